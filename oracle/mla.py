"""Float64 oracle of the absorbed MLA decode step.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only ``tests/`` and the CPU legs of
``bench.py`` use it; the CUDA library never reaches it.

KDA ledger, derivation DER2 ("MLA 矩阵吸收推导") for claim C4 (q absorbs W_UK and meets the latent c
directly; K and V are never decompressed), with the shapes of the ledger's symbol table
(c [B, T, r], W_UK [H, d_q, r], W_UV [H, d_v, r]):
    1. q_abs = q . W_UK                  [B, H, r]
    2. score = q_abs . c^T                [B, H, T]
    3. o_lat = softmax(score) . c         [B, H, r]
    4. o     = o_lat . W_UV^T             [B, H, d_v]
for one decode query per sequence over its T cached latent positions (the K3 MLA layer is a global
softmax attention without positional encoding: K3 architecture section, "NoPE").

Readings of what the pages leave open:
  * the softmax scale: not given; ``scale`` multiplies the scores, default 1/sqrt(d_q), the usual
    scale of the decompressed q . k product whose head dimension is d_q;
  * ragged caches: ``lengths[b]`` (default T) positions of sequence b take part, the rest are ignored.

``decompressed`` is the same attention with K and V materialised per head (K[t] = W_UK c_t,
V[t] = W_UV c_t) and the textbook softmax attention on them: the independent form that pins the
absorbed one.
"""
from __future__ import annotations

import numpy as np

from . import _f64


def _prep(q, W_UK, W_UV, c, scale, lengths):
    q, W_UK, W_UV, c = (_f64(x) for x in (q, W_UK, W_UV, c))
    B, H, d_q = q.shape
    Bc, T, r = c.shape
    if Bc != B or W_UK.shape != (H, d_q, r) or W_UV.shape[0] != H or W_UV.shape[2] != r:
        raise ValueError("shape mismatch")
    if scale is None:
        scale = 1.0 / np.sqrt(d_q)
    lengths = np.full(B, T, dtype=np.int64) if lengths is None else np.asarray(lengths, dtype=np.int64)
    if np.any(lengths < 1) or np.any(lengths > T):
        raise ValueError("lengths must be in [1, T]")
    return q, W_UK, W_UV, c, float(scale), lengths


def _softmax(x):
    m = np.max(x, axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def absorbed(q, W_UK, W_UV, c, *, scale=None, lengths=None):
    """DER2 steps 1-4 in order.  Returns o [B, H, d_v] (float64)."""
    q, W_UK, W_UV, c, scale, lengths = _prep(q, W_UK, W_UV, c, scale, lengths)
    B, H, _ = q.shape
    o = np.empty((B, H, W_UV.shape[1]))
    for b in range(B):
        L = lengths[b]
        q_abs = np.einsum("hd,hdr->hr", q[b], W_UK)        # step 1
        score = q_abs @ c[b, :L].T                          # step 2  [H, L]
        o_lat = _softmax(scale * score) @ c[b, :L]          # step 3  [H, r]
        o[b] = np.einsum("hr,hvr->hv", o_lat, W_UV)         # step 4
    return o


def decompressed(q, W_UK, W_UV, c, *, scale=None, lengths=None):
    """Softmax attention on K, V decompressed per head from the latent (never used by the GPU path)."""
    q, W_UK, W_UV, c, scale, lengths = _prep(q, W_UK, W_UV, c, scale, lengths)
    B, H, _ = q.shape
    o = np.empty((B, H, W_UV.shape[1]))
    for b in range(B):
        L = lengths[b]
        for h in range(H):
            Kh = c[b, :L] @ W_UK[h].T                       # [L, d_q]
            Vh = c[b, :L] @ W_UV[h].T                       # [L, d_v]
            p = _softmax(scale * (Kh @ q[b, h]))
            o[b, h] = p @ Vh
    return o
