"""GPU parity of the absorbed MLA decode (kda_mla_decode) against the float64 oracle (oracle.mla.absorbed,
pinned by the decompressed attention), on the same seeded bf16 bits.

Bar: max|o - o_ref| / max|o_ref| <= 5e-3, the bar of the other bf16 outputs; the output's own bf16
rounding costs up to 3.9e-3 of it.  Cases: the decode workload (B64 T4096 H96 d=128 r=512) with sampled
sequences, ragged lengths, head counts that are not a multiple of the 48-head tile, every (d_q, d_v, r)
built, a single cached position, a given scale.
"""
import numpy as np
import pytest
import torch

from oracle import mla
from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import MLA_DECODE, make_mla_inputs
from parity_util import TOL, rel_err

pytestmark = pytest.mark.gpu


def _run(x, scale=None):
    dev = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    o = kda.mla_decode(dev["q"], dev["W_UK"], dev["W_UV"], dev["c"], dev["lengths"], scale=scale)
    torch.cuda.synchronize()
    return o


def _check(x, o, rows, scale=None):
    L = None if x["lengths"] is None else x["lengths"][rows].numpy()
    ref = mla.absorbed(x["q"][rows], x["W_UK"], x["W_UV"], x["c"][rows], scale=scale, lengths=L)
    e = rel_err(o[rows].cpu(), ref)
    assert e <= TOL[torch.bfloat16], f"rel err {e:.3e}"


def test_decode_workload_sampled():
    x = make_mla_inputs(**MLA_DECODE)
    o = _run(x)
    _check(x, o, [0, 17, 42, 63])


@pytest.mark.parametrize("B,T,H,dq,dv,r", [(3, 100, 16, 64, 64, 128), (5, 700, 96, 128, 128, 512),
                                           (2, 333, 50, 128, 64, 256), (4, 1, 97, 64, 128, 512),
                                           (2, 4100, 48, 128, 128, 128)])
def test_shapes_ragged(B, T, H, dq, dv, r):
    x = make_mla_inputs(B, T, H, dq, dv, r, seed=7 + B, ragged=True)
    o = _run(x)
    _check(x, o, list(range(B)))


def test_full_lengths_and_scale():
    x = make_mla_inputs(3, 513, 24, 128, 128, 512, seed=11)
    o = _run(x, scale=0.05)
    _check(x, o, [0, 1, 2], scale=0.05)
