"""Seeded synthetic inputs for the KDA forward pass.

This module is shared by the tests, the benchmark and the smoke check.  It
holds none of the method's arithmetic: it only draws random tensors in the
shapes and distributions of the five workloads and casts them to the
workload's dtype.  L2-normalising q, k over K and applying a sigmoid to the
beta logits happen here because the op itself takes them as given
(KDA notes, "KDA 递归核心": beta is an input write strength; DeltaNet-family
digest: keys are assumed normalised).

Draw order (one ``torch.Generator`` seeded ``1000 + workload id``, float32):
q, k, v, g_raw, beta-logits, A_log, dt_bias, S0.
"""
from __future__ import annotations

import dataclasses
import math

import torch

GATE_NONE, GATE_SAFE, GATE_STANDARD = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    B: int
    T: int
    H: int
    HV: int
    K: int
    V: int
    chunk: int
    dtype: torch.dtype
    gate_mode: int
    lower_bound: float
    A_log_range: tuple | None      # U(lo, hi); None -> zeros
    dt_bias_mean: float
    dt_bias_std: float
    S0_std: float | None           # None -> no S0 (zeros)
    decode_steps: int = 0          # >0: T is the number of decode steps, one token each

    @property
    def pairs(self) -> int:
        return self.B * self.HV

    @property
    def is_decode(self) -> bool:
        return self.decode_steps > 0

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    1: Workload(1, "tiny fp32 recurrence B1 T64 H=HV=2 K=V=16 C16", 1, 64, 2, 2, 16, 16, 16,
                torch.float32, GATE_SAFE, -5.0, None, -4.0, 0.0, None),
    2: Workload(2, "GVA small prefill bf16 B2 T1024 H4->HV8 K=V=128 C64", 2, 1024, 4, 8, 128, 128, 64,
                torch.bfloat16, GATE_SAFE, -5.0, (-0.5, 0.5), -4.0, 0.1, None),
    3: Workload(3, "training-shaped prefill bf16 B8 T4096 H=HV=16 K=V=128 C64, S0 in, S_T out",
                8, 4096, 16, 16, 128, 128, 64, torch.bfloat16, GATE_SAFE, -5.0, (-0.5, 0.5), -4.0, 0.1,
                0.02),
    4: Workload(4, "long prefill bf16 B1 T65536 H8->HV32 K=V=128 C64, standard gate",
                1, 65536, 8, 32, 128, 128, 64, torch.bfloat16, GATE_STANDARD, 0.0, (-1.0, 0.5), -4.0, 0.0,
                None),
    5: Workload(5, "batched decode B256 HV=H=32 K=V=128, fp32 state in place, 128 steps",
                256, 128, 32, 32, 128, 128, 64, torch.bfloat16, GATE_SAFE, -5.0, None, -4.0, 0.0, 0.02,
                decode_steps=128),
}


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-6)


def make_inputs(w: Workload, seed: int | None = None, device: str = "cpu", raw: bool = False) -> dict:
    """Draw one workload's inputs.  Per-token tensors in ``w.dtype``; A_log, dt_bias, S0 fp32.

    ``raw=True`` returns the same draws without the two input-side steps: q and k as drawn (not
    normalised) and beta as its logits, each cast to ``w.dtype`` -- the inputs of the op's
    in-kernel input options.

    Returns a dict with q, k [B,T,H,K]; v [B,T,HV,V]; g [B,T,HV,K] (g_raw when the
    workload gates in the op); beta [B,T,HV]; A_log [HV]; dt_bias [HV,K]; S0
    [B,HV,K,V] or None.  For decode workloads T is the number of steps.
    """
    if seed is None:
        seed = 1000 + w.wid
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    B, T, H, HV, K, V = w.B, w.T, w.H, w.HV, w.K, w.V
    q = torch.randn(B, T, H, K, **f32)
    k = torch.randn(B, T, H, K, **f32)
    v = torch.randn(B, T, HV, V, **f32)
    g = torch.randn(B, T, HV, K, **f32)
    beta_logit = torch.randn(B, T, HV, **f32)
    if w.A_log_range is None:
        A_log = torch.zeros(HV, dtype=torch.float32, device=device)
    else:
        lo, hi = w.A_log_range
        A_log = lo + (hi - lo) * torch.rand(HV, **f32)
    dt_bias = w.dt_bias_mean + w.dt_bias_std * torch.randn(HV, K, **f32)
    S0 = None if w.S0_std is None else w.S0_std * torch.randn(B, HV, K, V, **f32)
    if raw:
        return dict(q=q.to(w.dtype), k=k.to(w.dtype), v=v.to(w.dtype), g=g.to(w.dtype), beta=beta_logit.to(w.dtype),
                    A_log=A_log, dt_bias=dt_bias.contiguous(), S0=S0)
    q = _l2norm(q).to(w.dtype)
    k = _l2norm(k).to(w.dtype)
    return dict(q=q, k=k, v=v.to(w.dtype), g=g.to(w.dtype), beta=torch.sigmoid(beta_logit).to(w.dtype),
                A_log=A_log, dt_bias=dt_bias.contiguous(), S0=S0)


def default_scale(K: int) -> float:
    return 1.0 / math.sqrt(K)


# Absorbed MLA decode, with the MLA sizes of the real K3 configuration (H = 96 heads, head dimension
# 128, kv_lora_rank r = 512) and a decode batch of 64 sequences with 4096 cached latent positions each.
MLA_DECODE = dict(B=64, T=4096, H=96, d_q=128, d_v=128, r=512)


def make_mla_inputs(B, T, H, d_q, d_v, r, seed=1006, device="cpu", ragged=False) -> dict:
    """q ~ N(0,1) [B,H,d_q]; W_UK ~ N(0,1/d_q) [H,d_q,r]; W_UV ~ N(0,1/r) [H,d_v,r]; c ~ N(0,1) [B,T,r];
    all bf16.  With ``ragged`` the lengths are drawn uniformly in [1, T] (int32), else None."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    q = torch.randn(B, H, d_q, **f32)
    W_UK = torch.randn(H, d_q, r, **f32) / math.sqrt(d_q)
    W_UV = torch.randn(H, d_v, r, **f32) / math.sqrt(r)
    c = torch.randn(B, T, r, **f32)
    lengths = None
    if ragged:
        lengths = torch.randint(1, T + 1, (B,), generator=gen, device=device, dtype=torch.int64).to(torch.int32)
    bf = torch.bfloat16
    return dict(q=q.to(bf), W_UK=W_UK.to(bf), W_UV=W_UV.to(bf), c=c.to(bf), lengths=lengths)
