"""Float64 reverse mode of the KDA recurrence and of the two gates.

TEST INFRASTRUCTURE ONLY, like the rest of this package: a reference for a
future backward pass, checked against central finite differences of the
forward oracle.  The pages give the forward method only; the adjoint below is
derived from the recurrence's four steps (KDA notes, "KDA 递归核心", §逐步公式)
and the gate definitions (KDA notes, "Gate 激活", table "两种 Gate"), one step
at a time and in reverse order.  Plain numpy with a loop over (b, hv) pairs
and tokens: meant for small cases.

Forward, per (b, hv) and token t, with head h = hv / (HV / H):
    a       = exp(g_t)                        (per key channel)
    S_dec   = diag(a) S_{t-1}
    r       = v_t - k_t^T S_dec
    S_t     = S_dec + beta_t k_t r^T
    o_t     = scale q_t^T S_t
Reverse, with dS the gradient of the loss with respect to S_t:
    dS     += scale q_t dO_t^T                 dq_t  += scale S_t dO_t
    dbeta_t = k_t^T dS r                       dr     = beta_t dS^T k_t
    dk_t   += beta_t dS r - S_dec dr           dv_t   = dr
    dS_dec  = dS - k_t dr^T
    dg_t    = a * rowsum(dS_dec * S_{t-1})     dS_{t-1} = diag(a) dS_dec
dq and dk of a q/k head add up over the value heads that read it.
"""
from __future__ import annotations

import numpy as np

from . import GATE_NONE, GATE_SAFE, GATE_STANDARD, _f64, _shapes, gate


def recurrent_backward(q, k, v, g, beta, S0=None, dO=None, dS_T=None, *, scale=None):
    """Gradients of ``sum(dO * o) + sum(dS_T * S_T)`` for the recurrence with log-decay ``g``.

    Returns a dict with ``dq``, ``dk`` ([B,T,H,K]), ``dv`` ([B,T,HV,V]), ``dg`` ([B,T,HV,K]),
    ``dbeta`` ([B,T,HV]) and ``dS0`` ([B,HV,K,V]), all float64.
    """
    q, k, v, g, beta, S0, dO, dS_T = (_f64(x) for x in (q, k, v, g, beta, S0, dO, dS_T))
    B, T, H, HV, K, V = _shapes(q, v)
    G = HV // H
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    dq, dk = np.zeros_like(q), np.zeros_like(k)
    dv, dg, dbeta = np.zeros_like(v), np.zeros_like(g), np.zeros_like(beta)
    dS0 = np.zeros((B, HV, K, V))
    for b in range(B):
        for hv in range(HV):
            h = hv // G
            # forward, keeping the state entering every token
            states = np.empty((T + 1, K, V))
            states[0] = 0.0 if S0 is None else S0[b, hv]
            for t in range(T):
                kt = k[b, t, h]
                S_dec = np.exp(g[b, t, hv])[:, None] * states[t]
                r = v[b, t, hv] - kt @ S_dec
                states[t + 1] = S_dec + beta[b, t, hv] * np.outer(kt, r)
            # reverse
            dS = np.zeros((K, V)) if dS_T is None else dS_T[b, hv].copy()
            for t in range(T - 1, -1, -1):
                qt, kt, bt = q[b, t, h], k[b, t, h], beta[b, t, hv]
                a = np.exp(g[b, t, hv])
                S_prev = states[t]
                S_dec = a[:, None] * S_prev
                r = v[b, t, hv] - kt @ S_dec
                if dO is not None:
                    dS += scale * np.outer(qt, dO[b, t, hv])
                    dq[b, t, h] += scale * (states[t + 1] @ dO[b, t, hv])
                dbeta[b, t, hv] = kt @ dS @ r
                dr = bt * (kt @ dS)
                dv[b, t, hv] = dr
                dk[b, t, h] += bt * (dS @ r) - S_dec @ dr
                dS_dec = dS - np.outer(kt, dr)
                dg[b, t, hv] = a * np.sum(dS_dec * S_prev, axis=1)
                dS = a[:, None] * dS_dec
            dS0[b, hv] = dS
    return {"dq": dq, "dk": dk, "dv": dv, "dg": dg, "dbeta": dbeta, "dS0": dS0}


def gate_backward(g_raw, A_log, dt_bias, dg, *, mode, lower_bound=None):
    """Chain ``dg`` (gradient with respect to the gate output) back through the gate.

    input x = g_raw + dt_bias, rate = exp(A_log):
      SAFE      g = L sigmoid(rate x):   dg/dx = L s (1 - s) rate,   dg/dA_log = L s (1 - s) rate x
      STANDARD  g = -rate softplus(x):   dg/dx = -rate sigmoid(x),   dg/dA_log = -rate softplus(x)
    Returns ``(dg_raw [.., HV, K], ddt_bias [HV, K] or None, dA_log [HV])``.
    """
    g_raw, A_log, dt_bias, dg = (_f64(x) for x in (g_raw, A_log, dt_bias, dg))
    HV, K = g_raw.shape[-2:]
    x = g_raw + (0.0 if dt_bias is None else dt_bias)
    rate = np.exp(A_log)[:, None]
    if mode == GATE_SAFE:
        if lower_bound is None or not np.isfinite(lower_bound):
            raise ValueError("safe gate needs a finite lower_bound")
        z = rate * x
        s = 1.0 / (1.0 + np.exp(-z))
        dgdx = lower_bound * s * (1.0 - s) * rate
        dgda = lower_bound * s * (1.0 - s) * z
    elif mode == GATE_STANDARD:
        s = 1.0 / (1.0 + np.exp(-x))
        sp = np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))
        dgdx = -rate * s
        dgda = -rate * sp
    else:
        raise ValueError(f"bad gate mode {mode}")
    dg_raw = dg * dgdx
    lead = tuple(range(dg.ndim - 2))
    ddt_bias = None if dt_bias is None else dg_raw.sum(axis=lead)
    dA_log = (dg * dgda).sum(axis=lead + (dg.ndim - 1,))
    return dg_raw, ddt_bias, dA_log


def backward(q, k, v, g, beta, A_log=None, dt_bias=None, S0=None, dO=None, dS_T=None, *, gate_mode=GATE_NONE,
             lower_bound=None, scale=None):
    """Reverse mode of ``oracle.forward``: the gate (when ``gate_mode`` is SAFE or STANDARD, ``g`` holds
    g_raw) then the recurrence.  Adds ``dg_raw``, ``ddt_bias`` and ``dA_log`` to the recurrence's
    gradients when a gate ran (``dg`` then stays the gradient with respect to the gate output)."""
    g_log = g if gate_mode == GATE_NONE else gate(g, A_log, dt_bias, mode=gate_mode, lower_bound=lower_bound)
    out = recurrent_backward(q, k, v, g_log, beta, S0, dO, dS_T, scale=scale)
    if gate_mode != GATE_NONE:
        out["dg_raw"], out["ddt_bias"], out["dA_log"] = gate_backward(g, A_log, dt_bias, out["dg"], mode=gate_mode,
                                                                      lower_bound=lower_bound)
    return out


def chunkwise_backward(q, k, v, g, beta, S0=None, dO=None, dS_T=None, *, chunk=64, scale=None):
    """The same gradients as ``recurrent_backward``, computed chunk by chunk in the form a chunked
    backward pass uses: the reverse mode of the chunkwise equations (DeltaNet-family digest,
    "Chunkwise KDA"), with every decay an explicit exponential of a prefix-sum difference.

    Per chunk of n tokens entering with state S (Gam_i = sum_{m<=i} g_m, e = exp):
        Ebar_i = beta_i (v_i - sum_d k_id e^{Gam_id} S[d,:])
        rho_ij = beta_i sum_d k_id k_jd e^{Gam_id - Gam_jd}              (j < i)
        E_i    = Ebar_i - sum_{j<i} rho_ij E_j
        a_ij   = scale sum_d q_id k_jd e^{Gam_id - Gam_jd}               (j <= i)
        O_i    = scale sum_d q_id e^{Gam_id} S[d,:] + sum_{j<=i} a_ij E_j
        S'[d,:] = e^{Gam_end,d} S[d,:] + sum_j k_jd e^{Gam_end,d - Gam_jd} E_j
    Reverse, given dO and dS' (the gradient with respect to S'):
        dE_j  = sum_{i>=j} a_ij dO_i + sum_d k_jd e^{Gam_end,d - Gam_jd} dS'[d,:]
        lam   = (I + rho)^{-T} dE          (back substitution; lam is the gradient of Ebar)
        drho_ij = -lam_i . E_j,  da_ij = dO_i . E_j
    and every factor above gives its q, k, beta, v, Gam and S terms; dg is the reverse cumulative
    sum of dGam within the chunk, and the S terms are the next (earlier) chunk's dS'.
    """
    q, k, v, g, beta, S0, dO, dS_T = (_f64(x) for x in (q, k, v, g, beta, S0, dO, dS_T))
    B, T, H, HV, K, V = _shapes(q, v)
    G = HV // H
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    if dO is None:
        dO = np.zeros((B, T, HV, V))
    dq, dk = np.zeros_like(q), np.zeros_like(k)
    dv, dg, dbeta = np.zeros_like(v), np.zeros_like(g), np.zeros_like(beta)
    dS0 = np.zeros((B, HV, K, V))
    starts = list(range(0, T, chunk))
    for b in range(B):
        for hv in range(HV):
            h = hv // G
            # forward over chunks, keeping the state entering each one
            S = np.zeros((K, V)) if S0 is None else S0[b, hv].copy()
            entering = []
            for c0 in starts:
                n = min(chunk, T - c0)
                qc, kc, vc = q[b, c0:c0 + n, h], k[b, c0:c0 + n, h], v[b, c0:c0 + n, hv]
                bc = beta[b, c0:c0 + n, hv]
                Gam = np.cumsum(g[b, c0:c0 + n, hv], axis=0)
                entering.append(S.copy())
                Ebar = bc[:, None] * (vc - (kc * np.exp(Gam)) @ S)
                E = np.zeros((n, V))
                for i in range(n):
                    acc = Ebar[i].copy()
                    for j in range(i):
                        rho = bc[i] * np.sum(kc[i] * kc[j] * np.exp(Gam[i] - Gam[j]))
                        acc -= rho * E[j]
                    E[i] = acc
                gend = Gam[n - 1]
                S = np.exp(gend)[:, None] * S + (kc * np.exp(gend - Gam)).T @ E
            # reverse over chunks
            dSn = np.zeros((K, V)) if dS_T is None else dS_T[b, hv].copy()   # gradient of S'
            for ci in range(len(starts) - 1, -1, -1):
                c0 = starts[ci]
                n = min(chunk, T - c0)
                S = entering[ci]
                qc, kc, vc = q[b, c0:c0 + n, h], k[b, c0:c0 + n, h], v[b, c0:c0 + n, hv]
                bc = beta[b, c0:c0 + n, hv]
                dOc = dO[b, c0:c0 + n, hv]
                Gam = np.cumsum(g[b, c0:c0 + n, hv], axis=0)
                gend = Gam[n - 1]
                # recompute the chunk's forward quantities
                eG = np.exp(Gam)                                   # [n, K]
                Kt = kc * eG                                       # k_i e^{Gam_i}
                Ebar = bc[:, None] * (vc - Kt @ S)
                rho = np.zeros((n, n))
                a = np.zeros((n, n))
                for i in range(n):
                    for j in range(n):
                        f = np.exp(Gam[i] - Gam[j])
                        if j < i:
                            rho[i, j] = bc[i] * np.sum(kc[i] * kc[j] * f)
                        if j <= i:
                            a[i, j] = scale * np.sum(qc[i] * kc[j] * f)
                E = np.zeros((n, V))
                for i in range(n):
                    E[i] = Ebar[i] - rho[i, :i] @ E[:i]
                Kend = kc * np.exp(gend - Gam)                     # k_j e^{Gam_end - Gam_j}
                # gradients of E, then of Ebar (back substitution through the unit lower solve)
                dE = a.T @ dOc + Kend @ dSn
                lam = np.zeros((n, V))
                for j in range(n - 1, -1, -1):
                    lam[j] = dE[j] - rho[j + 1:, j] @ lam[j + 1:]
                dGam = np.zeros((n, K))
                dkc = np.zeros((n, K))
                dqc = np.zeros((n, K))
                dS = np.exp(gend)[:, None] * dSn                  # from e^{Gam_end} S
                # O_i's direct term scale q_i e^{Gam_i} S
                QS_grad = dOc @ S.T                                # [n, K]: S[d,:] . dO_i
                dqc += scale * eG * QS_grad
                dGam += scale * qc * eG * QS_grad
                dS += scale * (qc * eG).T @ dOc
                # S' = e^{Gam_end} S + Kend^T E
                SdS = np.sum(S * dSn, axis=1)                       # S[d,:] . dS'[d,:]
                dGam[n - 1] += np.exp(gend) * SdS
                EdS = E @ dSn.T                                    # [n, K]: E_j . dS'[d,:]
                dkc += np.exp(gend - Gam) * EdS
                dGam[n - 1] += np.sum(Kend * EdS, axis=0)
                dGam -= Kend * EdS
                # Ebar_i = beta_i (v_i - Kt_i S)
                dv[b, c0:c0 + n, hv] = bc[:, None] * lam
                dbeta[b, c0:c0 + n, hv] += np.sum((vc - Kt @ S) * lam, axis=1)
                SL = lam @ S.T                                     # [n, K]: S[d,:] . lam_i
                dkc -= bc[:, None] * eG * SL
                dGam -= bc[:, None] * kc * eG * SL
                dS -= (bc[:, None] * Kt).T @ lam
                # rho and a
                drho = -(lam @ E.T)                                # drho_ij = -lam_i . E_j
                da = dOc @ E.T                                     # da_ij = dO_i . E_j
                for i in range(n):
                    for j in range(i + 1):
                        f = np.exp(Gam[i] - Gam[j])
                        if j < i:
                            w = drho[i, j]
                            dbeta[b, c0 + i, hv] += w * np.sum(kc[i] * kc[j] * f)
                            t_ = w * bc[i] * kc[i] * kc[j] * f
                            dkc[i] += w * bc[i] * kc[j] * f
                            dkc[j] += w * bc[i] * kc[i] * f
                            dGam[i] += t_
                            dGam[j] -= t_
                        w = da[i, j]
                        t_ = w * scale * qc[i] * kc[j] * f
                        dqc[i] += w * scale * kc[j] * f
                        dkc[j] += w * scale * qc[i] * f
                        dGam[i] += t_
                        dGam[j] -= t_
                dg[b, c0:c0 + n, hv] = np.cumsum(dGam[::-1], axis=0)[::-1]
                dq[b, c0:c0 + n, h] += dqc
                dk[b, c0:c0 + n, h] += dkc
                dSn = dS
            dS0[b, hv] = dSn
    return {"dq": dq, "dk": dk, "dv": dv, "dg": dg, "dbeta": dbeta, "dS0": dS0}
