"""fp64 model of the chunkwise (WY / UT) evaluation the CUDA kernels implement.

Test infrastructure.  This is NOT the oracle: it restates, in numpy, the
chunk-level algebra that the kernels use, so that the derivation can be checked
against the token-by-token oracle in fp64 and so that the effect of rounding
operands to bf16 at the kernels' cast points can be measured on the CPU.

Derivation (one sequence, one head; chunk of L <= C tokens, local index r; S
the state entering the chunk).  With g_r = sum_{i<=r} log_alpha_i (per key
channel) and gamma_r = exp(g_r), unrolling the update equation of the daiw.net
page (section "KDA 的更新式") inside the chunk gives

    S_r = Diag(gamma_r) S + sum_{i<=r} Diag(gamma_r / gamma_i) k_i u_i^T,
    u_r = beta_r (v_r - (gamma_r * k_r)^T S - sum_{i<r} <gamma_r*k_r, k_i/gamma_i> u_i).

So with K~ = k*gamma, K- = k/gamma, Q~ = q*gamma, K^ = k*gamma_{L-1}/gamma:

    A = strict_lower(diag(beta) K~ K-^T),   T = (I + A)^{-1},
    W = T diag(beta) K~,   U0 = T diag(beta) V,   U = U0 - W S,
    P = lower(Q~ K-^T)     (diagonal included: the read follows the write),
    O = d_k^{-1/2} (Q~ S + P U),
    S' = Diag(gamma_{L-1}) S + K^^T U.
"""
from __future__ import annotations

import numpy as np
import torch


def bf16(x):
    """Round an fp64 array to bf16 (round-to-nearest-even) and back."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def chunked_head(q, k, v, la, beta, S0, C=64, rnd=None):
    """One (sequence, head): q, k, la [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv].

    ``rnd`` is a dict of cast-point names -> rounding functions (default: none):
    'ops' (decayed MMA operands), 'T', 'wy' (stored W, U0), 'qk' (stored Q~, K^),
    'P', 'S' (state operand), 'U' (U operand), 'o' (output).
    """
    rnd = rnd or {}
    R = lambda name, x: rnd[name](x) if name in rnd else x
    T_, dk = q.shape
    scale = dk ** -0.5
    S = S0.copy()
    out = np.zeros((T_, v.shape[1]))
    for s in range(0, T_, C):
        e = min(s + C, T_)
        L = e - s
        g = np.cumsum(la[s:e], axis=0)
        gam = np.exp(g)
        Kt = R("ops", k[s:e] * gam)
        Kb = R("ops", k[s:e] / gam)
        Qt = q[s:e] * gam
        Kh = k[s:e] * np.exp(g[-1] - g)
        b = beta[s:e, None]
        A = np.tril(b * (Kt @ Kb.T), -1)
        Tm = R("T", np.linalg.inv(np.eye(L) + A))
        W = R("wy", Tm @ R("ops", b * k[s:e] * gam))
        U0 = R("wy", Tm @ R("ops", b * v[s:e]))
        P = R("P", np.tril(R("ops", Qt) @ Kb.T, 0))
        Qs, Khs = R("qk", Qt), R("qk", Kh)
        Sop = R("S", S)
        U = U0 - W @ Sop
        Uop = R("U", U)
        out[s:e] = R("o", scale * (Qs @ Sop + P @ Uop))
        S = np.exp(g[-1])[:, None] * S + Khs.T @ Uop
    return out, S
