"""Rounding model of the chunk algebra: which operand precisions the kernels can use.

Test infrastructure, like ``chunk_algebra.py``, whose algebra it repeats in a
form whose every product can round its operands the way a tensor-core kernel
would.  The plans it compares:
- the bf16-input path: tf32 A/P factors, fp16 everything else, fp32
  accumulation, bf16 output;
- two tensor-core forms of (I + A)^-1: the nilpotent product form and the
  blocked form with exact 16 x 16 diagonal blocks;
- the fp32-input path as single tf32 products or as split tf32 products
  (hi*hi + hi*lo + lo*hi).
Accumulation is modelled in fp64 (an fp32 accumulator adds about 1e-7).
"""
from __future__ import annotations

import numpy as np
import torch


def tf32(x):
    """Round to tf32 (10-bit mantissa, round to nearest even), back to fp64."""
    a = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    a = ((a + 0xFFF + ((a >> 13) & 1)) & ~np.uint64(0x1FFF)).astype(np.uint32)
    return a.view(np.float32).astype(np.float64)


def fp16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float16).double().numpy()


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def ident(x):
    return x


# ---- (I + A)^-1 for strictly lower A, operands of block products rounded by rnd
def inv_exact(A, rnd):
    return np.linalg.inv(np.eye(A.shape[0]) + A)


def inv_product(A, rnd):
    """(I + A)^-1 = prod_k (I + N^(2^k)), N = -A nilpotent: six factors cover 64 rows."""
    L = A.shape[0]
    N = -A
    P = np.eye(L) + N
    Np = N
    for _ in range(5):
        Np = rnd(Np) @ rnd(Np)
        P = P + rnd(P) @ rnd(Np)
    return P


def inv_blocked(A, rnd, bs=16):
    """Exact bs x bs diagonal blocks, then T21 = -T22 A21 T11, doubling the block."""
    L = A.shape[0]
    T = np.zeros((L, L))
    for s in range(0, L, bs):
        e = min(s + bs, L)
        T[s:e, s:e] = np.linalg.inv(np.eye(e - s) + A[s:e, s:e])
    b = bs
    while b < L:
        for s in range(0, L, 2 * b):
            m, e = s + b, min(s + 2 * b, L)
            if m >= L:
                continue
            X = rnd(A[m:e, s:m]) @ rnd(T[s:m, s:m])
            T[m:e, s:m] = -(rnd(T[m:e, m:e]) @ rnd(X))
        b *= 2
    return T


def bf16_path_head(q, k, v, la, beta, S0, inv=inv_exact, inv_rnd=ident, C=64, ops=tf32, mid=fp16):
    """The bf16-input plan: ``ops`` (tf32) for the split factors of A and P,
    ``mid`` (fp16) for T diag(beta), W, U0, P, Q~, K^, the state and U
    operands, bf16 output.  ops = mid = bf16 is the all-bf16 plan."""
    T_, dk = q.shape
    scale = dk ** -0.5
    S = S0.copy()
    out = np.zeros((T_, v.shape[1]))
    for s in range(0, T_, C):
        e = min(s + C, T_)
        L = e - s
        g = np.cumsum(la[s:e], axis=0)
        gm = g[(L - 1) // 2]
        Kl, Kr, Ql = ops(k[s:e] * np.exp(g - gm)), ops(k[s:e] * np.exp(gm - g)), ops(q[s:e] * np.exp(g - gm))
        b = beta[s:e]
        A = np.tril(b[:, None] * (Kl @ Kr.T), -1)
        Tb = mid(inv(A, inv_rnd) * b[None, :])
        W = mid(Tb @ mid(k[s:e] * np.exp(g)))
        U0 = mid(Tb @ v[s:e])
        P = mid(np.tril(Ql @ Kr.T, 0))
        Qt, Kh = mid(q[s:e] * np.exp(g)), mid(k[s:e] * np.exp(g[-1] - g))
        Sop = mid(S)
        Uop = mid(U0 - W @ Sop)
        out[s:e] = bf16(scale * (Qt @ Sop + P @ Uop))
        S = np.exp(g[-1])[:, None] * S + Kh.T @ Uop
    return out, S


def mm_tf32(X, Y):
    return f32(tf32(X) @ tf32(Y))


def mm_split_tf32(X, Y):
    Xh, Yh = tf32(X), tf32(Y)
    Xl, Yl = tf32(f32(X) - Xh), tf32(f32(Y) - Yh)
    return f32(Xh @ Yh + Xh @ Yl + Xl @ Yh)


def fp32_path_head(q, k, v, la, beta, S0, mm, C=64):
    """The fp32-input plan with every product done by ``mm``; the solve in fp32."""
    T_, dk = q.shape
    scale = dk ** -0.5
    S = f32(S0)
    out = np.zeros((T_, v.shape[1]))
    for s in range(0, T_, C):
        e = min(s + C, T_)
        L = e - s
        g = f32(np.cumsum(la[s:e], axis=0))
        gm = g[(L - 1) // 2]
        Kl, Kr, Ql = f32(k[s:e] * np.exp(g - gm)), f32(k[s:e] * np.exp(gm - g)), f32(q[s:e] * np.exp(g - gm))
        b = beta[s:e]
        A = np.tril(b[:, None] * mm(Kl, Kr.T), -1)
        Tb = f32(np.linalg.inv(np.eye(L) + A) * b[None, :])
        W, U0 = mm(Tb, f32(k[s:e] * np.exp(g))), mm(Tb, v[s:e])
        P = np.tril(mm(Ql, Kr.T), 0)
        Qt, Kh = f32(q[s:e] * np.exp(g)), f32(k[s:e] * np.exp(g[-1] - g))
        U = f32(U0 - mm(W, S))
        out[s:e] = f32(scale * (mm(Qt, S) + mm(P, U)))
        S = f32(np.exp(g[-1])[:, None] * S + mm(Kh.T, U))
    return out, S


def correlated_keys(T=512, dk=128, dv=128, seed=5):
    """Keys normalise(k0 + 0.1 noise), beta = 1, log_alpha = -1e-4: the powers
    of A grow combinatorially while (I + A)^-1 stays bounded."""
    g = torch.Generator().manual_seed(seed)
    k0 = torch.randn(dk, generator=g)
    k = k0[None, :] + 0.1 * torch.randn(T, dk, generator=g)
    k = (k / k.norm(dim=-1, keepdim=True)).to(torch.bfloat16).double()
    q = torch.randn(T, dk, generator=g)
    q = (q / q.norm(dim=-1, keepdim=True)).to(torch.bfloat16).double()
    v = torch.randn(T, dv, generator=g).to(torch.bfloat16).double()
    la = torch.full((T, dk), -1e-4, dtype=torch.float64)
    beta = torch.ones(T, dtype=torch.float64)
    return q.numpy(), k.numpy(), v.numpy(), la.numpy(), beta.numpy()
