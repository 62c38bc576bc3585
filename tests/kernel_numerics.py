"""Test-only CPU emulation of the tensor-core prefill's number formats, chunk by chunk.

The fused prefill (chunk_tc_kernel) evaluates the chunkwise WY form of tests/chunk_algebra.py
with every operand it hands the tensor core rounded to bf16 and every accumulation in fp32.
This module repeats that arithmetic in numpy at the same rounding points, so that the
precision of the design (not of a kernel) can be checked against the fp64 oracle on the CPU:

    g  = per-channel prefix of log2 alpha in the chunk,  m = (g_0 + g_C) / 2
    Ê  = bf16(bf16(b ⊙ k) ⊙ bf16(2^(g-m))),  Q̂ = bf16(q ⊙ bf16(2^(g-m))),  K̃ = bf16(k ⊙ bf16(2^(m-g)))
    U  = bf16(w ⊙ v)
    [A; P] = [Ê; Q̂] K̃^T (fp32),  T = (I + A)^-1 -> bf16,  P -> bf16
    W' = T Ê,  Ũ = T U (fp32);   Δ = Ũ - bf16(W') Z̃ (fp32) -> bf16,   Z̃ = bf16(Z)
    O  = Q̂ Z̃ + P Δ (fp32) -> output bf16
    Z += K̃^T Δ (fp32);  S = 2^(g_C - m) Z,  then Z' = 2^(m') S   (two fp32 multiplies, in turn)

Chunks whose span g_0 - g_C exceeds 120 nats take the kernel's wide-span branch; it is emulated
as fp32 arithmetic without operand rounding (A and P from 2^(g_r - g_i) <= 1 per element).
"""
import numpy as np

SPAN_MAX_LOG2 = 120.0 / np.log(2.0)


def bf16(x):
    """Round to bf16 (nearest, ties to even) through fp32; returned as fp64."""
    x32 = np.asarray(x, dtype=np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def ftz_exp2(x):
    """2^x in fp32 with results below the smallest normal fp32 flushed to zero."""
    y = f32(np.exp2(f32(x)))
    return np.where(y < np.finfo(np.float32).tiny, 0.0, y)


def emulate_chain(q, k, v, alpha, b, w, S0, C=64, combine_frame_factors=False, stored_u_bf16=False):
    """One chain ([T, d] arrays holding the stored token values, alpha fp32; S0 [K, V] or None).
    Returns (o [T, V] as bf16 values, S_T [K, V] fp32 values).  Between chunks the state is the
    fp32 S the kernel forms as sPost * Z; per chunk sS scales its bf16 copy for G3 and sZ the fp32
    copy that G5 accumulates into (fast chunks: sS = sZ = 2^m, sPost = 2^(g_C - m); wide chunks:
    sS = 1, sZ = 2^(g_C), sPost = 1).  combine_frame_factors=True instead takes sPost of one chunk
    and sS / sZ of the next as ONE factor, 2 to the sum of their exponents, flushed to zero below
    fp32's normal range as the GPU's ftz exp2 does: a design the kernel must not use, because at
    long-context decay rates that sum falls below -126 while each exponent alone does not.
    stored_u_bf16=True rounds Ũ = T U to bf16 as well, as a prefill split into a parallel build/solve
    kernel and a state walk would when it passes Ũ through HBM in bf16 (the fused kernel keeps it
    in fp32 in TMEM)."""
    T, K = q.shape
    V = v.shape[1]
    S = np.zeros((K, V)) if S0 is None else f32(S0)
    o = np.zeros((T, V))
    post = None   # combine_frame_factors: the previous chunk's sPost and accumulated Z
    tiny = np.finfo(np.float32).tiny
    for t0 in range(0, T, C):
        sl = slice(t0, min(T, t0 + C))
        L = sl.stop - sl.start
        g = f32(np.cumsum(f32(np.log2(np.maximum(alpha[sl], tiny))), axis=0))
        g0, gC = g[0], g[-1]
        wide = bool(np.any(g0 - gC > SPAN_MAX_LOG2))
        e, U = bf16(b[sl] * k[sl]), bf16(w[sl] * v[sl])
        if wide:   # A and P on CUDA cores from 2^(g_r - g_i) <= 1; unscaled factors (m = 0)
            Eh, Qh = bf16(b[sl] * k[sl] * np.exp2(g)), bf16(q[sl] * np.exp2(g))
            Kt = bf16(k[sl] * np.exp2(gC - g))
            diff = g[:, None, :] - g[None, :, :]
            keep = np.tril(np.ones((L, L), dtype=bool), 0)[:, :, None]
            dec = np.where(keep, np.exp2(np.where(keep, diff, 0.0)), 0.0)
            A = f32(np.einsum("rc,ic,ric->ri", b[sl] * k[sl], k[sl], dec)) * np.tril(np.ones((L, L)), -1)
            P = f32(np.einsum("rc,ic,ric->ri", q[sl], k[sl], dec))
            xS, xZ, xPost = np.zeros(K), gC, np.zeros(K)
        else:
            m = f32(0.5 * (g0 + gC))
            F = bf16(np.exp2(g - m))
            Eh, Qh = bf16(e * F), bf16(q[sl] * F)
            Kt = bf16(k[sl] * bf16(np.exp2(m - g)))
            with np.errstate(over="ignore"):   # products above the diagonal may overflow: masked below
                Full = f32(np.vstack([Eh, Qh]) @ Kt.T)
            A = np.tril(Full[:L], -1)
            P = np.tril(Full[L:], 0)
            xS = xZ = m
            xPost = f32(gC - m)
        sS, sZ, sPost = f32(np.exp2(xS)), f32(np.exp2(xZ)), f32(np.exp2(xPost))
        Tm = bf16(np.linalg.inv(np.eye(L) + A))
        Pb = bf16(P)
        Wp = f32(Tm @ Eh)
        Ut = f32(Tm @ U)
        if stored_u_bf16:
            Ut = bf16(Ut)
        if post is None:
            Zt = bf16(f32(sS[:, None] * S))
            Z = f32(sZ[:, None] * S)
        else:
            x_prev, Z_prev = post
            Zt = bf16(f32(ftz_exp2(x_prev + xS)[:, None] * Z_prev))
            Z = f32(ftz_exp2(x_prev + xZ)[:, None] * Z_prev)
        Delta = bf16(f32(Ut - bf16(Wp) @ Zt))
        o[sl] = bf16(f32(Qh @ Zt + Pb @ Delta))
        Z = f32(Z + Kt.T @ Delta)
        S = f32(sPost[:, None] * Z)
        if combine_frame_factors:
            post = (xPost, Z)
    return o, S
