"""Test-only fp64 chunkwise restatement of the recurrence's gradient (the WY backward form).

The forward chunk algebra is that of tests/chunk_algebra.py (page "NVIDIA представила
Gated DeltaNet-2 ...", the chunkwise WY form).  Per chunk of L tokens with incoming state S,
g = cumulative log alpha inside the chunk, Γ = exp(g), E = b ⊙ k, U = w ⊙ v:

    Ê = Γ ⊙ E,  Q̂ = Γ ⊙ Q,  Ǩ = exp(-g) ⊙ K,  A = strict_lower(Ê Ǩ^T),  P = lower(Q̂ Ǩ^T)
    R = U - Ê S,  Δ = (I + A)^-1 R,  O = Q̂ S + P Δ,  S' = Diag(γ) (S + Ǩ^T Δ),  γ = exp(g_{L-1})

Given dO and dS' (the gradient at the chunk's outgoing state) the chunk's gradients are matrix
products of the same shapes as the forward's:

    dΔ = P^T dO + Ǩ (γ ⊙ dS'),          dR = (I + A)^-T dΔ
    dA = -strict_lower(dR Δ^T),          dP = lower(dO Δ^T)
    dÊ = -dR S^T + dA Ǩ,                 dQ̂ = dO S^T + dP Ǩ
    dǨ = dA^T Ê + dP^T Q̂ + Δ (γ ⊙ dS')^T
    dS = Q̂^T dO - Ê^T dR + γ ⊙ dS'      (to the previous chunk)

then dq = Γ ⊙ dQ̂, de = Γ ⊙ dÊ, the key's own part exp(-g) ⊙ dǨ, and for the decay
dL/dg_r = (Q̂ ⊙ dQ̂ + Ê ⊙ dÊ - Ǩ ⊙ dǨ)_r, summed from the chunk's end back to each position,
plus rowsum(dS' ⊙ S') for the γ that scales the outgoing state.  This is the form a
tensor-core backward would evaluate; here it pins the step-wise oracle (tests/test_chunk_backward.py).
"""
import numpy as np


def chunk_grads(q, k, v, alpha, b, w, S, dO, dS_out):
    """One chunk ([L, d] fp64 arrays, S and dS_out [K, V]).
    Returns (dq, dk, dv, dalpha, db, dw, dS_in)."""
    L = q.shape[0]
    g = np.cumsum(np.log(alpha), axis=0)
    Gam, Ginv = np.exp(g), np.exp(-g)
    gam = Gam[-1]
    e, u = b * k, w * v
    Eh, Qh, Kc = Gam * e, Gam * q, Ginv * k
    strict = np.tril(np.ones((L, L)), -1)
    lower = np.tril(np.ones((L, L)), 0)
    A = (Eh @ Kc.T) * strict
    P = (Qh @ Kc.T) * lower
    IA = np.eye(L) + A
    R = u - Eh @ S
    Delta = np.linalg.solve(IA, R)
    S_out = gam[:, None] * (S + Kc.T @ Delta)

    gdS = gam[:, None] * dS_out
    dDelta = P.T @ dO + Kc @ gdS
    dR = np.linalg.solve(IA.T, dDelta)
    dA = -(dR @ Delta.T) * strict
    dP = (dO @ Delta.T) * lower
    dEh = -dR @ S.T + dA @ Kc
    dQh = dO @ S.T + dP @ Kc
    dKc = dA.T @ Eh + dP.T @ Qh + Delta @ gdS.T
    dS_in = Qh.T @ dO - Eh.T @ dR + gdS

    dq = Gam * dQh
    de = Gam * dEh
    dk = Ginv * dKc + b * de
    db = k * de
    dv = w * dR
    dw = v * dR
    h = Qh * dQh + Eh * dEh - Kc * dKc
    dlog = np.cumsum(h[::-1], axis=0)[::-1] + np.sum(dS_out * S_out, axis=1)[None, :]
    return dq, dk, dv, dlog / alpha, db, dw, dS_in


def chunked_grads(q, k, v, alpha, b, w, S0, dO, dST, C):
    """Whole chain ([T, d] arrays) in chunks of C (last one ragged): forward to collect each chunk's
    incoming state, then the chunks in reverse."""
    T, K = q.shape
    V = v.shape[1]
    S = np.zeros((K, V)) if S0 is None else np.array(S0, dtype=np.float64)
    starts = []
    for t0 in range(0, T, C):
        t1 = min(T, t0 + C)
        starts.append(S)
        g = np.cumsum(np.log(alpha[t0:t1]), axis=0)
        Gam = np.exp(g)
        e, u = b[t0:t1] * k[t0:t1], w[t0:t1] * v[t0:t1]
        Kc = np.exp(-g) * k[t0:t1]
        A = ((Gam * e) @ Kc.T) * np.tril(np.ones((t1 - t0, t1 - t0)), -1)
        Delta = np.linalg.solve(np.eye(t1 - t0) + A, u - (Gam * e) @ S)
        S = Gam[-1][:, None] * (S + Kc.T @ Delta)
    out = [np.zeros((T, K)), np.zeros((T, K)), np.zeros((T, V)), np.zeros((T, K)), np.zeros((T, K)),
           np.zeros((T, V))]
    dS = np.zeros((K, V)) if dST is None else np.array(dST, dtype=np.float64)
    for ci in range(len(starts) - 1, -1, -1):
        t0, t1 = ci * C, min(T, ci * C + C)
        sl = slice(t0, t1)
        g = chunk_grads(q[sl], k[sl], v[sl], alpha[sl], b[sl], w[sl], starts[ci], dO[sl], dS)
        for i in range(6):
            out[i][sl] = g[i]
        dS = g[6]
    return tuple(out) + (dS,)


def chunk_grads_framed(q, k, v, alpha, b, w, S, dO, dS_out):
    """chunk_grads with every decay factor taken around the chunk's per-channel midpoint
    m = (g_0 + g_{L-1}) / 2, as a tensor-core kernel must to keep its operands in range:
    Ê_m = exp(g - m) ⊙ E, Q̂_m = exp(g - m) ⊙ Q, Ǩ_m = exp(m - g) ⊙ K (A, P unchanged), the state
    in the frame Z = exp(m) ⊙ S, and dS entering as exp(g_{L-1} - m) ⊙ dS'.  The factors are then
    bounded by exp(span / 2) instead of exp(span); the products above the diagonal of A and P, which
    the masks drop, may still overflow and are selected away rather than multiplied by zero."""
    L = q.shape[0]
    g = np.cumsum(np.log(alpha), axis=0)
    m = 0.5 * (g[0] + g[-1])
    fm, fp = np.exp(g - m), np.exp(m - g)
    e = b * k
    Em, Qm, Km = fm * e, fm * q, fp * k
    strict = np.tril(np.ones((L, L), dtype=bool), -1)
    lower = np.tril(np.ones((L, L), dtype=bool), 0)
    with np.errstate(over="ignore"):   # entries above the diagonal may overflow: they are not kept
        A = np.where(strict, Em @ Km.T, 0.0)
        P = np.where(lower, Qm @ Km.T, 0.0)
    IA = np.eye(L) + A
    Z = np.exp(m)[:, None] * S
    Delta = np.linalg.solve(IA, w * v - Em @ Z)
    S_out = np.exp(g[-1])[:, None] * S + np.exp(g[-1] - m)[:, None] * (Km.T @ Delta)

    dSm = np.exp(g[-1] - m)[:, None] * dS_out
    dDelta = P.T @ dO + Km @ dSm
    dR = np.linalg.solve(IA.T, dDelta)
    dA = np.where(strict, -(dR @ Delta.T), 0.0)
    dP = np.where(lower, dO @ Delta.T, 0.0)
    dEm = -dR @ Z.T + dA @ Km
    dQm = dO @ Z.T + dP @ Km
    dKm = dA.T @ Em + dP.T @ Qm + Delta @ dSm.T
    dS_in = np.exp(m)[:, None] * (Qm.T @ dO - Em.T @ dR) + np.exp(g[-1])[:, None] * dS_out

    dq = fm * dQm
    de = fm * dEm
    dk = fp * dKm + b * de
    h = Qm * dQm + Em * dEm - Km * dKm       # frame-invariant: equals the unframed products
    dlog = np.cumsum(h[::-1], axis=0)[::-1] + np.sum(dS_out * S_out, axis=1)[None, :]
    return dq, dk, w * dR, dlog / alpha, k * de, v * dR, dS_in


def chunked_grads_framed(q, k, v, alpha, b, w, S0, dO, dST, C):
    """chunked_grads with chunk_grads_framed (the forward to each chunk's state is framed too)."""
    T, K = q.shape
    V = v.shape[1]
    S = np.zeros((K, V)) if S0 is None else np.array(S0, dtype=np.float64)
    starts = []
    for t0 in range(0, T, C):
        sl = slice(t0, min(T, t0 + C))
        L = sl.stop - sl.start
        starts.append(S)
        g = np.cumsum(np.log(alpha[sl]), axis=0)
        m = 0.5 * (g[0] + g[-1])
        Em, Km = np.exp(g - m) * b[sl] * k[sl], np.exp(m - g) * k[sl]
        with np.errstate(over="ignore"):
            A = np.where(np.tril(np.ones((L, L), dtype=bool), -1), Em @ Km.T, 0.0)
        Delta = np.linalg.solve(np.eye(L) + A, w[sl] * v[sl] - Em @ (np.exp(m)[:, None] * S))
        S = np.exp(g[-1])[:, None] * S + np.exp(g[-1] - m)[:, None] * (Km.T @ Delta)
    out = [np.zeros((T, K)), np.zeros((T, K)), np.zeros((T, V)), np.zeros((T, K)), np.zeros((T, K)),
           np.zeros((T, V))]
    dS = np.zeros((K, V)) if dST is None else np.array(dST, dtype=np.float64)
    for ci in range(len(starts) - 1, -1, -1):
        sl = slice(ci * C, min(T, ci * C + C))
        gr = chunk_grads_framed(q[sl], k[sl], v[sl], alpha[sl], b[sl], w[sl], starts[ci], dO[sl], dS)
        for i in range(6):
            out[i][sl] = gr[i]
        dS = gr[6]
    return tuple(out) + (dS,)


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def tf32(x):
    """Round to tf32 (10 explicit mantissa bits, nearest, ties to even) through fp32; fp64 result."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0xFFF + ((u >> 13) & 1)) & 0xFFFFE000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def chunked_grads_rounded(q, k, v, alpha, b, w, S0, dO, dST, C, rnd):
    """chunked_grads_framed with the number formats of a tensor-core kernel: every operand of a matrix
    product rounded by `rnd` (bf16 or tf32), every product accumulated and every other quantity held
    in fp32, the state carried in fp32, T = (I + A)^-1 formed in fp32.  Used to predict the accuracy
    such a kernel can reach, not as a reference."""
    mm = lambda x, y: _f32(rnd(x) @ rnd(y))
    T, K = q.shape
    V = v.shape[1]
    strict = lambda L: np.tril(np.ones((L, L), dtype=bool), -1)
    lower = lambda L: np.tril(np.ones((L, L), dtype=bool), 0)
    S = np.zeros((K, V)) if S0 is None else _f32(S0)
    saved = []
    for t0 in range(0, T, C):   # forward: each chunk's operands and its incoming state
        sl = slice(t0, min(T, t0 + C))
        L = sl.stop - sl.start
        g = _f32(np.cumsum(_f32(np.log(alpha[sl])), axis=0))
        m = _f32(0.5 * (g[0] + g[-1]))
        fm, fp = _f32(np.exp(g - m)), _f32(np.exp(m - g))
        Em, Qm, Km = _f32(fm * _f32(b[sl] * k[sl])), _f32(fm * q[sl]), _f32(fp * k[sl])
        with np.errstate(over="ignore", invalid="ignore"):
            A = np.where(strict(L), mm(Em, Km.T), 0.0)
            P = np.where(lower(L), mm(Qm, Km.T), 0.0)
        Tm = _f32(np.linalg.inv(np.eye(L) + A))
        Z = _f32(np.exp(m)[:, None] * S)
        Delta = mm(Tm, _f32(_f32(w[sl] * v[sl]) - mm(Em, Z)))
        S_out = _f32(_f32(np.exp(g[-1]))[:, None] * S + _f32(np.exp(g[-1] - m))[:, None] * mm(Km.T, Delta))
        saved.append((sl, L, g, m, fm, fp, Em, Qm, Km, P, Tm, Z, Delta, S_out))
        S = S_out
    out = [np.zeros((T, K)), np.zeros((T, K)), np.zeros((T, V)), np.zeros((T, K)), np.zeros((T, K)),
           np.zeros((T, V))]
    dS = np.zeros((K, V)) if dST is None else _f32(dST)
    for sl, L, g, m, fm, fp, Em, Qm, Km, P, Tm, Z, Delta, S_out in reversed(saved):
        dSm = _f32(_f32(np.exp(g[-1] - m))[:, None] * dS)
        dDelta = _f32(mm(P.T, dO[sl]) + mm(Km, dSm))
        dR = mm(Tm.T, dDelta)
        dA = np.where(strict(L), -mm(dR, Delta.T), 0.0)
        dP = np.where(lower(L), mm(dO[sl], Delta.T), 0.0)
        dEm = _f32(-mm(dR, Z.T) + mm(dA, Km))
        dQm = _f32(mm(dO[sl], Z.T) + mm(dP, Km))
        dKm = _f32(mm(dA.T, Em) + mm(dP.T, Qm) + mm(Delta, dSm.T))
        h = _f32(Qm * dQm + Em * dEm - Km * dKm)
        dlog = _f32(np.cumsum(h[::-1], axis=0)[::-1] + np.sum(dS * S_out, axis=1)[None, :])
        de = _f32(fm * dEm)
        out[0][sl] = _f32(fm * dQm)
        out[1][sl] = _f32(fp * dKm + b[sl] * de)
        out[2][sl] = _f32(w[sl] * dR)
        out[3][sl] = _f32(dlog / alpha[sl])
        out[4][sl] = _f32(k[sl] * de)
        out[5][sl] = _f32(v[sl] * dR)
        dS = _f32(_f32(np.exp(m))[:, None] * (mm(Qm.T, dO[sl]) - mm(Em.T, dR)) + _f32(np.exp(g[-1]))[:, None] * dS)
    return tuple(out) + (dS,)
