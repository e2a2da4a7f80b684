"""The chunked form of the RWKV-6 WKV operator, written out in float64 numpy and
checked against the oracle (CPU only).

The tensor-core kernels evaluate the recurrence blockwise ("RWKV Architecture
...", The Parallel Training Formulation): per chunk of L tokens in processing
order, with chunk-local cumulative log-decays, boundary states carried between
chunks, masked intra-chunk products, and the decay gradient assembled from
prefix and suffix sums.  This file restates that algebra on its own (it shares
nothing with the oracle or the CUDA code) in the order a chunk-parallel
evaluation would use it: first every chunk's boundary states (the forward state
entering the chunk and the adjoint leaving it), then each chunk's outputs and
gradients from those states alone, then the decay gradient's carries across
chunks.  Agreement with the oracle to rounding pins the algebra for any chunk
partition, including the one that gives both sweep directions the same time
chunks (the ragged chunk first in the anti-causal order).
"""
import numpy as np
import pytest

import oracle


def _case(T, N, seed):
    g = np.random.default_rng(seed)
    r, k, v, dy = (g.normal(0, 0.7, (T, N)) for _ in range(4))
    ew = -np.exp(g.uniform(-3.0, 0.0, (T, N)))
    u = g.normal(0, 0.5, N)
    return r, k, v, ew, u, dy


def _partition(n, L, ragged_first):
    """Chunks (index arrays, processing order) of a sequence of n positions."""
    if not ragged_first:
        return [np.arange(s, min(n, s + L)) for s in range(0, n, L)]
    head = n % L or L
    return [np.arange(0, head)] + [np.arange(s, s + L) for s in range(head, n, L)]


def _direction(r, k, v, ew, u, dy, chunks, bonus):
    """One sweep in processing order.  Returns y and (dr, dk, dv, dw) in processing
    order and du (bonus part only)."""
    T, N = r.shape
    nc = len(chunks)
    # chunk-local quantities: Lam_p = sum_{m<p} ew_m, Q = r e^Lam, Kt = k e^{-Lam_{s+1}}, Gam = e^{Lam_L}
    loc = []
    for idx in chunks:
        lam = np.concatenate([np.zeros((1, N)), np.cumsum(ew[idx], axis=0)])   # Lam_0 .. Lam_L
        loc.append(dict(idx=idx, E=np.exp(lam[:-1]), F=np.exp(-lam[1:]), gam=np.exp(lam[-1]),
                        Q=r[idx] * np.exp(lam[:-1]), Kt=k[idx] * np.exp(-lam[1:])))
    # ---- phase 1: boundary states.  S_in(c+1) = diag(Gam_c)(S_in(c) + Kt_c^T V_c);
    # G(c) = dL/dS_in(c) = Q_c^T dY_c + diag(Gam_c) G(c+1), G(nc) = 0; the chunk's own
    # state contribution receives Gt(c) = diag(Gam_c) G(c+1).
    S_in = [np.zeros((N, N))]
    for c in range(nc - 1):
        S_in.append(loc[c]["gam"][:, None] * (S_in[c] + loc[c]["Kt"].T @ v[loc[c]["idx"]]))
    G = [None] * (nc + 1)
    G[nc] = np.zeros((N, N))
    for c in range(nc - 1, -1, -1):
        G[c] = loc[c]["Q"].T @ dy[loc[c]["idx"]] + loc[c]["gam"][:, None] * G[c + 1]
    # ---- phase 2: every chunk on its own, from its boundary states
    y = np.zeros((T, N))
    dr, dk, dv = np.zeros((T, N)), np.zeros((T, N)), np.zeros((T, N))
    z, x = np.zeros((T, N)), np.zeros((T, N))
    du = np.zeros(N)
    for c, q in enumerate(loc):
        idx, Q, Kt, V, dY = q["idx"], q["Q"], q["Kt"], v[q["idx"]], dy[q["idx"]]
        n = len(idx)
        low = np.tril(np.ones((n, n)), -1)                 # s < p
        A = (Q @ Kt.T) * low
        dA = (dY @ V.T) * low
        Gt = q["gam"][:, None] * G[c + 1]
        y[idx] = Q @ S_in[c] + A @ V
        dQ = dA @ Kt + dY @ S_in[c].T
        dKt = dA.T @ Q + V @ Gt.T
        dr[idx] = q["E"] * dQ
        dk[idx] = q["F"] * dKt
        dv[idx] = A.T @ dY + Kt @ Gt
        z[idx] = Q * dQ                                     # r_t dr'_t
        x[idx] = Kt * dKt                                   # k_s dk'_s
        if bonus:
            vdy = np.sum(V * dY, axis=1)                    # dy_p . v_p
            cb = np.sum(r[idx] * u * k[idx], axis=1)
            y[idx] += cb[:, None] * V
            dr[idx] += u * k[idx] * vdy[:, None]
            dk[idx] += u * r[idx] * vdy[:, None]
            dv[idx] += cb[:, None] * dY
            du += np.sum(r[idx] * k[idx] * vdy[:, None], axis=0)
    # ---- phase 3: dw_m = sum_{t>m} z_t - sum_{s>=m} x_s, from chunk-local suffix sums
    # plus the totals of the later chunks (the carries)
    dw = np.zeros((T, N))
    zc, xc = np.zeros(N), np.zeros(N)
    for c in range(nc - 1, -1, -1):
        idx = loc[c]["idx"]
        zs = np.cumsum(z[idx][::-1], axis=0)[::-1]          # sum_{t >= p} within the chunk
        xs = np.cumsum(x[idx][::-1], axis=0)[::-1]
        dw[idx] = (zs - z[idx] + zc) - (xs + xc)
        zc, xc = zc + zs[0], xc + xs[0]
    return y, dr, dk, dv, dw, du


def _chunked(r, k, v, ew, u, dy, L, bidirectional, shared_time_chunks):
    T, N = r.shape
    out = [np.zeros((T, N)) for _ in range(5)]
    du = np.zeros(N)
    dirs = [(np.arange(T), True)]
    if bidirectional:
        dirs.append((np.arange(T)[::-1], False))
    for order, bonus in dirs:
        # the anti-causal order is the time order reversed: with shared time chunks its
        # ragged chunk (the last in time) comes first
        chunks = _partition(T, L, ragged_first=shared_time_chunks and not bonus)
        res = _direction(r[order], k[order], v[order], ew[order], u, dy[order], chunks, bonus)
        for o, a in zip(out, res[:5]):
            o[order] += a
        du += res[5]
    return out, du


@pytest.mark.parametrize("bidirectional", [False, True])
@pytest.mark.parametrize("T,L", [(1, 8), (7, 8), (8, 8), (37, 8), (50, 16), (33, 32)])
@pytest.mark.parametrize("shared", [False, True])
def test_chunked_form_matches_oracle(T, L, bidirectional, shared):
    N, H = 8, 1
    r, k, v, ew, u, dy = _case(T, N, seed=100 * T + L)
    (y, dr, dk, dv, dw), du = _chunked(r, k, v, ew, u, dy, L, bidirectional, shared)
    args = [a[None].astype(np.float64) for a in (r, k, v, ew)]
    y_ref = oracle.wkv6_fwd(*args, u, H=H, bidirectional=bidirectional)[0]
    g_ref = oracle.wkv6_bwd(*args, u, dy[None], H=H, bidirectional=bidirectional)
    for got, ref in zip((y, dr, dk, dv, dw), (y_ref,) + tuple(a[0] for a in g_ref[:4])):
        assert np.allclose(got, ref, rtol=1e-9, atol=1e-10)
    assert np.allclose(du, g_ref[4], rtol=1e-9, atol=1e-10)


def _anti_time_ordered(r, k, v, ew, dy, L):
    """The anti-causal sweep on time-ordered chunk tiles: per chunk the log-decay sums run
    over the later tokens (Lam^a_t = sum_{m>t} ew_m), Q^a_t = r_t e^{Lam^a_t},
    Kt^a_s = k_s e^{-(ew_s + Lam^a_s)}, the masks are strict-upper, the state enters a chunk
    from the later chunks and the adjoint from the earlier ones."""
    T, N = r.shape
    chunks = _partition(T, L, ragged_first=False)
    nc = len(chunks)
    loc = []
    for idx in chunks:
        suf = np.cumsum(ew[idx][::-1], axis=0)[::-1]          # sum_{m >= t}
        lam = suf - ew[idx]                                     # sum_{m > t}
        loc.append(dict(idx=idx, E=np.exp(lam), F=np.exp(-suf), gam=np.exp(suf[0]),
                        Q=r[idx] * np.exp(lam), Kt=k[idx] * np.exp(-suf)))
    S_in = [None] * nc
    S_in[nc - 1] = np.zeros((N, N))
    for j in range(nc - 2, -1, -1):
        q = loc[j + 1]
        S_in[j] = q["gam"][:, None] * (S_in[j + 1] + q["Kt"].T @ v[q["idx"]])
    G = [None] * (nc + 1)          # G[j + 1] = dL/dS_in(j); G[0] = 0
    G[0] = np.zeros((N, N))
    for j in range(nc):
        G[j + 1] = loc[j]["Q"].T @ dy[loc[j]["idx"]] + loc[j]["gam"][:, None] * G[j]
    y, dr, dk, dv, z, x = (np.zeros((T, N)) for _ in range(6))
    for j, q in enumerate(loc):
        idx, Q, Kt, V, dY = q["idx"], q["Q"], q["Kt"], v[q["idx"]], dy[q["idx"]]
        n = len(idx)
        up = np.triu(np.ones((n, n)), 1)                      # s > t
        A = (Q @ Kt.T) * up
        dA = (dY @ V.T) * up
        Gt = q["gam"][:, None] * G[j]
        y[idx] = Q @ S_in[j] + A @ V
        dQ = dA @ Kt + dY @ S_in[j].T
        dKt = dA.T @ Q + V @ Gt.T
        dr[idx], dk[idx], dv[idx] = q["E"] * dQ, q["F"] * dKt, A.T @ dY + Kt @ Gt
        z[idx], x[idx] = Q * dQ, Kt * dKt
    # dw_m = sum_{t<m} z_t - sum_{s<=m} x_s (the tokens processed after m come earlier in time)
    zc = np.cumsum(z, axis=0) - z
    xc = np.cumsum(x, axis=0)
    return y, dr, dk, dv, zc - xc


@pytest.mark.parametrize("T,L", [(7, 8), (37, 8), (50, 16), (33, 32)])
def test_anti_causal_sweep_on_time_ordered_tiles(T, L):
    """Causal part from the processing-order model plus the anti-causal part on time-ordered
    tiles reproduce the oracle's bidirectional forward and gradients."""
    N, H = 8, 1
    r, k, v, ew, u, dy = _case(T, N, seed=7 * T + L)
    (yc, drc, dkc, dvc, dwc), duc = _chunked(r, k, v, ew, u, dy, L, False, False)
    ya, dra, dka, dva, dwa = _anti_time_ordered(r, k, v, ew, dy, L)
    args = [a[None] for a in (r, k, v, ew)]
    y_ref = oracle.wkv6_fwd(*args, u, H=H, bidirectional=True)[0]
    g_ref = oracle.wkv6_bwd(*args, u, dy[None], H=H, bidirectional=True)
    got = (yc + ya, drc + dra, dkc + dka, dvc + dva, dwc + dwa)
    for a, ref in zip(got, (y_ref,) + tuple(g[0] for g in g_ref[:4])):
        assert np.allclose(a, ref, rtol=1e-9, atol=1e-10)
    assert np.allclose(duc, g_ref[4], rtol=1e-9, atol=1e-10)
