"""Brute-force O(T^2) sum forms of the WKV operator (numpy, float64).

These are deliberately written in a different shape from the oracle's O(T)
recurrences: every output is an explicit sum over pairs (t, s) with the decay
between them taken as exp of the sum of log-decays strictly between the two
positions.  They pin the oracle; they are never used to produce expected values
for the CUDA path.

RWKV-6 (one head; r,k,v,w: [T,N], u: [N]):
    y_t = sum_s A_ts v_s,   A_ts = sum_i r_t[i] k_s[i] D_ts[i]
    D_ts = exp(sum_{m strictly between s and t} w_m)   for s != t (per direction)
    D_tt = u
RWKV-4 (one channel; k,v: [T]; scalars w > 0, u):
    y_t = [sum_{s<t} e^{k_s - (t-1-s) w} v_s + e^{u+k_t} v_t] / [same without v]
"""
from __future__ import annotations

import numpy as np


def _D(w, s, t, u, past, future, bonus):
    if s == t:
        return u if bonus else None
    if s < t and past:
        return np.exp(w[s + 1:t].sum(axis=0)) if t - s > 1 else np.ones(w.shape[1])
    if s > t and future:
        return np.exp(w[t + 1:s].sum(axis=0)) if s - t > 1 else np.ones(w.shape[1])
    return None


def wkv6_head(r, k, v, w, u, past=True, future=False, bonus=True):
    r, k, v, w, u = (np.asarray(a, dtype=np.float64) for a in (r, k, v, w, u))
    T, N = r.shape
    y = np.zeros((T, N))
    for t in range(T):
        for s in range(T):
            D = _D(w, s, t, u, past, future, bonus)
            if D is None:
                continue
            y[t] += np.sum(r[t] * k[s] * D) * v[s]
    return y


def wkv6(r, k, v, w, u, H, past=True, future=False, bonus=True):
    """Apply wkv6_head to every (b, h) of [B,T,C] arrays."""
    B, T, C = r.shape
    N = C // H
    y = np.zeros((B, T, C))
    for b in range(B):
        for h in range(H):
            sl = slice(h * N, (h + 1) * N)
            y[b, :, sl] = wkv6_head(r[b, :, sl], k[b, :, sl], v[b, :, sl], w[b, :, sl], u[sl],
                                    past, future, bonus)
    return y


def wkv6_head_state(r, k, v, w, u, s0):
    """Causal pair form started from the state s0 ([N,N], row i = key channel).

    The initial state reaches y_t through the decays of tokens 0..t-1 and the
    final state holds every pair decayed to the end:
        y_t  = sum_s A_ts v_s + (r_t * exp(sum_{m<t} w_m)) . s0
        S_T-1 = diag(exp(sum_m w_m)) s0 + sum_s diag(exp(sum_{m>s} w_m)) k_s^T v_s
    """
    r, k, v, w, u, s0 = (np.asarray(a, dtype=np.float64) for a in (r, k, v, w, u, s0))
    T, N = r.shape
    y = wkv6_head(r, k, v, w, u)
    for t in range(T):
        y[t] += (r[t] * np.exp(w[:t].sum(axis=0))) @ s0
    sT = np.exp(w.sum(axis=0))[:, None] * s0
    for s in range(T):
        sT = sT + np.outer(k[s] * np.exp(w[s + 1:].sum(axis=0)), v[s])
    return y, sT


def wkv6_head_grads(r, k, v, w, u, dy, past=True, future=False):
    """Gradients of sum(dy * y) from the pair form (bonus always on).

    dA_ts = <dy_t, v_s>;  dv_s = sum_t A_ts dy_t;  dr_t = sum_s dA_ts k_s D_ts;
    dk_s = sum_t dA_ts r_t D_ts;  du = sum_t dA_tt r_t k_t;
    dw_m = sum_{s != t, m strictly between} dA_ts r_t k_s D_ts.
    """
    r, k, v, w, u, dy = (np.asarray(a, dtype=np.float64) for a in (r, k, v, w, u, dy))
    T, N = r.shape
    dr, dk, dv, dw = (np.zeros((T, N)) for _ in range(4))
    du = np.zeros(N)
    for t in range(T):
        for s in range(T):
            D = _D(w, s, t, u, past, future, True)
            if D is None:
                continue
            dA = float(dy[t] @ v[s])
            A = float(np.sum(r[t] * k[s] * D))
            dv[s] += A * dy[t]
            dr[t] += dA * k[s] * D
            dk[s] += dA * r[t] * D
            if s == t:
                du += dA * r[t] * k[t]
            else:
                lo, hi = min(s, t), max(s, t)
                for m in range(lo + 1, hi):
                    dw[m] += dA * r[t] * k[s] * D
    return dr, dk, dv, dw, du


def wkv4_channel(k, v, w, u):
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T = k.shape[0]
    y = np.zeros(T)
    for t in range(T):
        ex = np.array([k[s] - (t - 1 - s) * w for s in range(t)] + [u + k[t]])
        vs = np.concatenate([v[:t], v[t:t + 1]])
        m = ex.max()
        e = np.exp(ex - m)
        y[t] = float(e @ vs) / float(e.sum())
    return y


def wkv4(k, v, w, u):
    B, T, C = k.shape
    y = np.zeros((B, T, C))
    for b in range(B):
        for c in range(C):
            y[b, :, c] = wkv4_channel(k[b, :, c], v[b, :, c], float(w[c]), float(u[c]))
    return y
