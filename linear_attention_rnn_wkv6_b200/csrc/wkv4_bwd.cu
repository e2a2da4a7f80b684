// wkv4_bwd.cu -- RWKV-4 WKV backward for sm_100a.
//
// Gradients of L = sum_t dy_t y_t for wkv4_fwd ("RWKV Architecture ...", The
// Fundamental Mathematical Duality: y_t = N_t / D_t with the decayed pair weights
// E_ts = e^{k_s - (t-1-s) w} (s < t) and E_tt = e^{u + k_t}).  With g_t = dy_t / D_t:
//   dv_s = e^{k_s} alpha_s + g_s E_ss
//   dk_s = e^{k_s} (v_s alpha_s - beta_s) + g_s E_ss (v_s - y_s)
//   du   = sum_s g_s E_ss (v_s - y_s)
//   dw   = -sum_s e^{k_s} (v_s alpha'_s - beta'_s)
// where the future sums obey, backwards in time,
//   alpha_{s-1} = e^{-w} alpha_s + g_s,          beta_{s-1} = e^{-w} beta_s + g_s y_s,
//   alpha'_{s-1} = e^{-w} (alpha'_s + alpha_s),  beta'_{s-1} = e^{-w} (beta'_s + beta_s)
// (alpha_s = sum_{t>s} g_t e^{-(t-1-s)w}; the primed sums weight each term by t-1-s).
// All four share one log2 exponent q (the running maximum of their terms), like
// the forward's (a, b, p), so nothing overflows: e^{k_s} 2^q <= 1 because the
// step that dominates q includes token s in its own maximum.
//
// Layout as wkv4_fwd: a CTA covers 16 channels of one batch row and splits T
// into 32 segments.  Phases per thread (segment):
//   F1/F2  forward segment summary, then the forward state entering the segment
//   F3     forward rerun: y_t, the scaled g_t and the step's exponent m_t are
//          parked in dv, dk and the workspace (read back by the same thread);
//          the same pass sums the segment's own terms of the four future sums
//          as seen from t0 - 1 (token t weighs e^{-(t - t0) w}, and (t - t0)
//          times that in the primed sums), in time order
//   R2     the sums entering the segment from the right (a segment of length L
//          maps (a, a') to e^{-Lw} (a, a' + L a) before its own terms are added)
//   R3     reverse rerun: dk, dv per token, dw and du accumulated per thread,
//          reduced over the segments into per-(b, c) partials; a second kernel
//          sums the partials over b in a fixed order (deterministic, no atomics).
#include "wkv_launch.cuh"

namespace wkv {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kCh = 16;     // channels per CTA
constexpr int kSeg = 32;    // segments of T per channel
constexpr int kBat = 8;     // tokens whose loads are issued together (the summary pass)
constexpr int kBatR = 4;    // the same for the reruns, which load three or five arrays

__device__ __forceinline__ float ex2(float x) {   // 2^x; -inf gives 0
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct Fwd {
    float a, b, p;   // (a 2^p, b 2^p), p in log2 units
};

struct Rev {
    float al, be, al1, be1, q;   // (alpha, beta, alpha', beta') = (al, be, al1, be1) 2^q
};

__device__ __forceinline__ void fwd_update(Fwd &s, float k2, float v, float w2) {
    const float pd = s.p - w2;
    const float d = pd - k2;
    const float ex = ex2(-fabsf(d));
    const bool keep = d >= 0.f;
    const float e1 = keep ? 1.f : ex;
    const float e2 = keep ? ex : 1.f;
    s.a = fmaf(e1, s.a, e2 * v);
    s.b = fmaf(e1, s.b, e2);
    s.p = fmaxf(pd, k2);
}

// Add a term of the segment summary: x gh 2^{e} (x gh y 2^{e} for beta), weighted by dt in
// the primed sums, e = -m - dt w2 in log2 units for the token dt steps after the segment's
// start.
__device__ __forceinline__ void rev_term(Rev &r, float gh, float y, float m, float dt, float w2) {
    const float e = fmaf(-dt, w2, -m);
    const float qn = fmaxf(r.q, e);
    const float eo = ex2(r.q - qn), en = ex2(e - qn);
    const float g1 = en * gh, gy = g1 * y;
    r.al = fmaf(eo, r.al, g1);
    r.be = fmaf(eo, r.be, gy);
    r.al1 = fmaf(eo, r.al1, dt * g1);
    r.be1 = fmaf(eo, r.be1, dt * gy);
    r.q = qn;
}

// Include token s (scaled g = gh 2^{-m}, output y) into the future sums.
__device__ __forceinline__ void rev_update(Rev &r, float gh, float y, float m, float w2) {
    const float qd = r.q - w2;
    const float qn = fmaxf(qd, -m);
    const float eo = ex2(qd - qn), en = ex2(-m - qn);
    const float al = r.al, be = r.be;
    r.al = fmaf(eo, al, en * gh);
    r.be = fmaf(eo, be, en * gh * y);
    r.al1 = eo * (r.al1 + al);
    r.be1 = eo * (r.be1 + be);
    r.q = qn;
}

// x (+) y for two future-sum states referenced at the same position.
__device__ __forceinline__ Rev rev_add(const Rev &x, const Rev &y) {
    const float q = fmaxf(x.q, y.q);
    if (q == -INFINITY) return x;
    const float ex = ex2(x.q - q), ey = ex2(y.q - q);
    return Rev{fmaf(ex, x.al, ey * y.al), fmaf(ex, x.be, ey * y.be), fmaf(ex, x.al1, ey * y.al1),
               fmaf(ex, x.be1, ey * y.be1), q};
}

__global__ void __launch_bounds__(kCh * kSeg, 2)
wkv4_bwd_kernel(int T, int C, const float *__restrict__ k, const float *__restrict__ v,
                const float *__restrict__ w, const float *__restrict__ u, const float *__restrict__ dy,
                float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ mwork,
                float *__restrict__ dw_part, float *__restrict__ du_part) {
    __shared__ Fwd fsum[kSeg][kCh];
    __shared__ Rev rsum[kSeg][kCh];
    __shared__ float red[2][kSeg][kCh];
    const int tid = threadIdx.x;
    const int ch = tid & (kCh - 1), seg = tid / kCh;
    const int groups = (C + kCh - 1) / kCh;
    const int b = blockIdx.x / groups;
    const int c = (blockIdx.x % groups) * kCh + ch;
    const bool live = c < C;
    const int seglen = (T + kSeg - 1) / kSeg;
    const int t0 = min(T, seg * seglen), t1 = min(T, t0 + seglen);
    const float w2 = live ? w[c] * kLog2e : 0.f;
    const float u2 = live ? u[c] * kLog2e : 0.f;
    const size_t brow = (size_t)b * T * C;   // offsets inside a batch row fit in 32 bits
    const float *kr = k + brow, *vr = v + brow, *gr = dy + brow;
    float *dkr = dk + brow, *dvr = dv + brow, *mr = mwork + brow;

    // ---- F1: forward summary of the segment (the loads of kBat tokens issued before
    // any of them is used; the updates stay in token order)
    Fwd st{0.f, 0.f, -INFINITY};
    if (live)
        for (int t = t0; t < t1; t += kBat) {
            float kk[kBat], vv[kBat];
#pragma unroll
            for (int e = 0; e < kBat; ++e) {
                const int o = (t + e) * C + c;
                kk[e] = t + e < t1 ? kr[o] : 0.f;
                vv[e] = t + e < t1 ? vr[o] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < kBat; ++e)
                if (t + e < t1) fwd_update(st, kk[e] * kLog2e, vv[e], w2);
        }
    fsum[seg][ch] = st;
    __syncthreads();

    // ---- F2: forward state entering the segment
    Fwd in{0.f, 0.f, -INFINITY};
    for (int j = 0; j < seg; ++j) {
        const int L = min(T, (j + 1) * seglen) - min(T, j * seglen);
        const Fwd loc = fsum[j][ch];
        const float pd = in.p - (float)L * w2;
        const float q = fmaxf(pd, loc.p);
        if (q == -INFINITY) continue;
        const float e1 = ex2(pd - q), e2 = ex2(loc.p - q);
        in.a = fmaf(e1, in.a, e2 * loc.a);
        in.b = fmaf(e1, in.b, e2 * loc.b);
        in.p = q;
    }

    // ---- F3: forward rerun; park y, the scaled g and the exponent m of every step, and
    // sum the segment's terms of the future sums (seen from t0 - 1)
    st = in;
    Rev rs{0.f, 0.f, 0.f, 0.f, -INFINITY};
    if (live)
        for (int t = t0; t < t1; t += kBatR) {
            float kk[kBatR], vv[kBatR], gg[kBatR];
#pragma unroll
            for (int e = 0; e < kBatR; ++e) {
                const int o = (t + e) * C + c;
                kk[e] = t + e < t1 ? kr[o] : 0.f;
                vv[e] = t + e < t1 ? vr[o] : 0.f;
                gg[e] = t + e < t1 ? gr[o] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < kBatR; ++e) {
                const int o = (t + e) * C + c;
                if (t + e >= t1) break;
                if (!in_range((size_t)o, (size_t)T * C)) continue;   // y, g, m parked in this row of dv, dk, mwork
                const float k2 = kk[e] * kLog2e, vt = vv[e];
                const float uk = u2 + k2, d = st.p - uk;
                const float ex = ex2(-fabsf(d));
                const bool keep = d >= 0.f;
                const float e1 = keep ? 1.f : ex, e2 = keep ? ex : 1.f;
                const float den = fmaf(e1, st.b, e2);                 // >= 1
                const float yt = __fdividef(fmaf(e1, st.a, e2 * vt), den);   // y_t
                const float gh = __fdividef(gg[e], den);                     // g_t 2^{m_t}
                const float m = fmaxf(st.p, uk);                             // m_t (log2)
                dvr[o] = yt;
                dkr[o] = gh;
                mr[o] = m;
                rev_term(rs, gh, yt, m, (float)(t + e - t0), w2);
                fwd_update(st, k2, vt, w2);
            }
        }

    rsum[seg][ch] = rs;
    __syncthreads();

    // ---- R2: future sums entering the segment from the right (seen from t1 - 1)
    Rev ri{0.f, 0.f, 0.f, 0.f, -INFINITY};
    for (int j = kSeg - 1; j > seg; --j) {
        const int L = min(T, (j + 1) * seglen) - min(T, j * seglen);
        // carry ri through segment j, then add segment j's own terms
        const Rev carried{ri.al, ri.be, ri.al1 + (float)L * ri.al, ri.be1 + (float)L * ri.be, ri.q - (float)L * w2};
        ri = rev_add(carried, rsum[j][ch]);
    }

    // ---- R3: reverse rerun: dk, dv per token; dw, du per thread
    float dwa = 0.f, dua = 0.f;
    if (live)
        for (int t = t1 - 1; t >= t0; t -= kBatR) {
            float gg[kBatR], yy[kBatR], mm[kBatR], kk[kBatR], vv[kBatR];
#pragma unroll
            for (int e = 0; e < kBatR; ++e) {
                const int o = (t - e) * C + c;
                const bool in = t - e >= t0;
                gg[e] = in ? dkr[o] : 0.f;
                yy[e] = in ? dvr[o] : 0.f;
                mm[e] = in ? mr[o] : 0.f;
                kk[e] = in ? kr[o] : 0.f;
                vv[e] = in ? vr[o] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < kBatR; ++e) {
                const int o = (t - e) * C + c;
                if (t - e < t0) break;
                if (!in_range((size_t)o, (size_t)T * C)) continue;   // dk, dv: this batch row
                const float gh = gg[e], yt = yy[e], m = mm[e];
                const float k2 = kk[e] * kLog2e, vt = vv[e];
                const float E = ex2(k2 + ri.q);            // e^{k_s} 2^q
                const float F = ex2(u2 + k2 - m);          // bonus weight E_ss 2^{-m}
                const float gb = gh * F;                   // g_s E_ss
                dvr[o] = fmaf(E, ri.al, gb);
                dkr[o] = fmaf(E, fmaf(vt, ri.al, -ri.be), gb * (vt - yt));
                dwa = fmaf(-E, fmaf(vt, ri.al1, -ri.be1), dwa);
                dua = fmaf(gb, vt - yt, dua);
                rev_update(ri, gh, yt, m, w2);
            }
        }

    // ---- per-(b, c) partials: sum over the segments in a fixed order
    red[0][seg][ch] = dwa;
    red[1][seg][ch] = dua;
    __syncthreads();
    if (seg == 0 && live) {
        float sw = 0.f, su = 0.f;
        for (int j = 0; j < kSeg; ++j) {
            sw += red[0][j][ch];
            su += red[1][j][ch];
        }
        if (in_range((size_t)b * C + c, (size_t)(gridDim.x / groups) * C)) {
            dw_part[(size_t)b * C + c] = sw;
            du_part[(size_t)b * C + c] = su;
        }
    }
}

// dw[c] = sum_b dw_part[b][c], du likewise, in increasing b (deterministic).
__global__ void wkv4_bwd_reduce_kernel(int B, int C, const float *__restrict__ dw_part,
                                       const float *__restrict__ du_part, float *__restrict__ dw,
                                       float *__restrict__ du) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    // eight batches' loads in flight at a time; the additions stay in increasing b
    float sw = 0.f, su = 0.f;
    int b = 0;
    for (; b + 8 <= B; b += 8) {
        float xw[8], xu[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            xw[e] = dw_part[(size_t)(b + e) * C + c];
            xu[e] = du_part[(size_t)(b + e) * C + c];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sw += xw[e];
            su += xu[e];
        }
    }
    for (; b < B; ++b) {
        sw += dw_part[(size_t)b * C + c];
        su += du_part[(size_t)b * C + c];
    }
    if (in_range(c, (size_t)C)) {
        dw[c] = sw;
        du[c] = su;
    }
}

}  // namespace

cudaError_t wkv4_bwd_launch(int B, int T, int C, const float *k, const float *v, const float *w, const float *u,
                            const float *dy, float *dk, float *dv, float *dw, float *du, float *workspace,
                            cudaStream_t stream) {
    const int groups = (C + kCh - 1) / kCh;
    float *mwork = workspace;                               // [B][T][C]
    float *dw_part = workspace + (size_t)B * T * C;         // [B][C]
    float *du_part = dw_part + (size_t)B * C;               // [B][C]
    wkv4_bwd_kernel<<<(unsigned)(B * groups), kCh * kSeg, 0, stream>>>(T, C, k, v, w, u, dy, dk, dv, mwork,
                                                                       dw_part, du_part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wkv4_bwd_reduce_kernel<<<(C + 255) / 256, 256, 0, stream>>>(B, C, dw_part, du_part, dw, du);
    return cudaGetLastError();
}

}  // namespace wkv
