// wkv4_fwd.cu -- RWKV-4 WKV forward for sm_100a.
//
// Operation ("RWKV Architecture ...", The Fundamental Mathematical Duality and
// The Recurrent Inference Formulation), per (b, c), w >= 0, decay e^{-w}:
//   y_t = (a_{t-1} + e^{u+k_t} v_t) / (b_{t-1} + e^{u+k_t}),
//   a_t = e^{-w} a_{t-1} + e^{k_t} v_t,   b_t = e^{-w} b_{t-1} + e^{k_t},   a_{-1} = b_{-1} = 0.
// The pair (a, b) is carried in log space ("yarian.com RWKV overview", 3.2):
// the kernel stores (a, b, p) meaning (a e^p, b e^p), with p the running
// maximum exponent, so e^{k} never overflows and every exp has argument <= 0.
//
// The pages' parallel form computes the sums "via parallel associative prefix
// scans": here the T axis of each channel is split into SEG segments.  A CTA
// covers CH = 16 consecutive channels of one batch row and all SEG segments;
// a warp holds 16 channels x 2 segments (each load instruction reads two
// 64-byte row pieces), so the grid has B * C/16 equal CTAs, enough to spread
// evenly over the SMs.
//   phase 1  every thread folds its segment from the empty state -> (a, b, p)
//   phase 2  the thread of segment s combines the summaries of segments
//            0..s-1 (a segment of length L maps state X to e^{-L w} X (+)
//            local, where (+) is the log-space sum) -> the state entering it
//   phase 3  every thread reruns its segment from that state and writes y.
// Phase 3 re-reads k and v; the CTA's tile was read moments before, so the
// re-read is served by L2 and HBM traffic stays at the algorithmic bytes.
// Per element the work is a handful of FMAs and one ex2 per update or output
// (the larger exponent's factor is exactly 1, so every argument is <= 0 and
// the running denominator b stays >= 1, which the fast division relies on).
#include "wkv_launch.cuh"

namespace wkv {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kCh = 16;     // channels per CTA
constexpr int kSeg = 32;    // segments of T per channel
constexpr int kU = 4;       // tokens loaded ahead per step

struct Wkv4State {
    float a, b, p;   // p in log2 units; represents (a 2^p, b 2^p)
};

// 2^x for x <= 0 (x = -inf gives 0)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One token of the recurrence (log2 domain).  k2 = k*log2e; w2 = w*log2e.
__device__ __forceinline__ void wkv4_update(Wkv4State &s, float k2, float v, float w2) {
    const float pd = s.p - w2;              // decayed exponent
    const float d = pd - k2;
    const float ex = ex2(-fabsf(d));        // 0 when pd = -inf
    const bool keep = d >= 0.f;
    const float e1 = keep ? 1.f : ex;
    const float e2 = keep ? ex : 1.f;
    s.a = fmaf(e1, s.a, e2 * v);
    s.b = fmaf(e1, s.b, e2);
    s.p = fmaxf(pd, k2);
}

__device__ __forceinline__ float wkv4_output(const Wkv4State &s, float k2, float v, float u2) {
    const float d = s.p - (u2 + k2);
    const float ex = ex2(-fabsf(d));
    const bool keep = d >= 0.f;
    const float e1 = keep ? 1.f : ex;
    const float e2 = keep ? ex : 1.f;
    return __fdividef(fmaf(e1, s.a, e2 * v), fmaf(e1, s.b, e2));   // denominator >= 1
}

__global__ void __launch_bounds__(kCh * kSeg, 3)
wkv4_fwd_kernel(int T, int C, const float *__restrict__ k, const float *__restrict__ v,
                const float *__restrict__ w, const float *__restrict__ u, float *__restrict__ y) {
    __shared__ Wkv4State summ[kSeg][kCh];
    const int tid = threadIdx.x;
    const int ch = tid & (kCh - 1);
    const int seg = tid / kCh;
    const int groups = (C + kCh - 1) / kCh;
    const int b = blockIdx.x / groups;
    const int c = (blockIdx.x % groups) * kCh + ch;
    const bool live = c < C;
    const int seglen = (T + kSeg - 1) / kSeg;
    const int t0 = min(T, seg * seglen);
    const int t1 = min(T, t0 + seglen);
    const float w2 = live ? w[c] * kLog2e : 0.f;
    const float u2 = live ? u[c] * kLog2e : 0.f;
    // this batch row's arrays; offsets inside it fit in 32 bits (B*T*C < 2^31)
    const size_t brow = (size_t)b * T * C;
    const float *kr = k + brow, *vr = v + brow;
    float *yr = y + brow;

    // ---- phase 1: segment summary from the empty state ----
    Wkv4State st{0.f, 0.f, -INFINITY};
    int off = t0 * C + c;
    for (int t = t0; t < t1; t += kU) {
        float kb[kU], vb[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            const bool in = live && (t + i < t1);
            kb[i] = in ? __ldg(kr + off + i * C) : 0.f;
            vb[i] = in ? __ldg(vr + off + i * C) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < kU; ++i)
            if (t + i < t1) wkv4_update(st, kb[i] * kLog2e, vb[i], w2);
        off += kU * C;
    }
    summ[seg][ch] = st;
    __syncthreads();

    // ---- phase 2: state entering this segment ----
    Wkv4State in{0.f, 0.f, -INFINITY};
    for (int j = 0; j < seg; ++j) {
        const int L = min(T, (j + 1) * seglen) - min(T, j * seglen);
        const Wkv4State loc = summ[j][ch];
        const float pd = in.p - (float)L * w2;   // decay the carried state over segment j
        const float q = fmaxf(pd, loc.p);
        if (q == -INFINITY) continue;            // both empty
        const float e1 = ex2(pd - q), e2 = ex2(loc.p - q);
        in.a = fmaf(e1, in.a, e2 * loc.a);
        in.b = fmaf(e1, in.b, e2 * loc.b);
        in.p = q;
    }

    // ---- phase 3: rerun the segment, write y ----
    st = in;
    off = t0 * C + c;
    for (int t = t0; t < t1; t += kU) {
        float kb[kU], vb[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            const bool in_ = live && (t + i < t1);
            kb[i] = in_ ? __ldg(kr + off + i * C) : 0.f;
            vb[i] = in_ ? __ldg(vr + off + i * C) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            if (t + i < t1 && live) {
                const float k2 = kb[i] * kLog2e;
                const float yo = wkv4_output(st, k2, vb[i], u2);
                if (in_range((size_t)off + (size_t)i * C, (size_t)T * C)) yr[off + i * C] = yo;
                wkv4_update(st, k2, vb[i], w2);
            }
        }
        off += kU * C;
    }
}

// Four adjacent channels per thread (C % 4 == 0): one 16-byte load brings a token of
// all four, and their chains are independent work for the same thread.  A CTA
// covers 16 channels x kSegV segments (4 threads per token row), loads run one
// batch of kUV tokens ahead of the updates, and full segments skip the per-token
// bounds checks.  Phases as in wkv4_fwd_kernel, except that phase 2 is a
// log-depth (Kogge-Stone) scan over the segments: an element covering a span of
// n tokens is (a, b, p, n), and (left, right) combine to
// (e^{-n_right w} left (+) right, n_left + n_right), which is associative.
constexpr int kSegV = 32;                      // segments of T per channel
constexpr int kUV = 4;                         // tokens per load batch (two batches in flight)

constexpr int VEC = 4;                         // channels per thread (one float4); measured faster than 2
constexpr int kThrV = (kCh / VEC) * kSegV;     // 128 threads
using V = float4;
__device__ __forceinline__ float comp(const float4 &x, int i) { return i == 0 ? x.x : i == 1 ? x.y : i == 2 ? x.z : x.w; }
__device__ __forceinline__ float4 vmake(const float (&o)[4]) { return make_float4(o[0], o[1], o[2], o[3]); }

__global__ void __launch_bounds__(kThrV, 3)
wkv4_fwd_vec_kernel(int T, int C, const float *__restrict__ k, const float *__restrict__ v,
                    const float *__restrict__ w, const float *__restrict__ u, float *__restrict__ y) {
    constexpr int kQ = kCh / VEC;              // threads per token row of the CTA
    __shared__ Wkv4State summ[kSegV][kCh];
    __shared__ float sspan[kSegV][kQ];         // tokens covered by the scan element of each segment
    const int tid = threadIdx.x;
    const int cq = tid % kQ;                   // channel group within the CTA
    const int seg = tid / kQ;
    const int groups = (C + kCh - 1) / kCh;
    const int b = blockIdx.x / groups;
    const int c0 = (blockIdx.x % groups) * kCh + VEC * cq;
    const bool live = c0 < C;                  // C % VEC == 0: the group is whole or absent
    const int seglen = (T + kSegV - 1) / kSegV;
    const int t0 = min(T, seg * seglen);
    const int t1 = min(T, t0 + seglen);
    float w2[VEC], u2[VEC];
    {
        const V wv = live ? *reinterpret_cast<const V *>(w + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
        const V uv = live ? *reinterpret_cast<const V *>(u + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            w2[i] = comp(wv, i) * kLog2e;
            u2[i] = comp(uv, i) * kLog2e;
        }
    }
    const size_t brow = (size_t)b * T * C;
    const float *kr = k + brow + c0, *vr = v + brow + c0;
    float *yr = y + brow + c0;
    const bool full = live && (t1 - t0) == seglen && seglen % kUV == 0;
    auto load = [&](int t, V (&kb)[kUV], V (&vb)[kUV]) {
#pragma unroll
        for (int e = 0; e < kUV; ++e) {
            const bool in = live && t + e < t1;   // the look-ahead batch may pass the segment end
            kb[e] = in ? __ldg(reinterpret_cast<const V *>(kr + (size_t)(t + e) * C)) : make_float4(0.f, 0.f, 0.f, 0.f);
            vb[e] = in ? __ldg(reinterpret_cast<const V *>(vr + (size_t)(t + e) * C)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };

    // ---- phase 1: segment summaries from the empty state ----
    Wkv4State st[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) st[i] = Wkv4State{0.f, 0.f, -INFINITY};
    {
        V kb[kUV], vb[kUV];
        load(t0, kb, vb);
        for (int t = t0; t < t1; t += kUV) {
            V kn[kUV], vn[kUV];
            load(t + kUV, kn, vn);             // past t1 every load is predicated off
#pragma unroll
            for (int e = 0; e < kUV; ++e)
                if (full || t + e < t1) {
#pragma unroll
                    for (int i = 0; i < VEC; ++i) wkv4_update(st[i], comp(kb[e], i) * kLog2e, comp(vb[e], i), w2[i]);
                }
#pragma unroll
            for (int e = 0; e < kUV; ++e) {
                kb[e] = kn[e];
                vb[e] = vn[e];
            }
        }
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) summ[seg][VEC * cq + i] = st[i];
    sspan[seg][cq] = (float)(t1 - t0);
    __syncthreads();

    // ---- phase 2: inclusive scan over the segments, then the state entering this one ----
    {
        float span = (float)(t1 - t0);
#pragma unroll 1
        for (int o = 1; o < kSegV; o <<= 1) {
            Wkv4State left[VEC];
            float lspan = 0.f;
            if (seg >= o) {
#pragma unroll
                for (int i = 0; i < VEC; ++i) left[i] = summ[seg - o][VEC * cq + i];
                lspan = sspan[seg - o][cq];
            }
            __syncthreads();
            if (seg >= o) {
#pragma unroll
                for (int i = 0; i < VEC; ++i) {
                    const float pd = left[i].p - span * w2[i];   // the left span decays over this span
                    const float q = fmaxf(pd, st[i].p);
                    if (q == -INFINITY) continue;                // both empty
                    const float e1 = ex2(pd - q), e2 = ex2(st[i].p - q);
                    st[i].a = fmaf(e1, left[i].a, e2 * st[i].a);
                    st[i].b = fmaf(e1, left[i].b, e2 * st[i].b);
                    st[i].p = q;
                }
                span += lspan;
#pragma unroll
                for (int i = 0; i < VEC; ++i) summ[seg][VEC * cq + i] = st[i];
                sspan[seg][cq] = span;
            }
            __syncthreads();
        }
    }
    // the state entering segment seg is the inclusive scan of segment seg - 1
#pragma unroll
    for (int i = 0; i < VEC; ++i) st[i] = seg > 0 ? summ[seg - 1][VEC * cq + i] : Wkv4State{0.f, 0.f, -INFINITY};

    // ---- phase 3: rerun the segment, write y ----
    {
        V kb[kUV], vb[kUV];
        load(t0, kb, vb);
        for (int t = t0; t < t1; t += kUV) {
            V kn[kUV], vn[kUV];
            load(t + kUV, kn, vn);
#pragma unroll
            for (int e = 0; e < kUV; ++e)
                if (full || (live && t + e < t1)) {
                    float o[VEC];
#pragma unroll
                    for (int i = 0; i < VEC; ++i) {
                        const float k2 = comp(kb[e], i) * kLog2e, vv = comp(vb[e], i);
                        o[i] = wkv4_output(st[i], k2, vv, u2[i]);
                        wkv4_update(st[i], k2, vv, w2[i]);
                    }
                    if (in_range_vec((size_t)c0 + (size_t)(t + e) * C, VEC, (size_t)T * C))
                        *reinterpret_cast<V *>(yr + (size_t)(t + e) * C) = vmake(o);
                }
#pragma unroll
            for (int e = 0; e < kUV; ++e) {
                kb[e] = kn[e];
                vb[e] = vn[e];
            }
        }
    }
}

}  // namespace

cudaError_t wkv4_fwd_launch(int B, int T, int C, const float *k, const float *v, const float *w,
                            const float *u, float *y, cudaStream_t stream) {
    const int groups = (C + kCh - 1) / kCh;
    if (C % VEC == 0) {
        wkv4_fwd_vec_kernel<<<(unsigned)(B * groups), kThrV, 0, stream>>>(T, C, k, v, w, u, y);
        return cudaGetLastError();
    }
    wkv4_fwd_kernel<<<(unsigned)(B * groups), kCh * kSeg, 0, stream>>>(T, C, k, v, w, u, y);
    return cudaGetLastError();
}

}  // namespace wkv
