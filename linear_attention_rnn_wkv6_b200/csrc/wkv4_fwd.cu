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
// scans": here the T axis of each channel is split into SEG segments, one warp
// each (lane = channel, 32 consecutive channels per CTA for 128-byte loads):
//   phase 1  every warp folds its segment from the empty state -> (a, b, p)
//   phase 2  warp s combines the summaries of segments 0..s-1 (a segment of
//            length L maps state X to e^{-L w} X (+) local, where (+) is the
//            log-space sum) -> the state entering its segment
//   phase 3  every warp reruns its segment from that state and writes y.
// Phase 3 re-reads k and v; the CTA's tile was read moments before, so the
// re-read is served by L2 and HBM traffic stays at the algorithmic bytes.
#include "wkv_launch.cuh"

namespace wkv {

constexpr float kLog2e = 1.4426950408889634f;

struct Wkv4State {
    float a, b, p;   // p in log2 units; represents (a 2^p, b 2^p)
};

// One token of the recurrence (log2 domain).  k2 = k*log2e; w2 = w*log2e.
__device__ __forceinline__ void wkv4_update(Wkv4State &s, float k2, float v, float w2) {
    const float pd = s.p - w2;              // decayed exponent
    const float d = pd - k2;
    const float ex = exp2f(-fabsf(d));      // 0 when pd = -inf
    const bool keep = d >= 0.f;
    const float e1 = keep ? 1.f : ex;
    const float e2 = keep ? ex : 1.f;
    s.a = fmaf(e1, s.a, e2 * v);
    s.b = fmaf(e1, s.b, e2);
    s.p = fmaxf(pd, k2);
}

__device__ __forceinline__ float wkv4_output(const Wkv4State &s, float k2, float v, float u2) {
    const float uk = u2 + k2;
    const float d = s.p - uk;
    const float ex = exp2f(-fabsf(d));
    const bool keep = d >= 0.f;
    const float e1 = keep ? 1.f : ex;
    const float e2 = keep ? ex : 1.f;
    return __fdividef(fmaf(e1, s.a, e2 * v), fmaf(e1, s.b, e2));
}

template <int SEG, int U>
__global__ void __launch_bounds__(32 * SEG)
wkv4_fwd_kernel(int B, int T, int C, const float *__restrict__ k, const float *__restrict__ v,
                const float *__restrict__ w, const float *__restrict__ u, float *__restrict__ y) {
    __shared__ Wkv4State summ[SEG][32];
    const int lane = threadIdx.x & 31;
    const int seg = threadIdx.x >> 5;
    const int groups = (C + 31) / 32;
    const int b = blockIdx.x / groups;
    const int c = (blockIdx.x % groups) * 32 + lane;
    const bool live = c < C;
    const int seglen = (T + SEG - 1) / SEG;
    const int t0 = seg * seglen;
    const int t1 = min(T, t0 + seglen);
    const float w2 = live ? w[c] * kLog2e : 0.f;
    const float u2 = live ? u[c] * kLog2e : 0.f;
    const size_t base = (size_t)b * T * C + c;

    // ---- phase 1: segment summary from the empty state ----
    Wkv4State st{0.f, 0.f, -INFINITY};
    for (int t = t0; t < t1; t += U) {
        float kb[U], vb[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const bool in = live && (t + i < t1);
            kb[i] = in ? __ldg(k + base + (size_t)(t + i) * C) : 0.f;
            vb[i] = in ? __ldg(v + base + (size_t)(t + i) * C) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < U; ++i)
            if (t + i < t1) wkv4_update(st, kb[i] * kLog2e, vb[i], w2);
    }
    summ[seg][lane] = st;
    __syncthreads();

    // ---- phase 2: state entering this segment ----
    Wkv4State in{0.f, 0.f, -INFINITY};
    for (int j = 0; j < seg; ++j) {
        const int L = min(T, (j + 1) * seglen) - j * seglen;
        const Wkv4State loc = summ[j][lane];
        const float pd = in.p - (float)L * w2;   // decay the carried state over segment j
        const float q = fmaxf(pd, loc.p);
        if (q == -INFINITY) continue;            // both empty
        const float e1 = exp2f(pd - q), e2 = exp2f(loc.p - q);
        in.a = fmaf(e1, in.a, e2 * loc.a);
        in.b = fmaf(e1, in.b, e2 * loc.b);
        in.p = q;
    }

    // ---- phase 3: rerun the segment, write y ----
    st = in;
    for (int t = t0; t < t1; t += U) {
        float kb[U], vb[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const bool in_ = live && (t + i < t1);
            kb[i] = in_ ? __ldg(k + base + (size_t)(t + i) * C) : 0.f;
            vb[i] = in_ ? __ldg(v + base + (size_t)(t + i) * C) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < U; ++i) {
            if (t + i < t1 && live) {
                const float k2 = kb[i] * kLog2e;
                y[base + (size_t)(t + i) * C] = wkv4_output(st, k2, vb[i], u2);
                wkv4_update(st, k2, vb[i], w2);
            }
        }
    }
}

cudaError_t wkv4_fwd_launch(int B, int T, int C, const float *k, const float *v, const float *w,
                            const float *u, float *y, cudaStream_t stream) {
    constexpr int SEG = 16, U = 8;
    const int groups = (C + 31) / 32;
    wkv4_fwd_kernel<SEG, U><<<(unsigned)(B * groups), 32 * SEG, 0, stream>>>(B, T, C, k, v, w, u, y);
    return cudaGetLastError();
}

}  // namespace wkv
