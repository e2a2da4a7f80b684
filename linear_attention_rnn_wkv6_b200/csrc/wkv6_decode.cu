// wkv6_decode.cu -- one recurrent RWKV-6 step for B sequences (decode / streaming).
//
// The recurrent inference form ("RWKV Architecture ...", Recurrent Inference
// Formulation: the N x N state is all a step needs from the past) for a single
// token per sequence, with the state carried in HBM between calls:
//   y_b   = r_b (S_b + diag(u) k_b^T v_b)
//   S_b  <- diag(exp(ew_b)) S_b + k_b^T v_b        (in place)
// This is wkv6_fwd_state with T = 1 and the same buffer as initial and final
// state.  The step reads and writes each 16 KB state once, so it is bound by
// HBM (and, for small B*H, by launch latency).
//
// One CTA per (b, h), 256 threads: thread (q, j) owns value column j and the 16
// state rows 16q .. 16q+15, so every row access is one coalesced 256-byte row
// segment.  A thread issues all its state loads before its in-place stores.
#include "wkv_launch.cuh"

namespace wkv {

namespace {

constexpr int kDecThreads = 256;
constexpr int kRowsPerThread = kHead / (kDecThreads / kHead);   // 16 state rows per thread

__global__ void __launch_bounds__(kDecThreads)
wkv6_decode_kernel(int H, int C, const float *__restrict__ r, const float *__restrict__ k,
                   const float *__restrict__ v, const float *__restrict__ w, const float *__restrict__ u,
                   float *__restrict__ state, float *__restrict__ y) {
    static_assert(kRowsPerThread * (kDecThreads / kHead) == kHead, "thread layout covers the state");
    __shared__ float rs[kHead], ks[kHead], ds[kHead], vs[kHead];
    __shared__ float part[kDecThreads / kHead][kHead];
    __shared__ float bonus;
    const int tid = threadIdx.x;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const size_t io = (size_t)b * C + (size_t)h * kHead;   // this head's channels of token b
    const int j = tid & (kHead - 1), q = tid >> 6;

    if (tid < kHead) {
        rs[tid] = r[io + tid];
        ks[tid] = k[io + tid];
        vs[tid] = v[io + tid];
        ds[tid] = expf(w[io + tid]);
    }
    float *S = state + (size_t)bh * kHead * kHead + j;
    float sv[kRowsPerThread];
#pragma unroll
    for (int e = 0; e < kRowsPerThread; ++e) sv[e] = S[(size_t)(kRowsPerThread * q + e) * kHead];
    __syncthreads();

    // bonus scalar c = sum_i r_i u_i k_i (warp 0)
    if (tid < 32) {
        float c = rs[tid] * u[h * kHead + tid] * ks[tid] + rs[tid + 32] * u[h * kHead + tid + 32] * ks[tid + 32];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (tid == 0) bonus = c;
    }
    const float vj = vs[j];
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < kRowsPerThread; ++e) {
        const int i = kRowsPerThread * q + e;
        acc = fmaf(rs[i], sv[e], acc);
        S[(size_t)i * kHead] = fmaf(ds[i], sv[e], ks[i] * vj);
    }
    part[q][j] = acc;
    __syncthreads();
    if (q == 0) {
        float yj = bonus * vj;
#pragma unroll
        for (int qq = 0; qq < kDecThreads / kHead; ++qq) yj += part[qq][j];
        y[io + j] = yj;
    }
}

}  // namespace

cudaError_t wkv6_decode_launch(int B, int C, int H, const float *r, const float *k, const float *v,
                               const float *w, const float *u, float *state, float *y, cudaStream_t stream) {
    wkv6_decode_kernel<<<(unsigned)(B * H), kDecThreads, 0, stream>>>(H, C, r, k, v, w, u, state, y);
    return cudaGetLastError();
}

}  // namespace wkv
