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
// One CTA per (b, h), 256 threads: thread (q, g) owns the 4 x 4 block of rows
// 4q .. 4q+3 and columns 4g .. 4g+3, read and written as float4 (16 threads
// cover a 256-byte row); all state loads are issued before the in-place
// stores, and the column sums over the 16 row blocks go through shared memory.
#include "wkv_launch.cuh"

namespace wkv {

namespace {

constexpr int kDecThreads = 256;
constexpr int kColGroups = kHead / 4;                  // 16 float4 column groups per row
constexpr int kRowBlocks = kDecThreads / kColGroups;   // 16 blocks of 4 rows
static_assert(kRowBlocks * 4 == kHead, "thread layout covers the state");

__global__ void __launch_bounds__(kDecThreads, 4)
wkv6_decode_kernel(int H, int C, const float *__restrict__ r, const float *__restrict__ k,
                   const float *__restrict__ v, const float *__restrict__ w, const float *__restrict__ u,
                   float *__restrict__ state, float *__restrict__ y) {
    __shared__ __align__(16) float rs[kHead], ks[kHead], ds[kHead], vs[kHead];   // vs is read as float4
    __shared__ float4 part[kRowBlocks][kColGroups];
    __shared__ float bonus;
    const int tid = threadIdx.x;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const size_t io = (size_t)b * C + (size_t)h * kHead;   // this head's channels of token b
    const int g = tid % kColGroups, q = tid / kColGroups;

    float4 *S = reinterpret_cast<float4 *>(state + (size_t)bh * kHead * kHead) + g;
    float4 sv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) sv[e] = S[(size_t)(4 * q + e) * kColGroups];
    if (tid < kHead) {
        rs[tid] = r[io + tid];
        ks[tid] = k[io + tid];
        vs[tid] = v[io + tid];
        ds[tid] = expf(w[io + tid]);
    }
    __syncthreads();

    // bonus scalar c = sum_i r_i u_i k_i (warp 0)
    if (tid < 32) {
        float c = rs[tid] * u[h * kHead + tid] * ks[tid] + rs[tid + 32] * u[h * kHead + tid + 32] * ks[tid + 32];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (tid == 0) bonus = c;
    }
    const float4 vj = reinterpret_cast<const float4 *>(vs)[g];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int i = 4 * q + e;
        const float ri = rs[i], di = ds[i], ki = ks[i];
        acc.x = fmaf(ri, sv[e].x, acc.x);
        acc.y = fmaf(ri, sv[e].y, acc.y);
        acc.z = fmaf(ri, sv[e].z, acc.z);
        acc.w = fmaf(ri, sv[e].w, acc.w);
        const size_t si = (size_t)bh * kHead * kHead + (size_t)i * kHead + 4 * g;   // element index in state
        if (in_range_vec(si, 4, (size_t)gridDim.x * kHead * kHead))
            S[(size_t)i * kColGroups] = make_float4(fmaf(di, sv[e].x, ki * vj.x), fmaf(di, sv[e].y, ki * vj.y),
                                                    fmaf(di, sv[e].z, ki * vj.z), fmaf(di, sv[e].w, ki * vj.w));
    }
    part[q][g] = acc;
    __syncthreads();
    if (tid < kHead) {
        // y_j = c v_j + sum over the 16 row blocks of column j
        const float *pf = reinterpret_cast<const float *>(part);
        float yj = bonus * vs[tid];
#pragma unroll
        for (int qq = 0; qq < kRowBlocks; ++qq) yj += pf[qq * kHead + tid];
        if (in_range(io + tid, (size_t)(gridDim.x / H) * C)) y[io + tid] = yj;
    }
}

}  // namespace

cudaError_t wkv6_decode_launch(int B, int C, int H, const float *r, const float *k, const float *v,
                               const float *w, const float *u, float *state, float *y, cudaStream_t stream) {
    wkv6_decode_kernel<<<(unsigned)(B * H), kDecThreads, 0, stream>>>(H, C, r, k, v, w, u, state, y);
    return cudaGetLastError();
}

}  // namespace wkv
