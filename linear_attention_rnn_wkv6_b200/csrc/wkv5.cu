// wkv5.cu -- helpers of the RWKV-5 (static decay) backward in the recurrence test
// build (libwkv_recurrence.so; the product build runs the tensor-core backward
// with the static decay built in, wkv6_bwd_split.cu).
//
// RWKV-5 ("RWKV Architecture ...", RWKV-5 "Eagle") decays the matrix state by
// the static per-channel factor exp(-w); it is RWKV-6 with the log-decay
// ew_t = -w at every token.  Its backward can therefore run the RWKV-6 backward on
// that constant log-decay and fold the per-token decay gradient into one value
// per channel: dL/dw[c] = -sum_{b,t} dL/dew_t[b][c].  The two kernels here
// write the constant log-decay tensor and do that fold (a fixed summation
// order over b and t, so the result is deterministic).
#include <algorithm>

#include "wkv_launch.cuh"

#if WKV_RECURRENCE_PATHS
namespace wkv {

namespace {

// ew[b][t][c] = -w[c] (float4 along c; C is a multiple of 64)
__global__ void wkv5_expand_kernel(size_t n4, int C4, const float4 *__restrict__ w, float4 *__restrict__ ew) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n4; e += (size_t)gridDim.x * blockDim.x) {
        const float4 x = w[e % C4];
        if (in_range(e, n4)) ew[e] = make_float4(-x.x, -x.y, -x.z, -x.w);
    }
}

// dw[c] = -sum over rows (b, t) of dwtok[row][c], in two fixed-order stages so
// that the result is deterministic and the rows are read by many CTAs at once.
// Stage 1: a CTA of 32 x 8 threads takes 32 channels of one block of `blk` rows
// (64, or more when the rows would need over 65535 blocks); row group y sums rows
// y, y + 8, ... of the block, and the 8 group sums are added in order into
// part[block][c].
constexpr int kRowBlk = 64;
__global__ void wkv5_dw_partial_kernel(int rows, int blk, int C, const float *__restrict__ dwtok,
                                       float *__restrict__ part) {
    __shared__ float grp[8][32];
    const int c = blockIdx.x * 32 + threadIdx.x;
    const int r0 = blockIdx.y * blk, r1 = min(rows, r0 + blk);
    float acc = 0.f;
    if (c < C) {
#pragma unroll 8
        for (int row = r0 + threadIdx.y; row < r1; row += 8) acc += dwtok[(size_t)row * C + c];
    }
    grp[threadIdx.y][threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.y == 0 && c < C) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) s += grp[g][threadIdx.x];
        if (in_range((size_t)blockIdx.y * C + c, (size_t)gridDim.y * C)) part[(size_t)blockIdx.y * C + c] = s;
    }
}

// Stage 2: dw[c] = -(sum of the blocks' partials in block order), one thread per channel.
__global__ void wkv5_dw_final_kernel(int nblk, int C, const float *__restrict__ part, float *__restrict__ dw) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    float s = 0.f;
#pragma unroll 8
    for (int k = 0; k < nblk; ++k) s += part[(size_t)k * C + c];
    dw[c] = -s;
}

}  // namespace

cudaError_t wkv5_expand_launch(int B, int T, int C, const float *w, float *ew, cudaStream_t stream) {
    const size_t n4 = (size_t)B * T * C / 4;
    const unsigned grid = (unsigned)std::min<size_t>((n4 + 255) / 256, 148 * 16);
    wkv5_expand_kernel<<<grid, 256, 0, stream>>>(n4, C / 4, reinterpret_cast<const float4 *>(w),
                                                 reinterpret_cast<float4 *>(ew));
    return cudaGetLastError();
}

cudaError_t wkv5_dw_reduce_launch(int rows, int C, const float *dwtok, float *part, float *dw,
                                  cudaStream_t stream) {
    const int blk = std::max(kRowBlk, (rows + 65534) / 65535);   // at most 65535 blocks (grid y)
    const int nblk = (rows + blk - 1) / blk;
    wkv5_dw_partial_kernel<<<dim3((unsigned)((C + 31) / 32), (unsigned)nblk), dim3(32, 8), 0, stream>>>(
        rows, blk, C, dwtok, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wkv5_dw_final_kernel<<<(unsigned)((C + 255) / 256), 256, 0, stream>>>(nblk, C, part, dw);
    return cudaGetLastError();
}

}  // namespace wkv
#endif  // WKV_RECURRENCE_PATHS
