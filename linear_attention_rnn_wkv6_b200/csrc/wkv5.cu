// wkv5.cu -- helpers of the RWKV-5 (static decay) backward.
//
// RWKV-5 ("RWKV Architecture ...", RWKV-5 "Eagle") decays the matrix state by
// the static per-channel factor exp(-w); it is RWKV-6 with the log-decay
// ew_t = -w at every token.  Its backward therefore runs the RWKV-6 backward on
// that constant log-decay and folds the per-token decay gradient into one value
// per channel: dL/dw[c] = -sum_{b,t} dL/dew_t[b][c].  The two kernels here
// write the constant log-decay tensor and do that fold (a fixed summation
// order over b and t, so the result is deterministic).
#include <algorithm>

#include "wkv_launch.cuh"

namespace wkv {

namespace {

// ew[b][t][c] = -w[c] (float4 along c; C is a multiple of 64)
__global__ void wkv5_expand_kernel(size_t n4, int C4, const float4 *__restrict__ w, float4 *__restrict__ ew) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n4; e += (size_t)gridDim.x * blockDim.x) {
        const float4 x = w[e % C4];
        ew[e] = make_float4(-x.x, -x.y, -x.z, -x.w);
    }
}

// dw[c] = -sum over rows (b, t) of dwtok[row][c], rows in increasing order.
// A CTA of 32 x 8 threads covers 32 channels: each of the 8 row groups sums
// every 8th row, then the 8 partials are added in a fixed order.
__global__ void wkv5_dw_reduce_kernel(int rows, int C, const float *__restrict__ dwtok, float *__restrict__ dw) {
    __shared__ float part[8][32];
    const int c = blockIdx.x * 32 + threadIdx.x;
    float acc = 0.f;
    if (c < C)
        for (int row = threadIdx.y; row < rows; row += 8) acc += dwtok[(size_t)row * C + c];
    part[threadIdx.y][threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.y == 0 && c < C) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) s += part[g][threadIdx.x];
        dw[c] = -s;
    }
}

}  // namespace

cudaError_t wkv5_expand_launch(int B, int T, int C, const float *w, float *ew, cudaStream_t stream) {
    const size_t n4 = (size_t)B * T * C / 4;
    const unsigned grid = (unsigned)std::min<size_t>((n4 + 255) / 256, 148 * 16);
    wkv5_expand_kernel<<<grid, 256, 0, stream>>>(n4, C / 4, reinterpret_cast<const float4 *>(w),
                                                 reinterpret_cast<float4 *>(ew));
    return cudaGetLastError();
}

cudaError_t wkv5_dw_reduce_launch(int rows, int C, const float *dwtok, float *dw, cudaStream_t stream) {
    wkv5_dw_reduce_kernel<<<(unsigned)((C + 31) / 32), dim3(32, 8), 0, stream>>>(rows, C, dwtok, dw);
    return cudaGetLastError();
}

}  // namespace wkv
