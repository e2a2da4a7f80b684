// wkv_abi.cu -- the extern "C" entry points of libwkv.so (declared in include/wkv.h).
//
// Each entry point validates its arguments on the host (nothing is launched on
// an error), builds the TMA tensor maps the kernel needs, and enqueues the
// kernel(s) on the caller's stream.  No call allocates or synchronises.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/wkv.h"
#include "wkv_launch.cuh"

namespace wkv {

__device__ unsigned int g_wkv_faults = 0;

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D map over a [B][T][C] tensor; box = (box_c channels, box_t tokens, 1).
bool make_map(CUtensorMap *m, const void *ptr, bool bf16, int B, int T, int C, int box_c, int box_t,
              bool swizzle128 = false) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t es = bf16 ? 2 : 4;
    const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)C * es, (cuuint64_t)T * (cuuint64_t)C * es};
    const cuuint32_t box[3] = {(cuuint32_t)box_c, (cuuint32_t)box_t, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    std::memset(m, 0, sizeof(*m));
    CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                     const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// sm_100 check, cached per device (entry points may be called from several host threads).
int check_device() {
    static std::atomic<int> cached[64];   // 0 unknown, 1 ok, 2 bad
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WKV_ERR_CUDA;
    if (dev >= 0 && dev < 64 && cached[dev].load(std::memory_order_relaxed) == 1) return WKV_OK;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return WKV_ERR_CUDA;
    const bool ok = (major == 10 && minor == 0);
    if (dev >= 0 && dev < 64) cached[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
    return ok ? WKV_OK : WKV_ERR_DEVICE;
}

// Result of an entry point that enqueued work (e: the runtime's status after the
// launches).  In the debug build (-DWKV_DEVICE_CHECKS=1) the entry point also waits
// for the device and reports what its kernels' checks recorded in the fault word
// (then cleared): an index out of range as WKV_ERR_DEVICE_CHECK, a bounded wait
// that ran out as WKV_ERR_TIMEOUT.  The other builds never wait.
int launched(cudaError_t e) {
    if (e != cudaSuccess) return WKV_ERR_CUDA;
#if WKV_DEVICE_CHECKS
    if (cudaDeviceSynchronize() != cudaSuccess) return WKV_ERR_CUDA;
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_wkv_faults, sizeof(v)) != cudaSuccess) return WKV_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_wkv_faults, &zero, sizeof(zero)) != cudaSuccess) return WKV_ERR_CUDA;
    if (v & WKV_FAULT_INDEX) return WKV_ERR_DEVICE_CHECK;
    if (v & WKV_FAULT_TIMEOUT) return WKV_ERR_TIMEOUT;
#endif
    return WKV_OK;
}

// Shared checks of the RWKV-6 entry points.
int check_wkv6(int B, int T, int C, int H, std::initializer_list<const void *> ptrs) {
    if (B < 0 || T < 0 || C < 1 || H < 1 || C % H != 0) return WKV_ERR_ARG;
    for (const void *p : ptrs)
        if (p == nullptr) return WKV_ERR_ARG;
    if (C / H != kHead) return WKV_ERR_HEADSIZE;
    if ((long long)B * T * C >= (1ll << 31)) return WKV_ERR_TOO_LARGE;
    for (const void *p : ptrs)
        if (!aligned16(p)) return WKV_ERR_ALIGN;
    return WKV_OK;
}

// Tensor maps of the backward: inputs r, k, w, v, dy, then the outputs dr, dk,
// dv, dw (the second sweep reads back what the first sweep stored there).
bool make_bwd_maps(CUtensorMap (&maps)[kBwdMaps], bool bf16, int B, int T, int C, const void *r, const void *k,
                   const void *w, const void *v, const void *dy, const float *dr, const float *dk,
                   const float *dv, const float *dw) {
    const void *src[kBwdMaps] = {r, k, w, v, dy, dr, dk, dv, dw};
    for (int i = 0; i < kBwdMaps; ++i)
        if (!make_map(&maps[i], src[i], bf16 && i < 5, B, T, C, kHead, kBwdTC)) return false;
    return true;
}

// Algorithm of every entry point that has a chunked tensor-core form (the fp32 and
// bf16 forwards and backwards): fixed when the library is built.  The product
// library (libwkv.so) runs the chunked forms; the test library built with
// -DWKV_RECURRENCE_PATHS=1 (libwkv_recurrence.so) runs the token-by-token
// recurrence kernels behind the same entry points.
#ifndef WKV_RECURRENCE_PATHS
#define WKV_RECURRENCE_PATHS 0
#endif
constexpr bool kTensorCorePaths = !WKV_RECURRENCE_PATHS;

// Scratch of the tensor-core backward: per-batch du partials [B][C] and the S kind's
// per-channel z totals [B][C].
size_t bwd_tensor_workspace_floats(int B, int T, int C, bool bidir) {
    (void)T;
    (void)bidir;
    return 2 * (size_t)B * C;
}

// Shared by wkv6_bwd and wkv6_bwd_bf16 (inputs fp32 or bf16, gradients fp32).
int bwd_common(bool bf16, int B, int T, int C, int H, int bidirectional, const void *r, const void *k,
               const void *v, const void *w, const float *u, const void *dy, float *dr, float *dk, float *dv,
               float *dw, float *du, void *workspace, size_t workspace_bytes, wkv_stream_t stream) {
    int st = check_wkv6(B, T, C, H, {r, k, v, w, u, dy, dr, dk, dv, dw, du});
    if (st != WKV_OK) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (B == 0 || T == 0) {
        if ((st = check_device()) != WKV_OK) return st;
        return launched(cudaMemsetAsync(du, 0, sizeof(float) * (size_t)C, s));
    }
    const bool tensor = kTensorCorePaths;
    // the documented requirement (wkv6_bwd_workspace_bytes) in both builds, although
    // the recurrence uses only its first B*C floats
    const size_t need = bwd_tensor_workspace_floats(B, T, C, bidirectional != 0) * sizeof(float);
    if (workspace == nullptr || workspace_bytes < need) return WKV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return WKV_ERR_ALIGN;
    if ((st = check_device()) != WKV_OK) return st;
    if (tensor) {
        float *ws = static_cast<float *>(workspace);
        BwdParams prm{B, T, C, H, u, dr, dk, dv, dw, ws};
        return launched(wkv6_bwd_split_launch(bf16, bidirectional != 0, r, k, v, w, dy, prm, ws + (size_t)B * C, du, s));
    }
    CUtensorMap maps[kBwdMaps];
    if (!make_bwd_maps(maps, bf16, B, T, C, r, k, w, v, dy, dr, dk, dv, dw)) return WKV_ERR_CUDA;
    BwdParams prm{B, T, C, H, u, dr, dk, dv, dw, static_cast<float *>(workspace)};
    return launched(wkv6_bwd_launch(bf16, bidirectional != 0, maps, prm, du, s));
}

// w5 (RWKV-5): static per-channel decay rate [C]; then w is ignored (pass w5 for
// the argument checks) and the register recurrence runs with the constant log-decay.
// fused: decay prologue and norm/gate epilogue of wkv6_fwd_fused (fp32 kernels).
struct Fused {
    const float *wb, *g, *gn_w, *gn_b;
    float eps;
};

int fwd_common(bool bf16, bool bidir, int B, int T, int C, int H, const void *r, const void *k, const void *v,
               const void *w, const float *u, float *y, wkv_stream_t stream, const float *s0 = nullptr,
               float *sT = nullptr, const float *w5 = nullptr, const Fused *fused = nullptr) {
    int st = check_wkv6(B, T, C, H, {r, k, v, w, u, y});
    if (st != WKV_OK) return st;
    if (B == 0 || T == 0) return WKV_OK;
    if ((st = check_device()) != WKV_OK) return st;
    CUtensorMap mr, mk, mv, mw;
    if (bf16 && !bidir && s0 == nullptr && sT == nullptr && fused == nullptr && kTensorCorePaths) {
        constexpr int kTcChunk = 64;
        CUtensorMap my;
        if (!make_map(&mr, r, true, B, T, C, kHead, kTcChunk, true) ||
            !make_map(&mk, k, true, B, T, C, kHead, kTcChunk, true) ||
            !make_map(&mv, v, true, B, T, C, kHead, kTcChunk, true) ||
            !make_map(&mw, w5 != nullptr ? r : w, true, B, T, C, kHead, kTcChunk, true) ||
            !make_map(&my, y, false, B, T, C, kHead / 2, kTcChunk, true))
            return WKV_ERR_CUDA;
        FwdParams prm{B, T, C, H, u, y};
        prm.w5 = w5;
        return launched(wkv6_fwd_tc_launch(mr, mk, mv, mw, my, prm, reinterpret_cast<cudaStream_t>(stream)));
    }
    if (!bf16 && s0 == nullptr && sT == nullptr && w5 == nullptr && fused == nullptr && kTensorCorePaths &&
        wkv6_fwd_cluster_fits(B, T, H, bidir)) {
        // short sequence, few heads: every chunk of a (b, h) at once, in one cluster
        FwdParams prm{B, T, C, H, u, y};
        return launched(wkv6_fwd_cluster_launch(bidir, static_cast<const float *>(r), static_cast<const float *>(k),
                                                static_cast<const float *>(v), static_cast<const float *>(w), prm,
                                                reinterpret_cast<cudaStream_t>(stream)));
    }
    if (!bf16 && kTensorCorePaths) {
        // the chunked form (faster than the register recurrence at these sizes), with
        // the initial and final states of wkv6_fwd_state, the static decay of wkv5_fwd,
        // or the decay prologue and norm/gate epilogue when fused
        FwdParams prm{B, T, C, H, u, y};
        prm.s0 = s0;
        prm.sT = sT;
        prm.w5 = w5;
        if (fused != nullptr) {
            prm.wb = fused->wb;
            prm.g = fused->g;
            prm.gn_w = fused->gn_w;
            prm.gn_b = fused->gn_b;
            prm.gn_eps = fused->eps;
        }
        return launched(wkv6_fwd_split_launch(bidir, static_cast<const float *>(r), static_cast<const float *>(k),
                                     static_cast<const float *>(v), static_cast<const float *>(w), prm,
                                     reinterpret_cast<cudaStream_t>(stream)));
    }
    // a static decay leaves the w map unread: it is built over r only to be well formed
    if (!make_map(&mr, r, bf16, B, T, C, kHead, kFwdTC) || !make_map(&mk, k, bf16, B, T, C, kHead, kFwdTC) ||
        !make_map(&mv, v, bf16, B, T, C, kHead, kFwdTC) ||
        !make_map(&mw, w5 != nullptr ? r : w, bf16, B, T, C, kHead, kFwdTC))
        return WKV_ERR_CUDA;
    FwdParams prm{B, T, C, H, u, y};
    prm.s0 = s0;
    prm.sT = sT;
    prm.w5 = w5;
    if (!bf16 && fused == nullptr)
        // the test build's fp32 forwards without the fused prologue/epilogue: the
        // register recurrence fed by a transform warp
        return launched(wkv6_fwd_pipe_launch(bidir, mr, mk, mv, mw, prm, reinterpret_cast<cudaStream_t>(stream)));
    if (fused != nullptr) {
        prm.wb = fused->wb;
        prm.g = fused->g;
        prm.gn_w = fused->gn_w;
        prm.gn_b = fused->gn_b;
        prm.gn_eps = fused->eps;
    }
    return launched(wkv6_fwd_launch(bf16, bidir, mr, mk, mv, mw, prm, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace
}  // namespace wkv

using namespace wkv;

extern "C" {

int wkv6_fwd(int B, int T, int C, int H, const float *r, const float *k, const float *v, const float *w,
             const float *u, float *y, wkv_stream_t stream) {
    return fwd_common(false, false, B, T, C, H, r, k, v, w, u, y, stream);
}

int wkv6_fwd_bf16(int B, int T, int C, int H, const uint16_t *r, const uint16_t *k, const uint16_t *v,
                  const uint16_t *w, const float *u, float *y, wkv_stream_t stream) {
    return fwd_common(true, false, B, T, C, H, r, k, v, w, u, y, stream);
}

int wkv6_bidir_fwd(int B, int T, int C, int H, const float *r, const float *k, const float *v, const float *w,
                   const float *u, float *y, wkv_stream_t stream) {
    return fwd_common(false, true, B, T, C, H, r, k, v, w, u, y, stream);
}

int wkv6_fwd_state(int B, int T, int C, int H, const float *r, const float *k, const float *v, const float *w,
                   const float *u, const float *s0, float *y, float *sT, wkv_stream_t stream) {
    int st = check_wkv6(B, T, C, H, {r, k, v, w, u, y});
    if (st != WKV_OK) return st;
    if ((long long)B * H * kHead * kHead >= (1ll << 31)) return WKV_ERR_TOO_LARGE;
    if ((s0 != nullptr && !aligned16(s0)) || (sT != nullptr && !aligned16(sT))) return WKV_ERR_ALIGN;
    if (B == 0) return WKV_OK;
    if (T == 0) {
        // no tokens: the final state is the initial one
        if (sT == nullptr) return WKV_OK;
        if ((st = check_device()) != WKV_OK) return st;
        const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
        const size_t bytes = sizeof(float) * (size_t)B * H * kHead * kHead;
        if (s0 == sT) return WKV_OK;
        const cudaError_t e = s0 != nullptr ? cudaMemcpyAsync(sT, s0, bytes, cudaMemcpyDeviceToDevice, cs)
                                            : cudaMemsetAsync(sT, 0, bytes, cs);
        return launched(e);
    }
    return fwd_common(false, false, B, T, C, H, r, k, v, w, u, y, stream, s0, sT);
}

int wkv6_decode(int B, int C, int H, const float *r, const float *k, const float *v, const float *w,
                const float *u, float *state, float *y, wkv_stream_t stream) {
    if (B < 0 || C < 1 || H < 1 || C % H != 0) return WKV_ERR_ARG;
    if (!r || !k || !v || !w || !u || !state || !y) return WKV_ERR_ARG;
    if (C / H != kHead) return WKV_ERR_HEADSIZE;
    if ((long long)B * H * kHead * kHead >= (1ll << 31)) return WKV_ERR_TOO_LARGE;
    for (const void *p : {(const void *)r, (const void *)k, (const void *)v, (const void *)w, (const void *)u,
                          (const void *)state, (const void *)y})
        if (!aligned16(p)) return WKV_ERR_ALIGN;
    if (B == 0) return WKV_OK;
    const int st = check_device();
    if (st != WKV_OK) return st;
    return launched(wkv6_decode_launch(B, C, H, r, k, v, w, u, state, y, reinterpret_cast<cudaStream_t>(stream)));
}

size_t wkv6_bwd_workspace_bytes(int B, int T, int C, int H, int bidirectional) {
    (void)H;
    if (B < 1 || C < 1 || T < 0) return 0;
    // the tensor-core kernels' scratch (the recurrence needs only the first B*C floats)
    return bwd_tensor_workspace_floats(B, T, C, bidirectional != 0) * sizeof(float);
}

int wkv6_bwd(int B, int T, int C, int H, int bidirectional, const float *r, const float *k, const float *v,
             const float *w, const float *u, const float *dy, float *dr, float *dk, float *dv, float *dw,
             float *du, void *workspace, size_t workspace_bytes, wkv_stream_t stream) {
    return bwd_common(false, B, T, C, H, bidirectional, r, k, v, w, u, dy, dr, dk, dv, dw, du, workspace,
                      workspace_bytes, stream);
}

int wkv6_bwd_bf16(int B, int T, int C, int H, int bidirectional, const uint16_t *r, const uint16_t *k,
                  const uint16_t *v, const uint16_t *w, const float *u, const uint16_t *dy, float *dr, float *dk,
                  float *dv, float *dw, float *du, void *workspace, size_t workspace_bytes, wkv_stream_t stream) {
    return bwd_common(true, B, T, C, H, bidirectional, r, k, v, w, u, dy, dr, dk, dv, dw, du, workspace,
                      workspace_bytes, stream);
}

int wkv6_fwd_fused(int B, int T, int C, int H, int bidirectional, const float *r, const float *k, const float *v,
                   const float *ww, const float *w_base, const float *u, const float *g, const float *gn_weight,
                   const float *gn_bias, float eps, float *out, wkv_stream_t stream) {
    if (!(eps > 0.f) || !std::isfinite(eps)) return WKV_ERR_ARG;
    int st = check_wkv6(B, T, C, H, {w_base, g, gn_weight, gn_bias});
    if (st != WKV_OK) return st;
    const Fused f{w_base, g, gn_weight, gn_bias, eps};
    return fwd_common(false, bidirectional != 0, B, T, C, H, r, k, v, ww, u, out, stream, nullptr, nullptr, nullptr,
                      &f);
}

int wkv5_fwd(int B, int T, int C, int H, const float *r, const float *k, const float *v, const float *w,
             const float *u, float *y, wkv_stream_t stream) {
    return fwd_common(false, false, B, T, C, H, r, k, v, w, u, y, stream, nullptr, nullptr, w);
}

int wkv5_fwd_bf16(int B, int T, int C, int H, const uint16_t *r, const uint16_t *k, const uint16_t *v,
                  const float *w, const float *u, float *y, wkv_stream_t stream) {
    return fwd_common(true, false, B, T, C, H, r, k, v, w, u, y, stream, nullptr, nullptr, w);
}

size_t wkv5_bwd_workspace_bytes(int B, int T, int C, int H) {
    (void)H;
    if (B < 1 || T < 0 || C < 1) return 0;
    if (kTensorCorePaths)   // du partials and z totals (floats), two decay-gradient partials (doubles), [B][C] each
        return (2 * sizeof(float) + 2 * sizeof(double)) * (size_t)B * C;
    return sizeof(float) * (2 * (size_t)B * T * C + 2 * (size_t)B * C);
}

int wkv5_bwd(int B, int T, int C, int H, const float *r, const float *k, const float *v, const float *w,
             const float *u, const float *dy, float *dr, float *dk, float *dv, float *dw, float *du,
             void *workspace, size_t workspace_bytes, wkv_stream_t stream) {
    int st = check_wkv6(B, T, C, H, {r, k, v, w, u, dy, dr, dk, dv, dw, du});
    if (st != WKV_OK) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (B == 0 || T == 0) {
        if ((st = check_device()) != WKV_OK) return st;
        if (cudaMemsetAsync(dw, 0, sizeof(float) * (size_t)C, s) != cudaSuccess) return WKV_ERR_CUDA;
        return launched(cudaMemsetAsync(du, 0, sizeof(float) * (size_t)C, s));
    }
    if (workspace == nullptr || workspace_bytes < wkv5_bwd_workspace_bytes(B, T, C, H)) return WKV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return WKV_ERR_ALIGN;
    if ((st = check_device()) != WKV_OK) return st;
#if !WKV_RECURRENCE_PATHS
    // the tensor-core backward with the static log-decay: workspace = du partials [B][C]
    // and z totals [B][C] (floats), then the S and G kinds' decay-gradient partials [2][B][C]
    float *ws = static_cast<float *>(workspace);
    BwdParams prm{B, T, C, H, u, dr, dk, dv, dw, ws};
    prm.w5 = w;
    prm.w5_part = reinterpret_cast<double *>(ws + 2 * (size_t)B * C);
    return launched(wkv5_bwd_split_launch(r, k, v, dy, prm, ws + (size_t)B * C, du, s));
#else
    // workspace: the constant log-decay [B][T][C], its per-token gradient [B][T][C],
    // then the RWKV-6 backward's own 2 [B][C]
    float *ew = static_cast<float *>(workspace);
    float *dwtok = ew + (size_t)B * T * C;
    float *rest = dwtok + (size_t)B * T * C;
    if (wkv5_expand_launch(B, T, C, w, ew, s) != cudaSuccess) return WKV_ERR_CUDA;
    st = bwd_common(false, B, T, C, H, 0, r, k, v, ew, u, dy, dr, dk, dv, dwtok, du, rest,
                    2 * sizeof(float) * (size_t)B * C, stream);
    if (st != WKV_OK) return st;
    // the fold's per-block partials reuse the log-decay tensor, which the backward no longer reads
    return launched(wkv5_dw_reduce_launch(B * T, C, dwtok, ew, dw, s));
#endif
}

int wkv4_fwd(int B, int T, int C, const float *k, const float *v, const float *w, const float *u, float *y,
             wkv_stream_t stream) {
    if (B < 0 || T < 0 || C < 1 || !k || !v || !w || !u || !y) return WKV_ERR_ARG;
    if ((long long)B * T * C >= (1ll << 31)) return WKV_ERR_TOO_LARGE;
    if (!aligned16(k) || !aligned16(v) || !aligned16(w) || !aligned16(u) || !aligned16(y)) return WKV_ERR_ALIGN;
    if (B == 0 || T == 0) return WKV_OK;
    int st = check_device();
    if (st != WKV_OK) return st;
    return launched(wkv4_fwd_launch(B, T, C, k, v, w, u, y, reinterpret_cast<cudaStream_t>(stream)));
}

size_t wkv4_bwd_workspace_bytes(int B, int T, int C) {
    if (B < 1 || T < 0 || C < 1) return 0;
    return sizeof(float) * ((size_t)B * T * C + 2 * (size_t)B * C);
}

int wkv4_bwd(int B, int T, int C, const float *k, const float *v, const float *w, const float *u, const float *dy,
             float *dk, float *dv, float *dw, float *du, void *workspace, size_t workspace_bytes,
             wkv_stream_t stream) {
    if (B < 0 || T < 0 || C < 1 || !k || !v || !w || !u || !dy || !dk || !dv || !dw || !du) return WKV_ERR_ARG;
    if ((long long)B * T * C >= (1ll << 31)) return WKV_ERR_TOO_LARGE;
    for (const void *p : {(const void *)k, (const void *)v, (const void *)w, (const void *)u, (const void *)dy,
                          (const void *)dk, (const void *)dv, (const void *)dw, (const void *)du})
        if (!aligned16(p)) return WKV_ERR_ALIGN;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int st;
    if (B == 0 || T == 0) {
        if ((st = check_device()) != WKV_OK) return st;
        if (cudaMemsetAsync(dw, 0, sizeof(float) * (size_t)C, s) != cudaSuccess) return WKV_ERR_CUDA;
        return launched(cudaMemsetAsync(du, 0, sizeof(float) * (size_t)C, s));
    }
    if (workspace == nullptr || workspace_bytes < wkv4_bwd_workspace_bytes(B, T, C)) return WKV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return WKV_ERR_ALIGN;
    if ((st = check_device()) != WKV_OK) return st;
    return launched(wkv4_bwd_launch(B, T, C, k, v, w, u, dy, dk, dv, dw, du, static_cast<float *>(workspace), s));
}

const char *wkv_status_string(int status) {
    switch (status) {
        case WKV_OK: return "ok";
        case WKV_ERR_ARG: return "invalid argument (sizes < 0, C != H*N, or a NULL pointer)";
        case WKV_ERR_HEADSIZE: return "unsupported head size (N = C/H must be 64)";
        case WKV_ERR_ALIGN: return "pointer not 16-byte aligned";
        case WKV_ERR_WORKSPACE: return "workspace missing or too small";
        case WKV_ERR_CUDA: return "CUDA runtime or launch error";
        case WKV_ERR_DEVICE: return "current device is not sm_100 (B200)";
        case WKV_ERR_TOO_LARGE: return "problem too large (B*T*C must be < 2^31)";
        case WKV_ERR_DEVICE_CHECK: return "a kernel's index check failed (debug build)";
        case WKV_ERR_TIMEOUT: return "a kernel's bounded wait ran out (debug build)";
        default: return "unknown status";
    }
}

int wkv_take_device_faults(unsigned *faults) {
    if (!faults) return WKV_ERR_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return WKV_ERR_CUDA;
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_wkv_faults, sizeof(v)) != cudaSuccess) return WKV_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_wkv_faults, &zero, sizeof(zero)) != cudaSuccess) return WKV_ERR_CUDA;
    *faults = v;
    return WKV_OK;
}

int wkv_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------
// wkv6_bwd_noalloc: wkv6_bwd for callers that cannot allocate device memory.
//
// The only scratch wkv6_bwd needs is B*C floats of per-batch du partials.  Here
// they live in a fixed file-scope device array instead of a caller-supplied
// workspace.  In host code the array's name is only a host-side stand-in, so
// its device address is looked up with cudaGetSymbolAddress, once per device,
// with that device current (the first call on each device does this).
namespace wkv {
namespace {

constexpr size_t kNoAllocDuFloats = 262144;   // B*C limit: 1 MiB held by every device that loads the library
static __device__ __align__(256) float g_noalloc_du_partials[kNoAllocDuFloats];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float *g_noalloc_ptr[kMaxDevices];
CUcontext g_noalloc_ctx[kMaxDevices];   // the context the address above belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of the scratch array on the current device.  It is looked up
// (cudaGetSymbolAddress, with the device current) on the first call on each
// device, and again whenever the device's context has changed since (after a
// cudaDeviceReset the library's device code is loaded anew and the array may move).
int noalloc_scratch(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WKV_ERR_CUDA;
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (get_ctx == nullptr) return WKV_ERR_CUDA;
    CUcontext ctx = nullptr;   // null until the runtime has made the device's context current here
    if (get_ctx(&ctx) != CUDA_SUCCESS) return WKV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || g_noalloc_ctx[dev] != ctx) {
        void *p = nullptr;   // the lookup also makes the device's primary context current
        if (cudaGetSymbolAddress(&p, g_noalloc_du_partials) != cudaSuccess || p == nullptr) return WKV_ERR_CUDA;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return WKV_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<float *>(p);
        g_noalloc_ctx[dev] = ctx;
    }
    *out = g_noalloc_ptr[dev];
    return WKV_OK;
}

}  // namespace
}  // namespace wkv

extern "C" int wkv6_bwd_noalloc(int B, int T, int C, int H, int bidirectional, const float *r, const float *k,
                                const float *v, const float *w, const float *u, const float *dy, float *dr,
                                float *dk, float *dv, float *dw, float *du, wkv_stream_t stream) {
    int st = check_wkv6(B, T, C, H, {r, k, v, w, u, dy, dr, dk, dv, dw, du});
    if (st != WKV_OK) return st;
    if ((size_t)B * (size_t)C > kNoAllocDuFloats) return WKV_ERR_TOO_LARGE;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = check_device()) != WKV_OK) return st;
    if (B == 0 || T == 0)
        return launched(cudaMemsetAsync(du, 0, sizeof(float) * (size_t)C, s));
    float *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != WKV_OK) return st;
    CUtensorMap maps[kBwdMaps];
    if (!make_bwd_maps(maps, false, B, T, C, r, k, w, v, dy, dr, dk, dv, dw)) return WKV_ERR_CUDA;
    // Every per-batch partial the reduction reads is written first by the
    // backward kernel, so nothing left in the array by an earlier call leaks in.
    BwdParams prm{B, T, C, H, u, dr, dk, dv, dw, scratch};
    return launched(wkv6_bwd_launch(false, bidirectional != 0, maps, prm, du, s));
}

// ---------------------------------------------------------------------------
// wkv_selftest_wait_timeout: exercises the failure path every kernel's bounded
// waits share.  One thread waits on an mbarrier that nothing arrives on; the
// wait gives up after its time limit, records WKV_FAULT_TIMEOUT in the fault
// word and the kernel returns, so the context stays usable.

namespace wkv {
namespace {

__global__ void wkv_wait_selftest_kernel() {
    __shared__ alignas(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait_bounded(&bar, 0);   // phase 0 never completes: runs out after kWaitLimitNs
}

}  // namespace
}  // namespace wkv

extern "C" int wkv_selftest_wait_timeout(wkv_stream_t stream) {
    int st = wkv::check_device();
    if (st != WKV_OK) return st;
    wkv::wkv_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
    return launched(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// wkv_selftest_index_check: exercises the failure path of the index checks.  One
// thread attempts a store whose index equals the size of the array it targets; the
// check (the one every store of the debug build makes, applied here in every
// build) skips the store and records WKV_FAULT_INDEX, and the kernel returns.

namespace wkv {
namespace {

__device__ float g_selftest_sink[4];

__global__ void wkv_index_selftest_kernel(size_t idx, size_t n) {
    if (threadIdx.x == 0 && in_range_checked(idx, n)) g_selftest_sink[idx] = 1.f;
}

}  // namespace
}  // namespace wkv

extern "C" int wkv_selftest_index_check(wkv_stream_t stream) {
    int st = wkv::check_device();
    if (st != WKV_OK) return st;
    wkv::wkv_index_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(4, 4);
    return wkv::launched(cudaGetLastError());
}
