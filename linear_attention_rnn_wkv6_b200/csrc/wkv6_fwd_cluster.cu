// wkv6_fwd_cluster.cu -- RWKV-6 fp32 forward (causal and bidirectional) for short
// sequences and few heads: every chunk of a (b, h) at once, in one thread-block
// cluster, on the 5th-generation tensor cores.
//
// Same operation as wkv6_fwd_split.cu (chunks of L = 32 tokens, operands split
// exactly into three bf16 terms, six MMAs per product), but instead of one CTA
// carrying the state through the chunks of its (b, h) one after another, a
// cluster of kCw CTAs takes one chunk each (T <= kCw * L):
//   1. each CTA forms its chunk's tiles, in time order, with the chunk-local
//      cumulative log-decay Lam_p = sum_{m<p} ew_m and its total Lam_L:
//        causal  Q_p = r_p e^{Lam_p},          Kt_s = k_s e^{-Lam_{s+1}}
//        anti    Qa_p = r_p e^{Lam_L-Lam_{p+1}}, Kta_s = k_s e^{Lam_s-Lam_L}
//      and its local state contributions (the state each sweep would carry out of
//      the chunk from a zero state entering it, "RWKV Architecture ...", The
//      Parallel Training Formulation evaluated blockwise):
//        X  = diag(Gam) Kt^T V    (causal: the state after the chunk's last token)
//        Xa = diag(Gam) Kta^T V   (anti-causal: the state at the chunk's first token)
//      with Gam = e^{Lam_L} (the product of the chunk's decays), and the intra-chunk
//      matrices A = Q Kt^T (used below the diagonal) and Aa = Qa Kta^T (above it);
//   2. X, Xa and Gam go to shared memory; after a cluster barrier each CTA reads
//      those of the other chunks through distributed shared memory and folds them
//      into the states entering its own chunk ("How Custom CUDA Kernels
//      (wkv6_cuda.cu) ...", Forward Pass: the past-to-future state, and the
//      future-to-past one of the bidirectional form):
//        S_in  = fold over i = 0 .. j-1 of      F <- diag(Gam_i) F + X_i
//        Sa_in = fold over i = n-1 .. j+1 of    F <- diag(Gam_i) F + Xa_i
//   3. Y = A' V + Q S_in + Qa Sa_in with A' = strict-lower(A) + strict-upper(Aa)
//      + diag(c) (c_p = sum_i r_p u k_p, the bonus), one accumulator, one store.
// No chunk waits for another chunk's result beyond the one exchange, so the
// latency of a (b, h) is that of one chunk.  A chunk whose summed |ew| exceeds 80
// in some channel (fast-forgetting channels, decay exactly 0) computes X, Xa, Gam
// and y token by token on the CUDA cores instead, from the same folded states.
//
// One CTA of 128 threads per chunk, one cluster of kCw CTAs per (b, h) (CTAs past
// the last chunk only take part in the barriers).  Shared memory: the token tiles,
// A', the two folded states as bf16 terms and the two local states in fp32.
#include "wkv_launch.cuh"
#include "wkv_tc.cuh"

namespace wkv {

using namespace tc;

namespace {

constexpr int kCw = 8;                   // CTAs (chunks) per cluster
constexpr int kClusterMaxHeads = 32;     // at most this many (b, h) units: one cluster each
constexpr int kCL = 32;                  // tokens per chunk
constexpr int kCNT = 3;                  // bf16 terms per operand
constexpr int kCNP = 6;                  // products per contraction
constexpr int kCThr = 128;
constexpr int kCTok = kCL * kHead;       // bf16 elements of a 32 x 64 tile (4 KB)
constexpr int kCAp = kCL * kCL;          // bf16 elements of the 32 x 32 A' tile (2 KB)
constexpr int kCSt = kHead * kHead;      // bf16 elements of a 64 x 64 state tile (8 KB)
constexpr float kLog2eC = 1.4426950408889634f;
constexpr float kLamMaxC = 80.0f * kLog2eC;   // |Lam| bound of the tensor-core path, log2 units

__device__ __forceinline__ constexpr int cprod_a(int q) { return q == 2 ? 1 : q == 4 ? 1 : q == 5 ? 2 : 0; }
__device__ __forceinline__ constexpr int cprod_b(int q) { return q == 1 ? 1 : q == 3 ? 2 : q == 4 ? 1 : 0; }

constexpr uint32_t kHi16c = 0xFFFF0000u;
// x = t0 + t1 + t2 exactly: three bf16 values (the high halves of fp32 words) holding
// x's significand 8 bits at a time; the remainders are exact in fp32.
__device__ __forceinline__ void csplit3(float x, uint32_t &t0, uint32_t &t1, uint32_t &t2) {
    t0 = __float_as_uint(x) & kHi16c;
    const float r1 = x - __uint_as_float(t0);
    t1 = __float_as_uint(r1) & kHi16c;
    t2 = __float_as_uint(r1 - __uint_as_float(t1)) & kHi16c;
}
__device__ __forceinline__ uint32_t cpack(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7632); }

// values a, b at (row, col), (row, col + 1) of three 128B-swizzled term tiles
__device__ __forceinline__ void cput_pair3(__nv_bfloat16 (*tiles)[kCTok], int row, int col, float a, float b) {
    uint32_t a0, a1, a2, b0, b1, b2;
    csplit3(a, a0, a1, a2);
    csplit3(b, b0, b1, b2);
    const uint32_t o = swz(row, col);
    st_u32(tiles[0], o, cpack(a0, b0));
    st_u32(tiles[1], o, cpack(a1, b1));
    st_u32(tiles[2], o, cpack(a2, b2));
}

// No-swizzle K-major descriptor of A' (32 rows, 16-byte units 512 B apart), k-step ks.
__device__ __forceinline__ uint64_t cdesc_ap(const __nv_bfloat16 *tile, int ks) {
    return smem_desc(reinterpret_cast<const char *>(tile) + ks * 1024, 512, 128);
}
__device__ __forceinline__ uint64_t cdadd(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

__device__ __forceinline__ uint32_t cl_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cl_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address in CTA `rank`'s shared memory of what `local` is in this CTA's.
__device__ __forceinline__ uint32_t cl_map(const void *local, uint32_t rank) {
    uint32_t remote;
    asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    return remote;
}
// Loads from another CTA's shared memory, after a cluster barrier that ordered its stores.
__device__ __forceinline__ float4 cl_ld4(uint32_t addr) {
    float4 x;
    asm("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w) : "r"(addr));
    return x;
}
__device__ __forceinline__ float cl_ld1(uint32_t addr) {
    float x;
    asm("ld.shared::cluster.f32 %0, [%1];" : "=f"(x) : "r"(addr));
    return x;
}

struct ClusterSmem {
    // token tiles (32 rows of 64 bf16, 128B-swizzled), time order
    __nv_bfloat16 Q[kCNT][kCTok];       // K-major A of A = Q Kt^T and of Y += Q S_in
    __nv_bfloat16 Kt[kCNT][kCTok];      // K-major B of A; MN-major A of X = Kt^T V
    __nv_bfloat16 Qa[kCNT][kCTok];      // anti-causal counterparts
    __nv_bfloat16 Kta[kCNT][kCTok];
    __nv_bfloat16 V[kCNT][kCTok];       // MN-major B of X, Xa and of Y += A' V
    __nv_bfloat16 Ap[kCNT][kCAp];       // A' (row p, s contiguous), no swizzle
    __nv_bfloat16 Sin[kCNT][kCSt];      // S_in (row i, j contiguous), 128B-swizzled: MN-major B
    __nv_bfloat16 Sain[kCNT][kCSt];     // Sa_in likewise
    float X[kHead][kHead];              // local causal state (read by the later chunks)
    float Xa[kHead][kHead];             // local anti-causal state (read by the earlier chunks)
    float gam[kHead];                   // product of the chunk's decays per channel (read by the others)
    float psum[4][kHead], pabs[4][kHead];
    float cp[kCL];                      // bonus scalars per token
    float u[kHead];
    uint32_t tmem_base;
    alignas(8) uint64_t bar_a, bar_y, bar_fin;
};
static_assert(offsetof(ClusterSmem, Q) % 1024 == 0 && offsetof(ClusterSmem, Kt) % 1024 == 0 &&
                  offsetof(ClusterSmem, Qa) % 1024 == 0 && offsetof(ClusterSmem, Kta) % 1024 == 0 &&
                  offsetof(ClusterSmem, V) % 1024 == 0 && offsetof(ClusterSmem, Sin) % 1024 == 0 &&
                  offsetof(ClusterSmem, Sain) % 1024 == 0 && offsetof(ClusterSmem, X) % 16 == 0,
              "swizzled tiles on 1024-byte boundaries, states 16-byte aligned");
// exact chunks: raw fp32 inputs in the token tiles, the running state and y in the state tiles
struct ClusterExact {
    float r[kCL][kHead], k[kCL][kHead], v[kCL][kHead], d[kCL][kHead];
};
static_assert(sizeof(ClusterExact) <= offsetof(ClusterSmem, Ap) - offsetof(ClusterSmem, Q), "raw chunk fits");
struct ClusterExactState {
    float S[kHead][kHead];    // causal state entering the chunk, then running
    float Sa[kHead][kHead];   // anti-causal state entering the chunk, then running
    float y[kCL][kHead];      // the anti-causal sweep's outputs
    float red[2][kHead];      // the two row halves' partial sums of a readout
};
static_assert(sizeof(ClusterExactState) <= 2 * sizeof(__nv_bfloat16) * kCNT * kCSt, "exact state fits");

}  // namespace

template <bool BIDIR>
__global__ void __cluster_dims__(kCw, 1, 1) __launch_bounds__(kCThr, 1)
wkv6_fwd_cluster_kernel(const float *__restrict__ r, const float *__restrict__ k, const float *__restrict__ v,
                        const float *__restrict__ w, FwdParams prm) {
    extern __shared__ unsigned char smem_dyn[];
    ClusterSmem &sm = *reinterpret_cast<ClusterSmem *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    ClusterExact &xr = *reinterpret_cast<ClusterExact *>(&sm.Q[0][0]);
    ClusterExactState &xs = *reinterpret_cast<ClusterExactState *>(&sm.Sin[0][0]);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = prm.T, C = prm.C, H = prm.H;
    const uint32_t j = cl_rank();                       // this CTA's chunk
    const int bh = blockIdx.x / kCw;
    const int h = bh % H, b = bh / H;
    const int cbase = h * kHead;
    const int nch = (T + kCL - 1) / kCL;                // chunks of the sequence (<= kCw)
    const bool live = (int)j < nch;
    const int t0 = (int)j * kCL;
    const int n = live ? min(kCL, T - t0) : 0;          // tokens of this chunk
    const int ch = 2 * lane, pq = 8 * warp;             // transform: channels ch, ch + 1; tokens pq .. pq + 7
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const size_t nBTC = (size_t)prm.B * T * C;

    if (tid < kHead) sm.u[tid] = prm.u[cbase + tid];
    if (tid == 0) {
        mbar_init(&sm.bar_a, 1);
        mbar_init(&sm.bar_y, 1);
        mbar_init(&sm.bar_fin, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 256);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // TMEM (M = 64 layouts): X at 0..63, Xa at 64..127, A at 128..159, Aa at 160..191, Y at 192..255
    const uint32_t tX = sm.tmem_base, tXa = sm.tmem_base + 64, tA = sm.tmem_base + 128, tAa = sm.tmem_base + 160,
                   tY = sm.tmem_base + 192;

    // ---- load the chunk (tokens pq .. pq + 7 of this warp, channels ch, ch + 1)
    float2 xr_[8], xk_[8], xv_[8], xw_[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int p = pq + e;
        if (p < n) {
            const size_t o = ((size_t)b * T + t0 + p) * C + cbase + ch;
            xr_[e] = __ldg(reinterpret_cast<const float2 *>(r + o));
            xk_[e] = __ldg(reinterpret_cast<const float2 *>(k + o));
            xv_[e] = __ldg(reinterpret_cast<const float2 *>(v + o));
            xw_[e] = __ldg(reinterpret_cast<const float2 *>(w + o));
        } else {
            xr_[e] = xk_[e] = xv_[e] = xw_[e] = make_float2(0.f, 0.f);
        }
    }
    // ---- decay sums: this warp's quarter, then the prefix and the total per channel
    {
        float s0 = 0.f, s1 = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            s0 += xw_[e].x * kLog2eC;
            s1 += xw_[e].y * kLog2eC;
            a0 += fabsf(xw_[e].x * kLog2eC);
            a1 += fabsf(xw_[e].y * kLog2eC);
        }
        *reinterpret_cast<float2 *>(&sm.psum[warp][ch]) = make_float2(s0, s1);
        *reinterpret_cast<float2 *>(&sm.pabs[warp][ch]) = make_float2(a0, a1);
    }
    __syncthreads();
    float L0 = 0.f, L1 = 0.f, tot0 = 0.f, tot1 = 0.f, ab0 = 0.f, ab1 = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 ps = *reinterpret_cast<const float2 *>(&sm.psum[q][ch]);
        const float2 pa = *reinterpret_cast<const float2 *>(&sm.pabs[q][ch]);
        if (q < warp) {
            L0 += ps.x;
            L1 += ps.y;
        }
        tot0 += ps.x;
        tot1 += ps.y;
        ab0 += pa.x;
        ab1 += pa.y;
    }
    // every warp reads the same sums in the same order: the verdict is CTA-uniform
    const bool exact = __any_sync(0xffffffffu, !(ab0 <= kLamMaxC) || !(ab1 <= kLamMaxC));
    const float u0 = sm.u[ch], u1 = sm.u[ch + 1];
    {
        float bp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) bp[e] = fmaf(xr_[e].x * u0, xk_[e].x, xr_[e].y * u1 * xk_[e].y);
        const float cpv = transpose_reduce8(bp, lane);
        if ((lane & 3) == 0) sm.cp[pq + (lane >> 2)] = cpv;
    }
    bool ok = true;
    if (!exact) {
        if (warp == 0) *reinterpret_cast<float2 *>(&sm.gam[ch]) = make_float2(exp2f(tot0), exp2f(tot1));
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int p = pq + e;
            const float2 rr = xr_[e], kk = xk_[e];
            // L = Lam_p here; the anti-causal factors use Lam_L - Lam_{p+1} and Lam_p - Lam_L
            const float Lp0 = L0, Lp1 = L1;
            L0 += xw_[e].x * kLog2eC;
            L1 += xw_[e].y * kLog2eC;
            cput_pair3(sm.Q, p, ch, rr.x * fast_exp2(Lp0), rr.y * fast_exp2(Lp1));
            cput_pair3(sm.Kt, p, ch, kk.x * fast_exp2(-L0), kk.y * fast_exp2(-L1));
            if (BIDIR) {
                cput_pair3(sm.Qa, p, ch, rr.x * fast_exp2(tot0 - L0), rr.y * fast_exp2(tot1 - L1));
                cput_pair3(sm.Kta, p, ch, kk.x * fast_exp2(Lp0 - tot0), kk.y * fast_exp2(Lp1 - tot1));
            }
            cput_pair3(sm.V, p, ch, xv_[e].x, xv_[e].y);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int p = pq + e;
            *reinterpret_cast<float2 *>(&xr.r[p][ch]) = xr_[e];
            *reinterpret_cast<float2 *>(&xr.k[p][ch]) = xk_[e];
            *reinterpret_cast<float2 *>(&xr.v[p][ch]) = xv_[e];
            // decay factors; tokens past the chunk keep the state (d = 1, k = v = 0)
            *reinterpret_cast<float2 *>(&xr.d[p][ch]) =
                p < n ? make_float2(__expf(xw_[e].x), __expf(xw_[e].y)) : make_float2(1.f, 1.f);
        }
    }
    fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    constexpr uint32_t kTokB = kCTok * 2, kApB = kCAp * 2, kStB = kCSt * 2;
    constexpr uint32_t kIdA = idesc_bf16(64, 32, false, false);   // Q (K-major) x Kt (K-major)
    constexpr uint32_t kIdX = idesc_bf16(64, 64, true, true);     // Kt^T (MN) x V (MN)
    constexpr uint32_t kIdAV = idesc_bf16(64, 64, false, true);   // A' (K) x V (MN)
    constexpr uint32_t kIdQS = idesc_bf16(64, 64, false, true);   // Q (K) x S_in (MN)
    const uint64_t dQ = desc_k(sm.Q[0], 0), dKk = desc_k(sm.Kt[0], 0), dKm = desc_mn(sm.Kt[0], 0, 16);
    const uint64_t dQa = desc_k(sm.Qa[0], 0), dKak = desc_k(sm.Kta[0], 0), dKam = desc_mn(sm.Kta[0], 0, 16);
    const uint64_t dV = desc_mn(sm.V[0], 0, 16), dAp = cdesc_ap(sm.Ap[0], 0);
    const uint64_t dS = desc_mn(sm.Sin[0], 0, 16), dSa = desc_mn(sm.Sain[0], 0, 16);

    if (!exact) {
        // ===== X = Kt^T V, A = Q Kt^T (and Xa, Aa): one issuing thread =====
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int q = 0; q < kCNP; ++q)
                    mma_bf16(tX, cdadd(dKm, cprod_a(q) * kTokB + 2048 * ks), cdadd(dV, cprod_b(q) * kTokB + 2048 * ks),
                             kIdX, ks > 0 || q > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                for (int q = 0; q < kCNP; ++q)
                    mma_bf16(tA, cdadd(dQ, cprod_a(q) * kTokB + 32 * ks), cdadd(dKk, cprod_b(q) * kTokB + 32 * ks),
                             kIdA, ks > 0 || q > 0);
            if (BIDIR) {
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                    for (int q = 0; q < kCNP; ++q)
                        mma_bf16(tXa, cdadd(dKam, cprod_a(q) * kTokB + 2048 * ks),
                                 cdadd(dV, cprod_b(q) * kTokB + 2048 * ks), kIdX, ks > 0 || q > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int q = 0; q < kCNP; ++q)
                        mma_bf16(tAa, cdadd(dQa, cprod_a(q) * kTokB + 32 * ks),
                                 cdadd(dKak, cprod_b(q) * kTokB + 32 * ks), kIdA, ks > 0 || q > 0);
            }
            mma_commit(&sm.bar_a);
        }
        ok = mbar_wait_bounded(&sm.bar_a, 0);
        ok = __syncthreads_and(ok);
        fence_after_sync();
        if (ok) {
            // ===== local states: rows i of X (and Xa) times Gam_i, to shared memory (all warps) =====
            {
                const int q4 = lane & 3;
                float xv[32];
                tmem_ld_16x256b_x8(tX + lane_off, xv);
                tmem_wait_ld();
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int i = 16 * warp + (lane >> 2) + 8 * hr;
                    const float g = sm.gam[i];
#pragma unroll
                    for (int m = 0; m < 8; ++m)
                        *reinterpret_cast<float2 *>(&sm.X[i][8 * m + 2 * q4]) =
                            make_float2(g * xv[4 * m + 2 * hr], g * xv[4 * m + 2 * hr + 1]);
                }
                if (BIDIR) {
                    tmem_ld_16x256b_x8(tXa + lane_off, xv);
                    tmem_wait_ld();
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int i = 16 * warp + (lane >> 2) + 8 * hr;
                        const float g = sm.gam[i];
#pragma unroll
                        for (int m = 0; m < 8; ++m)
                            *reinterpret_cast<float2 *>(&sm.Xa[i][8 * m + 2 * q4]) =
                                make_float2(g * xv[4 * m + 2 * hr], g * xv[4 * m + 2 * hr + 1]);
                    }
                }
            }
            // ===== A' = strict-lower(A) + strict-upper(Aa) + diag(c) (warps 0, 1: rows p) =====
            if (warp < 2) {
                float a[16], aa[16];
                tmem_ld_16x256b_x4(tA + lane_off, a);
                if (BIDIR) tmem_ld_16x256b_x4(tAa + lane_off, aa);
                tmem_wait_ld();
                const int q4 = lane & 3;
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int p = 16 * warp + (lane >> 2) + 8 * hr;
                    const float cpp = sm.cp[p];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        float x[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int s2 = 8 * m + 2 * q4 + e;
                            const float up = BIDIR ? aa[4 * m + 2 * hr + e] : 0.f;
                            x[e] = s2 < p ? a[4 * m + 2 * hr + e] : (s2 == p ? cpp : up);
                        }
                        uint32_t x00, x01, x02, x10, x11, x12;
                        csplit3(x[0], x00, x01, x02);
                        csplit3(x[1], x10, x11, x12);
                        const uint32_t o = (uint32_t)(m * 512 + p * 16 + 4 * q4);
                        st_u32(sm.Ap[0], o, cpack(x00, x10));
                        st_u32(sm.Ap[1], o, cpack(x01, x11));
                        st_u32(sm.Ap[2], o, cpack(x02, x12));
                    }
                }
            }
        }
    } else {
        // ===== exact chunk: Gam and the local states token by token (CUDA cores) =====
        // thread (row i = tid / 2, columns 32 (tid % 2) .. + 31) of X and Xa
        const int i = tid >> 1, c0 = 32 * (tid & 1);
        float s[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) s[e] = 0.f;
        float g = 1.f;
        for (int p = 0; p < n; ++p) {
            const float dd = xr.d[p][i], kk = xr.k[p][i];
            g *= dd;
#pragma unroll
            for (int e = 0; e < 32; ++e) s[e] = fmaf(dd, s[e], kk * xr.v[p][c0 + e]);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) sm.X[i][c0 + e] = s[e];
        if ((tid & 1) == 0) sm.gam[i] = g;
        if (BIDIR) {
#pragma unroll
            for (int e = 0; e < 32; ++e) s[e] = 0.f;
            for (int p = n - 1; p >= 0; --p) {
                const float dd = xr.d[p][i], kk = xr.k[p][i];
#pragma unroll
                for (int e = 0; e < 32; ++e) s[e] = fmaf(dd, s[e], kk * xr.v[p][c0 + e]);
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) sm.Xa[i][c0 + e] = s[e];
        }
    }
    cl_barrier();   // every chunk's X, Xa and Gam are published

    // ===== fold: the states entering this chunk, thread (row i, 32 columns) =====
    {
        const int i = tid >> 1, c0 = 32 * (tid & 1);
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = 0.f;
        // causal: F <- diag(Gam_q) F + X_q for q = 0 .. j-1
        for (int q = 0; q < (int)j; ++q) {
            const float g = cl_ld1(cl_map(&sm.gam[i], q));
            const uint32_t base = cl_map(&sm.X[i][c0], q);
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
                const float4 x = cl_ld4(base + 16 * e4);
                f[4 * e4] = fmaf(g, f[4 * e4], x.x);
                f[4 * e4 + 1] = fmaf(g, f[4 * e4 + 1], x.y);
                f[4 * e4 + 2] = fmaf(g, f[4 * e4 + 2], x.z);
                f[4 * e4 + 3] = fmaf(g, f[4 * e4 + 3], x.w);
            }
        }
        if (!exact) {
            // three-term copy into the MN-major S_in tile (row i, columns c0 .. c0 + 31)
#pragma unroll
            for (int e8 = 0; e8 < 4; ++e8) {
                uint32_t t[3][8];
#pragma unroll
                for (int e = 0; e < 8; ++e) csplit3(f[8 * e8 + e], t[0][e], t[1][e], t[2][e]);
                const uint32_t o = swz(i, c0 + 8 * e8);
#pragma unroll
                for (int q = 0; q < 3; ++q)
                    st_u128(sm.Sin[q], o, make_uint4(cpack(t[q][0], t[q][1]), cpack(t[q][2], t[q][3]),
                                                     cpack(t[q][4], t[q][5]), cpack(t[q][6], t[q][7])));
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) xs.S[i][c0 + e] = f[e];
        }
        if (BIDIR) {
            // anti-causal: F <- diag(Gam_q) F + Xa_q for q = nch-1 .. j+1
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = 0.f;
            for (int q = nch - 1; q > (int)j; --q) {
                const float g = cl_ld1(cl_map(&sm.gam[i], q));
                const uint32_t base = cl_map(&sm.Xa[i][c0], q);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 x = cl_ld4(base + 16 * e4);
                    f[4 * e4] = fmaf(g, f[4 * e4], x.x);
                    f[4 * e4 + 1] = fmaf(g, f[4 * e4 + 1], x.y);
                    f[4 * e4 + 2] = fmaf(g, f[4 * e4 + 2], x.z);
                    f[4 * e4 + 3] = fmaf(g, f[4 * e4 + 3], x.w);
                }
            }
            if (!exact) {
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    uint32_t t[3][8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) csplit3(f[8 * e8 + e], t[0][e], t[1][e], t[2][e]);
                    const uint32_t o = swz(i, c0 + 8 * e8);
#pragma unroll
                    for (int q = 0; q < 3; ++q)
                        st_u128(sm.Sain[q], o, make_uint4(cpack(t[q][0], t[q][1]), cpack(t[q][2], t[q][3]),
                                                          cpack(t[q][4], t[q][5]), cpack(t[q][6], t[q][7])));
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) xs.Sa[i][c0 + e] = f[e];
            }
        }
    }
    fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    if (!exact) {
        // ===== Y = A' V + Q S_in + Qa Sa_in =====
        if (tid == 0 && ok) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int q = 0; q < kCNP; ++q)
                    mma_bf16(tY, cdadd(dAp, cprod_a(q) * kApB + 1024 * ks), cdadd(dV, cprod_b(q) * kTokB + 2048 * ks),
                             kIdAV, ks > 0 || q > 0);
            if (j > 0) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int q = 0; q < kCNP; ++q)
                        mma_bf16(tY, cdadd(dQ, cprod_a(q) * kTokB + 32 * ks), cdadd(dS, cprod_b(q) * kStB + 2048 * ks),
                                 kIdQS, true);
            }
            if (BIDIR && (int)j < nch - 1) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int q = 0; q < kCNP; ++q)
                        mma_bf16(tY, cdadd(dQa, cprod_a(q) * kTokB + 32 * ks),
                                 cdadd(dSa, cprod_b(q) * kStB + 2048 * ks), kIdQS, true);
            }
            mma_commit(&sm.bar_y);
        }
        if (ok) ok = mbar_wait_bounded(&sm.bar_y, 0);
        ok = __syncthreads_and(ok);
        fence_after_sync();
        if (ok && warp < 2 && live) {
            float yv[32];
            tmem_ld_16x256b_x8(tY + lane_off, yv);
            tmem_wait_ld();
            const int q4 = lane & 3;
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int p = 16 * warp + (lane >> 2) + 8 * hr;
                const size_t row = ((size_t)b * T + t0 + p) * C + cbase;
                if (p < n && in_range_vec(row, kHead, nBTC)) {
                    float2 *dst = reinterpret_cast<float2 *>(prm.y + row + 2 * q4);
#pragma unroll
                    for (int m = 0; m < 8; ++m) dst[4 * m] = make_float2(yv[4 * m + 2 * hr], yv[4 * m + 2 * hr + 1]);
                }
            }
        }
    } else {
        // ===== exact chunk: the sweeps token by token from the folded states (CUDA cores).
        // Thread (column jc, rows 32 hf .. 32 hf + 31); a readout's two row halves are
        // added in a fixed order, so the result is deterministic =====
        const int jc = tid & (kHead - 1), hf = tid >> 6;
        if (BIDIR) {
            // anti-causal, from the last token: y_p = r_p Sa; Sa <- diag(d_p) Sa + k_p^T v_p
            for (int p = n - 1; p >= 0; --p) {
                float part = 0.f;
#pragma unroll 8
                for (int ii = 0; ii < 32; ++ii) part = fmaf(xr.r[p][32 * hf + ii], xs.Sa[32 * hf + ii][jc], part);
                xs.red[hf][jc] = part;
                const float vj = xr.v[p][jc];
#pragma unroll 8
                for (int ii = 0; ii < 32; ++ii) {
                    const int i = 32 * hf + ii;
                    xs.Sa[i][jc] = fmaf(xr.d[p][i], xs.Sa[i][jc], xr.k[p][i] * vj);
                }
                __syncthreads();
                if (tid < kHead) xs.y[p][jc] = xs.red[0][jc] + xs.red[1][jc];
                __syncthreads();
            }
        }
        // causal: y_p += r_p (S + diag(u) k_p^T v_p); S <- diag(d_p) S + k_p^T v_p
        for (int p = 0; p < n; ++p) {
            const float vj = xr.v[p][jc];
            float part = 0.f;
#pragma unroll 8
            for (int ii = 0; ii < 32; ++ii) {
                const int i = 32 * hf + ii;
                part = fmaf(xr.r[p][i], fmaf(sm.u[i] * xr.k[p][i], vj, xs.S[i][jc]), part);
            }
            xs.red[hf][jc] = part;
#pragma unroll 8
            for (int ii = 0; ii < 32; ++ii) {
                const int i = 32 * hf + ii;
                xs.S[i][jc] = fmaf(xr.d[p][i], xs.S[i][jc], xr.k[p][i] * vj);
            }
            __syncthreads();
            if (tid < kHead) {
                const float yv = (BIDIR ? xs.y[p][jc] : 0.f) + (xs.red[0][jc] + xs.red[1][jc]);
                const size_t o = ((size_t)b * T + t0 + p) * C + cbase + jc;
                if (in_range(o, nBTC)) prm.y[o] = yv;
            }
            __syncthreads();
        }
    }
    if (!ok && tid == 0) {
        // a wait ran out: let every MMA issued so far finish before TMEM is released
        mma_commit(&sm.bar_fin);
        mbar_wait_bounded(&sm.bar_fin, 0);
    }
    // no CTA leaves (or frees its shared memory) while another may still read it
    cl_barrier();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(sm.tmem_base, 256);
}

namespace {
template <bool BIDIR>
cudaError_t launch_cluster(const float *r, const float *k, const float *v, const float *w, const FwdParams &prm,
                           cudaStream_t stream) {
    const size_t smem = sizeof(ClusterSmem) + 1024;
    auto kern = wkv6_fwd_cluster_kernel<BIDIR>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(prm.B * prm.H * kCw), kCThr, smem, stream>>>(r, k, v, w, prm);
    return cudaGetLastError();
}
}  // namespace

bool wkv6_fwd_cluster_fits(int B, int T, int H) {
    // every chunk in one cluster, and few enough (b, h) that one CTA per SM and chunk
    // beats carrying the state chunk by chunk (the chain of wkv6_fwd_split.cu)
    return T <= kCw * kCL && (long long)B * H <= kClusterMaxHeads;
}

cudaError_t wkv6_fwd_cluster_launch(bool bidir, const float *r, const float *k, const float *v, const float *w,
                                    const FwdParams &prm, cudaStream_t stream) {
    return bidir ? launch_cluster<true>(r, k, v, w, prm, stream) : launch_cluster<false>(r, k, v, w, prm, stream);
}

}  // namespace wkv
