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
//        S_in  = sum_{i<j} diag(prod_{m=i+1}^{j-1} Gam_m) X_i
//        Sa_in = sum_{i>j} diag(prod_{m=j+1}^{i-1} Gam_m) Xa_i
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
// at most this many (b, h) units, one cluster each (measured crossover with the chunk
// chain at T = 196: causal 24 units 34.8 against 36.9 us, 32 units 47.2 against 36.9 us;
// bidirectional 36 units 59.4 against 69.6 us, 48 units 75.8 against 70.6 us)
constexpr int kClusterMaxUnitsCausal = 24;
constexpr int kClusterMaxUnitsBidir = 36;
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
// Loads from another CTA's shared memory, after a cluster barrier that ordered its
// stores.  Eight 16-byte loads at addr + 2048 e (e = 0..7), issued
// back to back so that their latencies overlap: with addr = row r0 (of a 64 x 64
// fp32 state), column 4 c4, they are rows r0 + 8 e, columns 4 c4 .. 4 c4 + 3.
__device__ __forceinline__ void cl_ld_rows8(uint32_t addr, float (&x)[32]) {
    asm volatile(
        "ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%32];\n\t"
        "ld.shared::cluster.v4.f32 {%4, %5, %6, %7}, [%32 + 2048];\n\t"
        "ld.shared::cluster.v4.f32 {%8, %9, %10, %11}, [%32 + 4096];\n\t"
        "ld.shared::cluster.v4.f32 {%12, %13, %14, %15}, [%32 + 6144];\n\t"
        "ld.shared::cluster.v4.f32 {%16, %17, %18, %19}, [%32 + 8192];\n\t"
        "ld.shared::cluster.v4.f32 {%20, %21, %22, %23}, [%32 + 10240];\n\t"
        "ld.shared::cluster.v4.f32 {%24, %25, %26, %27}, [%32 + 12288];\n\t"
        "ld.shared::cluster.v4.f32 {%28, %29, %30, %31}, [%32 + 14336];"
        : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3]), "=f"(x[4]), "=f"(x[5]), "=f"(x[6]), "=f"(x[7]),
          "=f"(x[8]), "=f"(x[9]), "=f"(x[10]), "=f"(x[11]), "=f"(x[12]), "=f"(x[13]), "=f"(x[14]), "=f"(x[15]),
          "=f"(x[16]), "=f"(x[17]), "=f"(x[18]), "=f"(x[19]), "=f"(x[20]), "=f"(x[21]), "=f"(x[22]), "=f"(x[23]),
          "=f"(x[24]), "=f"(x[25]), "=f"(x[26]), "=f"(x[27]), "=f"(x[28]), "=f"(x[29]), "=f"(x[30]), "=f"(x[31])
        : "r"(addr));
}
// The decay totals of rows r0 + 8 e (e = 0..7) of another CTA, from addr = its gam[r0].
__device__ __forceinline__ void cl_ld_gam8(uint32_t addr, float (&g)[8]) {
    asm volatile(
        "ld.shared::cluster.f32 %0, [%8];\n\t"
        "ld.shared::cluster.f32 %1, [%8 + 32];\n\t"
        "ld.shared::cluster.f32 %2, [%8 + 64];\n\t"
        "ld.shared::cluster.f32 %3, [%8 + 96];\n\t"
        "ld.shared::cluster.f32 %4, [%8 + 128];\n\t"
        "ld.shared::cluster.f32 %5, [%8 + 160];\n\t"
        "ld.shared::cluster.f32 %6, [%8 + 192];\n\t"
        "ld.shared::cluster.f32 %7, [%8 + 224];"
        : "=f"(g[0]), "=f"(g[1]), "=f"(g[2]), "=f"(g[3]), "=f"(g[4]), "=f"(g[5]), "=f"(g[6]), "=f"(g[7])
        : "r"(addr));
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
    alignas(8) uint64_t bar_a, bar_a2, bar_y, bar_y2, bar_fin;
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
    ClusterSmem &sm = *reinterpret_cast<ClusterSmem *>(smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u));
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

    // ---- load the chunk first (tokens pq .. pq + 7 of this warp, channels ch, ch + 1): its
    // latency overlaps the set-up below
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
    if (tid < kHead) sm.u[tid] = prm.u[cbase + tid];
    if (tid == 0) {
        mbar_init(&sm.bar_a, 1);
        mbar_init(&sm.bar_a2, 1);
        mbar_init(&sm.bar_y, 1);
        mbar_init(&sm.bar_y2, 1);
        mbar_init(&sm.bar_fin, 2);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 256);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // TMEM (M = 64 layouts): X at 0..63, Xa at 64..127, A at 128..159, Aa at 160..191, Y at 192..255;
    // the second Y accumulator (Q S_in) reuses X's columns once X is in shared memory
    const uint32_t tX = sm.tmem_base, tXa = sm.tmem_base + 64, tA = sm.tmem_base + 128, tAa = sm.tmem_base + 160,
                   tY = sm.tmem_base + 192, tY2 = sm.tmem_base;

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
        // ===== X = Kt^T V, A = Q Kt^T (and Xa, Aa): two issuing threads (one thread issues
        // an MMA about every 47 cycles; a second issuer nearly halves the group's time).
        // Causal: thread 0 issues A, thread 32 X.  Bidirectional: thread 0 A and X, thread
        // 32 Aa and Xa =====
        if (tid == 0) {
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
                        mma_bf16(tX, cdadd(dKm, cprod_a(q) * kTokB + 2048 * ks), cdadd(dV, cprod_b(q) * kTokB + 2048 * ks),
                                 kIdX, ks > 0 || q > 0);
            }
            mma_commit(&sm.bar_a);
        } else if (tid == 32) {
            if (BIDIR) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int q = 0; q < kCNP; ++q)
                        mma_bf16(tAa, cdadd(dQa, cprod_a(q) * kTokB + 32 * ks),
                                 cdadd(dKak, cprod_b(q) * kTokB + 32 * ks), kIdA, ks > 0 || q > 0);
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                    for (int q = 0; q < kCNP; ++q)
                        mma_bf16(tXa, cdadd(dKam, cprod_a(q) * kTokB + 2048 * ks),
                                 cdadd(dV, cprod_b(q) * kTokB + 2048 * ks), kIdX, ks > 0 || q > 0);
            } else {
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                    for (int q = 0; q < kCNP; ++q)
                        mma_bf16(tX, cdadd(dKm, cprod_a(q) * kTokB + 2048 * ks), cdadd(dV, cprod_b(q) * kTokB + 2048 * ks),
                                 kIdX, ks > 0 || q > 0);
            }
            mma_commit(&sm.bar_a2);
        }
        ok = mbar_wait_bounded(&sm.bar_a, 0) && mbar_wait_bounded(&sm.bar_a2, 0);
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

    // ===== fold: the states entering this chunk,
    //   S_in  = sum_{q<j} diag(prod_{m=q+1}^{j-1} Gam_m) X_q,
    //   Sa_in = sum_{q>j} diag(prod_{m=j+1}^{q-1} Gam_m) Xa_q,
    // taken from the nearest chunk outwards with the decay product kept per row, so
    // that the CTAs' first remote reads go to different SMs.  Thread (warp w, lane l)
    // holds rows r0 + 8 e (r0 = 2 w + l / 16, e = 0..7), columns 4 (l % 16) .. + 3, so
    // that each remote load instruction of a warp reads 512 contiguous bytes (two rows;
    // no bank conflicts).  The remote reads dominate, so two chunks' states are in
    // flight per step: the next two causal predecessors, or (bidirectional) the next
    // causal predecessor and the next anti-causal successor =====
    if (live) {
        const int r0 = 2 * warp + (lane >> 4), c4 = 4 * (lane & 15);
        float fc[32], fa[32];   // [e][4]: row r0 + 8 e, columns c4 .. c4 + 3
        float pc[8], pa[8];     // decay products between the next chunk read and this one, per row
#pragma unroll
        for (int e = 0; e < 32; ++e) fc[e] = fa[e] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) pc[e] = pa[e] = 1.f;
        int qc = (int)j - 1, qa = (int)j + 1;   // next causal predecessor (down), anti-causal successor (up)
        while (qc >= 0 || (BIDIR && qa < nch)) {
            float x0[32], x1[32], g0[8], g1[8];
            // first item: a causal predecessor if one is left, else an anti-causal successor
            const bool first_c = qc >= 0;
            const int q_first = first_c ? qc : qa;
            // second item: bidirectional, the anti-causal successor (when the first was causal);
            // causal only, the next causal predecessor
            bool second = false, second_c = false;
            int q_second = 0;
            if (BIDIR) {
                if (first_c && qa < nch) {
                    second = true;
                    q_second = qa;
                }
            } else if (qc - 1 >= 0) {
                second = true;
                second_c = true;
                q_second = qc - 1;
            }
            cl_ld_rows8(cl_map(first_c ? &sm.X[r0][c4] : &sm.Xa[r0][c4], q_first), x0);
            cl_ld_gam8(cl_map(&sm.gam[r0], q_first), g0);
            if (second) {
                cl_ld_rows8(cl_map(second_c ? &sm.X[r0][c4] : &sm.Xa[r0][c4], q_second), x1);
                cl_ld_gam8(cl_map(&sm.gam[r0], q_second), g1);
            }
            // F += P X_q, then P *= Gam_q
            if (first_c) {
#pragma unroll
                for (int e = 0; e < 32; ++e) fc[e] = fmaf(pc[e >> 2], x0[e], fc[e]);
#pragma unroll
                for (int e = 0; e < 8; ++e) pc[e] *= g0[e];
                --qc;
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) fa[e] = fmaf(pa[e >> 2], x0[e], fa[e]);
#pragma unroll
                for (int e = 0; e < 8; ++e) pa[e] *= g0[e];
                ++qa;
            }
            if (second) {
                if (second_c) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) fc[e] = fmaf(pc[e >> 2], x1[e], fc[e]);
#pragma unroll
                    for (int e = 0; e < 8; ++e) pc[e] *= g1[e];
                    --qc;
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) fa[e] = fmaf(pa[e >> 2], x1[e], fa[e]);
#pragma unroll
                    for (int e = 0; e < 8; ++e) pa[e] *= g1[e];
                    ++qa;
                }
            }
        }
        if (!exact) {
            // three-term copies into the MN-major S_in tiles: 4 columns (8 bytes) per row and term
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int row = r0 + 8 * e;
                const uint32_t o = swz(row, c4);
                uint32_t t[3][4];
#pragma unroll
                for (int m = 0; m < 4; ++m) csplit3(fc[4 * e + m], t[0][m], t[1][m], t[2][m]);
#pragma unroll
                for (int q = 0; q < 3; ++q)
                    *reinterpret_cast<uint2 *>(reinterpret_cast<char *>(sm.Sin[q]) + o) =
                        make_uint2(cpack(t[q][0], t[q][1]), cpack(t[q][2], t[q][3]));
                if (BIDIR) {
#pragma unroll
                    for (int m = 0; m < 4; ++m) csplit3(fa[4 * e + m], t[0][m], t[1][m], t[2][m]);
#pragma unroll
                    for (int q = 0; q < 3; ++q)
                        *reinterpret_cast<uint2 *>(reinterpret_cast<char *>(sm.Sain[q]) + o) =
                            make_uint2(cpack(t[q][0], t[q][1]), cpack(t[q][2], t[q][3]));
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    xs.S[r0 + 8 * e][c4 + m] = fc[4 * e + m];
                    if (BIDIR) xs.Sa[r0 + 8 * e][c4 + m] = fa[4 * e + m];
                }
        }
    }
    fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    if (!exact) {
        // ===== Y = A' V + Qa Sa_in (thread 0, accumulator Y) and Q S_in (thread 32, accumulator
        // Y2 in X's columns), summed in the epilogue =====
        const bool has_s = j > 0, has_sa = BIDIR && (int)j < nch - 1;
        if (tid == 0 && ok) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int q = 0; q < kCNP; ++q)
                    mma_bf16(tY, cdadd(dAp, cprod_a(q) * kApB + 1024 * ks), cdadd(dV, cprod_b(q) * kTokB + 2048 * ks),
                             kIdAV, ks > 0 || q > 0);
            if (has_sa) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int q = 0; q < kCNP; ++q)
                        mma_bf16(tY, cdadd(dQa, cprod_a(q) * kTokB + 32 * ks),
                                 cdadd(dSa, cprod_b(q) * kStB + 2048 * ks), kIdQS, true);
            }
            mma_commit(&sm.bar_y);
        } else if (tid == 32 && ok && has_s) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                for (int q = 0; q < kCNP; ++q)
                    mma_bf16(tY2, cdadd(dQ, cprod_a(q) * kTokB + 32 * ks), cdadd(dS, cprod_b(q) * kStB + 2048 * ks),
                             kIdQS, ks > 0 || q > 0);
            mma_commit(&sm.bar_y2);
        }
        if (ok) ok = mbar_wait_bounded(&sm.bar_y, 0) && (!has_s || mbar_wait_bounded(&sm.bar_y2, 0));
        ok = __syncthreads_and(ok);
        fence_after_sync();
        if (ok && warp < 2 && live) {
            float yv[32];
            tmem_ld_16x256b_x8(tY + lane_off, yv);
            if (has_s) {
                float y2[32];
                tmem_ld_16x256b_x8(tY2 + lane_off, y2);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) yv[e] += y2[e];
            }
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
    if (!ok && (tid == 0 || tid == 32)) {
        // a wait ran out: let every MMA issued so far (by both issuing threads) finish
        // before TMEM is released
        mma_commit(&sm.bar_fin);
        if (tid == 0) mbar_wait_bounded(&sm.bar_fin, 0);
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

bool wkv6_fwd_cluster_fits(int B, int T, int H, bool bidir) {
    // every chunk in one cluster, and few enough (b, h) that one CTA per SM and chunk
    // beats carrying the state chunk by chunk (the chain of wkv6_fwd_split.cu)
    return T <= kCw * kCL && (long long)B * H <= (bidir ? kClusterMaxUnitsBidir : kClusterMaxUnitsCausal);
}

cudaError_t wkv6_fwd_cluster_launch(bool bidir, const float *r, const float *k, const float *v, const float *w,
                                    const FwdParams &prm, cudaStream_t stream) {
    return bidir ? launch_cluster<true>(r, k, v, w, prm, stream) : launch_cluster<false>(r, k, v, w, prm, stream);
}

}  // namespace wkv
