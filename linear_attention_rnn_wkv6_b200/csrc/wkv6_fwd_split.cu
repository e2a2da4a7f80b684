// wkv6_fwd_split.cu -- RWKV-6 fp32 forward (causal and bidirectional) on the
// 5th-generation tensor cores, with every operand split into three bf16 terms.
//
// Same operation as the fp32 register recurrences (wkv6_fwd_pipe.cu, wkv6_fwd.cu):
//   y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),   S_t = diag(d_t) S_{t-1} + k_t^T v_t,
// and, bidirectional ("How Custom CUDA Kernels (wkv6_cuda.cu) ...", Future-to-Past
// Pass), the same sweep run from the last token back to the first with no bonus,
// added to y.  The pages' parallel training form ("RWKV Architecture ...", The
// Parallel Training Formulation) is evaluated blockwise: a chunk of L = 32 tokens
// of one (b, h), in processing order p (time order for the causal sweep, reversed
// for the anti-causal one), with Lam_p = sum_{m<p} ew_m per channel (chunk-local),
//   Q_p = r_p exp(Lam_p),  Kt_s = k_s exp(-Lam_{s+1}),  c_p = sum_i r_p u k_p,
//   y_p   = Q_p S_in + sum_{s<p} (Q_p . Kt_s) v_s + c_p v_p      (c = 0 anti-causal)
//   S_out = diag(exp(Lam_L)) (S_in + Kt^T V).
// Four tcgen05 contractions per chunk (kind::f16, fp32 accumulators in tensor memory):
//   M1   A  = Q Kt^T          (M = 64 (p; rows 32..63 unused), N = 32 (s), K = 64 (i))
//   S    S += Kt^T V          (M = 64 (i), N = 64 (j), K = 32 (s)), issued beside M1
//   Y    Y  = A' V + Q S_in   (M = 64 (p), N = 64 (j), K = 32 (s) then 64 (i))
// with A' = strict-lower(A) + diag(c).  The state stays fp32 in tensor memory.
//
// Precision.  fp32 inputs need about 24 significant bits, bf16 carries 8: each
// operand x is written exactly as x0 + x1 + x2, three bf16 values holding its
// significand 8 bits at a time (truncation; the differences are exact in fp32),
// and a product a b is the six MMAs a0b0 + a0b1 + a1b0 + a0b2 + a1b1 + a2b0; the
// terms left out are below 2^-21 of |a b|.  (Two terms, three products, leave about 6e-6 relative
// L2 on the bidirectional workload: too close to the fp32 tolerance.)
//
// Exactness for any decay: |Lam| <= 80 keeps exp(-Lam) inside fp32 and bf16.  A
// chunk whose summed |ew| exceeds that in some channel (fast-forgetting channels,
// decay exactly 0, NaN) is evaluated by the token-by-token recurrence on the CUDA
// cores, from and back into the state in tensor memory.
//
// Fused form (wkv6_fwd_fused, "How the WKV ... Processes Images", the spatial-mix
// block): the loaded w is ww and the log-decay is -exp(w_base + ww); the last sweep
// replaces each finished y row of a head by (GroupNorm(y) * gn_w + gn_b) * g.  In
// the tensor-core epilogue a row's 64 outputs are 16 values in each of 4 lanes of
// one warp; in an exact chunk they are one value in each of threads 0..63.
//
// One CTA of 128 threads per (b, h), three CTAs per SM (70 KB of shared memory and
// 128 TMEM columns each), so the phases of one CTA (transform, MMA, mask, MMA,
// epilogue) overlap with those of the others.  Inputs are read with coalesced
// 8-byte loads into registers one chunk ahead.
#include "wkv_launch.cuh"
#include "wkv_tc.cuh"

namespace wkv {

using namespace tc;

namespace {

constexpr int kSL = 32;                  // tokens per chunk
constexpr int kNT = 3;                   // bf16 terms per operand
constexpr int kNP = 6;                   // products per contraction
constexpr int kThr = 128;
constexpr int kTokTile = kSL * kHead;    // bf16 elements of a 32 x 64 tile (4 KB)
constexpr int kApTile = kSL * kSL;       // bf16 elements of the 32 x 32 A' tile (2 KB)
constexpr int kStTile = kHead * kHead;   // bf16 elements of the 64 x 64 state tile (8 KB)
constexpr float kLog2eS = 1.4426950408889634f;
constexpr float kLamMaxS = 80.0f * kLog2eS;   // |Lam| bound of the tensor-core path, log2 units

// Products of the three-term split, as (term of the first operand, term of the second).
__device__ __forceinline__ constexpr int prod_a(int q) { return q == 2 ? 1 : q == 4 ? 1 : q == 5 ? 2 : 0; }
__device__ __forceinline__ constexpr int prod_b(int q) { return q == 1 ? 1 : q == 3 ? 2 : q == 4 ? 1 : 0; }

struct SplitSmem {
    // token tiles: 32 rows of 64 bf16, 128-byte rows, 128B-swizzled (row p / s, channel)
    __nv_bfloat16 Q[kNT][kTokTile];     // K-major A of Y += Q S_in and B of M1
    __nv_bfloat16 Kt[kNT][kTokTile];    // K-major A of M1; MN-major A of S += Kt^T V
    __nv_bfloat16 V[kNT][kTokTile];     // MN-major B of Y += A' V and S += Kt^T V
    // A' (row p, s contiguous), no swizzle: 4 units of 8 s-values x 32 rows (512 B each)
    __nv_bfloat16 Ap[kNT][kApTile];     // K-major A of Y += A' V
    __nv_bfloat16 Sin[kNT][kStTile];    // S_in (row i, j contiguous), 128B-swizzled: MN-major B
    float dec[kHead];                   // exp(Lam_L) per channel
    float cp[kSL];                      // bonus scalars per token
    float u[kHead];
    float gnw[kHead], gnb[kHead];       // fused epilogue: norm weight and bias of the head
    float red[4];                       // fused epilogue of exact chunks: two-warp sums
    uint32_t tmem_base;
    alignas(8) uint64_t bar_m1;
    alignas(8) uint64_t bar_p;
    alignas(8) uint64_t bar_s;
    alignas(8) uint64_t bar_fin;
};
static_assert(sizeof(SplitSmem) + 1024 <= 74 * 1024, "three CTAs per SM must fit");
static_assert(offsetof(SplitSmem, Q) % 1024 == 0 && offsetof(SplitSmem, Kt) % 1024 == 0 &&
                  offsetof(SplitSmem, V) % 1024 == 0 && offsetof(SplitSmem, Sin) % 1024 == 0,
              "swizzled tiles start on 1024-byte boundaries");

// Per-quarter decay sums live in the A' tiles while those are free (before M1).
struct DecaySums {
    float psum[4][kHead];
    float pabs[4][kHead];
};
static_assert(sizeof(DecaySums) <= sizeof(__nv_bfloat16) * kNT * kApTile, "decay sums fit in the A' tiles");

// Exact-chunk scratch: raw fp32 inputs in the Q, Kt, V tiles, partial sums in S_in.
constexpr int kPartStride = kHead + 4;   // floats per row of the partial-sum buffer
struct ExactRaw {
    float r[kSL][kHead], k[kSL][kHead], v[kSL][kHead], ew[kSL][kHead];
};
static_assert(sizeof(ExactRaw) <= 3 * sizeof(__nv_bfloat16) * kNT * kTokTile, "raw chunk fits in Q, Kt, V");
static_assert(sizeof(float) * kHead * kPartStride <= sizeof(__nv_bfloat16) * kNT * kStTile, "partials fit in S_in");

// x = t0 + t1 + t2 exactly, each term a bf16 value held as the high half of an fp32
// word: t0 keeps the sign, exponent and top 7 mantissa bits of x, the remainder
// x - t0 (exact) has at most 16 significant bits, its top 8 are t1 and the last 8 t2.
constexpr uint32_t kHi16 = 0xFFFF0000u;
__device__ __forceinline__ void split3(float x, uint32_t &t0, uint32_t &t1, uint32_t &t2) {
    t0 = __float_as_uint(x) & kHi16;
    const float r1 = x - __uint_as_float(t0);
    t1 = __float_as_uint(r1) & kHi16;
    t2 = __float_as_uint(r1 - __uint_as_float(t1)) & kHi16;
}
// bf16 pair (a low, b high) from two words whose low halves are zero.
__device__ __forceinline__ uint32_t pack_hi(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7632); }

// Store values a, b at (row, col), (row, col + 1) of the three term tiles.
__device__ __forceinline__ void put_pair3(__nv_bfloat16 (*tiles)[kTokTile], int row, int col, float a, float b) {
    uint32_t a0, a1, a2, b0, b1, b2;
    split3(a, a0, a1, a2);
    split3(b, b0, b1, b2);
    const uint32_t o = swz(row, col);
    st_u32(tiles[0], o, pack_hi(a0, b0));
    st_u32(tiles[1], o, pack_hi(a1, b1));
    st_u32(tiles[2], o, pack_hi(a2, b2));
}

// Eight consecutive values as three 16-byte term vectors.
__device__ __forceinline__ void split8(const float *x, uint4 &w0, uint4 &w1, uint4 &w2) {
    uint32_t a[3][8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split3(x[e], a[0][e], a[1][e], a[2][e]);
    w0 = make_uint4(pack_hi(a[0][0], a[0][1]), pack_hi(a[0][2], a[0][3]), pack_hi(a[0][4], a[0][5]),
                    pack_hi(a[0][6], a[0][7]));
    w1 = make_uint4(pack_hi(a[1][0], a[1][1]), pack_hi(a[1][2], a[1][3]), pack_hi(a[1][4], a[1][5]),
                    pack_hi(a[1][6], a[1][7]));
    w2 = make_uint4(pack_hi(a[2][0], a[2][1]), pack_hi(a[2][2], a[2][3]), pack_hi(a[2][4], a[2][5]),
                    pack_hi(a[2][6], a[2][7]));
}

// No-swizzle K-major descriptor of A' (32 rows, 16-byte units 512 B apart): k-step
// ks covers units 2 ks and 2 ks + 1.  Rows 32..63 of an M = 64 read fall on the
// next unit (or the next tile): those Y rows are never read.
__device__ __forceinline__ uint64_t desc_ap(const __nv_bfloat16 *tile, int ks) {
    return smem_desc(reinterpret_cast<const char *>(tile) + ks * 1024, 512, 128);
}

// A descriptor moved by `bytes` (a multiple of 16): the start address is the low field.
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity) {
    return mbar_wait_bounded(bar, parity);
}

// Barrier of warps 0 and 1 only (id 1; id 0 is __syncthreads).
__device__ __forceinline__ void sync_warps01() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace

template <bool BIDIR, bool FUSED>
__global__ void __launch_bounds__(kThr, 3) wkv6_fwd_split_kernel(const float *__restrict__ r,
                                                                 const float *__restrict__ k,
                                                                 const float *__restrict__ v,
                                                                 const float *__restrict__ w, FwdParams prm) {
    extern __shared__ unsigned char smem_dyn[];
    SplitSmem &sm = *reinterpret_cast<SplitSmem *>(smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u));
    DecaySums &ds = *reinterpret_cast<DecaySums *>(&sm.Ap[0][0]);
    ExactRaw &xr = *reinterpret_cast<ExactRaw *>(&sm.Q[0][0]);
    float *part = reinterpret_cast<float *>(&sm.Sin[0][0]);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = prm.T, C = prm.C, H = prm.H;
    const int h = blockIdx.x % H, b = blockIdx.x / H;
    const int cbase = h * kHead;
    const int nch = (T + kSL - 1) / kSL;
    const int ch = 2 * lane;          // transform: channels ch, ch + 1
    const int pq = 8 * warp;          // transform: tokens pq .. pq + 7 of the chunk
    const bool row_lane = lane < 16;  // 32x32b TMEM accesses: lanes 0..15 of each quarter hold M = 64 rows
    const int trow = 16 * warp + (lane & 15);   // exact chunks: state row i
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

    if (tid < kHead) sm.u[tid] = prm.u[cbase + tid];
    if (FUSED && tid < kHead) {
        sm.gnw[tid] = prm.gn_w[cbase + tid];
        sm.gnb[tid] = prm.gn_b[cbase + tid];
    }
    const float2 wb = FUSED ? __ldg(reinterpret_cast<const float2 *>(prm.wb + cbase + ch)) : make_float2(0.f, 0.f);
    if (tid == 0) {
        mbar_init(&sm.bar_m1, 1);
        mbar_init(&sm.bar_p, 1);
        mbar_init(&sm.bar_s, 1);
        mbar_init(&sm.bar_fin, 2);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 128);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // TMEM: A (32 columns) and Y (64) share columns 0..63, S at 64..127 (M = 64 layouts)
    const uint32_t tY = sm.tmem_base, tS = sm.tmem_base + 64;

    // base descriptors; every MMA below adds a compile-time offset (term tile, k-step)
    constexpr uint32_t kTokB = kTokTile * 2, kApB = kApTile * 2, kStB = kStTile * 2;   // tile bytes
    const uint64_t dQ = desc_k(sm.Q[0], 0), dKk = desc_k(sm.Kt[0], 0), dKm = desc_mn(sm.Kt[0], 0, 16);
    const uint64_t dV = desc_mn(sm.V[0], 0, 16), dA = desc_ap(sm.Ap[0], 0), dS = desc_mn(sm.Sin[0], 0, 16);
    constexpr uint32_t kIdM1 = idesc_bf16(64, 32, false, false);
    constexpr uint32_t kIdAV = idesc_bf16(64, 64, false, true);
    constexpr uint32_t kIdQS = idesc_bf16(64, 64, false, true);
    constexpr uint32_t kIdS = idesc_bf16(64, 64, true, true);

    // ---- register prefetch of one chunk: tokens pq..pq+7, channels ch, ch+1
    float2 xr_[8], xk_[8], xv_[8], xw_[8];
    // RWKV-5 (wkv5_fwd): the static log-decay -w5 of channels ch, ch + 1 at every token
    // of [0, T); the w argument is then the [C] array w5 and is not read per token
    const bool stat = !FUSED && prm.w5 != nullptr;
    const float2 w5ew = stat ? make_float2(-__ldg(prm.w5 + cbase + ch), -__ldg(prm.w5 + cbase + ch + 1))
                             : make_float2(0.f, 0.f);
    auto time_of = [&](int dir, int c, int p) { return dir > 0 ? c * kSL + p : T - 1 - (c * kSL + p); };
    auto load_chunk = [&](int dir, int c) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int p = pq + e;
            if (c * kSL + p < T) {
                const size_t o = ((size_t)b * T + time_of(dir, c, p)) * C + cbase + ch;
                xr_[e] = __ldg(reinterpret_cast<const float2 *>(r + o));
                xk_[e] = __ldg(reinterpret_cast<const float2 *>(k + o));
                xv_[e] = __ldg(reinterpret_cast<const float2 *>(v + o));
                xw_[e] = stat ? w5ew : __ldg(reinterpret_cast<const float2 *>(w + o));
            } else {
                xr_[e] = xk_[e] = xv_[e] = xw_[e] = make_float2(0.f, 0.f);
            }
        }
    };

    uint32_t ph_m1 = 0, ph_p = 0;
    bool ok = true;
    constexpr int ndir = BIDIR ? 2 : 1;
    const bool has_s0 = !BIDIR && !FUSED && prm.s0 != nullptr;   // wkv6_fwd_state
    load_chunk(BIDIR ? -1 : 1, 0);

    for (int di = 0; di < ndir && ok; ++di) {
        const int dir = (BIDIR && di == 0) ? -1 : 1;   // bidirectional: anti-causal sweep first
        const bool bonus = dir > 0;
        const bool accumulate_y = BIDIR && di == 1;    // the causal sweep adds to y
        const bool norm = FUSED && (!BIDIR || di == 1);  // the last sweep: norm/gate epilogue
        // S = 0 at the start of every sweep, or (causal, wkv6_fwd_state) the initial state:
        // lanes 0..15 of every warp own row i = trow; S_in's three-term copy as the epilogue
        // writes it
        if (has_s0) {
            float srow[64];
            const float *src = prm.s0 + ((size_t)b * H + h) * kHead * kHead + (size_t)trow * kHead;
#pragma unroll
            for (int g = 0; g < 16; ++g) {
                const float4 x4 = row_lane ? __ldg(reinterpret_cast<const float4 *>(src) + g)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
                srow[4 * g] = x4.x;
                srow[4 * g + 1] = x4.y;
                srow[4 * g + 2] = x4.z;
                srow[4 * g + 3] = x4.w;
            }
            float t32[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int e = 0; e < 32; ++e) t32[e] = srow[32 * half + e];
                tmem_st32(tS + lane_off + 32 * half, t32);
            }
            tmem_wait_st();
            if (row_lane) {
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    uint4 w0, w1, w2;
                    split8(srow + 8 * g, w0, w1, w2);
                    const uint32_t o = swz(trow, 8 * g);
                    st_u128(sm.Sin[0], o, w0);
                    st_u128(sm.Sin[1], o, w1);
                    st_u128(sm.Sin[2], o, w2);
                }
            }
        } else {
            float z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0.f;
            tmem_st32(tS + lane_off, z);
            tmem_st32(tS + lane_off + 32, z);
            tmem_wait_st();
        }
        for (int c = 0; c < nch; ++c) {
            // ================= transform =================
            if (FUSED) {
                // decay prologue, here rather than at the load so that the load stays in flight
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (c * kSL + pq + e < T)
                        xw_[e] = make_float2(-expf(wb.x + xw_[e].x), -expf(wb.y + xw_[e].y));
            }
            float s0 = 0.f, s1 = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                s0 += xw_[e].x * kLog2eS;
                s1 += xw_[e].y * kLog2eS;
                a0 += fabsf(xw_[e].x * kLog2eS);
                a1 += fabsf(xw_[e].y * kLog2eS);
            }
            *reinterpret_cast<float2 *>(&ds.psum[warp][ch]) = make_float2(s0, s1);
            *reinterpret_cast<float2 *>(&ds.pabs[warp][ch]) = make_float2(a0, a1);
            __syncthreads();
            float L0 = 0.f, L1 = 0.f, tot0 = 0.f, tot1 = 0.f, ab0 = 0.f, ab1 = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 ps = *reinterpret_cast<const float2 *>(&ds.psum[q][ch]);
                const float2 pa = *reinterpret_cast<const float2 *>(&ds.pabs[q][ch]);
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
            const bool exact = __any_sync(0xffffffffu, !(ab0 <= kLamMaxS) || !(ab1 <= kLamMaxS));
            const float u0 = sm.u[ch], u1 = sm.u[ch + 1];
            float bp[8];
            if (!exact) {
                if (warp == 0) *reinterpret_cast<float2 *>(&sm.dec[ch]) = make_float2(exp2f(tot0), exp2f(tot1));
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int p = pq + e;
                    const float2 rr = xr_[e], kk = xk_[e], vv = xv_[e];
                    bp[e] = bonus ? fmaf(rr.x * u0, kk.x, rr.y * u1 * kk.y) : 0.f;
                    const float q0 = rr.x * fast_exp2(L0), q1 = rr.y * fast_exp2(L1);
                    L0 += xw_[e].x * kLog2eS;
                    L1 += xw_[e].y * kLog2eS;
                    put_pair3(sm.Q, p, ch, q0, q1);
                    put_pair3(sm.Kt, p, ch, kk.x * fast_exp2(-L0), kk.y * fast_exp2(-L1));
                    put_pair3(sm.V, p, ch, vv.x, vv.y);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int p = pq + e;
                    const float2 rr = xr_[e], kk = xk_[e];
                    bp[e] = bonus ? fmaf(rr.x * u0, kk.x, rr.y * u1 * kk.y) : 0.f;
                    *reinterpret_cast<float2 *>(&xr.r[p][ch]) = rr;
                    *reinterpret_cast<float2 *>(&xr.k[p][ch]) = kk;
                    *reinterpret_cast<float2 *>(&xr.v[p][ch]) = xv_[e];
                    *reinterpret_cast<float2 *>(&xr.ew[p][ch]) = xw_[e];
                }
            }
            {
                const float cpv = transpose_reduce8(bp, lane);
                if ((lane & 3) == 0) sm.cp[pq + (lane >> 2)] = cpv;
            }
            // the registers are free: start the loads of the next chunk (or of the next sweep)
            if (c + 1 < nch) load_chunk(dir, c + 1);
            else if (BIDIR && di == 0) load_chunk(1, 0);
            fence_proxy_async_smem();
            fence_before_sync();
            __syncthreads();
            fence_after_sync();

            if (!exact) {
                // ===== M1: A = Q Kt^T (warp 0), and S += Kt^T V (warp 1): two issuing threads =====
                if (tid == 0) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                        for (int q = 0; q < kNP; ++q)
                            mma_bf16(tY, dadd(dQ, prod_a(q) * kTokB + 32 * ks), dadd(dKk, prod_b(q) * kTokB + 32 * ks),
                                     kIdM1, ks > 0 || q > 0);
                    mma_commit(&sm.bar_m1);
                } else if (tid == 32) {
                    // S (rescaled by the previous epilogue, or zero) += Kt^T V
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                        for (int q = 0; q < kNP; ++q)
                            mma_bf16(tS, dadd(dKm, prod_a(q) * kTokB + 2048 * ks), dadd(dV, prod_b(q) * kTokB + 2048 * ks),
                                     kIdS, true);
                    mma_commit(&sm.bar_s);
                }
                ok = wait_bar(&sm.bar_m1, ph_m1);
                ph_m1 ^= 1u;
                ok = __syncthreads_and(ok);
                if (!ok) break;
                fence_after_sync();
                // ================= mask: A' = strict-lower(A) + diag(c) =================
                // rows p = 16 warp + (lane / 4) and that + 8 (warps 0, 1); columns s = 8 m + 2 (lane % 4) + {0, 1}
                if (warp < 2) {
                    float a[16];
                    tmem_ld_16x256b_x4(tY + lane_off, a);
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
                                const float av = a[4 * m + 2 * hr + e];
                                x[e] = s2 < p ? av : (s2 == p ? cpp : 0.f);
                            }
                            uint32_t x00, x01, x02, x10, x11, x12;
                            split3(x[0], x00, x01, x02);
                            split3(x[1], x10, x11, x12);
                            const uint32_t o = (uint32_t)(m * 512 + p * 16 + 4 * q4);
                            st_u32(sm.Ap[0], o, pack_hi(x00, x10));
                            st_u32(sm.Ap[1], o, pack_hi(x01, x11));
                            st_u32(sm.Ap[2], o, pack_hi(x02, x12));
                        }
                    }
                }
                fence_proxy_async_smem();
                fence_before_sync();
                __syncthreads();
                fence_after_sync();
                // ================= Y = A' V + Q S_in =================
                if (tid == 0) {
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                        for (int q = 0; q < kNP; ++q)
                            mma_bf16(tY, dadd(dA, prod_a(q) * kApB + 1024 * ks), dadd(dV, prod_b(q) * kTokB + 2048 * ks),
                                     kIdAV, ks > 0 || q > 0);
                    if (c > 0 || has_s0) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                            for (int q = 0; q < kNP; ++q)
                                mma_bf16(tY, dadd(dQ, prod_a(q) * kTokB + 32 * ks),
                                         dadd(dS, prod_b(q) * kStB + 2048 * ks), kIdQS, true);
                    }
                    mma_commit(&sm.bar_p);
                }
                // fused: the gate values of this chunk's rows are loaded while Y is computed
                float2 gate[2][8];
                if (norm && warp < 2) {
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int p = 16 * warp + (lane >> 2) + 8 * hr;
                        const bool vd = c * kSL + p < T;
                        const float2 *gs = reinterpret_cast<const float2 *>(
                            prm.g + ((size_t)b * T + (vd ? time_of(dir, c, p) : 0)) * C + cbase + 2 * (lane & 3));
#pragma unroll
                        for (int m = 0; m < 8; ++m) gate[hr][m] = vd ? __ldg(gs + 4 * m) : make_float2(0.f, 0.f);
                    }
                }
                ok = wait_bar(&sm.bar_p, ph_p) && wait_bar(&sm.bar_s, ph_p);
                ph_p ^= 1u;
                ok = __syncthreads_and(ok);
                if (!ok) break;
                fence_after_sync();
                // ================= epilogue =================
                // fragment rows r0 = 16 warp + (lane / 4) and r0 + 8; columns 8 m + 2 (lane % 4) + {0, 1}
                const int q4 = lane & 3;
                if (warp < 2) {
                    // y rows p: the anti-causal part is loaded first, all loads before any store
                    float2 prev[2][8];
                    float2 *dst[2];
                    bool valid[2];
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int p = 16 * warp + (lane >> 2) + 8 * hr;
                        valid[hr] = c * kSL + p < T &&   // the head's 64 channels of the token
                                    in_range_vec(((size_t)b * T + time_of(dir, c, p)) * C + cbase, kHead,
                                                 (size_t)prm.B * T * C);
                        dst[hr] = reinterpret_cast<float2 *>(
                            prm.y + ((size_t)b * T + (valid[hr] ? time_of(dir, c, p) : 0)) * C + cbase + 2 * q4);
#pragma unroll
                        for (int m = 0; m < 8; ++m)
                            prev[hr][m] = (accumulate_y && valid[hr]) ? dst[hr][4 * m] : make_float2(0.f, 0.f);
                    }
                    float yv[32];
                    tmem_ld_16x256b_x8(tY + lane_off, yv);
                    tmem_wait_ld();
                    if (norm) {
                        // a row's 64 outputs: 16 here, the rest in the lanes differing in bits 0, 1
#pragma unroll
                        for (int hr = 0; hr < 2; ++hr) {
                            float yr[16];
                            float s1 = 0.f;
#pragma unroll
                            for (int m = 0; m < 8; ++m) {
                                yr[2 * m] = yv[4 * m + 2 * hr] + prev[hr][m].x;
                                yr[2 * m + 1] = yv[4 * m + 2 * hr + 1] + prev[hr][m].y;
                                s1 += yr[2 * m] + yr[2 * m + 1];
                            }
                            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
                            s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
                            const float mu = s1 * (1.f / kHead);
                            float s2 = 0.f;
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                yr[e] -= mu;
                                s2 = fmaf(yr[e], yr[e], s2);
                            }
                            s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
                            s2 += __shfl_xor_sync(0xffffffffu, s2, 2);
                            const float rstd = rsqrtf(s2 * (1.f / kHead) + prm.gn_eps);
                            if (valid[hr]) {
#pragma unroll
                                for (int m = 0; m < 8; ++m) {
                                    const int j = 8 * m + 2 * q4;
                                    dst[hr][4 * m] =
                                        make_float2(fmaf(yr[2 * m] * rstd, sm.gnw[j], sm.gnb[j]) * gate[hr][m].x,
                                                    fmaf(yr[2 * m + 1] * rstd, sm.gnw[j + 1], sm.gnb[j + 1]) *
                                                        gate[hr][m].y);
                                }
                            }
                        }
                    } else {
#pragma unroll
                        for (int hr = 0; hr < 2; ++hr)
                            if (valid[hr]) {
#pragma unroll
                                for (int m = 0; m < 8; ++m)
                                    dst[hr][4 * m] = make_float2(yv[4 * m + 2 * hr] + prev[hr][m].x,
                                                                 yv[4 * m + 2 * hr + 1] + prev[hr][m].y);
                            }
                    }
                }
                {
                    // S rows i scaled by exp(Lam_L[i]), back to TMEM, three-term copy into S_in
                    float sv[32];
                    tmem_ld_16x256b_x8(tS + lane_off, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        const int i = 16 * warp + (lane >> 2) + 8 * hr;
                        const float dsc = sm.dec[i];
#pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            const float s0 = sv[4 * m + 2 * hr] * dsc, s1 = sv[4 * m + 2 * hr + 1] * dsc;
                            sv[4 * m + 2 * hr] = s0;
                            sv[4 * m + 2 * hr + 1] = s1;
                            uint32_t x00, x01, x02, x10, x11, x12;
                            split3(s0, x00, x01, x02);
                            split3(s1, x10, x11, x12);
                            const uint32_t o = swz(i, 8 * m + 2 * q4);
                            st_u32(sm.Sin[0], o, pack_hi(x00, x10));
                            st_u32(sm.Sin[1], o, pack_hi(x01, x11));
                            st_u32(sm.Sin[2], o, pack_hi(x02, x12));
                        }
                    }
                    tmem_st_16x256b_x8(tS + lane_off, sv);
                    tmem_wait_st();
                }
            } else {
                // ================= exact chunk: token-by-token recurrence =================
                // lanes 0..15 of every warp own state row i = trow (64 values in registers)
                const int i = trow;
                float srow[64];
                {
                    float t32[32];
                    tmem_ld32(tS + lane_off, t32);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) srow[e] = t32[e];
                    tmem_ld32(tS + lane_off + 32, t32);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) srow[32 + e] = t32[e];
                }
                for (int p = 0; p < kSL; ++p) {
                    if (c * kSL + p >= T) break;   // uniform
                    if (row_lane) {
                        const float rr = xr.r[p][i];
#pragma unroll
                        for (int g = 0; g < 16; ++g)
                            *reinterpret_cast<float4 *>(&part[i * kPartStride + 4 * g]) =
                                make_float4(rr * srow[4 * g], rr * srow[4 * g + 1], rr * srow[4 * g + 2],
                                            rr * srow[4 * g + 3]);
                    }
                    __syncthreads();
                    if (tid < kHead) {
                        const int j = tid;
                        float acc = sm.cp[p] * xr.v[p][j];
                        for (int ii = 0; ii < kHead; ++ii) acc += part[ii * kPartStride + j];
                        const size_t o = ((size_t)b * T + time_of(dir, c, p)) * C + cbase + j;
                        float *dst = prm.y + o;
                        const bool ok = in_range(o, (size_t)prm.B * T * C);
                        float yo = (accumulate_y && ok) ? *dst + acc : acc;
                        if (norm) {
                            // the token's 64 outputs are one per thread of warps 0 and 1
                            const float gt = ok ? __ldg(prm.g + o) : 0.f;
                            float s1 = warp_sum(yo);
                            if (lane == 0) sm.red[warp] = s1;
                            sync_warps01();
                            const float mu = (sm.red[0] + sm.red[1]) * (1.f / kHead);
                            const float d = yo - mu;
                            const float s2 = warp_sum(d * d);
                            if (lane == 0) sm.red[2 + warp] = s2;
                            sync_warps01();
                            const float rstd = rsqrtf((sm.red[2] + sm.red[3]) * (1.f / kHead) + prm.gn_eps);
                            yo = fmaf(d * rstd, sm.gnw[j], sm.gnb[j]) * gt;
                        }
                        if (ok) *dst = yo;
                    }
                    if (row_lane) {
                        const float dd = __expf(xr.ew[p][i]), kk = xr.k[p][i];
#pragma unroll
                        for (int j = 0; j < kHead; ++j) srow[j] = fmaf(dd, srow[j], kk * xr.v[p][j]);
                    }
                    __syncthreads();
                }
                {
                    float t32[32];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) t32[e] = srow[32 * half + e];
                        tmem_st32(tS + lane_off + 32 * half, t32);
                    }
                    tmem_wait_st();
                }
                if (row_lane) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        uint4 w0, w1, w2;
                        split8(srow + 8 * g, w0, w1, w2);
                        const uint32_t o = swz(i, 8 * g);
                        st_u128(sm.Sin[0], o, w0);
                        st_u128(sm.Sin[1], o, w1);
                        st_u128(sm.Sin[2], o, w2);
                    }
                }
            }
            fence_proxy_async_smem();
            fence_before_sync();
            __syncthreads();
            fence_after_sync();
        }
    }
    if (ok && !BIDIR && !FUSED && prm.sT != nullptr) {
        // wkv6_fwd_state: every chunk's epilogue left S_out = diag(exp(Lam_L)) (S_in + Kt^T V)
        // in TMEM, and tokens past T were zero (k = v = 0, log-decay 0): the state S_{T-1}
        const size_t nstate = (size_t)prm.B * H * kHead * kHead;
        float *dst = prm.sT + ((size_t)b * H + h) * kHead * kHead + (size_t)trow * kHead;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float t32[32];
            tmem_ld32(tS + lane_off + 32 * half, t32);
            tmem_wait_ld();
            if (row_lane) {
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const size_t o = ((size_t)b * H + h) * kHead * kHead + (size_t)trow * kHead + 32 * half + 4 * g;
                    if (in_range_vec(o, 4, nstate))
                        *reinterpret_cast<float4 *>(dst + 32 * half + 4 * g) =
                            make_float4(t32[4 * g], t32[4 * g + 1], t32[4 * g + 2], t32[4 * g + 3]);
                }
            }
        }
    }
    if (!ok && (tid == 0 || tid == 32)) {
        // a wait ran out: let every MMA issued so far (by both issuing threads) finish
        // before TMEM is released
        mma_commit(&sm.bar_fin);
        if (tid == 0) mbar_wait_bounded(&sm.bar_fin, 0);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(sm.tmem_base, 128);
}

cudaError_t wkv6_fwd_split_launch(bool bidir, const float *r, const float *k, const float *v, const float *w,
                                  const FwdParams &prm, cudaStream_t stream) {
    const size_t smem = sizeof(SplitSmem) + 1024;
    const bool fused = prm.gn_w != nullptr;
    auto kern = bidir ? (fused ? wkv6_fwd_split_kernel<true, true> : wkv6_fwd_split_kernel<true, false>)
                      : (fused ? wkv6_fwd_split_kernel<false, true> : wkv6_fwd_split_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(prm.B * prm.H), kThr, smem, stream>>>(r, k, v, w, prm);
    return cudaGetLastError();
}

}  // namespace wkv
