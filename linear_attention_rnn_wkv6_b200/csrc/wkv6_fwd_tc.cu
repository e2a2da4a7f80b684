// wkv6_fwd_tc.cu -- chunked RWKV-6 causal forward on the 5th-generation tensor cores.
//
// Same operation as wkv6_fwd.cu (bf16 r, k, v, w; fp32 u, state and y):
//   y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),   S_t = diag(d_t) S_{t-1} + k_t^T v_t.
// The pages' parallel training form ("RWKV Architecture ...", The Parallel
// Training Formulation) evaluates the decayed sums blockwise instead of token
// by token; here a chunk of L = 64 tokens of one (b, h) is three dense
// 64 x 64 x 64 contractions on tcgen05 (kind::tf32, fp32 accumulators in TMEM).
//
// Chunk algebra.  With Lam_p = sum_{m<p} ew_m (per row i, exclusive, chunk-local),
// Q_p = r_p * exp(Lam_p), Kt_s = k_s * exp(-Lam_{s+1}) and c_p = sum_i r_p u k_p:
//   y_p   = Q_p S_in + sum_{s<p} (Q_p . Kt_s) v_s + c_p v_p
//   S_out = diag(exp(Lam_L)) (S_in + Kt^T V)
//   M1  A  = Q Kt^T                                  (TMEM cols [0,64))
//   M2  Y  = Q S_in + A' V,  A' = strict-lower(A) + diag(c)   (TMEM cols [64,128))
//   M3  S += Kt^T V, then rows scaled by exp(Lam_L)  (TMEM cols [128,192))
// All operands are K-major (TF32 operands in MN-major form give no result on
// this hardware), staged in the 128-byte-swizzled canonical layout so both
// row-wise and column-wise shared-memory writes are bank-conflict free; Kt is
// kept in two orientations and V and S_in are stored transposed.
// |Lam| <= 80 keeps exp(-Lam) inside fp32.  A chunk whose cumulative decay
// leaves that range (fast-forgetting channels) is evaluated instead by the
// exact token-by-token recurrence on the CUDA cores, starting from the state
// held in TMEM, so any decay down to exactly 0 stays exact.
//
// Warp roles (one CTA per (b, h), 13 warps):
//   warp 0      TMA loads (2-stage ring) and, from one thread, all MMAs
//   warps 1..8  transform: chunk operands for the MMAs, then the masked A'
//   warps 9..12 epilogue: y out of TMEM, state rescale and its transposed copy
// Operand sets are double buffered, so the transform of chunk c+1 overlaps the
// MMAs and epilogue of chunk c.  Hand-offs are mbarriers; every wait is bounded
// and a shared abort flag stops all roles after the first timeout.
#include "wkv_launch.cuh"
#include "wkv_tc.cuh"

namespace wkv {

namespace {

constexpr int kL = 64;                 // tokens per chunk
constexpr float kLamMax = 80.0f;       // |Lam| bound of the tensor-core path
constexpr int kTW = 8;                 // transform warps
constexpr int kEW = 4;                 // epilogue warps
constexpr int kThreads = 32 * (1 + kTW + kEW);
constexpr int kTT = 32 * kTW;          // transform threads
constexpr int kET = 32 * kEW;          // epilogue threads

struct Tc2Smem {
    __nv_bfloat16 raw[2][4][kL][kHead];   // r, k, v, w stages (TMA, 128B-swizzled), 64 KB
    float Q[2][kL * kHead];               // (row p, k = i)            A of M1, M2
    float K[2][kL * kHead];               // (row s, k = i), B of M1; then A' (row p, k = s), A of M2
    float KT[2][kHead * kL];              // (row i, k = s)            A of M3
    float VT[2][kHead * kL];              // (row j, k = s)            B of M2, M3
    float ST[kHead * kHead];              // S_in^T (row j, k = i)     B of M2
    float dec[4][kHead];                  // exp(Lam_L) per row (ring of 4 chunks)
    float cp[2][kL];                      // bonus scalars per token
    float part_sum[kTW][kHead];           // per-octet log2-decay sums (prefix exchange)
    float u[kHead];
    int flag[4];                          // chunk c is flagged iff flag[c & 3] == c + 1
    int abort_;
    uint32_t tmem_base;
    alignas(8) uint64_t full[2];
    alignas(8) uint64_t t_done, m1_done, a_done, mma_done, s_ready;
    alignas(8) uint64_t set_free[2];
    alignas(8) uint64_t final_bar;
};

enum { R_ = 0, K_ = 1, V_ = 2, W_ = 3 };

__device__ __forceinline__ float raw_at(const __nv_bfloat16 (&t)[kL][kHead], int row, int col) {
    const int chunk = (col >> 3) ^ (row & 7);
    return __bfloat162float(t[row][chunk * 8 + (col & 7)]);
}

// Float index of element (row r, k) of a 64 x 64 tf32 K-major tile in the
// 128-byte-swizzled canonical layout: two K-blocks of [64 rows][32 floats],
// 16-byte chunk c of row r stored at chunk c ^ (r & 7).
__device__ __forceinline__ int swz(int r, int k) {
    return (k >> 5) * 2048 + r * 32 + ((((k & 31) >> 2) ^ (r & 7)) << 2) + (k & 3);
}

// Descriptor of the kstep-th group of 8 K values of such a tile.
__device__ __forceinline__ uint64_t desc_sw(const float *tile, int kstep) {
    const char *p = reinterpret_cast<const char *>(tile) + (kstep >> 2) * 8192 + (kstep & 3) * 32;
    return tc::smem_desc(p, 16, 1024) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait that gives up at once when another thread has already aborted.
__device__ __forceinline__ bool wait_or_abort(Tc2Smem &sm, uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*(volatile int *)&sm.abort_) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_wkv_faults, WKV_FAULT_TIMEOUT);
            *(volatile int *)&sm.abort_ = 1;
            return false;
        }
        __nanosleep(64);
    }
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
wkv6_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_r, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_w,
                   FwdParams prm) {
    extern __shared__ unsigned char smem_dyn[];
    Tc2Smem &sm = *reinterpret_cast<Tc2Smem *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = prm.T, C = prm.C, H = prm.H;
    const int h = blockIdx.x % H, b = blockIdx.x / H;
    const int cbase = h * kHead;
    const int nch = (T + kL - 1) / kL;
    constexpr uint32_t kStageBytes = 4u * kL * kHead * sizeof(__nv_bfloat16);

    if (tid < kHead) sm.u[tid] = prm.u[cbase + tid];
    if (tid < 4) sm.flag[tid] = 0;
    if (tid == 0) {
        sm.abort_ = 0;
        prefetch_tensormap(&map_r);
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
        prefetch_tensormap(&map_w);
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        mbar_init(&sm.t_done, kTT);
        mbar_init(&sm.m1_done, 1);
        mbar_init(&sm.a_done, kTT);
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.s_ready, kET);
        mbar_init(&sm.set_free[0], 1);
        mbar_init(&sm.set_free[1], 1);
        mbar_init(&sm.final_bar, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem_base, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.tmem_base;
    const uint32_t tA = tbase, tY = tbase + 64, tS = tbase + 128;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's TMEM lane quarter
    const int qrow = 16 * (warp & 3) + lane;                          // accumulator row (lane < 16)
    const bool rowlane = lane < 16;

    auto issue = [&](int c) {
        const int s = c & 1;
        mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
        tma_load_3d(&sm.raw[s][R_][0][0], &map_r, cbase, c * kL, b, &sm.full[s]);
        tma_load_3d(&sm.raw[s][K_][0][0], &map_k, cbase, c * kL, b, &sm.full[s]);
        tma_load_3d(&sm.raw[s][V_][0][0], &map_v, cbase, c * kL, b, &sm.full[s]);
        tma_load_3d(&sm.raw[s][W_][0][0], &map_w, cbase, c * kL, b, &sm.full[s]);
    };

    if (warp == 0) {
        // ===================== TMA + MMA issue (one thread) =====================
        if (lane == 0) {
            constexpr uint32_t kId = tc::idesc_tf32(64, 64, false, false);
            int issued = 0;
            issue(0);
            ++issued;
            if (nch > 1) {
                issue(1);
                ++issued;
            }
            uint32_t ph_t = 0, ph_a = 0;
            int s_seen = 0;   // s_ready phases observed
            bool ok = true;
            for (int c = 0; c < nch && ok; ++c) {
                const int set = c & 1;
                ok = wait_or_abort(sm, &sm.t_done, ph_t);
                ph_t ^= 1;
                if (!ok) break;
                tc::fence_after_sync();
                const bool flagged = *(volatile int *)&sm.flag[c & 3] == c + 1;
                if (!flagged) {
                    if (c + 2 < nch) {
                        fence_proxy_async_smem();
                        issue(c + 2);
                        ++issued;
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        tc::mma_tf32(tA, desc_sw(sm.Q[set], k), desc_sw(sm.K[set], k), kId, k > 0);
                    tc::mma_commit(&sm.m1_done);
                    ok = wait_or_abort(sm, &sm.a_done, ph_a);
                    ph_a ^= 1;
                    while (ok && s_seen <= c - 1) {
                        ok = wait_or_abort(sm, &sm.s_ready, s_seen & 1);
                        ++s_seen;
                    }
                    if (!ok) break;
                    tc::fence_after_sync();
                    if (c > 0) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            tc::mma_tf32(tY, desc_sw(sm.Q[set], k), desc_sw(sm.ST, k), kId, k > 0);
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        tc::mma_tf32(tY, desc_sw(sm.K[set], k), desc_sw(sm.VT[set], k), kId, c > 0 || k > 0);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        tc::mma_tf32(tS, desc_sw(sm.KT[set], k), desc_sw(sm.VT[set], k), kId, c > 0 || k > 0);
                    tc::mma_commit(&sm.mma_done);
                    tc::mma_commit(&sm.set_free[set]);
                } else {
                    // the transform warps evaluate this chunk exactly; they read the
                    // raw stage until they publish the chunk's state
                    while (ok && s_seen <= c) {
                        ok = wait_or_abort(sm, &sm.s_ready, s_seen & 1);
                        ++s_seen;
                    }
                    if (!ok) break;
                    if (c + 2 < nch) {
                        fence_proxy_async_smem();
                        issue(c + 2);
                        ++issued;
                    }
                    mbar_arrive(&sm.mma_done);
                    mbar_arrive(&sm.set_free[set]);
                }
            }
            // every MMA issued so far must finish before TMEM is released
            tc::mma_commit(&sm.final_bar);
            mbar_wait_bounded(&sm.final_bar, 0);
            if (!ok) {
                // let copies still in flight land before the CTA exits (bounded)
                for (int cc = max(0, issued - 2); cc < issued; ++cc)
                    mbar_wait_bounded(&sm.full[cc & 1], (cc >> 1) & 1);
            }
        }
    } else if (warp <= kTW) {
        // ===================== transform warps =====================
        // warp tw handles tokens [8 tw, 8 tw + 8) of the chunk; lane handles
        // channels (2 lane, 2 lane + 1): bf16x2 loads, 8-byte Q / Kt stores and
        // 16-byte stores of the transposed tiles, 8 independent tokens per thread.
        const int t = tid - 32;               // 0 .. kTT-1
        const int tw = warp - 1;              // transform warp index = token octet
        const int ch = 2 * lane;              // first of this thread's two channels
        const int p0 = 8 * tw;
        const uint32_t raw_off = (uint32_t)(((lane & 3) << 2));   // byte offset inside the 16-byte chunk
        const float u0 = sm.u[ch], u1 = sm.u[ch + 1];
        uint32_t ph_m1 = 0;
        for (int c = 0; c < nch; ++c) {
            const int set = c & 1, stg = c & 1;
            const int t0 = c * kL;
            // waits never make these threads leave early on their own: a timeout sets
            // the shared abort flag, and all transform threads leave together at the
            // first named barrier below, so none is left waiting at a barrier
            bool ok = true;
            if (c >= 2) ok = wait_or_abort(sm, &sm.set_free[set], ((c - 2) >> 1) & 1);
            if (ok) ok = wait_or_abort(sm, &sm.full[stg], (c >> 1) & 1);
            const auto &R = sm.raw[stg][R_];
            const auto &Kr = sm.raw[stg][K_];
            const auto &V = sm.raw[stg][V_];
            const auto &W = sm.raw[stg][W_];
            auto ld2 = [&](const __nv_bfloat16 (&tile)[kL][kHead], int e, float &a, float &b2) {
                const int p = p0 + e;
                const uint32_t off = (uint32_t)p * 128u + (((uint32_t)(lane >> 2) ^ (uint32_t)(e & 7)) << 4) + raw_off;
                const uint32_t v = *reinterpret_cast<const uint32_t *>(reinterpret_cast<const char *>(&tile[0][0]) + off);
                a = __uint_as_float(v << 16);
                b2 = __uint_as_float(v & 0xFFFF0000u);
            };
            // ---- cumulative log2-decay of this thread's 8 tokens, quarter exchange
            float e0[8], e1[8];
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ld2(W, e, e0[e], e1[e]);
                e0[e] *= 1.4426950408889634f;
                e1[e] *= 1.4426950408889634f;
                s0 += e0[e];
                s1 += e1[e];
            }
            *reinterpret_cast<float2 *>(&sm.part_sum[tw][ch]) = make_float2(s0, s1);
            named_sync(1, kTT);
            if (*(volatile int *)&sm.abort_) break;        // uniform: every thread passed the barrier
            float L0 = 0.f, L1 = 0.f;
            for (int q = 0; q < tw; ++q) {
                const float2 ps = *reinterpret_cast<const float2 *>(&sm.part_sum[q][ch]);
                L0 += ps.x;
                L1 += ps.y;
            }
            float l0[9], l1[9];
            float mx = fmaxf(fabsf(L0), fabsf(L1));
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                l0[e] = L0;
                l1[e] = L1;
                L0 += e0[e];
                L1 += e1[e];
                mx = fmaxf(mx, fmaxf(fabsf(L0), fabsf(L1)));
            }
            l0[8] = L0;
            l1[8] = L1;
            if (tw == kTW - 1) *reinterpret_cast<float2 *>(&sm.dec[c & 3][ch]) = make_float2(exp2f(L0), exp2f(L1));
            if (!(mx <= kLamMax * 1.4426950408889634f)) atomicMax(&sm.flag[c & 3], c + 1);
            // ---- r, k, v of the 8 tokens; bonus partials r u k
            float r0[8], r1[8], k0[8], k1[8], v0[8], v1[8], bp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ld2(R, e, r0[e], r1[e]);
                ld2(Kr, e, k0[e], k1[e]);
                ld2(V, e, v0[e], v1[e]);
                bp[e] = fmaf(r0[e] * u0, k0[e], r1[e] * u1 * k1[e]);
            }
            // transpose-reduce the 8 partials over the 32 lanes: lane ends with token (lane >> 2)
            {
                const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
                float a4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float keep = b4 ? bp[4 + q] : bp[q];
                    const float send = b4 ? bp[q] : bp[4 + q];
                    a4[q] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
                float a2[2];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float keep = b3 ? a4[2 + q] : a4[q];
                    const float send = b3 ? a4[q] : a4[2 + q];
                    a2[q] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
                float a1 = (b2 ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? a2[0] : a2[1], 4);
                a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
                a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
                if ((lane & 3) == 0) sm.cp[set][p0 + (lane >> 2)] = a1;
            }
            named_sync(1, kTT);
            const bool flagged = *(volatile int *)&sm.flag[c & 3] == c + 1;
            if (!flagged) {
                // ---- chunk operands
                float *Qs = sm.Q[set], *Ks = sm.K[set], *KT = sm.KT[set], *VT = sm.VT[set];
                float kt0[8], kt1[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int p = p0 + e;
                    const float q0 = r0[e] * exp2f(l0[e]), q1 = r1[e] * exp2f(l1[e]);
                    kt0[e] = k0[e] * exp2f(-l0[e + 1]);
                    kt1[e] = k1[e] * exp2f(-l1[e + 1]);
                    *reinterpret_cast<float2 *>(&Qs[swz(p, ch)]) = make_float2(q0, q1);
                    *reinterpret_cast<float2 *>(&Ks[swz(p, ch)]) = make_float2(kt0[e], kt1[e]);
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int pb = p0 + 4 * hh;
                    *reinterpret_cast<float4 *>(&KT[swz(ch, pb)]) =
                        make_float4(kt0[4 * hh], kt0[4 * hh + 1], kt0[4 * hh + 2], kt0[4 * hh + 3]);
                    *reinterpret_cast<float4 *>(&KT[swz(ch + 1, pb)]) =
                        make_float4(kt1[4 * hh], kt1[4 * hh + 1], kt1[4 * hh + 2], kt1[4 * hh + 3]);
                    *reinterpret_cast<float4 *>(&VT[swz(ch, pb)]) =
                        make_float4(v0[4 * hh], v0[4 * hh + 1], v0[4 * hh + 2], v0[4 * hh + 3]);
                    *reinterpret_cast<float4 *>(&VT[swz(ch + 1, pb)]) =
                        make_float4(v1[4 * hh], v1[4 * hh + 1], v1[4 * hh + 2], v1[4 * hh + 3]);
                }
                fence_proxy_async_smem();
                mbar_arrive(&sm.t_done);
                // ---- masked A' = strict-lower(Q Kt^T) + diag(c) into the K buffer
                wait_or_abort(sm, &sm.m1_done, ph_m1);   // on a timeout: garbage, then leave at the next barrier
                ph_m1 ^= 1;
                tc::fence_after_sync();
                {
                    const int col0 = 32 * (tw >> 2);        // warps 1..4 columns 0..31, warps 5..8 32..63
                    float a[32];
                    tc::tmem_ld32(tA + lane_off + col0, a);
                    tc::tmem_wait_ld();
                    if (rowlane) {
                        const int p = qrow;
                        const float cpp = sm.cp[set][p];
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            float x[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int s = col0 + 4 * g + e;
                                x[e] = s < p ? a[4 * g + e] : (s == p ? cpp : 0.f);
                            }
                            *reinterpret_cast<float4 *>(&Ks[swz(p, col0 + 4 * g)]) = make_float4(x[0], x[1], x[2], x[3]);
                        }
                    }
                }
                fence_proxy_async_smem();
                tc::fence_before_sync();
                mbar_arrive(&sm.a_done);
            } else {
                mbar_arrive(&sm.t_done);
                // ---- exact token-by-token evaluation of this chunk on the CUDA cores
                if (c > 0) wait_or_abort(sm, &sm.s_ready, (c - 1) & 1);
                tc::fence_after_sync();
                const bool worker = tw < 4 && rowlane;   // warps 1..4 hold the 64 state rows
                float Sr[64];
                {
                    float s0[32], s1[32];
                    tc::tmem_ld32(tS + lane_off, s0);
                    tc::tmem_ld32(tS + lane_off + 32, s1);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        Sr[j] = c > 0 ? s0[j] : 0.f;
                        Sr[32 + j] = c > 0 ? s1[j] : 0.f;
                    }
                }
                float *part = sm.Q[set];                  // [64 rows][64 cols] scratch
                for (int p = 0; p < kL; ++p) {
                    if (worker) {
                        const float rr = raw_at(R, p, qrow);
#pragma unroll
                        for (int j = 0; j < 64; ++j) part[qrow * 64 + j] = rr * Sr[j];
                    }
                    named_sync(1, kTT);
                    if (t < kHead) {
                        float acc = 0.f;
                        for (int r = 0; r < kHead; ++r) acc += part[r * 64 + t];
                        if (t0 + p < T)
                            prm.y[((size_t)b * T + t0 + p) * C + cbase + t] = fmaf(sm.cp[set][p], raw_at(V, p, t), acc);
                    }
                    if (worker) {
                        const float d = __expf(raw_at(W, p, qrow));
                        const float kk = raw_at(Kr, p, qrow);
#pragma unroll
                        for (int j = 0; j < 64; ++j) Sr[j] = fmaf(d, Sr[j], kk * raw_at(V, p, j));
                    }
                    named_sync(1, kTT);
                }
                {
                    float s0[32], s1[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        s0[j] = Sr[j];
                        s1[j] = Sr[32 + j];
                    }
                    if (tw < 4) {
                        tc::tmem_st32(tS + lane_off, s0);
                        tc::tmem_st32(tS + lane_off + 32, s1);
                        tc::tmem_wait_st();
                    }
                    if (worker) {
#pragma unroll
                        for (int j = 0; j < 64; ++j) sm.ST[swz(j, qrow)] = Sr[j];
                    }
                }
                fence_proxy_async_smem();
                tc::fence_before_sync();
                // the epilogue warps skip flagged chunks: the state hand-off is ours
                for (int r = 0; r < kET / kTT + (t < kET % kTT ? 1 : 0); ++r) mbar_arrive(&sm.s_ready);
            }
        }
    } else {
        // ===================== epilogue warps =====================
        const int e_t = tid - 32 * (1 + kTW);    // 0 .. kET-1
        (void)e_t;
        for (int c = 0; c < nch; ++c) {
            const int t0 = c * kL;
            if (!wait_or_abort(sm, &sm.mma_done, c & 1)) break;
            tc::fence_after_sync();
            if (*(volatile int *)&sm.flag[c & 3] == c + 1) continue;
            // ---- y = Y (the bonus is already on A's diagonal)
            {
                float y0[32], y1[32];
                tc::tmem_ld32(tY + lane_off, y0);
                tc::tmem_ld32(tY + lane_off + 32, y1);
                tc::tmem_wait_ld();
                const int t = t0 + qrow;
                if (rowlane && t < T) {
                    float4 *dst = reinterpret_cast<float4 *>(prm.y + ((size_t)b * T + t) * C + cbase);
#pragma unroll
                    for (int g = 0; g < 8; ++g) dst[g] = make_float4(y0[4 * g], y0[4 * g + 1], y0[4 * g + 2], y0[4 * g + 3]);
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        dst[8 + g] = make_float4(y1[4 * g], y1[4 * g + 1], y1[4 * g + 2], y1[4 * g + 3]);
                }
            }
            // ---- S rows scaled by exp(Lam_L); back to TMEM and transposed into ST
            {
                float s0[32], s1[32];
                tc::tmem_ld32(tS + lane_off, s0);
                tc::tmem_ld32(tS + lane_off + 32, s1);
                tc::tmem_wait_ld();
                const float dsc = rowlane ? sm.dec[c & 3][qrow] : 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    s0[j] *= dsc;
                    s1[j] *= dsc;
                }
                tc::tmem_st32(tS + lane_off, s0);
                tc::tmem_st32(tS + lane_off + 32, s1);
                if (rowlane) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        sm.ST[swz(j, qrow)] = s0[j];
                        sm.ST[swz(32 + j, qrow)] = s1[j];
                    }
                }
                tc::tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            mbar_arrive(&sm.s_ready);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}

cudaError_t wkv6_fwd_tc_launch(const CUtensorMap &mr, const CUtensorMap &mk, const CUtensorMap &mv,
                               const CUtensorMap &mw, const FwdParams &prm, cudaStream_t stream) {
    const size_t smem = sizeof(Tc2Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(wkv6_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    wkv6_fwd_tc_kernel<<<(unsigned)(prm.B * prm.H), kThreads, smem, stream>>>(mr, mk, mv, mw, prm);
    return cudaGetLastError();
}

}  // namespace wkv
