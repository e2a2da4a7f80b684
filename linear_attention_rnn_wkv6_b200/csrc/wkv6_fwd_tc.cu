// wkv6_fwd_tc.cu -- chunked RWKV-6 causal forward on the 5th-generation tensor cores.
//
// Same operation as wkv6_fwd.cu (bf16 r, k, v, w; fp32 u, state and y):
//   y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),   S_t = diag(d_t) S_{t-1} + k_t^T v_t.
// The pages' parallel training form ("RWKV Architecture ...", The Parallel
// Training Formulation) evaluates the decayed sums blockwise instead of token
// by token; here a chunk of L = 64 tokens of one (b, h) becomes three
// tcgen05 contractions (kind::f16, bf16 operands, fp32 accumulators in tensor
// memory; the state itself stays fp32 in tensor memory from chunk to chunk).
//
// Chunk algebra.  With Lam_p = sum_{m<p} ew_m (per row i, exclusive, chunk-local),
// Q_p = r_p * exp(Lam_p), Kt_s = k_s * exp(-Lam_{s+1}) and c_p = sum_i r_p u k_p:
//   y_p   = Q_p S_in + sum_{s<p} (Q_p . Kt_s) v_s + c_p v_p
//   S_out = diag(exp(Lam_L)) (S_in + Kt^T V)
// The products are arranged so that every operand is either a tile exactly as
// the TMA wrote it or a tile whose rows a thread writes contiguously:
//   M1   A^T          = Kt Q^T                 (M = 64 (s), N = 64 (p), K = i; two TMEM buffers)
//   P2   [Y ; S]     += [Q ; 0] S_in           (M = 128, N = 64 (j), K = i)
//   P34  [Y ; S]     += [A' ; Kt^T] V          (M = 128, N = 64 (j), K = s)
// where A' = strict-lower(A) + diag(c).  One M = 128 accumulator holds Y in
// TMEM lanes 0..63 (row p) and the fp32 state S in lanes 64..127 (row i).
// Q and Kt overwrite r and k in place in the TMA stage (same 128-byte-swizzled
// rows); an all-zero tile follows Q so that [Q ; 0] is one K-major operand;
// A'^T (written row s by row s) and Kt form the two 64-wide atoms of P34's
// MN-major A, V is P34's MN-major B as loaded, and S_in (bf16, written row i
// by row i) is P2's MN-major B.  After P34 the epilogue stores y, clears Y,
// scales row i of S by exp(Lam_L[i]) in TMEM and writes the bf16 copy S_in.
// On this hardware a tcgen05.mma costs about the same issue time for any of
// these shapes, so the kernel minimises the instruction count: 12 per chunk.
// |Lam| <= 80 keeps exp(-Lam) inside fp32.  A chunk whose summed |ew| exceeds
// that (fast-forgetting channels, decay down to exactly 0) is evaluated by the
// exact token-by-token recurrence on the CUDA cores, from the state in TMEM.
//
// Warp roles (one CTA per (b, h), 13 warps, two CTAs per SM):
//   warp 0       TMA loads (3-stage r/k/v ring, 2-stage w ring) and, from one
//                thread, all MMAs, in a fixed order
//   warps 1..4   transform: Q, Kt, the bonus scalars c, exp(Lam_L), chunk flag
//   warps 5..8   mask: A'^T from TMEM into shared memory
//   warps 9..12  epilogue: the two warps on TMEM lanes 0..63 stage y in the
//                chunk's Q/Kt slots for a TMA store, the two on lanes 64..127
//                rescale the state; all four run exact chunks
// Hand-offs are mbarriers; every wait is bounded and a shared abort flag stops
// all roles after the first timeout.
#include "wkv_launch.cuh"
#include "wkv_tc.cuh"

namespace wkv {

using namespace tc;

namespace {

constexpr int kL = 64;                       // tokens per chunk
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLamMax2 = 80.0f * kLog2e;   // |Lam| bound of the tensor-core path, log2 units
constexpr int kTW = 4;                       // transform warps (16 tokens each)
constexpr int kAW = 4;                       // mask warps
constexpr int kEW = 4;                       // epilogue warps
constexpr int kThreads = 32 * (1 + kTW + kAW + kEW);
constexpr int kTT = 32 * kTW;
constexpr int kAT = 32 * kAW;
constexpr int kET = 32 * kEW;
constexpr int kTokW = kL / kTW;              // tokens per transform warp
constexpr int kTile = kL * kHead;            // bf16 elements of one 64 x 64 tile (8 KB)

enum { R_ = 0, K_ = 1, V_ = 2, kSlots = 3 };
constexpr int kStages = 3;                   // r, k, v ring (freed by P34)
constexpr int kWStages = 2;                  // w ring (freed once the transform has read it)

struct TcSmem {
    __nv_bfloat16 Ap[kTile];             // A'^T (row s, p contiguous): first A atom of P34
    __nv_bfloat16 Sin[kTile];            // bf16 S_in (row i, j contiguous): B of P2
    __nv_bfloat16 raw[kStages][kSlots][kTile];   // stages: r -> Q, k -> Kt, v (TMA, swizzled)
    __nv_bfloat16 wt[kWStages][kTile];   // log-decay tiles (TMA, swizzled)
    float dec[4][kHead];                 // exp(Lam_L) per row i (ring of 4 chunks)
    float cp[4][kL];                     // bonus scalars per token (ring of 4 chunks)
    float psum[2][kTW][kHead];           // per-warp log2-decay sums, by chunk parity
    float pabs[2][kTW][kHead];           // per-warp sums of |log2-decay|
    float u[kHead];
    float ew5[kHead];                    // RWKV-5 static log-decay -w (natural log), unused otherwise
    float ypart[2][2][kHead];            // exact chunks: per-warp column sums, by token parity
    int flag[4];                         // chunk c is exact-evaluated iff flag[c & 3] == c + 1
    int abort_;
    uint32_t tmem_base;
    alignas(8) uint64_t full[kStages];   // r, k, v of the stage landed
    alignas(8) uint64_t wfull[kWStages]; // w of the w stage landed
    alignas(8) uint64_t t_done[kStages]; // transform of the stage's chunk done
    alignas(8) uint64_t m1_done[2];      // per TMEM A buffer: A^T ready
    alignas(8) uint64_t a_done[2];       // per TMEM A buffer: A'^T in shared memory, buffer read
    alignas(8) uint64_t ap_free;         // the A'^T buffer has been read (one phase per chunk)
    alignas(8) uint64_t stage_free[kStages];   // every reader of the stage finished
    alignas(8) uint64_t mma_done;        // Y and S of the chunk complete
    alignas(8) uint64_t s_ready;         // y stored and Y cleared, state rescaled, S_in written
    alignas(8) uint64_t final_bar;
};

// Two CTAs per SM: 228 KB of shared memory less 1 KB reserved per CTA, with the
// 1 KB alignment slack of the dynamic allocation.
static_assert(sizeof(TcSmem) + 1024 <= 113 * 1024, "two CTAs per SM must fit");

// try_wait with a suspend-time hint: the thread is parked by the hardware until
// the phase completes or about `ns` nanoseconds pass, without issuing anything.
__device__ __forceinline__ bool mbar_try_wait_for(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return done != 0;
}

// Bounded wait that gives up at once when another thread has already aborted.
// Waiting threads stay parked in the barrier (20 us at a time) instead of
// spinning, so they take no issue slots from the warps doing the work.
__device__ __forceinline__ bool wait_or_abort(TcSmem &sm, uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_for(bar, parity, 20000u)) return true;
        if (*(volatile int *)&sm.abort_) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_wkv_faults, WKV_FAULT_TIMEOUT);
            *(volatile int *)&sm.abort_ = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ bool is_flagged(const TcSmem &sm, int c) {
    return *(const volatile int *)&sm.flag[c & 3] == c + 1;
}

}  // namespace

template <bool STATIC>
__global__ void __launch_bounds__(kThreads, 2)
wkv6_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_r, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_w,
                   const __grid_constant__ CUtensorMap map_y, FwdParams prm) {
    extern __shared__ unsigned char smem_dyn[];
    TcSmem &sm = *reinterpret_cast<TcSmem *>(smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = prm.T, C = prm.C, H = prm.H;
    const int h = blockIdx.x % H, b = blockIdx.x / H;
    const int cbase = h * kHead;
    const int nch = (T + kL - 1) / kL;
    constexpr uint32_t kStageBytes = 3u * kTile * sizeof(__nv_bfloat16);   // r, k, v
    constexpr uint32_t kWBytes = kTile * sizeof(__nv_bfloat16);

    // RWKV-5 (STATIC): a static decay exp(-w5) per channel replaces the loaded w tiles
    constexpr bool stat = STATIC;
    if (tid < kHead) {
        sm.u[tid] = prm.u[cbase + tid];
        sm.ew5[tid] = stat ? -prm.w5[cbase + tid] : 0.f;
    }
    if (tid < 4) sm.flag[tid] = 0;
    if (tid == 0) {
        sm.abort_ = 0;
        prefetch_tensormap(&map_r);
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
        prefetch_tensormap(&map_w);
        prefetch_tensormap(&map_y);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.t_done[i], kTT);
            mbar_init(&sm.stage_free[i], 1);
        }
        for (int i = 0; i < kWStages; ++i) mbar_init(&sm.wfull[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.m1_done[i], 1);
            mbar_init(&sm.a_done[i], kAT);
        }
        mbar_init(&sm.ap_free, 1);
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.s_ready, kET);
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
    // TMEM columns: A^T buffers at 0 and 64 (M = 64 layout); [Y ; S] at 128 and P2's
    // Q S_in at 192 (M = 128: lane = row; only lanes 0..63 of the latter are read)
    const uint32_t tbase = sm.tmem_base;
    const uint32_t tD = tbase + 128, tD2 = tbase + 192;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's TMEM lane quarter

    if (warp == 0) {
        // ===================== TMA + MMA issue (one thread) =====================
        if (lane == 0) {
            auto issue = [&](int c) {
                const int s = c % kStages;
                mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
                tma_load_3d(sm.raw[s][R_], &map_r, cbase, c * kL, b, &sm.full[s]);
                tma_load_3d(sm.raw[s][K_], &map_k, cbase, c * kL, b, &sm.full[s]);
                tma_load_3d(sm.raw[s][V_], &map_v, cbase, c * kL, b, &sm.full[s]);
                // the load of chunk c + kStages waits for this stage's chunk to retire;
                // start its HBM reads now so that it is served from L2
                if (c + kStages < nch) {
                    tma_prefetch_l2_3d(&map_r, cbase, (c + kStages) * kL, b);
                    tma_prefetch_l2_3d(&map_k, cbase, (c + kStages) * kL, b);
                    tma_prefetch_l2_3d(&map_v, cbase, (c + kStages) * kL, b);
                }
            };
            // The thread's bookkeeping stays in scalars: an array indexed by a runtime
            // value would live in local memory, one L2 round trip per access under load.
            static_assert(kWStages == 2, "the w bookkeeping below has two stages");
            int last_w0 = -1, last_w1 = -1;     // latest chunk loaded into each w stage (-1: none)
            auto issue_w = [&](int c) {
                if (stat) return;   // no w tiles with a static decay
                const int s = c & 1;
                if (s) last_w1 = c; else last_w0 = c;
                mbar_arrive_expect_tx(&sm.wfull[s], kWBytes);
                tma_load_3d(sm.wt[s], &map_w, cbase, c * kL, b, &sm.wfull[s]);
            };
            constexpr uint32_t kIdM1 = idesc_bf16(64, 64, false, false);
            constexpr uint32_t kIdP2 = idesc_bf16(128, 64, false, true);
            constexpr uint32_t kIdP34 = idesc_bf16(128, 64, true, true);
            for (int c = 0; c < kStages && c < nch; ++c) issue(c);
            for (int c = 0; c < kWStages && c < nch; ++c) issue_w(c);
            int next_tma = min(nch, kStages);   // next chunk to load (r, k, v)
            // exact chunk whose w stage waits for its epilogue, per w stage (-1: none); a
            // slot cannot be reused before it is resolved, since the chunk that would
            // reuse it needs the pending load first
            int w_pend0 = -1, w_pend1 = -1;
            bool ok = true;
            // A fixed issue order, waiting on one barrier at a time (the waiting thread
            // is parked by the hardware and resumes as soon as the phase completes):
            //   M1(0), P2(0), then for every chunk c:  P34(c), M1(c+1), P2(c+1), load c+3.
            // Every input of a step comes from steps issued before it, so the order
            // cannot deadlock; M1 runs at most one chunk ahead of P34, a stage is
            // reloaded only after its chunk's last reader released it, and every parity
            // wait is on the oldest phase not yet observed, so none is ambiguous.
            auto step_m1 = [&](int c) -> bool {
                const int set = c & 1, s = c % kStages;
                if (!wait_or_abort(sm, &sm.t_done[s], (c / kStages) & 1)) return false;
                tc::fence_after_sync();
                if (!is_flagged(sm, c)) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tbase + 64 * set, desc_k(sm.raw[s][K_], k), desc_k(sm.raw[s][R_], k), kIdM1,
                                 k > 0);
                    tc::mma_commit(&sm.m1_done[set]);
                    if (c + kWStages < nch) issue_w(c + kWStages);   // the transform is done with w
                } else {
                    mbar_arrive(&sm.m1_done[set]);   // the mask warps skip this chunk
                    if (c & 1) w_pend1 = c; else w_pend0 = c;   // the exact evaluation still reads w
                }
                return true;
            };
            auto step_p2 = [&](int c) -> bool {
                // the epilogue of chunk c - 1 is done (the initial phase stands for c = 0)
                if (!wait_or_abort(sm, &sm.s_ready, c & 1)) return false;
                tc::fence_after_sync();
                // exact chunks up to c - 1 have released their w stage
                if (w_pend0 >= 0 && w_pend0 <= c - 1) {
                    if (w_pend0 + kWStages < nch) issue_w(w_pend0 + kWStages);
                    w_pend0 = -1;
                }
                if (w_pend1 >= 0 && w_pend1 <= c - 1) {
                    if (w_pend1 + kWStages < nch) issue_w(w_pend1 + kWStages);
                    w_pend1 = -1;
                }
                if (!is_flagged(sm, c)) {
                    const int s = c % kStages;
                    // [Q ; next tile] S_in: rows 64..127 land in TMEM lanes that are never read
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tD2, desc_k(sm.raw[s][R_], k), desc_mn(sm.Sin, k, 16), kIdP2, k > 0);
                }
                return true;
            };
            auto step_p34 = [&](int c) -> bool {
                const int set = c & 1, s = c % kStages;
                if (!wait_or_abort(sm, &sm.a_done[set], (c >> 1) & 1)) return false;
                tc::fence_after_sync();
                if (!is_flagged(sm, c)) {
                    const uint32_t lbo = smem_u32(sm.raw[s][K_]) - smem_u32(sm.Ap);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tD, desc_mn(sm.Ap, k, lbo), desc_mn(sm.raw[s][V_], k, 16), kIdP34, true);
                    tc::mma_commit(&sm.mma_done);
                    tc::mma_commit(&sm.ap_free);
                } else {
                    // the epilogue evaluates this chunk exactly and then releases its stage;
                    // the A'^T buffer phase is completed by a commit, in order behind P34(c - 1)
                    mbar_arrive(&sm.mma_done);
                    tc::mma_commit(&sm.ap_free);
                }
                return true;
            };
            ok = step_m1(0) && step_p2(0);
            for (int c = 0; c < nch && ok; ++c) {
                ok = step_p34(c);
                if (ok && c + 1 < nch) ok = step_m1(c + 1) && step_p2(c + 1);
                if (ok && next_tma < nch) {
                    // the stage of chunk next_tma - kStages (= c once the ring is full) is
                    // released by the epilogue once its y store has read the staging tiles
                    // (or its exact evaluation is done); P2(c + 1) already waited for the
                    // rest of that epilogue, so this wait is short
                    const int cc = next_tma - kStages;
                    ok = wait_or_abort(sm, &sm.stage_free[cc % kStages], (cc / kStages) & 1);
                    if (ok) {
                        fence_proxy_async_smem();
                        issue(next_tma);
                        ++next_tma;
                    }
                }
            }
            // every MMA issued so far must finish before TMEM is released
            tc::mma_commit(&sm.final_bar);
            mbar_wait_bounded(&sm.final_bar, 0);
            if (!ok) {
                // drain the loads still in flight (the last kStages r/k/v loads, the w loads)
                for (int cc = max(0, next_tma - kStages); cc < next_tma; ++cc)
                    mbar_wait_bounded(&sm.full[cc % kStages], (cc / kStages) & 1);
                if (last_w0 >= 0) mbar_wait_bounded(&sm.wfull[0], (last_w0 / kWStages) & 1);
                if (last_w1 >= 0) mbar_wait_bounded(&sm.wfull[1], (last_w1 / kWStages) & 1);
            }
        }
    } else if (warp <= kTW) {
        // ===================== transform warps =====================
        // warp tw handles tokens [16 tw, 16 tw + 16) of the chunk; lane handles
        // channels (2 lane, 2 lane + 1), i.e. 4 bytes of 16-byte chunk lane / 4
        const int tw = warp - 1;
        const int ch = 2 * lane;
        const int p0 = kTokW * tw;
        const uint32_t in_chunk = (uint32_t)(lane & 3) << 2;
        const uint32_t chunk = (uint32_t)(lane >> 2);
        for (int c = 0; c < nch; ++c) {
            const int stg = c % kStages, par = c & 1;
            // a timeout sets the shared abort flag; all transform threads leave
            // together after the named barrier below, so none is left waiting there
            wait_or_abort(sm, &sm.full[stg], (c / kStages) & 1);
            if (!stat) wait_or_abort(sm, &sm.wfull[c % kWStages], (c / kWStages) & 1);
            __nv_bfloat16 *Rb = sm.raw[stg][R_], *Kb = sm.raw[stg][K_];
            const __nv_bfloat16 *Wb = sm.wt[c % kWStages];
            auto off = [&](int e) -> uint32_t {
                const int p = p0 + e;
                return (uint32_t)p * 128u + ((chunk ^ (uint32_t)(p & 7)) << 4) + in_chunk;
            };
            float L0, L1, tot0, tot1, ab0, ab1;
            if (stat) {
                const float st0 = sm.ew5[ch] * kLog2e, st1 = sm.ew5[ch + 1] * kLog2e;   // static log2-decay
                // closed-form decay powers: Lam_p = p ew, the chunk total is L ew; no
                // w tiles and no sums across the warps (each warp sees every channel)
                if (*(volatile int *)&sm.abort_) break;
                L0 = (float)p0 * st0;
                L1 = (float)p0 * st1;
                tot0 = (float)kL * st0;
                tot1 = (float)kL * st1;
                ab0 = fabsf(tot0);
                ab1 = fabsf(tot1);
            } else {
                // ---- log2-decay sums of this warp's 16 tokens (signed and absolute)
                float s0 = 0.f, s1 = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int e = 0; e < kTokW; ++e) {
                    const uint32_t wv = ld_u32(Wb, off(e));
                    const float x0 = bf_lo(wv) * kLog2e, x1 = bf_hi(wv) * kLog2e;
                    s0 += x0;
                    s1 += x1;
                    a0 += fabsf(x0);
                    a1 += fabsf(x1);
                }
                *reinterpret_cast<float2 *>(&sm.psum[par][tw][ch]) = make_float2(s0, s1);
                *reinterpret_cast<float2 *>(&sm.pabs[par][tw][ch]) = make_float2(a0, a1);
                named_sync(1, kTT);
                if (*(volatile int *)&sm.abort_) break;        // uniform: every thread passed the barrier
                L0 = 0.f, L1 = 0.f, tot0 = 0.f, tot1 = 0.f, ab0 = 0.f, ab1 = 0.f;
#pragma unroll
                for (int q = 0; q < kTW; ++q) {
                    const float2 ps = *reinterpret_cast<const float2 *>(&sm.psum[par][q][ch]);
                    const float2 pa = *reinterpret_cast<const float2 *>(&sm.pabs[par][q][ch]);
                    if (q < tw) {
                        L0 += ps.x;
                        L1 += ps.y;
                    }
                    tot0 += ps.x;
                    tot1 += ps.y;
                    ab0 += pa.x;
                    ab1 += pa.y;
                }
            }
            // sum |ew| bounds every |Lam_p| of the chunk; every warp reads the same
            // sums in the same order, so all four reach the same verdict
            const bool flagged = __any_sync(0xffffffffu, !(ab0 <= kLamMax2) || !(ab1 <= kLamMax2));
            if (tw == 0) {
                *reinterpret_cast<float2 *>(&sm.dec[c & 3][ch]) = make_float2(exp2f(tot0), exp2f(tot1));
                if (lane == 0 && flagged) sm.flag[c & 3] = c + 1;
            }
            // ---- Q and Kt in place of r and k; bonus scalars c_p, 8 tokens at a time
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float bp[8];
                // flagged is warp-uniform: keeping the branch outside the token loop
                // leaves one straight-line body whose loads and exponentials overlap
                // per-channel constants are re-read from shared memory here rather than
                // held in registers across the chunk loop
                const float u0 = sm.u[ch], u1 = sm.u[ch + 1];
                if (!flagged) {
                    const float st0 = sm.ew5[ch] * kLog2e, st1 = sm.ew5[ch + 1] * kLog2e;
                    // four tokens at a time, loads first: the in-place stores below may
                    // alias them as far as the compiler can tell, so loads issued after a
                    // store would serialise (batches of four keep the registers in bounds)
#pragma unroll
                    for (int sb = 0; sb < 2; ++sb) {
                        uint32_t rv[4], kv[4], wv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t o = off(8 * half + 4 * sb + e);
                            rv[e] = ld_u32(Rb, o);
                            kv[e] = ld_u32(Kb, o);
                            wv[e] = stat ? 0u : ld_u32(Wb, o);
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t o = off(8 * half + 4 * sb + e);
                            const float r0 = bf_lo(rv[e]), r1 = bf_hi(rv[e]), k0 = bf_lo(kv[e]), k1 = bf_hi(kv[e]);
                            bp[4 * sb + e] = fmaf(r0 * u0, k0, r1 * u1 * k1);
                            const float q0 = r0 * fast_exp2(L0), q1 = r1 * fast_exp2(L1);
                            L0 += stat ? st0 : bf_lo(wv[e]) * kLog2e;
                            L1 += stat ? st1 : bf_hi(wv[e]) * kLog2e;
                            st_u32(Rb, o, pack_bf16(q0, q1));
                            st_u32(Kb, o, pack_bf16(k0 * fast_exp2(-L0), k1 * fast_exp2(-L1)));
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t o = off(8 * half + e);
                        const uint32_t rv = ld_u32(Rb, o), kv = ld_u32(Kb, o);
                        bp[e] = fmaf(bf_lo(rv) * u0, bf_lo(kv), bf_hi(rv) * u1 * bf_hi(kv));
                    }
                }
                const float cpv = transpose_reduce8(bp, lane);
                if ((lane & 3) == 0) sm.cp[c & 3][p0 + 8 * half + (lane >> 2)] = cpv;
            }
            fence_proxy_async_smem();
            mbar_arrive(&sm.t_done[stg]);
        }
    } else if (warp <= kTW + kAW) {
        // ===================== mask warps: A'^T = strict-upper(A^T) + diag(c) =====================
        const int s = 16 * (warp & 3) + (lane & 15);   // A^T row (M = 64 layout: lanes 0..15 of the quarter)
        const bool rowlane = lane < 16;
        for (int c = 0; c < nch; ++c) {
            const int set = c & 1;
            if (!wait_or_abort(sm, &sm.m1_done[set], (c >> 1) & 1)) break;
            if (!is_flagged(sm, c)) {
                // the single A'^T buffer: P34 of the previous chunk must have read it
                if (c > 0 && !wait_or_abort(sm, &sm.ap_free, (c - 1) & 1)) break;
                tc::fence_after_sync();
                const float cps = sm.cp[c & 3][s];
                __nv_bfloat16 *Ab = sm.Ap;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float a[32];
                    tc::tmem_ld32(tbase + 64 * set + lane_off + 32 * half, a);
                    tc::tmem_wait_ld();
                    if (rowlane) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            float x[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int p = 32 * half + 8 * g + e;
                                x[e] = p > s ? a[8 * g + e] : (p == s ? cps : 0.f);
                            }
                            st_u128(Ab, swz(s, 32 * half + 8 * g),
                                    make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                                               pack_bf16(x[6], x[7])));
                        }
                    }
                }
                fence_proxy_async_smem();
                tc::fence_before_sync();
            }
            // every chunk arrives once, so the buffer's phase count stays chunk >> 1
            mbar_arrive(&sm.a_done[set]);
        }
    } else {
        // ===================== epilogue warps =====================
        const int et = tid - 32 * (1 + kTW + kAW);   // 0 .. kET-1
        const int q = warp & 3;                       // TMEM lane quarter
        const bool yrole = q < 2;                     // lanes 0..63: Y rows; lanes 64..127: S rows
        const int row = 32 * (q & 1) + lane;          // p (Y) or i (S)
        // everything starts at zero: Y, S and the bf16 copy S_in
        {
            float z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0.f;
            tc::tmem_st32(tD + lane_off, z);
            tc::tmem_st32(tD + lane_off + 32, z);
            uint4 *st = reinterpret_cast<uint4 *>(sm.Sin);
            for (int i = et; i < kTile * 2 / 16; i += kET) st[i] = make_uint4(0u, 0u, 0u, 0u);
            tc::tmem_wait_st();
            fence_proxy_async_smem();
            tc::fence_before_sync();
            mbar_arrive(&sm.s_ready);
        }
        for (int c = 0; c < nch; ++c) {
            const int t0 = c * kL, stg = c % kStages;
            wait_or_abort(sm, &sm.mma_done, c & 1);
            named_sync(2, kET);
            if (*(volatile int *)&sm.abort_) break;        // uniform: every thread passed the barrier
            tc::fence_after_sync();
            const bool exact = is_flagged(sm, c);
            if (!exact) {
                if (yrole) {
                    // ---- y row p = (A' V) row p + (Q S_in) row p, then clear Y for the next
                    // chunk.  The row goes to two 128B-swizzled fp32 staging tiles (columns
                    // 0..31 and 32..63) in the Q and Kt slots of the chunk's stage, which no
                    // MMA reads any more; one thread then stores them with the TMA, which
                    // writes whole lines and leaves out the rows past T.
#pragma unroll 1
                    for (int qt = 0; qt < 4; ++qt) {   // 16 columns at a time keeps registers low
                        float v[16], v2[16];
                        tc::tmem_ld16(tD + lane_off + 16 * qt, v);
                        tc::tmem_ld16(tD2 + lane_off + 16 * qt, v2);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] += v2[e];
                        char *box = reinterpret_cast<char *>(sm.raw[stg][R_ + (qt >> 1)]) + row * 128;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int j = 4 * (qt & 1) + g;   // 16-byte chunk of the 128-byte row
                            *reinterpret_cast<float4 *>(box + ((j ^ (row & 7)) << 4)) =
                                make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                        }
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = 0.f;
                        tc::tmem_st16(tD + lane_off + 16 * qt, v);
                    }
                } else {
                    // ---- S row i scaled by exp(Lam_L[i]), back to TMEM, bf16 copy into S_in
                    const float dsc = sm.dec[c & 3][row];
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        float v[32];
                        tc::tmem_ld32(tD + lane_off + 32 * half, v);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] *= dsc;
                        tc::tmem_st32(tD + lane_off + 32 * half, v);
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            st_u128(sm.Sin, swz(row, 32 * half + 8 * g),
                                    make_uint4(pack_bf16(v[8 * g], v[8 * g + 1]), pack_bf16(v[8 * g + 2], v[8 * g + 3]),
                                               pack_bf16(v[8 * g + 4], v[8 * g + 5]),
                                               pack_bf16(v[8 * g + 6], v[8 * g + 7])));
                    }
                }
                tc::tmem_wait_st();
            } else {
                // ---- exact token-by-token evaluation of this chunk on the CUDA cores.
                // The S warps own rows i of S and form per-warp column sums of
                // r_p[i] S[i][j]; the Y warps add the two halves and the bonus and store y.
                const __nv_bfloat16 *R = sm.raw[stg][R_], *Kr = sm.raw[stg][K_];
                const __nv_bfloat16 *V = sm.raw[stg][V_], *W = sm.wt[c % kWStages];
                for (int p = 0; p < kL; ++p) {
                    if (!yrole) {
                        const float rr = raw_at(R, p, row), kk = raw_at(Kr, p, row);
                        const float dd = __expf(stat ? sm.ew5[row] : raw_at(W, p, row));
#pragma unroll 1
                        for (int m = 0; m < 4; ++m) {
                            float s16[16];
                            tc::tmem_ld16(tD + lane_off + 16 * m, s16);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                float pr[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) pr[e] = rr * s16[8 * hh + e];
                                const float colsum = transpose_reduce8(pr, lane);   // column 16 m + 8 hh + (lane >> 2)
                                if ((lane & 3) == 0) sm.ypart[p & 1][q - 2][16 * m + 8 * hh + (lane >> 2)] = colsum;
                            }
                        }
                        // update after every column sum of this token has read the old S
#pragma unroll 1
                        for (int m = 0; m < 4; ++m) {
                            float s16[16];
                            tc::tmem_ld16(tD + lane_off + 16 * m, s16);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e) s16[e] = fmaf(dd, s16[e], kk * raw_at(V, p, 16 * m + e));
                            tc::tmem_st16(tD + lane_off + 16 * m, s16);
                            tc::tmem_wait_st();
                        }
                    }
                    named_sync(2, kET);
                    if (yrole && t0 + p < T && in_range(((size_t)b * T + t0 + p) * C + cbase + row, (size_t)prm.B * T * C)) {
                        const int jj = row;   // 0..63
                        prm.y[((size_t)b * T + t0 + p) * C + cbase + jj] =
                            sm.ypart[p & 1][0][jj] + sm.ypart[p & 1][1][jj] + sm.cp[c & 3][p] * raw_at(V, p, jj);
                    }
                }
                if (!yrole) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float v[32];
                        tc::tmem_ld32(tD + lane_off + 32 * half, v);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            st_u128(sm.Sin, swz(row, 32 * half + 8 * g),
                                    make_uint4(pack_bf16(v[8 * g], v[8 * g + 1]), pack_bf16(v[8 * g + 2], v[8 * g + 3]),
                                               pack_bf16(v[8 * g + 4], v[8 * g + 5]),
                                               pack_bf16(v[8 * g + 6], v[8 * g + 7])));
                    }
                }
                // every epilogue thread is done with the raw stage: release it
                named_sync(2, kET);
                if (et == 0) {
                    fence_proxy_async_smem();
                    mbar_arrive(&sm.stage_free[stg]);
                }
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            mbar_arrive(&sm.s_ready);
            if (yrole && !exact) {
                // every Y row is staged (and fenced for the async proxy): store the tiles,
                // then release the stage once the TMA has read them
                named_sync(3, kET / 2);
                if (row == 0) {
                    tma_store_3d(&map_y, sm.raw[stg][R_], cbase, t0, b);
                    tma_store_3d(&map_y, sm.raw[stg][K_], cbase + kHead / 2, t0, b);
                    bulk_commit_group();
                    bulk_wait_read_all();
                    mbar_arrive(&sm.stage_free[stg]);
                }
            }
        }
        if (yrole && row == 0) bulk_wait_all();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}

cudaError_t wkv6_fwd_tc_launch(const CUtensorMap &mr, const CUtensorMap &mk, const CUtensorMap &mv,
                               const CUtensorMap &mw, const CUtensorMap &my, const FwdParams &prm,
                               cudaStream_t stream) {
    const size_t smem = sizeof(TcSmem) + 1024;
    auto kern = prm.w5 != nullptr ? wkv6_fwd_tc_kernel<true> : wkv6_fwd_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(prm.B * prm.H), kThreads, smem, stream>>>(mr, mk, mv, mw, my, prm);
    return cudaGetLastError();
}

}  // namespace wkv
