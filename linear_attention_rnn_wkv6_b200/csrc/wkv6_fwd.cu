// wkv6_fwd.cu -- RWKV-6 WKV forward (causal and bidirectional) for sm_100a: the
// first register-recurrence kernel, which the test build (WKV_RECURRENCE_PATHS)
// runs for the bf16 causal forward and the fused fp32 forwards; every other
// recurrence-form forward runs the pipelined kernel of wkv6_fwd_pipe.cu.
//
// Operation (per batch b, head h; N = 64; d_t = exp(ew_t)):
//   causal : y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),  S_t = diag(d_t) S_{t-1} + k_t^T v_t
//   bidir  : adds r_t S^b_{t+1} with S^b_t = diag(d_t) S^b_{t+1} + k_t^T v_t (no bonus)
// ("RWKV Architecture ...", RWKV-5 matrix state / RWKV-6 dynamic decay;
//  "How Custom CUDA Kernels (wkv6_cuda.cu) ...", Forward Pass Implementation.)
//
// Design (B200-first; the pages' one-thread-per-column kernel is prior art only)
// -----------------------------------------------------------------------------
// * One CTA per (b, h, group of CW = 16*WARPS value columns).  Value columns j
//   of S are independent (decay scales rows, x_t = k_t^T v_t is an outer
//   product), so a head's 64 columns may be split over CTAs.
// * Inputs are staged in chunks of TC tokens by TMA (3-D tensor maps over
//   [B][T][C], boxes of TC x 64 for r, k, w and TC x CW for v) into a
//   double-buffered shared-memory ring, one mbarrier per stage.  Rows outside
//   [0, T) come back zero filled: zero r, k, v contribute nothing and a zero
//   log-decay keeps the state, so ragged chunks need no masking except on the
//   y store.
// * Scaled state.  Inside a chunk (tokens in processing order p = 0..TC-1) the
//   kernel keeps S' with S_before(p) = diag(exp(L_p)) S', where L_p is the sum
//   of the log-decays of the chunk's tokens before p.  Then
//       readout  y_p  = (r_p * exp(L_p)) . S'                   (1 FMA / element)
//       update   S'  += (k_p * exp(-L_{p+1})) v_p^T               (1 FMA / element)
//   instead of 3 operations per element for the plain recurrence.  A
//   "renorm step" ends every run: S' <- diag(exp(L_p + ew_p)) S' + k_p v_p^T,
//   after which L restarts at 0.  The last token of each chunk is always a
//   renorm step, and so is any token whose |ew| exceeds kTheta / TC in some
//   row, so |L| <= kTheta inside a run and exp(+-L) stays inside fp32.  For an
//   arbitrary decay (down to exactly 0) the result is the plain recurrence's.
// * Register state: warp w owns columns [16w, 16w+16) of the CTA's group;
//   lane (rg = lane & 7, cg = lane >> 3) holds rows {4rg..4rg+3, 32+4rg..32+4rg+3}
//   x columns {4cg..4cg+3}: 32 fp32 state registers.  The readout sums over
//   rows with a 3-level butterfly reduce-scatter (4 shuffles).
// * The bonus term (r_t . u . k_t) v_t is a per-token scalar c_t times v_t;
//   c_t is formed once per token in the transform step.
// * RWKV-5 ("RWKV Architecture ...", RWKV-5 "Eagle": S_t = exp(-w) . S_{t-1} +
//   k_t^T v_t with a static per-channel w) runs the same kernel with the
//   log-decay -w of each channel in shared memory instead of the loaded w tile,
//   so a stage carries r, k and v only.
// * Fused prologue and epilogue (fp32).  RWKV-6 computes the decay from a base
//   and a low-rank term, w_t = w_base + tanh(x_t W1) W2, and hands the kernel
//   ew = -exp(w_t); a head's output is then group-normalised and gated
//   ("RWKV Architecture ...", RWKV-6 "Finch" and RWKV-5 "Eagle"; the spatial-mix
//   block of "How the WKV ... Processes Images").  With FwdParams::wb the loaded
//   tile is ww = tanh(x W1) W2 and is turned into ew in shared memory; with
//   FwdParams::gn_w each finished y row of a head (the 16 lanes of a half warp)
//   is normalised, scaled, shifted and multiplied by the gate before its store.
//   Neither w nor the un-normalised y makes a trip through HBM.
#include <type_traits>

#include "wkv_launch.cuh"

namespace wkv {

[[maybe_unused]] constexpr float kTheta = 40.0f;  // bound on |L| inside a run (exp(40) ~ 2.4e17)

template <typename Tin, int WARPS, int TC>
struct FwdSmem {
    static constexpr int CW = 16 * WARPS;
    // raw TMA landing buffers (2 stages)
    Tin raw_r[2][TC][kHead];
    Tin raw_k[2][TC][kHead];
    Tin raw_w[2][TC][kHead];
    Tin raw_v[2][TC][CW];
    // transformed chunk, processing order
    float rs[TC][kHead];     // r_p * exp(L_p)
    float ks[TC][kHead];     // k_p * exp(-L_{p+1})  (k_p on renorm steps)
    float al[TC][kHead];     // exp(L_p + ew_p) on renorm steps
    float vs[TC][CW];        // v_p (fp32), this CTA's columns
    float ybuf[TC][CW];      // y_p, this CTA's columns
    float c[TC];             // bonus scalar sum_i r_p u k_p
    float u[kHead];
    float ew5[kHead];        // static log-decay -w5 (RWKV-5), unused otherwise
    float wbase[kHead];      // w_base of the decay prologue, unused otherwise
    uint32_t renorm_mask;    // bit p set: token p is a renorm step
    alignas(8) uint64_t full[2];
};

// Chunk g of the CTA's sweep sequence: pass 0 is anti-causal when bidirectional.
struct ChunkPos {
    int dir;     // +1 past->future, -1 future->past
    int t_lo;    // first token (lowest t) of the TMA box; may be < 0 for dir -1
    int pass;
    int c;       // chunk index within the pass
};

__device__ __forceinline__ ChunkPos chunk_pos(int g, int nch, int T, int TC, bool bidir) {
    ChunkPos cp;
    cp.pass = bidir ? (g / nch) : 1;
    cp.c = bidir ? (g % nch) : g;
    cp.dir = (bidir && cp.pass == 0) ? -1 : +1;
    cp.t_lo = (cp.dir > 0) ? cp.c * TC : (T - (cp.c + 1) * TC);
    return cp;
}

template <typename Tin, int WARPS, int TC, bool BIDIR>
__global__ void __launch_bounds__(32 * WARPS, 3)
wkv6_fwd_kernel(const __grid_constant__ CUtensorMap map_r, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_w,
                FwdParams prm) {
    using Smem = FwdSmem<Tin, WARPS, TC>;
    constexpr int CW = Smem::CW;
    constexpr int NT = 32 * WARPS;
    constexpr int GROUPS = kHead / CW;
    constexpr uint32_t kStageBytes = (3 * TC * kHead + TC * CW) * sizeof(Tin);
    constexpr uint32_t kWBytes = TC * kHead * sizeof(Tin);
    extern __shared__ unsigned char smem_dyn[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_dyn + ((128u - (smem_u32(smem_dyn) & 127u)) & 127u));

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int T = prm.T, C = prm.C, H = prm.H;
    const int grp = blockIdx.x % GROUPS;
    const int bh = blockIdx.x / GROUPS;
    const int h = bh % H;
    const int b = bh / H;
    const int cbase = h * kHead;             // first channel of the head
    const int col0 = grp * CW;               // first value column of this CTA (head-relative)
    const int nch = (T + TC - 1) / TC;
    const int nchunks = BIDIR ? 2 * nch : nch;

    // RWKV-5: one log-decay per channel for every token; the w map is not read
    const bool stat = prm.w5 != nullptr;
    // decay prologue (fp32 only): the loaded tile is ww, turned into ew = -exp(w_base + ww)
    const bool pro = std::is_same<Tin, float>::value && prm.wb != nullptr;
    if (tid < kHead) {
        sm.u[tid] = prm.u[cbase + tid];
        sm.ew5[tid] = stat ? -prm.w5[cbase + tid] : 0.f;
        sm.wbase[tid] = pro ? prm.wb[cbase + tid] : 0.f;
    }
    if (tid == 0) {
        prefetch_tensormap(&map_r);
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
        prefetch_tensormap(&map_w);
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        fence_barrier_init();
    }
    __syncthreads();

    auto issue = [&](int g) {
        const ChunkPos cp = chunk_pos(g, nch, T, TC, BIDIR);
        const int s = g & 1;
        mbar_arrive_expect_tx(&sm.full[s], stat ? kStageBytes - kWBytes : kStageBytes);
        tma_load_3d(&sm.raw_r[s][0][0], &map_r, cbase, cp.t_lo, b, &sm.full[s]);
        tma_load_3d(&sm.raw_k[s][0][0], &map_k, cbase, cp.t_lo, b, &sm.full[s]);
        if (!stat) tma_load_3d(&sm.raw_w[s][0][0], &map_w, cbase, cp.t_lo, b, &sm.full[s]);
        tma_load_3d(&sm.raw_v[s][0][0], &map_v, cbase + col0, cp.t_lo, b, &sm.full[s]);
    };
    if (tid == 0) {
        issue(0);
        if (nchunks > 1) issue(1);
    }

    // register state: rows R(q) = (q < 4 ? 4*rg + q : 32 + 4*rg + q - 4), cols 4*cg + j
    const int rg = lane & 7;
    const int cg = lane >> 3;
    const int rowA = 4 * rg;
    const int rowB = 32 + 4 * rg;
    const int jc = 16 * warp + 4 * cg;       // CTA-relative first column of this lane
    const int jj = (rg >> 1) & 3;            // column (of the 4) this lane holds after the reduce
    const bool b2 = (rg & 4) != 0, b1 = (rg & 2) != 0;
    // packed fp32: S2[qq][j] = (S[row 2qq][j], S[row 2qq+1][j]) for the row pairs
    // (rowA, rowA+1), (rowA+2, rowA+3), (rowB, rowB+1), (rowB+2, rowB+3); one
    // __ffma2_rn does two multiply-adds
    constexpr float2 kZero2 = {0.f, 0.f};
    float2 S2[4][4];
#pragma unroll
    for (int qq = 0; qq < 4; ++qq)
#pragma unroll
        for (int j = 0; j < 4; ++j) S2[qq][j] = kZero2;
    // state row of pair qq, half e (0: first row of the pair, 1: second)
    auto prow = [&](int qq, int e) { return (qq < 2 ? rowA + 2 * qq : rowB + 2 * (qq - 2)) + e; };
    const size_t state_off = ((size_t)b * H + h) * kHead * kHead + col0 + jc;
    if (!BIDIR && prm.s0 != nullptr) {
        // initial state: the scaled state equals the true state at a chunk start
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const float4 x0 = *reinterpret_cast<const float4 *>(prm.s0 + state_off + (size_t)prow(qq, 0) * kHead);
            const float4 x1 = *reinterpret_cast<const float4 *>(prm.s0 + state_off + (size_t)prow(qq, 1) * kHead);
            S2[qq][0] = make_float2(x0.x, x1.x);
            S2[qq][1] = make_float2(x0.y, x1.y);
            S2[qq][2] = make_float2(x0.z, x1.z);
            S2[qq][3] = make_float2(x0.w, x1.w);
        }
    }

    // group-norm weight and bias of the 4 output columns this thread writes (the same
    // columns in every write-out round)
    static_assert(NT % (CW / 4) == 0, "a thread writes the same columns in every round");
    float4 gnw = make_float4(0.f, 0.f, 0.f, 0.f), gnb = gnw;
    if (prm.gn_w != nullptr) {
        const int j4 = (tid % (CW / 4)) * 4;
        gnw = __ldg(reinterpret_cast<const float4 *>(prm.gn_w + cbase + col0 + j4));
        gnb = __ldg(reinterpret_cast<const float4 *>(prm.gn_b + cbase + col0 + j4));
    }

    for (int g = 0; g < nchunks; ++g) {
        const ChunkPos cp = chunk_pos(g, nch, T, TC, BIDIR);
        const int s = g & 1;
        const bool with_bonus = !(BIDIR && cp.pass == 0);
        if (BIDIR && g == nch) {             // pass boundary: fresh state
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
#pragma unroll
                for (int j = 0; j < 4; ++j) S2[qq][j] = kZero2;
        }
        // ---- wait for the chunk ----
        const bool ok = mbar_wait_bounded(&sm.full[s], (g >> 1) & 1);
        if (!__syncthreads_and(ok)) {         // a bounded wait ran out: stop (fault recorded)
            drain_two_stage(sm.full, g, nchunks);
            return;
        }

        // log-decay of box row `row` (token cp.t_lo + row), channel i; a static decay
        // applies to tokens inside [0, T) only, like the zero fill of the loaded w
        auto ew_at = [&](int row, int i) -> float {
            if (!stat) return to_f32(sm.raw_w[s][row][i]);
            const int t = cp.t_lo + row;
            return (t >= 0 && t < T) ? sm.ew5[i] : 0.f;
        };
        // ---- transform: renorm flags ----
        // a token is a renorm step if some row has |ew| > kTheta / TC (or NaN)
        int bad = 0;
        if constexpr (std::is_same<Tin, float>::value) {
            if (pro) {
                // decay prologue, in place: rows outside [0, T) keep the zero log-decay
                for (int e = tid; e < TC * kHead; e += NT) {
                    const int row = e / kHead, i = e % kHead, t = cp.t_lo + row;
                    const float ew = (t >= 0 && t < T) ? -expf(sm.wbase[i] + sm.raw_w[s][row][i]) : 0.f;
                    sm.raw_w[s][row][i] = ew;
                    bad |= !(fabsf(ew) <= kTheta / TC);
                }
                fence_proxy_async_smem();   // the stage is reloaded by the TMA later
            }
        }
        if (!pro)
            for (int e = tid; e < TC * kHead; e += NT) {
                const float ew = ew_at(e / kHead, e % kHead);
                bad |= !(fabsf(ew) <= kTheta / TC);
            }
        const int any_bad = __syncthreads_or(bad);
        if (tid < 32) {
            uint32_t mask = 1u << (TC - 1);
            if (any_bad) {
                for (int p = 0; p < TC - 1; ++p) {
                    const int row = cp.dir > 0 ? p : TC - 1 - p;
                    const float e0 = ew_at(row, lane);
                    const float e1 = ew_at(row, lane + 32);
                    const bool bad = !(fabsf(e0) <= kTheta / TC) || !(fabsf(e1) <= kTheta / TC);
                    if (__any_sync(0xffffffffu, bad)) mask |= 1u << p;
                }
            }
            if (tid == 0) sm.renorm_mask = mask;
        }
        __syncthreads();
        const uint32_t rmask = sm.renorm_mask;
        // ---- transform: scaled r, k per row (sequential over the chunk) ----
        // two threads per row i, each half of the chunk; the second one first sums
        // the decays of the first half (with the renorm resets)
        {
            static_assert(NT == 2 * kHead && TC % 2 == 0, "transform split assumes 2 threads per row");
            constexpr int TH = TC / 2;
            const int i = tid & (kHead - 1), p0 = (tid >> 6) * TH;
            float L = 0.f;
            for (int p = 0; p < p0; ++p) {
                const int row = cp.dir > 0 ? p : TC - 1 - p;
                L = ((rmask >> p) & 1u) ? 0.f : L + ew_at(row, i);
            }
            float ew[TH], rr[TH], kk[TH];
#pragma unroll
            for (int e = 0; e < TH; ++e) {
                const int p = p0 + e, row = cp.dir > 0 ? p : TC - 1 - p;
                ew[e] = ew_at(row, i);
                rr[e] = to_f32(sm.raw_r[s][row][i]);
                kk[e] = to_f32(sm.raw_k[s][row][i]);
            }
#pragma unroll
            for (int e = 0; e < TH; ++e) {
                const int p = p0 + e;
                sm.rs[p][i] = rr[e] * __expf(L);
                if ((rmask >> p) & 1u) {
                    sm.al[p][i] = __expf(L + ew[e]);
                    sm.ks[p][i] = kk[e];
                    L = 0.f;
                } else {
                    L += ew[e];
                    sm.ks[p][i] = kk[e] * __expf(-L);
                }
            }
        }
        // ---- transform: v (this CTA's columns) and the bonus scalar ----
        for (int e = tid; e < TC * CW; e += NT) {
            const int p = e / CW, j = e % CW;
            const int row = cp.dir > 0 ? p : TC - 1 - p;
            sm.vs[p][j] = to_f32(sm.raw_v[s][row][j]);
        }
        for (int p = warp; p < TC; p += WARPS) {
            const int row = cp.dir > 0 ? p : TC - 1 - p;
            float part = to_f32(sm.raw_r[s][row][lane]) * sm.u[lane] * to_f32(sm.raw_k[s][row][lane]) +
                         to_f32(sm.raw_r[s][row][lane + 32]) * sm.u[lane + 32] *
                             to_f32(sm.raw_k[s][row][lane + 32]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == 0) sm.c[p] = with_bonus ? part : 0.f;
        }
        __syncthreads();
        // the raw stage is consumed: refill it with chunk g + 2
        if (tid == 0 && g + 2 < nchunks) {
            fence_proxy_async_smem();
            issue(g + 2);
        }

        // ---- recurrence over the chunk ----
#pragma unroll 2
        for (int p = 0; p < TC; ++p) {
            const float4 ra = *reinterpret_cast<const float4 *>(&sm.rs[p][rowA]);
            const float4 rb = *reinterpret_cast<const float4 *>(&sm.rs[p][rowB]);
            const float4 ka = *reinterpret_cast<const float4 *>(&sm.ks[p][rowA]);
            const float4 kb = *reinterpret_cast<const float4 *>(&sm.ks[p][rowB]);
            const float4 vv = *reinterpret_cast<const float4 *>(&sm.vs[p][jc]);
            const float2 rr2[4] = {make_float2(ra.x, ra.y), make_float2(ra.z, ra.w), make_float2(rb.x, rb.y),
                                   make_float2(rb.z, rb.w)};
            const float2 kr2[4] = {make_float2(ka.x, ka.y), make_float2(ka.z, ka.w), make_float2(kb.x, kb.y),
                                   make_float2(kb.z, kb.w)};
            const float2 v2[4] = {make_float2(vv.x, vv.x), make_float2(vv.y, vv.y), make_float2(vv.z, vv.z),
                                  make_float2(vv.w, vv.w)};
            float yp[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float2 acc = __ffma2_rn(rr2[0], S2[0][j], kZero2);
#pragma unroll
                for (int qq = 1; qq < 4; ++qq) acc = __ffma2_rn(rr2[qq], S2[qq][j], acc);
                yp[j] = acc.x + acc.y;
            }
            if ((rmask >> p) & 1u) {
                const float4 aa = *reinterpret_cast<const float4 *>(&sm.al[p][rowA]);
                const float4 ab = *reinterpret_cast<const float4 *>(&sm.al[p][rowB]);
                const float2 al2[4] = {make_float2(aa.x, aa.y), make_float2(aa.z, aa.w), make_float2(ab.x, ab.y),
                                       make_float2(ab.z, ab.w)};
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        S2[qq][j] = __ffma2_rn(S2[qq][j], al2[qq], __ffma2_rn(kr2[qq], v2[j], kZero2));
            } else {
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
#pragma unroll
                    for (int j = 0; j < 4; ++j) S2[qq][j] = __ffma2_rn(kr2[qq], v2[j], S2[qq][j]);
            }
            // reduce-scatter the 4 column partials over the 8 row groups (lanes xor 4, 2, 1)
            float k0 = b2 ? yp[2] : yp[0];
            float k1 = b2 ? yp[3] : yp[1];
            const float s0 = b2 ? yp[0] : yp[2];
            const float s1 = b2 ? yp[1] : yp[3];
            k0 += __shfl_xor_sync(0xffffffffu, s0, 4);
            k1 += __shfl_xor_sync(0xffffffffu, s1, 4);
            float kk = b1 ? k1 : k0;
            const float s2 = b1 ? k0 : k1;
            kk += __shfl_xor_sync(0xffffffffu, s2, 2);
            kk += __shfl_xor_sync(0xffffffffu, kk, 1);
            if ((rg & 1) == 0) {
                const float vj = sm.vs[p][jc + jj];
                sm.ybuf[p][jc + jj] = fmaf(sm.c[p], vj, kk);
            }
        }
        __syncthreads();

        // ---- write y for the chunk (float4, coalesced along channels) ----
        constexpr int V4 = CW / 4;
        static_assert((TC * V4) % NT == 0, "y write-out assumes whole rounds of the block");
        constexpr int kRounds = TC * V4 / NT;
        // pass 1 adds the anti-causal part that pass 0 of this CTA stored: all of
        // this thread's loads are issued before its stores, so their latencies overlap
        float4 old[kRounds];
        if (BIDIR && cp.pass == 1) {
#pragma unroll
            for (int m = 0; m < kRounds; ++m) {
                const int e = tid + m * NT, p = e / V4, j4 = (e % V4) * 4;
                const int t = cp.dir > 0 ? cp.t_lo + p : cp.t_lo + TC - 1 - p;
                old[m] = (t >= 0 && t < T)
                             ? *reinterpret_cast<const float4 *>(prm.y + ((size_t)b * T + t) * C + cbase + col0 + j4)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        // norm/gate epilogue on the finished y (the causal sweep, or the second pass);
        // the gate loads are issued first so that their latency overlaps the statistics
        const bool epi = prm.gn_w != nullptr && (!BIDIR || cp.pass == 1);
        float4 gate[kRounds];
        if (epi) {
#pragma unroll
            for (int m = 0; m < kRounds; ++m) {
                const int e = tid + m * NT, p = e / V4, j4 = (e % V4) * 4;
                const int t = cp.dir > 0 ? cp.t_lo + p : cp.t_lo + TC - 1 - p;
                gate[m] = (t >= 0 && t < T)
                              ? __ldg(reinterpret_cast<const float4 *>(prm.g + ((size_t)b * T + t) * C + cbase +
                                                                       col0 + j4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int m = 0; m < kRounds; ++m) {
            const int e = tid + m * NT, p = e / V4, j4 = (e % V4) * 4;
            const int t = cp.dir > 0 ? cp.t_lo + p : cp.t_lo + TC - 1 - p;
            const bool valid = t >= 0 && t < T;
            float4 val = *reinterpret_cast<const float4 *>(&sm.ybuf[p][j4]);
            if (BIDIR && cp.pass == 1) {
                val.x += old[m].x;
                val.y += old[m].y;
                val.z += old[m].z;
                val.w += old[m].w;
            }
            const size_t off = ((size_t)b * T + t) * C + cbase + col0 + j4;
            if (epi) {
                static_assert(V4 == 16, "a head row is the 16 lanes of a half warp");
                // mean and variance of the head's 64 outputs (two passes, exact order)
                float sm1 = (val.x + val.y) + (val.z + val.w);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) sm1 += __shfl_xor_sync(0xffffffffu, sm1, o);
                const float mu = sm1 * (1.f / kHead);
                const float4 d = make_float4(val.x - mu, val.y - mu, val.z - mu, val.w - mu);
                float q = (d.x * d.x + d.y * d.y) + (d.z * d.z + d.w * d.w);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
                const float rstd = rsqrtf(q * (1.f / kHead) + prm.gn_eps);
                const float4 gg = gate[m];
                val = make_float4(fmaf(d.x * rstd, gnw.x, gnb.x) * gg.x, fmaf(d.y * rstd, gnw.y, gnb.y) * gg.y,
                                  fmaf(d.z * rstd, gnw.z, gnb.z) * gg.z, fmaf(d.w * rstd, gnw.w, gnb.w) * gg.w);
            }
            if (valid && in_range_vec(off, 4, (size_t)prm.B * T * C)) *reinterpret_cast<float4 *>(prm.y + off) = val;
        }
        if (BIDIR && g == nch - 1) __syncthreads();  // pass-0 y stores visible before pass-1 reads
    }
    if (!BIDIR && prm.sT != nullptr) {
        // every chunk ends with a renorm step, so the scaled state is the true
        // state S_{T-1} here (tokens past T were zero-filled: k = 0, ew = 0)
        const size_t nstate = (size_t)prm.B * H * kHead * kHead;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            if (in_range_vec(state_off + (size_t)prow(qq, 0) * kHead, 4, nstate))
                *reinterpret_cast<float4 *>(prm.sT + state_off + (size_t)prow(qq, 0) * kHead) =
                    make_float4(S2[qq][0].x, S2[qq][1].x, S2[qq][2].x, S2[qq][3].x);
            if (in_range_vec(state_off + (size_t)prow(qq, 1) * kHead, 4, nstate))
                *reinterpret_cast<float4 *>(prm.sT + state_off + (size_t)prow(qq, 1) * kHead) =
                    make_float4(S2[qq][0].y, S2[qq][1].y, S2[qq][2].y, S2[qq][3].y);
        }
    }
}

// ------------------------------------------------------------------ launchers

template <typename Tin, int WARPS, int TC, bool BIDIR>
static cudaError_t launch_fwd(const CUtensorMap &mr, const CUtensorMap &mk, const CUtensorMap &mv,
                              const CUtensorMap &mw, const FwdParams &prm, cudaStream_t stream) {
    using Smem = FwdSmem<Tin, WARPS, TC>;
    auto kern = wkv6_fwd_kernel<Tin, WARPS, TC, BIDIR>;
    const size_t smem = sizeof(Smem) + 128;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int groups = kHead / Smem::CW;
    const unsigned grid = (unsigned)(prm.B * prm.H * groups);
    kern<<<grid, 32 * WARPS, smem, stream>>>(mr, mk, mv, mw, prm);
    return cudaGetLastError();
}

cudaError_t wkv6_fwd_launch(bool bf16, bool bidir, const CUtensorMap &mr, const CUtensorMap &mk,
                            const CUtensorMap &mv, const CUtensorMap &mw, const FwdParams &prm,
                            cudaStream_t stream) {
    // Reached only in the library built with WKV_RECURRENCE_PATHS: there the bf16
    // causal forward and the fused fp32 forwards run this kernel (the other fp32
    // forwards run the pipelined recurrence there).
#if WKV_RECURRENCE_PATHS
    constexpr int TC = kFwdTC;
    if (bf16) return bidir ? cudaErrorNotSupported : launch_fwd<__nv_bfloat16, 4, TC, false>(mr, mk, mv, mw, prm, stream);
    if (bidir) return launch_fwd<float, 4, TC, true>(mr, mk, mv, mw, prm, stream);
    return launch_fwd<float, 4, TC, false>(mr, mk, mv, mw, prm, stream);
#else
    (void)bf16;
    (void)bidir;
    (void)mr;
    (void)mk;
    (void)mv;
    (void)mw;
    (void)prm;
    (void)stream;
    return cudaErrorNotSupported;
#endif
}

}  // namespace wkv
