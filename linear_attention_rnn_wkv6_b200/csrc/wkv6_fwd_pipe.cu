// wkv6_fwd_pipe.cu -- RWKV-6 fp32 forward (causal and bidirectional) as a
// register recurrence fed by a dedicated transform warp (sm_100a).
//
// Operation (per batch b, head h; N = 64; d_t = exp(ew_t)):
//   causal : y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),  S_t = diag(d_t) S_{t-1} + k_t^T v_t
//   bidir  : adds r_t S^b_{t+1} with S^b_t = diag(d_t) S^b_{t+1} + k_t^T v_t (no bonus)
// ("RWKV Architecture ...", RWKV-6 "Finch" dynamic decay; "How Custom CUDA
//  Kernels (wkv6_cuda.cu) ...", Forward Pass Implementation: the Past-to-Future
//  and Future-to-Past passes.)
//
// The arithmetic is 2 FMAs per state element per token (readout and update on
// the scaled state below), 4096 elements per head: at N = 64 the forward is
// bound by the FP32 pipe and by shared-memory delivery of the per-token
// vectors, not by HBM.  The kernel is laid out so that the warps holding the
// state issue little besides those FMAs:
//
// * One CTA per (b, h): four state warps and one transform warp.  State warp w
//   holds value columns [16w, 16w + 16) for all 64 rows; lane (rg = lane & 7,
//   cg = lane >> 3) holds rows {4rg + e, 32 + 4rg + e : e in 0..3} x columns
//   16w + 4cg + {0..3}: 32 fp32 values as 16 packed row pairs, so one
//   fma.rn.f32x2 does two multiply-adds.  Per token a lane reads 20 floats
//   (8 scaled r, 8 scaled k, 4 v; five conflict-free 16-byte loads, the next
//   token's issued before this token's arithmetic), and the readout sums its 8
//   rows in registers and the 8 row groups with 4 shuffles.  Columns are
//   independent, so the four state warps never wait for each other.
// * Scaled state (per run of tokens, L_p = sum of the run's log-decays before
//   token p): S_before(p) = diag(e^{L_p}) S', readout y_p = (r_p e^{L_p}) . S',
//   update S' += (k_p e^{-L_{p+1}}) v_p^T.  A run ends at every stage's last
//   token, where S' <- diag(e^{L_p + ew_p}) S' + k_p v_p^T and L restarts at 0;
//   a stage in which some |ew| exceeds 40/16 (or is NaN) ends a run at every
//   token, which is the plain recurrence.  So |L| <= 40, e^{+-L} stays inside
//   fp32, and any decay down to exactly 0 is handled.
// * The transform warp owns the staging: TMA loads of r, k, w, v in stages of
//   16 tokens (a 4-stage ring), then in place r -> r e^{L_p}, k -> k e^{-L_{p+1}},
//   w -> e^{L_p + ew_p} at run ends, the bonus scalar c_p = sum_i r u k (zero in
//   the anti-causal sweep) and the run ends.  It works one stage ahead of the
//   state warps; three mbarriers per stage (loaded, transformed, consumed)
//   order the roles, and every wait is bounded.
// * y: the lane that ends up holding column j of token t after the readout
//   writes y[t][j] (a warp's 16 such lanes: 64 contiguous bytes per token).
//   The bidirectional form runs the anti-causal sweep first and stores its
//   part; the causal sweep adds its part with one atomic add onto that store
//   (made by the same lane): one addition per element, so the result is the
//   same whatever the timing.
// * The library built with WKV_RECURRENCE_PATHS runs every non-fused fp32 forward
//   here.  RWKV-5 (static decay, FwdParams::w5, wkv5_fwd): the transform warp uses
//   -w5 for every token inside [0, T) and the w tile is not loaded.  Initial and
//   final states (FwdParams::s0, sT, causal only, wkv6_fwd_state): the scaled state
//   equals the true state at every stage boundary.
#include "wkv_launch.cuh"

namespace wkv {

namespace {

constexpr int kPT = 16;                       // tokens per stage
constexpr int kPS = 4;                        // stages in the ring
constexpr int kPStateWarps = 4;               // 16 value columns each
constexpr int kPThreads = 32 * (kPStateWarps + 1);
constexpr float kPRunBound = 40.0f / kPT;     // |ew| above this ends a run
constexpr float kPLog2e = 1.4426950408889634f;
static_assert(kPT == kFwdTC, "the entry points build the r, k, v, w maps with boxes of kFwdTC tokens");

struct alignas(128) PipeStage {
    float r[kPT][kHead];   // raw r, then r e^{L_p}
    float k[kPT][kHead];   // raw k, then k e^{-L_{p+1}} (k at a run end)
    float w[kPT][kHead];   // raw log-decay, then e^{L_p + ew_p} at run ends
    float v[kPT][kHead];
};

struct PipeSmem {
    PipeStage st[kPS];
    float c[kPS][kPT];          // bonus scalar per token (processing order)
    uint32_t runend[kPS];       // bit p: token p ends a run
    float u[kHead];
    float ew5[kHead];           // static log-decay -w5 (RWKV-5)
    alignas(8) uint64_t full[kPS];    // TMA bytes landed
    alignas(8) uint64_t ready[kPS];   // transformed (32 arrivals)
    alignas(8) uint64_t empty[kPS];   // read by the state warps (128 arrivals)
    int abort;
};

__device__ __forceinline__ float ex2a(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Stage g of the CTA's sequence: the anti-causal sweep first when bidirectional.
struct PipePos {
    int dir;    // +1 past->future, -1 future->past
    int t_lo;   // first token of the TMA box (may be < 0)
    int pass;   // 0: anti-causal sweep of the bidirectional form, 1: causal sweep
};

__device__ __forceinline__ PipePos pipe_pos(int g, int nch, int T, bool bidir) {
    PipePos p;
    p.pass = (bidir && g < nch) ? 0 : 1;
    const int c = bidir ? (g % nch) : g;
    p.dir = p.pass == 0 ? -1 : 1;
    p.t_lo = p.dir > 0 ? c * kPT : T - (c + 1) * kPT;
    return p;
}

// The 16 per-lane values v[0..15] summed over the warp; lane l ends with the sum
// for index l >> 1 (both lanes of a pair hold it).  16 shuffles.
__device__ __forceinline__ float transpose_reduce16(float (&v)[kPT], int lane) {
#pragma unroll
    for (int lvl = 0; lvl < 4; ++lvl) {
        const int half = 8 >> lvl;                  // values kept after this level
        const bool hi = (lane >> (4 - lvl)) & 1;    // lane bits 4, 3, 2, 1
#pragma unroll
        for (int q = 0; q < half; ++q) {
            const float keep = hi ? v[q + half] : v[q];
            const float send = hi ? v[q] : v[q + half];
            v[q] = keep + __shfl_xor_sync(0xffffffffu, send, 16 >> lvl);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

template <bool BIDIR>
__global__ void __launch_bounds__(kPThreads, 3)
wkv6_fwd_pipe_kernel(const __grid_constant__ CUtensorMap map_r, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_w,
                     FwdParams prm) {
    // the 128-byte aligned start as an offset into the shared array, so that every
    // access through `sm` stays a shared-memory access (an integer round trip of the
    // pointer would turn them into generic ones)
    extern __shared__ unsigned char smem_dyn[];
    PipeSmem &sm = *reinterpret_cast<PipeSmem *>(smem_dyn + ((128u - (smem_u32(smem_dyn) & 127u)) & 127u));

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int T = prm.T, C = prm.C, H = prm.H;
    const int h = blockIdx.x % H;
    const int b = blockIdx.x / H;
    const int cbase = h * kHead;
    const int nch = (T + kPT - 1) / kPT;
    const int nst = BIDIR ? 2 * nch : nch;
    const bool stat = prm.w5 != nullptr;
    const size_t nBTC = (size_t)prm.B * T * C;

    if (tid < kHead) {
        sm.u[tid] = prm.u[cbase + tid];
        sm.ew5[tid] = stat ? -prm.w5[cbase + tid] : 0.f;
    }
    if (tid == 0) {
        for (int s = 0; s < kPS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.ready[s], 32);
            mbar_init(&sm.empty[s], 32 * kPStateWarps);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kPStateWarps) {
        // ========================= transform warp =========================
        constexpr uint32_t kBox = kPT * kHead * sizeof(float);
        auto issue = [&](int g) {
            const PipePos pp = pipe_pos(g, nch, T, BIDIR);
            PipeStage &S = sm.st[g % kPS];
            uint64_t *bar = &sm.full[g % kPS];
            mbar_arrive_expect_tx(bar, stat ? 3 * kBox : 4 * kBox);
            tma_load_3d(&S.r[0][0], &map_r, cbase, pp.t_lo, b, bar);
            tma_load_3d(&S.k[0][0], &map_k, cbase, pp.t_lo, b, bar);
            tma_load_3d(&S.v[0][0], &map_v, cbase, pp.t_lo, b, bar);
            if (!stat) tma_load_3d(&S.w[0][0], &map_w, cbase, pp.t_lo, b, bar);
        };
        int issued = 0;
        if (lane == 0) {
            prefetch_tensormap(&map_r);
            prefetch_tensormap(&map_k);
            prefetch_tensormap(&map_v);
            prefetch_tensormap(&map_w);
            for (; issued < kPS && issued < nst; ++issued) issue(issued);
        }
        issued = __shfl_sync(0xffffffffu, issued, 0);
        const int i0 = 2 * lane;
        const float2 u2 = make_float2(sm.u[i0], sm.u[i0 + 1]);
        const float2 e5 = make_float2(sm.ew5[i0], sm.ew5[i0 + 1]);
        bool ok = true;
        int g = 0;
        for (; g < nst && ok; ++g) {
            const int s = g % kPS;
            const PipePos pp = pipe_pos(g, nch, T, BIDIR);
            ok = mbar_wait_bounded(&sm.full[s], (g / kPS) & 1) && !*(volatile int *)&sm.abort;
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            PipeStage &S = sm.st[s];
            auto row_of = [&](int p) { return pp.dir > 0 ? p : kPT - 1 - p; };
            // the stage's log-decays (log2 units); a stage with any |ew| above the
            // bound (or NaN) ends a run at every token: the plain recurrence
            float2 e2[kPT];
            bool big = false;
#pragma unroll
            for (int p = 0; p < kPT; ++p) {
                const int row = row_of(p);
                float2 ew;
                if (stat) {
                    const int t = pp.t_lo + row;
                    ew = (t >= 0 && t < T) ? e5 : make_float2(0.f, 0.f);
                } else {
                    ew = *reinterpret_cast<const float2 *>(&S.w[row][i0]);
                }
                big |= !(fabsf(ew.x) <= kPRunBound) || !(fabsf(ew.y) <= kPRunBound);
                e2[p] = make_float2(ew.x * kPLog2e, ew.y * kPLog2e);
            }
            const uint32_t runend = __any_sync(0xffffffffu, big) ? 0xffffu : 1u << (kPT - 1);
            // scaled r and k, decay factors at run ends, bonus partials
            float L0 = 0.f, L1 = 0.f;
            float bon[kPT];
#pragma unroll
            for (int p = 0; p < kPT; ++p) {
                const int row = row_of(p);
                const float2 r2 = *reinterpret_cast<const float2 *>(&S.r[row][i0]);
                const float2 k2 = *reinterpret_cast<const float2 *>(&S.k[row][i0]);
                bon[p] = fmaf(r2.x * u2.x, k2.x, r2.y * u2.y * k2.y);
                *reinterpret_cast<float2 *>(&S.r[row][i0]) = make_float2(r2.x * ex2a(L0), r2.y * ex2a(L1));
                if ((runend >> p) & 1u) {
                    *reinterpret_cast<float2 *>(&S.w[row][i0]) = make_float2(ex2a(L0 + e2[p].x), ex2a(L1 + e2[p].y));
                    L0 = 0.f;
                    L1 = 0.f;
                    // k stays as loaded
                } else {
                    L0 += e2[p].x;
                    L1 += e2[p].y;
                    *reinterpret_cast<float2 *>(&S.k[row][i0]) = make_float2(k2.x * ex2a(-L0), k2.y * ex2a(-L1));
                }
            }
            const float csum = transpose_reduce16(bon, lane);
            if ((lane & 1) == 0) sm.c[s][lane >> 1] = pp.pass == 1 ? csum : 0.f;
            if (lane == 0) sm.runend[s] = runend;
            mbar_arrive(&sm.ready[s]);   // every lane: its stores are released with its arrival
            // refill the stage the state warps finished last
            if (g >= 1 && issued < nst) {
                const int gp = g - 1;
                ok = mbar_wait_bounded(&sm.empty[gp % kPS], (gp / kPS) & 1);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                if (lane == 0) issue(issued);
                ++issued;
            }
        }
        if (!ok) {
            // a wait ran out: stop the state warps and let the loads in flight land
            // before the CTA's shared memory goes away
            *(volatile int *)&sm.abort = 1;
            if (lane == 0)
                for (int g2 = g; g2 < issued; ++g2) mbar_wait_bounded(&sm.full[g2 % kPS], (g2 / kPS) & 1);
        }
        return;
    }

    // ============================ state warps ============================
    // lane (rg = lane & 7, cg = lane >> 3): rows {4rg + e, 32 + 4rg + e : e in 0..3}
    // (packed pairs qq: (4rg, 4rg+1), (4rg+2, 4rg+3), (32+4rg, ..), (34+4rg, ..)) x
    // columns jc + j, j in 0..3, with jc = 16 warp + 4 cg
    const int rg = lane & 7, cg = lane >> 3;
    const int jc = 16 * warp + 4 * cg;
    const int jj = (rg >> 1) & 3;           // the column (of the lane's 4) it holds after the readout
    const bool b2 = (rg & 4) != 0, b1 = (rg & 2) != 0;
    const bool writer = (rg & 1) == 0;
    constexpr float2 kZ2 = {0.f, 0.f};
    float2 S2[4][4];
#pragma unroll
    for (int qq = 0; qq < 4; ++qq)
#pragma unroll
        for (int j = 0; j < 4; ++j) S2[qq][j] = kZ2;
    auto prow = [&](int qq, int e) { return (qq < 2 ? 4 * rg + 2 * qq : 32 + 4 * rg + 2 * (qq - 2)) + e; };
    const size_t state_off = ((size_t)b * H + h) * kHead * kHead + jc;
    if (!BIDIR && prm.s0 != nullptr) {
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
    const size_t ycol = (size_t)cbase + jc + jj;

    // readout of S' with the scaled r of one token (4 column partials over this
    // lane's 8 rows), then the update, or at a run end (alrow >= 0) the update with
    // the row's decay factors
    auto step = [&](const float4 &ra, const float4 &rb, const float4 &ka, const float4 &kb, const float4 &vv,
                    const PipeStage &S, int alrow, float (&yp)[4]) {
        const float2 rr2[4] = {make_float2(ra.x, ra.y), make_float2(ra.z, ra.w), make_float2(rb.x, rb.y),
                               make_float2(rb.z, rb.w)};
        const float2 kr2[4] = {make_float2(ka.x, ka.y), make_float2(ka.z, ka.w), make_float2(kb.x, kb.y),
                               make_float2(kb.z, kb.w)};
        const float2 v2[4] = {make_float2(vv.x, vv.x), make_float2(vv.y, vv.y), make_float2(vv.z, vv.z),
                              make_float2(vv.w, vv.w)};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float2 acc = __ffma2_rn(rr2[0], S2[0][j], kZ2);
#pragma unroll
            for (int qq = 1; qq < 4; ++qq) acc = __ffma2_rn(rr2[qq], S2[qq][j], acc);
            yp[j] = acc.x + acc.y;
        }
        if (alrow >= 0) {
            const float4 aa = *reinterpret_cast<const float4 *>(&S.w[alrow][4 * rg]);
            const float4 ab = *reinterpret_cast<const float4 *>(&S.w[alrow][32 + 4 * rg]);
            const float2 al2[4] = {make_float2(aa.x, aa.y), make_float2(aa.z, aa.w), make_float2(ab.x, ab.y),
                                   make_float2(ab.z, ab.w)};
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
#pragma unroll
                for (int j = 0; j < 4; ++j) S2[qq][j] = __ffma2_rn(S2[qq][j], al2[qq], __fmul2_rn(kr2[qq], v2[j]));
        } else {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
#pragma unroll
                for (int j = 0; j < 4; ++j) S2[qq][j] = __ffma2_rn(kr2[qq], v2[j], S2[qq][j]);
        }
    };
    // sum the 4 column partials over the 8 row groups (reduce-scatter over lanes xor
    // 4, 2, 1) and add the bonus: y of column jc + jj
    auto reduce = [&](const float (&yp)[4], float vj, float cp) -> float {
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
        return fmaf(cp, vj, kk);
    };
    auto vsel = [&](const float4 &vv) { return jj == 0 ? vv.x : jj == 1 ? vv.y : jj == 2 ? vv.z : vv.w; };

    for (int g = 0; g < nst; ++g) {
        const int s = g % kPS;
        const PipePos pp = pipe_pos(g, nch, T, BIDIR);
        if (BIDIR && g == nch) {   // the causal sweep starts from the empty state
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
#pragma unroll
                for (int j = 0; j < 4; ++j) S2[qq][j] = kZ2;
        }
        bool ok = mbar_wait_bounded(&sm.ready[s], (g / kPS) & 1) && !*(volatile int *)&sm.abort;
        if (!__all_sync(0xffffffffu, ok)) {
            *(volatile int *)&sm.abort = 1;
            return;
        }
        const PipeStage &S = sm.st[s];
        const uint32_t runend = sm.runend[s];
        const bool add = BIDIR && pp.pass == 1;
        // y: a plain store, or (causal sweep of the bidirectional form) one atomic add
        // onto this lane's own anti-causal store: a single add, so the result does not
        // depend on timing.  Predicated, so that the unrolled token loop stays one block.
        auto put = [&](int p, float yv) {
            const int t = pp.dir > 0 ? pp.t_lo + p : pp.t_lo + kPT - 1 - p;
            const size_t off = ((size_t)b * T + (t >= 0 && t < T ? t : 0)) * C + ycol;
            const uint32_t on = writer && t >= 0 && t < T && in_range(off, nBTC);
            float *dst = prm.y + off;
            if (add)
                asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q red.global.add.f32 [%0], %1;\n\t}"
                             ::"l"(dst), "f"(yv), "r"(on));
            else
                asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.global.f32 [%0], %1;\n\t}"
                             ::"l"(dst), "f"(yv), "r"(on));
        };
        auto row_of = [&](int p) { return pp.dir > 0 ? p : kPT - 1 - p; };
        auto load = [&](int p, float4 &xa, float4 &xb, float4 &ya, float4 &yb, float4 &xv) {
            const int row = row_of(p);
            xa = *reinterpret_cast<const float4 *>(&S.r[row][4 * rg]);
            xb = *reinterpret_cast<const float4 *>(&S.r[row][32 + 4 * rg]);
            ya = *reinterpret_cast<const float4 *>(&S.k[row][4 * rg]);
            yb = *reinterpret_cast<const float4 *>(&S.k[row][32 + 4 * rg]);
            xv = *reinterpret_cast<const float4 *>(&S.v[row][jc]);
        };
        if (runend == 1u << (kPT - 1)) {
            // one run per stage.  Software pipelined: token p + 1's operands are loaded
            // and token p - 1's row-group sum and store run while token p computes.
            float4 ra, rb, ka, kb, vv;
            load(0, ra, rb, ka, kb, vv);
            float ypv[4], vjv = 0.f;
#pragma unroll
            for (int p = 0; p < kPT; ++p) {
                float4 nra, nrb, nka, nkb, nvv;
                if (p + 1 < kPT) load(p + 1, nra, nrb, nka, nkb, nvv);
                float ypc[4];
                step(ra, rb, ka, kb, vv, S, p == kPT - 1 ? row_of(p) : -1, ypc);
                if (p > 0) put(p - 1, reduce(ypv, vjv, sm.c[s][p - 1]));
#pragma unroll
                for (int j = 0; j < 4; ++j) ypv[j] = ypc[j];
                vjv = vsel(vv);
                if (p + 1 < kPT) {
                    ra = nra;
                    rb = nrb;
                    ka = nka;
                    kb = nkb;
                    vv = nvv;
                }
            }
            put(kPT - 1, reduce(ypv, vjv, sm.c[s][kPT - 1]));
        } else {
            // every token ends a run (a stage with a large or non-finite log-decay)
#pragma unroll 1
            for (int p = 0; p < kPT; ++p) {
                float4 ra, rb, ka, kb, vv;
                load(p, ra, rb, ka, kb, vv);
                float yp[4];
                step(ra, rb, ka, kb, vv, S, row_of(p), yp);
                put(p, reduce(yp, vsel(vv), sm.c[s][p]));
            }
        }
        mbar_arrive(&sm.empty[s]);
    }
    if (!BIDIR && prm.sT != nullptr) {
        // the last token of every stage ends a run: S' is the true state S_{T-1}
        // (tokens past T were zero filled: k = v = 0 and ew = 0)
        const size_t nstate = (size_t)prm.B * H * kHead * kHead;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const size_t o0 = state_off + (size_t)prow(qq, 0) * kHead, o1 = state_off + (size_t)prow(qq, 1) * kHead;
            if (in_range_vec(o0, 4, nstate))
                *reinterpret_cast<float4 *>(prm.sT + o0) =
                    make_float4(S2[qq][0].x, S2[qq][1].x, S2[qq][2].x, S2[qq][3].x);
            if (in_range_vec(o1, 4, nstate))
                *reinterpret_cast<float4 *>(prm.sT + o1) =
                    make_float4(S2[qq][0].y, S2[qq][1].y, S2[qq][2].y, S2[qq][3].y);
        }
    }
}

}  // namespace

cudaError_t wkv6_fwd_pipe_launch(bool bidir, const CUtensorMap &mr, const CUtensorMap &mk, const CUtensorMap &mv,
                                 const CUtensorMap &mw, const FwdParams &prm, cudaStream_t stream) {
    if (bidir && (prm.s0 != nullptr || prm.sT != nullptr)) return cudaErrorInvalidValue;
    if (prm.wb != nullptr || prm.gn_w != nullptr) return cudaErrorInvalidValue;
    const size_t smem = sizeof(PipeSmem) + 128;
    auto kern = bidir ? wkv6_fwd_pipe_kernel<true> : wkv6_fwd_pipe_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(prm.B * prm.H), kPThreads, smem, stream>>>(mr, mk, mv, mw, prm);
    return cudaGetLastError();
}

}  // namespace wkv
