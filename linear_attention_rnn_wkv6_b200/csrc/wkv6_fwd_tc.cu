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
// Q_p = r_p * exp(Lam_p) and Kt_s = k_s * exp(-Lam_{s+1}):
//   y_p   = Q_p S_in + sum_{s<p} (Q_p . Kt_s) v_s + c_p v_p        (c_p = sum_i r u k)
//   S_out = diag(exp(Lam_L)) (S_in + Kt^T V)
//   M1  A  = Q Kt^T                       (TMEM cols [0,64))
//   M2  Y  = Q S_in + tril_strict(A) V     (TMEM cols [64,128))
//   M3  S += Kt^T V                        (TMEM cols [128,192)), then rows scaled by exp(Lam_L)
// Every operand is staged K-major (the contraction index contiguous): TF32
// operands in the transposed (MN-major) form produce no result on this
// hardware, so Kt is kept in two layouts and V and S_in are stored transposed.
// |Lam| <= 80 keeps exp(-Lam) inside fp32.  A chunk whose cumulative decay
// leaves that range (fast-forgetting channels) is evaluated instead by the
// exact token-by-token recurrence on the CUDA cores, starting from the state
// held in TMEM, so any decay value down to exactly 0 stays exact.
//
// One CTA (128 threads) per (b, h); thread 0 issues the MMAs; all threads do
// the decay transform and the TMEM epilogues.  Inputs arrive by TMA with the
// 128-byte swizzle (bank-conflict-free column reads of the bf16 tiles).
#include "wkv_launch.cuh"
#include "wkv_tc.cuh"

namespace wkv {

namespace {

constexpr int kL = 64;                 // tokens per chunk
constexpr float kLamMax = 80.0f;       // |Lam| bound of the tensor-core path
constexpr int kLamPad = kHead + 4;     // padded row of the Lam table (bank spread)

struct TcSmem {
    __nv_bfloat16 raw[2][4][kL][kHead];   // r, k, v, w stages (TMA, 128B-swizzled), 64 KB
    float Qs[16][kL][4];                  // Q    : unit over i, row p   (A of M1, M2)
    float Ks[16][kL][4];                  // Kt   : unit over i, row s   (B of M1)
    float KT[16][kHead][4];               // Kt^T : unit over s, row i   (A of M3)
    float VT[16][kHead][4];               // V^T  : unit over s, row j   (B of M2, M3)
    float As[16][kL][4];                  // A    : unit over s, row p, masked (A of M2)
    float ST[16][kHead][4];               // S_in^T: unit over i, row j  (B of M2)
    float lam[kL + 1][kLamPad];           // exclusive cumulative log-decay, rows p = 0..64
    float dec[kHead];                     // exp(Lam_L)
    float c[kL];                          // bonus scalars
    float u[kHead];
    uint32_t tmem_base;
    int flag;
    alignas(8) uint64_t full[2];
    alignas(8) uint64_t mma_bar;
};

enum { R_ = 0, K_ = 1, V_ = 2, W_ = 3 };

// Element (row, col) of a 64 x 64 bf16 tile written by TMA with the 128-byte swizzle.
__device__ __forceinline__ float raw_at(const __nv_bfloat16 (&t)[kL][kHead], int row, int col) {
    const int chunk = (col >> 3) ^ (row & 7);
    return __bfloat162float(t[row][chunk * 8 + (col & 7)]);
}

}  // namespace

__global__ void __launch_bounds__(128, 1)
wkv6_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_r, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_w,
                   FwdParams prm) {
    extern __shared__ unsigned char smem_dyn[];
    TcSmem &sm = *reinterpret_cast<TcSmem *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = prm.T, C = prm.C, H = prm.H;
    const int h = blockIdx.x % H, b = blockIdx.x / H;
    const int cbase = h * kHead;
    const int nch = (T + kL - 1) / kL;
    constexpr uint32_t kStageBytes = 4u * kL * kHead * sizeof(__nv_bfloat16);

    if (tid < kHead) sm.u[tid] = prm.u[cbase + tid];
    if (tid == 0) {
        prefetch_tensormap(&map_r);
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
        prefetch_tensormap(&map_w);
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        mbar_init(&sm.mma_bar, 1);
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
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;   // this warp's TMEM lane quarter

    auto issue = [&](int c) {
        const int s = c & 1;
        mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
        tma_load_3d(&sm.raw[s][R_][0][0], &map_r, cbase, c * kL, b, &sm.full[s]);
        tma_load_3d(&sm.raw[s][K_][0][0], &map_k, cbase, c * kL, b, &sm.full[s]);
        tma_load_3d(&sm.raw[s][V_][0][0], &map_v, cbase, c * kL, b, &sm.full[s]);
        tma_load_3d(&sm.raw[s][W_][0][0], &map_w, cbase, c * kL, b, &sm.full[s]);
    };
    if (tid == 0) {
        issue(0);
        if (nch > 1) issue(1);
    }

    uint32_t mma_phase = 0;
    bool failed = false;
    const int prow = 16 * warp + lane;       // accumulator row of this thread (valid for lane < 16)
    const bool rowlane = lane < 16;
    constexpr uint32_t kIdK_K = tc::idesc_tf32(64, 64, false, false);   // A and B K-major

    for (int c = 0; c < nch; ++c) {
        const int s = c & 1;
        const int t0 = c * kL;
        const bool ok = mbar_wait_bounded(&sm.full[s], (c >> 1) & 1);
        if (!__syncthreads_and(ok)) {
            failed = true;
            drain_two_stage(sm.full, c, nch);
            break;
        }
        // ---- T1: cumulative log-decay per row (threads 0..63), bonus scalars (64..127)
        int bad = 0;
        if (tid < kHead) {
            const int i = tid;
            float L = 0.f, mx = 0.f;
            for (int p = 0; p < kL; ++p) {
                sm.lam[p][i] = L;
                L += raw_at(sm.raw[s][W_], p, i);
                mx = fmaxf(mx, fabsf(L));
            }
            sm.lam[kL][i] = L;
            sm.dec[i] = __expf(L);
            bad = !(mx <= kLamMax);
        } else {
            const int p = tid - kHead;
            float acc = 0.f;
            for (int i = 0; i < kHead; ++i)
                acc = fmaf(raw_at(sm.raw[s][R_], p, i) * sm.u[i], raw_at(sm.raw[s][K_], p, i), acc);
            sm.c[p] = acc;
        }
        const bool flagged = __syncthreads_or(bad) != 0;

        if (!flagged) {
            // ---- T2: Q, Kt, V into the operand tiles (lane -> 8 rows x 4 units per quarter warp)
            for (int e = tid; e < kL * 16; e += 128) {
                const int pl = e & 7, ul = (e >> 3) & 3, blk = e >> 5;     // blk: 32 blocks of 8 rows x 4 units
                const int p = (blk & 7) * 8 + pl;
                const int u4 = (blk >> 3) * 4 + ul;
                const int i0 = 4 * u4;
                float q[4], kt[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    const int i = i0 + e2;
                    q[e2] = raw_at(sm.raw[s][R_], p, i) * __expf(sm.lam[p][i]);
                    kt[e2] = raw_at(sm.raw[s][K_], p, i) * __expf(-sm.lam[p + 1][i]);
                }
                *reinterpret_cast<float4 *>(&sm.Qs[u4][p][0]) = make_float4(q[0], q[1], q[2], q[3]);
                *reinterpret_cast<float4 *>(&sm.Ks[u4][p][0]) = make_float4(kt[0], kt[1], kt[2], kt[3]);
            }
            // transposed tiles: 4 consecutive tokens of one channel per thread
            for (int e = tid; e < kL * 16; e += 128) {
                const int il = e & 7, sl = (e >> 3) & 3, blk = e >> 5;
                const int i = (blk & 7) * 8 + il;
                const int su = (blk >> 3) * 4 + sl;
                float kt[4], vv[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    const int tok = 4 * su + e2;
                    kt[e2] = raw_at(sm.raw[s][K_], tok, i) * __expf(-sm.lam[tok + 1][i]);
                    vv[e2] = raw_at(sm.raw[s][V_], tok, i);
                }
                *reinterpret_cast<float4 *>(&sm.KT[su][i][0]) = make_float4(kt[0], kt[1], kt[2], kt[3]);
                *reinterpret_cast<float4 *>(&sm.VT[su][i][0]) = make_float4(vv[0], vv[1], vv[2], vv[3]);
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            // the raw stage is consumed: refill it
            if (tid == 0 && c + 2 < nch) {
                fence_proxy_async_smem();
                issue(c + 2);
            }
            // ---- M1: A = Q Kt^T
            if (tid == 0) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc::mma_tf32(tA, tc::desc_kmajor(sm.Qs, k), tc::desc_kmajor(sm.Ks, k), kIdK_K, k > 0);
                tc::mma_commit(&sm.mma_bar);
            }
            if (!mbar_wait_bounded(&sm.mma_bar, mma_phase)) failed = true;
            mma_phase ^= 1;
            tc::fence_after_sync();
            // ---- E_A: strictly-lower mask, A -> As (unit over s, row p)
            {
                float a0[32], a1[32];
                tc::tmem_ld32(tA + lane_off, a0);
                tc::tmem_ld32(tA + lane_off + 32, a1);
                tc::tmem_wait_ld();
                if (rowlane) {
#pragma unroll
                    for (int u4 = 0; u4 < 16; ++u4) {
                        float x[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int sc = 4 * u4 + e2;
                            const float val = sc < 32 ? a0[sc] : a1[sc - 32];
                            x[e2] = sc < prow ? val : 0.f;
                        }
                        *reinterpret_cast<float4 *>(&sm.As[u4][prow][0]) = make_float4(x[0], x[1], x[2], x[3]);
                    }
                }
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            // ---- M2: Y = Q S_in + A V;  M3: S += Kt^T V
            if (tid == 0) {
                if (c > 0) {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        tc::mma_tf32(tY, tc::desc_kmajor(sm.Qs, k), tc::desc_kmajor(sm.ST, k), kIdK_K, k > 0);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc::mma_tf32(tY, tc::desc_kmajor(sm.As, k), tc::desc_kmajor(sm.VT, k), kIdK_K, c > 0 || k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc::mma_tf32(tS, tc::desc_kmajor(sm.KT, k), tc::desc_kmajor(sm.VT, k), kIdK_K, c > 0 || k > 0);
                tc::mma_commit(&sm.mma_bar);
            }
            if (!mbar_wait_bounded(&sm.mma_bar, mma_phase)) failed = true;
            mma_phase ^= 1;
            tc::fence_after_sync();
            // ---- E_Y: y = Y + c_p v_p, straight to global
            {
                float y0[32], y1[32];
                tc::tmem_ld32(tY + lane_off, y0);
                tc::tmem_ld32(tY + lane_off + 32, y1);
                tc::tmem_wait_ld();
                const int t = t0 + prow;
                if (rowlane && t < T) {
                    float *dst = prm.y + ((size_t)b * T + t) * C + cbase;
                    const float cp = sm.c[prow];
                    const float *vrow = &sm.VT[prow >> 2][0][prow & 3];   // v_p[j] at vrow[4 * j]
#pragma unroll
                    for (int u4 = 0; u4 < 16; ++u4) {
                        const float *src = u4 < 8 ? &y0[4 * u4] : &y1[4 * (u4 - 8)];
                        *reinterpret_cast<float4 *>(dst + 4 * u4) =
                            make_float4(fmaf(cp, vrow[4 * (4 * u4)], src[0]), fmaf(cp, vrow[4 * (4 * u4 + 1)], src[1]),
                                        fmaf(cp, vrow[4 * (4 * u4 + 2)], src[2]), fmaf(cp, vrow[4 * (4 * u4 + 3)], src[3]));
                    }
                }
            }
            // ---- E_S: S rows scaled by exp(Lam_L); back to TMEM and to Ss for the next chunk
            {
                float s0[32], s1[32];
                tc::tmem_ld32(tS + lane_off, s0);
                tc::tmem_ld32(tS + lane_off + 32, s1);
                tc::tmem_wait_ld();
                const float dsc = rowlane ? sm.dec[prow] : 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    s0[j] *= dsc;
                    s1[j] *= dsc;
                }
                tc::tmem_st32(tS + lane_off, s0);
                tc::tmem_st32(tS + lane_off + 32, s1);
                if (rowlane) {
                    float *dstT = &sm.ST[prow >> 2][0][prow & 3];         // S[i][j] at dstT[4 * j]
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        dstT[4 * j] = s0[j];
                        dstT[4 * (32 + j)] = s1[j];
                    }
                }
                tc::tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
        } else {
            // ---- exact token-by-token fallback on the CUDA cores for this chunk
            // state row i = prow (lane < 16) in registers; y via a shared-memory column sum
            float Sr[64];
            if (c > 0) {
                float s0[32], s1[32];
                tc::tmem_ld32(tS + lane_off, s0);
                tc::tmem_ld32(tS + lane_off + 32, s1);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    Sr[j] = s0[j];
                    Sr[32 + j] = s1[j];
                }
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) Sr[j] = 0.f;
            }
            float (*part)[kHead] = reinterpret_cast<float (*)[kHead]>(&sm.As[0][0][0]);   // [64 rows][64 cols]
            for (int p = 0; p < kL; ++p) {
                if (rowlane) {
                    const float rr = raw_at(sm.raw[s][R_], p, prow);
#pragma unroll
                    for (int j = 0; j < 64; ++j) part[prow][j] = rr * Sr[j];
                }
                __syncthreads();
                if (tid < kHead) {
                    const int j = tid;
                    float acc = 0.f;
                    for (int i = 0; i < kHead; ++i) acc += part[i][j];
                    const int t = t0 + p;
                    if (t < T) prm.y[((size_t)b * T + t) * C + cbase + j] = fmaf(sm.c[p], raw_at(sm.raw[s][V_], p, j), acc);
                }
                if (rowlane) {
                    const float d = __expf(raw_at(sm.raw[s][W_], p, prow));
                    const float kk = raw_at(sm.raw[s][K_], p, prow);
#pragma unroll
                    for (int j = 0; j < 64; ++j) Sr[j] = fmaf(d, Sr[j], kk * raw_at(sm.raw[s][V_], p, j));
                }
                __syncthreads();
            }
            {
                float s0[32], s1[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    s0[j] = Sr[j];
                    s1[j] = Sr[32 + j];
                }
                tc::tmem_st32(tS + lane_off, s0);
                tc::tmem_st32(tS + lane_off + 32, s1);
                if (rowlane) {
                    float *dstT = &sm.ST[prow >> 2][0][prow & 3];
#pragma unroll
                    for (int j = 0; j < 64; ++j) dstT[4 * j] = Sr[j];
                }
                tc::tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            if (tid == 0 && c + 2 < nch) {
                fence_proxy_async_smem();
                issue(c + 2);
            }
        }
        if (failed) break;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}

cudaError_t wkv6_fwd_tc_launch(const CUtensorMap &mr, const CUtensorMap &mk, const CUtensorMap &mv,
                               const CUtensorMap &mw, const FwdParams &prm, cudaStream_t stream) {
    const size_t smem = sizeof(TcSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(wkv6_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    wkv6_fwd_tc_kernel<<<(unsigned)(prm.B * prm.H), 128, smem, stream>>>(mr, mk, mv, mw, prm);
    return cudaGetLastError();
}

}  // namespace wkv
