// wkv_launch.cuh -- kernel parameter blocks and launcher prototypes (internal to libwkv.so).
#pragma once

#include "wkv_common.cuh"

namespace wkv {

struct FwdParams {
    int B, T, C, H;
    const float *u;
    float *y;
    // causal recurrence only: initial state S_{-1} and final state S_{T-1},
    // [B][H][N][N] (row i = key channel, column j = value channel); null = none
    const float *s0 = nullptr;
    float *sT = nullptr;
    // RWKV-5 static decay rate w5[C] >= 0 (log-decay -w5 at every token); when set
    // the w tensor map is not read
    const float *w5 = nullptr;
    // fp32 kernels (recurrence and tensor-core).  Decay prologue: when wb (w_base [C]) is set, the
    // w map holds ww [B][T][C] and the log-decay is ew = -exp(wb + ww).  Norm/gate
    // epilogue: when gn_w is set, y receives (GroupNorm_head(y) * gn_w + gn_b) * g,
    // with g [B][T][C], gn_w and gn_b [C] and the variance offset gn_eps.
    const float *wb = nullptr;
    const float *g = nullptr, *gn_w = nullptr, *gn_b = nullptr;
    float gn_eps = 0.f;
};

struct BwdParams {
    int B, T, C, H;
    const float *u;
    float *dr, *dk, *dv, *dw;
    float *du_part;   // [B][C] per-batch du partials (caller's workspace)
    // RWKV-5 (tensor-core backward only): static decay rate w5[C] >= 0, the log-decay
    // -w5 at every token (the w pointer is not read), and dw is not written: the
    // kernels add each token's decay gradient into w5_part[2][B][C] (S kind, G kind)
    const float *w5 = nullptr;
    double *w5_part = nullptr;
};

constexpr int kFwdTC = 16;   // tokens per TMA chunk, forward recurrence kernels
constexpr int kBwdTC = 8;    // tokens per TMA chunk, backward kernel

cudaError_t wkv6_fwd_launch(bool bf16, bool bidir, const CUtensorMap &mr, const CUtensorMap &mk,
                            const CUtensorMap &mv, const CUtensorMap &mw, const FwdParams &prm,
                            cudaStream_t stream);
// my: fp32 y map, box 32 channels x 64 tokens, 128-byte swizzle (TMA stores).
cudaError_t wkv6_fwd_tc_launch(const CUtensorMap &mr, const CUtensorMap &mk, const CUtensorMap &mv,
                               const CUtensorMap &mw, const CUtensorMap &my, const FwdParams &prm,
                               cudaStream_t stream);
// fp32 causal or bidirectional forward on the tensor cores (split-bf16 operands);
// r, k, v, w are [B][T][C] fp32 device pointers, 8-byte aligned.  Causal and not
// fused: prm.s0 / prm.sT, when set, are the initial and final states; prm.w5, when
// set, is the static decay rate [C] (w is then not read).
cudaError_t wkv6_fwd_split_launch(bool bidir, const float *r, const float *k, const float *v, const float *w,
                                  const FwdParams &prm, cudaStream_t stream);
// fp32 causal or bidirectional forward for short sequences and few heads: one
// thread-block cluster per (b, h), one chunk per CTA, the chunk states exchanged
// through distributed shared memory.  fits: whether (B, T, H) is such a problem for
// the causal or the bidirectional form.
bool wkv6_fwd_cluster_fits(int B, int T, int H, bool bidir);
cudaError_t wkv6_fwd_cluster_launch(bool bidir, const float *r, const float *k, const float *v, const float *w,
                                    const FwdParams &prm, cudaStream_t stream);
// fp32 causal or bidirectional forward as a register recurrence: four warps hold a
// head's state, a fifth stages and transforms the inputs (maps: fp32, box 64
// channels x kFwdTC tokens); supports s0/sT (causal) and w5, not the fused forms.
cudaError_t wkv6_fwd_pipe_launch(bool bidir, const CUtensorMap &mr, const CUtensorMap &mk, const CUtensorMap &mv,
                                 const CUtensorMap &mw, const FwdParams &prm, cudaStream_t stream);
// One recurrent step for B sequences (state [B][H][N][N] updated in place).
cudaError_t wkv6_decode_launch(int B, int C, int H, const float *r, const float *k, const float *v,
                               const float *w, const float *u, float *state, float *y, cudaStream_t stream);
// maps: kBwdMaps tensor maps, in the order r, k, w, v, dy, dr, dk, dv, dw
constexpr int kBwdMaps = 9;
// bf16: r, k, w, v, dy are bf16 (their maps describe bf16 tensors); gradients stay fp32
cudaError_t wkv6_bwd_launch(bool bf16, bool bidir, const CUtensorMap *maps, const BwdParams &prm, float *du,
                            cudaStream_t stream);
// du[c] = sum_b part[b][c] in increasing b.
cudaError_t wkv6_du_reduce_launch(int B, int C, const float *part, float *du, cudaStream_t stream);
// Backward on the tensor cores (split-bf16 operands; r, k, v, w, dy fp32 or, bf16,
// bfloat16): an S-kind and a G-kind launch and the du reduction; ztot is B*C floats
// of workspace (per-channel z totals).
cudaError_t wkv6_bwd_split_launch(bool bf16, bool bidir, const void *r, const void *k, const void *v, const void *w,
                                  const void *dy, const BwdParams &prm, float *ztot, float *du,
                                  cudaStream_t stream);
// RWKV-5 backward on the tensor cores: the causal S- and G-kind kernels with the static
// log-decay -prm.w5, the du reduction, and dw[c] = -sum_b (w5_part[0][b][c] + w5_part[1][b][c]).
cudaError_t wkv5_bwd_split_launch(const float *r, const float *k, const float *v, const float *dy,
                                  const BwdParams &prm, float *ztot, float *du, cudaStream_t stream);
// RWKV-4 backward; workspace: [B][T][C] + 2 [B][C] floats (see wkv4_bwd_workspace_bytes)
// RWKV-5 backward helpers: ew[b][t][c] = -w[c]; dw[c] = -sum_rows dwtok[row][c].
cudaError_t wkv5_expand_launch(int B, int T, int C, const float *w, float *ew, cudaStream_t stream);
// dw[c] = -sum over the rows of dwtok; `part` holds up to rows x C floats of scratch (ceil(rows / 64) x C in practice)
cudaError_t wkv5_dw_reduce_launch(int rows, int C, const float *dwtok, float *part, float *dw, cudaStream_t stream);
cudaError_t wkv4_bwd_launch(int B, int T, int C, const float *k, const float *v, const float *w, const float *u,
                            const float *dy, float *dk, float *dv, float *dw, float *du, float *workspace,
                            cudaStream_t stream);
cudaError_t wkv4_fwd_launch(int B, int T, int C, const float *k, const float *v, const float *w,
                            const float *u, float *y, cudaStream_t stream);

}  // namespace wkv
