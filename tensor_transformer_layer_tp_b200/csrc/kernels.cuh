// Host launchers of the bandwidth-bound kernels and of attention.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tp_common.cuh"

namespace tp {

// ---------------------------------------------------------------- device error words
// Each reads and clears the error word of one translation unit's waiting
// kernels (synchronise first); return a cudaError_t value.
int attention_read_clear_error(unsigned int* value);
int layernorm_read_clear_error(unsigned int* value);
int elementwise_read_clear_error(unsigned int* value);

// ---------------------------------------------------------------- LayerNorm
// y = (x - mean) * rstd * gamma + beta over rows of width h (bf16 in/out),
// biased variance; mean and rstd are saved (fp32, one per row), or, with
// stats_given, read (a forward rebuilt from saved statistics).
int launch_layernorm_fwd(const void* x, const void* gamma, const void* beta, float eps, int rows,
                         int h, void* y, float* mean, float* rstd, cudaStream_t s,
                         bool stats_given = false);

// dx = dres + rstd * (g - mean(g) - xhat * mean(g * xhat)), g = dy * gamma.
// Per-block partial column sums go to `partial` ([planes][blocks][h] fp32,
// layernorm_bwd_blocks() blocks): dy*xhat and dy, and with extra_sums also
// dres and dx (the bias gradients whose inputs these are).  row_sums, when
// given: float2 [row_parts][rows] partial sums of (g, g * xhat) per row (the
// EPI_LN_ROWSTATS epilogue of the GEMM that produced dy), so the kernel does
// not read dy and x for them.
int layernorm_bwd_blocks(int rows);
int launch_layernorm_bwd(const void* dy, const void* x, const void* gamma, const float* mean,
                         const float* rstd, const void* dres, int rows, int h, void* dx,
                         float* partial, bool extra_sums, cudaStream_t s,
                         const void* row_sums = nullptr, int row_parts = 0);

// ---------------------------------------------------------------- column sums
// out[g][j] = bf16( sum_r partial[g][r][j] ), partial is [groups][nrows][n]
// fp32, for up to kMaxSumJobs independent jobs in one launch: finishes the
// dgamma / dbeta and bias gradients of a backward pass together at its end.
constexpr int kMaxSumJobs = 6;
struct SumRowsJob {
  const float* partial;
  int groups, nrows, n;
  void* out[8];
};
int launch_sum_rows_multi(const SumRowsJob* jobs, int njobs, cudaStream_t s);

// ---------------------------------------------------------------- dropout
// Backward of a hidden-output dropout (the site d over [rows, h], h % 8 == 0,
// h <= 4096): out = g * keep * d.scale (bf16; may alias g) and per-block
// column sums of out into partial [dropout_bwd_blocks(rows)][h] fp32.
int dropout_bwd_blocks(int rows);
// out = residual + drop(sum + bias), [rows][h] bf16 (h % 8 == 0): the finish
// of a row-parallel linear whose partition sum was formed outside the library.
int launch_bias_drop_residual(const void* sum, const void* bias, const void* residual, void* out,
                              int rows, int h, const DropSite& d, cudaStream_t s);
int launch_dropout_bwd(const void* g, void* out, int rows, int h, const DropSite& d, float* partial,
                       cudaStream_t s);

// ---------------------------------------------------------------- attention
struct AttnArgs {
  int batch, seq, heads, head_dim, t;   // heads: total; heads/t live in each partition
  int causal;
  const int32_t* valid_len;             // [batch] or null
  // Per partition: fused projection buffer [tokens][3*hp*d] = [Q heads | K heads | V heads].
  const void* qkv[8];
  void* o[8];                           // [tokens][hp*d]
  float* lse;                           // [batch][heads][seq], base 2 of the scaled scores
  // backward only
  const void* d_o[8];                   // [tokens][hp*d]
  void* dqkv[8];                        // [tokens][3*hp*d]
  float* delta;                         // [batch][heads][seq] fp32 scratch
  // Column partials of dQKV_i per 32-row block of each sequence (the bias
  // gradient db_qkv,i = their sum): [t][batch * ceil(seq/32)][3*hp*d] fp32.
  float* colsum;
  // fp32 dQ accumulator, per partition [tokens][hp*d] back to back (head
  // dims up to 96 accumulate dQ here from every key tile).
  float* dq_acc;
  // Dropout of the attention probabilities (thresh 0: none); rows are
  // (batch * heads_total + head0 + head) * seq + query, columns keys, where
  // head counts the heads of this call and head0 / heads_total place them in
  // the whole layer (a rank-local call holds one partition's heads).
  DropSite drop;
  int head0;         // global index of this call's first head (0: the whole layer)
  int heads_total;   // heads of the whole layer (0: heads)
};
// Forward (tcgen05): O and lse.
int launch_attention_fwd_tc(const AttnArgs& a, cudaStream_t s);
// Backward (tcgen05).  Head dims up to 96: delta = rowsum(dO * O) (and a zeroed
// dQ accumulator), one fused kernel per key tile for dK, dV and the dQ
// partials, and a dQ conversion.  Head dim 128: a dQ kernel (also computes
// delta) and a dK/dV kernel.
int launch_attention_bwd_tc(const AttnArgs& a, cudaStream_t s);
int attention_bwd_launches(int head_dim);

// ---------------------------------------------------------------- loss
// Per (partition, token) statistics of fp32 logits z_i [T][Vp]:
// stats[0][i][n] = max_v z, stats[1][i][n] = sum_v exp(z - max),
// stats[2][i][n] = z[target - i*Vp] if the target lies in partition i else 0.
int launch_xent_stats(int t, int tokens, int vp, const float* const* logits, const int32_t* target,
                      float* stats, cudaStream_t s);
// Combine the t triples: lse[n], loss_tok[n] = lse - z_target, loss = mean.
// `lse` must hold tokens + ceil(tokens / 256) floats (the tail keeps block sums).
int launch_xent_combine(int t, int tokens, const float* stats, float* lse, float* loss_tok,
                        float* loss, cudaStream_t s);
// dz_i = (exp(z_i - lse) - onehot) / T  (bf16 out)
int launch_xent_grad(int t, int tokens, int vp, const float* const* logits, const int32_t* target,
                     const float* lse, void* const* dlogits, cudaStream_t s);

// Fused path.  tile_stats [t][ntiles][tokens] float2 = (max, sum 2^(x - max))
// of x = z log2(e) per 256-column logits tile (the logits GEMM's EPI_XENT
// epilogue), ztgt [tokens] the target logits: lse, loss_tok, loss as
// launch_xent_combine (lse holds tokens + ceil(tokens / 8) floats).
int launch_xent_tile_combine(int t, int tokens, int ntiles, int vocab, const float2* tile_stats,
                             const float* ztgt, const int32_t* target, float* lse, float* loss_tok,
                             float* loss, cudaStream_t s);
// dz_i = (exp(z_i - lse) - onehot) / T from bf16 logits z_i [T][vp], written
// over them in bf16; logits[i] is vocab partition i + group0.
int launch_xent_grad_bf16(int t, int tokens, int vp, void* const* logits, const int32_t* target,
                          const float* lse, cudaStream_t s, int group0 = 0);
// Loss across devices, one vocab partition per call (comm [3][tokens] fp32,
// the values the caller reduces over ranks):
//   fold:   lse_loc = lse over the slice (from the tile statistics), comm[0] =
//           lse_loc, comm[2] = the target logit or 0
//   exp:    comm[1] = exp(lse_loc - comm[0])         (comm[0] = max over ranks)
//   finish: lse = comm[0] + log comm[1], loss_tok = lse - comm[2], loss = mean
//           (comm[1], comm[2] = sums over ranks; lse holds tokens +
//           ceil(tokens / 8) floats)
int launch_xent_rank_fold(int tokens, int ntiles, const float2* tile_stats, const float* ztgt,
                          float* lse_loc, float* comm, cudaStream_t s);
int launch_xent_rank_exp(int tokens, const float* lse_loc, float* comm, cudaStream_t s);
int launch_xent_rank_finish(int tokens, const float* comm, float* lse, float* loss_tok, float* loss,
                            cudaStream_t s);

}  // namespace tp
