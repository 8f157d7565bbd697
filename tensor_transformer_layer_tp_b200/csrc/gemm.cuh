// Grouped / partition-summed bf16 GEMM on the sm_100a tensor cores.
//
// One launch computes, for t logical tensor-parallel partitions g = 0..t-1,
//   grouped mode : C_g = A_g . B_g                 (column-parallel linear: every
//                                                  partition owns its own output)
//   summed  mode : C   = sum_g A_g . B_g           (row-parallel linear followed by
//                                                  the all-reduce; the sum runs in
//                                                  the K-loop, in one fp32 TMEM
//                                                  accumulator, so no partial is
//                                                  ever written to HBM)
// with fused epilogues (bias, GeLU, residual, GeLU derivative).  This is the
// ColumnParallelLinear / RowParallelLinear pair of the Megatron-LM ParallelMLP
// (rkmt.cn guide, section 3.1; Megatron-LM show notes, the MLP split outline
// item) and the same split applied to Q/K/V and the attention output
// projection (section 3.2).
#pragma once

#include "tp_common.cuh"

namespace tp {

constexpr int kMaxGroups = 8;

enum Epilogue : int {
  EPI_BF16 = 0,       // C = bf16(acc)
  EPI_F32 = 1,        // C = acc
  EPI_BIAS_BF16 = 2,  // C_g = bf16(acc + bias_g[n])
  // C_g = bf16(gelu'(U)), C2_g = bf16(gelu(U)), U = acc + bias_g[n]: the
  // activation and the derivative the backward needs, from one CDF / PDF
  EPI_BIAS_GELU = 3,
  // C = bf16(aux[m, n] + drop(acc + bias[n]))  (aux = residual stream; drop =
  // the hidden-output dropout of the `drop` site, identity when it is off)
  EPI_BIAS_RES = 4,
  EPI_DGELU = 5,      // C_g = bf16(acc * aux_g[m, n])             (aux = saved gelu'(U))
  // Vocab-parallel loss statistics of a logits tile (acc = z, group g = vocab
  // partition g + xent_group0): per (row m, column tile nt) the max x of
  // x = z log2(e) over the tile's columns and sum 2^(x - max), into
  // xent_stats[g][nt][m]; the target's logit z[m, target[m] - (g +
  // xent_group0) N] into xent_ztgt[m] by the one tile that holds it; and,
  // when out[g] is given, bf16(z) into C_g.
  EPI_XENT = 6,
  // C = bf16(acc), and the LayerNorm-backward row sums of the rounded output
  // dy against the LayerNorm's input x (aux), gain gamma (bias[0]) and saved
  // row statistics: per (column tile nt, row m), sum_n dy g and
  // sum_n dy g (x - mean) rstd over the tile's columns, into
  // ln_rows[nt][m].  For a partition-summed GEMM (one output).
  EPI_LN_ROWSTATS = 7,
};

struct GemmMaps {
  CUtensorMap a[kMaxGroups];
  CUtensorMap b[kMaxGroups];
  // Output tensor maps (out, out2) for the epilogue's tensor stores
  // (GemmParams::tma_out): the groups' outputs stacked as [groups * M] rows,
  // box 32 columns x 32 rows, swizzled to the row width (64 bytes for bf16,
  // 128 bytes for fp32).  Two maps rather than one per group keep the kernel
  // parameters under 4 KB (above that every launch took a few microseconds
  // longer).
  CUtensorMap c;
  CUtensorMap c2;
};

struct GemmParams {
  int groups;
  int sum_groups;
  // concat = 1: the groups share A and their N ranges are tiled as one
  //             [M, groups*N] problem; concat = 2: the groups share B and
  //             their M ranges are tiled as one [groups*M, N] problem.
  int concat;
  int M, N, K;      // per group
  int Mv, Nv;       // extents the tiles cover (groups*M or groups*N when concatenated)
  int m_tiles, n_tiles, k_blocks;
  int band_w;       // concat = 1: column tiles per band of the tile order
  int tiles_per_group;
  int total_tiles;
  int epi;
  int tma_out;      // 1: outputs staged in shared memory and written by tensor stores
  long long ldc;    // output row stride (elements)
  long long ldaux;  // aux row stride (elements)
  float* colsum;    // optional: per-32-row column partials of the output, [g][ceil(M/32)][N]
  void* out[kMaxGroups];
  void* out2[kMaxGroups];
  const void* bias[kMaxGroups];
  const void* aux[kMaxGroups];
  const int32_t* xent_target;   // EPI_XENT: [M] target ids over the whole vocabulary
  float2* xent_stats;           // EPI_XENT: [groups][n_tiles][M] (max, sum), log2 units
  float* xent_ztgt;             // EPI_XENT: [M] target logit
  int xent_group0;              // EPI_XENT: vocab partition index of group 0
  DropSite drop;                // EPI_BIAS_RES: dropout of (acc + bias), rows = m, cols = n
  const float* ln_mean;         // EPI_LN_ROWSTATS: [M] saved mean and rstd of the LayerNorm
  const float* ln_rstd;
  float2* ln_rows;              // EPI_LN_ROWSTATS: [n_tiles][M] row sums
};


// Host-side description of one GEMM call.
struct GemmDesc {
  int groups = 1;
  int sum_groups = 0;
  int M = 0, N = 0, K = 0;
  // A is [M, K]; a_mn = false: stored row-major [M][K] (K contiguous),
  //                a_mn = true : stored as [K][M] (M contiguous).
  bool a_mn = false;
  // B is [K, N]; b_mn = false: stored as [N][K] (K contiguous),
  //                b_mn = true : stored row-major [K][N] (N contiguous).
  bool b_mn = false;
  const void* a[kMaxGroups] = {};
  const void* b[kMaxGroups] = {};
  long long lda = 0, ldb = 0;   // row strides of the stored matrices (elements)
  int epi = EPI_BF16;
  void* out[kMaxGroups] = {};
  void* out2[kMaxGroups] = {};
  const void* bias[kMaxGroups] = {};
  const void* aux[kMaxGroups] = {};
  long long ldc = 0, ldaux = 0;
  // Optional: column sums of the fp32 output values (before rounding) written
  // as partials per 32-row block, colsum[g][ceil(M/32)][N] (a bias gradient
  // folded into the producing GEMM; finish with a sum over the row blocks).
  float* colsum = nullptr;
  // EPI_XENT outputs (see Epilogue); out[g] may be null (statistics only).
  // The call is tiled per group (no concatenation) so that every column tile
  // lies in one vocab partition; xent_stats holds ceil(N / tile width) tiles
  // per group (gemm_pick_bn, or force_bn).
  const int32_t* xent_target = nullptr;
  float2* xent_stats = nullptr;
  float* xent_ztgt = nullptr;
  int xent_group0 = 0;   // vocab partition of group 0 (a rank-local call: its rank)
  DropSite drop = {};   // EPI_BIAS_RES dropout (thresh 0: none)
  // EPI_LN_ROWSTATS: aux[0] = the LayerNorm input, bias[0] = its gain, these
  // its saved row statistics, and the [ceil(N / tile width)][M] row sums out
  const float* ln_mean = nullptr;
  const float* ln_rstd = nullptr;
  float2* ln_rows = nullptr;
  // Grouped calls whose groups share one operand (the same A pointer, or the
  // same B pointer) tile the other operand's groups as one concatenated
  // dimension, so that no tile is cut short at a group edge.  Needs the
  // concatenated extent per group to be a multiple of 64.
  bool allow_concat = true;
  int force_bn = 0;     // 0: heuristic
  int force_pair = -1;  // -1: heuristic (CTA pairs when M > 128), 0: single CTAs, 1: pairs
};

// 2-D bf16 TMA descriptor: `inner` contiguous elements per row, `outer` rows,
// `ld` elements between rows; box = 64 x box_outer elements, 128-byte swizzle,
// zero fill outside the tensor.
bool make_map(CUtensorMap* map, const void* base, long long inner, long long outer, long long ld,
              int box_outer);

// 2-D fp32 TMA descriptor without swizzle: box = box_inner x box_outer
// elements (box_inner * 4 bytes a multiple of 16), for tile stores / reductions.
bool make_map_f32(CUtensorMap* map, const void* base, long long inner, long long outer,
                  long long ld, int box_inner, int box_outer);

// Number of SMs of the current device.
int num_sms();

// Enqueue the GEMM on `stream`.  Returns 0 or a cudaError_t value.
int launch_gemm(const GemmDesc& d, cudaStream_t stream);

// Tile width (128 or 256) the launcher picks for a problem.
int gemm_pick_bn(int M, int N, int groups, bool summed, bool pair);

// Reads and clears the device error word of the GEMM kernels on the current
// device (synchronises `stream` first).  Returns a cudaError_t value.
int gemm_read_clear_error(unsigned int* value, cudaStream_t stream);

}  // namespace tp
