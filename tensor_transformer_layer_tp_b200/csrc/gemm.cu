// tcgen05 GEMM kernel and its host launcher.  See gemm.cuh for what it computes.
//
// Structure (one CTA per SM, persistent over output tiles):
//   warp 0      : TMA producer.  Streams 128x64 A tiles and BNx64 B tiles into
//                 a STAGES-deep shared-memory ring (128-byte swizzle).
//   warp 1      : allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN,
//                 K=16 per instruction) into one of two TMEM accumulators and
//                 frees ring slots with tcgen05.commit.
//   warps 2..5  : epilogue.  tcgen05.ld the finished accumulator (one TMEM lane
//                 = one output row per thread), apply the fused epilogue and
//                 store (straight from registers, or for the epilogues that
//                 would otherwise bound the GEMM staged in shared memory and
//                 written by TMA tensor stores); the other accumulator is
//                 being filled meanwhile.
#include <cudaTypedefs.h>

#include <mutex>

#include "gemm.cuh"

namespace tp {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr uint32_t A_STAGE_BYTES = BM * BK * 2;
constexpr int kEpilogueThreads = 128;
constexpr int kGemmThreads = 64 + kEpilogueThreads;
// Epilogue modes, one kernel instance each: lane-per-row stores; tensor
// stores through shared-memory staging (4 epilogue warps, two staging
// buffers each); lane-per-row stores plus the LayerNorm-backward row sums.
// For CTA pairs after a short K loop, where the epilogue bounds the tile,
// the store modes also come with 8 epilogue warps -- two per TMEM lane
// quarter, each on half of the tile's columns (one staging buffer each).
constexpr int kEmDirect = 0, kEmStaged = 1, kEmLnRows = 2, kEmStaged8 = 3, kEmDirect8 = 4;
// Epilogue staging for tensor stores: per epilogue warp two buffers of 4 KB
// (a 32 x 32 chunk of fp32, or of bf16 out + out2).
constexpr uint32_t kStgBufBytes = 4096;
constexpr uint32_t kStgBytes = (kEpilogueThreads / 32) * 2 * kStgBufBytes;

template <int BN>
struct GemmCfg {
  static constexpr uint32_t B_STAGE_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr int STAGES = (BN >= 256) ? 4 : (BN >= 192 ? 5 : 6);
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
  static constexpr size_t SMEM_BYTES = 1024 + size_t(STAGES) * STAGE_BYTES + 256;
  // with the epilogue's tensor-store staging after a 1 KB barrier block
  static constexpr size_t SMEM_BYTES_STG = 1024 + size_t(STAGES) * STAGE_BYTES + 1024 + kStgBytes;
  static_assert(STAGE_BYTES % 1024 == 0, "barriers and staging follow the ring 1024-aligned");
  static_assert(SMEM_BYTES_STG <= 232448, "GEMM exceeds 227 KB of shared memory");
};

__device__ __forceinline__ void decode_tile(const GemmParams& p, int tile, int& g, int& mt,
                                            int& nt) {
  if (p.concat == 1) {
    // Bands of band_w column tiles, row-tile major inside a band: the tiles in
    // flight together share their A rows and a narrow range of B columns.
    g = 0;
    const int band_tiles = p.m_tiles * p.band_w;
    const int b = tile / band_tiles;
    const int r = tile - b * band_tiles;
    const int w = min(p.band_w, p.n_tiles - b * p.band_w);
    mt = r / w;
    nt = b * p.band_w + (r - mt * w);
    return;
  }
  if (p.sum_groups || p.concat) {
    g = 0;
  } else {
    g = tile / p.tiles_per_group;
    tile -= g * p.tiles_per_group;
  }
  mt = tile / p.n_tiles;
  nt = tile - mt * p.n_tiles;
}

// Splits a coordinate v of a concatenated dimension (groups x ext) into the
// group and the coordinate inside it.  Past the end it stays in the last
// group, where the coordinate is out of range (TMA fills zeros, the epilogue
// stores nothing).
__device__ __forceinline__ void split_concat(int v, int ext, int groups, int& g, int& local) {
  g = v / ext;
  if (g > groups - 1) g = groups - 1;
  local = v - g * ext;
}

// Where the 64-row chunks of one operand tile come from, fixed per tile: the
// group (-1: the k-loop's group) and the row coordinate inside that group.
template <int NCH>
struct ChunkPlan {
  int g[NCH];
  int r[NCH];
};

template <int NCH>
__device__ __forceinline__ void plan_chunks(ChunkPlan<NCH>& cp, bool concat, int ext, int groups,
                                            int r0) {
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    cp.g[c] = -1;
    cp.r[c] = r0 + c * 64;
    if (concat) split_concat(r0 + c * 64, ext, groups, cp.g[c], cp.r[c]);
  }
}

// Loads an operand tile as NCH chunks of 64 rows (K-major: 64 rows x 64 K;
// MN-major: 64 M/N x 64 K), 8 KB apart in shared memory.
template <bool MN, bool PAIR, int NCH>
__device__ __forceinline__ void load_chunks(uint32_t dst, const CUtensorMap* maps, int gg,
                                            const ChunkPlan<NCH>& cp, int kx, uint32_t bar) {
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int g = cp.g[c] >= 0 ? cp.g[c] : gg;
    const int x = MN ? cp.r[c] : kx, y = MN ? kx : cp.r[c];
    if (PAIR)
      tma_load_2d_pair(dst + c * 8192u, &maps[g], x, y, bar);
    else
      tma_load_2d(dst + c * 8192u, &maps[g], x, y, bar);
  }
}

// Optional bias-gradient partials: column sums over this warp's 32 rows.
// Called by all 32 lanes of the warp (rows >= M contribute zeros).
__device__ __forceinline__ void epilogue_colsum(const GemmParams& p, int go, int m, int n0,
                                                const float (&vals)[32]) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = (m < p.M) ? vals[j] : 0.f;
  warp_colsum32(v);
  const int lane = threadIdx.x & 31;
  const int mblocks = (p.M + 31) / 32;
  const int rb = (m - lane) / 32;     // the warp's 32-row block
  if (rb < mblocks && n0 + lane < p.N)
    p.colsum[((long long)go * mblocks + rb) * p.N + n0 + lane] = v[0];
}

// Fused epilogue for 32 consecutive columns [n0, n0+32) of output row m.
// Called by all 32 lanes of a warp (rows >= M store nothing).
__device__ __forceinline__ bool epi_has_aux(int epi) {
  return epi == EPI_BIAS_RES || epi == EPI_DGELU || epi == EPI_LN_ROWSTATS;
}

// The aux operand (residual or saved pre-activation) of row m, columns
// [n0, n0+32), as 16 bf16 pairs; zeros outside the matrix.
__device__ __forceinline__ void load_aux(const GemmParams& p, int go, int m, int n0,
                                         uint32_t (&w)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = 0u;
  if (!epi_has_aux(p.epi) || m >= p.M || n0 >= p.N) return;
  const __nv_bfloat16* aux =
      static_cast<const __nv_bfloat16*>(p.aux[go]) + (long long)m * p.ldaux + n0;
  if (n0 + 32 <= p.N) {
    const uint4* a4 = reinterpret_cast<const uint4*>(aux);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = a4[q];
      w[4 * q] = u.x;
      w[4 * q + 1] = u.y;
      w[4 * q + 2] = u.z;
      w[4 * q + 3] = u.w;
    }
  } else {
    const uint16_t* a16 = reinterpret_cast<const uint16_t*>(aux);
    for (int j = 0; j < 32 && n0 + j < p.N; ++j)
      w[j >> 1] |= static_cast<uint32_t>(a16[j]) << (16 * (j & 1));
  }
}

// Pulls the aux row segment [n0, n0+cols) of row m into L2 ahead of its use.
__device__ __forceinline__ void prefetch_aux_l2(const GemmParams& p, int go, int m, int n0,
                                                int cols) {
  if (!epi_has_aux(p.epi) || m >= p.M || n0 >= p.N) return;
  const char* row = reinterpret_cast<const char*>(static_cast<const __nv_bfloat16*>(p.aux[go]) +
                                                  (long long)m * p.ldaux + n0);
  const int bytes = 2 * min(cols, p.N - n0);
  for (int b = 0; b < bytes; b += 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(row + b));
}

// EPI_XENT, one 32-column chunk [n0, n0+32) of row m of group g's logits:
// folds the chunk into the row's running (max, sum of 2^(x - max)) over the
// tile (x = z log2 e, columns >= N excluded), picks out the target's logit
// (lt = target column inside the group) and optionally stores bf16(z).
// Called by all 32 lanes of a warp.
__device__ __forceinline__ void epilogue_xent_chunk(const GemmParams& p, int g, int m, int n0,
                                                    const uint32_t (&r)[32], int lt, float& xm,
                                                    float& xs) {
  constexpr float kLog2e = 1.4426950408889634f;
  float x[32];
  float cmax = -INFINITY;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    x[j] = (n0 + j < p.N) ? __uint_as_float(r[j]) * kLog2e : -INFINITY;
    cmax = fmaxf(cmax, x[j]);
  }
  if (cmax > xm) {
    xs = (xm == -INFINITY) ? 0.f : xs * exp2f(xm - cmax);
    xm = cmax;
  }
  if (xm != -INFINITY) {
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      a += exp2f(x[j] - xm);
      b += exp2f(x[j + 1] - xm);
    }
    xs += a + b;
  }
  if (m >= p.M) return;
  // the target's column, if it is a valid column of this chunk (another
  // partition's index can land in the padding past N: not ours)
  if (lt >= n0 && lt < n0 + 32 && lt < p.N) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (lt - n0 == j) p.xent_ztgt[m] = __uint_as_float(r[j]);
  }
  if (p.out[g]) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out[g]) + (long long)m * p.ldc + n0;
    if (n0 + 32 <= p.N) {
      uint4* o4 = reinterpret_cast<uint4*>(out);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o4[q] = make_uint4(pack_bf16(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                           pack_bf16(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                           pack_bf16(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                           pack_bf16(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n0 + j < p.N) out[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
    }
  }
}

// EPI_XENT, end of a tile: the row's (max, sum) for column tile nt of group g.
__device__ __forceinline__ void epilogue_xent_flush(const GemmParams& p, int g, int nt, int m,
                                                    float xm, float xs) {
  if (m < p.M) p.xent_stats[((long long)g * p.n_tiles + nt) * p.M + m] = make_float2(xm, xs);
}

template <bool LNS>
__device__ __forceinline__ void epilogue_chunk(const GemmParams& p, int g, int m, int n0,
                                               const uint32_t (&r)[32],
                                               const uint32_t (&aux_w)[16], float2 lnst,
                                               float& ls1, float& ls2) {
  float v[32], r2[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  const int go = p.sum_groups ? 0 : g;
  const bool full = (n0 + 32 <= p.N);
  const int epi = p.epi;

  if (epi == EPI_BIAS_BF16 || epi == EPI_BIAS_GELU || epi == EPI_BIAS_RES) {
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias[go]);
    if (full) {
      const uint4* b4 = reinterpret_cast<const uint4*>(bias + n0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 u = __ldg(b4 + q);
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[q * 8 + 2 * e] += bf16_lo(w[e]);
          v[q * 8 + 2 * e + 1] += bf16_hi(w[e]);
        }
      }
    } else {
      for (int j = 0; j < 32; ++j)
        if (n0 + j < p.N) v[j] += __bfloat162float(bias[n0 + j]);
    }
  }
  if ((epi == EPI_BIAS_RES || epi == EPI_DGELU) && m < p.M) {
    float a[32];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      a[2 * e] = bf16_lo(aux_w[e]);
      a[2 * e + 1] = bf16_hi(aux_w[e]);
    }
    if (epi == EPI_BIAS_RES) {
      if (p.drop.thresh) {   // hidden-output dropout before the residual add
        const uint32_t keep = drop_keep32(p.drop, static_cast<uint32_t>(m), static_cast<uint32_t>(n0));
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = ((keep >> j) & 1u) ? v[j] * p.drop.scale : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += a[j];
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= a[j];
    }
  }

  if (p.colsum) epilogue_colsum(p, go, m, n0, v);
  if (m >= p.M) return;

  if (LNS) {
    // LayerNorm-backward row sums of the stored (rounded) output dy against the
    // gain and the normalised input: dy g and dy g (x - mean) rstd
    const __nv_bfloat16* gam = static_cast<const __nv_bfloat16*>(p.bias[0]);
    float gv[32];
    if (full) {
      const uint4* g4 = reinterpret_cast<const uint4*>(gam + n0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 u = __ldg(g4 + q);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          gv[q * 8 + 2 * e] = bf16_lo(w[e]);
          gv[q * 8 + 2 * e + 1] = bf16_hi(w[e]);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) gv[j] = (n0 + j < p.N) ? __bfloat162float(gam[n0 + j]) : 0.f;
    }
    const float c = -lnst.x * lnst.y;   // xhat = x rstd - mean rstd
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t yb = pack_bf16(v[2 * e], v[2 * e + 1]);   // the stored values
      const float d0 = bf16_lo(yb) * gv[2 * e], d1 = bf16_hi(yb) * gv[2 * e + 1];
      ls1 += d0 + d1;
      ls2 = fmaf(d0, fmaf(bf16_lo(aux_w[e]), lnst.y, c), fmaf(d1, fmaf(bf16_hi(aux_w[e]), lnst.y, c), ls2));
    }
  }

  if (epi == EPI_F32) {
    float* out = static_cast<float*>(p.out[go]) + (long long)m * p.ldc + n0;
    if (full) {
      float4* o4 = reinterpret_cast<float4*>(out);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        o4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
      for (int j = 0; j < 32; ++j)
        if (n0 + j < p.N) out[j] = v[j];
    }
    return;
  }

  if (epi == EPI_BIAS_GELU) {
    // out2 <- gelu(U), and U is replaced by gelu'(U) for the store to out below
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float g, dg;
      gelu_and_grad(v[j], g, dg);
      v[j] = dg;
      r2[j] = g;
    }
    __nv_bfloat16* out2 = static_cast<__nv_bfloat16*>(p.out2[go]) + (long long)m * p.ldc + n0;
    if (full) {
      uint4* o4 = reinterpret_cast<uint4*>(out2);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o4[q] = make_uint4(pack_bf16(r2[8 * q], r2[8 * q + 1]), pack_bf16(r2[8 * q + 2], r2[8 * q + 3]),
                           pack_bf16(r2[8 * q + 4], r2[8 * q + 5]),
                           pack_bf16(r2[8 * q + 6], r2[8 * q + 7]));
    } else {
      for (int j = 0; j < 32; ++j)
        if (n0 + j < p.N) out2[j] = __float2bfloat16_rn(r2[j]);
    }
  }
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out[go]) + (long long)m * p.ldc + n0;
  if (full) {
    uint4* o4 = reinterpret_cast<uint4*>(out);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      o4[q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                         pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                         pack_bf16(v[8 * q + 6], v[8 * q + 7]));
  } else {
    for (int j = 0; j < 32; ++j)
      if (n0 + j < p.N) out[j] = __float2bfloat16_rn(v[j]);
  }
}

// The fused epilogue of 32 consecutive columns [n0, n0+32) of output row m:
// on return v holds the values of `out` and, for EPI_BIAS_GELU, v2 those of
// `out2`; the optional column-sum partials are written.  Called by all 32
// lanes of a warp.
__device__ __forceinline__ void epilogue_values(const GemmParams& p, int g, int m, int n0,
                                                const uint32_t (&r)[32],
                                                const uint32_t (&aux_w)[16], float (&v)[32],
                                                float (&v2)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  const int go = p.sum_groups ? 0 : g;
  const bool full = (n0 + 32 <= p.N);
  const int epi = p.epi;

  if (epi == EPI_BIAS_BF16 || epi == EPI_BIAS_GELU || epi == EPI_BIAS_RES) {
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias[go]);
    if (full) {
      const uint4* b4 = reinterpret_cast<const uint4*>(bias + n0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 u = __ldg(b4 + q);
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[q * 8 + 2 * e] += bf16_lo(w[e]);
          v[q * 8 + 2 * e + 1] += bf16_hi(w[e]);
        }
      }
    } else {
      for (int j = 0; j < 32; ++j)
        if (n0 + j < p.N) v[j] += __bfloat162float(bias[n0 + j]);
    }
  }
  if ((epi == EPI_BIAS_RES || epi == EPI_DGELU) && m < p.M) {
    float a[32];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      a[2 * e] = bf16_lo(aux_w[e]);
      a[2 * e + 1] = bf16_hi(aux_w[e]);
    }
    if (epi == EPI_BIAS_RES) {
      if (p.drop.thresh) {   // hidden-output dropout before the residual add
        const uint32_t keep = drop_keep32(p.drop, static_cast<uint32_t>(m), static_cast<uint32_t>(n0));
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = ((keep >> j) & 1u) ? v[j] * p.drop.scale : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += a[j];
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= a[j];
    }
  }

  if (p.colsum) epilogue_colsum(p, go, m, n0, v);

  if (epi == EPI_BIAS_GELU) {
    // out2 <- gelu(U); out <- gelu'(U)
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float gl, dg;
      gelu_and_grad(v[j], gl, dg);
      v[j] = dg;
      v2[j] = gl;
    }
  }
}

// Stores a chunk through the TMA unit.  The warp writes its 32 rows x 32
// columns into staging buffer k % NB of its own (laid out as the output tensor
// map's swizzle expects: 16-byte unit u of row r at unit u ^ ((r >> 1) & 3)
// of a 64-byte bf16 row, u ^ (r & 7) of a 128-byte fp32 row, which also keeps
// the warp's shared-memory writes free of bank conflicts), and lane 0 issues
// the tensor store(s) as one bulk group; the tensor map drops columns >= N
// and rows past the stacked outputs (with several groups M % 32 == 0, so a
// warp's rows stay inside its group).  m0: the warp's first row, in group
// coordinates.  Stores
// straight from registers, one row per lane, touch 32 cache lines per
// instruction and made the two-output GeLU epilogue (and the epilogue of
// short-K GEMMs) the bottleneck; the tensor store writes whole lines and
// leaves the epilogue warps free for the next chunk.  Where the epilogue hides
// under the next tile's K loop anyway, its extra synchronisation made the
// last tile's epilogue longer, so the launcher picks it per call (tma_out).
template <int NB>
__device__ __forceinline__ void store_chunk_staged(const GemmMaps& maps, const GemmParams& p,
                                                   int go, int m0, int n0, const float (&v)[32],
                                                   const float (&v2)[32], uint8_t* stg,
                                                   uint32_t k) {
  const int lane = threadIdx.x & 31;
  uint8_t* buf = stg + (NB == 2 ? (k & 1u) * kStgBufBytes : 0u);
  // the bulk group of chunk k - NB (this buffer's last reader) has read it
  if (lane == 0) {
    if (NB == 2)
      bulk_wait_group_read1();
    else
      bulk_wait_group_read0();
  }
  __syncwarp();
  if (p.epi == EPI_F32) {
    uint8_t* row = buf + lane * 128;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      *reinterpret_cast<float4*>(row + ((u ^ (lane & 7)) << 4)) =
          make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
  } else {
    const int sw = (lane >> 1) & 3;
    uint8_t* row = buf + lane * 64;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      *reinterpret_cast<uint4*>(row + ((u ^ sw) << 4)) =
          make_uint4(pack_bf16(v[8 * u], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                     pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
    if (p.epi == EPI_BIAS_GELU) {
      uint8_t* row2 = row + kStgBufBytes / 2;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4*>(row2 + ((u ^ sw) << 4)) = make_uint4(
            pack_bf16(v2[8 * u], v2[8 * u + 1]), pack_bf16(v2[8 * u + 2], v2[8 * u + 3]),
            pack_bf16(v2[8 * u + 4], v2[8 * u + 5]), pack_bf16(v2[8 * u + 6], v2[8 * u + 7]));
    }
  }
  fence_proxy_async_smem();   // the writes are visible to the TMA unit
  __syncwarp();
  if (lane == 0) {
    if (m0 < p.M && n0 < p.N) {
      const int y = go * p.M + m0;   // the groups' outputs are stacked in the maps' rows
      tma_store_2d(&maps.c, smem_u32(buf), n0, y);
      if (p.epi == EPI_BIAS_GELU) tma_store_2d(&maps.c2, smem_u32(buf + kStgBufBytes / 2), n0, y);
    }
    bulk_commit_group();   // one group per chunk (possibly empty), see the wait above
  }
}

// Tensor-store epilogue: the output maps fetched ahead of the first store ...
__device__ __forceinline__ void epilogue_stg_prefetch(const GemmMaps& maps, const GemmParams& p) {
  if (p.epi != EPI_XENT && threadIdx.x == 64) {
    tma_prefetch_desc(&maps.c);
    if (p.epi == EPI_BIAS_GELU) tma_prefetch_desc(&maps.c2);
  }
}
// ... and, before the CTA's shared memory goes, every store has read its
// staging (the global writes complete with the grid).
__device__ __forceinline__ void epilogue_stg_drain(const GemmParams& p) {
  if (p.epi != EPI_XENT && (threadIdx.x & 31) == 0) bulk_wait_group_read0();
  __syncwarp();
}

template <int BN, bool A_MN, bool B_MN, int EM>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmParams p) {
  using Cfg = GemmCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr uint32_t IDESC = make_idesc_bf16(BM, BN, A_MN, B_MN);
  // Byte offsets of the descriptors for the k-th 16-wide K slice of a stage.
  constexpr uint32_t A_K_STEP = A_MN ? 16 * 128 : 32;
  constexpr uint32_t B_K_STEP = B_MN ? 16 * 128 : 32;
  constexpr uint32_t MN_CHUNK_BYTES = BK * 128;   // one 64-wide M/N chunk of a MN-major tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::B_STAGE_BYTES);
  uint8_t* sStg = reinterpret_cast<uint8_t*>(bars) + 1024;   // epilogue staging (kEmStaged)
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES;
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* aborted = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull_bar[a]), 1);
      mbar_init(smem_u32(&tempty_bar[a]), kEpilogueThreads);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *aborted = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.groups; ++g) {
      tma_prefetch_desc(&maps.a[g]);
      tma_prefetch_desc(&maps.b[g]);
    }
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kb_total = p.sum_groups ? p.groups * p.k_blocks : p.k_blocks;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      const bool cm = p.concat == 2, cn = p.concat == 1;
      for (int tile = blockIdx.x; tile < p.total_tiles && !*aborted; tile += gridDim.x) {
        int g, mt, nt;
        decode_tile(p, tile, g, mt, nt);
        ChunkPlan<BM / 64> pa;
        ChunkPlan<BN / 64> pb;
        plan_chunks(pa, cm, p.M, p.groups, mt * BM);
        plan_chunks(pb, cn, p.N, p.groups, nt * BN);
        // summed mode walks the groups' K ranges one after another; (gg, kk)
        // advance incrementally (a division here stalls the ring)
        int gg = p.sum_groups ? 0 : g, kk = 0;
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1, DEV_ERR_TIMEOUT_EMPTY, 1)) {
            *aborted = 1;
            break;
          }
          const uint32_t fb = smem_u32(&full_bar[stage]);
          mbar_arrive_expect_tx(fb, Cfg::STAGE_BYTES);
          const uint32_t a_dst = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * Cfg::B_STAGE_BYTES);
          if (!A_MN && !cm)
            tma_load_2d(a_dst, &maps.a[gg], kk * BK, mt * BM, fb);
          else
            load_chunks<A_MN, false>(a_dst, maps.a, gg, pa, kk * BK, fb);
          if (!B_MN && !cn)
            tma_load_2d(b_dst, &maps.b[gg], kk * BK, nt * BN, fb);
          else
            load_chunks<B_MN, false>(b_dst, maps.b, gg, pb, kk * BK, fb);
          ++issued;
          if (++kk == p.k_blocks && p.sum_groups) {
            kk = 0;
            ++gg;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*aborted) {
        // Let every copy this thread issued land before the CTA exits.
        const int outstanding = issued < STAGES ? issued : STAGES;
        for (int i = 1; i <= outstanding; ++i) {
          int s = stage - i;
          uint32_t ph = phase;
          if (s < 0) {
            s += STAGES;
            ph ^= 1;
          }
          mbar_wait(smem_u32(&full_bar[s]), ph, DEV_ERR_TIMEOUT_DRAIN, 1);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < p.total_tiles && !*aborted; tile += gridDim.x) {
        if (!mbar_wait(smem_u32(&tempty_bar[acc]), acc_phase ^ 1, DEV_ERR_TIMEOUT_ACC, 2)) {
          *aborted = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!mbar_wait(smem_u32(&full_bar[stage]), phase, DEV_ERR_TIMEOUT_FULL, 2)) {
            *aborted = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * Cfg::B_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_MN ? sw128_desc(a0 + k * A_K_STEP, MN_CHUNK_BYTES, 1024)
                                     : sw128_desc(a0 + k * A_K_STEP, 16, 1024);
            const uint64_t bd = B_MN ? sw128_desc(b0 + k * B_K_STEP, MN_CHUNK_BYTES, 1024)
                                     : sw128_desc(b0 + k * B_K_STEP, 16, 1024);
            tc_mma_bf16(d_tmem, ad, bd, IDESC, (kb > 0 || k > 0) ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(smem_u32(&empty_bar[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&tfull_bar[acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (*aborted && issued_any) {
        // Make sure no MMA still writes TMEM before it is released.
        tc_commit(smem_u32(drain_bar));
        mbar_wait(smem_u32(drain_bar), 0, DEV_ERR_TIMEOUT_DRAIN, 2);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;   // accumulator row owned by this thread
    uint8_t* my_stg = sStg + (warp - 2) * (2 * kStgBufBytes);
    uint32_t nchunk = 0;
    if (EM == kEmStaged) epilogue_stg_prefetch(maps, p);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x) {
      int g, mt, nt;
      decode_tile(p, tile, g, mt, nt);
      int ge = g, m = mt * BM + row;
      if (p.concat == 2) split_concat(m, p.M, p.groups, ge, m);   // one group per warp
      int gc = ge, n0 = nt * BN;
      if (p.concat == 1) split_concat(nt * BN, p.N, p.groups, gc, n0);
      // The aux operand (residual / saved pre-activation) of chunk 0 is loaded
      // before the accumulator is waited for, that of chunk c+1 while chunk c
      // is processed, and the next tile's rows are pulled into L2 now.
      uint32_t aux_cur[16], aux_nxt[16];
      load_aux(p, gc, m, n0, aux_cur);
      if (epi_has_aux(p.epi) && tile + (int)gridDim.x < p.total_tiles) {
        int g2, mt2, nt2;
        decode_tile(p, tile + (int)gridDim.x, g2, mt2, nt2);
        int ge2 = g2, m2 = mt2 * BM + row, gc2 = g2, n2 = nt2 * BN;
        if (p.concat == 2) split_concat(m2, p.M, p.groups, ge2, m2);
        gc2 = ge2;
        if (p.concat == 1) split_concat(nt2 * BN, p.N, p.groups, gc2, n2);
        prefetch_aux_l2(p, gc2, m2, n2, BN);
      }
      const bool stop = __any_sync(0xffffffffu, *aborted != 0);   // warp-uniform
      if (stop ||
          !mbar_wait_warp(smem_u32(&tfull_bar[acc]), acc_phase, DEV_ERR_TIMEOUT_ACC, 3)) {
        *aborted = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      // EPI_XENT: the row's running statistics over this tile, and the
      // target's column inside the group (tiles never cross groups there)
      const bool xent = p.epi == EPI_XENT;
      float xm = -INFINITY, xs = 0.f;
      const int xg = gc, xnt = nt;
      const int lt = (xent && m < p.M) ? p.xent_target[m] - (gc + p.xent_group0) * p.N : -1;
      // EPI_LN_ROWSTATS: the row's saved statistics and its sums over this tile
      const bool lns = EM == kEmLnRows && m < p.M;
      const float2 lnst = lns ? make_float2(p.ln_mean[m], p.ln_rstd[m]) : make_float2(0.f, 0.f);
      float ls1 = 0.f, ls2 = 0.f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        if (nt * BN + c * 32 >= p.Nv) break;   // warp-uniform
        int gn = gc, nn = n0 + 32;
        if (p.concat == 1 && nn >= p.N && gn < p.groups - 1) {   // next group's columns
          nn -= p.N;
          ++gn;
        }
        if (c + 1 < BN / 32) load_aux(p, gn, m, nn, aux_nxt);
        uint32_t r[32];
        tmem_ld32_wait(t_row + c * 32, r);
        if (xent) {
          epilogue_xent_chunk(p, gc, m, n0, r, lt, xm, xs);
        } else if (EM == kEmStaged) {
          float v[32], v2[32];
          epilogue_values(p, gc, m, n0, r, aux_cur, v, v2);
          store_chunk_staged<2>(maps, p, p.sum_groups ? 0 : gc, m - lane, n0, v, v2, my_stg, nchunk++);
        } else {
          epilogue_chunk<EM == kEmLnRows>(p, gc, m, n0, r, aux_cur, lnst, ls1, ls2);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) aux_cur[e] = aux_nxt[e];
        gc = gn;
        n0 = nn;
      }
      if (xent) epilogue_xent_flush(p, xg, xnt, m, xm, xs);
      if (lns) p.ln_rows[(long long)nt * p.M + m] = make_float2(ls1, ls2);
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty_bar[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    if (EM == kEmStaged) epilogue_stg_drain(p);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA-pair kernel
//
// Same computation with 256-row tiles shared by a cluster of two CTAs on
// neighbouring SMs (tcgen05 cta_group::2).  CTA r of the pair loads rows
// [128r, 128r+128) of the A tile and columns [r*BN/2, (r+1)*BN/2) of the B
// tile into its own shared memory; one MMA instruction issued by CTA 0 reads
// both halves and writes the 128 accumulator rows of each CTA into that CTA's
// TMEM.  Each SM therefore streams half the B tile: 32 KB per 64-deep K step
// at BN = 256 instead of 48 KB, and the ring holds 6 such stages.
//
// Barriers: stage "full" lives in CTA 0 (its producer arms it with both CTAs'
// bytes; both CTAs' TMA loads complete on it); stage "empty" and accumulator
// "full" exist in both CTAs and are signalled by CTA 0's commits, multicast
// to the pair; accumulator "empty" lives in CTA 0 and collects the epilogue
// threads of both CTAs.  No TMA load uses multicast.

constexpr int kPairRows = 256;

template <int BN>
struct GemmPairCfg {
  static constexpr int BNH = BN / 2;   // B columns held by each CTA
  static constexpr uint32_t B_STAGE_BYTES = BNH * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;   // per CTA
  static constexpr int STAGES = (BN >= 256) ? 6 : 8;
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
  static constexpr size_t SMEM_BYTES = 1024 + size_t(STAGES) * STAGE_BYTES + 256;
  // with the epilogue's tensor-store staging after a 1 KB barrier block
  static constexpr size_t SMEM_BYTES_STG = 1024 + size_t(STAGES) * STAGE_BYTES + 1024 + kStgBytes;
  static_assert(STAGE_BYTES % 1024 == 0, "barriers and staging follow the ring 1024-aligned");
  static_assert(SMEM_BYTES_STG <= 232448, "GEMM exceeds 227 KB of shared memory");
};

template <int BN, bool A_MN, bool B_MN, int EM>
__global__ void __cluster_dims__(2, 1, 1)
    __launch_bounds__((EM == kEmStaged8 || EM == kEmDirect8) ? 64 + 256 : kGemmThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmParams p) {
  using Cfg = GemmPairCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr bool STGD = EM == kEmStaged || EM == kEmStaged8;   // tensor-store epilogue
  constexpr int EPI_WARPS = (EM == kEmStaged8 || EM == kEmDirect8) ? 8 : 4;
  constexpr int BNH = Cfg::BNH;
  constexpr uint32_t IDESC = make_idesc_bf16(kPairRows, BN, A_MN, B_MN);
  constexpr uint32_t A_K_STEP = A_MN ? 16 * 128 : 32;
  constexpr uint32_t B_K_STEP = B_MN ? 16 * 128 : 32;
  constexpr uint32_t MN_CHUNK_BYTES = BK * 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::B_STAGE_BYTES);
  uint8_t* sStg = reinterpret_cast<uint8_t*>(bars) + 1024;   // epilogue staging (kEmStaged)
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES;
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* aborted = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull_bar[a]), 1);
      mbar_init(smem_u32(&tempty_bar[a]), 2 * 32 * EPI_WARPS);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *aborted = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.groups; ++g) {
      tma_prefetch_desc(&maps.a[g]);
      tma_prefetch_desc(&maps.b[g]);
    }
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kb_total = p.sum_groups ? p.groups * p.k_blocks : p.k_blocks;
  const int cl = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(num_clusters_x());

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      bool issued_any = false;
      const bool cm = p.concat == 2, cn = p.concat == 1;
      for (int tile = cl; tile < p.total_tiles && !*aborted; tile += ncl) {
        int g, mt, nt;
        decode_tile(p, tile, g, mt, nt);
        const int row0 = mt * kPairRows + static_cast<int>(rank) * BM;
        const int col0 = nt * BN + static_cast<int>(rank) * BNH;
        ChunkPlan<BM / 64> pa;
        ChunkPlan<BNH / 64> pb;
        plan_chunks(pa, cm, p.M, p.groups, row0);
        plan_chunks(pb, cn, p.N, p.groups, col0);
        // summed mode walks the groups' K ranges one after another; (gg, kk)
        // advance incrementally (a division here stalls the ring)
        int gg = p.sum_groups ? 0 : g, kk = 0;
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1, DEV_ERR_TIMEOUT_EMPTY, 5)) {
            *aborted = 1;
            break;
          }
          const uint32_t fb_local = smem_u32(&full_bar[stage]);
          if (leader) mbar_arrive_expect_tx(fb_local, 2 * Cfg::STAGE_BYTES);
          const uint32_t fb = mapa_shared(fb_local, 0);
          const uint32_t a_dst = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * Cfg::B_STAGE_BYTES);
          if (!A_MN && !cm)
            tma_load_2d_pair(a_dst, &maps.a[gg], kk * BK, row0, fb);
          else
            load_chunks<A_MN, true>(a_dst, maps.a, gg, pa, kk * BK, fb);
          if (!B_MN && !cn)
            tma_load_2d_pair(b_dst, &maps.b[gg], kk * BK, col0, fb);
          else
            load_chunks<B_MN, true>(b_dst, maps.b, gg, pb, kk * BK, fb);
          issued_any = true;
          if (++kk == p.k_blocks && p.sum_groups) {
            kk = 0;
            ++gg;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*aborted && issued_any) {
        // Completion of this CTA's copies is counted in CTA 0; give them a
        // bounded moment to land before the CTA leaves.
        const unsigned long long t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------------- MMA issuer (CTA 0)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued_any = false;
      for (int tile = cl; tile < p.total_tiles && !*aborted; tile += ncl) {
        if (!mbar_wait(smem_u32(&tempty_bar[acc]), acc_phase ^ 1, DEV_ERR_TIMEOUT_ACC, 6)) {
          *aborted = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!mbar_wait(smem_u32(&full_bar[stage]), phase, DEV_ERR_TIMEOUT_FULL, 6)) {
            *aborted = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * Cfg::B_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_MN ? sw128_desc(a0 + k * A_K_STEP, MN_CHUNK_BYTES, 1024)
                                     : sw128_desc(a0 + k * A_K_STEP, 16, 1024);
            const uint64_t bd = B_MN ? sw128_desc(b0 + k * B_K_STEP, MN_CHUNK_BYTES, 1024)
                                     : sw128_desc(b0 + k * B_K_STEP, 16, 1024);
            tc_mma_bf16_pair(d_tmem, ad, bd, IDESC, (kb > 0 || k > 0) ? 1u : 0u);
          }
          issued_any = true;
          tc_commit_pair_mc(smem_u32(&empty_bar[stage]), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(smem_u32(&tfull_bar[acc]), 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (*aborted && issued_any) {
        tc_commit_pair_mc(smem_u32(drain_bar), 0x1);
        mbar_wait(smem_u32(drain_bar), 0, DEV_ERR_TIMEOUT_DRAIN, 6);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    // with 8 epilogue warps, warps 2..5 take the tile's first half of the
    // columns and warps 6..9 the second
    const int c_begin = EPI_WARPS == 8 ? ((warp - 2) >> 2) * (BN / 64) : 0;
    const int c_end = EPI_WARPS == 8 ? c_begin + BN / 64 : BN / 32;
    uint8_t* my_stg = sStg + (warp - 2) * ((EPI_WARPS == 8 ? 1 : 2) * kStgBufBytes);
    uint32_t nchunk = 0;
    if (STGD) epilogue_stg_prefetch(maps, p);
    const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&tempty_bar[0]), 0),
                                       mapa_shared(smem_u32(&tempty_bar[1]), 0)};
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cl; tile < p.total_tiles; tile += ncl) {
      int g, mt, nt;
      decode_tile(p, tile, g, mt, nt);
      int ge = g, m = mt * kPairRows + static_cast<int>(rank) * BM + row;
      if (p.concat == 2) split_concat(m, p.M, p.groups, ge, m);   // one group per warp
      int gc = ge, n0 = nt * BN + c_begin * 32;
      if (p.concat == 1) split_concat(nt * BN + c_begin * 32, p.N, p.groups, gc, n0);
      // The aux operand (residual / saved pre-activation) of chunk 0 is loaded
      // before the accumulator is waited for, that of chunk c+1 while chunk c
      // is processed, and the next tile's rows are pulled into L2 now.
      uint32_t aux_cur[16], aux_nxt[16];
      load_aux(p, gc, m, n0, aux_cur);
      if (epi_has_aux(p.epi) && tile + ncl < p.total_tiles) {
        int g2, mt2, nt2;
        decode_tile(p, tile + ncl, g2, mt2, nt2);
        int ge2 = g2, m2 = mt2 * kPairRows + static_cast<int>(rank) * BM + row, gc2 = g2,
            n2 = nt2 * BN + c_begin * 32;
        if (p.concat == 2) split_concat(m2, p.M, p.groups, ge2, m2);
        gc2 = ge2;
        if (p.concat == 1) split_concat(nt2 * BN + c_begin * 32, p.N, p.groups, gc2, n2);
        prefetch_aux_l2(p, gc2, m2, n2, (c_end - c_begin) * 32);
      }
      const bool stop = __any_sync(0xffffffffu, *aborted != 0);   // warp-uniform
      if (stop ||
          !mbar_wait_warp(smem_u32(&tfull_bar[acc]), acc_phase, DEV_ERR_TIMEOUT_ACC, 7)) {
        *aborted = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      // EPI_XENT: the row's running statistics over this tile, and the
      // target's column inside the group (tiles never cross groups there)
      const bool xent = p.epi == EPI_XENT;
      float xm = -INFINITY, xs = 0.f;
      const int xg = gc, xnt = nt;
      const int lt = (xent && m < p.M) ? p.xent_target[m] - (gc + p.xent_group0) * p.N : -1;
      // EPI_LN_ROWSTATS: the row's saved statistics and its sums over this tile
      const bool lns = EM == kEmLnRows && m < p.M;
      const float2 lnst = lns ? make_float2(p.ln_mean[m], p.ln_rstd[m]) : make_float2(0.f, 0.f);
      float ls1 = 0.f, ls2 = 0.f;
#pragma unroll 1
      for (int c = c_begin; c < c_end; ++c) {
        if (nt * BN + c * 32 >= p.Nv) break;   // warp-uniform
        int gn = gc, nn = n0 + 32;
        if (p.concat == 1 && nn >= p.N && gn < p.groups - 1) {   // next group's columns
          nn -= p.N;
          ++gn;
        }
        if (c + 1 < c_end) load_aux(p, gn, m, nn, aux_nxt);
        uint32_t r[32];
        tmem_ld32_wait(t_row + c * 32, r);
        if (xent) {
          epilogue_xent_chunk(p, gc, m, n0, r, lt, xm, xs);
        } else if (STGD) {
          float v[32], v2[32];
          epilogue_values(p, gc, m, n0, r, aux_cur, v, v2);
          store_chunk_staged<EPI_WARPS == 8 ? 1 : 2>(maps, p, p.sum_groups ? 0 : gc, m - lane, n0, v,
                                                     v2, my_stg, nchunk++);
        } else {
          epilogue_chunk<EM == kEmLnRows>(p, gc, m, n0, r, aux_cur, lnst, ls1, ls2);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) aux_cur[e] = aux_nxt[e];
        gc = gn;
        n0 = nn;
      }
      if (xent) epilogue_xent_flush(p, xg, xnt, m, xm, xs);
      if (lns) p.ln_rows[(long long)nt * p.M + m] = make_float2(ls1, ls2);
      tc_fence_before();
      mbar_arrive_cluster(tempty_leader[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    if (STGD) epilogue_stg_drain(p);
  }

  tc_fence_before();
  __syncwarp();
  __syncthreads();
  cluster_sync();   // the peer's MMAs, copies and arrivals are done before TMEM and smem go
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

}  // namespace

// 2-D bf16 tensor map: `inner` contiguous elements per row, `outer` rows,
// `ld` elements between rows; box = 64 inner x box_outer, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, long long inner, long long outer, long long ld,
              int box_outer) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map_f32(CUtensorMap* map, const void* base, long long inner, long long outer,
                  long long ld, int box_inner, int box_outer) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 4)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output tensor map for the epilogue's tensor stores: box 32 x 32 elements,
// swizzled to the box row (64 bytes of bf16: 64-byte swizzle; 128 bytes of
// fp32: 128-byte swizzle).  Needs a 16-byte aligned base and row stride.
static bool make_map_out(CUtensorMap* map, const void* base, long long inner, long long outer,
                  long long ld, bool f32) {
  auto enc = get_encode_fn();
  const int esz = f32 ? 4 : 2;
  if (!enc || !base || (reinterpret_cast<uintptr_t>(base) & 15) || (ld * esz) % 16 || ld < inner)
    return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * esz)};
  cuuint32_t box[2] = {32u, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (n[dev] == 0) cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
  return n[dev] > 0 ? n[dev] : 148;
}

namespace {

// One kernel instance per epilogue mode: the tensor-store path and its shared
// memory, and the LayerNorm row sums, exist only in the instances that use
// them (kernels carrying several store paths measured 1-4 % slower on the
// plain epilogues).
template <int BN, bool A_MN, bool B_MN, int EM>
int launch_inst(const GemmMaps& maps, const GemmParams& prm, cudaStream_t stream) {
  using Cfg = GemmCfg<BN>;
  auto kern = gemm_tc_kernel<BN, A_MN, B_MN, EM>;
  constexpr size_t smem = (EM == kEmStaged || EM == kEmStaged8) ? Cfg::SMEM_BYTES_STG : Cfg::SMEM_BYTES;
  static int configured_dev_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured_dev_mask & (1 << (dev & 31)))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << (dev & 31);
  }
  const int grid = prm.total_tiles < num_sms() ? prm.total_tiles : num_sms();
  kern<<<grid, kGemmThreads, smem, stream>>>(maps, prm);
  return cudaGetLastError();
}

template <int BN, bool A_MN, bool B_MN, int EM>
int launch_pair_inst(const GemmMaps& maps, const GemmParams& prm, cudaStream_t stream) {
  using Cfg = GemmPairCfg<BN>;
  auto kern = gemm_tc2_kernel<BN, A_MN, B_MN, EM>;
  constexpr size_t smem = (EM == kEmStaged || EM == kEmStaged8) ? Cfg::SMEM_BYTES_STG : Cfg::SMEM_BYTES;
  static int configured_dev_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured_dev_mask & (1 << (dev & 31)))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << (dev & 31);
  }
  const int pairs = num_sms() / 2;
  const int clusters = prm.total_tiles < pairs ? prm.total_tiles : pairs;
  kern<<<2 * clusters, (EM == kEmStaged8 || EM == kEmDirect8) ? 64 + 256 : kGemmThreads, smem,
         stream>>>(maps, prm);
  return cudaGetLastError();
}

// The row sums serve the input-gradient GEMMs (K-major operands) only.
template <int BN, bool A_MN, bool B_MN>
int launch_pair_stg(const GemmMaps& maps, const GemmParams& prm, cudaStream_t s) {
  if (prm.epi == EPI_LN_ROWSTATS) {
    if constexpr (!A_MN && !B_MN) return launch_pair_inst<BN, A_MN, B_MN, kEmLnRows>(maps, prm, s);
    return cudaErrorInvalidValue;
  }
  // after a short K loop the epilogue bounds the tile: twice the warps for it
  // (not for the loss statistics, which keep running row state over a tile)
  const int kb_total = prm.sum_groups ? prm.groups * prm.k_blocks : prm.k_blocks;
  const bool short_k = kb_total <= 16;
  if (!prm.tma_out)
    return short_k && prm.epi != EPI_XENT ? launch_pair_inst<BN, A_MN, B_MN, kEmDirect8>(maps, prm, s)
                                          : launch_pair_inst<BN, A_MN, B_MN, kEmDirect>(maps, prm, s);
  return short_k ? launch_pair_inst<BN, A_MN, B_MN, kEmStaged8>(maps, prm, s)
                 : launch_pair_inst<BN, A_MN, B_MN, kEmStaged>(maps, prm, s);
}

template <int BN, bool A_MN, bool B_MN>
int launch_stg(const GemmMaps& maps, const GemmParams& prm, cudaStream_t s) {
  if (prm.epi == EPI_LN_ROWSTATS) {
    if constexpr (!A_MN && !B_MN) return launch_inst<BN, A_MN, B_MN, kEmLnRows>(maps, prm, s);
    return cudaErrorInvalidValue;
  }
  return prm.tma_out ? launch_inst<BN, A_MN, B_MN, kEmStaged>(maps, prm, s)
                     : launch_inst<BN, A_MN, B_MN, kEmDirect>(maps, prm, s);
}

template <int BN>
int dispatch_pair(bool a_mn, bool b_mn, const GemmMaps& maps, const GemmParams& prm,
                  cudaStream_t s) {
  if (!a_mn && !b_mn) return launch_pair_stg<BN, false, false>(maps, prm, s);
  if (!a_mn && b_mn) return launch_pair_stg<BN, false, true>(maps, prm, s);
  if (a_mn && b_mn) return launch_pair_stg<BN, true, true>(maps, prm, s);
  return launch_pair_stg<BN, true, false>(maps, prm, s);
}

template <int BN>
int dispatch_major(bool a_mn, bool b_mn, const GemmMaps& maps, const GemmParams& prm,
                   cudaStream_t s) {
  if (!a_mn && !b_mn) return launch_stg<BN, false, false>(maps, prm, s);
  if (!a_mn && b_mn) return launch_stg<BN, false, true>(maps, prm, s);
  if (a_mn && b_mn) return launch_stg<BN, true, true>(maps, prm, s);
  return launch_stg<BN, true, false>(maps, prm, s);
}

}  // namespace

int gemm_read_clear_error(unsigned int* value, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  return read_clear_unit_error(value);
}

// Tile choice, from timing every layer GEMM shape on B200: 256-column tiles
// beat 128-column ones everywhere (a 128-wide tile moves 1.5x the operand bytes
// per flop and starves on L2 -> SM bandwidth), CTA pairs beat single CTAs
// from M = 512 up, single CTAs win for short M (fewer idle half-pairs).
bool gemm_use_pair(int M) { return M >= 512; }

int gemm_pick_bn(int M, int N, int groups, bool summed, bool pair) {
  (void)M;
  (void)groups;
  (void)summed;
  (void)pair;
  return N <= 128 ? 128 : 256;
}

int launch_gemm(const GemmDesc& d, cudaStream_t stream) {
  if (d.groups < 1 || d.groups > kMaxGroups || d.M <= 0 || d.N <= 0 || d.K <= 0)
    return cudaErrorInvalidValue;
  int concat = 0;
  if (d.epi == EPI_XENT && (d.sum_groups || !d.xent_target || !d.xent_stats || !d.xent_ztgt))
    return cudaErrorInvalidValue;
  if (!d.sum_groups && d.groups > 1 && d.allow_concat && d.epi != EPI_XENT) {
    bool same_a = true, same_b = true;
    for (int g = 1; g < d.groups; ++g) {
      same_a = same_a && d.a[g] == d.a[0];
      same_b = same_b && d.b[g] == d.b[0];
    }
    if (same_a && !same_b && d.N % 64 == 0) concat = 1;
    if (same_b && !same_a && d.M % 64 == 0) concat = 2;
    // A K-major operand that already fills whole tiles gains nothing and
    // would be loaded in more, smaller chunks.
    const int bn_est = gemm_pick_bn(d.M, concat == 1 ? d.groups * d.N : d.N, d.groups, false, true);
    if (concat == 1 && !d.b_mn && d.N % bn_est == 0) concat = 0;
    if (concat == 2 && !d.a_mn && d.M % kPairRows == 0) concat = 0;
  }
  const int Mv = concat == 2 ? d.groups * d.M : d.M;
  const int Nv = concat == 1 ? d.groups * d.N : d.N;
  const bool pair = d.force_pair >= 0 ? d.force_pair != 0 : gemm_use_pair(Mv);
  const int bn = d.force_bn ? d.force_bn : gemm_pick_bn(Mv, Nv, d.groups, d.sum_groups, pair);
  const int rows = pair ? kPairRows : BM;
  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  for (int g = 0; g < d.groups; ++g) {
    bool ok;
    // K-major operands of a concatenated dimension load in 64-row chunks
    if (!d.a_mn)
      ok = make_map(&maps.a[g], d.a[g], d.K, d.M, d.lda, concat == 2 ? 64 : BM);
    else
      ok = make_map(&maps.a[g], d.a[g], d.M, d.K, d.lda, BK);
    if (ok) {
      if (!d.b_mn)
        ok = make_map(&maps.b[g], d.b[g], d.K, d.N, d.ldb, concat == 1 ? 64 : (pair ? bn / 2 : bn));
      else
        ok = make_map(&maps.b[g], d.b[g], d.N, d.K, d.ldb, BK);
    }
    if (!ok) return cudaErrorInvalidValue;
  }
  GemmParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.groups = d.groups;
  prm.sum_groups = d.sum_groups;
  prm.concat = concat;
  prm.M = d.M;
  prm.N = d.N;
  prm.K = d.K;
  prm.Mv = Mv;
  prm.Nv = Nv;
  prm.m_tiles = (Mv + rows - 1) / rows;
  prm.n_tiles = (Nv + bn - 1) / bn;
  prm.k_blocks = (d.K + BK - 1) / BK;
  prm.tiles_per_group = prm.m_tiles * prm.n_tiles;
  prm.band_w = (d.N + bn - 1) / bn;   // about one group's columns per band
  prm.total_tiles = prm.tiles_per_group * (d.sum_groups || concat ? 1 : d.groups);
  prm.epi = d.epi;
  prm.ldc = d.ldc;
  prm.ldaux = d.ldaux;
  prm.colsum = d.colsum;
  prm.xent_target = d.xent_target;
  prm.xent_stats = d.xent_stats;
  prm.xent_ztgt = d.xent_ztgt;
  prm.xent_group0 = d.xent_group0;
  prm.drop = d.drop;
  prm.ln_mean = d.ln_mean;
  prm.ln_rstd = d.ln_rstd;
  prm.ln_rows = d.ln_rows;
  if (d.epi == EPI_LN_ROWSTATS && ((d.groups != 1 && !d.sum_groups) || !d.ln_mean || !d.ln_rstd ||
                                   !d.ln_rows || !d.aux[0] || !d.bias[0]))
    return cudaErrorInvalidValue;
  for (int g = 0; g < kMaxGroups; ++g) {
    prm.out[g] = d.out[g];
    prm.out2[g] = d.out2[g];
    prm.bias[g] = d.bias[g];
    prm.aux[g] = d.aux[g];
  }
  // Tensor stores for the epilogues that would otherwise bound the GEMM (two
  // outputs and the GeLU; a plain output after a short K loop), when the
  // groups' outputs are stacked ([groups][M][ldc], 16-byte aligned base and
  // row stride) so that one tensor map per output covers them all.
  prm.tma_out = 0;
  const long long k_total = (long long)d.K * (d.sum_groups ? d.groups : 1);
  const bool plain = d.epi == EPI_BF16 || d.epi == EPI_BIAS_BF16 || d.epi == EPI_F32;
  if (d.epi == EPI_BIAS_GELU || (plain && k_total <= 1024)) {
    const int nout = d.sum_groups ? 1 : d.groups;
    const long long esz = d.epi == EPI_F32 ? 4 : 2;
    const long long gstride = (long long)d.M * d.ldc * esz;
    // a warp's 32 rows must not run past its group's M into the next group
    bool ok = nout == 1 || d.M % 32 == 0;
    for (int g = 1; ok && g < nout; ++g) {
      ok = static_cast<const char*>(d.out[g]) == static_cast<const char*>(d.out[0]) + g * gstride;
      if (d.epi == EPI_BIAS_GELU)
        ok = ok && static_cast<const char*>(d.out2[g]) == static_cast<const char*>(d.out2[0]) + g * gstride;
    }
    ok = ok && make_map_out(&maps.c, d.out[0], d.N, (long long)nout * d.M, d.ldc, d.epi == EPI_F32);
    if (ok && d.epi == EPI_BIAS_GELU)
      ok = make_map_out(&maps.c2, d.out2[0], d.N, (long long)nout * d.M, d.ldc, false);
    prm.tma_out = ok ? 1 : 0;
  }
  if (pair) {
    switch (bn) {
      case 128: return dispatch_pair<128>(d.a_mn, d.b_mn, maps, prm, stream);
      case 256: return dispatch_pair<256>(d.a_mn, d.b_mn, maps, prm, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (bn) {
    case 128: return dispatch_major<128>(d.a_mn, d.b_mn, maps, prm, stream);
    case 256: return dispatch_major<256>(d.a_mn, d.b_mn, maps, prm, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tp
