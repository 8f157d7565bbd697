// LayerNorm forward/backward and column reductions (bandwidth-bound kernels).
//
// LayerNorm is replicated in Megatron-LM's intra-layer parallelism rather than
// split (Megatron-LM show notes, the outline item on dropout, layer
// normalisation and residual connections being duplicated to avoid
// communication), so on one device it runs once over the full hidden width.
// The forward stages one row per warp in shared memory; the backward runs one
// block per SM over a contiguous range of rows, row statistics by warps, then
// dx and the column partials by column owners.  Accesses are 16-byte vectors
// along the hidden dimension and row statistics use warp shuffles.
#include <string.h>

#include <mutex>
#include <set>
#include <utility>

#include "kernels.cuh"
#include "tp_common.cuh"

namespace tp {

namespace {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
  f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z);
  f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                    pack_bf16(f[6], f[7]));
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kLnBlocks = 148;   // the backward: one block per SM of a B200
constexpr uint32_t kLnSmemBudget = 224u * 1024u;   // dynamic shared memory a block may take

// ---------------------------------------------------------------- forward, one warp per row
// A warp copies its row into shared memory with 16-byte asynchronous copies,
// all issued at once, so the SM has every row of its warps in flight (8 rows
// a block, up to 4 blocks of 48 KB per SM at h = 3072: a 4096-row tensor is
// one wave of warps); registers stay few.  Mean and variance come from two
// passes over the staged row (the mean, then the squared deviations from it:
// the textbook stable form, and fewer instructions than merging per-vector
// partial moments).  Gamma and beta are read through the cache (the same for
// every row).
constexpr int kLnFwdWarps = 8;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kLnFwdWarps * 32)
    ln_fwd_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ gamma,
                  const __nv_bfloat16* __restrict__ beta, float eps, int rows, int h, bool stats_given,
                  __nv_bfloat16* __restrict__ y, float* __restrict__ mean, float* __restrict__ rstd) {
  extern __shared__ uint4 ln_rows[];   // [kLnFwdWarps][h / 8]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = blockIdx.x * kLnFwdWarps + warp;
  if (r >= rows) return;   // warp-uniform; no block-wide synchronisation below
  const int nvec = h >> 3;
  uint4* row = ln_rows + (size_t)warp * nvec;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (long long)r * h);
  for (int c = lane; c < nvec; c += 32) cp_async16(row + c, xr + c);
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncwarp();
  float mu, rs;
  if (stats_given) {
    mu = mean[r];
    rs = rstd[r];
  } else {
    // two passes over the staged row: the mean, then the squared deviations
    float sum = 0.f;
    for (int c = lane; c < nvec; c += 32) {
      float v[8];
      unpack8(row[c], v);
      sum += ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
    }
    mu = warp_sum(sum) / h;
    float sq = 0.f;
    for (int c = lane; c < nvec; c += 32) {
      float v[8];
      unpack8(row[c], v);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = v[e] - mu;
        sq = fmaf(d, d, sq);
      }
    }
    rs = rsqrtf(warp_sum(sq) / h + eps);
  }
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  const uint4* b4 = reinterpret_cast<const uint4*>(beta);
  uint4* yr = reinterpret_cast<uint4*>(y + (long long)r * h);
#pragma unroll 4
  for (int c = lane; c < nvec; c += 32) {
    float v[8], g[8], b[8], o[8];
    unpack8(row[c], v);
    unpack8(__ldg(g4 + c), g);
    unpack8(__ldg(b4 + c), b);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = fmaf((v[e] - mu) * rs, g[e], b[e]);
    yr[c] = pack8(o);
  }
  if (lane == 0 && !stats_given) {
    mean[r] = mu;
    rstd[r] = rs;
  }
}

// ---------------------------------------------------------------- backward
// One block per SM over a contiguous slab of rows [r0, r1), in two phases:
//  1. row statistics, one warp per row (16-byte loads along the row, a warp
//     shuffle reduction, no block barrier): m1 = sum_j dy_j g_j / h and
//     m2 = sum_j dy_j g_j xhat_j / h, kept in shared memory with the row's
//     mean and rstd;
//  2. after the block's one barrier, column owners: thread (c, q) owns the
//     hidden columns [8c, 8c+8) of rows r0 + q, r0 + q + RS, ... (RS row lanes
//     fill the block when the row has fewer than 512 vectors of 8) and writes
//     dx = rstd (dy g - (xhat m2 + m1)) + dres; the column partials of dgamma,
//     dbeta (and the extra sums) accumulate in registers, then across the RS
//     row lanes in shared memory.
// The second reads of dy and x come from L2: a block's slab (28 rows of 12 KB
// at h = 3072) was read a few microseconds before.  (A column-owner kernel
// that reduced every row's sums across the whole block took two block
// barriers per group of four rows and reached 40 % of HBM bandwidth.)
// Per-block column partials go to `partial`:
//   plane 0: sum dy * xhat (dgamma)      plane 1: sum dy (dbeta)
//   plane 2: sum dres                    plane 3: sum dx      (only if extra)
// so a caller whose residual gradient and output are themselves the inputs of
// bias gradients gets those column sums from the same pass.
constexpr int kLnBwdThreads = 512;        // block = (h / 8) x RS threads, at most this
constexpr int kLnBwdMaxSlabRows = 4096;   // row statistics in shared memory: 64 KB

__host__ __device__ inline int ln_bwd_rows_per_block(int rows) {
  int rpb = (rows + kLnBlocks - 1) / kLnBlocks;
  return rpb < kLnBwdMaxSlabRows ? rpb : kLnBwdMaxSlabRows;
}
inline int ln_bwd_row_lanes(int h) {
  const int rs = kLnBwdThreads / (h / 8);
  return rs > 0 ? rs : 1;
}

template <bool EXTRA>
__global__ void __launch_bounds__(kLnBwdThreads, 1) ln_bwd_kernel(
    const __nv_bfloat16* __restrict__ dy, const __nv_bfloat16* __restrict__ x,
    const __nv_bfloat16* __restrict__ gamma, const float* __restrict__ mean,
    const float* __restrict__ rstd, const __nv_bfloat16* __restrict__ dres, int rows, int h,
    int rows_per_block, int rs_lanes, const float2* __restrict__ row_sums, int row_parts,
    __nv_bfloat16* __restrict__ dx, float* __restrict__ partial) {
  extern __shared__ float4 ln_bwd_smem[];   // [rows_per_block] (mean, rstd, m1, m2); scratch
  const int nvec = h >> 3;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;   // whole warps (a partial last warp skips phase 1)
  const int r0 = blockIdx.x * rows_per_block;
  const int r1 = min(rows, r0 + rows_per_block);
  const float inv_h = 1.0f / h;
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  float4* st = ln_bwd_smem;

  // ---- phase 1: row statistics.  Given (row_sums: per-column-tile partial
  // sums from the GEMM that produced dy), one thread per row adds them up in
  // order; otherwise one warp per row reads dy and x.
  if (row_sums) {
    for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
      float s1 = 0.f, s2 = 0.f;
      for (int k = 0; k < row_parts; ++k) {
        const float2 v = row_sums[(long long)k * rows + r];
        s1 += v.x;
        s2 += v.y;
      }
      st[r - r0] = make_float4(mean[r], rstd[r], s1 * inv_h, s2 * inv_h);
    }
  } else if (warp < nwarps) {
    for (int r = r0 + warp; r < r1; r += nwarps) {
      const uint4* dyr = reinterpret_cast<const uint4*>(dy + (long long)r * h);
      const uint4* xr = reinterpret_cast<const uint4*>(x + (long long)r * h);
      const float mu = mean[r], rs = rstd[r];
      float s1 = 0.f, s2 = 0.f;
#pragma unroll 12
      for (int c = lane; c < nvec; c += 32) {
        float d[8], xv[8], g[8];
        unpack8(dyr[c], d);
        unpack8(xr[c], xv);
        unpack8(__ldg(g4 + c), g);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float gd = d[e] * g[e];
          s1 += gd;
          s2 = fmaf(gd, (xv[e] - mu) * rs, s2);
        }
      }
      s1 = warp_sum(s1);
      s2 = warp_sum(s2);
      if (lane == 0) st[r - r0] = make_float4(mu, rs, s1 * inv_h, s2 * inv_h);
    }
  }
  __syncthreads();

  // ---- phase 2: dx and the column partials, column owners
  const int c = threadIdx.x % nvec, q = threadIdx.x / nvec;
  const bool owner = q < rs_lanes;   // threads past nvec x RS only join the barriers
  float g[8], a_dg[8], a_db[8], a_dr[8], a_dx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) g[e] = a_dg[e] = a_db[e] = a_dr[e] = a_dx[e] = 0.f;
  if (owner) unpack8(__ldg(g4 + c), g);
  const uint4* dy4 = reinterpret_cast<const uint4*>(dy);
  const uint4* x4 = reinterpret_cast<const uint4*>(x);
  const uint4* dr4 = reinterpret_cast<const uint4*>(dres);
  uint4* dx4 = reinterpret_cast<uint4*>(dx);
  auto step = [&](const uint4& ud, const uint4& ux, const uint4& ur, const float4& sr,
                  long long off) {
    float d[8], xv[8], rv[8], o[8];
    unpack8(ud, d);
    unpack8(ux, xv);
    unpack8(ur, rv);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float xh = (xv[e] - sr.x) * sr.y;
      o[e] = fmaf(sr.y, fmaf(d[e], g[e], -fmaf(xh, sr.w, sr.z)), rv[e]);
      a_dg[e] = fmaf(d[e], xh, a_dg[e]);
      a_db[e] += d[e];
      if (EXTRA) {
        a_dr[e] += rv[e];
        a_dx[e] += __bfloat162float(__float2bfloat16_rn(o[e]));   // sum of the stored dx
      }
    }
    dx4[off] = pack8(o);
  };
  if (owner) {
    int r = r0 + q;
    // four rows' loads in flight at a time (dy and x mostly come back from L1
    // or L2: phase 1 read them moments ago)
    for (; r + 3 * rs_lanes < r1; r += 4 * rs_lanes) {
      uint4 ud[4], ux[4], ur[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const long long off = (long long)(r + u * rs_lanes) * nvec + c;
        ud[u] = dy4[off];
        ux[u] = x4[off];
        ur[u] = dr4[off];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        step(ud[u], ux[u], ur[u], st[r + u * rs_lanes - r0], (long long)(r + u * rs_lanes) * nvec + c);
    }
    for (; r < r1; r += rs_lanes) {
      const long long off = (long long)r * nvec + c;
      step(dy4[off], x4[off], dr4[off], st[r - r0], off);
    }
  }

  // ---- the block's column partials (summed over the RS row lanes)
  const long long nb = gridDim.x;
  float* scratch = reinterpret_cast<float*>(ln_bwd_smem + rows_per_block);   // [RS][h]
  auto put = [&](int plane, const float (&a)[8]) {
    if (rs_lanes > 1) {
      __syncthreads();   // the previous plane's scratch has been read
      if (owner) {
        float4* sc = reinterpret_cast<float4*>(scratch + (size_t)q * h + c * 8);
        sc[0] = make_float4(a[0], a[1], a[2], a[3]);
        sc[1] = make_float4(a[4], a[5], a[6], a[7]);
      }
      __syncthreads();
    }
    if (q != 0) return;
    float t[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = a[e];
    for (int k = 1; k < rs_lanes; ++k) {
      const float4* sc = reinterpret_cast<const float4*>(scratch + (size_t)k * h + c * 8);
      const float4 u0 = sc[0], u1 = sc[1];
      t[0] += u0.x; t[1] += u0.y; t[2] += u0.z; t[3] += u0.w;
      t[4] += u1.x; t[5] += u1.y; t[6] += u1.z; t[7] += u1.w;
    }
    float4* dst = reinterpret_cast<float4*>(partial + ((plane * nb + blockIdx.x) * h) + c * 8);
    dst[0] = make_float4(t[0], t[1], t[2], t[3]);
    dst[1] = make_float4(t[4], t[5], t[6], t[7]);
  };
  put(0, a_dg);
  put(1, a_db);
  if (EXTRA) {
    put(2, a_dr);
    put(3, a_dx);
  }
}

struct OutPtrs {
  __nv_bfloat16* p[8];
};

// out[g][j] = sum_r partial[g][r][j] for one 32-column block: 8 row-lanes.
__device__ __forceinline__ void sum_rows_block(const float* __restrict__ partial, int nrows, int n,
                                               int g, int cblock, __nv_bfloat16* out) {
  __shared__ float red[8][33];
  const int cl = threadIdx.x & 31, rl = threadIdx.x >> 5;
  const int col = cblock * 32 + cl;
  const float* base = partial + (long long)g * nrows * n;
  float s = 0.f;
  if (col < n) {
#pragma unroll 8
    for (int r = rl; r < nrows; r += 8) s += base[(long long)r * n + col];
  }
  red[rl][cl] = s;
  __syncthreads();
  if (rl == 0 && col < n) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += red[k][cl];
    out[col] = __float2bfloat16_rn(t);
  }
}

struct SumJobs {
  const float* partial[kMaxSumJobs];
  int groups[kMaxSumJobs], nrows[kMaxSumJobs], n[kMaxSumJobs];
  OutPtrs out[kMaxSumJobs];
};

// Several independent row sums in one launch: blockIdx.z picks the job,
// blockIdx.y the group, blockIdx.x the 32-column block (blocks past a job's
// extent return at once).
__global__ void __launch_bounds__(256) sum_rows_multi_kernel(const __grid_constant__ SumJobs jobs) {
  const int j = blockIdx.z, g = blockIdx.y;
  if (g >= jobs.groups[j] || (int)blockIdx.x * 32 >= jobs.n[j]) return;
  sum_rows_block(jobs.partial[j], jobs.nrows[j], jobs.n[j], g, blockIdx.x, jobs.out[j].p[g]);
}

// Opts a kernel in to the large dynamic shared memory of the staged kernels
// (once per kernel and device).
cudaError_t allow_ln_smem(const void* kern) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kern, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kLnSmemBudget + 1024));
  if (e == cudaSuccess) done.insert({kern, dev});
  return e;
}

}  // namespace

int layernorm_read_clear_error(unsigned int* value) { return read_clear_unit_error(value); }

int launch_layernorm_fwd(const void* x, const void* gamma, const void* beta, float eps, int rows,
                         int h, void* y, float* mean, float* rstd, cudaStream_t s,
                         bool stats_given) {
  if (h % 8 != 0 || h > 4096 || rows <= 0) return cudaErrorInvalidValue;
  const size_t smem = (size_t)kLnFwdWarps * h * 2;   // 64 KB at most
  cudaError_t e = allow_ln_smem(reinterpret_cast<const void*>(ln_fwd_kernel));
  if (e != cudaSuccess) return e;
  const unsigned blocks = static_cast<unsigned>((rows + kLnFwdWarps - 1) / kLnFwdWarps);
  ln_fwd_kernel<<<blocks, kLnFwdWarps * 32, smem, s>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(gamma),
      static_cast<const __nv_bfloat16*>(beta), eps, rows, h, stats_given, static_cast<__nv_bfloat16*>(y),
      mean, rstd);
  return cudaGetLastError();
}

int layernorm_bwd_blocks(int rows) {
  const int rpb = ln_bwd_rows_per_block(rows);
  return (rows + rpb - 1) / rpb;
}

int launch_layernorm_bwd(const void* dy, const void* x, const void* gamma, const float* mean,
                         const float* rstd, const void* dres, int rows, int h, void* dx,
                         float* partial, bool extra_sums, cudaStream_t s, const void* row_sums,
                         int row_parts) {
  if (h % 8 != 0 || h > 8 * kLnBwdThreads || rows <= 0 || (row_sums && row_parts < 1))
    return cudaErrorInvalidValue;
  auto RS = static_cast<const float2*>(row_sums);
  const int rpb = ln_bwd_rows_per_block(rows);
  const int blocks = (rows + rpb - 1) / rpb;
  const int rs = ln_bwd_row_lanes(h);
  const int threads = (h / 8) * rs;
  const size_t smem = (size_t)rpb * sizeof(float4) + (rs > 1 ? (size_t)rs * h * sizeof(float) : 0);
  auto DY = static_cast<const __nv_bfloat16*>(dy);
  auto X = static_cast<const __nv_bfloat16*>(x);
  auto G = static_cast<const __nv_bfloat16*>(gamma);
  auto DR = static_cast<const __nv_bfloat16*>(dres);
  auto DX = static_cast<__nv_bfloat16*>(dx);
  if (extra_sums) {
    cudaError_t e = allow_ln_smem(reinterpret_cast<const void*>(ln_bwd_kernel<true>));
    if (e != cudaSuccess) return e;
    ln_bwd_kernel<true><<<blocks, threads, smem, s>>>(DY, X, G, mean, rstd, DR, rows, h, rpb, rs, RS,
                                                      row_parts, DX, partial);
  } else {
    cudaError_t e = allow_ln_smem(reinterpret_cast<const void*>(ln_bwd_kernel<false>));
    if (e != cudaSuccess) return e;
    ln_bwd_kernel<false><<<blocks, threads, smem, s>>>(DY, X, G, mean, rstd, DR, rows, h, rpb, rs,
                                                       RS, row_parts, DX, partial);
  }
  return cudaGetLastError();
}

int launch_sum_rows_multi(const SumRowsJob* jobs, int njobs, cudaStream_t s) {
  if (njobs < 1 || njobs > kMaxSumJobs) return cudaErrorInvalidValue;
  SumJobs J;
  memset(&J, 0, sizeof(J));
  int max_n = 0, max_g = 0;
  for (int j = 0; j < njobs; ++j) {
    const SumRowsJob& b = jobs[j];
    if (b.groups < 1 || b.groups > 8 || b.n <= 0 || b.nrows <= 0 || !b.partial)
      return cudaErrorInvalidValue;
    J.partial[j] = b.partial;
    J.groups[j] = b.groups;
    J.nrows[j] = b.nrows;
    J.n[j] = b.n;
    for (int g = 0; g < b.groups; ++g) J.out[j].p[g] = static_cast<__nv_bfloat16*>(b.out[g]);
    max_n = b.n > max_n ? b.n : max_n;
    max_g = b.groups > max_g ? b.groups : max_g;
  }
  dim3 grid((max_n + 31) / 32, max_g, njobs);
  sum_rows_multi_kernel<<<grid, 256, 0, s>>>(J);
  return cudaGetLastError();
}

}  // namespace tp
