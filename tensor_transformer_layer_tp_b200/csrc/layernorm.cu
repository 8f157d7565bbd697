// LayerNorm forward/backward and column reductions (bandwidth-bound kernels).
//
// LayerNorm is replicated in Megatron-LM's intra-layer parallelism rather than
// split (Megatron-LM show notes, the outline item on dropout, layer
// normalisation and residual connections being duplicated to avoid
// communication), so on one device it runs once over the full hidden width.
// The forward keeps one row per warp in registers; the backward streams
// groups of rows through shared memory with bulk async copies into a ring,
// one block per SM over a contiguous range of rows.  Accesses are 16-byte
// vectors along the hidden dimension and row statistics use warp shuffles.
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

// Eight warp-wide sums at once by recursive halving: at each of the first
// three levels a lane keeps half of its values and adds the partner's copy of
// them, so 9 shuffles replace 8 x 5.  Returns the total of value
// (lane >> 2) & 7 (every lane holds one of the eight totals).
__device__ __forceinline__ float warp_reduce8(float (&v)[8]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int w = 16, n = 4; w >= 4; w >>= 1, n >>= 1) {
    const bool hi = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = hi ? v[i] : v[i + n];
      const float keep = hi ? v[i + n] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  float r = v[0];
  r += __shfl_xor_sync(0xffffffffu, r, 2);
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r;
}

// The backward streams its rows through shared memory with bulk async copies
// (one copy per row and tensor, completion counted on an mbarrier), one block
// per SM over a contiguous range of rows, so that the next rows are in flight
// while the current ones are reduced.
constexpr int kLnBlocks = 148;   // one block per SM of a B200
constexpr uint32_t kLnSmemBudget = 224u * 1024u;   // ring bytes per block

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Rows per block for `rows` rows split over at most kLnBlocks blocks, a
// multiple of `mult`.
__host__ __device__ inline int ln_rows_per_block(int rows, int mult) {
  int nb = (rows + mult - 1) / mult;
  if (nb > kLnBlocks) nb = kLnBlocks;
  int rpb = (rows + nb - 1) / nb;
  return (rpb + mult - 1) / mult * mult;
}

// ---------------------------------------------------------------- forward, one warp per row
// A warp copies its row into shared memory with 16-byte asynchronous copies,
// all issued at once, so the SM has every row of its warps in flight (8 rows
// a block, up to 4 blocks of 48 KB per SM at h = 3072: a 4096-row tensor is
// one wave of warps); registers stay few.  Mean and variance come from one
// pass over the staged row: each 8-value vector's own mean and sum of squared
// deviations (exact two-pass over 8 values), merged into the lane's running
// pair and then across lanes by the pairwise update of Chan, Golub and
// LeVeque (1979) -- as stable as a two-pass variance.  Gamma and beta are read
// through the cache (the same for every row).
constexpr int kLnFwdWarps = 8;

// (n, mean, m2) <- the union of (n, mean, m2) and (nb, mb, m2b): counts,
// means and sums of squared deviations of two disjoint sets.
__device__ __forceinline__ void chan_merge(float& n, float& mean, float& m2, float nb, float mb,
                                           float m2b) {
  const float nt = n + nb;
  if (nt == 0.f) return;
  const float d = mb - mean;
  const float wb = nb / nt;
  mean = fmaf(d, wb, mean);
  m2 = m2 + m2b + d * d * n * wb;
  n = nt;
}

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
    float n = 0.f, m = 0.f, m2 = 0.f;
    for (int c = lane; c < nvec; c += 32) {
      float v[8];
      unpack8(row[c], v);
      const float vm = (((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]))) * 0.125f;
      float vq = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = v[e] - vm;
        vq = fmaf(d, d, vq);
      }
      chan_merge(n, m, m2, 8.f, vm, vq);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float nb = __shfl_xor_sync(0xffffffffu, n, o);
      const float mb = __shfl_xor_sync(0xffffffffu, m, o);
      const float qb = __shfl_xor_sync(0xffffffffu, m2, o);
      chan_merge(n, m, m2, nb, mb, qb);
    }
    mu = m;
    rs = rsqrtf(m2 / h + eps);
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
// Column-owner layout: thread j owns hidden columns [CPT*j, CPT*j+CPT) and
// walks the block's rows kLnBwdRows at a time (one block reduction per
// group).  Groups arrive through a ring of `stages` buffers, each holding dy,
// x and dres of kLnBwdRows rows.  CPT = 4 (up to 768 threads, h <= 3072)
// keeps registers low enough for 24 warps per SM; CPT = 8 serves h <= 4096.
// Per-block column partials go to `partial`:
//   plane 0: sum dy * xhat (dgamma)      plane 1: sum dy (dbeta)
//   plane 2: sum dres                    plane 3: sum dx      (only if extra)
// so a caller whose residual gradient and output are themselves the inputs of
// bias gradients gets those column sums from the same pass.
constexpr int kLnBwdRows = 4;

template <int CPT> struct LnVec;
template <> struct LnVec<8> { using T = uint4; };
template <> struct LnVec<4> { using T = uint2; };

__device__ __forceinline__ void unpackv(const uint4& u, float (&f)[8]) { unpack8(u, f); }
__device__ __forceinline__ void unpackv(const uint2& u, float (&f)[4]) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
  f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
}
__device__ __forceinline__ uint4 packv(const float (&f)[8]) { return pack8(f); }
__device__ __forceinline__ uint2 packv(const float (&f)[4]) {
  return make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
}

template <bool EXTRA, int CPT>
__global__ void __launch_bounds__(CPT == 4 ? 768 : 512, 1) ln_bwd_kernel(
    const __nv_bfloat16* __restrict__ dy, const __nv_bfloat16* __restrict__ x,
    const __nv_bfloat16* __restrict__ gamma, const float* __restrict__ mean,
    const float* __restrict__ rstd, const __nv_bfloat16* __restrict__ dres, int rows, int h,
    int rows_per_block, int stages, bool stats_in_smem, __nv_bfloat16* __restrict__ dx,
    float* __restrict__ partial) {
  constexpr int R = kLnBwdRows;
  using V = typename LnVec<CPT>::T;
  extern __shared__ __align__(128) uint8_t ln_smem[];
  __shared__ float red[2][2 * R][32];   // [buffer][s1 rows | s2 rows][warp]
  const uint32_t row_bytes = static_cast<uint32_t>(h) * 2u;
  const uint32_t stage_bytes = 3u * R * row_bytes;   // [tensor][row][h]
  uint64_t* full = reinterpret_cast<uint64_t*>(ln_smem + (size_t)stages * stage_bytes);
  const int nvec = h / CPT;
  const int j = threadIdx.x;
  const bool active = j < nvec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int r0 = blockIdx.x * rows_per_block;
  const int r1 = min(rows, r0 + rows_per_block);
  const int ngroups = (r1 - r0 + R - 1) / R;
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) mbar_init(smem_u32(&full[i]), 1);
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int k) {   // thread 0: group k into stage k % stages
    const int g0 = r0 + k * R;
    const int cnt = min(R, r1 - g0);
    uint8_t* st = ln_smem + (size_t)(k % stages) * stage_bytes;
    const uint32_t bar = smem_u32(&full[k % stages]);
    mbar_arrive_expect_tx(bar, 3u * cnt * row_bytes);
    for (int t = 0; t < 3; ++t)
      for (int i = 0; i < cnt; ++i)
        bulk_load(smem_u32(st + (size_t)(t * R + i) * row_bytes),
                  (t == 0 ? dy : (t == 1 ? x : dres)) + (long long)(g0 + i) * h, row_bytes, bar);
  };
  int last_issued = -1;   // thread 0 only
  if (threadIdx.x == 0)
    for (int k = 0; k < min(stages, ngroups); ++k) issue(last_issued = k);
  // the block's row statistics, read once (when they fit: stats_in_smem)
  float2* stats = reinterpret_cast<float2*>(full + stages);
  if (stats_in_smem)
    for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x)
      stats[r - r0] = make_float2(mean[r], rstd[r]);

  float g[CPT], acc_dg[CPT], acc_db[CPT], acc_dr[CPT], acc_dx[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) g[e] = acc_dg[e] = acc_db[e] = acc_dr[e] = acc_dx[e] = 0.f;
  // threads past the hidden width hold zeros (0 * uninitialised could be NaN)
  if (active) unpackv(__ldg(reinterpret_cast<const V*>(gamma) + j), g);
  const float inv_h = 1.0f / h;
  bool ok = true;
  int k = 0;
  for (; k < ngroups; ++k) {
    const int rb = r0 + k * R;
    // thread 0 polls the barrier; the block barrier passes the arrival on
    // (768 threads spinning on try_wait would take most of the issue slots)
    if (threadIdx.x == 0)
      ok = mbar_wait(smem_u32(&full[k % stages]), (k / stages) & 1, DEV_ERR_TIMEOUT_FULL, 81);
    ok = !__syncthreads_or(!ok);
    if (!ok) break;   // block-uniform exit on a timeout
    const uint8_t* st = ln_smem + (size_t)(k % stages) * stage_bytes;
    V udy[R], ux[R], ures[R];
    float mu[R], rs[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int r = rb + i;
      const bool on = active && r < r1;
      udy[i] = on ? reinterpret_cast<const V*>(st + (size_t)(0 * R + i) * row_bytes)[j] : V{};
      ux[i] = on ? reinterpret_cast<const V*>(st + (size_t)(1 * R + i) * row_bytes)[j] : V{};
      ures[i] = on ? reinterpret_cast<const V*>(st + (size_t)(2 * R + i) * row_bytes)[j] : V{};
      const float2 st2 = r >= r1         ? make_float2(0.f, 0.f)
                         : stats_in_smem ? stats[r - r0]
                                         : make_float2(mean[r], rstd[r]);
      mu[i] = st2.x;
      rs[i] = st2.y;
    }
    float s1[R], s2[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      float d[CPT], xv[CPT];
      unpackv(udy[i], d);
      unpackv(ux[i], xv);
      s1[i] = s2[i] = 0.f;
#pragma unroll
      for (int e = 0; e < CPT; ++e) {
        const float xh = (xv[e] - mu[i]) * rs[i];
        const float gd = d[e] * g[e];
        s1[i] += gd;
        s2[i] = fmaf(gd, xh, s2[i]);
        acc_dg[e] = fmaf(d[e], xh, acc_dg[e]);
        acc_db[e] += d[e];
      }
    }
    static_assert(2 * R == 8, "the row sums of a group fill one 8-value warp reduction");
    float (*slot)[32] = red[k & 1];
    {
      float v8[8];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        v8[i] = s1[i];
        v8[R + i] = s2[i];
      }
      const float tot = warp_reduce8(v8);
      if ((lane & 3) == 0) slot[(lane >> 2) & 7][warp] = tot;
    }
    __syncthreads();   // also: every thread has read stage k % stages
    if (threadIdx.x == 0 && k + stages < ngroups) issue(last_issued = k + stages);
    // every warp folds the per-warp partials itself: lane w loads warp w's
    // eight sums, one 8-value reduction, then the totals are broadcast
    float t1s[R], t2s[R];
    {
      float v8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v8[q] = lane < nwarps ? slot[q][lane] : 0.f;
      const float tot = warp_reduce8(v8);
#pragma unroll
      for (int i = 0; i < R; ++i) {
        t1s[i] = __shfl_sync(0xffffffffu, tot, i << 2);
        t2s[i] = __shfl_sync(0xffffffffu, tot, (R + i) << 2);
      }
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const float t1 = t1s[i], t2 = t2s[i];
      const int r = rb + i;
      if (active && r < r1) {
        const float m1 = t1 * inv_h, m2 = t2 * inv_h;
        // row statistics read again rather than kept live across the barrier
        const float2 st2 = stats_in_smem ? stats[r - r0] : make_float2(mean[r], rstd[r]);
        float d[CPT], xv[CPT], rv[CPT], o[CPT];
        unpackv(udy[i], d);
        unpackv(ux[i], xv);
        unpackv(ures[i], rv);
#pragma unroll
        for (int e = 0; e < CPT; ++e) {
          const float xh = (xv[e] - st2.x) * st2.y;
          o[e] = fmaf(st2.y, fmaf(d[e], g[e], -fmaf(xh, m2, m1)), rv[e]);
          if (EXTRA) {
            acc_dr[e] += rv[e];
            acc_dx[e] += __bfloat162float(__float2bfloat16_rn(o[e]));   // sum of the stored dx
          }
        }
        reinterpret_cast<V*>(dx + (long long)r * h)[j] = packv(o);
      }
    }
  }
  if (!ok && threadIdx.x == 0) {
    // After a timeout: let the copies still in flight land before the block exits.
    for (int q = k; q <= last_issued; ++q)
      mbar_wait(smem_u32(&full[q % stages]), (q / stages) & 1, DEV_ERR_TIMEOUT_DRAIN, 82);
  }
  if (active) {
    const long long nb = gridDim.x;
    auto put = [&](int plane, const float (&a)[CPT]) {
      float4* dst = reinterpret_cast<float4*>(partial + ((plane * nb + blockIdx.x) * h) + j * CPT);
#pragma unroll
      for (int q = 0; q < CPT / 4; ++q)
        dst[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
    };
    put(0, acc_dg);
    put(1, acc_db);
    if (EXTRA) {
      put(2, acc_dr);
      put(3, acc_dx);
    }
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
  const int rpb = ln_rows_per_block(rows, kLnBwdRows);
  return (rows + rpb - 1) / rpb;
}

int launch_layernorm_bwd(const void* dy, const void* x, const void* gamma, const float* mean,
                         const float* rstd, const void* dres, int rows, int h, void* dx,
                         float* partial, bool extra_sums, cudaStream_t s) {
  if (h % 8 != 0 || h > 4096 || rows <= 0) return cudaErrorInvalidValue;
  const int cpt = h <= 3072 ? 4 : 8;
  const int threads = ((h / cpt + 31) / 32) * 32;
  const uint32_t stage_bytes = 3u * kLnBwdRows * static_cast<uint32_t>(h) * 2u;
  const int rpb = ln_rows_per_block(rows, kLnBwdRows);
  const bool stats_in_smem = rpb <= 2048;   // 16 KB of (mean, rstd) pairs at most
  const uint32_t stats_bytes = stats_in_smem ? 8u * rpb : 0u;
  const int stages = min(4, static_cast<int>((kLnSmemBudget - stats_bytes) / stage_bytes));
  const size_t smem = (size_t)stages * (stage_bytes + 8) + stats_bytes;
  const int blocks = (rows + rpb - 1) / rpb;
  auto DY = static_cast<const __nv_bfloat16*>(dy);
  auto X = static_cast<const __nv_bfloat16*>(x);
  auto G = static_cast<const __nv_bfloat16*>(gamma);
  auto DR = static_cast<const __nv_bfloat16*>(dres);
  auto DX = static_cast<__nv_bfloat16*>(dx);
#define TP_LN_BWD(EX, C)                                                                       \
  {                                                                                            \
    cudaError_t e = allow_ln_smem(reinterpret_cast<const void*>(ln_bwd_kernel<EX, C>));        \
    if (e != cudaSuccess) return e;                                                            \
    ln_bwd_kernel<EX, C><<<blocks, threads, smem, s>>>(DY, X, G, mean, rstd, DR, rows, h, rpb, \
                                                       stages, stats_in_smem, DX, partial);    \
  }
  if (extra_sums) {
    if (cpt == 4) TP_LN_BWD(true, 4) else TP_LN_BWD(true, 8)
  } else {
    if (cpt == 4) TP_LN_BWD(false, 4) else TP_LN_BWD(false, 8)
  }
#undef TP_LN_BWD
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
