// Vocab-parallel cross-entropy kernels (bandwidth-bound).
//
// The output embedding is split along the vocabulary; instead of gathering
// the b x s x v logits, every partition reduces its own slice to three numbers
// per token -- the max, the sum of exp(z - max), and the target logit if the
// target falls in its slice -- and only those are combined (Megatron-LM show
// notes, the outline item on parallelising the output embedding over the
// vocabulary and fusing the loss; rkmt.cn guide, section 3.3: the all-gather
// of the output layer is deferred and fused with the cross-entropy).
//
// One warp streams one (partition, token) row of fp32 logits with 16-byte
// loads; the statistics use an online max / rescaled sum and warp shuffles.
#include "kernels.cuh"
#include "tp_common.cuh"

namespace tp {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct LogitPtrs {
  const float* p[8];
};
struct GradPtrs {
  __nv_bfloat16* p[8];
};

__device__ __forceinline__ float4 ld_stream(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

// Merge (m2, s2) into (m, s), both in the log2 domain: s = sum 2^(x - m).
__device__ __forceinline__ void merge_ms(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;
  s = s * exp2f(m - mn) + s2 * exp2f(m2 - mn);
  m = mn;
}

__global__ void __launch_bounds__(256) xent_stats_kernel(int t, int T, int vp, LogitPtrs z,
                                                         const int32_t* __restrict__ target,
                                                         float* __restrict__ stats) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (gw >= t * T) return;
  const int i = gw / T;
  const int n = gw - i * T;
  const float* row = z.p[i] + (long long)n * vp;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  const int nv = vp >> 2;
  // Work in the log2 domain: x = z * log2(e).
  float m = -INFINITY, s = 0.f;
  int c = lane;
  for (; c + 96 < nv; c += 128) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = ld_stream(row4 + c + 32 * u);
    float mx = m;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      mx = fmaxf(mx, fmaxf(fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w)) * kLog2e);
    if (mx != m) {
      s *= exp2f(m - mx);
      m = mx;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      s += exp2f(fmaf(v[u].x, kLog2e, -m)) + exp2f(fmaf(v[u].y, kLog2e, -m)) +
           exp2f(fmaf(v[u].z, kLog2e, -m)) + exp2f(fmaf(v[u].w, kLog2e, -m));
    }
  }
  for (; c < nv; c += 32) {
    const float4 v = ld_stream(row4 + c);
    const float mx = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)) * kLog2e);
    if (mx != m) {
      s *= exp2f(m - mx);
      m = mx;
    }
    s += exp2f(fmaf(v.x, kLog2e, -m)) + exp2f(fmaf(v.y, kLog2e, -m)) +
         exp2f(fmaf(v.z, kLog2e, -m)) + exp2f(fmaf(v.w, kLog2e, -m));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    merge_ms(m, s, m2, s2);
  }
  if (lane == 0) {
    const int local = target[n] - i * vp;
    const float zt = (local >= 0 && local < vp) ? row[local] : 0.f;
    const long long tt = (long long)t * T;
    stats[gw] = m * kLn2;                 // natural-log max
    stats[tt + gw] = s;                   // sum exp(z - max)
    stats[2 * tt + gw] = zt;
  }
}

// lse[n] = M + log(sum_i s_i exp(m_i - M)), loss_tok[n] = lse - sum_i z_i;
// block partial sums of loss_tok go to block_sum.
__global__ void __launch_bounds__(256) xent_combine_kernel(int t, int T,
                                                           const float* __restrict__ stats,
                                                           float* __restrict__ lse,
                                                           float* __restrict__ loss_tok,
                                                           float* __restrict__ block_sum) {
  __shared__ float red[8];
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  float tok = 0.f;
  if (n < T) {
    const long long tt = (long long)t * T;
    float mx = -INFINITY;
    for (int i = 0; i < t; ++i) mx = fmaxf(mx, stats[i * T + n]);
    float ssum = 0.f, zt = 0.f;
    for (int i = 0; i < t; ++i) {
      ssum += stats[tt + i * T + n] * expf(stats[i * T + n] - mx);
      zt += stats[2 * tt + i * T + n];
    }
    const float l = mx + logf(ssum);
    tok = l - zt;
    lse[n] = l;
    if (loss_tok) loss_tok[n] = tok;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tok += __shfl_xor_sync(0xffffffffu, tok, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = tok;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b += red[w];
    block_sum[blockIdx.x] = b;
  }
}

__global__ void __launch_bounds__(1024) xent_mean_kernel(const float* __restrict__ block_sum,
                                                         int nblocks, int T,
                                                         float* __restrict__ loss) {
  __shared__ float red[32];
  float v = 0.f;
  for (int b = threadIdx.x; b < nblocks; b += blockDim.x) v += block_sum[b];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
    *loss = s / T;
  }
}

// dz = (exp(z - lse) - onehot) / T, streamed per (partition, token) row.
__global__ void __launch_bounds__(256) xent_grad_kernel(int t, int T, int vp, LogitPtrs z,
                                                        const int32_t* __restrict__ target,
                                                        const float* __restrict__ lse,
                                                        GradPtrs dz) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (gw >= t * T) return;
  const int i = gw / T;
  const int n = gw - i * T;
  const float4* row4 = reinterpret_cast<const float4*>(z.p[i] + (long long)n * vp);
  uint2* out2 = reinterpret_cast<uint2*>(dz.p[i] + (long long)n * vp);
  const float l2 = lse[n] * kLog2e;
  const float inv_t = 1.0f / T;
  const int local = target[n] - i * vp;
  const int nv = vp >> 2;
  int c = lane;
  for (; c + 96 < nv; c += 128) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = ld_stream(row4 + c + 32 * u);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e0 = (c + 32 * u) * 4;
      float g0 = exp2f(fmaf(v[u].x, kLog2e, -l2)), g1 = exp2f(fmaf(v[u].y, kLog2e, -l2));
      float g2 = exp2f(fmaf(v[u].z, kLog2e, -l2)), g3 = exp2f(fmaf(v[u].w, kLog2e, -l2));
      if (local >= e0 && local < e0 + 4) {
        const int k = local - e0;
        if (k == 0) g0 -= 1.f;
        if (k == 1) g1 -= 1.f;
        if (k == 2) g2 -= 1.f;
        if (k == 3) g3 -= 1.f;
      }
      out2[c + 32 * u] = make_uint2(pack_bf16(g0 * inv_t, g1 * inv_t), pack_bf16(g2 * inv_t, g3 * inv_t));
    }
  }
  for (; c < nv; c += 32) {
    const float4 v = ld_stream(row4 + c);
    const int e0 = c * 4;
    float g0 = exp2f(fmaf(v.x, kLog2e, -l2)), g1 = exp2f(fmaf(v.y, kLog2e, -l2));
    float g2 = exp2f(fmaf(v.z, kLog2e, -l2)), g3 = exp2f(fmaf(v.w, kLog2e, -l2));
    if (local >= e0 && local < e0 + 4) {
      const int k = local - e0;
      if (k == 0) g0 -= 1.f;
      if (k == 1) g1 -= 1.f;
      if (k == 2) g2 -= 1.f;
      if (k == 3) g3 -= 1.f;
    }
    out2[c] = make_uint2(pack_bf16(g0 * inv_t, g1 * inv_t), pack_bf16(g2 * inv_t, g3 * inv_t));
  }
}

// ---------------------------------------------------------------- fused path
//
// The logits GEMM's epilogue has already reduced every (token, 256-column
// tile) of every partition to (max, sum 2^(x - max)) in log2 units and picked
// out the target's logit, so no fp32 logit reaches HBM.  Here each partition's
// tiles are folded into its (max, sum-exp) pair -- the triple the method has
// each partition report -- and the t triples are combined as in
// xent_combine_kernel.
// One warp per token: for each partition, the lanes fold its tiles (a lane
// per tile, then a shuffle merge of the lanes' pairs), giving the partition's
// (max, sum-exp); lane 0 combines the t pairs.
__device__ __forceinline__ void warp_merge_ms(float& m, float& s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    merge_ms(m, s, m2, s2);
  }
}

__global__ void __launch_bounds__(256) xent_tile_combine_kernel(
    int t, int T, int ntiles, int vocab, const float2* __restrict__ tile_stats,
    const float* __restrict__ ztgt, const int32_t* __restrict__ target, float* __restrict__ lse,
    float* __restrict__ loss_tok, float* __restrict__ block_sum) {
  __shared__ float red[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = blockIdx.x * 8 + warp;
  float tok = 0.f;
  if (n < T) {
    float big = -INFINITY, ssum = 0.f;
    for (int i = 0; i < t; ++i) {            // partition i: fold its tiles
      float m = -INFINITY, sum = 0.f;
      for (int k = lane; k < ntiles; k += 32) {
        const float2 v = tile_stats[((long long)i * ntiles + k) * T + n];
        merge_ms(m, sum, v.x, v.y);
      }
      warp_merge_ms(m, sum);
      merge_ms(big, ssum, m, sum);             // combine the partitions' pairs
    }
    const int y = target[n];
    const float zt = (y >= 0 && y < vocab) ? ztgt[n] : 0.f;
    const float l = (big + log2f(ssum)) * kLn2;
    tok = l - zt;
    if (lane == 0) {
      lse[n] = l;
      if (loss_tok) loss_tok[n] = tok;
    }
  }
  if (lane == 0) red[warp] = tok;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f;
    for (int w = 0; w < 8; ++w) b += red[w];
    block_sum[blockIdx.x] = b;
  }
}

// ---------------------------------------------------------------- loss across devices
// Partition `rank` of the vocabulary on this device (one partition per call).
// Step 1 (after the logits GEMM): fold the partition's tiles of every token
// to its log-sum-exp over the slice, lse_i (natural units), into lse_loc and
// comm[0]; the target logit, or 0 when the target lies in another slice, into
// comm[2].  The caller then takes the max over ranks of comm[0] (M).
__global__ void __launch_bounds__(256) xent_rank_fold_kernel(int T, int ntiles,
                                                             const float2* __restrict__ tile_stats,
                                                             const float* __restrict__ ztgt,
                                                             float* __restrict__ lse_loc,
                                                             float* __restrict__ comm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = blockIdx.x * 8 + warp;
  if (n >= T) return;
  float m = -INFINITY, sum = 0.f;
  for (int k = lane; k < ntiles; k += 32) {
    const float2 v = tile_stats[(long long)k * T + n];
    merge_ms(m, sum, v.x, v.y);
  }
  warp_merge_ms(m, sum);
  if (lane == 0) {
    const float l = (m + log2f(sum)) * kLn2;
    lse_loc[n] = l;
    comm[n] = l;
    comm[2LL * T + n] = ztgt[n];
  }
}

// Step 2 (comm[0] = M, the max over ranks): comm[1] = exp(lse_i - M); the
// caller then sums comm[1] and comm[2] over ranks (S, and the target logit).
__global__ void __launch_bounds__(256) xent_rank_exp_kernel(int T, const float* __restrict__ lse_loc,
                                                            float* __restrict__ comm) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n < T) comm[T + n] = __expf(lse_loc[n] - comm[n]);
}

// Step 3: lse = M + log S and the per-token loss lse - z_target, with
// per-block sums for the mean (block_sum[ceil(T / 256)]).
__global__ void __launch_bounds__(256) xent_rank_finish_kernel(int T, const float* __restrict__ comm,
                                                               float* __restrict__ lse,
                                                               float* __restrict__ loss_tok,
                                                               float* __restrict__ block_sum) {
  __shared__ float red[8];
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  float tok = 0.f;
  if (n < T) {
    const float l = comm[n] + logf(comm[T + n]);
    tok = l - comm[2LL * T + n];
    lse[n] = l;
    if (loss_tok) loss_tok[n] = tok;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tok += __shfl_xor_sync(0xffffffffu, tok, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = tok;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f;
    for (int w = 0; w < 8; ++w) b += red[w];
    block_sum[blockIdx.x] = b;
  }
}

// 2^x on the special-function unit (ex2.approx.ftz: relative error about
// 2^-22, results below the normal range flush to zero).  The logit gradient
// is rounded to bf16 (2^-9), so this is exact enough, and one instruction
// per element keeps the in-place gradient pass on the memory roofline.
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct BfPtrs {
  __nv_bfloat16* p[8];
};

__device__ __forceinline__ uint4 ld_stream_u4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// dz = (exp(z - lse) - onehot) / T from the bf16 logits the fused GEMM
// stored, written over them (bf16), streamed per (partition, token) row with
// 16-byte accesses.
__global__ void __launch_bounds__(256) xent_grad_bf16_kernel(int t, int T, int vp, int group0, BfPtrs z,
                                                             const int32_t* __restrict__ target,
                                                             const float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (gw >= t * T) return;
  const int i = gw / T;
  const int n = gw - i * T;
  uint4* row = reinterpret_cast<uint4*>(z.p[i] + (long long)n * vp);
  const float l2 = lse[n] * kLog2e;
  const float inv_t = 1.0f / T;
  const int local = target[n] - (i + group0) * vp;
  const int nv = vp >> 3;
  auto grad8 = [&](uint4 u, int e0) -> uint4 {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float g[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      g[2 * k] = ex2_fast(fmaf(bf16_lo(w[k]), kLog2e, -l2));
      g[2 * k + 1] = ex2_fast(fmaf(bf16_hi(w[k]), kLog2e, -l2));
    }
    if (local >= e0 && local < e0 + 8) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (local - e0 == k) g[k] -= 1.f;
    }
    return make_uint4(pack_bf16(g[0] * inv_t, g[1] * inv_t), pack_bf16(g[2] * inv_t, g[3] * inv_t),
                      pack_bf16(g[4] * inv_t, g[5] * inv_t), pack_bf16(g[6] * inv_t, g[7] * inv_t));
  };
  int c = lane;
  for (; c + 96 < nv; c += 128) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = ld_stream_u4(row + c + 32 * u);
#pragma unroll
    for (int u = 0; u < 4; ++u) row[c + 32 * u] = grad8(v[u], (c + 32 * u) * 8);
  }
  for (; c < nv; c += 32) row[c] = grad8(ld_stream_u4(row + c), c * 8);
}

}  // namespace

int launch_xent_stats(int t, int tokens, int vp, const float* const* logits, const int32_t* target,
                      float* stats, cudaStream_t s) {
  if (t < 1 || t > 8 || vp % 4 != 0 || tokens <= 0) return cudaErrorInvalidValue;
  LogitPtrs z;
  for (int i = 0; i < 8; ++i) z.p[i] = i < t ? logits[i] : nullptr;
  const long long rows = (long long)t * tokens;
  xent_stats_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(t, tokens, vp, z, target, stats);
  return cudaGetLastError();
}

int launch_xent_combine(int t, int tokens, const float* stats, float* lse, float* loss_tok,
                        float* loss, cudaStream_t s) {
  // Block partial sums of the per-token loss are kept right after lse, so the
  // caller's lse buffer holds tokens + ceil(tokens / 256) floats.
  const int nb = (tokens + 255) / 256;
  float* block_sum = lse + tokens;
  xent_combine_kernel<<<nb, 256, 0, s>>>(t, tokens, stats, lse, loss_tok, block_sum);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  xent_mean_kernel<<<1, 1024, 0, s>>>(block_sum, nb, tokens, loss);
  return cudaGetLastError();
}

int launch_xent_grad(int t, int tokens, int vp, const float* const* logits, const int32_t* target,
                     const float* lse, void* const* dlogits, cudaStream_t s) {
  if (t < 1 || t > 8 || vp % 4 != 0 || tokens <= 0) return cudaErrorInvalidValue;
  LogitPtrs z;
  GradPtrs g;
  for (int i = 0; i < 8; ++i) {
    z.p[i] = i < t ? logits[i] : nullptr;
    g.p[i] = i < t ? static_cast<__nv_bfloat16*>(dlogits[i]) : nullptr;
  }
  const long long rows = (long long)t * tokens;
  xent_grad_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(t, tokens, vp, z, target, lse, g);
  return cudaGetLastError();
}

}  // namespace tp

namespace tp {

int launch_xent_tile_combine(int t, int tokens, int ntiles, int vocab, const float2* tile_stats,
                             const float* ztgt, const int32_t* target, float* lse, float* loss_tok,
                             float* loss, cudaStream_t s) {
  if (t < 1 || t > 8 || tokens <= 0 || ntiles <= 0) return cudaErrorInvalidValue;
  // 8 tokens per block: block_sum needs ceil(tokens / 8) floats, which the
  // caller's lse buffer provides (tokens + ceil(tokens / 8) floats)
  const int nb = (tokens + 7) / 8;
  float* block_sum = lse + tokens;
  xent_tile_combine_kernel<<<nb, 256, 0, s>>>(t, tokens, ntiles, vocab, tile_stats, ztgt, target,
                                               lse, loss_tok, block_sum);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  xent_mean_kernel<<<1, 1024, 0, s>>>(block_sum, nb, tokens, loss);
  return cudaGetLastError();
}

int launch_xent_rank_fold(int tokens, int ntiles, const float2* tile_stats, const float* ztgt,
                          float* lse_loc, float* comm, cudaStream_t s) {
  if (tokens <= 0 || ntiles <= 0) return cudaErrorInvalidValue;
  xent_rank_fold_kernel<<<(tokens + 7) / 8, 256, 0, s>>>(tokens, ntiles, tile_stats, ztgt, lse_loc, comm);
  return cudaGetLastError();
}

int launch_xent_rank_exp(int tokens, const float* lse_loc, float* comm, cudaStream_t s) {
  if (tokens <= 0) return cudaErrorInvalidValue;
  xent_rank_exp_kernel<<<(tokens + 255) / 256, 256, 0, s>>>(tokens, lse_loc, comm);
  return cudaGetLastError();
}

int launch_xent_rank_finish(int tokens, const float* comm, float* lse, float* loss_tok, float* loss,
                            cudaStream_t s) {
  if (tokens <= 0) return cudaErrorInvalidValue;
  // block sums after lse: the caller's lse buffer holds tokens + ceil(tokens / 8) floats
  const int nb = (tokens + 255) / 256;
  float* block_sum = lse + tokens;
  xent_rank_finish_kernel<<<nb, 256, 0, s>>>(tokens, comm, lse, loss_tok, block_sum);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  xent_mean_kernel<<<1, 1024, 0, s>>>(block_sum, nb, tokens, loss);
  return cudaGetLastError();
}

int launch_xent_grad_bf16(int t, int tokens, int vp, void* const* logits, const int32_t* target,
                          const float* lse, cudaStream_t s, int group0) {
  if (t < 1 || t > 8 || vp % 8 != 0 || tokens <= 0) return cudaErrorInvalidValue;
  BfPtrs z;
  for (int i = 0; i < 8; ++i) z.p[i] = i < t ? static_cast<__nv_bfloat16*>(logits[i]) : nullptr;
  const long long rows = (long long)t * tokens;
  xent_grad_bf16_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(t, tokens, vp, group0, z, target,
                                                                    lse);
  return cudaGetLastError();
}

}  // namespace tp
