// LayerNorm forward/backward and column reductions (bandwidth-bound kernels).
//
// LayerNorm is replicated in Megatron-LM's intra-layer parallelism rather than
// split (Megatron-LM show notes, the outline item on dropout, layer
// normalisation and residual connections being duplicated to avoid
// communication), so on one device it runs once over the full hidden width.
// All loads and stores are 16-byte vectors along the hidden dimension; row
// statistics use warp shuffles.
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

// One warp per row; lane l owns 8-element vectors l, l+32, ... (NV of them).
template <int NV>
__global__ void __launch_bounds__(256) ln_fwd_kernel(const __nv_bfloat16* __restrict__ x,
                                                     const __nv_bfloat16* __restrict__ gamma,
                                                     const __nv_bfloat16* __restrict__ beta,
                                                     float eps, int rows, int h,
                                                     __nv_bfloat16* __restrict__ y,
                                                     float* __restrict__ mean,
                                                     float* __restrict__ rstd) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int nvec = h >> 3;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (long long)row * h);
  float v[NV][8];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = i * 32 + lane;
    if (c < nvec) {
      unpack8(xr[c], v[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) s += v[i][e];
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
    }
  }
  const float mu = warp_sum(s) / h;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    if (i * 32 + lane < nvec) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = v[i][e] - mu;
        q += d * d;
      }
    }
  }
  const float rs = rsqrtf(warp_sum(q) / h + eps);
  uint4* yr = reinterpret_cast<uint4*>(y + (long long)row * h);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  const uint4* b4 = reinterpret_cast<const uint4*>(beta);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = i * 32 + lane;
    if (c < nvec) {
      float g[8], b[8], o[8];
      unpack8(__ldg(g4 + c), g);
      unpack8(__ldg(b4 + c), b);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = (v[i][e] - mu) * rs * g[e] + b[e];
      yr[c] = pack8(o);
    }
  }
  if (lane == 0) {
    mean[row] = mu;
    rstd[row] = rs;
  }
}

constexpr int kLnBwdRowsPerBlock = 16;
constexpr int kLnBwdRowsPerSync = 4;

// Column-owner layout: thread j owns hidden columns [8j, 8j+8) and walks
// kLnBwdRowsPerBlock rows, kLnBwdRowsPerSync at a time (one block reduction
// per group of rows).  Per-block column partials go to `partial`:
//   plane 0: sum dy * xhat (dgamma)      plane 1: sum dy (dbeta)
//   plane 2: sum dres                    plane 3: sum dx      (only if extra)
// so a caller whose residual gradient and output are themselves the inputs of
// bias gradients gets those column sums from the same pass.
template <bool EXTRA>
__global__ void __launch_bounds__(512) ln_bwd_kernel(
    const __nv_bfloat16* __restrict__ dy, const __nv_bfloat16* __restrict__ x,
    const __nv_bfloat16* __restrict__ gamma, const float* __restrict__ mean,
    const float* __restrict__ rstd, const __nv_bfloat16* __restrict__ dres, int rows, int h,
    __nv_bfloat16* __restrict__ dx, float* __restrict__ partial) {
  constexpr int R = kLnBwdRowsPerSync;
  __shared__ float2 red[2][R][16];
  const int nvec = h >> 3;
  const int j = threadIdx.x;
  const bool active = j < nvec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  float g[8], acc_dg[8], acc_db[8], acc_dr[8], acc_dx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc_dg[e] = acc_db[e] = acc_dr[e] = acc_dx[e] = 0.f;
  if (active) unpack8(__ldg(reinterpret_cast<const uint4*>(gamma) + j), g);
  const int r0 = blockIdx.x * kLnBwdRowsPerBlock;
  for (int rb = r0, it = 0; rb < min(rows, r0 + kLnBwdRowsPerBlock); rb += R, ++it) {
    // All loads of the row group first (packed bf16): one memory round trip per R rows.
    uint4 udy[R], ux[R], ures[R];
    float mu[R], rs[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int r = rb + k;
      const bool ok = active && r < rows;
      udy[k] = ok ? reinterpret_cast<const uint4*>(dy + (long long)r * h)[j] : make_uint4(0, 0, 0, 0);
      ux[k] = ok ? reinterpret_cast<const uint4*>(x + (long long)r * h)[j] : make_uint4(0, 0, 0, 0);
      ures[k] = ok ? reinterpret_cast<const uint4*>(dres + (long long)r * h)[j] : make_uint4(0, 0, 0, 0);
      mu[k] = r < rows ? mean[r] : 0.f;
      rs[k] = r < rows ? rstd[r] : 0.f;
    }
    float s1[R], s2[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      float d[8], xv[8];
      unpack8(udy[k], d);
      unpack8(ux[k], xv);
      s1[k] = s2[k] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xh = (xv[e] - mu[k]) * rs[k];
        const float gd = d[e] * g[e];
        s1[k] += gd;
        s2[k] += gd * xh;
        acc_dg[e] += d[e] * xh;
        acc_db[e] += d[e];
      }
    }
#pragma unroll
    for (int k = 0; k < R; ++k) {
      s1[k] = warp_sum(s1[k]);
      s2[k] = warp_sum(s2[k]);
    }
    float2 (*slot)[16] = red[it & 1];
    if (lane == 0) {
#pragma unroll
      for (int k = 0; k < R; ++k) slot[k][warp] = make_float2(s1[k], s2[k]);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < R; ++k) {
      float t1 = 0.f, t2 = 0.f;
      for (int w = 0; w < nwarps; ++w) {
        t1 += slot[k][w].x;
        t2 += slot[k][w].y;
      }
      const int r = rb + k;
      if (active && r < rows) {
        const float inv_h = 1.0f / h;
        const float m1 = t1 * inv_h, m2 = t2 * inv_h;
        float d[8], xv[8], rv[8], o[8];
        unpack8(udy[k], d);
        unpack8(ux[k], xv);
        unpack8(ures[k], rv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xh = (xv[e] - mu[k]) * rs[k];
          o[e] = rv[e] + rs[k] * (d[e] * g[e] - m1 - xh * m2);
          if (EXTRA) {
            acc_dr[e] += rv[e];
            acc_dx[e] += __bfloat162float(__float2bfloat16_rn(o[e]));   // sum of the stored dx
          }
        }
        reinterpret_cast<uint4*>(dx + (long long)r * h)[j] = pack8(o);
      }
    }
  }
  if (active) {
    const long long nb = gridDim.x;
    auto put = [&](int plane, const float (&a)[8]) {
      float4* dst = reinterpret_cast<float4*>(partial + ((plane * nb + blockIdx.x) * h) + j * 8);
      dst[0] = make_float4(a[0], a[1], a[2], a[3]);
      dst[1] = make_float4(a[4], a[5], a[6], a[7]);
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

// out[g][j] = sum_r partial[g][r][j]: 32 columns x 8 row-lanes per block.
__global__ void __launch_bounds__(256) sum_rows_kernel(const float* __restrict__ partial,
                                                       int nrows, int n, OutPtrs outs) {
  __shared__ float red[8][33];
  const int g = blockIdx.y;
  const int cl = threadIdx.x & 31, rl = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + cl;
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
    outs.p[g][col] = __float2bfloat16_rn(t);
  }
}

}  // namespace

int launch_layernorm_fwd(const void* x, const void* gamma, const void* beta, float eps, int rows,
                         int h, void* y, float* mean, float* rstd, cudaStream_t s) {
  if (h % 8 != 0 || h > 4096 || rows <= 0) return cudaErrorInvalidValue;
  const int nv = (h / 8 + 31) / 32;
  const int warps = 8;
  dim3 grid((rows + warps - 1) / warps);
  auto X = static_cast<const __nv_bfloat16*>(x);
  auto G = static_cast<const __nv_bfloat16*>(gamma);
  auto B = static_cast<const __nv_bfloat16*>(beta);
  auto Y = static_cast<__nv_bfloat16*>(y);
#define TP_LN_CASE(N)                                                                    \
  case N:                                                                                \
    ln_fwd_kernel<N><<<grid, warps * 32, 0, s>>>(X, G, B, eps, rows, h, Y, mean, rstd); \
    break;
  switch (nv) {
    TP_LN_CASE(1) TP_LN_CASE(2) TP_LN_CASE(3) TP_LN_CASE(4) TP_LN_CASE(5) TP_LN_CASE(6)
    TP_LN_CASE(7) TP_LN_CASE(8) TP_LN_CASE(9) TP_LN_CASE(10) TP_LN_CASE(11) TP_LN_CASE(12)
    TP_LN_CASE(13) TP_LN_CASE(14) TP_LN_CASE(15) TP_LN_CASE(16)
    default: return cudaErrorInvalidValue;
  }
#undef TP_LN_CASE
  return cudaGetLastError();
}

int layernorm_bwd_blocks(int rows) { return (rows + kLnBwdRowsPerBlock - 1) / kLnBwdRowsPerBlock; }

int launch_layernorm_bwd(const void* dy, const void* x, const void* gamma, const float* mean,
                         const float* rstd, const void* dres, int rows, int h, void* dx,
                         float* partial, bool extra_sums, cudaStream_t s) {
  if (h % 8 != 0 || h > 4096 || rows <= 0) return cudaErrorInvalidValue;
  const int threads = ((h / 8 + 31) / 32) * 32;
  auto DY = static_cast<const __nv_bfloat16*>(dy);
  auto X = static_cast<const __nv_bfloat16*>(x);
  auto G = static_cast<const __nv_bfloat16*>(gamma);
  auto DR = static_cast<const __nv_bfloat16*>(dres);
  auto DX = static_cast<__nv_bfloat16*>(dx);
  if (extra_sums)
    ln_bwd_kernel<true><<<layernorm_bwd_blocks(rows), threads, 0, s>>>(DY, X, G, mean, rstd, DR,
                                                                      rows, h, DX, partial);
  else
    ln_bwd_kernel<false><<<layernorm_bwd_blocks(rows), threads, 0, s>>>(DY, X, G, mean, rstd, DR,
                                                                       rows, h, DX, partial);
  return cudaGetLastError();
}

int launch_sum_rows(const float* partial, int groups, int nrows, int n, void* const* out,
                    cudaStream_t s) {
  if (groups < 1 || groups > 8 || n <= 0 || nrows <= 0) return cudaErrorInvalidValue;
  OutPtrs o;
  for (int g = 0; g < 8; ++g) o.p[g] = g < groups ? static_cast<__nv_bfloat16*>(out[g]) : nullptr;
  dim3 grid((n + 31) / 32, groups);
  sum_rows_kernel<<<grid, 256, 0, s>>>(partial, nrows, n, o);
  return cudaGetLastError();
}

}  // namespace tp
