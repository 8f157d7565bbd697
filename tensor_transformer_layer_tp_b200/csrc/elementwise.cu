// tp_gelu_eval: the device GeLU and its derivative (the functions the fused
// GEMM epilogues apply), evaluated elementwise for tests and reuse.
#include "../../include/tplayer.h"
#include "kernels.cuh"
#include "tp_common.cuh"

namespace tp {
namespace {

__global__ void __launch_bounds__(256) gelu_eval_kernel(int n, const float* __restrict__ x,
                                                        float* __restrict__ g,
                                                        float* __restrict__ dg) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float v = x[i];
    if (g) g[i] = gelu_f(v);
    if (dg) dg[i] = gelu_grad_f(v);
  }
}

}  // namespace
}  // namespace tp

extern "C" int tp_gelu_eval(int n, const float* x, float* gelu, float* dgelu, void* stream) {
  if (n < 0 || (n > 0 && !x)) return TP_ERR_INVALID_ARG;
  if (n == 0 || (!gelu && !dgelu)) return TP_OK;
  const int blocks = (n + 255) / 256 < 4 * 148 ? (n + 255) / 256 : 4 * 148;
  tp::gelu_eval_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(n, x, gelu, dgelu);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// tp_partition_sum: the all-reduce of a row-parallel linear done the explicit
// way -- every partition has written its fp32 partial product, and one pass
// sums them and applies the epilogue:
//   out[r][c] = bf16( sum_i partial_i[r][c] + bias[c] + residual[r][c] ).
namespace tp {
namespace {

struct PartialPtrs {
  const float* p[8];
};

__global__ void __launch_bounds__(256) partition_sum_kernel(int t, int rows, int cols, long long ld,
                                                            PartialPtrs parts,
                                                            const __nv_bfloat16* __restrict__ bias,
                                                            const __nv_bfloat16* __restrict__ res,
                                                            __nv_bfloat16* __restrict__ out) {
  const int c4n = cols / 4;
  const long long total = (long long)rows * c4n;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = static_cast<int>(i / c4n), c = static_cast<int>(i - (long long)r * c4n) * 4;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < t; ++g) {
      const float4 v = *reinterpret_cast<const float4*>(parts.p[g] + (long long)r * ld + c);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    if (bias) {
      const uint2 b = *reinterpret_cast<const uint2*>(bias + c);
      s.x += bf16_lo(b.x);
      s.y += bf16_hi(b.x);
      s.z += bf16_lo(b.y);
      s.w += bf16_hi(b.y);
    }
    if (res) {
      const uint2 a = *reinterpret_cast<const uint2*>(res + (long long)r * cols + c);
      s.x += bf16_lo(a.x);
      s.y += bf16_hi(a.x);
      s.z += bf16_lo(a.y);
      s.w += bf16_hi(a.y);
    }
    *reinterpret_cast<uint2*>(out + (long long)r * cols + c) =
        make_uint2(pack_bf16(s.x, s.y), pack_bf16(s.z, s.w));
  }
}

}  // namespace
}  // namespace tp

extern "C" int tp_partition_sum(int t, int rows, int cols, const float* const* partials,
                                long long ld, const void* bias, const void* residual, void* out,
                                void* stream) {
  if (t < 1 || t > 8 || rows <= 0 || cols <= 0 || cols % 4 != 0 || ld < cols || ld % 4 != 0 ||
      !partials || !out)
    return TP_ERR_INVALID_ARG;
  tp::PartialPtrs pp{};
  for (int g = 0; g < t; ++g) {
    if (!partials[g] || (reinterpret_cast<uintptr_t>(partials[g]) & 15)) return TP_ERR_INVALID_ARG;
    pp.p[g] = partials[g];
  }
  if ((reinterpret_cast<uintptr_t>(out) & 7) || (reinterpret_cast<uintptr_t>(bias) & 7) ||
      (reinterpret_cast<uintptr_t>(residual) & 7))
    return TP_ERR_INVALID_ARG;
  const long long work = (long long)rows * (cols / 4);
  const long long want = (work + 255) / 256;
  const int blocks = static_cast<int>(want < 148 * 8 ? want : 148 * 8);
  tp::partition_sum_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      t, rows, cols, ld, pp, static_cast<const __nv_bfloat16*>(bias),
      static_cast<const __nv_bfloat16*>(residual), static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// Backward of a hidden-output dropout: out = g * keep / (1 - p) over [rows, h]
// bf16, with per-block column sums of out (the bias gradient of the dropped
// output is their total).  Block b walks rows [b rpb, (b+1) rpb); thread j
// owns the 8-column chunks j, j + 256, ... (16-byte accesses; two generator
// calls per chunk and row).
namespace tp {
namespace {

constexpr int kDropBwdThreads = 256;
constexpr int kDropBwdChunks = 2;   // 8-column chunks per thread: h <= 4096

__global__ void __launch_bounds__(kDropBwdThreads) dropout_bwd_kernel(
    const __nv_bfloat16* __restrict__ g, __nv_bfloat16* __restrict__ out, int rows, int h, int rpb,
    DropSite d, float* __restrict__ partial) {
  const int r0 = blockIdx.x * rpb, r1 = min(rows, r0 + rpb);
  const int nchunk = h / 8;
  float acc[kDropBwdChunks][8];
#pragma unroll
  for (int c = 0; c < kDropBwdChunks; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[c][e] = 0.f;
  for (int r = r0; r < r1; ++r) {
#pragma unroll
    for (int c = 0; c < kDropBwdChunks; ++c) {
      const int ch = threadIdx.x + c * kDropBwdThreads;
      if (ch >= nchunk) continue;
      const long long off = (long long)r * h + ch * 8;
      const uint4 u = *reinterpret_cast<const uint4*>(g + off);
      const uint32_t keep = drop_keep4(d, static_cast<uint32_t>(r), 2u * ch) |
                            (drop_keep4(d, static_cast<uint32_t>(r), 2u * ch + 1u) << 4);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      float v[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = ((keep >> (2 * e)) & 1u) ? bf16_lo(w[e]) * d.scale : 0.f;
        v[2 * e + 1] = ((keep >> (2 * e + 1)) & 1u) ? bf16_hi(w[e]) * d.scale : 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[c][e] += v[e];
      *reinterpret_cast<uint4*>(out + off) = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                        pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
    }
  }
#pragma unroll
  for (int c = 0; c < kDropBwdChunks; ++c) {
    const int ch = threadIdx.x + c * kDropBwdThreads;
    if (ch >= nchunk) continue;
    float4* dst = reinterpret_cast<float4*>(partial + (long long)blockIdx.x * h + ch * 8);
    dst[0] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
    dst[1] = make_float4(acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
  }
}

int dropout_bwd_rows_per_block(int rows) {
  const int blocks = rows < 2 * 148 ? rows : 2 * 148;
  return (rows + blocks - 1) / blocks;
}

}  // namespace

int dropout_bwd_blocks(int rows) {
  const int rpb = dropout_bwd_rows_per_block(rows);
  return (rows + rpb - 1) / rpb;
}

int launch_dropout_bwd(const void* g, void* out, int rows, int h, const DropSite& d, float* partial,
                       cudaStream_t s) {
  if (rows <= 0 || h % 8 || h / 8 > kDropBwdThreads * kDropBwdChunks) return cudaErrorInvalidValue;
  const int rpb = dropout_bwd_rows_per_block(rows);
  dropout_bwd_kernel<<<dropout_bwd_blocks(rows), kDropBwdThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(g), static_cast<__nv_bfloat16*>(out), rows, h, rpb, d,
      partial);
  return cudaGetLastError();
}

// out = residual + drop(sum + bias) over [rows][h] bf16: the row-parallel
// linear's output once its partition sum has arrived from the other devices
// (the same values the summed GEMM's bias / dropout / residual epilogue forms
// when all partitions share one device; the dropout mask is keyed by the
// element's global (row, column)).  One thread per 8 columns of a row.
__global__ void __launch_bounds__(256) bias_drop_residual_kernel(
    const __nv_bfloat16* __restrict__ sum, const __nv_bfloat16* __restrict__ bias,
    const __nv_bfloat16* __restrict__ residual, __nv_bfloat16* __restrict__ out, int rows, int h,
    DropSite d) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nchunk = h / 8;
  if (idx >= (long long)rows * nchunk) return;
  const int r = static_cast<int>(idx / nchunk), ch = static_cast<int>(idx - (long long)r * nchunk);
  const long long off = (long long)r * h + ch * 8;
  const uint4 a = *reinterpret_cast<const uint4*>(sum + off);
  const uint4 bb = *reinterpret_cast<const uint4*>(bias + ch * 8);
  const uint4 rr = *reinterpret_cast<const uint4*>(residual + off);
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {bb.x, bb.y, bb.z, bb.w},
                 wr[4] = {rr.x, rr.y, rr.z, rr.w};
  const uint32_t keep = d.thresh ? (drop_keep4(d, static_cast<uint32_t>(r), 2u * ch) |
                                    (drop_keep4(d, static_cast<uint32_t>(r), 2u * ch + 1u) << 4))
                                 : 0xFFu;
  const float sc = d.thresh ? d.scale : 1.f;
  float o[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float v0 = bf16_lo(wa[e]) + bf16_lo(wb[e]), v1 = bf16_hi(wa[e]) + bf16_hi(wb[e]);
    o[2 * e] = bf16_lo(wr[e]) + (((keep >> (2 * e)) & 1u) ? v0 * sc : 0.f);
    o[2 * e + 1] = bf16_hi(wr[e]) + (((keep >> (2 * e + 1)) & 1u) ? v1 * sc : 0.f);
  }
  *reinterpret_cast<uint4*>(out + off) = make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]),
                                                    pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
}

int launch_bias_drop_residual(const void* sum, const void* bias, const void* residual, void* out,
                              int rows, int h, const DropSite& d, cudaStream_t s) {
  if (rows <= 0 || h % 8) return cudaErrorInvalidValue;
  const long long n = (long long)rows * (h / 8);
  bias_drop_residual_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(sum), static_cast<const __nv_bfloat16*>(bias),
      static_cast<const __nv_bfloat16*>(residual), static_cast<__nv_bfloat16*>(out), rows, h, d);
  return cudaGetLastError();
}

}  // namespace tp

// tp_selftest_wait_timeout: one thread waits on a shared-memory barrier that
// nothing arrives on; the bounded wait gives up after its time limit, records
// a timeout in this unit's error word and the kernel returns.
namespace tp {
namespace {

__global__ void wait_timeout_selftest_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, DEV_ERR_TIMEOUT_FULL, 99);
}

}  // namespace

int elementwise_read_clear_error(unsigned int* value) { return read_clear_unit_error(value); }

}  // namespace tp

extern "C" int tp_selftest_wait_timeout(void* stream) {
  tp::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}
