// Vocab-parallel input embedding (rkmt.cn guide, section 3.3: the input layer
// is split along the vocabulary and its outputs are summed by an all-reduce).
//
// Partition i holds rows [i V/t, (i+1) V/t) of E and outputs E_i[id - i V/t]
// for the tokens whose id falls in its range, zeros for the others; the t
// outputs are summed.  Exactly one partition owns each valid id, so the sum
// has one non-zero term: the kernel reads that term from the owning
// partition's buffer directly (an id outside [0, V) gives zeros, as the sum
// of t zero contributions).  The backward scatters each token's output
// gradient into the owner's rows: an fp32 accumulator over all V rows, added
// to with vector atomics, then rounded to bf16 into each partition's gradient
// (optionally added to what is there: the tied output-embedding gradient).
#include "../../include/tplayer.h"
#include "kernels.cuh"
#include "tp_common.cuh"

namespace tp {
namespace {

struct EmbPtrs {
  const __nv_bfloat16* p[8];
};
struct EmbGradPtrs {
  __nv_bfloat16* p[8];
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// One warp per token, 16-byte accesses.
__global__ void __launch_bounds__(256) embedding_fwd_kernel(int tokens, int h, int vp, int t,
                                                            const int32_t* __restrict__ ids,
                                                            EmbPtrs emb,
                                                            __nv_bfloat16* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= tokens) return;
  const int id = ids[n];
  const int part = id >= 0 ? id / vp : -1;
  uint4* dst = reinterpret_cast<uint4*>(out + (long long)n * h);
  const int nv = h >> 3;
  if (part < 0 || part >= t) {
    for (int c = lane; c < nv; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(emb.p[part] + (long long)(id - part * vp) * h);
  for (int c = lane; c < nv; c += 32) dst[c] = __ldg(src + c);
}

// acc[id] += dout[n] for every token with a valid id (fp32, vector atomics).
__global__ void __launch_bounds__(256) embedding_scatter_kernel(int tokens, int h, int vocab,
                                                                const int32_t* __restrict__ ids,
                                                                const __nv_bfloat16* __restrict__ dout,
                                                                float* __restrict__ acc) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= tokens) return;
  const int id = ids[n];
  if (id < 0 || id >= vocab) return;
  const uint2* src = reinterpret_cast<const uint2*>(dout + (long long)n * h);
  float4* dst = reinterpret_cast<float4*>(acc + (long long)id * h);
  for (int c = lane; c < (h >> 2); c += 32) {
    const uint2 u = src[c];
    atomicAdd(dst + c, make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y)));
  }
}

__global__ void __launch_bounds__(256) zero_f32_kernel(float4* __restrict__ p, long long n4) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// demb_i[r] = bf16(acc[i vp + r] (+ demb_i[r])), 4 columns per thread.
__global__ void __launch_bounds__(256) embedding_finish_kernel(int t, int vp, int h, int accumulate,
                                                               const float* __restrict__ acc,
                                                               EmbGradPtrs demb) {
  const long long per = (long long)vp * h / 4;
  const long long total = per * t;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int part = static_cast<int>(i / per);
    const long long j = i - part * per;
    float4 v = reinterpret_cast<const float4*>(acc)[i];
    uint2* d = reinterpret_cast<uint2*>(demb.p[part]) + j;
    if (accumulate) {
      const uint2 u = *d;
      v.x += bf16_lo(u.x);
      v.y += bf16_hi(u.x);
      v.z += bf16_lo(u.y);
      v.w += bf16_hi(u.y);
    }
    *d = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
  }
}

int grid_for(long long work) {
  const long long b = (work + 255) / 256;
  return static_cast<int>(b < 148 * 8 ? (b > 0 ? b : 1) : 148 * 8);
}

}  // namespace
}  // namespace tp

using namespace tp;

extern "C" {

int vocab_parallel_embedding_forward(int t, int tokens, int hidden, int vocab, const int32_t* ids,
                                     const void* const* emb, void* out, void* stream) {
  if (t < 1 || tokens <= 0 || hidden <= 0 || vocab <= 0 || !ids || !emb || !out)
    return TP_ERR_INVALID_ARG;
  if (t > TP_MAX_PARTITIONS || vocab % t || hidden % 8) return TP_ERR_UNSUPPORTED;
  EmbPtrs e{};
  for (int i = 0; i < t; ++i) {
    if (!emb[i] || !aligned16(emb[i])) return TP_ERR_INVALID_ARG;
    e.p[i] = static_cast<const __nv_bfloat16*>(emb[i]);
  }
  if (!aligned16(out)) return TP_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  embedding_fwd_kernel<<<(tokens + 7) / 8, 256, 0, s>>>(tokens, hidden, vocab / t, t, ids, e,
                                                        static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

size_t tp_embedding_backward_workspace_bytes(int t, int tokens, int hidden, int vocab) {
  if (t < 1 || t > TP_MAX_PARTITIONS || tokens <= 0 || hidden <= 0 || vocab <= 0 || vocab % t ||
      hidden % 8)
    return 0;
  return (size_t)vocab * hidden * 4;
}

int vocab_parallel_embedding_backward(int t, int tokens, int hidden, int vocab, const int32_t* ids,
                                      const void* dout, void* const* demb, int accumulate,
                                      void* ws, size_t ws_bytes, void* stream) {
  if (t < 1 || tokens <= 0 || hidden <= 0 || vocab <= 0 || !ids || !dout || !demb || !ws)
    return TP_ERR_INVALID_ARG;
  if (t > TP_MAX_PARTITIONS || vocab % t || hidden % 8) return TP_ERR_UNSUPPORTED;
  if (ws_bytes < tp_embedding_backward_workspace_bytes(t, tokens, hidden, vocab))
    return TP_ERR_WORKSPACE;
  EmbGradPtrs g{};
  for (int i = 0; i < t; ++i) {
    if (!demb[i] || !aligned16(demb[i])) return TP_ERR_INVALID_ARG;
    g.p[i] = static_cast<__nv_bfloat16*>(demb[i]);
  }
  if (!aligned16(dout) || !aligned16(ws)) return TP_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* acc = static_cast<float*>(ws);
  const long long n4 = (long long)vocab * hidden / 4;
  zero_f32_kernel<<<grid_for(n4), 256, 0, s>>>(reinterpret_cast<float4*>(acc), n4);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  embedding_scatter_kernel<<<(tokens + 7) / 8, 256, 0, s>>>(
      tokens, hidden, vocab, ids, static_cast<const __nv_bfloat16*>(dout), acc);
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  embedding_finish_kernel<<<grid_for(n4), 256, 0, s>>>(t, vocab / t, hidden, accumulate ? 1 : 0,
                                                         acc, g);
  return cudaGetLastError() == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

}  // extern "C"
