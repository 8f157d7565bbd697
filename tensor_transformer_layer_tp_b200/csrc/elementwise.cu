// tp_gelu_eval: the device GeLU and its derivative (the functions the fused
// GEMM epilogues apply), evaluated elementwise for tests and reuse.
#include "../../include/tplayer.h"
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
