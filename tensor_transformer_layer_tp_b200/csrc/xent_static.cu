// vocab_parallel_xent_static: the vocab-parallel cross-entropy for callers
// that cannot allocate device memory.
//
// Who needs it: a caller whose device memory is entirely owned by another
// component -- for example a serving process or framework allocator that
// reserves the GPU at start-up and forbids further cudaMalloc -- or a plain C
// caller with no allocator at hand that cannot size, allocate and keep a
// workspace between calls.  Such a caller still owns its inputs and outputs,
// but has nowhere to put the intermediate logits, partition statistics and
// logit gradient that vocab_parallel_xent keeps in its `ws` argument.
//
// This variant keeps that scratch in a fixed array in the library's own device
// memory (g_xent_scratch below, TP_XENT_STATIC_SCRATCH_BYTES = 64 MiB).  Every
// GPU that loads the library holds the array until the process exits.
//
// Host code must not use the array's name as a device address (on the host it
// names a stand-in object): the address is looked up with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device (and again if a later call runs under another CUDA context of
// the device, e.g. after cudaDeviceReset).  Make that first call before any
// stream capture on the device.
//
// All calls share the one array and it keeps whatever the last call left in
// it.  Nothing in it needs to start at zero: every element a call reads was
// written earlier in the same call.  Calls that overlap on the GPU (on
// different streams, or from different threads without ordering) race on the
// array and give wrong results; order them on one stream.
#include <cuda.h>

#include <mutex>

#include "../../include/tplayer.h"

namespace {

constexpr size_t kScratchBytes = TP_XENT_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_xent_scratch[kScratchBytes];

// The array's device address belongs to the CUDA context the module was
// loaded into: it is looked up once per (device, context) and looked up again
// when the calling thread's current context is another one (after
// cudaDeviceReset created a new primary context, or under a context the
// caller made current itself).  cuCtxGetCurrent is reached through the
// runtime's driver entry-point query, so the library needs no libcuda link.
constexpr int kMaxDevices = 64;
struct CachedAddress {
  CUcontext ctx;
  void* addr;
};
std::mutex g_mu;
CachedAddress g_cache[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

// Device address of g_xent_scratch in the current context of the current device.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TP_ERR_UNSUPPORTED;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (!get_ctx) return TP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return TP_ERR_CUDA;
  CachedAddress& c = g_cache[dev];
  if (!ctx || ctx != c.ctx || !c.addr) {
    void* p = nullptr;   // the lookup makes the device's primary context current if none is
    if (cudaGetSymbolAddress(&p, g_xent_scratch) != cudaSuccess || !p) return TP_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return TP_ERR_CUDA;
    c.ctx = ctx;
    c.addr = p;
  }
  *out = c.addr;
  return TP_OK;
}

}  // namespace

extern "C" int vocab_parallel_xent_static(int t, int tokens, int hidden, int vocab,
                                          const void* x, const void* const* emb,
                                          const int32_t* target, float* loss,
                                          float* loss_per_token, void* dx, void* const* demb,
                                          void* stream) {
  if (t < 1 || tokens <= 0 || hidden <= 0 || vocab <= 0) return TP_ERR_INVALID_ARG;
  const size_t need = tp_xent_workspace_bytes(t, tokens, hidden, vocab);
  if (need == 0) return TP_ERR_UNSUPPORTED;
  if (need > kScratchBytes) return TP_ERR_WORKSPACE;   // beyond the fixed scratch
  void* ws = nullptr;
  const int st = scratch_address(&ws);
  if (st != TP_OK) return st;
  return vocab_parallel_xent(t, tokens, hidden, vocab, x, emb, target, loss, loss_per_token, dx,
                             demb, ws, kScratchBytes, stream);
}
