// C-ABI entry points: argument checks, carving of the saved-activation and
// scratch buffers, and the launch sequence of each call.
//
// Forward of the layer (F1..F7) and backward (B1..B7), all on one stream:
//   F1 LN1           Xn1 = LN(X)
//   F2 QKV           QKV_i = Xn1 W_qkv,i + b_qkv,i          (grouped GEMM, t outputs)
//   F3 attention     O_i, lse                               (per head of partition i)
//   F4 out-proj      H1 = X + b_o + sum_i O_i W_o,i         (partition sum in the K-loop)
//   F5 LN2           Xn2 = LN(H1)
//   F6 FC1 + GeLU    U_i = Xn2 A_i + b1_i, G_i = GeLU(U_i)  (grouped GEMM)
//   F7 FC2           Y = H1 + b2 + sum_i G_i B_i            (partition sum in the K-loop)
//   B1 FC2 bwd       dU_i = (dY B_i^T) * GeLU'(U_i); dB_i = G_i^T dY; db2 = sum_n dY
//   B2 FC1 bwd       dA_i = Xn2^T dU_i; db1_i = sum_n dU_i; dXn2 = sum_i dU_i A_i^T
//   B3 LN2 bwd       dH1 = dY + LN2'(dXn2); dgamma2, dbeta2
//   B4 out-proj bwd  dO_i = dH1 W_o,i^T; dW_o,i = O_i^T dH1; db_o = sum_n dH1
//   B5 attention bwd dQKV_i
//   B6 QKV bwd       dW_qkv,i = Xn1^T dQKV_i; db_qkv,i; dXn1 = sum_i dQKV_i W_qkv,i^T
//   B7 LN1 bwd       dX = dH1 + LN1'(dXn1); dgamma1, dbeta1
// The four sums over partitions are the all-reduce points of Megatron-LM's
// intra-layer parallelism (Megatron-LM show notes: 2 all-reduces per module,
// 4 per layer across forward and backward).
#include <string.h>

#include <cmath>
#include <mutex>
#include <vector>

#include "../../include/tplayer.h"
#include "gemm.cuh"
#include "kernels.cuh"

namespace tp {
namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Carver {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const tp_layer_dims* d) {
  if (!d) return TP_ERR_INVALID_ARG;
  if (d->t <= 0 || d->batch <= 0 || d->seq <= 0 || d->hidden <= 0 || d->heads <= 0 ||
      d->ffn <= 0 || !(d->ln_eps > 0.f))
    return TP_ERR_INVALID_ARG;
  if (!(d->dropout_attn >= 0.f && d->dropout_attn < 1.f) ||
      !(d->dropout_hidden >= 0.f && d->dropout_hidden < 1.f) ||
      (d->recompute != 0 && d->recompute != 1))
    return TP_ERR_INVALID_ARG;
  if (d->t > TP_MAX_PARTITIONS) return TP_ERR_UNSUPPORTED;
  if (d->heads % d->t || d->ffn % d->t || d->hidden % d->heads) return TP_ERR_UNSUPPORTED;
  const int hd = d->hidden / d->heads;
  if (hd != 64 && hd != 96 && hd != 128) return TP_ERR_UNSUPPORTED;
  if (d->hidden % 64 || d->hidden > 4096) return TP_ERR_UNSUPPORTED;
  if ((d->ffn / d->t) % 64) return TP_ERR_UNSUPPORTED;
  const long long n = (long long)d->batch * d->seq;
  if (n > (1LL << 30) / d->hidden) return TP_ERR_UNSUPPORTED;
  // attention-probability dropout numbers its rows (batch * heads + head) * seq + query in 32 bits
  if (d->dropout_attn > 0.f && (long long)d->batch * d->heads * d->seq > 0xFFFFFFFFLL)
    return TP_ERR_UNSUPPORTED;
  return TP_OK;
}

// A dropout site of the layer: drop when the 32-bit draw is below
// floor(p 2^32), scale kept values by 1 / (1 - p); rates below 2^-32 are off.
DropSite make_drop(float p, unsigned long long seed, uint32_t stream) {
  DropSite d{};
  const double t = std::floor(static_cast<double>(p) * 4294967296.0);
  d.thresh = t >= 4294967295.0 ? 0xFFFFFFFFu : static_cast<uint32_t>(t);
  d.scale = d.thresh ? static_cast<float>(1.0 / (1.0 - static_cast<double>(p))) : 1.f;
  d.key = make_uint2(static_cast<uint32_t>(seed & 0xFFFFFFFFull), static_cast<uint32_t>(seed >> 32));
  d.stream = stream;
  return d;
}

// Per-row statistics the forward keeps in either mode: LayerNorm mean / rstd
// of both LayerNorms and the attention log-sum-exp.
struct Stats {
  size_t mu1, rs1, lse, mu2, rs2, total;
};

// `parts`: how many of the d.t partitions the buffers hold -- all of them
// (d.t) for the whole layer on one device, 1 for a rank-local pass.
Stats stats_layout(const tp_layer_dims& d, Carver& c, int parts) {
  const size_t n = (size_t)d.batch * d.seq;
  Stats s;
  s.mu1 = c.take(n * 4);
  s.rs1 = c.take(n * 4);
  s.lse = c.take((size_t)d.batch * (d.heads / d.t) * parts * d.seq * 4);
  s.mu2 = c.take(n * 4);
  s.rs2 = c.take(n * 4);
  s.total = c.off;
  return s;
}

// The activations the backward reads: saved by the forward (recompute = 0),
// or rebuilt at the start of the backward (recompute = 1).
struct Acts {
  size_t xn1, qkv, o, h1, xn2, dgelu, g, lse_scratch, total;
};

Acts acts_layout(const tp_layer_dims& d, Carver& c, int parts) {
  const size_t n = (size_t)d.batch * d.seq, h = d.hidden;
  const size_t hp = h / d.t * parts, fp = (size_t)d.ffn / d.t * parts;   // widths held
  Acts a;
  a.xn1 = c.take(n * h * 2);
  a.qkv = c.take(n * 3 * hp * 2);
  a.o = c.take(n * hp * 2);
  a.h1 = c.take(n * h * 2);
  a.xn2 = c.take(n * h * 2);
  a.dgelu = c.take(n * fp * 2);   // GeLU'(U) of the FC1 pre-activation U
  a.g = c.take(n * fp * 2);
  // recompute: the rebuilt attention forward writes its log-sum-exp here
  // (identical to the saved one, which the backward reads)
  a.lse_scratch = d.recompute ? c.take((size_t)d.batch * d.heads * d.seq * 4) : 0;
  a.total = c.off;
  return a;
}

// The `saved` buffer: statistics, then (recompute = 0) the activations.
struct Saved {
  Stats st;
  Acts act;
  size_t total;
};

Saved saved_layout(const tp_layer_dims& d, int parts) {
  Carver c;
  Saved s;
  s.st = stats_layout(d, c, parts);
  if (!d.recompute) s.act = acts_layout(d, c, parts);
  s.total = c.off;
  return s;
}

// Forward scratch: the activations (recompute = 1 only).
struct FwdWork {
  size_t acts, total;
  Acts act;
};

FwdWork fwd_work_layout(const tp_layer_dims& d) {
  Carver c;
  FwdWork f{};
  if (d.recompute) {
    f.acts = c.off;
    Carver a;
    f.act = acts_layout(d, a, d.t);
    c.take(f.act.total);
  }
  f.total = c.off;
  return f;
}

size_t forward_ws_bytes(const tp_layer_dims& d) { return fwd_work_layout(d).total; }

struct Work {
  size_t du, dxn2, dh1, d_o, dqkv, delta, dq_acc, dxn1, ln_part2, ln_part1, col_fc1, col_qkv;
  size_t ln_rows;   // LayerNorm-backward row sums from the dgrad GEMMs' epilogue
  size_t dz2, da1, drop_part2, drop_part1;   // hidden-output dropout (rate > 0)
  size_t acts;                               // rebuilt activations (recompute)
  Acts act;
  size_t total;
};

Work work_layout(const tp_layer_dims& d, int parts) {
  const size_t n = (size_t)d.batch * d.seq, h = d.hidden;
  const size_t hp = h / d.t * parts, fp = (size_t)d.ffn / d.t * parts;   // widths held
  Carver c;
  Work w{};
  w.du = c.take(n * fp * 2);
  w.dxn2 = c.take(n * h * 2);
  w.dh1 = c.take(n * h * 2);
  w.d_o = c.take(n * hp * 2);
  w.dqkv = c.take(n * 3 * hp * 2);
  w.delta = c.take((size_t)d.batch * (d.heads / d.t) * parts * d.seq * 4);
  w.dq_acc = c.take(n * hp * 4);
  w.dxn1 = c.take(n * h * 2);
  // per-row partial sums (float2) of each column tile of the dXn GEMMs,
  // at most ceil(h / 128) tiles; LN2's, then (reused) LN1's
  w.ln_rows = c.take(((h + 127) / 128) * n * 8);
  // column partials, all summed by one launch at the end of the backward:
  // LayerNorm 2 (4 planes) and 1 (2 planes), one row per LayerNorm block
  w.ln_part2 = c.take((size_t)4 * layernorm_bwd_blocks((int)n) * h * 4);
  w.ln_part1 = c.take((size_t)2 * layernorm_bwd_blocks((int)n) * h * 4);
  // bias-gradient partials, [t][blocks][width / t]: db1 per 32-token block,
  // db_qkv per 32-row block of each sequence
  w.col_fc1 = c.take(((n + 31) / 32) * fp * 4);
  w.col_qkv = c.take((size_t)d.batch * ((d.seq + 31) / 32) * 3 * hp * 4);
  if (d.dropout_hidden > 0.f) {
    // gradients of the dropped outputs (the inputs of b2 / B and of b_o / W_o)
    w.dz2 = c.take(n * h * 2);
    w.da1 = c.take(n * h * 2);
    w.drop_part2 = c.take((size_t)dropout_bwd_blocks((int)n) * h * 4);
    w.drop_part1 = c.take((size_t)dropout_bwd_blocks((int)n) * h * 4);
  }
  if (d.recompute) {
    w.acts = c.off;
    Carver a;
    w.act = acts_layout(d, a, parts);
    c.take(w.act.total);
  }
  w.total = c.off;
  return w;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

#define TP_TRY(expr)                               \
  do {                                             \
    int _e = (expr);                               \
    if (_e != 0) return TP_ERR_CUDA;               \
  } while (0)

// ---------------------------------------------------------------- profiling

struct ProfRecord {
  int kind;
  int kernels;
  cudaEvent_t start, stop;
};

struct Profiler {
  std::mutex mu;
  bool on = false;
  bool overflow = false;
  std::vector<cudaEvent_t> events;   // 2 per record
  std::vector<ProfRecord> records;
};

Profiler& profiler() {
  static Profiler p;
  return p;
}

bool profiling_on() {
  Profiler& P = profiler();
  std::lock_guard<std::mutex> lock(P.mu);
  return P.on;
}

// Run `launch` (which enqueues `kernels` kernels of class `kind` on `s`),
// bracketed by CUDA events when profiling is enabled.
template <typename F>
int timed(int kind, int kernels, cudaStream_t s, F&& launch) {
  Profiler& P = profiler();
  std::unique_lock<std::mutex> lock(P.mu);
  if (!P.on) {
    lock.unlock();
    return launch();
  }
  const size_t i = P.records.size();
  if (2 * (i + 1) > P.events.size()) {
    P.overflow = true;
    lock.unlock();
    return launch();
  }
  ProfRecord r{kind, kernels, P.events[2 * i], P.events[2 * i + 1]};
  cudaEventRecord(r.start, s);
  const int rc = launch();
  cudaEventRecord(r.stop, s);
  P.records.push_back(r);
  return rc;
}

#define TP_RUN(kind, nk, expr) TP_TRY(timed((kind), (nk), s, [&]() -> int { return (expr); }))
// The same, enqueued on stream `st`.
#define TP_RUN_ON(st, kind, nk, expr) \
  TP_TRY(timed((kind), (nk), (st), [&]() -> int { return (expr); }))

// ---------------------------------------------------------------- side stream
//
// The backward's weight-gradient GEMMs (dB_i, dA_i, dW_o,i, dW_qkv,i) read
// only tensors the main stream has already produced and write only their own
// gradients, so they run on a second stream: forked after their inputs exist,
// joined before the final bias / gamma / beta sums.  They fill the partly idle
// last wave of the input-gradient GEMMs and run beside the LayerNorm and
// attention backward instead of after them.  One side stream and its events
// per device, created by the first backward on that device (before any stream
// capture; capture follows the fork and join); a mutex keeps one backward's
// fork / join sequence from interleaving with another host thread's.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork[4] = {};
  cudaEvent_t join = nullptr;
  std::mutex mu;
};

constexpr int kMaxSideDevices = 64;
SideStream g_side[kMaxSideDevices];
std::mutex g_side_init;

int side_stream(SideStream** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) return TP_ERR_CUDA;
  SideStream& ss = g_side[dev];
  std::lock_guard<std::mutex> lock(g_side_init);
  if (!ss.stream) {
    cudaStream_t st = nullptr;
    int lo = 0, hi = 0;   // numerically greatest = lowest priority
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess ||
        cudaStreamCreateWithPriority(&st, cudaStreamNonBlocking, lo) != cudaSuccess)
      return TP_ERR_CUDA;
    for (auto& e : ss.fork)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return TP_ERR_CUDA;
    if (cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) return TP_ERR_CUDA;
    ss.stream = st;
  }
  *out = &ss;
  return TP_OK;
}

// The side stream waits for everything enqueued on `s` so far.
int fork_to(SideStream& ss, int i, cudaStream_t s) {
  if (cudaEventRecord(ss.fork[i], s) != cudaSuccess) return TP_ERR_CUDA;
  return cudaStreamWaitEvent(ss.stream, ss.fork[i], 0) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

// `s` waits for everything enqueued on the side stream so far.
int join_from(SideStream& ss, cudaStream_t s) {
  if (cudaEventRecord(ss.join, ss.stream) != cudaSuccess) return TP_ERR_CUDA;
  return cudaStreamWaitEvent(s, ss.join, 0) == cudaSuccess ? TP_OK : TP_ERR_CUDA;
}

#define TP_FORK(i) \
  do {               \
    if (!serial) TP_TRY(fork_to(*side, (i), s)); \
  } while (0)

}  // namespace
}  // namespace tp

namespace tp {
namespace {

constexpr int kXentTileN = 256;   // column tile of the logits GEMM (force_bn)

struct XentFusedLayout {
  size_t stats, ztgt, lse, z, small, total;
};

XentFusedLayout xent_fused_layout(int t, int tokens, int vocab) {
  const size_t vp = vocab / t;
  const size_t ntiles = (vp + kXentTileN - 1) / kXentTileN;
  Carver c;
  XentFusedLayout L;
  L.stats = c.take((size_t)t * ntiles * tokens * 8);
  L.ztgt = c.take((size_t)tokens * 4);
  L.lse = c.take(((size_t)tokens + (tokens + 7) / 8) * 4);   // + block sums of the combine
  L.small = c.off;
  L.z = c.take((size_t)t * tokens * vp * 2);
  L.total = c.off;
  return L;
}

// Scratch of one vocab partition's loss on its own device: its tile
// statistics and target logit, its slice's log-sum-exp, the combined lse (+
// block sums of the mean), and with a gradient its bf16 logits.
struct XentRankLayout {
  size_t stats, ztgt, lse_loc, lse, small, z, total;
};

XentRankLayout xent_rank_layout(int t, int tokens, int vocab) {
  const size_t vp = vocab / t;
  const size_t ntiles = (vp + kXentTileN - 1) / kXentTileN;
  Carver c;
  XentRankLayout L;
  L.stats = c.take(ntiles * tokens * 8);
  L.ztgt = c.take((size_t)tokens * 4);
  L.lse_loc = c.take((size_t)tokens * 4);
  L.lse = c.take(((size_t)tokens + (tokens + 7) / 8) * 4);
  L.small = c.off;
  L.z = c.take((size_t)tokens * vp * 2);
  L.total = c.off;
  return L;
}

}  // namespace
}  // namespace tp

namespace tp {
namespace {

// Device pointers of the statistics and activations one layer pass uses.
struct ActPtrs {
  __nv_bfloat16 *xn1, *qkv, *o, *h1, *xn2, *dgelu, *g;
  float *mu1, *rs1, *lse, *mu2, *rs2;
};

ActPtrs act_ptrs(void* stats_base, const Stats& st, void* act_base, const Acts& a) {
  ActPtrs P;
  P.mu1 = at<float>(stats_base, st.mu1);
  P.rs1 = at<float>(stats_base, st.rs1);
  P.lse = at<float>(stats_base, st.lse);
  P.mu2 = at<float>(stats_base, st.mu2);
  P.rs2 = at<float>(stats_base, st.rs2);
  P.xn1 = at<__nv_bfloat16>(act_base, a.xn1);
  P.qkv = at<__nv_bfloat16>(act_base, a.qkv);
  P.o = at<__nv_bfloat16>(act_base, a.o);
  P.h1 = at<__nv_bfloat16>(act_base, a.h1);
  P.xn2 = at<__nv_bfloat16>(act_base, a.xn2);
  P.dgelu = at<__nv_bfloat16>(act_base, a.dgelu);
  P.g = at<__nv_bfloat16>(act_base, a.g);
  return P;
}

int check_weights(const tp_layer_dims& d, const tp_layer_weights* w) {
  if (!w->ln1_g || !w->ln1_b || !w->ln2_g || !w->ln2_b || !w->b_o || !w->b_fc2)
    return TP_ERR_INVALID_ARG;
  for (int i = 0; i < d.t; ++i)
    if (!w->w_qkv[i] || !w->b_qkv[i] || !w->w_o[i] || !w->w_fc1[i] || !w->b_fc1[i] ||
        !w->w_fc2[i] || !aligned16(w->w_qkv[i]) || !aligned16(w->w_o[i]) ||
        !aligned16(w->w_fc1[i]) || !aligned16(w->w_fc2[i]) || !aligned16(w->b_qkv[i]) ||
        !aligned16(w->b_fc1[i]))
      return TP_ERR_INVALID_ARG;
  return TP_OK;
}

// A rank-local pass: partition `rank` of the d.t partitions, on this device,
// with every sum over partitions left to the caller (a collective across
// devices).  The pass is cut at the sum points into segments; `partial`
// ([N, h] bf16) receives this partition's term at the end of a segment and
// holds the sum over all partitions when the next segment starts.  The
// weights and gradients of the partition are at index 0 of their arrays, and
// the per-partition buffers hold that one partition.
struct RankCtx {
  int rank;
  int segment;
  __nv_bfloat16* partial;
};

// F1..F6 (and F7 when y is given) into the activation pointers P.  With
// stats_given the LayerNorms apply the statistics in P instead of computing
// them; the attention writes its log-sum-exp to lse_out.  With rk, one
// segment of the rank-local forward: 0 = F1..F3 and O_i W_o,i; 1 = H1 from
// the summed partial, F5, F6 and G_i B_i; 2 = Y from the summed partial.
int run_forward(const tp_layer_dims& d, const tp_layer_weights* w, const void* x,
                const int32_t* valid_len, void* y, const ActPtrs& P, bool stats_given,
                float* lse_out, cudaStream_t s, const RankCtx* rk = nullptr) {
  const int t = d.t;
  const int np = rk ? 1 : t;   // partitions this call computes
  const int n = d.batch * d.seq, h = d.hidden, f = d.ffn;
  const int hd = h / d.heads;
  const int qkv_w = 3 * h / t, o_w = h / t, f_w = f / t;
  const int seg = rk ? rk->segment : -1;

  if (rk && seg == 1) {
    // H1 = X + drop(sum_i O_i W_o,i + b_o), the sum formed by the caller
    TP_RUN(TP_KERNEL_ELEMENTWISE, 1,
           launch_bias_drop_residual(rk->partial, w->b_o, x, P.h1, n, h,
                                     make_drop(d.dropout_hidden, d.seed, DROP_ATTN_OUT), s));
  }
  if (rk && seg == 2) {
    // Y = H1 + drop(sum_i G_i B_i + b2)
    TP_RUN(TP_KERNEL_ELEMENTWISE, 1,
           launch_bias_drop_residual(rk->partial, w->b_fc2, P.h1, y, n, h,
                                     make_drop(d.dropout_hidden, d.seed, DROP_MLP_OUT), s));
    return TP_OK;
  }
  if (!rk || seg == 0) {
  // F1
  TP_RUN(TP_KERNEL_LN_FWD, 1, launch_layernorm_fwd(x, w->ln1_g, w->ln1_b, d.ln_eps, n, h, P.xn1,
                                                   P.mu1, P.rs1, s, stats_given));
  // F2
  {
    GemmDesc gd;
    gd.groups = np;
    gd.M = n; gd.N = qkv_w; gd.K = h;
    gd.a_mn = false; gd.lda = h;
    gd.b_mn = true; gd.ldb = qkv_w;
    gd.epi = EPI_BIAS_BF16; gd.ldc = qkv_w;
    for (int i = 0; i < np; ++i) {
      gd.a[i] = P.xn1;
      gd.b[i] = w->w_qkv[i];
      gd.bias[i] = w->b_qkv[i];
      gd.out[i] = P.qkv + (size_t)i * n * qkv_w;
    }
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  }
  // F3
  {
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.batch = d.batch; a.seq = d.seq; a.heads = d.heads / t * np; a.head_dim = hd; a.t = np;
    a.causal = d.causal; a.valid_len = valid_len;
    a.head0 = rk ? rk->rank * (d.heads / t) : 0;
    a.heads_total = d.heads;
    for (int i = 0; i < np; ++i) {
      a.qkv[i] = P.qkv + (size_t)i * n * qkv_w;
      a.o[i] = P.o + (size_t)i * n * o_w;
    }
    a.lse = lse_out;
    a.drop = make_drop(d.dropout_attn, d.seed, DROP_ATTN_PROBS);
    TP_RUN(TP_KERNEL_ATTN_FWD, 1, launch_attention_fwd_tc(a, s));
  }
  // F4: H1 = X + drop(sum_i O_i W_o,i + b_o); rank-local: the term O_i W_o,i
  {
    GemmDesc gd;
    gd.groups = np; gd.sum_groups = 1;
    gd.M = n; gd.N = h; gd.K = o_w;
    gd.a_mn = false; gd.lda = o_w;
    gd.b_mn = true; gd.ldb = h;
    gd.ldc = h; gd.ldaux = h;
    for (int i = 0; i < np; ++i) {
      gd.a[i] = P.o + (size_t)i * n * o_w;
      gd.b[i] = w->w_o[i];
    }
    if (rk) {
      gd.epi = EPI_BF16;
      gd.out[0] = rk->partial;
    } else {
      gd.epi = EPI_BIAS_RES;
      gd.out[0] = P.h1; gd.bias[0] = w->b_o; gd.aux[0] = x;
      gd.drop = make_drop(d.dropout_hidden, d.seed, DROP_ATTN_OUT);
    }
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  }
  if (rk) return TP_OK;
  }
  // F5
  TP_RUN(TP_KERNEL_LN_FWD, 1, launch_layernorm_fwd(P.h1, w->ln2_g, w->ln2_b, d.ln_eps, n, h, P.xn2,
                                                   P.mu2, P.rs2, s, stats_given));
  // F6
  {
    GemmDesc gd;
    gd.groups = np;
    gd.M = n; gd.N = f_w; gd.K = h;
    gd.a_mn = false; gd.lda = h;
    gd.b_mn = true; gd.ldb = f_w;
    gd.epi = EPI_BIAS_GELU; gd.ldc = f_w;
    for (int i = 0; i < np; ++i) {
      gd.a[i] = P.xn2;
      gd.b[i] = w->w_fc1[i];
      gd.bias[i] = w->b_fc1[i];
      gd.out[i] = P.dgelu + (size_t)i * n * f_w;
      gd.out2[i] = P.g + (size_t)i * n * f_w;
    }
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  }
  if (!y && !rk) return TP_OK;
  // F7: Y = H1 + drop(sum_i G_i B_i + b2); rank-local: the term G_i B_i
  {
    GemmDesc gd;
    gd.groups = np; gd.sum_groups = 1;
    gd.M = n; gd.N = h; gd.K = f_w;
    gd.a_mn = false; gd.lda = f_w;
    gd.b_mn = true; gd.ldb = h;
    gd.ldc = h; gd.ldaux = h;
    for (int i = 0; i < np; ++i) {
      gd.a[i] = P.g + (size_t)i * n * f_w;
      gd.b[i] = w->w_fc2[i];
    }
    if (rk) {
      gd.epi = EPI_BF16;
      gd.out[0] = rk->partial;
    } else {
      gd.epi = EPI_BIAS_RES;
      gd.out[0] = y; gd.bias[0] = w->b_fc2; gd.aux[0] = P.h1;
      gd.drop = make_drop(d.dropout_hidden, d.seed, DROP_MLP_OUT);
    }
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  }
  return TP_OK;
}

// B1..B7 and the bias / gamma / beta sums, from the activations P.  With
// rk, one segment of the rank-local backward: 0 = dropout of dY, B1 and B2
// with the term dU_i A_i^T of dXn2 into the partial; 1 = B3 from the summed
// dXn2, B4, B5 and B6 with the term dQKV_i W_qkv,i^T of dXn1; 2 = B7 from the
// summed dXn1 and the sums.  The weight-gradient GEMMs of segments 0 and 1
// may still run on the side stream when the call returns (beside the
// caller's collective); segment 2 joins them.
int run_backward(const tp_layer_dims& d, const tp_layer_weights* w, const void* x,
                 const int32_t* valid_len, const ActPtrs& P, const void* dy, void* dx,
                 const tp_layer_grads* gr, void* ws, const Work& W, cudaStream_t s,
                 const RankCtx* rk = nullptr) {
  SideStream* side = nullptr;
  TP_TRY(side_stream(&side));
  std::lock_guard<std::mutex> side_lock(side->mu);
  // With per-launch timing on, everything runs on `s`: a recorded duration is
  // then one kernel's alone, not a share of two overlapping ones.
  const bool serial = profiling_on();
  const cudaStream_t ss = serial ? s : side->stream;
  const int t = d.t;
  const int np = rk ? 1 : t;   // partitions this call computes
  const int seg = rk ? rk->segment : -1;
  const int n = d.batch * d.seq, h = d.hidden, f = d.ffn;
  const int hd = h / d.heads;
  const int qkv_w = 3 * h / t, o_w = h / t, f_w = f / t;
  const bool hdrop = d.dropout_hidden > 0.f && make_drop(d.dropout_hidden, d.seed, 0).thresh;
  auto* du = at<__nv_bfloat16>(ws, W.du);
  auto* dxn2 = rk ? rk->partial : at<__nv_bfloat16>(ws, W.dxn2);
  auto* dh1 = at<__nv_bfloat16>(ws, W.dh1);
  auto* d_o = at<__nv_bfloat16>(ws, W.d_o);
  auto* dqkv = at<__nv_bfloat16>(ws, W.dqkv);
  auto* dxn1 = rk ? rk->partial : at<__nv_bfloat16>(ws, W.dxn1);
  float2* ln_rows = at<float2>(ws, W.ln_rows);
  const int ln_tile = gemm_pick_bn(n, h, np, true, true);   // the dXn GEMMs' column tile
  const int ln_row_parts = (h + ln_tile - 1) / ln_tile;
  float* ln_part2 = at<float>(ws, W.ln_part2);
  float* ln_part1 = at<float>(ws, W.ln_part1);
  float* col_fc1 = at<float>(ws, W.col_fc1);
  float* col_qkv = at<float>(ws, W.col_qkv);

  // Gradient of the FC2 output before its dropout: dZ2 = dY * keep / (1 - p)
  // (b2's gradient is its column sum); dY itself without dropout.
  const void* dz2 = hdrop ? at<__nv_bfloat16>(ws, W.dz2) : dy;
  const void* da1 = hdrop ? at<__nv_bfloat16>(ws, W.da1) : dh1;
  if (!rk || seg == 0) {
  if (hdrop) {
    TP_RUN(TP_KERNEL_REDUCE, 1,
           launch_dropout_bwd(dy, const_cast<void*>(dz2), n, h,
                              make_drop(d.dropout_hidden, d.seed, DROP_MLP_OUT),
                              at<float>(ws, W.drop_part2), s));
  }
  // B1: dU_i (FC2 dgrad with the GeLU' epilogue), dB_i  (db2 comes with B3)
  {
    GemmDesc gd;
    gd.groups = np;
    gd.M = n; gd.N = f_w; gd.K = h;
    gd.a_mn = false; gd.lda = h;
    gd.b_mn = false; gd.ldb = h;
    gd.epi = EPI_DGELU; gd.ldc = f_w; gd.ldaux = f_w;
    gd.colsum = col_fc1;    // db1_i partials come out of this epilogue
    for (int i = 0; i < np; ++i) {
      gd.a[i] = dz2;
      gd.b[i] = w->w_fc2[i];
      gd.aux[i] = P.dgelu + (size_t)i * n * f_w;
      gd.out[i] = du + (size_t)i * n * f_w;
    }
    GemmDesc wg;
    wg.groups = np;
    wg.M = f_w; wg.N = h; wg.K = n;
    wg.a_mn = true; wg.lda = f_w;
    wg.b_mn = true; wg.ldb = h;
    wg.epi = EPI_BF16; wg.ldc = h;
    for (int i = 0; i < np; ++i) {
      wg.a[i] = P.g + (size_t)i * n * f_w;
      wg.b[i] = dz2;
      wg.out[i] = gr->w_fc2[i];
    }
    // dB_i = G_i^T dZ2 on the side stream, enqueued after the dgrad on the
    // critical path so that the dgrad's CTAs are placed first
    TP_FORK(0);
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
    TP_RUN_ON(ss, TP_KERNEL_GEMM, 1, launch_gemm(wg, ss));
  }
  // B2: dA_i, db1_i, dXn2 = sum_i dU_i A_i^T
  {
    GemmDesc wg;
    wg.groups = np;
    wg.M = h; wg.N = f_w; wg.K = n;
    wg.a_mn = true; wg.lda = h;
    wg.b_mn = true; wg.ldb = f_w;
    wg.epi = EPI_BF16; wg.ldc = f_w;
    for (int i = 0; i < np; ++i) {
      wg.a[i] = P.xn2;
      wg.b[i] = du + (size_t)i * n * f_w;
      wg.out[i] = gr->w_fc1[i];
    }
    GemmDesc gd;
    gd.groups = np; gd.sum_groups = 1;
    gd.M = n; gd.N = h; gd.K = f_w;
    gd.a_mn = false; gd.lda = f_w;
    gd.b_mn = false; gd.ldb = f_w;
    gd.epi = EPI_BF16; gd.ldc = h;
    for (int i = 0; i < np; ++i) {
      gd.a[i] = du + (size_t)i * n * f_w;
      gd.b[i] = w->w_fc1[i];
    }
    gd.out[0] = dxn2;
    if (!rk) {   // dXn2 complete here: LN2's backward row sums from the epilogue
      gd.epi = EPI_LN_ROWSTATS;
      gd.aux[0] = P.h1; gd.ldaux = h; gd.bias[0] = w->ln2_g;
      gd.ln_mean = P.mu2; gd.ln_rstd = P.rs2; gd.ln_rows = ln_rows;
    }
    TP_FORK(1);   // dA_i = Xn2^T dU_i on the side stream
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
    TP_RUN_ON(ss, TP_KERNEL_GEMM, 1, launch_gemm(wg, ss));
  }
  if (rk) return TP_OK;
  }
  if (!rk || seg == 1) {
  // B3: dH1 = dY + LN2'(dXn2); dgamma2, dbeta2, and (without dropout) the
  // column sums of dY (= db2) and of dH1 (= db_o) from the same pass
  TP_RUN(TP_KERNEL_LN_BWD, 1,
         launch_layernorm_bwd(dxn2, P.h1, w->ln2_g, P.mu2, P.rs2, dy, n, h, dh1, ln_part2, !hdrop,
                              s, rk ? nullptr : ln_rows, ln_row_parts));
  // Gradient of the out-projection output before its dropout
  if (hdrop) {
    TP_RUN(TP_KERNEL_REDUCE, 1,
           launch_dropout_bwd(dh1, const_cast<void*>(da1), n, h,
                              make_drop(d.dropout_hidden, d.seed, DROP_ATTN_OUT),
                              at<float>(ws, W.drop_part1), s));
  }
  // B4: dO_i, dW_o,i
  {
    GemmDesc gd;
    gd.groups = np;
    gd.M = n; gd.N = o_w; gd.K = h;
    gd.a_mn = false; gd.lda = h;
    gd.b_mn = false; gd.ldb = h;
    gd.epi = EPI_BF16; gd.ldc = o_w;
    for (int i = 0; i < np; ++i) {
      gd.a[i] = da1;
      gd.b[i] = w->w_o[i];
      gd.out[i] = d_o + (size_t)i * n * o_w;
    }
    GemmDesc wg;
    wg.groups = np;
    wg.M = o_w; wg.N = h; wg.K = n;
    wg.a_mn = true; wg.lda = o_w;
    wg.b_mn = true; wg.ldb = h;
    wg.epi = EPI_BF16; wg.ldc = h;
    for (int i = 0; i < np; ++i) {
      wg.a[i] = P.o + (size_t)i * n * o_w;
      wg.b[i] = da1;
      wg.out[i] = gr->w_o[i];
    }
    TP_FORK(2);   // dW_o,i = O_i^T dA1 on the side stream, beside the attention backward
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
    TP_RUN_ON(ss, TP_KERNEL_GEMM, 1, launch_gemm(wg, ss));
  }
  // B5: attention backward
  {
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.batch = d.batch; a.seq = d.seq; a.heads = d.heads / t * np; a.head_dim = hd; a.t = np;
    a.causal = d.causal; a.valid_len = valid_len;
    a.head0 = rk ? rk->rank * (d.heads / t) : 0;
    a.heads_total = d.heads;
    for (int i = 0; i < np; ++i) {
      a.qkv[i] = P.qkv + (size_t)i * n * qkv_w;
      a.o[i] = P.o + (size_t)i * n * o_w;
      a.d_o[i] = d_o + (size_t)i * n * o_w;
      a.dqkv[i] = dqkv + (size_t)i * n * qkv_w;
    }
    a.lse = P.lse;
    a.delta = at<float>(ws, W.delta);
    a.dq_acc = at<float>(ws, W.dq_acc);
    a.colsum = col_qkv;     // db_qkv,i partials come out of the attention backward
    a.drop = make_drop(d.dropout_attn, d.seed, DROP_ATTN_PROBS);
    TP_RUN(TP_KERNEL_ATTN_BWD, attention_bwd_launches(hd), launch_attention_bwd_tc(a, s));
  }
  // B6: dW_qkv,i, db_qkv,i, dXn1 = sum_i dQKV_i W_qkv,i^T
  {
    GemmDesc wg;
    wg.groups = np;
    wg.M = h; wg.N = qkv_w; wg.K = n;
    wg.a_mn = true; wg.lda = h;
    wg.b_mn = true; wg.ldb = qkv_w;
    wg.epi = EPI_BF16; wg.ldc = qkv_w;
    for (int i = 0; i < np; ++i) {
      wg.a[i] = P.xn1;
      wg.b[i] = dqkv + (size_t)i * n * qkv_w;
      wg.out[i] = gr->w_qkv[i];
    }
    GemmDesc gd;
    gd.groups = np; gd.sum_groups = 1;
    gd.M = n; gd.N = h; gd.K = qkv_w;
    gd.a_mn = false; gd.lda = qkv_w;
    gd.b_mn = false; gd.ldb = qkv_w;
    gd.epi = EPI_BF16; gd.ldc = h;
    for (int i = 0; i < np; ++i) {
      gd.a[i] = dqkv + (size_t)i * n * qkv_w;
      gd.b[i] = w->w_qkv[i];
    }
    gd.out[0] = dxn1;
    if (!rk) {   // LN1's backward row sums from the epilogue
      gd.epi = EPI_LN_ROWSTATS;
      gd.aux[0] = x; gd.ldaux = h; gd.bias[0] = w->ln1_g;
      gd.ln_mean = P.mu1; gd.ln_rstd = P.rs1; gd.ln_rows = ln_rows;
    }
    TP_FORK(3);   // dW_qkv,i = Xn1^T dQKV_i on the side stream
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
    TP_RUN_ON(ss, TP_KERNEL_GEMM, 1, launch_gemm(wg, ss));
  }
  if (rk) return TP_OK;
  }
  // B7: dX = dH1 + LN1'(dXn1)
  TP_RUN(TP_KERNEL_LN_BWD, 1,
         launch_layernorm_bwd(dxn1, x, w->ln1_g, P.mu1, P.rs1, dh1, n, h, dx, ln_part1, false, s,
                              rk ? nullptr : ln_rows, ln_row_parts));
  // the weight gradients are done before the backward returns
  if (!serial) TP_TRY(join_from(*side, s));
  // Every bias / gamma / beta gradient from its partial rows, in one launch
  {
    SumRowsJob jobs[kMaxSumJobs] = {};
    int nj = 0;
    const int lnb = layernorm_bwd_blocks(n);
    if (!hdrop) {
      jobs[nj++] = {ln_part2, 4, lnb, h, {gr->ln2_g, gr->ln2_b, gr->b_fc2, gr->b_o}};
    } else {
      jobs[nj++] = {ln_part2, 2, lnb, h, {gr->ln2_g, gr->ln2_b}};
      jobs[nj++] = {at<float>(ws, W.drop_part2), 1, dropout_bwd_blocks(n), h, {gr->b_fc2}};
      jobs[nj++] = {at<float>(ws, W.drop_part1), 1, dropout_bwd_blocks(n), h, {gr->b_o}};
    }
    jobs[nj++] = {ln_part1, 2, lnb, h, {gr->ln1_g, gr->ln1_b}};
    SumRowsJob& jf = jobs[nj++];
    jf = {col_fc1, np, (n + 31) / 32, f_w, {}};
    SumRowsJob& jq = jobs[nj++];
    jq = {col_qkv, np, d.batch * ((d.seq + 31) / 32), qkv_w, {}};
    for (int i = 0; i < np; ++i) {
      jf.out[i] = gr->b_fc1[i];
      jq.out[i] = gr->b_qkv[i];
    }
    TP_RUN(TP_KERNEL_REDUCE, 1, launch_sum_rows_multi(jobs, nj, s));
  }
  return TP_OK;
}

}  // namespace
}  // namespace tp

using namespace tp;

extern "C" {

size_t tp_layer_saved_bytes(const tp_layer_dims* dims) {
  if (check_dims(dims) != TP_OK) return 0;
  return saved_layout(*dims, dims->t).total;
}

size_t tp_layer_forward_workspace_bytes(const tp_layer_dims* dims) {
  if (check_dims(dims) != TP_OK) return 0;
  return forward_ws_bytes(*dims);
}

size_t tp_layer_workspace_bytes(const tp_layer_dims* dims) {
  if (check_dims(dims) != TP_OK) return 0;
  return work_layout(*dims, dims->t).total;
}

int tp_layer_forward(const tp_layer_dims* dims, const tp_layer_weights* w, const void* x,
                     const int32_t* valid_len, void* y, void* saved, size_t saved_bytes, void* ws,
                     size_t ws_bytes, void* stream) {
  int st = check_dims(dims);
  if (st != TP_OK) return st;
  if (!w || !x || !y || !saved) return TP_ERR_INVALID_ARG;
  const tp_layer_dims& d = *dims;
  const Saved L = saved_layout(d, d.t);
  if (saved_bytes < L.total) return TP_ERR_WORKSPACE;
  const FwdWork F = fwd_work_layout(d);
  if (F.total && (!ws || ws_bytes < F.total)) return TP_ERR_WORKSPACE;
  if ((st = check_weights(d, w)) != TP_OK) return st;
  if (!aligned16(x) || !aligned16(y) || !aligned16(saved) || (F.total && !aligned16(ws)))
    return TP_ERR_INVALID_ARG;
  const ActPtrs P = d.recompute ? act_ptrs(saved, L.st, at<uint8_t>(ws, F.acts), F.act)
                                : act_ptrs(saved, L.st, saved, L.act);
  return run_forward(d, w, x, valid_len, y, P, false, P.lse, static_cast<cudaStream_t>(stream));
}

int tp_layer_backward(const tp_layer_dims* dims, const tp_layer_weights* w, const void* x,
                      const int32_t* valid_len, const void* saved, size_t saved_bytes,
                      const void* dy, void* dx, const tp_layer_grads* gr, void* ws,
                      size_t ws_bytes, void* stream) {
  int st = check_dims(dims);
  if (st != TP_OK) return st;
  if (!w || !x || !saved || !dy || !dx || !gr || !ws) return TP_ERR_INVALID_ARG;
  const tp_layer_dims& d = *dims;
  const int t = d.t;
  const Work W = work_layout(d, d.t);
  const Saved L = saved_layout(d, d.t);
  if (ws_bytes < W.total || saved_bytes < L.total) return TP_ERR_WORKSPACE;
  if (!gr->ln1_g || !gr->ln1_b || !gr->ln2_g || !gr->ln2_b || !gr->b_o || !gr->b_fc2)
    return TP_ERR_INVALID_ARG;
  if ((st = check_weights(d, w)) != TP_OK) return st;
  for (int i = 0; i < t; ++i)
    if (!gr->w_qkv[i] || !gr->b_qkv[i] || !gr->w_o[i] || !gr->w_fc1[i] || !gr->b_fc1[i] ||
        !gr->w_fc2[i] || !aligned16(gr->w_qkv[i]) || !aligned16(gr->w_o[i]) ||
        !aligned16(gr->w_fc1[i]) || !aligned16(gr->w_fc2[i]))
      return TP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dx) || !aligned16(dy) || !aligned16(saved) || !aligned16(ws))
    return TP_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* sv = const_cast<void*>(saved);
  ActPtrs P;
  if (d.recompute) {
    // rebuild the activations from X with the forward's kernels, applying the
    // saved LayerNorm statistics; the rebuilt attention writes its (identical)
    // log-sum-exp to scratch, the backward reads the saved one
    P = act_ptrs(sv, L.st, at<uint8_t>(ws, W.acts), W.act);
    const int rc = run_forward(d, w, x, valid_len, nullptr, P, true,
                               at<float>(at<uint8_t>(ws, W.acts), W.act.lse_scratch), s);
    if (rc != TP_OK) return rc;
  } else {
    P = act_ptrs(sv, L.st, sv, L.act);
  }
  return run_backward(d, w, x, valid_len, P, dy, dx, gr, ws, W, s);
}

// ---------------------------------------------------------------- rank-local layer

namespace {
int check_rank_call(const tp_layer_dims* dims, int rank, int segment) {
  const int st = check_dims(dims);
  if (st != TP_OK) return st;
  if (rank < 0 || rank >= dims->t || segment < 0 || segment > 2) return TP_ERR_INVALID_ARG;
  if (dims->recompute) return TP_ERR_UNSUPPORTED;
  return TP_OK;
}

// The rank's tensors at index 0; the replicated ones whole.
int check_rank_weights(const tp_layer_weights* w) {
  if (!w || !w->ln1_g || !w->ln1_b || !w->ln2_g || !w->ln2_b || !w->b_o || !w->b_fc2)
    return TP_ERR_INVALID_ARG;
  if (!w->w_qkv[0] || !w->b_qkv[0] || !w->w_o[0] || !w->w_fc1[0] || !w->b_fc1[0] || !w->w_fc2[0] ||
      !aligned16(w->w_qkv[0]) || !aligned16(w->w_o[0]) || !aligned16(w->w_fc1[0]) ||
      !aligned16(w->w_fc2[0]) || !aligned16(w->b_qkv[0]) || !aligned16(w->b_fc1[0]) ||
      !aligned16(w->b_o) || !aligned16(w->b_fc2))
    return TP_ERR_INVALID_ARG;
  return TP_OK;
}
}  // namespace

size_t tp_layer_rank_saved_bytes(const tp_layer_dims* dims) {
  if (check_rank_call(dims, 0, 0) != TP_OK) return 0;
  return saved_layout(*dims, 1).total;
}

size_t tp_layer_rank_workspace_bytes(const tp_layer_dims* dims) {
  if (check_rank_call(dims, 0, 0) != TP_OK) return 0;
  return work_layout(*dims, 1).total;
}

int tp_layer_rank_forward(const tp_layer_dims* dims, int rank, int segment, const tp_layer_weights* w,
                          const void* x, const int32_t* valid_len, void* partial, void* y, void* saved,
                          size_t saved_bytes, void* stream) {
  int st = check_rank_call(dims, rank, segment);
  if (st != TP_OK) return st;
  if ((st = check_rank_weights(w)) != TP_OK) return st;
  if (!x || !partial || !saved || (segment == 2 && !y)) return TP_ERR_INVALID_ARG;
  const tp_layer_dims& d = *dims;
  const Saved L = saved_layout(d, 1);
  if (saved_bytes < L.total) return TP_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(partial) || !aligned16(saved) || (y && !aligned16(y)))
    return TP_ERR_INVALID_ARG;
  const ActPtrs P = act_ptrs(saved, L.st, saved, L.act);
  const RankCtx rk{rank, segment, static_cast<__nv_bfloat16*>(partial)};
  return run_forward(d, w, x, valid_len, y, P, false, P.lse, static_cast<cudaStream_t>(stream), &rk);
}

int tp_layer_rank_backward(const tp_layer_dims* dims, int rank, int segment, const tp_layer_weights* w,
                           const void* x, const int32_t* valid_len, const void* saved,
                           size_t saved_bytes, const void* dy, void* partial, void* dx,
                           const tp_layer_grads* gr, void* ws, size_t ws_bytes, void* stream) {
  int st = check_rank_call(dims, rank, segment);
  if (st != TP_OK) return st;
  if ((st = check_rank_weights(w)) != TP_OK) return st;
  if (!x || !saved || !dy || !partial || !gr || !ws || (segment == 2 && !dx)) return TP_ERR_INVALID_ARG;
  const tp_layer_dims& d = *dims;
  const Work W = work_layout(d, 1);
  const Saved L = saved_layout(d, 1);
  if (ws_bytes < W.total || saved_bytes < L.total) return TP_ERR_WORKSPACE;
  if (!gr->ln1_g || !gr->ln1_b || !gr->ln2_g || !gr->ln2_b || !gr->b_o || !gr->b_fc2 ||
      !gr->w_qkv[0] || !gr->b_qkv[0] || !gr->w_o[0] || !gr->w_fc1[0] || !gr->b_fc1[0] ||
      !gr->w_fc2[0] || !aligned16(gr->w_qkv[0]) || !aligned16(gr->w_o[0]) ||
      !aligned16(gr->w_fc1[0]) || !aligned16(gr->w_fc2[0]))
    return TP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(partial) || !aligned16(saved) || !aligned16(ws) ||
      (dx && !aligned16(dx)))
    return TP_ERR_INVALID_ARG;
  void* sv = const_cast<void*>(saved);
  const ActPtrs P = act_ptrs(sv, L.st, sv, L.act);
  const RankCtx rk{rank, segment, static_cast<__nv_bfloat16*>(partial)};
  return run_backward(d, w, x, valid_len, P, dy, dx, gr, ws, W, static_cast<cudaStream_t>(stream), &rk);
}

// ---------------------------------------------------------------- rank-local loss

size_t tp_xent_rank_workspace_bytes(int t, int tokens, int hidden, int vocab) {
  if (t < 1 || t > TP_MAX_PARTITIONS || tokens <= 0 || hidden <= 0 || vocab <= 0) return 0;
  if (vocab % t || (vocab / t) % 8 || hidden % 8) return 0;
  return xent_rank_layout(t, tokens, vocab).total;
}

int vocab_parallel_xent_rank(int t, int rank, int segment, int tokens, int hidden, int vocab,
                             const void* x, const void* emb, const int32_t* target, float* comm,
                             float* loss, float* loss_per_token, void* dx, void* demb, void* ws,
                             size_t ws_bytes, void* stream) {
  if (t < 1 || tokens <= 0 || hidden <= 0 || vocab <= 0) return TP_ERR_INVALID_ARG;
  if (rank < 0 || rank >= t || segment < 0 || segment > 2) return TP_ERR_INVALID_ARG;
  if (t > TP_MAX_PARTITIONS || vocab % t || (vocab / t) % 8 || hidden % 8) return TP_ERR_UNSUPPORTED;
  if (!x || !emb || !target || !comm || !ws || (segment == 2 && !loss)) return TP_ERR_INVALID_ARG;
  if (dx && !demb) return TP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(emb) || !aligned16(ws) || (dx && (!aligned16(dx) || !aligned16(demb))))
    return TP_ERR_INVALID_ARG;
  const XentRankLayout L = xent_rank_layout(t, tokens, vocab);
  if (ws_bytes < (dx ? L.total : L.small)) return TP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int vp = vocab / t;
  const int ntiles = (vp + kXentTileN - 1) / kXentTileN;
  float* lse_loc = at<float>(ws, L.lse_loc);
  float* lse = at<float>(ws, L.lse);
  void* z = dx ? at<__nv_bfloat16>(ws, L.z) : nullptr;
  if (segment == 0) {
    // the target logit stays 0 unless the target lies in this slice
    if (cudaMemsetAsync(at<float>(ws, L.ztgt), 0, (size_t)tokens * 4, s) != cudaSuccess)
      return TP_ERR_CUDA;
    GemmDesc gd;
    gd.groups = 1;
    gd.M = tokens; gd.N = vp; gd.K = hidden;
    gd.a_mn = false; gd.lda = hidden;
    gd.b_mn = false; gd.ldb = hidden;
    gd.epi = EPI_XENT; gd.ldc = vp;
    gd.force_bn = kXentTileN;
    gd.xent_target = target;
    gd.xent_stats = at<float2>(ws, L.stats);
    gd.xent_ztgt = at<float>(ws, L.ztgt);
    gd.xent_group0 = rank;
    gd.a[0] = x;
    gd.b[0] = emb;
    gd.out[0] = z;
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
    TP_RUN(TP_KERNEL_XENT_COMBINE, 1,
           launch_xent_rank_fold(tokens, ntiles, at<float2>(ws, L.stats), at<float>(ws, L.ztgt), lse_loc,
                                 comm, s));
    return TP_OK;
  }
  if (segment == 1) {
    TP_RUN(TP_KERNEL_XENT_COMBINE, 1, launch_xent_rank_exp(tokens, lse_loc, comm, s));
    return TP_OK;
  }
  TP_RUN(TP_KERNEL_XENT_COMBINE, 2, launch_xent_rank_finish(tokens, comm, lse, loss_per_token, loss, s));
  if (!dx) return TP_OK;
  void* zp[1] = {z};
  TP_RUN(TP_KERNEL_XENT_GRAD, 1, launch_xent_grad_bf16(1, tokens, vp, zp, target, lse, s, rank));
  {
    GemmDesc wg;   // this partition's rows of dE = dz^T X
    wg.groups = 1;
    wg.M = vp; wg.N = hidden; wg.K = tokens;
    wg.a_mn = true; wg.lda = vp;
    wg.b_mn = true; wg.ldb = hidden;
    wg.epi = EPI_BF16; wg.ldc = hidden;
    wg.a[0] = z;
    wg.b[0] = x;
    wg.out[0] = demb;
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(wg, s));
    GemmDesc gd;   // this partition's term of dX = dz E
    gd.groups = 1;
    gd.M = tokens; gd.N = hidden; gd.K = vp;
    gd.a_mn = false; gd.lda = vp;
    gd.b_mn = true; gd.ldb = hidden;
    gd.epi = EPI_BF16; gd.ldc = hidden;
    gd.a[0] = z;
    gd.b[0] = emb;
    gd.out[0] = dx;
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  }
  return TP_OK;
}

// ---------------------------------------------------------------- loss, fused path
//
// The logits tile never leaves the SM in fp32: the logits GEMM's epilogue
// reduces every (token, 256-column tile) to (max, sum-exp) and picks out the
// target logit; one small kernel folds those per partition and combines the
// partitions' triples.  Only when a gradient is wanted does the epilogue also
// store the logits in bf16, which the gradient pass turns into dz in place.

size_t tp_xent_workspace_bytes(int t, int tokens, int hidden, int vocab) {
  if (t < 1 || t > TP_MAX_PARTITIONS || tokens <= 0 || hidden <= 0 || vocab <= 0) return 0;
  if (vocab % t || (vocab / t) % 8 || hidden % 8) return 0;
  return xent_fused_layout(t, tokens, vocab).total;
}

size_t tp_xent_forward_workspace_bytes(int t, int tokens, int hidden, int vocab) {
  if (tp_xent_workspace_bytes(t, tokens, hidden, vocab) == 0) return 0;
  return xent_fused_layout(t, tokens, vocab).small;
}

int vocab_parallel_xent(int t, int tokens, int hidden, int vocab, const void* x,
                        const void* const* emb, const int32_t* target, float* loss,
                        float* loss_per_token, void* dx, void* const* demb, void* ws,
                        size_t ws_bytes, void* stream) {
  if (t < 1 || tokens <= 0 || hidden <= 0 || vocab <= 0) return TP_ERR_INVALID_ARG;
  if (t > TP_MAX_PARTITIONS || vocab % t || (vocab / t) % 8 || hidden % 8)
    return TP_ERR_UNSUPPORTED;
  if (!x || !emb || !target || !loss || !ws) return TP_ERR_INVALID_ARG;
  if (dx && !demb) return TP_ERR_INVALID_ARG;
  for (int i = 0; i < t; ++i) {
    if (!emb[i] || !aligned16(emb[i])) return TP_ERR_INVALID_ARG;
    if (dx && (!demb[i] || !aligned16(demb[i]))) return TP_ERR_INVALID_ARG;
  }
  if (!aligned16(x) || !aligned16(ws) || (dx && !aligned16(dx))) return TP_ERR_INVALID_ARG;
  const XentFusedLayout L = xent_fused_layout(t, tokens, vocab);
  if (ws_bytes < (dx ? L.total : L.small)) return TP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int vp = vocab / t;
  const int ntiles = (vp + kXentTileN - 1) / kXentTileN;
  float2* stats = at<float2>(ws, L.stats);
  float* ztgt = at<float>(ws, L.ztgt);
  float* lse = at<float>(ws, L.lse);
  void* zp[TP_MAX_PARTITIONS] = {};
  if (dx)
    for (int i = 0; i < t; ++i) zp[i] = at<__nv_bfloat16>(ws, L.z) + (size_t)i * tokens * vp;
  // X1 + X2: z_i = X E_i^T, reduced to tile statistics in the epilogue
  {
    GemmDesc gd;
    gd.groups = t;
    gd.M = tokens; gd.N = vp; gd.K = hidden;
    gd.a_mn = false; gd.lda = hidden;
    gd.b_mn = false; gd.ldb = hidden;
    gd.epi = EPI_XENT; gd.ldc = vp;
    gd.force_bn = kXentTileN;
    gd.xent_target = target;
    gd.xent_stats = stats;
    gd.xent_ztgt = ztgt;
    for (int i = 0; i < t; ++i) {
      gd.a[i] = x;
      gd.b[i] = emb[i];
      gd.out[i] = zp[i];
    }
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  }
  // X3: per-partition triples combined into lse, the per-token and mean loss
  TP_RUN(TP_KERNEL_XENT_COMBINE, 2,
         launch_xent_tile_combine(t, tokens, ntiles, vocab, stats, ztgt, target, lse,
                                  loss_per_token, loss, s));
  if (!dx) return TP_OK;
  // X4: dz_i over the bf16 logits
  TP_RUN(TP_KERNEL_XENT_GRAD, 1, launch_xent_grad_bf16(t, tokens, vp, zp, target, lse, s));
  // X5: dE_i = dz_i^T X on the side stream, beside dX = sum_i dz_i E_i (the
  // 128 tiles of dX leave the last of its two waves of CTA pairs 27 % idle)
  {
    SideStream* side = nullptr;
    TP_TRY(side_stream(&side));
    std::lock_guard<std::mutex> side_lock(side->mu);
    const bool serial = profiling_on();
    const cudaStream_t ss = serial ? s : side->stream;
    GemmDesc wg;
    wg.groups = t;
    wg.M = vp; wg.N = hidden; wg.K = tokens;
    wg.a_mn = true; wg.lda = vp;
    wg.b_mn = true; wg.ldb = hidden;
    wg.epi = EPI_BF16; wg.ldc = hidden;
    for (int i = 0; i < t; ++i) {
      wg.a[i] = zp[i];
      wg.b[i] = x;
      wg.out[i] = demb[i];
    }
    GemmDesc gd;
    gd.groups = t; gd.sum_groups = 1;
    gd.M = tokens; gd.N = hidden; gd.K = vp;
    gd.a_mn = false; gd.lda = vp;
    gd.b_mn = true; gd.ldb = hidden;
    gd.epi = EPI_BF16; gd.ldc = hidden;
    for (int i = 0; i < t; ++i) {
      gd.a[i] = zp[i];
      gd.b[i] = emb[i];
    }
    gd.out[0] = dx;
    if (!serial) TP_TRY(fork_to(*side, 0, s));
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
    TP_RUN_ON(ss, TP_KERNEL_GEMM, 1, launch_gemm(wg, ss));
    if (!serial) TP_TRY(join_from(*side, s));
  }
  return TP_OK;
}

// ---------------------------------------------------------------- loss, explicit path

size_t tp_xent_explicit_workspace_bytes(int t, int tokens, int hidden, int vocab) {
  if (t < 1 || t > TP_MAX_PARTITIONS || tokens <= 0 || hidden <= 0 || vocab <= 0) return 0;
  if (vocab % t || (vocab / t) % 8 || hidden % 8) return 0;
  const size_t vp = vocab / t;
  Carver c;
  c.take((size_t)t * tokens * vp * 4);      // logits
  c.take((size_t)3 * t * tokens * 4);       // statistics
  c.take(((size_t)tokens + (tokens + 255) / 256) * 4);   // lse + block sums
  c.take((size_t)t * tokens * vp * 2);      // logit gradient
  return c.off;
}

int vocab_parallel_xent_explicit(int t, int tokens, int hidden, int vocab, const void* x,
                                 const void* const* emb, const int32_t* target, float* loss,
                                 float* loss_per_token, void* dx, void* const* demb, void* ws,
                                 size_t ws_bytes, void* stream) {
  if (t < 1 || tokens <= 0 || hidden <= 0 || vocab <= 0) return TP_ERR_INVALID_ARG;
  if (t > TP_MAX_PARTITIONS || vocab % t || (vocab / t) % 8 || hidden % 8)
    return TP_ERR_UNSUPPORTED;
  if (!x || !emb || !target || !loss || !ws) return TP_ERR_INVALID_ARG;
  if (dx && !demb) return TP_ERR_INVALID_ARG;
  for (int i = 0; i < t; ++i) {
    if (!emb[i] || !aligned16(emb[i])) return TP_ERR_INVALID_ARG;
    if (dx && (!demb[i] || !aligned16(demb[i]))) return TP_ERR_INVALID_ARG;
  }
  if (!aligned16(x) || !aligned16(ws) || (dx && !aligned16(dx))) return TP_ERR_INVALID_ARG;
  const size_t need = tp_xent_explicit_workspace_bytes(t, tokens, hidden, vocab);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int vp = vocab / t;
  Carver c;
  float* logits = at<float>(ws, c.take((size_t)t * tokens * vp * 4));
  float* stats = at<float>(ws, c.take((size_t)3 * t * tokens * 4));
  float* lse = at<float>(ws, c.take(((size_t)tokens + (tokens + 255) / 256) * 4));
  __nv_bfloat16* dlogits = at<__nv_bfloat16>(ws, c.take((size_t)t * tokens * vp * 2));
  const float* zp[TP_MAX_PARTITIONS];
  void* dzp[TP_MAX_PARTITIONS];
  for (int i = 0; i < t; ++i) {
    zp[i] = logits + (size_t)i * tokens * vp;
    dzp[i] = dlogits + (size_t)i * tokens * vp;
  }
  // X1: z_i = X E_i^T (fp32)
  {
    GemmDesc gd;
    gd.groups = t;
    gd.M = tokens; gd.N = vp; gd.K = hidden;
    gd.a_mn = false; gd.lda = hidden;
    gd.b_mn = false; gd.ldb = hidden;
    gd.epi = EPI_F32; gd.ldc = vp;
    for (int i = 0; i < t; ++i) {
      gd.a[i] = x;
      gd.b[i] = emb[i];
      gd.out[i] = const_cast<float*>(zp[i]);
    }
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  }
  // X2, X3: per-partition (max, sum-exp, target logit), combined into the loss
  TP_RUN(TP_KERNEL_XENT_STATS, 1, launch_xent_stats(t, tokens, vp, zp, target, stats, s));
  TP_RUN(TP_KERNEL_XENT_COMBINE, 2, launch_xent_combine(t, tokens, stats, lse, loss_per_token, loss, s));
  if (!dx) return TP_OK;
  // X4: dz_i
  TP_RUN(TP_KERNEL_XENT_GRAD, 1, launch_xent_grad(t, tokens, vp, zp, target, lse, dzp, s));
  // X5: dE_i = dz_i^T X ; dX = sum_i dz_i E_i
  {
    GemmDesc wg;
    wg.groups = t;
    wg.M = vp; wg.N = hidden; wg.K = tokens;
    wg.a_mn = true; wg.lda = vp;
    wg.b_mn = true; wg.ldb = hidden;
    wg.epi = EPI_BF16; wg.ldc = hidden;
    for (int i = 0; i < t; ++i) {
      wg.a[i] = dzp[i];
      wg.b[i] = x;
      wg.out[i] = demb[i];
    }
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(wg, s));
    GemmDesc gd;
    gd.groups = t; gd.sum_groups = 1;
    gd.M = tokens; gd.N = hidden; gd.K = vp;
    gd.a_mn = false; gd.lda = vp;
    gd.b_mn = true; gd.ldb = hidden;
    gd.epi = EPI_BF16; gd.ldc = hidden;
    for (int i = 0; i < t; ++i) {
      gd.a[i] = dzp[i];
      gd.b[i] = emb[i];
    }
    gd.out[0] = dx;
    TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  }
  return TP_OK;
}

int tp_gemm(int groups, int sum_groups, int m, int n, int k, const void* const* a, int a_layout,
            const void* const* b, int b_layout, void* const* c, int c_fp32, int tile_n,
            int cta_pair, void* stream) {
  if (groups < 1 || m <= 0 || n <= 0 || k <= 0 || !a || !b || !c) return TP_ERR_INVALID_ARG;
  if (groups > TP_MAX_PARTITIONS || m % 8 || n % 8 || k % 8) return TP_ERR_UNSUPPORTED;
  if ((tile_n != 0 && tile_n != 128 && tile_n != 256) || cta_pair < -1 || cta_pair > 1)
    return TP_ERR_INVALID_ARG;
  GemmDesc gd;
  gd.groups = groups;
  gd.sum_groups = sum_groups ? 1 : 0;
  gd.M = m; gd.N = n; gd.K = k;
  gd.a_mn = a_layout != 0;
  gd.lda = a_layout ? m : k;
  gd.b_mn = b_layout == 0;
  gd.ldb = b_layout ? k : n;
  gd.epi = c_fp32 ? EPI_F32 : EPI_BF16;
  gd.ldc = n;
  gd.force_bn = tile_n;
  gd.force_pair = cta_pair;
  for (int i = 0; i < groups; ++i) {
    if (!a[i] || !b[i] || !aligned16(a[i]) || !aligned16(b[i])) return TP_ERR_INVALID_ARG;
    gd.a[i] = a[i];
    gd.b[i] = b[i];
  }
  const int nout = sum_groups ? 1 : groups;
  for (int i = 0; i < nout; ++i) {
    if (!c[i] || !aligned16(c[i])) return TP_ERR_INVALID_ARG;
    gd.out[i] = c[i];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  TP_RUN(TP_KERNEL_GEMM, 1, launch_gemm(gd, s));
  return TP_OK;
}

int tp_profile_enable(int max_records) {
  Profiler& P = profiler();
  std::lock_guard<std::mutex> lock(P.mu);
  for (cudaEvent_t e : P.events) cudaEventDestroy(e);
  P.events.clear();
  P.records.clear();
  P.overflow = false;
  P.on = false;
  if (max_records <= 0) return TP_OK;
  P.events.resize(2 * (size_t)max_records);
  for (auto& e : P.events)
    if (cudaEventCreate(&e) != cudaSuccess) return TP_ERR_CUDA;
  P.records.reserve(max_records);
  P.on = true;
  return TP_OK;
}

int tp_profile_reset(void) {
  Profiler& P = profiler();
  std::lock_guard<std::mutex> lock(P.mu);
  P.records.clear();
  P.overflow = false;
  return TP_OK;
}

int tp_profile_summary(int kind, int* kernels, double* total_ms) {
  if (kind < 0 || kind >= TP_KERNEL_CLASSES || !kernels || !total_ms) return TP_ERR_INVALID_ARG;
  Profiler& P = profiler();
  std::lock_guard<std::mutex> lock(P.mu);
  int k = 0;
  double ms = 0.0;
  for (const ProfRecord& r : P.records) {
    if (r.kind != kind) continue;
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return TP_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) return TP_ERR_CUDA;
    k += r.kernels;
    ms += t;
  }
  *kernels = k;
  *total_ms = ms;
  return P.overflow ? TP_ERR_WORKSPACE : TP_OK;
}

int tp_profile_record(int index, int* kind, int* kernels, double* ms) {
  if (!kind || !kernels || !ms) return TP_ERR_INVALID_ARG;
  Profiler& P = profiler();
  std::lock_guard<std::mutex> lock(P.mu);
  if (index < 0 || (size_t)index >= P.records.size()) return TP_ERR_INVALID_ARG;
  const ProfRecord& r = P.records[index];
  if (cudaEventSynchronize(r.stop) != cudaSuccess) return TP_ERR_CUDA;
  float t = 0.f;
  if (cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) return TP_ERR_CUDA;
  *kind = r.kind;
  *kernels = r.kernels;
  *ms = t;
  return TP_OK;
}

int tp_device_status(void* stream) {
  unsigned int v = 0, any = 0;
  // synchronises the stream, then every unit's error word is read and cleared
  if (gemm_read_clear_error(&v, static_cast<cudaStream_t>(stream)) != 0) return TP_ERR_CUDA;
  any |= v;
  int (*const readers[])(unsigned int*) = {attention_read_clear_error, layernorm_read_clear_error,
                                           elementwise_read_clear_error};
  for (auto rd : readers) {
    v = 0;
    if (rd(&v) != 0) return TP_ERR_CUDA;
    any |= v;
  }
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  return any ? TP_ERR_TIMEOUT : TP_OK;
}

const char* tp_status_string(int status) {
  switch (status) {
    case TP_OK: return "ok";
    case TP_ERR_INVALID_ARG: return "invalid argument";
    case TP_ERR_UNSUPPORTED: return "unsupported shape";
    case TP_ERR_WORKSPACE: return "workspace too small";
    case TP_ERR_CUDA: return "CUDA error";
    case TP_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
