/*
 * tplayer — one Megatron-style tensor-parallel transformer layer and the
 * vocab-parallel cross-entropy, forward and backward, on one NVIDIA B200
 * (sm_100a).  C ABI: plain pointers and sizes only.
 *
 * What is computed (Megatron-LM show notes, "intra-layer parallel
 * implementation" outline; rkmt.cn guide, section 3 "Transformer layer
 * splitting"):
 *   pre-LN layer   H1 = X + b_o + sum_i O_i W_o,i
 *                  O_i = attention over the heads of partition i of
 *                        Q/K/V_i = LN1(X) W_qkv,i + b_qkv,i
 *                  Y  = H1 + b2 + sum_i GeLU(LN2(H1) A_i + b1_i) B_i
 *   loss           z_i = X E_i^T (vocab rows of partition i),
 *                  loss = mean_n [ logsumexp_v z_n - z_n[target_n] ],
 *                  combined from per-partition (max, sum-exp, target logit).
 * The t tensor-parallel partitions are t logical slices on one device: every
 * partition-owned tensor is passed as t separate buffers, and the all-reduce
 * points of the method (after W_o and B in the forward, into the inputs of
 * the column-split linears in the backward, the loss triple, the loss input
 * gradient) are sums over those buffers done on the device.
 *
 * Conventions
 *   - bf16 storage, fp32 accumulation.  "bf16" below means IEEE bfloat16.
 *   - Row-major.  Activations are [batch, seq, hidden] (token n = b*seq + pos).
 *   - Weights are stored input-major as the pages write the MLP (X A, Y B):
 *       w_qkv[i] [h][3h/t]  columns = [Q of its heads | K of its heads | V ...],
 *                           head-major, head_dim contiguous; partition i owns
 *                           heads [i*H/t, (i+1)*H/t)
 *       w_o[i]   [h/t][h]   rows of W_o belonging to those heads
 *       w_fc1[i] [h][f/t]   columns [i*f/t, (i+1)*f/t) of A
 *       w_fc2[i] [f/t][h]   the same rows of B
 *       b_qkv[i] [3h/t], b_fc1[i] [f/t] (split with their columns);
 *       b_o, b_fc2, ln*_g, ln*_b [h] are replicated (added once).
 *       emb[i]   [V/t][h]   vocabulary rows [i*V/t, (i+1)*V/t)
 *   - Ownership: the caller owns every buffer (all device memory unless
 *     stated).  The library never allocates, frees or synchronises, except
 *     tp_device_status().  Work is enqueued on `stream` (a cudaStream_t;
 *     NULL = legacy default stream).
 *   - Gradients are overwritten, not accumulated.
 *   - Errors: argument and support errors return before any launch; a failed
 *     launch returns TP_ERR_CUDA.  Every wait inside a kernel is bounded;
 *     a wait that runs out sets a device-side error word that
 *     tp_device_status() reports as TP_ERR_TIMEOUT.
 *   - Support: 1 <= t <= 8, H % t == 0, f % t == 0, V % t == 0, h % H == 0,
 *     head_dim in {64, 96, 128}, h % 64 == 0, h <= 4096, f/t % 64 == 0,
 *     (V/t) % 8 == 0, 1 <= seq, batch.  Outside: TP_ERR_UNSUPPORTED, no
 *     fallback.  Every device pointer must be 16-byte aligned.
 */
#ifndef TPLAYER_H_
#define TPLAYER_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TP_MAX_PARTITIONS 8

#if defined(__GNUC__)
#define TP_API __attribute__((visibility("default")))
#else
#define TP_API
#endif

typedef enum {
  TP_OK = 0,
  TP_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad alignment */
  TP_ERR_UNSUPPORTED = 2, /* outside the support matrix above */
  TP_ERR_WORKSPACE = 3,   /* workspace smaller than the *_workspace_bytes() value */
  TP_ERR_CUDA = 4,        /* a CUDA call or launch failed */
  TP_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out (see tp_device_status) */
} tp_status;

/* Layer shape and options.  causal = 1: key k attends only to query
 * positions >= k (GPT); causal = 0: bidirectional (BERT), optionally with key
 * padding.
 *
 * Dropout (Megatron-LM show notes: dropout is replicated on every partition,
 * not split): dropout_attn on the attention probabilities, dropout_hidden on
 * the outputs of the out-projection and of FC2 before their residual adds;
 * rates in [0, 1), 0 = off.  A value is dropped when its 32-bit draw is below
 * floor(rate * 2^32); kept values are scaled by 1 / (1 - rate).  The draws
 * come from the counter-based generator Philox-4x32-10 (Salmon et al., SC
 * 2011) under key (seed mod 2^32, seed div 2^32): element (row, col) takes
 * word col % 4 of the block at counter (col / 4, row, site, 0), with rows and
 * columns global -- (token, hidden column) for the hidden outputs (site 1
 * after the out-projection, 2 after FC2), ((batch * heads + head) * seq +
 * query, key) for the attention probabilities (site 0) -- so the masks do not
 * depend on t, and the backward regenerates exactly the forward's masks.
 * Attention dropout needs batch * heads * seq < 2^32.
 *
 * recompute = 1 (activation recomputation): the forward keeps only the
 * LayerNorm statistics and the attention log-sum-exp in `saved`; its other
 * activations go to the forward workspace, and the backward rebuilds them
 * from x (applying the saved statistics) before computing the gradients,
 * which equal those of recompute = 0. */
typedef struct {
  int t;       /* tensor-parallel partitions (1..8) */
  int batch;   /* B */
  int seq;     /* s */
  int hidden;  /* h */
  int heads;   /* H */
  int ffn;     /* f (4h in Megatron-LM) */
  int causal;
  float ln_eps;
  float dropout_attn;        /* rate on the attention probabilities */
  float dropout_hidden;      /* rate on the out-projection and FC2 outputs */
  unsigned long long seed;   /* dropout generator key */
  int recompute;             /* 0: save activations; 1: rebuild them in the backward */
} tp_layer_dims;

/* Parameters (device pointers, bf16).  Arrays hold t partition buffers. */
typedef struct {
  const void* ln1_g;
  const void* ln1_b;
  const void* w_qkv[TP_MAX_PARTITIONS];
  const void* b_qkv[TP_MAX_PARTITIONS];
  const void* w_o[TP_MAX_PARTITIONS];
  const void* b_o;
  const void* ln2_g;
  const void* ln2_b;
  const void* w_fc1[TP_MAX_PARTITIONS];
  const void* b_fc1[TP_MAX_PARTITIONS];
  const void* w_fc2[TP_MAX_PARTITIONS];
  const void* b_fc2;
} tp_layer_weights;

/* Parameter gradients: same shapes and layout as tp_layer_weights, written. */
typedef struct {
  void* ln1_g;
  void* ln1_b;
  void* w_qkv[TP_MAX_PARTITIONS];
  void* b_qkv[TP_MAX_PARTITIONS];
  void* w_o[TP_MAX_PARTITIONS];
  void* b_o;
  void* ln2_g;
  void* ln2_b;
  void* w_fc1[TP_MAX_PARTITIONS];
  void* b_fc1[TP_MAX_PARTITIONS];
  void* w_fc2[TP_MAX_PARTITIONS];
  void* b_fc2;
} tp_layer_grads;

/* Bytes of the activation buffer the forward fills and the backward reads:
 * the LayerNorm statistics and the attention log-sum-exp, and with
 * recompute = 0 also the LN outputs, per-partition Q/K/V and attention
 * outputs, H1, the GeLU output and its derivative at the GeLU input.
 * 0 if dims unsupported. */
TP_API size_t tp_layer_saved_bytes(const tp_layer_dims* dims);

/* Bytes of scratch the forward needs: 0 with recompute = 0; with
 * recompute = 1 the activations that the backward will rebuild.  Nothing in
 * it needs to start at zero.  0 also if dims unsupported (check
 * tp_layer_saved_bytes). */
TP_API size_t tp_layer_forward_workspace_bytes(const tp_layer_dims* dims);

/* Bytes of scratch the backward needs: gradients of the intermediate
 * activations, the fp32 dQ accumulator of the attention backward, the column
 * partials of the bias / gamma / beta gradients, with hidden dropout the
 * gradients of the dropped outputs, and with recompute the rebuilt
 * activations.  Nothing in it needs to start at zero.  0 if unsupported. */
TP_API size_t tp_layer_workspace_bytes(const tp_layer_dims* dims);

/* Forward of one layer.
 *   x          [B, s, h] bf16 input
 *   valid_len  [B] int32 device array of unpadded lengths (keys at positions
 *              >= valid_len[b] are masked), or NULL for no padding
 *   y          [B, s, h] bf16 output
 *   saved      saved_bytes bytes, written; pass unchanged to backward.
 *              saved_bytes < tp_layer_saved_bytes(dims) returns
 *              TP_ERR_WORKSPACE before any launch.
 *   ws         ws_bytes >= tp_layer_forward_workspace_bytes(dims) bytes of
 *              scratch (may be NULL with 0 bytes when that is 0), else
 *              TP_ERR_WORKSPACE before any launch; free again once the
 *              enqueued work is done (the backward does not read it)
 * (Megatron-LM show notes: 2 all-reduces per layer in the forward -- here the
 * sums over partitions inside the W_o and B GEMMs.) */
TP_API int tp_layer_forward(const tp_layer_dims* dims, const tp_layer_weights* w, const void* x,
                            const int32_t* valid_len, void* y, void* saved, size_t saved_bytes,
                            void* ws, size_t ws_bytes, void* stream);

/* Backward of one layer for upstream gradient dy [B, s, h] bf16.
 *   saved      the buffer the forward filled (saved_bytes as passed there;
 *              a short one returns TP_ERR_WORKSPACE before any launch)
 *   dx         [B, s, h] bf16 input gradient, written
 *   grads      every pointer written (bf16)
 *   ws         ws_bytes >= tp_layer_workspace_bytes() bytes of scratch, else
 *              TP_ERR_WORKSPACE before any launch
 * (2 more all-reduces: into the inputs of the Q/K/V and A projections.)
 *
 * The weight-gradient GEMMs (dW_qkv,i, dW_o,i, dA_i, dB_i) run on a second,
 * low-priority library stream of the device, which waits for `stream` where
 * their inputs are ready; `stream` waits for it again before the last launch,
 * so all of the backward's work is ordered before whatever is enqueued on
 * `stream` next.  Calls from several host threads are serialised on it.
 *
 * Both calls only enqueue kernels (no allocation, no synchronisation), so a
 * forward + backward can be recorded once with CUDA stream capture and
 * replayed as a graph on the same buffers (the capture follows the fork and
 * join).  The first call on a device does one-time setup (kernel attributes,
 * and for the backward its side stream and events); make it before any
 * capture. */
TP_API int tp_layer_backward(const tp_layer_dims* dims, const tp_layer_weights* w, const void* x,
                             const int32_t* valid_len, const void* saved, size_t saved_bytes,
                             const void* dy, void* dx, const tp_layer_grads* grads, void* ws,
                             size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- rank-local layer
 *
 * Partition `rank` of the dims->t partitions on the calling device, for
 * tensor parallelism across devices (partition i on device i, Megatron-LM show
 * notes: two all-reduces per module, four per layer; rkmt.cn guide, section
 * 2.1: tensor parallelism inside one NVLink domain).  The same kernels as
 * tp_layer_forward / tp_layer_backward restricted to the partition's heads and
 * MLP columns; the four sums over partitions are left to the caller (an
 * all-reduce across the group, in bf16 as the layer's activations).  Each pass
 * is cut at its sum points into three segments:
 *
 *   forward  segment 0: LN1, QKV_i, attention of its heads, and the term
 *                       O_i W_o,i                        -> partial
 *            (caller: partial = sum over ranks of partial)
 *            segment 1: H1 = X + drop(partial + b_o), LN2, FC1_i + GeLU, and
 *                       the term G_i B_i                 -> partial
 *            (caller: sum)
 *            segment 2: Y = H1 + drop(partial + b2)      -> y
 *   backward segment 0: dropout of dY, dU_i, dB_i, db1_i, dA_i, and the term
 *                       dU_i A_i^T of dXn2               -> partial
 *            (caller: sum)
 *            segment 1: dH1 = dY + LN2'(partial), dW_o,i, attention backward
 *                       of its heads, dW_qkv,i, db_qkv,i, and the term
 *                       dQKV_i W_qkv,i^T of dXn1         -> partial
 *            (caller: sum)
 *            segment 2: dX = dH1 + LN1'(partial), and the replicated
 *                       parameters' gradients (LayerNorms, b_o, b2)
 *
 * The replicated steps (LayerNorm, residual, dropout of the hidden outputs,
 * gradients of the replicated parameters) run identically on every rank;
 * dropout masks are keyed by global positions (attention: global head
 * index), so the ranks together draw exactly the masks of the one-device
 * layer.  Arguments as for tp_layer_forward / tp_layer_backward, except:
 *   rank      0 .. dims->t - 1
 *   segment   0, 1 or 2, called in order for one pass; the same saved, ws,
 *             partial, x, dy and grads buffers throughout the pass
 *   w, grads  the partition's tensors at index 0 of the per-partition arrays
 *             (w_qkv[0] [h][3h/t], w_o[0] [h/t][h], w_fc1[0] [h][f/t],
 *             w_fc2[0] [f/t][h], b_qkv[0], b_fc1[0]); the replicated ones whole
 *   partial   [B, s, h] bf16, written at the end of segments 0 and 1, read
 *             (as the sum over ranks) at the start of segments 1 and 2
 *   saved     tp_layer_rank_saved_bytes(dims) bytes; ws
 *             tp_layer_rank_workspace_bytes(dims) bytes (backward only)
 * y is needed by forward segment 2 only, dx and grads by backward segment 2
 * (grads of the partition's own tensors are written from segment 0 on).
 * Recompute (dims->recompute = 1) is not supported here: TP_ERR_UNSUPPORTED.
 * After backward segments 0 and 1 return, weight-gradient GEMMs of the
 * segment may still run on the library's side stream of the device (beside
 * the caller's all-reduce, which only touches `partial`); backward segment 2
 * joins them into `stream`. */
TP_API size_t tp_layer_rank_saved_bytes(const tp_layer_dims* dims);
TP_API size_t tp_layer_rank_workspace_bytes(const tp_layer_dims* dims);
TP_API int tp_layer_rank_forward(const tp_layer_dims* dims, int rank, int segment,
                                 const tp_layer_weights* w, const void* x,
                                 const int32_t* valid_len, void* partial, void* y, void* saved,
                                 size_t saved_bytes, void* stream);
TP_API int tp_layer_rank_backward(const tp_layer_dims* dims, int rank, int segment,
                                  const tp_layer_weights* w, const void* x,
                                  const int32_t* valid_len, const void* saved, size_t saved_bytes,
                                  const void* dy, void* partial, void* dx,
                                  const tp_layer_grads* grads, void* ws, size_t ws_bytes,
                                  void* stream);

/* ---------------------------------------------------------------- rank-local loss
 *
 * Vocab partition `rank` of t (rows [rank V/t, (rank+1) V/t) of E) on the
 * calling device, the combine over partitions left to the caller (rkmt.cn
 * guide, section 3.3: each device keeps its slice of the logits and only
 * per-token statistics cross devices).  Three segments, with the caller's
 * collectives over `comm` ([3][tokens] fp32) in between:
 *   segment 0: the logits X E_rank^T, reduced in the GEMM epilogue to the
 *              slice's log-sum-exp per token       -> comm[0]
 *              and the target logit, 0 when the target lies in another
 *              slice                                 -> comm[2]
 *   (caller: comm[0] = max over ranks of comm[0])
 *   segment 1: comm[1] = exp(slice log-sum-exp - comm[0])
 *   (caller: comm[1] and comm[2] = sums over ranks)
 *   segment 2: lse = comm[0] + log comm[1], loss_per_token = lse - comm[2],
 *              *loss = their mean; with dx: dz = (softmax - onehot) / T over
 *              the slice, demb = dz^T X (the partition's rows of dE), and
 *              dx = dz E_rank, this partition's term of dX
 *   (caller, with dx: dx = sum over ranks of dx)
 * emb / demb: [V/t][h] bf16 of this partition; x [tokens][h] bf16; target
 * [tokens] int32 over the whole vocabulary.  dx and demb NULL for the loss
 * alone, and the same pointers in all three segments (segment 0 keeps the
 * bf16 logits in ws only when dx is given).  ws:
 * tp_xent_rank_workspace_bytes(t, tokens, hidden, vocab) bytes with a
 * gradient, else its statistics part; the same buffer in all three segments.
 * Errors as vocab_parallel_xent, plus TP_ERR_INVALID_ARG for a rank or
 * segment out of range. */
TP_API size_t tp_xent_rank_workspace_bytes(int t, int tokens, int hidden, int vocab);
TP_API int vocab_parallel_xent_rank(int t, int rank, int segment, int tokens, int hidden, int vocab,
                                    const void* x, const void* emb, const int32_t* target,
                                    float* comm, float* loss, float* loss_per_token, void* dx,
                                    void* demb, void* ws, size_t ws_bytes, void* stream);

/* Scratch bytes for vocab_parallel_xent with a gradient (dx != NULL): the
 * per-(token, 256-column tile) statistics, the target logits, the
 * log-sum-exp, and the bf16 logits of every partition, which the gradient
 * pass overwrites with the logit gradient.  0 if unsupported. */
TP_API size_t tp_xent_workspace_bytes(int t, int tokens, int hidden, int vocab);

/* Scratch bytes for vocab_parallel_xent without a gradient (dx == NULL):
 * the statistics, target logits and log-sum-exp only (no logits are stored).
 * 0 if unsupported. */
TP_API size_t tp_xent_forward_workspace_bytes(int t, int tokens, int hidden, int vocab);

/* Vocab-parallel output embedding fused with cross-entropy (Megatron-LM show
 * notes, output-embedding outline item; rkmt.cn guide, section 3.3).
 *   x               [tokens, hidden] bf16
 *   emb             host array of t device pointers, emb[i] = [V/t, hidden] bf16
 *   target          [tokens] int32 device array, values in [0, vocab)
 *   loss            [1] fp32 device: mean over tokens
 *   loss_per_token  [tokens] fp32 device, or NULL
 *   dx              [tokens, hidden] bf16 gradient of loss w.r.t. x, or NULL
 *                   for forward only
 *   demb            host array of t device pointers ([V/t, hidden] bf16
 *                   gradients), or NULL (required when dx is given)
 *   ws, ws_bytes    scratch: tp_xent_workspace_bytes() bytes with dx,
 *                   tp_xent_forward_workspace_bytes() without; smaller
 *                   returns TP_ERR_WORKSPACE before any launch
 * Full logits are never gathered: each partition reduces its own logits to
 * (max, sum-exp, target logit) and only those triples are combined.  The
 * logits GEMM does that reduction in its epilogue from the fp32 accumulator
 * (256 vocabulary columns at a time), so no fp32 logit is written to memory
 * and the loss has fp32 accuracy.  With dx, the epilogue also stores the
 * logits rounded to bf16, and the gradient (exp(z - lse) - onehot) / tokens
 * is formed from those in place before the two gradient GEMMs; the dE GEMM
 * runs on the library's side stream of the device beside the dX GEMM and is
 * joined into `stream` before the call returns (as in tp_layer_backward). */
TP_API int vocab_parallel_xent(int t, int tokens, int hidden, int vocab, const void* x,
                               const void* const* emb, const int32_t* target, float* loss,
                               float* loss_per_token, void* dx, void* const* demb, void* ws,
                               size_t ws_bytes, void* stream);

/* Scratch bytes for vocab_parallel_xent_explicit: fp32 logits of every
 * partition, the per-partition statistics, the bf16 logit gradient.
 * 0 if unsupported. */
TP_API size_t tp_xent_explicit_workspace_bytes(int t, int tokens, int hidden, int vocab);

/* The same loss realised step by step, as the method describes it: every
 * partition writes its fp32 logits z_i = X E_i^T, one pass reduces each
 * partition's logits to its (max, sum-exp, target logit) triple, the triples
 * are combined, and a second pass over the fp32 logits forms the bf16 logit
 * gradient.  Same arguments and results as vocab_parallel_xent (ws_bytes >=
 * tp_xent_explicit_workspace_bytes()); it moves the fp32 logits through
 * memory three times and serves as the reference realisation. */
TP_API int vocab_parallel_xent_explicit(int t, int tokens, int hidden, int vocab, const void* x,
                                        const void* const* emb, const int32_t* target, float* loss,
                                        float* loss_per_token, void* dx, void* const* demb,
                                        void* ws, size_t ws_bytes, void* stream);

/* vocab_parallel_xent for callers that cannot allocate device memory (no
 * counterpart in the paper: an interface convenience of this library).
 * Some callers cannot call cudaMalloc -- their device memory is owned by
 * another component (a serving process or framework allocator that reserves
 * the GPU up front and forbids later allocation), or they have no allocator at
 * hand to create and keep a workspace.  This entry point takes the same
 * arguments as vocab_parallel_xent minus ws/ws_bytes and keeps the scratch in
 * a fixed array of TP_XENT_STATIC_SCRATCH_BYTES inside the library, held on
 * every GPU that loads the library until the process exits.  It allocates
 * and frees nothing.
 *   - Size limit: calls whose tp_xent_workspace_bytes() exceeds
 *     TP_XENT_STATIC_SCRATCH_BYTES return TP_ERR_WORKSPACE before any launch
 *     (e.g. 1024 tokens x vocab 8192 fits; 8192 x 50304 does not).
 *   - The first call on a device looks up the array's device address (with
 *     that device current), and the first call with a gradient creates the
 *     library's side stream of the device (as vocab_parallel_xent does; no
 *     device memory); make it before any stream capture on the device.
 *     The address is kept per device and CUDA context: a call under another
 *     context of the device (after cudaDeviceReset, or a context the caller
 *     made current) looks it up again, so make that call outside capture too.
 *   - All calls share the array: calls that overlap on the GPU race; order them
 *     on one stream.  Nothing in the array needs to start at zero. */
#define TP_XENT_STATIC_SCRATCH_BYTES (64u << 20)
TP_API int vocab_parallel_xent_static(int t, int tokens, int hidden, int vocab, const void* x,
                                      const void* const* emb, const int32_t* target, float* loss,
                                      float* loss_per_token, void* dx, void* const* demb,
                                      void* stream);

/* Vocab-parallel input embedding (rkmt.cn guide, section 3.3: the input
 * layer is split along the vocabulary and its outputs are summed by an
 * all-reduce).  Partition i holds emb[i] = rows [i V/t, (i+1) V/t) of E
 * ([V/t, hidden] bf16); out[n] = sum_i (E_i[ids[n] - i V/t] if ids[n] is in
 * partition i's range, else 0) = E[ids[n]].  Exactly one partition owns a
 * valid id, so the sum is formed by reading the owner's row; an id outside
 * [0, vocab) gives a zero row.
 *   ids   [tokens] int32 device;  emb  host array of t device pointers
 *   out   [tokens, hidden] bf16 device, written
 * Requires 1 <= t <= 8, vocab % t == 0, hidden % 8 == 0 (TP_ERR_UNSUPPORTED
 * otherwise); NULL or unaligned pointers give TP_ERR_INVALID_ARG.  Enqueued
 * on `stream`; no allocation. */
TP_API int vocab_parallel_embedding_forward(int t, int tokens, int hidden, int vocab,
                                            const int32_t* ids, const void* const* emb, void* out,
                                            void* stream);

/* Scratch bytes of vocab_parallel_embedding_backward: an fp32 accumulator of
 * vocab x hidden.  0 if unsupported. */
TP_API size_t tp_embedding_backward_workspace_bytes(int t, int tokens, int hidden, int vocab);

/* Backward of vocab_parallel_embedding_forward: for every partition i and its
 * row r, demb[i][r] = sum of dout[n] over the tokens with ids[n] = i V/t + r
 * (accumulate = 1: added to the bf16 values already in demb[i], e.g. the
 * gradient of an output layer that shares E).  The sums run in fp32 through
 * `ws` with atomic adds, so their order (and the last bit of a row shared by
 * many tokens) can change from run to run; the result is rounded to bf16 once.
 *   dout  [tokens, hidden] bf16;  demb  host array of t device pointers
 *   ws    ws_bytes >= tp_embedding_backward_workspace_bytes(), else
 *         TP_ERR_WORKSPACE before any launch; nothing in it needs to start
 *         at zero. */
TP_API int vocab_parallel_embedding_backward(int t, int tokens, int hidden, int vocab,
                                             const int32_t* ids, const void* dout,
                                             void* const* demb, int accumulate, void* ws,
                                             size_t ws_bytes, void* stream);

/* Plain grouped / partition-summed GEMM exposed for testing and reuse:
 *   sum_groups = 0 : C_g = A_g B_g for g < groups (column-parallel linear)
 *   sum_groups = 1 : C   = sum_g A_g B_g          (row-parallel linear + all-reduce)
 * A_g is m x k: a_layout 0 = stored [m][k], 1 = stored [k][m].
 * B_g is k x n: b_layout 0 = stored [k][n], 1 = stored [n][k].
 * Dense leading dimensions (k or m for A, n or k for B, n for C).
 * c_fp32 = 1 writes fp32, else bf16.  a, b, c: host arrays of device pointers
 * (c has 1 entry when summing).  Requires m, n, k > 0 and multiples of 8.
 * Grouped calls whose groups all pass the same A pointer (or all the same B
 * pointer) are tiled as one problem with the groups' n (or m) ranges
 * concatenated when that extent is a multiple of 64 (tiles then cross group
 * edges); the results are the same.
 * Kernel choice (for tests and tuning; the layer calls always use the
 * automatic choice): tile_n = 0 (auto), 128 or 256 output columns per tile;
 * cta_pair = -1 (auto: pairs when m >= 512), 0 (one CTA per 128-row tile) or
 * 1 (two CTAs on neighbouring SMs share a 256-row tile). */
TP_API int tp_gemm(int groups, int sum_groups, int m, int n, int k, const void* const* a, int a_layout,
            const void* const* b, int b_layout, void* const* c, int c_fp32, int tile_n,
            int cta_pair, void* stream);

/* The GeLU nonlinearity of the MLP block (rkmt.cn guide, section 3.1: the
 * first linear's output goes through GeLU before the second) and its
 * derivative, exactly as the fused GEMM epilogues evaluate them:
 *   gelu[i]  = x Phi(x),   dgelu[i] = Phi(x) + x phi(x),   x = x[i], i < n,
 * Phi / phi the standard normal CDF / density.  x, gelu, dgelu: device fp32
 * arrays of n elements; gelu or dgelu may be NULL.  Enqueued on `stream`;
 * n = 0 is a no-op.  Returns TP_ERR_INVALID_ARG for n < 0 or a NULL x with
 * n > 0, TP_ERR_CUDA if the launch fails.  For tests and reuse. */
TP_API int tp_gelu_eval(int n, const float* x, float* gelu, float* dgelu, void* stream);

/* The all-reduce of a row-parallel linear done explicitly (Megatron-LM show
 * notes, the MLP split outline item: the row-split second linear's partial
 * outputs are summed by an all-reduce; rkmt.cn guide, section 3.1): every
 * partition g < t has written its fp32 partial product (e.g. tp_gemm with
 * sum_groups = 0, c_fp32 = 1), and this pass forms
 *   out[r][c] = bf16( sum_g partials[g][r][c] + bias[c] + residual[r][c] ).
 * The layer entry points do not use it: they sum inside the consuming GEMM's
 * K-loop (no partial reaches HBM).  This is the reference realisation, for
 * validation and for comparing its cost.
 *   partials   host array of t device pointers, fp32 [rows][ld], 16-byte aligned
 *   bias       bf16 [cols] device or NULL;  residual  bf16 [rows][cols] or NULL
 *   out        bf16 [rows][cols] device
 * Requires 1 <= t <= 8, cols and ld multiples of 4, ld >= cols; returns
 * TP_ERR_INVALID_ARG otherwise (before any launch), TP_ERR_CUDA if the launch
 * fails.  Enqueued on `stream`. */
TP_API int tp_partition_sum(int t, int rows, int cols, const float* const* partials, long long ld,
                            const void* bias, const void* residual, void* out, void* stream);

/* ---------------------------------------------------------------- profiling
 * Opt-in timing of the library's own kernels, for roofline reports.  While
 * enabled, every launch is bracketed by two CUDA events on its stream (host
 * resources created here, at enable time; no device memory is allocated).
 * Kernel classes: */
enum {
  TP_KERNEL_GEMM = 0,       /* tcgen05 GEMM (all linears, logits, their grads) */
  TP_KERNEL_ATTN_FWD = 1,   /* attention forward */
  TP_KERNEL_ATTN_BWD = 2,   /* attention backward (delta, main, dQ conversion) */
  TP_KERNEL_LN_FWD = 3,     /* LayerNorm forward */
  TP_KERNEL_LN_BWD = 4,     /* LayerNorm backward (+ residual gradient) */
  TP_KERNEL_REDUCE = 5,     /* column sums: bias, gamma and beta gradients */
  TP_KERNEL_XENT_STATS = 6, /* per-partition (max, sum-exp, target) statistics */
  TP_KERNEL_XENT_COMBINE = 7, /* combine of the triples and the mean loss */
  TP_KERNEL_XENT_GRAD = 8,  /* logit gradient */
  TP_KERNEL_ELEMENTWISE = 9, /* bias + dropout + residual after a sum formed by the caller */
  TP_KERNEL_CLASSES = 10
};

/* max_records > 0: enable with room for that many launches (events are
 * created now); 0: disable and release the events.  Returns a tp_status.
 * While enabled, tp_layer_backward enqueues its weight-gradient GEMMs on the
 * caller's stream too (instead of its internal side stream), so that every
 * recorded duration is that launch's alone. */
TP_API int tp_profile_enable(int max_records);

/* Forget the records taken so far (keeps profiling enabled). */
TP_API int tp_profile_reset(void);

/* Waits for the recorded launches and reports, for kernel class `kind`, the
 * number of kernels launched and their summed device time in milliseconds.
 * Returns TP_ERR_INVALID_ARG for an unknown class, TP_ERR_WORKSPACE if more
 * launches happened than max_records (the surplus was not timed). */
TP_API int tp_profile_summary(int kind, int* kernels, double* total_ms);

/* Per-launch record `index` (0 = the first launch recorded since enable or
 * reset, in enqueue order): its kernel class, the number of kernels it
 * launched and its device time in milliseconds (waits for it).  Returns
 * TP_ERR_INVALID_ARG when index is past the last record. */
TP_API int tp_profile_record(int index, int* kind, int* kernels, double* ms);

/* Self-test of the failure path (no counterpart in the pages): enqueues one
 * kernel whose wait on a shared-memory barrier is never satisfied.  The wait
 * is bounded like every wait in the library (0.5 s); when it runs out the
 * kernel records a timeout and returns, so the next tp_device_status() on
 * that stream reports TP_ERR_TIMEOUT (and clears it), and the context stays
 * usable.  Nothing is left waiting on the GPU.  Returns TP_ERR_CUDA if the
 * launch fails. */
TP_API int tp_selftest_wait_timeout(void* stream);

/* Synchronises `stream` and reports a device-side error (TP_ERR_TIMEOUT) or a
 * CUDA error (TP_ERR_CUDA); clears the device error word. */
TP_API int tp_device_status(void* stream);

TP_API const char* tp_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* TPLAYER_H_ */
