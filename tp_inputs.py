"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module only draws random numbers and lays them out; it holds none of the
layer's or the loss's arithmetic.  Both the CUDA path and the fp64 oracle are
fed from here, so they see bit-identical bf16 inputs.

Draw order (one torch CPU generator per workload, seeded once):
  1. the activation input X (or the cross-entropy input),
  2. every parameter, unpartitioned, in the order of ``LAYER_PARAM_ORDER``,
  3. the upstream gradient dY (layer-only workloads),
  4. target ids, then the per-sequence padding draw u_b.
Every floating value is rounded once to bf16 (round-to-nearest-even).

Workloads follow the Megatron-LM shapes the pages discuss: GPT-2 355M, the
8.3B GPT-2-style model and the 3.9B BERT model (Megatron-LM show notes, the
"model size vs. performance" outline items), with the layer split t ways
(intra-layer model parallelism) and the output embedding split by vocabulary.
"""
from __future__ import annotations

import dataclasses

import torch

# Parameter draw order; also the order of the C-ABI weight struct.
LAYER_PARAM_ORDER = (
    "ln1_g", "ln1_b",
    "w_q", "w_k", "w_v", "b_q", "b_k", "b_v",
    "w_o", "b_o",
    "ln2_g", "ln2_b",
    "w_fc1", "b_fc1", "w_fc2", "b_fc2",
)

WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class LayerDims:
    batch: int
    seq: int
    hidden: int
    heads: int
    ffn: int
    t: int
    causal: bool = True
    padding: float = 0.0     # max fraction of each sequence that is padding (BERT workload)
    vocab: int = 0           # >0: the layer output feeds a vocab-parallel loss
    ln_eps: float = 1e-5

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    @property
    def head_dim(self) -> int:
        return self.hidden // self.heads


@dataclasses.dataclass(frozen=True)
class XentDims:
    tokens: int
    hidden: int
    vocab: int
    t: int


# Named workloads (sizes as the benchmark and parity tests use them).
WORKLOADS = {
    # tiny GPT layer + loss, t=2
    "tiny_gpt_t2": LayerDims(batch=2, seq=128, hidden=256, heads=4, ffn=1024, t=2, vocab=1024),
    # GPT-2 355M-shape layer
    "gpt2_355m_t1": LayerDims(batch=8, seq=1024, hidden=1024, heads=16, ffn=4096, t=1),
    "gpt2_355m_t2": LayerDims(batch=8, seq=1024, hidden=1024, heads=16, ffn=4096, t=2),
    "gpt2_355m_t4": LayerDims(batch=8, seq=1024, hidden=1024, heads=16, ffn=4096, t=4),
    # 8.3B-scale GPT layer, 8 logical partitions
    "gpt_8p3b_t8": LayerDims(batch=4, seq=1024, hidden=3072, heads=32, ffn=12288, t=8),
    # 3.9B-scale BERT layer: bidirectional, key padding 0-10% per sequence
    "bert_3p9b_t4": LayerDims(batch=16, seq=512, hidden=2560, heads=40, ffn=10240, t=4,
                              causal=False, padding=0.10),
}
XENT_WORKLOADS = {
    f"xent_50k_t{t}": XentDims(tokens=8192, hidden=1024, vocab=50304, t=t) for t in (1, 2, 4, 8)
}


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def _normal(gen, shape, std=1.0, mean=0.0):
    return _bf16(torch.randn(*shape, generator=gen, dtype=torch.float32) * std + mean)


def param_shapes(d: LayerDims) -> dict:
    h, f = d.hidden, d.ffn
    return {
        "ln1_g": (h,), "ln1_b": (h,),
        "w_q": (h, h), "w_k": (h, h), "w_v": (h, h),
        "b_q": (h,), "b_k": (h,), "b_v": (h,),
        "w_o": (h, h), "b_o": (h,),
        "ln2_g": (h,), "ln2_b": (h,),
        "w_fc1": (h, f), "b_fc1": (f,), "w_fc2": (f, h), "b_fc2": (h,),
    }


def make_layer_inputs(d: LayerDims, seed: int = 0, need_dy: bool = True) -> dict:
    """Unpartitioned bf16 inputs of one layer workload (CPU tensors).

    Weights are stored input-major, as the pages write the MLP: Y = GeLU(X A),
    Z = Y B, so A is [h, f] and B is [f, h]; W_q/W_k/W_v are [h, h] with head j
    owning columns [j*d, (j+1)*d).
    """
    gen = torch.Generator().manual_seed(seed)
    out = {"x": _normal(gen, (d.batch, d.seq, d.hidden))}
    shapes = param_shapes(d)
    for name in LAYER_PARAM_ORDER:
        if name in ("ln1_g", "ln2_g"):
            out[name] = _normal(gen, shapes[name], std=WEIGHT_STD, mean=1.0)
        else:
            out[name] = _normal(gen, shapes[name], std=WEIGHT_STD)
    if d.vocab:
        out["emb"] = _normal(gen, (d.vocab, d.hidden), std=WEIGHT_STD)
    if need_dy and not d.vocab:
        out["dy"] = _normal(gen, (d.batch, d.seq, d.hidden))
    if d.vocab:
        out["target"] = torch.randint(0, d.vocab, (d.tokens,), generator=gen, dtype=torch.int32)
    if d.padding > 0:
        u = torch.rand(d.batch, generator=gen, dtype=torch.float64)
        pads = torch.floor(u * d.padding * d.seq).to(torch.int32)
        out["valid_len"] = (d.seq - pads).to(torch.int32)
    return out


def make_xent_inputs(d: XentDims, seed: int = 0) -> dict:
    gen = torch.Generator().manual_seed(seed)
    x = _normal(gen, (d.tokens, d.hidden))
    emb = _normal(gen, (d.vocab, d.hidden), std=WEIGHT_STD)
    target = torch.randint(0, d.vocab, (d.tokens,), generator=gen, dtype=torch.int32)
    return {"x": x, "emb": emb, "target": target}


def partition_layer_params(p: dict, t: int, heads: int) -> dict:
    """Slice unpartitioned parameters into t partitions (pure layout).

    Partition i owns heads [i*H/t, (i+1)*H/t): its fused QKV weight is the
    concatenation [W_q cols | W_k cols | W_v cols] of those heads, [h, 3h/t].
    It owns MLP columns [i*f/t, (i+1)*f/t) of A (FC1) and the same rows of B
    (FC2), and rows [i*h/t, (i+1)*h/t) of W_o.  Row-split biases b_o, b_fc2 and
    the LayerNorm parameters stay whole (replicated).
    """
    h = p["w_q"].shape[0]
    f = p["w_fc1"].shape[1]
    assert heads % t == 0 and f % t == 0
    hs, fs = h // t, f // t
    parts = {k: [] for k in ("w_qkv", "b_qkv", "w_o", "w_fc1", "b_fc1", "w_fc2")}
    for i in range(t):
        c = slice(i * hs, (i + 1) * hs)
        parts["w_qkv"].append(torch.cat([p["w_q"][:, c], p["w_k"][:, c], p["w_v"][:, c]], 1).contiguous())
        parts["b_qkv"].append(torch.cat([p["b_q"][c], p["b_k"][c], p["b_v"][c]]).contiguous())
        parts["w_o"].append(p["w_o"][c, :].contiguous())
        m = slice(i * fs, (i + 1) * fs)
        parts["w_fc1"].append(p["w_fc1"][:, m].contiguous())
        parts["b_fc1"].append(p["b_fc1"][m].contiguous())
        parts["w_fc2"].append(p["w_fc2"][m, :].contiguous())
    for k in ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "b_o", "b_fc2"):
        parts[k] = p[k]
    return parts


def partition_vocab(emb: torch.Tensor, t: int) -> list:
    """Rows [i*V/t, (i+1)*V/t) of the output embedding go to partition i."""
    v = emb.shape[0]
    assert v % t == 0
    vs = v // t
    return [emb[i * vs:(i + 1) * vs].contiguous() for i in range(t)]


def layer_flops(d: LayerDims, valid_len=None) -> float:
    """Algorithmic matmul flops of one layer forward+backward.

    GEMMs: forward 2N(3h*h + h*h + h*f + f*h), backward twice that.  Attention
    counts only kept (query, key) pairs: forward 2 matmuls, backward 4, each
    2*d flops per pair per head.  No recompute, LayerNorm or element-wise work.
    """
    n, h, f = d.tokens, d.hidden, d.ffn
    gemm = 3 * 2 * n * (3 * h * h + h * h + 2 * h * f)
    if d.causal:
        pairs = d.batch * d.seq * (d.seq + 1) // 2
    elif valid_len is not None:
        pairs = d.seq * int(sum(int(v) for v in valid_len))
    else:
        pairs = d.batch * d.seq * d.seq
    attn = 12 * h * pairs      # (2 fwd + 4 bwd matmuls) * 2 flops * d * heads = 12*h per pair
    return float(gemm + attn)


def xent_flops(d: XentDims) -> float:
    """Logits GEMM forward plus the two backward GEMMs."""
    return float(3 * 2 * d.tokens * d.hidden * d.vocab)


def xent_stream_bytes(d: XentDims) -> float:
    """Algorithmic HBM bytes of the bandwidth-bound loss kernels.

    Read the fp32 logits once for the partition statistics, once for the
    gradient, and write the bf16 logit gradient once.
    """
    return float(d.tokens * d.vocab * (4 + 4 + 2))


def xent_fused_stream_bytes(d: XentDims) -> float:
    """Algorithmic HBM bytes of the fused loss's one bandwidth-bound pass: the
    bf16 logits the GEMM epilogue stored are read once and the bf16 logit
    gradient written over them."""
    return float(d.tokens * d.vocab * (2 + 2))


def padded_len_summary(valid_len) -> str:
    vals = [int(v) for v in valid_len]
    return f"min {min(vals)} max {max(vals)} mean {sum(vals) / len(vals):.1f}"


def assemble_layer_grads(g: dict, t: int) -> dict:
    """Inverse of partition_layer_params for gradients: partition buffers -> unpartitioned."""
    out = {k: g[k] for k in ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "b_o", "b_fc2")}
    hs = g["w_qkv"][0].shape[1] // 3
    for j, nm in enumerate("qkv"):
        out["w_" + nm] = torch.cat([w[:, j * hs:(j + 1) * hs] for w in g["w_qkv"]], 1)
        out["b_" + nm] = torch.cat([b[j * hs:(j + 1) * hs] for b in g["b_qkv"]], 0)
    out["w_o"] = torch.cat(list(g["w_o"]), 0)
    out["w_fc1"] = torch.cat(list(g["w_fc1"]), 1)
    out["b_fc1"] = torch.cat(list(g["b_fc1"]), 0)
    out["w_fc2"] = torch.cat(list(g["w_fc2"]), 0)
    return out
