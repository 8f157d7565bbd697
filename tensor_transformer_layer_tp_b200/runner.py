"""Buffer management around the C-ABI calls (torch is used for device memory only)."""
from __future__ import annotations

import torch

from . import binding as B

PARTITIONED = ("w_qkv", "b_qkv", "w_o", "w_fc1", "b_fc1", "w_fc2")
REPLICATED = ("ln1_g", "ln1_b", "b_o", "ln2_g", "ln2_b", "b_fc2")


def params_to(parts: dict, device) -> dict:
    """Move partitioned parameters (dict of tensors / lists of tensors) to `device`."""
    out = {}
    for k in REPLICATED:
        out[k] = parts[k].to(device).contiguous()
    for k in PARTITIONED:
        out[k] = [p.to(device).contiguous() for p in parts[k]]
    return out


def empty_grads_like(params: dict) -> dict:
    g = {k: torch.empty_like(params[k]) for k in REPLICATED}
    for k in PARTITIONED:
        g[k] = [torch.empty_like(p) for p in params[k]]
    return g


class LayerRunner:
    """Owns the output, saved-activation, gradient and scratch buffers of one layer."""

    def __init__(self, dims: B.tp_layer_dims, params: dict, device="cuda"):
        self.dims = dims
        self.params = params
        n = dims.batch * dims.seq
        self.y = torch.empty(dims.batch, dims.seq, dims.hidden, dtype=torch.bfloat16, device=device)
        self.dx = torch.empty_like(self.y)
        self.saved = torch.empty(B.tp_layer_saved_bytes(dims), dtype=torch.uint8, device=device)
        self.ws = torch.empty(B.tp_layer_workspace_bytes(dims), dtype=torch.uint8, device=device)
        fws = B.tp_layer_forward_workspace_bytes(dims)
        self.fws = torch.empty(fws, dtype=torch.uint8, device=device) if fws else None
        self.grads = empty_grads_like(params)
        assert self.saved.numel() > 0 and self.ws.numel() > 0 and n > 0

    def forward(self, x, valid_len=None, stream=None):
        B.tp_layer_forward(self.dims, self.params, x, valid_len, self.y, self.saved, stream,
                           ws=self.fws)
        return self.y

    def backward(self, x, dy, valid_len=None, stream=None):
        B.tp_layer_backward(self.dims, self.params, x, valid_len, self.saved, dy, self.dx,
                            self.grads, self.ws, stream)
        return self.dx, self.grads

    def capture_step(self, x, dy, valid_len=None):
        """Record forward + backward on these input buffers as a CUDA graph;
        `graph.replay()` reruns the step (refill x / dy in place between
        replays).  One eager step on a side stream first does the library's
        one-time setup; per-launch profiling is off while recording."""
        import torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.forward(x, valid_len)
            self.backward(x, dy, valid_len)
        torch.cuda.current_stream().wait_stream(side)
        B.tp_profile_enable(0)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.forward(x, valid_len)
            self.backward(x, dy, valid_len)
        return graph


class XentRunner:
    """Owns the loss outputs, gradients and scratch of one vocab-parallel loss
    shape.  explicit=True runs the step-by-step fp32-logit realisation."""

    def __init__(self, t, tokens, hidden, vocab, device="cuda", with_grad=True, explicit=False):
        self.t, self.tokens, self.hidden, self.vocab = t, tokens, hidden, vocab
        self.explicit = explicit
        if explicit:
            nbytes = B.tp_xent_explicit_workspace_bytes(t, tokens, hidden, vocab)
        elif with_grad:
            nbytes = B.tp_xent_workspace_bytes(t, tokens, hidden, vocab)
        else:
            nbytes = B.tp_xent_forward_workspace_bytes(t, tokens, hidden, vocab)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.loss = torch.empty(1, dtype=torch.float32, device=device)
        self.loss_tok = torch.empty(tokens, dtype=torch.float32, device=device)
        self.dx = torch.empty(tokens, hidden, dtype=torch.bfloat16, device=device) if with_grad else None
        self.demb = ([torch.empty(vocab // t, hidden, dtype=torch.bfloat16, device=device)
                      for _ in range(t)] if with_grad else None)

    def __call__(self, x, emb: list, target, stream=None):
        B.vocab_parallel_xent(self.t, self.tokens, self.hidden, self.vocab, x, emb, target,
                              self.loss, self.loss_tok, self.dx, self.demb, self.ws, stream,
                              explicit=self.explicit)
        return self.loss


class StackRunner:
    """A GPT stack with tied embeddings, composed from the C-ABI calls: the
    vocab-parallel input embedding, `len(layer_params)` layers, the
    vocab-parallel loss on the last layer's output with the same embedding
    partitions as the output layer, and the backward through all of them, the
    input embedding's gradient added to the output layer's (one shared E).
    Owns every buffer; every step runs in the library's kernels."""

    def __init__(self, dims: B.tp_layer_dims, layer_params: list, emb_parts: list, vocab: int,
                 device="cuda"):
        self.dims, self.emb, self.vocab = dims, emb_parts, vocab
        self.n = dims.batch * dims.seq
        self.layers = [LayerRunner(dims, p, device) for p in layer_params]
        self.xent = XentRunner(dims.t, self.n, dims.hidden, vocab, device)
        self.x0 = torch.empty(dims.batch, dims.seq, dims.hidden, dtype=torch.bfloat16, device=device)
        self.ews = torch.empty(B.tp_embedding_backward_workspace_bytes(dims.t, self.n, dims.hidden, vocab),
                               dtype=torch.uint8, device=device)

    def step(self, ids, targets, stream=None):
        """Forward and backward of one batch: returns the loss tensor; the
        gradients are in self.demb (shared E) and self.layers[l].grads."""
        d = self.dims
        B.vocab_parallel_embedding_forward(d.t, self.n, d.hidden, self.vocab, ids, self.emb, self.x0,
                                           stream)
        inputs = [self.x0]
        for r in self.layers:
            inputs.append(r.forward(inputs[-1], None, stream))
        self.xent(inputs[-1].view(self.n, d.hidden), self.emb, targets, stream)
        dy = self.xent.dx.view(d.batch, d.seq, d.hidden)
        for r, x in zip(reversed(self.layers), reversed(inputs[:-1])):
            dy, _ = r.backward(x, dy, None, stream)
        B.vocab_parallel_embedding_backward(d.t, self.n, d.hidden, self.vocab, ids, dy, self.xent.demb,
                                            True, self.ews, stream)
        return self.xent.loss

    @property
    def demb(self):
        return self.xent.demb


class RankRunner:
    """Owns the buffers of partition `rank` of one layer on this device (the
    rank-local calls): `params` holds the rank's partitioned tensors as
    one-element lists (PartitionShard.slice_params, wrapped) and the replicated
    ones whole.  forward / backward walk the three segments of a pass and call
    `all_reduce(partial)` -- a sum over the group, in place -- at each of the
    two sum points; every step on this device runs in the library's kernels."""

    def __init__(self, dims: B.tp_layer_dims, rank: int, params: dict, device="cuda"):
        self.dims, self.rank, self.params = dims, rank, params
        self.y = torch.empty(dims.batch, dims.seq, dims.hidden, dtype=torch.bfloat16, device=device)
        self.dx = torch.empty_like(self.y)
        self.partial = torch.empty_like(self.y)
        self.saved = torch.empty(B.tp_layer_rank_saved_bytes(dims), dtype=torch.uint8, device=device)
        self.ws = torch.empty(B.tp_layer_rank_workspace_bytes(dims), dtype=torch.uint8, device=device)
        self.grads = empty_grads_like(params)
        assert self.saved.numel() > 0 and self.ws.numel() > 0

    def forward_segment(self, segment, x, valid_len=None, stream=None):
        B.tp_layer_rank_forward(self.dims, self.rank, segment, self.params, x, valid_len, self.partial,
                                self.y, self.saved, stream)

    def backward_segment(self, segment, x, dy, valid_len=None, stream=None):
        B.tp_layer_rank_backward(self.dims, self.rank, segment, self.params, x, valid_len, self.saved, dy,
                                 self.partial, self.dx, self.grads, self.ws, stream)

    def forward(self, x, all_reduce, valid_len=None, stream=None):
        for seg in range(3):
            if seg:
                all_reduce(self.partial)
            self.forward_segment(seg, x, valid_len, stream)
        return self.y

    def backward(self, x, dy, all_reduce, valid_len=None, stream=None):
        for seg in range(3):
            if seg:
                all_reduce(self.partial)
            self.backward_segment(seg, x, dy, valid_len, stream)
        return self.dx, self.grads


class RankXentRunner:
    """Owns the buffers of vocab partition `rank`'s loss on this device: the
    [3][tokens] fp32 values the ranks reduce (`comm`), the loss outputs, and
    with a gradient this partition's dX term and dE rows.  __call__ walks the
    three segments with the caller's collectives in between:
    all_reduce_max(comm[0:1]), then all_reduce_sum(comm[1:3]), and (with a
    gradient) all_reduce_sum(dx) at the end."""

    def __init__(self, t, rank, tokens, hidden, vocab, device="cuda", with_grad=True):
        self.t, self.rank, self.tokens, self.hidden, self.vocab = t, rank, tokens, hidden, vocab
        nbytes = B.tp_xent_rank_workspace_bytes(t, tokens, hidden, vocab)
        assert nbytes > 0
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.comm = torch.empty(3, tokens, dtype=torch.float32, device=device)
        self.loss = torch.empty(1, dtype=torch.float32, device=device)
        self.loss_tok = torch.empty(tokens, dtype=torch.float32, device=device)
        self.dx = torch.empty(tokens, hidden, dtype=torch.bfloat16, device=device) if with_grad else None
        self.demb = (torch.empty(vocab // t, hidden, dtype=torch.bfloat16, device=device)
                     if with_grad else None)

    def segment(self, seg, x, emb, target, stream=None):
        B.vocab_parallel_xent_rank(self.t, self.rank, seg, self.tokens, self.hidden, self.vocab, x, emb,
                                   target, self.comm, self.loss, self.loss_tok, self.dx, self.demb,
                                   self.ws, stream)

    def __call__(self, x, emb, target, all_reduce_max, all_reduce_sum, stream=None):
        self.segment(0, x, emb, target, stream)
        all_reduce_max(self.comm[0])
        self.segment(1, x, emb, target, stream)
        all_reduce_sum(self.comm[1:3])
        self.segment(2, x, emb, target, stream)
        if self.dx is not None:
            all_reduce_sum(self.dx)
        return self.loss
