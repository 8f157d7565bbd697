"""Partition i of the layer on GPU i: the plumbing of cross-device tensor parallelism.

Megatron-LM's intra-layer parallelism puts partition i -- heads
[i H/t, (i+1) H/t), MLP columns [i f/t, (i+1) f/t), vocabulary rows
[i V/t, (i+1) V/t) -- on GPU i, and joins the partitions with two
all-reduces per module, four per layer, and the loss's combine of the
per-partition (max, sum-exp, target logit) triples (Megatron-LM show notes,
the outline items on the MLP / self-attention split and the output
embedding; rkmt.cn guide, section 2.1: tensor parallelism inside one NVLink
domain).  On one GPU the library runs these sums inside the GEMMs' K-loops.
Across GPUs they become collectives; this module holds what does not depend
on where the kernels run:

* ``Collective``: the sums and maxima over the tensor-parallel group, over
  torch.distributed (NCCL between GPUs, gloo on CPU for tests).
* ``PartitionShard``: what rank i owns, and its slices of unpartitioned
  parameters (weights are stored input-major: W_qkv [h, 3h], W_o [h, h],
  A [h, f], B [f, h], E [V, h]).
* ``LAYER_FORWARD`` / ``LAYER_BACKWARD``: the order of rank-local steps and
  collectives of one layer, and ``run_schedule`` that walks it, calling a
  rank-local compute object for every local step and the collective at every
  sum point.
* ``combine_loss_triples``: the vocab-parallel loss across ranks.

The rank-local steps are the library's kernels restricted to one partition:
``tp_layer_rank_forward`` / ``tp_layer_rank_backward`` (``runner.RankRunner``)
run the spans between the sum points on this device, and ``run_rank_layer``
below joins them with the group's all-reduce (NCCL between GPUs).  The
kernels are checked on one GPU with the ranks run one after another and the
sums formed on the host between segments; the schedule is checked with gloo
ranks on CPU.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Dict, List, Sequence

import torch


class Collective:
    """Sums and maxima over the ranks of a tensor-parallel group (in place)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)

    def all_reduce_sum(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
        return t

    def all_reduce_max(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)
        return t


@dataclasses.dataclass(frozen=True)
class PartitionShard:
    """What partition `rank` of `t` owns in a layer of `heads` heads, MLP
    width `ffn`, hidden size `hidden` and (optionally) vocabulary `vocab`."""
    rank: int
    t: int
    hidden: int
    heads: int
    ffn: int
    vocab: int = 0

    def __post_init__(self):
        if not 0 <= self.rank < self.t:
            raise ValueError("rank outside the group")
        if self.heads % self.t or self.ffn % self.t or (self.vocab and self.vocab % self.t):
            raise ValueError("heads, ffn and vocab must split evenly into t partitions")

    @property
    def head_range(self):
        hp = self.heads // self.t
        return range(self.rank * hp, (self.rank + 1) * hp)

    @property
    def hidden_cols(self) -> slice:
        """Columns of Q, K, V (and rows of W_o) of this partition's heads."""
        w = self.hidden // self.t
        return slice(self.rank * w, (self.rank + 1) * w)

    @property
    def ffn_cols(self) -> slice:
        w = self.ffn // self.t
        return slice(self.rank * w, (self.rank + 1) * w)

    @property
    def vocab_rows(self) -> slice:
        w = self.vocab // self.t
        return slice(self.rank * w, (self.rank + 1) * w)

    def slice_params(self, p: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
        """This partition's parameters from unpartitioned ones: the fused Q|K|V
        columns of its heads, its W_o rows, its A columns and B rows; the
        LayerNorm parameters and the row-split biases b_o, b_fc2 stay whole
        (replicated, added once after the sum)."""
        c, m = self.hidden_cols, self.ffn_cols
        out = {
            "w_qkv": torch.cat([p["w_q"][:, c], p["w_k"][:, c], p["w_v"][:, c]], 1).contiguous(),
            "b_qkv": torch.cat([p["b_q"][c], p["b_k"][c], p["b_v"][c]]).contiguous(),
            "w_o": p["w_o"][c, :].contiguous(),
            "w_fc1": p["w_fc1"][:, m].contiguous(),
            "b_fc1": p["b_fc1"][m].contiguous(),
            "w_fc2": p["w_fc2"][m, :].contiguous(),
        }
        for k in ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "b_o", "b_fc2"):
            out[k] = p[k]
        return out


# --------------------------------------------------------------------- the schedule of one layer
#
# Local steps name rank-local computations (one partition's heads / columns;
# replicated steps run identically on every rank); ("sum", name) marks an
# all-reduce of the named partial.  Forward: the sums after the row-parallel
# W_o and B; backward: the sums into the inputs of the column-parallel A and
# Q/K/V projections (the f / g operators of the show notes' MLP split).

SUM = "sum"

LAYER_FORWARD = (
    "ln1",                 # Xn1 = LN1(X)                        (replicated)
    "qkv",                 # QKV_i = Xn1 W_qkv,i + b_qkv,i        (own heads)
    "attention",           # O_i                                  (own heads)
    "attn_out_partial",    # P1 = O_i W_o,i
    (SUM, "attn_out_partial"),
    "residual1",           # H1 = X + drop(P1 + b_o)              (replicated)
    "ln2",                 # Xn2 = LN2(H1)                        (replicated)
    "fc1",                 # G_i = GeLU(Xn2 A_i + b1_i)           (own columns)
    "mlp_out_partial",     # P2 = G_i B_i
    (SUM, "mlp_out_partial"),
    "residual2",           # Y = H1 + drop(P2 + b2)               (replicated)
)

LAYER_BACKWARD = (
    "mlp_out_grad",        # dZ2 = drop'(dY); db2; dB_i = G_i^T dZ2; dU_i
    "fc1_grad",            # dA_i, db1_i; partial dXn2_i = dU_i A_i^T
    (SUM, "dxn2_partial"),
    "ln2_grad",            # dH1 = dY + LN2'(dXn2)                (replicated)
    "attn_out_grad",       # dA1 = drop'(dH1); db_o; dW_o,i; dO_i
    "attention_grad",      # dQKV_i                               (own heads)
    "qkv_grad",            # dW_qkv,i, db_qkv,i; partial dXn1_i = dQKV_i W_qkv,i^T
    (SUM, "dxn1_partial"),
    "ln1_grad",            # dX = dH1 + LN1'(dXn1)                (replicated)
)


def sum_points(schedule: Sequence) -> List[str]:
    return [s[1] for s in schedule if isinstance(s, tuple) and s[0] == SUM]


def run_schedule(schedule: Sequence, compute, state: dict, coll: Collective) -> dict:
    """Walk a layer schedule on this rank: every local step calls
    compute.<step>(state) (which reads and adds entries of `state`); every sum
    point all-reduces state[name] in place over the group."""
    for step in schedule:
        if isinstance(step, tuple):
            coll.all_reduce_sum(state[step[1]])
        else:
            getattr(compute, step)(state)
    return state


# --------------------------------------------------------------------- the loss across ranks

def combine_loss_triples(m_local: torch.Tensor, s_local: torch.Tensor, z_local: torch.Tensor,
                         coll: Collective):
    """Vocab-parallel loss from each rank's (max, sum exp(z - max), target
    logit or 0) per token: M = max over ranks, S = sum over ranks of
    s exp(m - M), lse = M + log S, loss_n = lse - sum over ranks of z.
    Two all-reduces of [tokens] values (one max, one sum of [2, tokens]);
    no logit crosses ranks.  Returns (mean loss, per-token loss, lse)."""
    big = coll.all_reduce_max(m_local.clone())
    both = torch.stack([s_local * torch.exp(m_local - big), z_local])
    coll.all_reduce_sum(both)
    lse = big + torch.log(both[0])
    tok = lse - both[1]
    return tok.mean(), tok, lse


# --------------------------------------------------------------------- partition i on device i

# The rank-local calls cut each pass at its two sum points into three
# segments (include/tplayer.h): forward segment 0 = ln1 .. attn_out_partial,
# segment 1 = residual1 .. mlp_out_partial, segment 2 = residual2; backward
# segment 0 = mlp_out_grad, fc1_grad; segment 1 = ln2_grad .. qkv_grad;
# segment 2 = ln1_grad.  The sums between them are LAYER_FORWARD's and
# LAYER_BACKWARD's sum points.
def split_at_sums(schedule: Sequence) -> tuple:
    """The local steps between consecutive sum points of a schedule."""
    segs, cur = [], []
    for step in schedule:
        if isinstance(step, tuple) and step[0] == SUM:
            segs.append(tuple(cur))
            cur = []
        else:
            cur.append(step)
    segs.append(tuple(cur))
    return tuple(segs)


RANK_SEGMENTS_FORWARD = split_at_sums(LAYER_FORWARD)
RANK_SEGMENTS_BACKWARD = split_at_sums(LAYER_BACKWARD)


def run_rank_layer(runner, x, dy, coll: Collective, valid_len=None):
    """Forward and backward of partition coll.rank of one layer on this device
    (runner: runner.RankRunner for that rank): the library's rank-local
    segments, with coll's all-reduce over `runner.partial` at the four sum
    points.  Every rank gets the whole output and input gradient, its own
    partitions' weight gradients and the replicated parameters' gradients."""
    y = runner.forward(x, coll.all_reduce_sum, valid_len)
    dx, grads = runner.backward(x, dy, coll.all_reduce_sum, valid_len)
    return y, dx, grads


def run_rank_xent(runner, x, emb, target, coll: Collective):
    """Vocab partition coll.rank's loss on this device (runner:
    runner.RankXentRunner): the library's three rank-local segments with the
    group's max and sum all-reduces of the per-token statistics between them,
    and the sum of the partitions' dX terms at the end.  Only [3, tokens]
    statistics and the [tokens, h] dX cross devices, never a logit."""
    return runner(x, emb, target, coll.all_reduce_max, coll.all_reduce_sum)
