"""The rank-local layer (partition i alone, the four sums over partitions left
to the caller) through the C-ABI, against the fp64 oracle of the whole layer.

Partition i on device i is the pages' deployment (Megatron-LM show notes: two
all-reduces per module, four per layer).  Here every rank runs on the one GPU
of the test, one after another: each rank's segment is launched and finished,
then the host forms the sum over ranks of the `partial` buffers (the
all-reduce, in bf16 like the layer's activations) and hands it back to every
rank before the next segment.  No kernel of one rank waits for another
rank's; the collective across real devices is torch.distributed's, over the
same buffers (tensor_transformer_layer_tp_b200.parallel.run_rank_layer).

Checks: every rank's output and input gradient, and the gradients assembled
from the ranks' partitions, against the oracle (max|err| <= 2e-2 max|ref|);
the replicated gradients agree between ranks; with dropout, the ranks draw
the masks of the one-device layer (the oracle with the same Philox key).  The
vocab-parallel loss likewise: each rank's loss (1e-5 relative), the sum of the
ranks' dX terms and their dE slices against the oracle, with targets on every
slice edge.
"""
import pytest
import torch

from helpers import LOSS_RTOL, assert_close, f64
from oracle import tp_oracle as O
from test_gpu_layer import GRAD_NAMES, check_grad
from test_gpu_xent import boundary_targets
from tensor_transformer_layer_tp_b200 import binding as B
from tensor_transformer_layer_tp_b200.runner import RankRunner, RankXentRunner
from tp_inputs import (LayerDims, XentDims, assemble_layer_grads, make_layer_inputs, make_xent_inputs,
                       partition_layer_params, partition_vocab)

pytestmark = pytest.mark.gpu

REPLICATED = ("ln1_g", "ln1_b", "b_o", "ln2_g", "ln2_b", "b_fc2")
PARTITIONED = ("w_qkv", "b_qkv", "w_o", "w_fc1", "b_fc1", "w_fc2")
SEED = 0x0DD5_EED5_0000_7777


def rank_params(parts: dict, rank: int) -> dict:
    out = {k: parts[k].cuda().contiguous() for k in REPLICATED}
    for k in PARTITIONED:
        out[k] = [parts[k][rank].cuda().contiguous()]
    return out


def emulated_all_reduce(runners):
    """Sum the ranks' partials (fp32 accumulation, bf16 result) into each."""
    torch.cuda.synchronize()
    total = torch.zeros_like(runners[0].partial, dtype=torch.float32)
    for r in runners:
        total += r.partial.float()
    for r in runners:
        r.partial.copy_(total)


def run_ranks(d: LayerDims, inp, p_attn=0.0, p_hidden=0.0):
    dims = B.make_dims(d.t, d.batch, d.seq, d.hidden, d.heads, d.ffn, d.causal, d.ln_eps,
                       dropout_attn=p_attn, dropout_hidden=p_hidden, seed=SEED)
    parts = partition_layer_params(inp, d.t, d.heads)
    runners = [RankRunner(dims, r, rank_params(parts, r)) for r in range(d.t)]
    x, dy = inp["x"].cuda(), inp["dy"].cuda()
    vl = inp["valid_len"].cuda() if "valid_len" in inp else None
    for seg in range(3):
        if seg:
            emulated_all_reduce(runners)
        for r in runners:
            r.forward_segment(seg, x, vl)
    for seg in range(3):
        if seg:
            emulated_all_reduce(runners)
        for r in runners:
            r.backward_segment(seg, x, dy, vl)
    torch.cuda.synchronize()
    B.tp_device_status()
    return runners


def oracle(d: LayerDims, inp, drop=None):
    p = O.to_f64({k: inp[k] for k in GRAD_NAMES})
    vl = inp["valid_len"].numpy() if "valid_len" in inp else None
    y, cache = O.layer_forward(f64(inp["x"]), p, d.heads, d.causal, vl, d.ln_eps, drop=drop)
    dx, gr = O.layer_backward(f64(inp["dy"]), cache, p, d.heads, d.causal, vl, drop=drop)
    return y, dx, gr


def check(runners, d, y, dx, gr):
    for r in runners:
        assert_close(f"y (rank {r.rank})", r.y, y)
        assert_close(f"dx (rank {r.rank})", r.dx, dx)
    g = {k: runners[0].grads[k] for k in REPLICATED}
    for k in PARTITIONED:
        g[k] = [r.grads[k][0] for r in runners]
    full = assemble_layer_grads(g, d.t)
    for k in GRAD_NAMES:
        check_grad(k, full[k], gr, d.seq)
    for k in REPLICATED:
        for r in runners[1:]:
            assert torch.allclose(r.grads[k].float(), g[k].float(), rtol=0, atol=1e-2 * float(
                g[k].float().abs().max()) + 1e-6), f"replicated gradient {k} differs between ranks"


CASES = {
    "causal t2": LayerDims(batch=2, seq=128, hidden=512, heads=8, ffn=2048, t=2),
    "causal t4 head_dim 96 ragged": LayerDims(batch=1, seq=200, hidden=384, heads=4, ffn=1536, t=4),
    "bert padding t2 head_dim 128": LayerDims(batch=3, seq=160, hidden=256, heads=2, ffn=1024, t=2,
                                              causal=False, padding=0.5),
    "t8": LayerDims(batch=2, seq=96, hidden=512, heads=8, ffn=2048, t=8),
}


@pytest.mark.parametrize("name", list(CASES))
def test_rank_local_layer_matches_oracle(name):
    d = CASES[name]
    inp = make_layer_inputs(d, seed=4)
    check(run_ranks(d, inp), d, *oracle(d, inp))


@pytest.mark.parametrize("name", ["causal t2", "causal t4 head_dim 96 ragged"])
def test_rank_local_dropout_draws_the_one_device_masks(name):
    d = CASES[name]
    inp = make_layer_inputs(d, seed=5)
    drop = O.Dropout(seed=SEED, p_attn=0.1, p_hidden=0.1)
    check(run_ranks(d, inp, p_attn=0.1, p_hidden=0.1), d, *oracle(d, inp, drop))


def test_rank_local_argument_errors():
    d = CASES["causal t2"]
    dims = B.make_dims(d.t, d.batch, d.seq, d.hidden, d.heads, d.ffn)
    inp = make_layer_inputs(d, seed=6)
    r = RankRunner(dims, 0, rank_params(partition_layer_params(inp, d.t, d.heads), 0))
    x = inp["x"].cuda()
    with pytest.raises(B.TPError):
        B.tp_layer_rank_forward(dims, 2, 0, r.params, x, None, r.partial, r.y, r.saved)   # rank >= t
    with pytest.raises(B.TPError):
        B.tp_layer_rank_forward(dims, 0, 3, r.params, x, None, r.partial, r.y, r.saved)   # segment
    with pytest.raises(B.TPError):
        B.tp_layer_rank_forward(dims, 0, 0, r.params, x, None, r.partial, r.y, r.saved[:16])  # short
    rec = B.make_dims(d.t, d.batch, d.seq, d.hidden, d.heads, d.ffn, recompute=True)
    assert B.tp_layer_rank_saved_bytes(rec) == 0   # recompute is not offered rank-locally


# ---------------------------------------------------------------- the loss across devices

def run_xent_ranks(d: XentDims, inp, with_grad=True):
    """Every vocab partition's loss segments on the one GPU, one rank after
    another, the ranks' statistics reduced on the host between segments."""
    x, tgt = inp["x"].cuda(), inp["target"].cuda()
    emb = [e.cuda() for e in partition_vocab(inp["emb"], d.t)]
    rs = [RankXentRunner(d.t, r, d.tokens, d.hidden, d.vocab, with_grad=with_grad) for r in range(d.t)]
    for r in rs:
        r.segment(0, x, emb[r.rank], tgt)
    torch.cuda.synchronize()
    big = torch.stack([r.comm[0] for r in rs]).amax(0)
    for r in rs:
        r.comm[0].copy_(big)
    for r in rs:
        r.segment(1, x, emb[r.rank], tgt)
    torch.cuda.synchronize()
    both = torch.stack([r.comm[1:3] for r in rs]).sum(0)
    for r in rs:
        r.comm[1:3].copy_(both)
    for r in rs:
        r.segment(2, x, emb[r.rank], tgt)
    torch.cuda.synchronize()
    dx = None
    if with_grad:
        dx = torch.stack([r.dx.float() for r in rs]).sum(0)
    B.tp_device_status()
    return rs, dx


@pytest.mark.parametrize("edges", [False, True])
@pytest.mark.parametrize("t", [2, 4, 8])
def test_rank_local_loss_matches_oracle(t, edges):
    # vocab 8 * 136: slice widths 544 / 272 / 136 are not multiples of the
    # 256-column statistics tile, and with edges every target sits on the first
    # or last row of a slice
    d = XentDims(tokens=300, hidden=256, vocab=8 * 136, t=t)
    inp = make_xent_inputs(d, seed=7)
    if edges:
        inp["target"] = boundary_targets(d.tokens, d.vocab, t)
    rs, dx = run_xent_ranks(d, inp)
    x64, e64, y = f64(inp["x"]), f64(inp["emb"]), inp["target"].numpy()
    loss, tok, lse = O.cross_entropy(x64, e64, y)
    dx64, de64 = O.cross_entropy_backward(x64, e64, y, lse)
    for r in rs:
        assert abs(r.loss.item() - loss) <= LOSS_RTOL * abs(loss), (r.rank, r.loss.item(), loss)
        assert_close(f"loss per token (rank {r.rank})", r.loss_tok, tok, tol=1e-4)
    assert_close("dX (sum of the ranks' terms)", dx, dx64)
    assert_close("dE (the ranks' slices)", torch.cat([r.demb for r in rs]), de64)


def test_rank_local_loss_without_gradient():
    d = XentDims(tokens=128, hidden=64, vocab=8 * 136, t=4)
    inp = make_xent_inputs(d, seed=8)
    rs, _ = run_xent_ranks(d, inp, with_grad=False)
    loss, _, _ = O.cross_entropy(f64(inp["x"]), f64(inp["emb"]), inp["target"].numpy())
    for r in rs:
        assert abs(r.loss.item() - loss) <= LOSS_RTOL * abs(loss)
