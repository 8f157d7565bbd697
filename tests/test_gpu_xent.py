"""Vocab-parallel cross-entropy through the C-ABI vs the fp64 oracle.

Loss: relative error <= 1e-5.  dx, dE: max|err| <= 2e-2 * max|ref|.
Small ragged cases here; the full 8192 x 1024 x 50304 workload is in
test_gpu_fullsize.py.
"""
import math

import numpy as np
import pytest
import torch

from helpers import LOSS_RTOL, assert_close, f64
from oracle import tp_oracle as O
from tensor_transformer_layer_tp_b200.runner import XentRunner
from tp_inputs import XentDims, make_xent_inputs, partition_vocab

pytestmark = pytest.mark.gpu


def run_gpu(d: XentDims, inp, with_grad=True, explicit=False):
    r = XentRunner(d.t, d.tokens, d.hidden, d.vocab, with_grad=with_grad, explicit=explicit)
    x = inp["x"].cuda()
    emb = [e.cuda() for e in partition_vocab(inp["emb"], d.t)]
    tgt = inp["target"].cuda()
    r(x, emb, tgt)
    torch.cuda.synchronize()
    return r


PATHS = {"fused": False, "explicit": True}


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("t", [1, 2, 4, 8])
@pytest.mark.parametrize("tokens,hidden,vocab", [(300, 256, 2048), (128, 64, 8 * 136),
                                                 (520, 128, 8 * 312)])
def test_xent_matches_oracle(t, tokens, hidden, vocab, path):
    # 520 tokens: ragged over the 256-row CTA-pair tiles; 8 x 312 vocabulary:
    # partition widths 1248 .. 312 end inside a 256-column tile
    d = XentDims(tokens=tokens, hidden=hidden, vocab=vocab, t=t)
    inp = make_xent_inputs(d, seed=3)
    r = run_gpu(d, inp, explicit=PATHS[path])
    x, e, y = f64(inp["x"]), f64(inp["emb"]), inp["target"].numpy()
    loss, tok, lse = O.cross_entropy(x, e, y)
    assert abs(r.loss.item() - loss) <= LOSS_RTOL * abs(loss)
    assert_close("loss_per_token", r.loss_tok, tok, tol=1e-5)
    dx, de = O.cross_entropy_backward(x, e, y, lse)
    assert_close("dx", r.dx, dx)
    assert_close("demb", torch.cat([g.cpu() for g in r.demb], 0), de)


@pytest.mark.parametrize("path", list(PATHS))
def test_xent_zero_input_gives_log_vocab(path):
    # every logit is 0: loss = ln V, dE = 0 (closed form)
    d = XentDims(tokens=256, hidden=128, vocab=4096, t=4)
    inp = make_xent_inputs(d, seed=4)
    inp["x"] = torch.zeros_like(inp["x"])
    r = run_gpu(d, inp, explicit=PATHS[path])
    assert abs(r.loss.item() - math.log(d.vocab)) <= LOSS_RTOL * math.log(d.vocab)
    for g in r.demb:
        assert torch.count_nonzero(g).item() == 0


@pytest.mark.parametrize("path", list(PATHS))
def test_xent_forward_only_and_split_invariance(path):
    # the same data split t = 1 and t = 8 ways gives the same loss, forward only
    d1 = XentDims(512, 256, 8192, 1)
    inp = make_xent_inputs(d1, seed=6)
    losses = []
    for t in (1, 8):
        r = run_gpu(XentDims(512, 256, 8192, t), inp, with_grad=False, explicit=PATHS[path])
        losses.append(r.loss.item())
    assert abs(losses[0] - losses[1]) <= 1e-6 * abs(losses[0])
    loss, _, _ = O.cross_entropy(f64(inp["x"]), f64(inp["emb"]), inp["target"].numpy())
    assert abs(losses[0] - loss) <= LOSS_RTOL * abs(loss)


def test_fused_and_explicit_paths_agree():
    # the two realisations of the same loss, on one workload: fp32-accurate
    # losses agree closely; gradients within the bf16 tolerance
    d = XentDims(tokens=700, hidden=256, vocab=8 * 520, t=8)
    inp = make_xent_inputs(d, seed=11)
    a, b = run_gpu(d, inp), run_gpu(d, inp, explicit=True)
    assert abs(a.loss.item() - b.loss.item()) <= LOSS_RTOL * abs(b.loss.item())
    assert_close("loss_per_token", a.loss_tok, b.loss_tok, tol=LOSS_RTOL)
    assert_close("dx", a.dx, b.dx)
    for i in range(d.t):
        assert_close(f"demb[{i}]", a.demb[i], b.demb[i])


def boundary_targets(tokens: int, vocab: int, t: int) -> torch.Tensor:
    """Targets on every partition edge: the first and last vocabulary row of
    each partition (i*V/t and i*V/t - 1 for every i, 0 and V - 1), cycled over
    the tokens.  These are the rows where the owning partition changes, so a
    wrong offset of the target into a partition's slice picks the neighbour's
    logit or none."""
    vp = vocab // t
    edges = sorted({0, vocab - 1} | {i * vp for i in range(1, t)} | {i * vp - 1 for i in range(1, t)})
    return torch.tensor([edges[n % len(edges)] for n in range(tokens)], dtype=torch.int32)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("t", [2, 4, 8])
def test_xent_targets_on_partition_edges(t, path):
    # vocab 8 * 136: partition widths 544 / 272 / 136 are not multiples of the
    # GEMM tile, so every edge also falls inside a tile
    d = XentDims(tokens=200, hidden=256, vocab=8 * 136, t=t)
    inp = make_xent_inputs(d, seed=9)
    inp["target"] = boundary_targets(d.tokens, d.vocab, t)
    r = run_gpu(d, inp, explicit=PATHS[path])
    x, e, y = f64(inp["x"]), f64(inp["emb"]), inp["target"].numpy()
    loss, tok, lse = O.cross_entropy(x, e, y)
    assert abs(r.loss.item() - loss) <= LOSS_RTOL * abs(loss)
    assert_close("loss_per_token", r.loss_tok, tok, tol=LOSS_RTOL)
    dx, de = O.cross_entropy_backward(x, e, y, lse)
    assert_close("dx", r.dx, dx)
    assert_close("demb", torch.cat([g.cpu() for g in r.demb], 0), de)
