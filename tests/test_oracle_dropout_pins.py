"""Pins for the oracle's dropout (CPU only), against things other than itself.

* the counter-based generator against the published known-answer vectors of
  Philox-4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
  easy as 1, 2, 3", SC 2011; the vectors distributed with that paper's
  Random123 library),
* the keep masks against the binomial law of their rate,
* the layer backward with dropout against central finite differences,
* the attention with dropout against a torch fp64 autograd composition,
* the partition identity with dropout: the masks are keyed by global
  coordinates, so splitting the layer t ways draws the same masks and gives
  the same result (Megatron-LM show notes: dropout is replicated on every
  partition),
* rate 0 reduces to the dropout-free layer,
* and a planted mistake (masks keyed by the partition-local head) fails a pin.
"""
import numpy as np
import pytest
import torch

from oracle import tp_oracle as O
from test_oracle_pins import LAYER_TINY, RNG, _expect_failure, _fd_check, _layer_args, rel

M = 0xFFFFFFFF


@pytest.mark.parametrize("counter,key,expected", [
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((M, M, M, M), (M, M), (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
])
def test_philox_known_answers(counter, key, expected):
    got = O.philox4x32(counter, key)
    assert tuple(int(w) for w in got) == expected


@pytest.mark.parametrize("p", [0.1, 0.5])
def test_keep_rate_is_binomial(p):
    rows, cols = 512, 1000
    keep = O.keep_mask(seed=0x1234_5678_9ABC, p=p, stream=1, rows=np.arange(rows), ncols=cols)
    n = rows * cols
    kept = keep.sum()
    sigma = np.sqrt(n * p * (1 - p))
    assert abs(kept - n * (1 - p)) <= 6 * sigma
    # different streams and seeds give different masks; rate 0 keeps everything
    other = O.keep_mask(0x1234_5678_9ABC, p, 2, np.arange(rows), cols)
    assert 0.3 * n * p < np.sum(keep != other)
    assert O.keep_mask(7, 0.0, 1, np.arange(4), 9).all()


def _drop():
    return O.Dropout(seed=0xDEAD_BEEF_0042, p_attn=0.2, p_hidden=0.3)


@pytest.mark.parametrize("causal,padded", [(True, False), (False, True)])
def test_layer_backward_with_dropout_finite_differences(causal, padded):
    c = LAYER_TINY
    args = _layer_args(c["b"], c["s"], c["h"], c["heads"], c["f"])
    valid = np.array([8, 5]) if padded else None
    dy = RNG.normal(0, 1, args["x"].shape)
    drop = _drop()

    def loss(a):
        y, _ = O.layer_forward(a["x"], a, c["heads"], causal, valid, drop=drop)
        return float(np.sum(y * dy))

    y, cache = O.layer_forward(args["x"], args, c["heads"], causal, valid, drop=drop)
    dx, gr = O.layer_backward(dy, cache, args, c["heads"], causal, valid, drop=drop)
    gr = dict(gr, x=dx)
    _fd_check(loss, args, gr, ["x"] + sorted(k for k in gr if k != "x"))


def test_attention_with_dropout_matches_torch_autograd():
    b, s, hh, d = 2, 7, 3, 4
    q, k, v = (RNG.normal(0, 1, (b, s, hh, d)) for _ in range(3))
    drop = O.Dropout(seed=99, p_attn=0.4)
    w = RNG.normal(0, 1, (b, s, hh, d))
    o, _ = O.attention(q, k, v, True, None, drop)
    dq, dk, dv = O.attention_backward(w, q, k, v, True, None, drop)
    T = [torch.from_numpy(a).requires_grad_() for a in (q, k, v)]
    scale = 1.0 / np.sqrt(d)
    mask = torch.tril(torch.ones(s, s, dtype=torch.bool))
    outs = []
    for bb in range(b):
        for j in range(hh):
            sc = (T[0][bb, :, j] @ T[1][bb, :, j].T) * scale
            pr = torch.softmax(sc.masked_fill(~mask, float("-inf")), dim=-1)
            keep = torch.from_numpy(O.attn_keep(drop, bb, j, hh, s))
            outs.append((pr * keep / (1 - drop.p_attn)) @ T[2][bb, :, j])
    ot = torch.stack(outs).reshape(b, hh, s, d).transpose(1, 2)
    assert rel(o, ot.detach().numpy()) < 1e-12
    ot.backward(torch.from_numpy(w))
    for got, t in zip((dq, dk, dv), T):
        assert rel(got, t.grad.numpy()) < 1e-11


@pytest.mark.parametrize("t", [1, 2, 4])
def test_partitioned_layer_with_dropout_equals_unpartitioned(t):
    b, s, h, heads, f = 2, 8, 64, 8, 256
    args = _layer_args(b, s, h, heads, f)
    drop = _drop()
    y, cache = O.layer_forward(args["x"], args, heads, True, drop=drop)
    assert rel(O.layer_forward_partitioned(args["x"], args, heads, t, True, drop=drop), y) < 1e-12
    dy = RNG.normal(0, 1, y.shape)
    dx, gr = O.layer_backward(dy, cache, args, heads, True, drop=drop)
    dxp, grp = O.layer_backward_partitioned(dy, args["x"], args, heads, t, True, drop=drop)
    assert rel(dxp, dx) < 1e-12
    for k in gr:
        assert np.max(np.abs(grp[k] - gr[k])) <= 1e-12 * max(1.0, np.max(np.abs(gr[k]))), k


def test_rate_zero_is_the_dropout_free_layer():
    c = LAYER_TINY
    args = _layer_args(c["b"], c["s"], c["h"], c["heads"], c["f"])
    y0, cache0 = O.layer_forward(args["x"], args, c["heads"], True)
    y1, cache1 = O.layer_forward(args["x"], args, c["heads"], True, drop=O.Dropout(seed=5))
    assert np.array_equal(y0, y1)
    dy = RNG.normal(0, 1, y0.shape)
    dx0, g0 = O.layer_backward(dy, cache0, args, c["heads"], True)
    dx1, g1 = O.layer_backward(dy, cache1, args, c["heads"], True, drop=O.Dropout(seed=5))
    assert np.array_equal(dx0, dx1) and all(np.array_equal(g0[k], g1[k]) for k in g0)


def test_dropout_changes_the_output():
    c = LAYER_TINY
    args = _layer_args(c["b"], c["s"], c["h"], c["heads"], c["f"])
    y0, _ = O.layer_forward(args["x"], args, c["heads"], True)
    y1, _ = O.layer_forward(args["x"], args, c["heads"], True, drop=_drop())
    assert rel(y1, y0) > 1e-2


def test_planted_local_head_keying_is_caught(monkeypatch):
    # keying the attention masks by the partition-local head makes the mask
    # depend on t: the partition identity must fail
    orig = O.attention

    def local_keyed(q, k, v, causal, valid_len=None, drop=None, head0=0, heads_total=None):
        return orig(q, k, v, causal, valid_len, drop, 0, heads_total)
    monkeypatch.setattr(O, "attention", local_keyed)
    _expect_failure(lambda: test_partitioned_layer_with_dropout_equals_unpartitioned(2))
