"""Pins for the oracle's vocab-parallel input embedding and the tied-embedding
layer stack (CPU only).

* the split input embedding (rkmt.cn guide, section 3.3: the input layer is
  split along the vocabulary and its outputs are summed by an all-reduce)
  equals the plain lookup for t = 1, 2, 4, 8, with ids on every partition edge,
* the embedding backward against torch's embedding and autograd,
* the whole stack (embedding, layers, tied output embedding, loss) against a
  torch fp64 autograd composition of library primitives, and its gradient with
  respect to the shared embedding against central finite differences: a
  dropped input or output half of the tied gradient fails both,
* a planted mistake (the input half of the tied gradient left out) fails.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import tp_oracle as O
from test_oracle_pins import RNG, _expect_failure, rel, tiny_params


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_vocab_parallel_embedding_equals_lookup(t):
    v, h = 64, 16
    emb = RNG.normal(0, 1, (v, h))
    vs = v // t
    edges = sorted({0, v - 1} | {i * vs for i in range(1, t)} | {i * vs - 1 for i in range(1, t)})
    ids = np.concatenate([np.array(edges), RNG.integers(0, v, 50)])
    out = O.vocab_parallel_embedding(ids, emb, t)
    assert np.array_equal(out, O.embedding(ids, emb))
    assert np.array_equal(out, F.embedding(torch.from_numpy(ids), torch.from_numpy(emb)).numpy())


def test_embedding_backward_matches_torch():
    v, h, n = 40, 8, 300           # many repeated ids
    emb = RNG.normal(0, 1, (v, h))
    ids = RNG.integers(0, v, n)
    dout = RNG.normal(0, 1, (n, h))
    et = torch.from_numpy(emb).requires_grad_()
    F.embedding(torch.from_numpy(ids), et).backward(torch.from_numpy(dout))
    assert rel(O.embedding_backward(ids, dout, v), et.grad.numpy()) < 1e-12


def _stack_case(layers=2):
    b, s, h, heads, f, v = 2, 6, 16, 2, 64, 24
    emb = RNG.normal(0, 0.5, (v, h))
    params = [tiny_params(h, f) for _ in range(layers)]
    ids = RNG.integers(0, v, (b, s))
    targets = RNG.integers(0, v, (b, s))
    return ids, targets, emb, params, heads


def test_stack_matches_torch_autograd():
    ids, targets, emb, params, heads = _stack_case()
    loss, de, grads = O.stack_forward_backward(ids, targets, emb, params, heads)
    b, s = ids.shape
    h = emb.shape[1]
    E = torch.from_numpy(emb).requires_grad_()
    P = [{k: torch.from_numpy(v).requires_grad_() for k, v in p.items()} for p in params]
    x = F.embedding(torch.from_numpy(ids), E)
    split = lambda a: a.view(b, s, heads, h // heads).transpose(1, 2)
    for T in P:
        xn1 = F.layer_norm(x, (h,), T["ln1_g"], T["ln1_b"], 1e-5)
        q, k, v = (split(F.linear(xn1, T["w_" + n].T, T["b_" + n])) for n in "qkv")
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(b, s, h)
        h1 = x + F.linear(o, T["w_o"].T, T["b_o"])
        xn2 = F.layer_norm(h1, (h,), T["ln2_g"], T["ln2_b"], 1e-5)
        x = h1 + F.linear(F.gelu(F.linear(xn2, T["w_fc1"].T, T["b_fc1"])), T["w_fc2"].T, T["b_fc2"])
    lt = F.cross_entropy(x.reshape(b * s, h) @ E.T, torch.from_numpy(targets.reshape(-1)))
    lt.backward()
    assert abs(loss - lt.item()) <= 1e-12 * abs(loss)
    assert rel(de, E.grad.numpy()) < 1e-10
    for g, T in zip(grads, P):
        for name in g:
            ref = T[name].grad.numpy()
            assert np.max(np.abs(g[name] - ref)) <= 1e-10 * max(1.0, np.max(np.abs(ref))), name


def test_stack_tied_gradient_finite_differences():
    ids, targets, emb, params, heads = _stack_case(layers=1)
    _, de, _ = O.stack_forward_backward(ids, targets, emb, params, heads)
    eps = 1e-6
    for _ in range(3):
        vdir = RNG.normal(0, 1, emb.shape)
        lp = O.stack_forward_backward(ids, targets, emb + eps * vdir, params, heads)[0]
        lm = O.stack_forward_backward(ids, targets, emb - eps * vdir, params, heads)[0]
        fd = (lp - lm) / (2 * eps)
        an = float(np.sum(de * vdir))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (fd, an)


def test_planted_missing_input_half_is_caught(monkeypatch):
    monkeypatch.setattr(O, "embedding_backward", lambda ids, dout, vocab: np.zeros((vocab, dout.shape[1])))
    _expect_failure(test_stack_tied_gradient_finite_differences)
