"""Pins for the fp64 oracle, against things other than itself.

* library routines (torch fp64 CPU: layer_norm, gelu, scaled_dot_product_attention,
  cross_entropy, autograd),
* closed forms and special cases (s=1 attention, zero queries, zero logits),
* central finite differences for every backward,
* the partition identities the pages rest on: column split + per-partition GeLU +
  row split + sum equals the unpartitioned MLP; per-head attention split; the
  vocab-split loss with a combined (max, sum-exp, target) triple equals the
  closed-form log-sum-exp (Megatron-LM show notes, outline items on the MLP and
  self-attention split, the 4 all-reduces per layer and the output embedding;
  rkmt.cn guide, sections 3.1-3.3).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import tp_oracle as O

RNG = np.random.default_rng(1234)


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def tiny_params(h, f, rng=RNG):
    p = {}
    for n, shp in dict(w_q=(h, h), w_k=(h, h), w_v=(h, h), w_o=(h, h), w_fc1=(h, f),
                       w_fc2=(f, h)).items():
        p[n] = rng.normal(0, 0.3, shp)
    for n, shp in dict(b_q=h, b_k=h, b_v=h, b_o=h, b_fc1=f, b_fc2=h, ln1_b=h, ln2_b=h).items():
        p[n] = rng.normal(0, 0.1, shp)
    p["ln1_g"] = 1 + rng.normal(0, 0.1, h)
    p["ln2_g"] = 1 + rng.normal(0, 0.1, h)
    return p


# ------------------------------------------------------------ primitives vs library

def test_layer_norm_matches_torch():
    x = RNG.normal(0, 2, (3, 5, 48)) + 0.7
    g, b = RNG.normal(1, 0.2, 48), RNG.normal(0, 0.2, 48)
    y, (mu, rstd) = O.layer_norm(x, g, b, 1e-5)
    ref = F.layer_norm(torch.from_numpy(x), (48,), torch.from_numpy(g), torch.from_numpy(b), 1e-5)
    assert rel(y, ref.numpy()) < 1e-13
    dy = RNG.normal(0, 1, x.shape)
    dx, dg, db = O.layer_norm_backward(dy, x, g, mu, rstd)
    xt, gt, bt = (torch.from_numpy(a).requires_grad_() for a in (x, g, b))
    F.layer_norm(xt, (48,), gt, bt, 1e-5).backward(torch.from_numpy(dy))
    assert rel(dx, xt.grad.numpy()) < 1e-12
    assert rel(dg, gt.grad.numpy()) < 1e-12
    assert rel(db, bt.grad.numpy()) < 1e-12


def test_gelu_matches_torch_exact_form():
    u = np.linspace(-8, 8, 2001)
    ut = torch.from_numpy(u).requires_grad_()
    ref = F.gelu(ut, approximate="none")
    assert rel(O.gelu(u), ref.detach().numpy()) < 1e-14
    ref.sum().backward()
    assert rel(O.gelu_grad(u), ut.grad.numpy()) < 1e-13
    # closed forms: gelu(0) = 0, gelu(x) - gelu(-x) = x, gelu'(0) = 1/2
    assert O.gelu(np.array(0.0)) == 0.0
    assert rel(O.gelu(u) - O.gelu(-u), u) < 1e-14
    assert abs(O.gelu_grad(np.array(0.0)) - 0.5) < 1e-15


def _sdpa(q, k, v, mask):
    # torch layout [B, H, s, d]
    qt, kt, vt = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask).permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("causal,padded", [(True, False), (False, True), (False, False)])
def test_attention_matches_sdpa(causal, padded):
    b, s, hh, d = 2, 9, 3, 8
    q, k, v = (RNG.normal(0, 1, (b, s, hh, d)) for _ in range(3))
    valid = np.array([9, 6]) if padded else None
    o, lse = O.attention(q, k, v, causal, valid)
    # reference mask built independently of the oracle: torch.tril for causal, key < valid_len for padding
    mask = torch.ones(b, 1, s, s, dtype=torch.bool)
    if causal:
        mask &= torch.tril(torch.ones(s, s, dtype=torch.bool))
    if valid is not None:
        mask &= (torch.arange(s)[None, :] < torch.from_numpy(valid)[:, None])[:, None, None, :]
    assert rel(o, _sdpa(q, k, v, mask)) < 1e-13
    scores = torch.einsum("bqhd,bkhd->bhqk", torch.from_numpy(q), torch.from_numpy(k)) / math.sqrt(d)
    scores = scores.masked_fill(~mask, float("-inf"))
    assert rel(lse, torch.logsumexp(scores, -1).numpy()) < 1e-13


def test_attention_special_cases():
    # s = 1: the only key is the query itself, so O = V
    q, k, v = (RNG.normal(0, 1, (2, 1, 2, 8)) for _ in range(3))
    o, lse = O.attention(q, k, v, causal=True)
    assert rel(o, v) < 1e-15
    # Q = 0: uniform weights over allowed keys -> running mean of V (causal), lse = log(#keys)
    s = 7
    q0 = np.zeros((1, s, 1, 4))
    k, v = RNG.normal(0, 1, (1, s, 1, 4)), RNG.normal(0, 1, (1, s, 1, 4))
    o, lse = O.attention(q0, k, v, causal=True)
    run_mean = np.cumsum(v[0, :, 0, :], axis=0) / np.arange(1, s + 1)[:, None]
    assert rel(o[0, :, 0, :], run_mean) < 1e-14
    assert rel(lse[0, 0], np.log(np.arange(1, s + 1))) < 1e-14
    # key padding with Q = 0: mean of the first valid_len values for every query
    o, _ = O.attention(q0, k, v, causal=False, valid_len=np.array([4]))
    assert rel(o[0, :, 0, :], np.broadcast_to(v[0, :4, 0, :].mean(0), (s, 4))) < 1e-14


def _fd_check(fn, args, grads, names, eps=1e-6, tol=1e-6, rng=RNG):
    """Directional central differences: (L(a+e v) - L(a-e v)) / 2e == <grad, v>."""
    for nm in names:
        vdir = rng.normal(0, 1, np.shape(args[nm]))
        plus = dict(args); plus[nm] = args[nm] + eps * vdir
        minus = dict(args); minus[nm] = args[nm] - eps * vdir
        fd = (fn(plus) - fn(minus)) / (2 * eps)
        an = float(np.sum(grads[nm] * vdir))
        assert abs(fd - an) <= tol * max(1.0, abs(an)), (nm, fd, an)


@pytest.mark.parametrize("causal,padded", [(True, False), (False, True)])
def test_attention_backward_finite_differences(causal, padded):
    b, s, hh, d = 2, 6, 2, 4
    args = {n: RNG.normal(0, 1, (b, s, hh, d)) for n in ("q", "k", "v")}
    valid = np.array([6, 4]) if padded else None
    w = RNG.normal(0, 1, (b, s, hh, d))
    fn = lambda a: float(np.sum(O.attention(a["q"], a["k"], a["v"], causal, valid)[0] * w))
    dq, dk, dv = O.attention_backward(w, args["q"], args["k"], args["v"], causal, valid)
    _fd_check(fn, args, {"q": dq, "k": dk, "v": dv}, ("q", "k", "v"))


# ------------------------------------------------------------ loss

def test_cross_entropy_matches_torch_and_closed_forms():
    n, h, v = 11, 16, 40
    x, e = RNG.normal(0, 1, (n, h)), RNG.normal(0, 0.5, (v, h))
    y = RNG.integers(0, v, n)
    loss, tok, lse = O.cross_entropy(x, e, y)
    z = torch.from_numpy(x) @ torch.from_numpy(e).T
    assert abs(loss - F.cross_entropy(z, torch.from_numpy(y)).item()) < 1e-13
    assert rel(tok, F.cross_entropy(z, torch.from_numpy(y), reduction="none").numpy()) < 1e-13
    # zero input: every logit is 0, loss = ln V exactly; gradient rows = (1/V - onehot)/n
    loss0, _, lse0 = O.cross_entropy(np.zeros((n, h)), e, y)
    assert abs(loss0 - math.log(v)) < 1e-13
    dx, de = O.cross_entropy_backward(np.zeros((n, h)), e, y, lse0)
    dz = np.full((n, v), 1.0 / v)
    dz[np.arange(n), y] -= 1
    assert rel(dx, (dz / n) @ e) < 1e-13
    assert np.max(np.abs(de)) == 0.0     # x = 0 => dE = dz^T x = 0


def test_cross_entropy_backward_matches_torch_and_fd():
    n, h, v = 9, 12, 30
    x, e = RNG.normal(0, 1, (n, h)), RNG.normal(0, 0.5, (v, h))
    y = RNG.integers(0, v, n)
    loss, tok, lse = O.cross_entropy(x, e, y)
    dx, de = O.cross_entropy_backward(x, e, y, lse)
    xt, et = torch.from_numpy(x).requires_grad_(), torch.from_numpy(e).requires_grad_()
    F.cross_entropy(xt @ et.T, torch.from_numpy(y)).backward()
    assert rel(dx, xt.grad.numpy()) < 1e-12 and rel(de, et.grad.numpy()) < 1e-12
    fn = lambda a: float(O.cross_entropy(a["x"], a["e"], y)[0])
    _fd_check(fn, {"x": x, "e": e}, {"x": dx, "e": de}, ("x", "e"))


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_vocab_parallel_loss_equals_logsumexp(t):
    n, h, v = 33, 16, 64
    x, e = RNG.normal(0, 2, (n, h)), RNG.normal(0, 1, (v, h))
    y = RNG.integers(0, v, n)
    loss, tok, lse = O.vocab_parallel_cross_entropy(x, e, y, t)
    z = x @ e.T
    m = z.max(1)
    closed = m + np.log(np.exp(z - m[:, None]).sum(1))          # log-sum-exp written out
    assert rel(lse, closed) < 1e-13
    assert rel(tok, closed - z[np.arange(n), y]) < 1e-13
    loss_u, tok_u, _ = O.cross_entropy(x, e, y)
    assert abs(loss - loss_u) <= 1e-13 * abs(loss_u)


@pytest.mark.parametrize("t", [2, 4, 8])
def test_vocab_parallel_loss_targets_on_partition_edges(t):
    # every target on a partition's first or last row (i*V/t, i*V/t - 1, 0, V-1):
    # the split loss still equals the log-sum-exp closed form row by row
    n, h, v = 40, 16, 64
    vs = v // t
    edges = sorted({0, v - 1} | {i * vs for i in range(1, t)} | {i * vs - 1 for i in range(1, t)})
    x, e = RNG.normal(0, 2, (n, h)), RNG.normal(0, 1, (v, h))
    y = np.array([edges[k % len(edges)] for k in range(n)])
    _, tok, lse = O.vocab_parallel_cross_entropy(x, e, y, t)
    z = x @ e.T
    m = z.max(1)
    closed = m + np.log(np.exp(z - m[:, None]).sum(1))
    assert rel(tok, closed - z[np.arange(n), y]) < 1e-13


# ------------------------------------------------------------ the layer

LAYER_TINY = dict(b=2, s=8, h=32, heads=4, f=128)


def _layer_args(b, s, h, heads, f):
    p = tiny_params(h, f)
    p["x"] = RNG.normal(0, 1, (b, s, h))
    return p


@pytest.mark.parametrize("causal,padded", [(True, False), (False, True)])
def test_layer_backward_finite_differences(causal, padded):
    c = LAYER_TINY
    args = _layer_args(c["b"], c["s"], c["h"], c["heads"], c["f"])
    valid = np.array([8, 5]) if padded else None
    dy = RNG.normal(0, 1, args["x"].shape)

    def loss(a):
        y, _ = O.layer_forward(a["x"], a, c["heads"], causal, valid)
        return float(np.sum(y * dy))

    y, cache = O.layer_forward(args["x"], args, c["heads"], causal, valid)
    dx, gr = O.layer_backward(dy, cache, args, c["heads"], causal, valid)
    gr = dict(gr, x=dx)
    _fd_check(loss, args, gr, ["x"] + sorted(k for k in gr if k != "x"))


def test_layer_matches_torch_autograd_composition():
    """Cross-check against torch fp64 library primitives + autograd (layout of heads, bias placement)."""
    c = LAYER_TINY
    args = _layer_args(c["b"], c["s"], c["h"], c["heads"], c["f"])
    dy = RNG.normal(0, 1, args["x"].shape)
    y, cache = O.layer_forward(args["x"], args, c["heads"], True)
    dx, gr = O.layer_backward(dy, cache, args, c["heads"], True)
    T = {k: torch.from_numpy(v).requires_grad_() for k, v in args.items()}
    b, s, h, hh = c["b"], c["s"], c["h"], c["heads"]
    xn1 = F.layer_norm(T["x"], (h,), T["ln1_g"], T["ln1_b"], 1e-5)
    heads = lambda a: a.view(b, s, hh, h // hh).transpose(1, 2)
    q, k, v = (heads(F.linear(xn1, T["w_" + n].T, T["b_" + n])) for n in "qkv")
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(b, s, h)
    h1 = T["x"] + F.linear(o, T["w_o"].T, T["b_o"])
    xn2 = F.layer_norm(h1, (h,), T["ln2_g"], T["ln2_b"], 1e-5)
    yt = h1 + F.linear(F.gelu(F.linear(xn2, T["w_fc1"].T, T["b_fc1"])), T["w_fc2"].T, T["b_fc2"])
    assert rel(y, yt.detach().numpy()) < 1e-12
    yt.backward(torch.from_numpy(dy))
    assert rel(dx, T["x"].grad.numpy()) < 1e-11
    for name, g in gr.items():
        ref = T[name].grad.numpy()
        assert np.max(np.abs(g - ref)) <= 1e-11 * max(1.0, np.max(np.abs(ref))), name
    # closed form: a key bias shifts every score of a query row by the same q.b_k,
    # which softmax ignores, so its gradient is zero
    assert np.max(np.abs(gr["b_k"])) < 1e-12


@pytest.mark.parametrize("t", [1, 2, 4, 8])
@pytest.mark.parametrize("causal,padded", [(True, False), (False, True)])
def test_partitioned_layer_equals_unpartitioned(t, causal, padded):
    b, s, h, heads, f = 2, 8, 64, 8, 256
    args = _layer_args(b, s, h, heads, f)
    valid = np.array([8, 6]) if padded else None
    y, cache = O.layer_forward(args["x"], args, heads, causal, valid)
    yp = O.layer_forward_partitioned(args["x"], args, heads, t, causal, valid)
    assert rel(yp, y) < 1e-12
    dy = RNG.normal(0, 1, y.shape)
    dx, gr = O.layer_backward(dy, cache, args, heads, causal, valid)
    dxp, grp = O.layer_backward_partitioned(dy, args["x"], args, heads, t, causal, valid)
    assert rel(dxp, dx) < 1e-12
    assert set(grp) == set(gr)
    for k in gr:
        # b_k's gradient is exactly zero (softmax shift invariance): compare on a floor of 1
        assert np.max(np.abs(grp[k] - gr[k])) <= 1e-12 * max(1.0, np.max(np.abs(gr[k]))), k


# ------------------------------------------------------------ the pins have teeth

def _expect_failure(fn):
    with pytest.raises(AssertionError):
        fn()


def test_planted_mistakes_are_caught(monkeypatch):
    """Plant plausible mistakes in the oracle (CPU only) and check a pin fails for each."""
    # wrong sign inside the GeLU derivative
    monkeypatch.setattr(O, "gelu_grad", lambda u: 0.5 * (1 + O.erf(u / O.SQRT2)) - u * O.INV_SQRT_2PI * np.exp(-0.5 * u * u))
    _expect_failure(lambda: test_layer_backward_finite_differences(True, False))
    monkeypatch.undo()
    # dropped mean term in the LayerNorm backward
    orig_lnb = O.layer_norm_backward

    def lnb_drop(dy, x, gamma, mu, rstd):
        dx, dg, db = orig_lnb(dy, x, gamma, mu, rstd)
        return dx + rstd[..., None] * (dy * gamma).sum(-1, keepdims=True) / x.shape[-1], dg, db
    monkeypatch.setattr(O, "layer_norm_backward", lnb_drop)
    _expect_failure(test_layer_norm_matches_torch)
    monkeypatch.undo()
    # transposed key operand in attention (S = Q K instead of Q K^T on square heads)
    orig_attn = O.attention

    def attn_t(q, k, v, causal, valid_len=None):
        return orig_attn(q, np.swapaxes(k, 1, 3) if k.shape[1] == k.shape[3] else k[:, ::-1], v, causal, valid_len)
    monkeypatch.setattr(O, "attention", attn_t)
    _expect_failure(lambda: test_attention_matches_sdpa(True, False))
    monkeypatch.undo()
    # off-by-one causal mask (k < q instead of k <= q)
    monkeypatch.setattr(O, "attention_mask",
                        lambda s, c, vl: (np.arange(s)[None, :] < np.arange(s)[:, None]) | np.eye(s, k=1, dtype=bool)
                        if c else np.ones((s, s), bool))
    _expect_failure(lambda: test_attention_matches_sdpa(True, False))
    monkeypatch.undo()
    # row-split bias added once per partition instead of once
    orig_lfp = O.layer_forward_partitioned

    def lfp_bias(x, p, heads, t, causal, valid_len=None, eps=1e-5):
        return orig_lfp(x, p, heads, t, causal, valid_len, eps) + (t - 1) * p["b_fc2"]
    monkeypatch.setattr(O, "layer_forward_partitioned", lfp_bias)
    _expect_failure(lambda: test_partitioned_layer_equals_unpartitioned(2, True, False))
    monkeypatch.undo()
    # target logit taken from the wrong partition offset in the split loss
    orig_vp = O.vocab_parallel_cross_entropy

    def vp_bad(x, emb, target, t):
        return orig_vp(x, emb, (target + 1) % emb.shape[0], t)
    monkeypatch.setattr(O, "vocab_parallel_cross_entropy", vp_bad)
    _expect_failure(lambda: test_vocab_parallel_loss_equals_logsumexp(2))
    monkeypatch.undo()
