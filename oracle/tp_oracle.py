"""fp64 CPU oracle for the tensor-parallel transformer layer and the vocab-parallel loss.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this module.  The CUDA
library never calls it and shares no code with it.

What it computes
----------------
The plain, unpartitioned definition of one pre-LN transformer layer and of the
output-embedding cross-entropy, forward and backward, in float64 with no
intermediate rounding.  Megatron-LM's intra-layer model parallelism is an exact
re-association of these matmuls (Megatron-LM show notes, "intra-layer parallel
implementation" outline: MLP weight split, per-head Q/K/V split, 2 all-reduces
per module; rkmt.cn selection guide, section 3 "extreme splitting of the
Transformer layer"), so the definition below is what the partitioned method
must reach up to rounding.  ``*_partitioned`` functions walk the t partitions
explicitly (column split, per-partition GeLU, row split, explicit sum standing
for the all-reduce, per-partition max/sum-exp/target triple for the loss) and
exist only so tests can pin that equivalence.

Readings where the pages are silent (each also listed in the design notes):
  * GeLU is the exact form x*Phi(x) = x/2 * (1 + erf(x/sqrt 2)).
  * LayerNorm: biased variance over the hidden dimension, eps = 1e-5, affine.
  * The layer is pre-LN (the BERT re-ordering the show notes describe) for
    both GPT and BERT workloads:  H1 = X + Attn(LN1(X)),  Y = H1 + MLP(LN2(H1)).
  * All four linears carry a bias; row-split biases are added once after the sum.
  * Attention scale 1/sqrt(d).  Causal: key k <= query q.  Key padding:
    keys at positions >= valid_len[b] are excluded; padded queries are kept.
  * Dropout is off unless a ``Dropout`` is passed.  When on, it sits where
    Megatron-LM puts it: on the attention probabilities (inside the heads of
    each partition) and on the two replicated hidden outputs, after the
    out-projection and after FC2 (before each residual add); the show notes
    say only that dropout is replicated on every partition.  Masks come from a
    counter-based generator (Philox-4x32-10) keyed by the seed and by each
    element's global coordinates, so every partition count t draws the same
    mask (see ``keep_mask``).  Kept values are scaled by 1/(1-p).
  * Loss = mean over all tokens of logsumexp(z) - z[target].

Parity pins: see tests/test_oracle_pins.py.  Every function here is pinned
(library routine, closed form, finite differences or partition identity).
"""
from __future__ import annotations

import dataclasses

import numpy as np
from scipy.special import erf

SQRT2 = np.sqrt(2.0)
INV_SQRT_2PI = 1.0 / np.sqrt(2.0 * np.pi)


# ---------------------------------------------------------------- primitives

def layer_norm(x, gamma, beta, eps):
    """y = (x - mean) / sqrt(var + eps) * gamma + beta over the last axis (biased var)."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (x - mu) * rstd
    return xhat * gamma + beta, (mu[..., 0], rstd[..., 0])


def layer_norm_backward(dy, x, gamma, mu, rstd):
    """Gradients of layer_norm w.r.t. x, gamma, beta (reduction over all leading axes)."""
    h = x.shape[-1]
    xhat = (x - mu[..., None]) * rstd[..., None]
    g = dy * gamma
    dx = rstd[..., None] * (g - g.sum(-1, keepdims=True) / h
                            - xhat * (g * xhat).sum(-1, keepdims=True) / h)
    lead = tuple(range(dy.ndim - 1))
    return dx, (dy * xhat).sum(axis=lead), dy.sum(axis=lead)


def gelu(u):
    """Exact GeLU: u * Phi(u)."""
    return 0.5 * u * (1.0 + erf(u / SQRT2))


def gelu_grad(u):
    """d/du [u * Phi(u)] = Phi(u) + u * phi(u)."""
    return 0.5 * (1.0 + erf(u / SQRT2)) + u * INV_SQRT_2PI * np.exp(-0.5 * u * u)


def attention_mask(seq, causal, valid_len_b):
    """Boolean [s, s] matrix of allowed (query, key) pairs for one sequence."""
    q = np.arange(seq)[:, None]
    k = np.arange(seq)[None, :]
    allowed = np.ones((seq, seq), dtype=bool)
    if causal:
        allowed &= k <= q
    if valid_len_b is not None:
        allowed &= k < valid_len_b
    return allowed


def attention(q, k, v, causal, valid_len=None, drop=None, head0=0, heads_total=None):
    """Per (batch, head) softmax attention.

    q, k, v: [B, s, H, d].  Returns O [B, s, H, d] and lse [B, H, s] where
    lse = log sum_k exp(S_qk) over allowed keys and S = q k^T / sqrt(d).
    With a Dropout, O = (P * keep / (1 - p_attn)) V; local head j is global
    head head0 + j of heads_total (partitions pass their first head).
    """
    b_, s_, hh, d = q.shape
    heads_total = hh if heads_total is None else heads_total
    scale = 1.0 / np.sqrt(d)
    o = np.empty_like(q)
    lse = np.empty((b_, hh, s_))
    for b in range(b_):
        allowed = attention_mask(s_, causal, None if valid_len is None else int(valid_len[b]))
        for j in range(hh):
            s = (q[b, :, j, :] @ k[b, :, j, :].T) * scale
            s = np.where(allowed, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            z = e.sum(axis=1, keepdims=True)
            pr = e / z
            keep = attn_keep(drop, b, head0 + j, heads_total, s_)
            if keep is not None:
                pr = pr * keep / (1.0 - drop.p_attn)
            o[b, :, j, :] = pr @ v[b, :, j, :]
            lse[b, j, :] = (m + np.log(z))[:, 0]
    return o, lse


def attention_backward(do, q, k, v, causal, valid_len=None, drop=None, head0=0, heads_total=None):
    """Gradients of attention() w.r.t. q, k, v (softmax Jacobian written out)."""
    b_, s_, hh, d = q.shape
    heads_total = hh if heads_total is None else heads_total
    scale = 1.0 / np.sqrt(d)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(b_):
        allowed = attention_mask(s_, causal, None if valid_len is None else int(valid_len[b]))
        for j in range(hh):
            qq, kk, vv, g = q[b, :, j, :], k[b, :, j, :], v[b, :, j, :], do[b, :, j, :]
            s = np.where(allowed, (qq @ kk.T) * scale, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            keep = attn_keep(drop, b, head0 + j, heads_total, s_)
            mult = 1.0 if keep is None else keep / (1.0 - drop.p_attn)
            dv[b, :, j, :] = (p * mult).T @ g        # O = (P * mult) V
            dp = (g @ vv.T) * mult                    # gradient w.r.t. P
            ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
            dq[b, :, j, :] = (ds @ kk) * scale
            dk[b, :, j, :] = (ds.T @ qq) * scale
    return dq, dk, dv


# ---------------------------------------------------------------- dropout masks

PHILOX_M = (0xD2511F53, 0xCD9E8D57)   # round multipliers
PHILOX_W = (0x9E3779B9, 0xBB67AE85)   # key increments (golden ratio, sqrt(3) - 1)
_M32 = np.uint64(0xFFFFFFFF)


def philox4x32(counter, key, rounds=10):
    """Philox-4x32 counter-based generator (Salmon, Moraes, Dror and Shaw,
    "Parallel random numbers: as easy as 1, 2, 3", SC 2011), element-wise over
    numpy arrays.  counter: 4 arrays (or ints) of 32-bit words, key: 2 words.
    Each round multiplies words 0 and 2 by the two multipliers, keeps the low
    halves as the new words 1 and 3, folds the high halves into words 1 and 3
    of the input and the key (xor) as the new words 0 and 2; the key grows by
    the two increments between rounds.  Returns 4 uint64 arrays of 32-bit words.
    """
    c = [np.asarray(v, dtype=np.uint64) & _M32 for v in counter]
    k0, k1 = (np.asarray(v, dtype=np.uint64) & _M32 for v in key)
    m0, m1 = np.uint64(PHILOX_M[0]), np.uint64(PHILOX_M[1])
    for _ in range(rounds):
        p0 = m0 * c[0]                  # 32 x 32 -> 64 bits, exact in uint64
        p1 = m1 * c[2]
        c = [(p1 >> np.uint64(32)) ^ c[1] ^ k0, p1 & _M32,
             (p0 >> np.uint64(32)) ^ c[3] ^ k1, p0 & _M32]
        k0 = (k0 + np.uint64(PHILOX_W[0])) & _M32
        k1 = (k1 + np.uint64(PHILOX_W[1])) & _M32
    return c


# Generator streams of the three dropout sites.
STREAM_ATTN_PROBS, STREAM_ATTN_OUT, STREAM_MLP_OUT = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Dropout:
    """Dropout of the layer: rate p_attn on the attention probabilities, rate
    p_hidden on the outputs of the out-projection and of FC2, masks drawn from
    a 64-bit seed."""
    seed: int
    p_attn: float = 0.0
    p_hidden: float = 0.0


def drop_threshold(p):
    """A value is dropped when its 32-bit draw is below floor(p * 2^32)."""
    assert 0.0 <= p < 1.0
    return min(int(np.floor(p * 2.0 ** 32)), 2 ** 32 - 1)


def keep_mask(seed, p, stream, rows, ncols):
    """Boolean keep mask [len(rows), ncols] of one dropout site.

    Element (row, col) draws word col % 4 of Philox-4x32-10 at counter
    (col // 4, row, stream, 0) under key (seed mod 2^32, seed div 2^32): the
    coordinates are global (token and hidden column for the hidden outputs;
    (batch * heads + head) * seq + query and key for the attention
    probabilities), so the mask does not depend on how the layer is split.
    """
    rows = np.asarray(rows, dtype=np.uint64)[:, None]
    groups = np.arange((ncols + 3) // 4, dtype=np.uint64)[None, :]
    words = philox4x32((groups, rows, np.uint64(stream), np.uint64(0)),
                       (np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32)))
    w = np.stack(words, axis=-1).reshape(rows.shape[0], -1)[:, :ncols]
    return w >= np.uint64(drop_threshold(p))


def hidden_keep(drop, stream, n_tokens, h):
    """Keep mask of a hidden-output dropout over [tokens, h], or None when off
    (a rate whose threshold floor(p 2^32) is 0 drops nothing: off)."""
    if drop is None or drop_threshold(drop.p_hidden) == 0:
        return None
    return keep_mask(drop.seed, drop.p_hidden, stream, np.arange(n_tokens), h)


def attn_keep(drop, b, head, heads, seq):
    """Keep mask [seq, seq] of the attention probabilities of (batch b, global
    head `head`), or None when off."""
    if drop is None or drop_threshold(drop.p_attn) == 0:
        return None
    rows = (b * heads + head) * seq + np.arange(seq)
    return keep_mask(drop.seed, drop.p_attn, STREAM_ATTN_PROBS, rows, seq)


# ---------------------------------------------------------------- the layer

def _hidden_dropout(a, drop, stream):
    """a * keep / (1 - p_hidden) over [B, s, h] (identity when off)."""
    keep = hidden_keep(drop, stream, a.shape[0] * a.shape[1], a.shape[2])
    if keep is None:
        return a
    return a * keep.reshape(a.shape) / (1.0 - drop.p_hidden)


def layer_forward(x, p, heads, causal, valid_len=None, eps=1e-5, drop=None):
    """Unpartitioned pre-LN transformer layer.  x: [B, s, h]; p: dict of fp64 arrays.

    Returns (y, cache) with y [B, s, h].  With a Dropout:
    H1 = X + drop(O W_o + b_o), Y = H1 + drop(G B + b2), attention probabilities dropped.
    """
    b_, s_, h = x.shape
    d = h // heads
    xn1, st1 = layer_norm(x, p["ln1_g"], p["ln1_b"], eps)
    q = (xn1 @ p["w_q"] + p["b_q"]).reshape(b_, s_, heads, d)
    k = (xn1 @ p["w_k"] + p["b_k"]).reshape(b_, s_, heads, d)
    v = (xn1 @ p["w_v"] + p["b_v"]).reshape(b_, s_, heads, d)
    o, lse = attention(q, k, v, causal, valid_len, drop)
    o2 = o.reshape(b_, s_, h)
    h1 = x + _hidden_dropout(o2 @ p["w_o"] + p["b_o"], drop, STREAM_ATTN_OUT)
    xn2, st2 = layer_norm(h1, p["ln2_g"], p["ln2_b"], eps)
    u = xn2 @ p["w_fc1"] + p["b_fc1"]
    g = gelu(u)
    y = h1 + _hidden_dropout(g @ p["w_fc2"] + p["b_fc2"], drop, STREAM_MLP_OUT)
    cache = dict(x=x, xn1=xn1, st1=st1, q=q, k=k, v=v, o=o2, lse=lse, h1=h1,
                 xn2=xn2, st2=st2, u=u, g=g)
    return y, cache


def layer_backward(dy, cache, p, heads, causal, valid_len=None, drop=None):
    """Exact gradients of the layer for upstream gradient dy (L = sum(Y * dY))."""
    c = cache
    b_, s_, h = dy.shape
    d = h // heads
    flat = lambda a: a.reshape(-1, a.shape[-1])
    gr = {}
    # MLP: Y = H1 + drop(G B + b2), G = gelu(U), U = Xn2 A + b1
    dz2 = _hidden_dropout(dy, drop, STREAM_MLP_OUT)
    gr["b_fc2"] = flat(dz2).sum(0)
    gr["w_fc2"] = flat(c["g"]).T @ flat(dz2)
    dg = dz2 @ p["w_fc2"].T
    du = dg * gelu_grad(c["u"])
    gr["w_fc1"] = flat(c["xn2"]).T @ flat(du)
    gr["b_fc1"] = flat(du).sum(0)
    dxn2 = du @ p["w_fc1"].T
    dh1_ln, gr["ln2_g"], gr["ln2_b"] = layer_norm_backward(dxn2, c["h1"], p["ln2_g"], *c["st2"])
    dh1 = dy + dh1_ln
    # attention block: H1 = X + drop(O W_o + b_o)
    da1 = _hidden_dropout(dh1, drop, STREAM_ATTN_OUT)
    gr["b_o"] = flat(da1).sum(0)
    gr["w_o"] = flat(c["o"]).T @ flat(da1)
    do = (da1 @ p["w_o"].T).reshape(b_, s_, heads, d)
    dq, dk, dv = attention_backward(do, c["q"], c["k"], c["v"], causal, valid_len, drop)
    dq, dk, dv = (a.reshape(b_, s_, h) for a in (dq, dk, dv))
    xn1 = flat(c["xn1"])
    gr["w_q"], gr["w_k"], gr["w_v"] = xn1.T @ flat(dq), xn1.T @ flat(dk), xn1.T @ flat(dv)
    gr["b_q"], gr["b_k"], gr["b_v"] = flat(dq).sum(0), flat(dk).sum(0), flat(dv).sum(0)
    dxn1 = dq @ p["w_q"].T + dk @ p["w_k"].T + dv @ p["w_v"].T
    dx_ln, gr["ln1_g"], gr["ln1_b"] = layer_norm_backward(dxn1, c["x"], p["ln1_g"], *c["st1"])
    dx = dh1 + dx_ln
    return dx, gr


# ---------------------------------------------------------------- the loss

def cross_entropy(x, emb, target):
    """Unpartitioned loss: logits z = x E^T, l_n = logsumexp(z_n) - z_n[y_n], mean over n.

    Returns (loss, per-token loss, lse).
    """
    z = x @ emb.T
    m = z.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0]
    tok = lse - z[np.arange(z.shape[0]), target]
    return tok.mean(), tok, lse


def cross_entropy_backward(x, emb, target, lse):
    """d loss / d x and d loss / d E for the mean loss (dloss = 1)."""
    n = x.shape[0]
    z = x @ emb.T
    dz = np.exp(z - lse[:, None])
    dz[np.arange(n), target] -= 1.0
    dz /= n
    return dz @ emb, dz.T @ x


# ---------------------------------------------------------------- partitioned forms (pins only)

def slice_partitions(p, t, heads):
    """The oracle's own slicing of unpartitioned parameters into t partitions."""
    h = p["w_q"].shape[0]
    f = p["w_fc1"].shape[1]
    hs, fs = h // t, f // t
    out = []
    for i in range(t):
        c, m = slice(i * hs, (i + 1) * hs), slice(i * fs, (i + 1) * fs)
        out.append(dict(w_q=p["w_q"][:, c], w_k=p["w_k"][:, c], w_v=p["w_v"][:, c],
                        b_q=p["b_q"][c], b_k=p["b_k"][c], b_v=p["b_v"][c],
                        w_o=p["w_o"][c, :], w_fc1=p["w_fc1"][:, m], b_fc1=p["b_fc1"][m],
                        w_fc2=p["w_fc2"][m, :]))
    return out


def layer_forward_partitioned(x, p, heads, t, causal, valid_len=None, eps=1e-5, drop=None):
    """Same layer, computed as t partitions plus an explicit sum at each all-reduce point.

    Partition i: heads [i H/t, (i+1) H/t) (Q/K/V column split), W_o rows of those
    heads (row split), MLP columns of A and rows of B.  LayerNorm, residual and
    the row-split biases are replicated, i.e. computed once.
    """
    b_, s_, h = x.shape
    d = h // heads
    hp = heads // t
    parts = slice_partitions(p, t, heads)
    xn1, _ = layer_norm(x, p["ln1_g"], p["ln1_b"], eps)
    attn_partials = []
    for i, pi in enumerate(parts):
        q = (xn1 @ pi["w_q"] + pi["b_q"]).reshape(b_, s_, hp, d)
        k = (xn1 @ pi["w_k"] + pi["b_k"]).reshape(b_, s_, hp, d)
        v = (xn1 @ pi["w_v"] + pi["b_v"]).reshape(b_, s_, hp, d)
        o, _ = attention(q, k, v, causal, valid_len, drop, i * hp, heads)
        attn_partials.append(o.reshape(b_, s_, h // t) @ pi["w_o"])
    # all-reduce after the row-split W_o; the replicated dropout and residual follow
    h1 = x + _hidden_dropout(sum(attn_partials) + p["b_o"], drop, STREAM_ATTN_OUT)
    xn2, _ = layer_norm(h1, p["ln2_g"], p["ln2_b"], eps)
    mlp_partials = [gelu(xn2 @ pi["w_fc1"] + pi["b_fc1"]) @ pi["w_fc2"] for pi in parts]
    # all-reduce after the row-split B
    return h1 + _hidden_dropout(sum(mlp_partials) + p["b_fc2"], drop, STREAM_MLP_OUT)


def layer_backward_partitioned(dy, x, p, heads, t, causal, valid_len=None, eps=1e-5, drop=None):
    """Backward through t partitions; the input gradients of the column-split
    linears are summed over partitions (the backward all-reduce of the f operator).

    Returns (dx, grads) with grads unpartitioned (partition slices re-assembled).
    """
    b_, s_, h = x.shape
    d = h // heads
    hp = heads // t
    parts = slice_partitions(p, t, heads)
    flat = lambda a: a.reshape(-1, a.shape[-1])
    xn1, st1 = layer_norm(x, p["ln1_g"], p["ln1_b"], eps)
    pc = []
    for i, pi in enumerate(parts):
        q = (xn1 @ pi["w_q"] + pi["b_q"]).reshape(b_, s_, hp, d)
        k = (xn1 @ pi["w_k"] + pi["b_k"]).reshape(b_, s_, hp, d)
        v = (xn1 @ pi["w_v"] + pi["b_v"]).reshape(b_, s_, hp, d)
        o, _ = attention(q, k, v, causal, valid_len, drop, i * hp, heads)
        pc.append(dict(q=q, k=k, v=v, o=o.reshape(b_, s_, h // t)))
    h1 = x + _hidden_dropout(sum(c["o"] @ pi["w_o"] for c, pi in zip(pc, parts)) + p["b_o"],
                             drop, STREAM_ATTN_OUT)
    xn2, st2 = layer_norm(h1, p["ln2_g"], p["ln2_b"], eps)
    us = [xn2 @ pi["w_fc1"] + pi["b_fc1"] for pi in parts]
    gp = [dict() for _ in range(t)]
    dxn2_partials = []
    dz2 = _hidden_dropout(dy, drop, STREAM_MLP_OUT)    # replicated on every partition
    for i, pi in enumerate(parts):
        g = gelu(us[i])
        gp[i]["w_fc2"] = flat(g).T @ flat(dz2)
        du = (dz2 @ pi["w_fc2"].T) * gelu_grad(us[i])
        gp[i]["w_fc1"] = flat(xn2).T @ flat(du)
        gp[i]["b_fc1"] = flat(du).sum(0)
        dxn2_partials.append(du @ pi["w_fc1"].T)
    dxn2 = sum(dxn2_partials)                           # backward all-reduce (MLP)
    dh1_ln, g2, b2 = layer_norm_backward(dxn2, h1, p["ln2_g"], *st2)
    dh1 = dy + dh1_ln
    da1 = _hidden_dropout(dh1, drop, STREAM_ATTN_OUT)  # replicated on every partition
    dxn1_partials = []
    for i, (c, pi) in enumerate(zip(pc, parts)):
        gp[i]["w_o"] = flat(c["o"]).T @ flat(da1)
        do = (da1 @ pi["w_o"].T).reshape(b_, s_, hp, d)
        dq, dk, dv = attention_backward(do, c["q"], c["k"], c["v"], causal, valid_len, drop,
                                        i * hp, heads)
        dq, dk, dv = (a.reshape(b_, s_, h // t) for a in (dq, dk, dv))
        for nm, a in (("q", dq), ("k", dk), ("v", dv)):
            gp[i]["w_" + nm] = flat(xn1).T @ flat(a)
            gp[i]["b_" + nm] = flat(a).sum(0)
        dxn1_partials.append(dq @ pi["w_q"].T + dk @ pi["w_k"].T + dv @ pi["w_v"].T)
    dxn1 = sum(dxn1_partials)                           # backward all-reduce (attention)
    dx_ln, g1, b1 = layer_norm_backward(dxn1, x, p["ln1_g"], *st1)
    grads = {"ln1_g": g1, "ln1_b": b1, "ln2_g": g2, "ln2_b": b2,
             "b_o": flat(da1).sum(0), "b_fc2": flat(dz2).sum(0)}
    for nm in ("w_q", "w_k", "w_v", "w_fc1"):
        grads[nm] = np.concatenate([g[nm] for g in gp], axis=1)
    for nm in ("b_q", "b_k", "b_v", "b_fc1"):
        grads[nm] = np.concatenate([g[nm] for g in gp], axis=0)
    for nm in ("w_o", "w_fc2"):
        grads[nm] = np.concatenate([g[nm] for g in gp], axis=0)
    return dh1 + dx_ln, grads


def vocab_parallel_cross_entropy(x, emb, target, t):
    """The method's loss: each vocab partition reports (max, sum-exp, target logit),
    the triples are combined (the all-reduce of three scalars per token), and no
    partition ever sees the other partitions' logits.

    Returns (loss, per-token loss, lse).
    """
    v = emb.shape[0]
    vs = v // t
    n = x.shape[0]
    m_i, s_i, z_i = np.empty((t, n)), np.empty((t, n)), np.zeros((t, n))
    for i in range(t):
        zi = x @ emb[i * vs:(i + 1) * vs].T
        m_i[i] = zi.max(axis=1)
        s_i[i] = np.exp(zi - m_i[i][:, None]).sum(axis=1)
        mine = (target >= i * vs) & (target < (i + 1) * vs)
        rows = np.nonzero(mine)[0]
        z_i[i, rows] = zi[rows, target[rows] - i * vs]
    big_m = m_i.max(axis=0)
    big_s = (s_i * np.exp(m_i - big_m)).sum(axis=0)
    lse = big_m + np.log(big_s)
    tok = lse - z_i.sum(axis=0)
    return tok.mean(), tok, lse


# ---------------------------------------------------------------- input embedding and the stack

def embedding(ids, emb):
    """Plain lookup X[n] = E[ids[n]]."""
    return emb[ids]


def vocab_parallel_embedding(ids, emb, t):
    """The method's input embedding (rkmt.cn guide, section 3.3: the input layer
    is split along the vocabulary and its outputs are summed by an all-reduce):
    partition i holds rows [i V/t, (i+1) V/t) and outputs its row for the
    tokens in that range and zeros for the others; the t outputs are summed."""
    v = emb.shape[0]
    vs = v // t
    out = np.zeros((len(ids), emb.shape[1]))
    for i in range(t):
        mine = (ids >= i * vs) & (ids < (i + 1) * vs)
        part = np.zeros_like(out)
        part[mine] = emb[i * vs:(i + 1) * vs][ids[mine] - i * vs]
        out += part                                   # the all-reduce
    return out


def embedding_backward(ids, dout, vocab):
    """dE[v] = sum of dout[n] over the tokens n with ids[n] = v."""
    de = np.zeros((vocab, dout.shape[1]))
    np.add.at(de, ids, dout)
    return de


def stack_forward_backward(ids, targets, emb, layers, heads, causal=True, eps=1e-5):
    """A GPT stack with tied embeddings: X0 = E[ids], X_{l+1} = layer_l(X_l),
    loss = cross_entropy(X_L, E, targets) (the output layer reuses the input
    embedding E; no final LayerNorm, as for the single layer with its loss).

    ids, targets: [B, s] ints; emb [V, h]; layers: list of parameter dicts.
    Returns (loss, dE, per-layer parameter gradients), dE = input + output part.
    """
    b_, s_ = ids.shape
    x = embedding(ids.reshape(-1), emb).reshape(b_, s_, -1)
    caches = []
    for p in layers:
        x, c = layer_forward(x, p, heads, causal, None, eps)
        caches.append(c)
    flat = x.reshape(b_ * s_, -1)
    loss, _, lse = cross_entropy(flat, emb, targets.reshape(-1))
    dflat, de_out = cross_entropy_backward(flat, emb, targets.reshape(-1), lse)
    dx = dflat.reshape(x.shape)
    grads = []
    for p, c in zip(reversed(layers), reversed(caches)):
        dx, g = layer_backward(dx, c, p, heads, causal)
        grads.append(g)
    de_in = embedding_backward(ids.reshape(-1), dx.reshape(b_ * s_, -1), emb.shape[0])
    return loss, de_out + de_in, grads[::-1]


def to_f64(params):
    """Widen a dict of bf16/fp32 torch tensors or arrays to fp64 numpy (exact)."""
    out = {}
    for k, v in params.items():
        if hasattr(v, "detach"):
            v = v.detach().to("cpu")
            if v.is_floating_point():
                v = v.double()
            v = v.numpy()
        out[k] = np.asarray(v, dtype=np.float64) if np.asarray(v).dtype.kind == "f" else np.asarray(v)
    return out
