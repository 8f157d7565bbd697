"""Parity at the workloads' full sizes, in the configuration bench.py times.

The fp64 oracle runs the whole unpartitioned layer (or loss) once per model
and every partition count t is compared against it: the GPT-2 355M layer at
t = 1, 2, 4; the 8.3B-scale layer at t = 8; the 3.9B BERT layer (key padding)
at t = 4; the 8192 x 1024 x 50304 vocab-parallel loss at t = 1, 2, 4, 8.
"""
import functools

import numpy as np
import pytest
import torch

from helpers import LOSS_RTOL, assert_close, f64
from oracle import tp_oracle as O
from test_gpu_layer import GRAD_NAMES, check_grad, gpu_layer
from tp_inputs import (WORKLOADS, XENT_WORKLOADS, XentDims, assemble_layer_grads, make_layer_inputs,
                       make_xent_inputs, partition_vocab)
from tensor_transformer_layer_tp_b200.runner import XentRunner

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@functools.lru_cache(maxsize=1)
def layer_reference(base: str):
    d = WORKLOADS[base]
    inp = make_layer_inputs(d, seed=0)
    p = O.to_f64({k: inp[k] for k in GRAD_NAMES})
    vl = inp["valid_len"].numpy() if "valid_len" in inp else None
    y, cache = O.layer_forward(f64(inp["x"]), p, d.heads, d.causal, vl, d.ln_eps)
    dx, gr = O.layer_backward(f64(inp["dy"]), cache, p, d.heads, d.causal, vl)
    return inp, y, dx, gr


LAYER_CASES = [("gpt2_355m_t1", "gpt2_355m_t1"), ("gpt2_355m_t1", "gpt2_355m_t2"),
               ("gpt2_355m_t1", "gpt2_355m_t4"), ("gpt_8p3b_t8", "gpt_8p3b_t8"),
               ("bert_3p9b_t4", "bert_3p9b_t4")]


@pytest.mark.parametrize("base,name", LAYER_CASES)
def test_full_size_layer(base, name):
    inp, y, dx, gr = layer_reference(base)
    d = WORKLOADS[name]
    r = gpu_layer(d, inp, inp["dy"])
    assert_close("y", r.y, y)
    assert_close("dx", r.dx, dx)
    g = assemble_layer_grads(r.grads, d.t)
    for k in GRAD_NAMES:
        check_grad(k, g[k], gr, d.seq)


@functools.lru_cache(maxsize=1)
def xent_reference():
    d = XENT_WORKLOADS["xent_50k_t1"]
    inp = make_xent_inputs(d, seed=0)
    x, e, y = f64(inp["x"]), f64(inp["emb"]), inp["target"].numpy()
    n = d.tokens
    toks, dx, de = [], [], np.zeros_like(e)
    for c0 in range(0, n, 1024):      # chunks of tokens bound the fp64 logits to 0.4 GB
        xc, yc = x[c0:c0 + 1024], y[c0:c0 + 1024]
        _, tok, lse = O.cross_entropy(xc, e, yc)
        dxc, dec = O.cross_entropy_backward(xc, e, yc, lse)
        w = len(xc) / n               # chunk means -> mean over all tokens
        toks.append(tok)
        dx.append(dxc * w)
        de += dec * w
    tok = np.concatenate(toks)
    return inp, tok.mean(), tok, np.concatenate(dx), de


@pytest.mark.parametrize("explicit", [False, True])
@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_full_size_xent(t, explicit):
    inp, loss, tok, dx, de = xent_reference()
    d = XENT_WORKLOADS[f"xent_50k_t{t}"]
    r = XentRunner(d.t, d.tokens, d.hidden, d.vocab, explicit=explicit)
    r(inp["x"].cuda(), [e.cuda() for e in partition_vocab(inp["emb"], t)], inp["target"].cuda())
    torch.cuda.synchronize()
    assert abs(r.loss.item() - loss) <= LOSS_RTOL * abs(loss)
    assert_close("loss_per_token", r.loss_tok, tok, tol=LOSS_RTOL)
    assert_close("dx", r.dx, dx)
    assert_close("demb", torch.cat([g.cpu() for g in r.demb], 0), de)
