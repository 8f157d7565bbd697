"""Dropout (Philox-keyed masks) and activation recomputation through the C-ABI,
against the fp64 oracle with the same masks.

The masks are keyed by global coordinates, so the GPU and the oracle draw the
same keep bits element by element, and every partition count t draws the same
masks (Megatron-LM show notes: dropout is replicated on every partition).
Tolerance: max|err| <= 2e-2 max|ref| per tensor, as for every layer output.
"""
import numpy as np
import pytest
import torch

from helpers import TENSOR_TOL, assert_close, f64
from oracle import tp_oracle as O
from test_gpu_layer import GRAD_NAMES, check_grad
from tensor_transformer_layer_tp_b200 import binding as B
from tensor_transformer_layer_tp_b200.runner import LayerRunner, params_to
from tp_inputs import LayerDims, assemble_layer_grads, make_layer_inputs, partition_layer_params

pytestmark = pytest.mark.gpu

SEED = 0x5EED_0000_1234_ABCD


def run_gpu(d: LayerDims, inp, p_attn=0.0, p_hidden=0.0, seed=SEED, recompute=False):
    dims = B.make_dims(d.t, d.batch, d.seq, d.hidden, d.heads, d.ffn, d.causal, d.ln_eps,
                       dropout_attn=p_attn, dropout_hidden=p_hidden, seed=seed,
                       recompute=recompute)
    r = LayerRunner(dims, params_to(partition_layer_params(inp, d.t, d.heads), "cuda"))
    x = inp["x"].cuda()
    vl = inp["valid_len"].cuda() if "valid_len" in inp else None
    r.forward(x, vl)
    r.backward(x, inp["dy"].cuda(), vl)
    torch.cuda.synchronize()
    B.tp_device_status()
    return r


def run_oracle(d: LayerDims, inp, drop):
    p = O.to_f64({k: inp[k] for k in GRAD_NAMES})
    vl = inp["valid_len"].numpy() if "valid_len" in inp else None
    y, cache = O.layer_forward(f64(inp["x"]), p, d.heads, d.causal, vl, d.ln_eps, drop=drop)
    dx, gr = O.layer_backward(f64(inp["dy"]), cache, p, d.heads, d.causal, vl, drop=drop)
    return y, dx, gr


def check(r, d, y, dx, gr):
    assert_close("y", r.y, y)
    assert_close("dx", r.dx, dx)
    g = assemble_layer_grads(r.grads, d.t)
    for k in GRAD_NAMES:
        check_grad(k, g[k], gr, d.seq)


CASES = {
    "causal t2": LayerDims(batch=2, seq=128, hidden=512, heads=8, ffn=2048, t=2),
    "causal t4 ragged seq": LayerDims(batch=1, seq=200, hidden=384, heads=4, ffn=1536, t=4),
    "bert padding t2": LayerDims(batch=3, seq=96, hidden=256, heads=4, ffn=1024, t=2, causal=False,
                                 padding=0.5),
    "head_dim 128": LayerDims(batch=2, seq=128, hidden=256, heads=2, ffn=1024, t=2),
}


@pytest.mark.parametrize("name", list(CASES))
def test_dropout_matches_oracle(name):
    d = CASES[name]
    inp = make_layer_inputs(d, seed=21)
    drop = O.Dropout(seed=SEED, p_attn=0.15, p_hidden=0.1)
    r = run_gpu(d, inp, drop.p_attn, drop.p_hidden)
    check(r, d, *run_oracle(d, inp, drop))


def test_dropout_masks_do_not_depend_on_t():
    base = LayerDims(batch=2, seq=128, hidden=512, heads=8, ffn=2048, t=1)
    inp = make_layer_inputs(base, seed=22)
    outs = []
    for t in (1, 2, 8):
        d = LayerDims(batch=2, seq=128, hidden=512, heads=8, ffn=2048, t=t)
        r = run_gpu(d, inp, 0.2, 0.2)
        outs.append((f64(r.y), f64(r.dx)))
    for y, dx in outs[1:]:
        assert np.max(np.abs(y - outs[0][0])) <= 1e-2 * np.max(np.abs(outs[0][0]))
        assert np.max(np.abs(dx - outs[0][1])) <= 1e-2 * np.max(np.abs(outs[0][1]))


def test_seed_changes_the_masks_and_rate_zero_is_off():
    d = CASES["causal t2"]
    inp = make_layer_inputs(d, seed=23)
    a = run_gpu(d, inp, 0.1, 0.1, seed=1)
    b = run_gpu(d, inp, 0.1, 0.1, seed=2)
    assert torch.count_nonzero(a.y != b.y).item() > 0.05 * a.y.numel()
    off = run_gpu(d, inp, 0.0, 0.0, seed=1)
    plain = run_gpu(d, inp, 0.0, 0.0, seed=99)
    assert torch.equal(off.y, plain.y)


@pytest.mark.parametrize("name", ["causal t2", "bert padding t2", "head_dim 128"])
@pytest.mark.parametrize("with_dropout", [False, True])
def test_recompute_matches_saved_mode_and_oracle(name, with_dropout):
    d = CASES[name]
    inp = make_layer_inputs(d, seed=24)
    pa, ph = (0.1, 0.1) if with_dropout else (0.0, 0.0)
    saved = run_gpu(d, inp, pa, ph)
    rec = run_gpu(d, inp, pa, ph, recompute=True)
    # the same forward kernels rebuild the same activations: the output is
    # bitwise equal, the gradients equal up to the order of the dQ reduce-add
    assert torch.equal(saved.y, rec.y)
    assert_close("dx (recompute vs saved)", rec.dx, f64(saved.dx), tol=2e-3)
    gs, gr_ = assemble_layer_grads(saved.grads, d.t), assemble_layer_grads(rec.grads, d.t)
    for k in GRAD_NAMES:
        ref = f64(gs[k])
        if np.max(np.abs(ref)) > 0:
            assert np.max(np.abs(f64(gr_[k]) - ref)) <= 2e-3 * np.max(np.abs(ref)) + 1e-6, k
    drop = O.Dropout(seed=SEED, p_attn=pa, p_hidden=ph) if with_dropout else None
    check(rec, d, *run_oracle(d, inp, drop))
    # the saved buffer holds only the LayerNorm statistics and the log-sum-exp
    assert rec.saved.numel() < saved.saved.numel() // 20
