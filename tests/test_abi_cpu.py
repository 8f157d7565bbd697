"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports every
function include/tplayer.h declares, sizes its buffers, and rejects bad
arguments before any launch."""
import ctypes

import pytest

from tensor_transformer_layer_tp_b200 import binding as B
from tp_inputs import WORKLOADS


def test_library_exports_every_header_function():
    names = B.header_functions()
    assert len(names) >= 9
    lib = B.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    assert B.status_string(B.TP_OK) == "ok"
    assert "workspace" in B.status_string(B.TP_ERR_WORKSPACE)
    assert B.status_string(99) == "unknown status"


def _dims(name, t=None):
    d = WORKLOADS[name]
    return B.make_dims(t or d.t, d.batch, d.seq, d.hidden, d.heads, d.ffn, d.causal, d.ln_eps)


def test_saved_and_workspace_sizes_cover_the_activations():
    d = _dims("gpt_8p3b_t8")
    n, h, f = 4 * 1024, 3072, 12288
    saved = B.tp_layer_saved_bytes(d)
    # Xn1, QKV (3h), O, H1, Xn2 in bf16 + U and G (f each) + stats + lse
    assert saved >= 2 * n * (h + 3 * h + h + h + h + 2 * f)
    assert saved < 1.1 * 2 * n * (7 * h + 2 * f) + 64 * n
    ws = B.tp_layer_workspace_bytes(d)
    assert ws >= 2 * n * (f + 4 * h + 3 * h)   # dU, dXn2, dH1, dO, dXn1, dQKV (bf16)
    # sizes do not depend on t
    assert B.tp_layer_saved_bytes(_dims("gpt_8p3b_t8", 1)) == saved


@pytest.mark.parametrize("field,value,status", [
    ("t", 3, B.TP_ERR_UNSUPPORTED),        # 32 heads not divisible by 3
    ("t", 16, B.TP_ERR_UNSUPPORTED),       # above 8 partitions
    ("heads", 40, B.TP_ERR_UNSUPPORTED),   # hidden % heads != 0
    ("hidden", 3000, B.TP_ERR_UNSUPPORTED),
    ("batch", 0, B.TP_ERR_INVALID_ARG),    # empty input
    ("seq", -1, B.TP_ERR_INVALID_ARG),
])
def test_bad_dims_are_rejected_before_launch(field, value, status):
    d = _dims("gpt_8p3b_t8")
    setattr(d, field, value)
    assert B.tp_layer_saved_bytes(d) == 0
    w = B.tp_layer_weights()
    rc = B.lib().tp_layer_forward(ctypes.byref(d), ctypes.byref(w), None, None, None, None, 0, None,
                                  0, None)
    assert rc == status


def test_null_pointers_are_rejected():
    d = _dims("tiny_gpt_t2")
    w = B.tp_layer_weights()
    assert B.lib().tp_layer_forward(ctypes.byref(d), ctypes.byref(w), None, None, None, None, 0,
                                    None, 0, None) == B.TP_ERR_INVALID_ARG
    g = B.tp_layer_grads()
    assert B.lib().tp_layer_backward(ctypes.byref(d), ctypes.byref(w), None, None, None, 0, None,
                                     None, ctypes.byref(g), None, 0, None) == B.TP_ERR_INVALID_ARG


def test_short_workspace_is_rejected():
    d = _dims("tiny_gpt_t2")
    w = B.tp_layer_weights()
    g = B.tp_layer_grads()
    fake = 1 << 20   # never dereferenced: the size check fails first
    full_saved = B.tp_layer_saved_bytes(d)
    full_ws = B.tp_layer_workspace_bytes(d)
    rc = B.lib().tp_layer_backward(ctypes.byref(d), ctypes.byref(w), fake, None, fake, full_saved,
                                   fake, fake, ctypes.byref(g), fake, 16, None)
    assert rc == B.TP_ERR_WORKSPACE
    # a short saved-activation buffer, in the forward (written) and the backward (read)
    rc = B.lib().tp_layer_backward(ctypes.byref(d), ctypes.byref(w), fake, None, fake,
                                   full_saved - 256, fake, fake, ctypes.byref(g), fake, full_ws, None)
    assert rc == B.TP_ERR_WORKSPACE


def test_short_saved_buffer_is_rejected_by_the_forward():
    d = _dims("tiny_gpt_t2")
    fake = 1 << 20
    ptrs = {k: fake for k in ("ln1_g", "ln1_b", "b_o", "ln2_g", "ln2_b", "b_fc2")}
    for k in ("w_qkv", "b_qkv", "w_o", "w_fc1", "b_fc1", "w_fc2"):
        ptrs[k] = [fake] * d.t
    w = B._fill(B.tp_layer_weights, ptrs, d.t)
    rc = B.lib().tp_layer_forward(ctypes.byref(d), ctypes.byref(w), fake, None, fake, fake,
                                  B.tp_layer_saved_bytes(d) - 1, None, 0, None)
    assert rc == B.TP_ERR_WORKSPACE


def test_xent_argument_checks():
    L = B.lib()
    # fused path: bf16 logits (2 bytes per logit) plus per-tile statistics
    assert B.tp_xent_workspace_bytes(8, 8192, 1024, 50304) >= 8192 * 50304 * 2
    assert B.tp_xent_forward_workspace_bytes(8, 8192, 1024, 50304) < 8192 * 50304 // 16
    # explicit path: fp32 logits and a bf16 gradient (6 bytes per logit)
    assert B.tp_xent_explicit_workspace_bytes(8, 8192, 1024, 50304) > 8192 * 50304 * 6
    assert B.tp_xent_workspace_bytes(5, 8192, 1024, 50304) == 0      # V not divisible by t
    assert B.tp_xent_workspace_bytes(1, 0, 1024, 50304) == 0         # no tokens
    emb = (ctypes.c_void_p * 1)(None)
    rc = L.vocab_parallel_xent(1, 16, 64, 1000, None, emb, None, None, None, None, None, None, 0, None)
    assert rc == B.TP_ERR_INVALID_ARG
    rc = L.vocab_parallel_xent(3, 16, 64, 1000, None, emb, None, None, None, None, None, None, 0, None)
    assert rc == B.TP_ERR_UNSUPPORTED
    for fn in (L.vocab_parallel_xent, L.vocab_parallel_xent_explicit):
        fake = 1 << 20   # never dereferenced: the workspace check fails first
        e1 = (ctypes.c_void_p * 1)(fake)
        rc = fn(1, 16, 64, 1024, fake, e1, fake, fake, None, None, None, fake, 64, None)
        assert rc == B.TP_ERR_WORKSPACE


def test_gemm_argument_checks():
    L = B.lib()
    p = (ctypes.c_void_p * 1)(None)
    assert L.tp_gemm(1, 0, 0, 8, 8, p, 0, p, 0, p, 0, 0, -1, None) == B.TP_ERR_INVALID_ARG
    assert L.tp_gemm(9, 0, 8, 8, 8, p, 0, p, 0, p, 0, 0, -1, None) == B.TP_ERR_UNSUPPORTED
    assert L.tp_gemm(1, 0, 8, 12, 8, p, 0, p, 0, p, 0, 0, -1, None) == B.TP_ERR_UNSUPPORTED
    assert L.tp_gemm(1, 0, 8, 8, 8, p, 0, p, 0, p, 0, 192, -1, None) == B.TP_ERR_INVALID_ARG


def test_gelu_eval_argument_checks():
    L = B.lib()
    assert L.tp_gelu_eval(-1, None, None, None, None) == B.TP_ERR_INVALID_ARG
    assert L.tp_gelu_eval(4, None, None, None, None) == B.TP_ERR_INVALID_ARG
    assert L.tp_gelu_eval(0, None, None, None, None) == B.TP_OK       # nothing to do


def test_partition_sum_argument_checks():
    L = B.lib()
    p = (ctypes.c_void_p * 1)(None)
    assert L.tp_partition_sum(0, 4, 4, p, 4, None, None, None, None) == B.TP_ERR_INVALID_ARG
    assert L.tp_partition_sum(9, 4, 4, p, 4, None, None, None, None) == B.TP_ERR_INVALID_ARG
    assert L.tp_partition_sum(1, 4, 6, p, 8, None, None, None, None) == B.TP_ERR_INVALID_ARG
    assert L.tp_partition_sum(1, 4, 4, p, 4, None, None, None, None) == B.TP_ERR_INVALID_ARG


@pytest.mark.parametrize("field,value,status", [
    ("dropout_attn", 1.0, B.TP_ERR_INVALID_ARG),     # rates live in [0, 1)
    ("dropout_hidden", -0.1, B.TP_ERR_INVALID_ARG),
    ("dropout_attn", float("nan"), B.TP_ERR_INVALID_ARG),
    ("recompute", 2, B.TP_ERR_INVALID_ARG),
])
def test_bad_options_are_rejected(field, value, status):
    d = _dims("tiny_gpt_t2")
    setattr(d, field, value)
    assert B.tp_layer_saved_bytes(d) == 0
    w = B.tp_layer_weights()
    rc = B.lib().tp_layer_forward(ctypes.byref(d), ctypes.byref(w), None, None, None, None, 0, None,
                                  0, None)
    assert rc == status


def test_attention_dropout_row_numbering_limit():
    # (batch * heads + head) * seq + query must fit 32 bits with attention dropout
    d = B.make_dims(1, 2 ** 16, 2 ** 12, 256, 4, 1024, dropout_attn=0.1)
    assert B.tp_layer_saved_bytes(d) == 0
    d.dropout_attn = 0.0
    d.batch = 2 ** 8
    assert B.tp_layer_saved_bytes(d) > 0


def test_recompute_moves_activations_out_of_saved():
    base = _dims("gpt_8p3b_t8")
    rec = _dims("gpt_8p3b_t8")
    rec.recompute = 1
    n = base.batch * base.seq
    stats = 4 * n * 4 + base.batch * base.heads * base.seq * 4
    assert B.tp_layer_forward_workspace_bytes(base) == 0
    assert stats <= B.tp_layer_saved_bytes(rec) <= stats + 5 * 256
    # the activations move to the forward scratch and into the backward scratch
    act = B.tp_layer_saved_bytes(base) - B.tp_layer_saved_bytes(rec)
    assert B.tp_layer_forward_workspace_bytes(rec) >= act
    assert B.tp_layer_workspace_bytes(rec) >= B.tp_layer_workspace_bytes(base) + act
    # hidden dropout needs the gradients of the dropped outputs
    drop = _dims("gpt_8p3b_t8")
    drop.dropout_hidden = 0.1
    assert B.tp_layer_workspace_bytes(drop) >= B.tp_layer_workspace_bytes(base) + 2 * n * base.hidden * 2


def test_recompute_forward_needs_its_workspace():
    d = _dims("tiny_gpt_t2")
    d.recompute = 1
    fake = 1 << 20
    ptrs = {k: fake for k in ("ln1_g", "ln1_b", "b_o", "ln2_g", "ln2_b", "b_fc2")}
    for k in ("w_qkv", "b_qkv", "w_o", "w_fc1", "b_fc1", "w_fc2"):
        ptrs[k] = [fake] * d.t
    w = B._fill(B.tp_layer_weights, ptrs, d.t)
    rc = B.lib().tp_layer_forward(ctypes.byref(d), ctypes.byref(w), fake, None, fake, fake,
                                  B.tp_layer_saved_bytes(d), None, 0, None)
    assert rc == B.TP_ERR_WORKSPACE


def test_rank_local_sizes():
    """A rank-local pass holds one partition's tensors: with t = 1 its saved
    and scratch sizes are the whole layer's; with t > 1 they are smaller, and
    unsupported options (recompute) report size 0."""
    one = B.make_dims(1, 2, 128, 512, 8, 2048)
    assert B.tp_layer_rank_saved_bytes(one) == B.tp_layer_saved_bytes(one) > 0
    assert B.tp_layer_rank_workspace_bytes(one) == B.tp_layer_workspace_bytes(one) > 0
    four = B.make_dims(4, 2, 128, 512, 8, 2048)
    assert 0 < B.tp_layer_rank_saved_bytes(four) < B.tp_layer_saved_bytes(four)
    assert 0 < B.tp_layer_rank_workspace_bytes(four) < B.tp_layer_workspace_bytes(four)
    assert B.tp_layer_rank_saved_bytes(B.make_dims(4, 2, 128, 512, 8, 2048, recompute=True)) == 0


def test_rank_local_loss_sizes_and_checks():
    """One vocab partition's loss scratch is a slice of the one-device loss's;
    a rank or segment out of range and an unsplittable vocabulary are refused
    before any launch (no GPU needed for that)."""
    whole = B.tp_xent_workspace_bytes(8, 8192, 1024, 50304)
    part = B.tp_xent_rank_workspace_bytes(8, 8192, 1024, 50304)
    assert 0 < part < whole
    assert B.tp_xent_rank_workspace_bytes(4, 8192, 1024, 50300) == 0   # slices of 12575 rows
    f = B.lib().vocab_parallel_xent_rank
    for rank, seg in ((8, 0), (-1, 0), (0, 3)):
        assert f(8, rank, seg, 8192, 1024, 50304, None, None, None, None, None, None, None, None,
                 None, 0, None) == B.TP_ERR_INVALID_ARG
