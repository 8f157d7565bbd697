"""vocab_parallel_xent_static, the cross-entropy entry point for callers that
cannot allocate device memory (their GPU memory is owned by another component,
or they have no allocator to create and keep a workspace).  It must give what
vocab_parallel_xent gives with a caller workspace, call after call, although
every call reuses the same fixed scratch array inside the library.

This file is collected last so that a failure here does not stop the rest of
a `pytest -x` run; it also passes on its own in a fresh process."""
import pytest
import torch

from helpers import LOSS_RTOL, assert_close
from tensor_transformer_layer_tp_b200 import binding as B
from tensor_transformer_layer_tp_b200.runner import XentRunner
from tp_inputs import XentDims, make_xent_inputs, partition_vocab

pytestmark = pytest.mark.gpu


def _outputs(d: XentDims):
    return (torch.empty(1, dtype=torch.float32, device="cuda"),
            torch.empty(d.tokens, dtype=torch.float32, device="cuda"),
            torch.empty(d.tokens, d.hidden, dtype=torch.bfloat16, device="cuda"),
            [torch.empty(d.vocab // d.t, d.hidden, dtype=torch.bfloat16, device="cuda")
             for _ in range(d.t)])


def test_static_scratch_matches_workspace_entry_point_on_two_calls():
    d = XentDims(tokens=1000, hidden=512, vocab=8192, t=4)   # ~49 MB of scratch
    assert B.tp_xent_workspace_bytes(d.t, d.tokens, d.hidden, d.vocab) <= B.XENT_STATIC_SCRATCH_BYTES
    ref = XentRunner(d.t, d.tokens, d.hidden, d.vocab)
    for seed in (7, 8):                      # two calls in a row, different data
        inp = make_xent_inputs(d, seed=seed)
        x = inp["x"].cuda()
        emb = [e.cuda() for e in partition_vocab(inp["emb"], d.t)]
        tgt = inp["target"].cuda()
        ref(x, emb, tgt)
        loss, tok, dx, demb = _outputs(d)
        B.vocab_parallel_xent_static(d.t, d.tokens, d.hidden, d.vocab, x, emb, tgt, loss, tok,
                                     dx, demb)
        torch.cuda.synchronize()
        B.tp_device_status()
        assert abs(loss.item() - ref.loss.item()) <= LOSS_RTOL * abs(ref.loss.item())
        assert_close("loss_per_token", tok, ref.loss_tok, tol=LOSS_RTOL)
        assert_close("dx", dx, ref.dx)
        for i in range(d.t):
            assert_close(f"demb[{i}]", demb[i], ref.demb[i])


def test_static_scratch_rejects_calls_beyond_its_size():
    d = XentDims(tokens=8192, hidden=1024, vocab=50304, t=8)   # needs ~2.5 GB
    x = torch.zeros(16, 16, dtype=torch.bfloat16, device="cuda")   # never read: rejected first
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    with pytest.raises(B.TPError) as err:
        B.vocab_parallel_xent_static(d.t, d.tokens, d.hidden, d.vocab, x, [x] * d.t, x, loss)
    assert err.value.status == B.TP_ERR_WORKSPACE
