"""The vocab-parallel input embedding and a tied-embedding GPT stack through
the C-ABI, against the fp64 oracle (rkmt.cn guide, section 3.3: the input
layer split along the vocabulary with an all-reduce of its outputs; the
output layer split the same way and fused with the loss)."""
import numpy as np
import pytest
import torch

from helpers import assert_close, f64
from oracle import tp_oracle as O
from test_gpu_layer import GRAD_NAMES, check_grad
from tensor_transformer_layer_tp_b200 import binding as B
from tensor_transformer_layer_tp_b200.runner import StackRunner, params_to
from tp_inputs import (LayerDims, WEIGHT_STD, assemble_layer_grads, make_layer_inputs,
                       partition_layer_params, partition_vocab)

pytestmark = pytest.mark.gpu


def _edge_ids(n, vocab, t, gen):
    vp = vocab // t
    edges = sorted({0, vocab - 1} | {i * vp for i in range(1, t)} | {i * vp - 1 for i in range(1, t)})
    ids = torch.randint(0, vocab, (n,), generator=gen, dtype=torch.int32)
    ids[:len(edges)] = torch.tensor(edges, dtype=torch.int32)
    return ids


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_embedding_forward_is_the_owner_row(t):
    gen = torch.Generator().manual_seed(30 + t)
    vocab, h, n = 8 * 136, 256, 700
    emb = (torch.randn(vocab, h, generator=gen) * WEIGHT_STD).to(torch.bfloat16)
    ids = _edge_ids(n, vocab, t, gen)
    ids[-3:] = torch.tensor([-1, vocab, 10 * vocab], dtype=torch.int32)   # outside: zero rows
    out = torch.empty(n, h, dtype=torch.bfloat16, device="cuda")
    B.vocab_parallel_embedding_forward(t, n, h, vocab, ids.cuda(), [e.cuda() for e in partition_vocab(emb, t)], out)
    torch.cuda.synchronize()
    ref = O.vocab_parallel_embedding(ids[:-3].numpy(), f64(emb), t)
    assert np.array_equal(f64(out[:-3]), ref)          # a copy: bit-exact
    assert torch.count_nonzero(out[-3:]).item() == 0


@pytest.mark.parametrize("accumulate", [False, True])
@pytest.mark.parametrize("t", [1, 2, 8])
def test_embedding_backward_matches_oracle(t, accumulate):
    gen = torch.Generator().manual_seed(40 + t)
    vocab, h, n = 8 * 136, 256, 3000          # many repeated ids
    ids = _edge_ids(n, vocab, t, gen)
    dout = torch.randn(n, h, generator=gen).to(torch.bfloat16)
    base = (torch.randn(vocab, h, generator=gen) * 0.1).to(torch.bfloat16)
    demb = [p.cuda() for p in partition_vocab(base, t)] if accumulate else \
        [torch.empty(vocab // t, h, dtype=torch.bfloat16, device="cuda") for _ in range(t)]
    ws = torch.empty(B.tp_embedding_backward_workspace_bytes(t, n, h, vocab), dtype=torch.uint8,
                     device="cuda")
    B.vocab_parallel_embedding_backward(t, n, h, vocab, ids.cuda(), dout.cuda(), demb, accumulate, ws)
    torch.cuda.synchronize()
    ref = O.embedding_backward(ids.numpy(), f64(dout), vocab) + (f64(base) if accumulate else 0.0)
    got = torch.cat([g.cpu() for g in demb], 0)
    assert_close("demb", got, ref, tol=1e-2)


def test_tied_stack_matches_oracle():
    t, layers = 2, 2
    d = LayerDims(batch=2, seq=128, hidden=256, heads=4, ffn=1024, t=t)
    vocab = 1024
    gen = torch.Generator().manual_seed(50)
    emb = (torch.randn(vocab, d.hidden, generator=gen) * WEIGHT_STD).to(torch.bfloat16)
    ids = torch.randint(0, vocab, (d.batch, d.seq), generator=gen, dtype=torch.int32)
    targets = torch.randint(0, vocab, (d.batch, d.seq), generator=gen, dtype=torch.int32)
    inps = [make_layer_inputs(d, seed=60 + l) for l in range(layers)]
    dims = B.make_dims(t, d.batch, d.seq, d.hidden, d.heads, d.ffn, d.causal, d.ln_eps)
    emb_parts = [e.cuda() for e in partition_vocab(emb, t)]
    st = StackRunner(dims, [params_to(partition_layer_params(p, t, d.heads), "cuda") for p in inps],
                     emb_parts, vocab)
    loss = st.step(ids.view(-1).cuda(), targets.view(-1).cuda())
    torch.cuda.synchronize()
    B.tp_device_status()

    p64 = [O.to_f64({k: p[k] for k in GRAD_NAMES}) for p in inps]
    loss64, de64, grads64 = O.stack_forward_backward(ids.numpy(), targets.numpy(), f64(emb), p64, d.heads)
    # the loss sees bf16 hidden states after two layers (see the layer + loss reading)
    assert abs(loss.item() - loss64) <= 2e-4 * abs(loss64)
    assert_close("dE (tied: input + output halves)", torch.cat([g.cpu() for g in st.demb], 0), de64)
    for l in range(layers):
        g = assemble_layer_grads(st.layers[l].grads, t)
        for k in GRAD_NAMES:
            check_grad(k, g[k], grads64[l], d.seq)
