"""Cross-device tensor-parallel plumbing with two gloo ranks on CPU: partition
i on rank i, the four per-layer sums and the loss triple as collectives.

The rank-local steps here are the oracle's own fp64 arithmetic restricted to
the rank's partition (this test stands in for the per-rank kernels, which
need GPUs); what is under test is the package's ownership slicing, the
schedule of local steps and sums, and the loss combine across ranks, checked
against the unpartitioned fp64 oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleRankCompute:
    """Rank-local steps from the oracle's arithmetic on one partition (test only)."""

    def __init__(self, O, shard, p_local, heads, causal, eps=1e-5):
        self.O, self.sh, self.p, self.heads, self.causal, self.eps = O, shard, p_local, heads, causal, eps

    def _split(self, a):
        b, s, _ = a.shape
        hp = self.heads // self.sh.t
        return a.reshape(b, s, hp, -1)

    # forward
    def ln1(self, st):
        st["xn1"], st["st1"] = self.O.layer_norm(st["x"], self.p["ln1_g"], self.p["ln1_b"], self.eps)

    def qkv(self, st):
        q_k_v = st["xn1"] @ self.p["w_qkv"] + self.p["b_qkv"]
        w = q_k_v.shape[-1] // 3
        st["q"], st["k"], st["v"] = (self._split(q_k_v[..., i * w:(i + 1) * w]) for i in range(3))

    def attention(self, st):
        o, _ = self.O.attention(st["q"], st["k"], st["v"], self.causal)
        st["o"] = o.reshape(o.shape[0], o.shape[1], -1)

    def attn_out_partial(self, st):
        st["attn_out_partial"] = torch.from_numpy(st["o"] @ self.p["w_o"])

    def residual1(self, st):
        st["h1"] = st["x"] + st["attn_out_partial"].numpy() + self.p["b_o"]

    def ln2(self, st):
        st["xn2"], st["st2"] = self.O.layer_norm(st["h1"], self.p["ln2_g"], self.p["ln2_b"], self.eps)

    def fc1(self, st):
        st["u"] = st["xn2"] @ self.p["w_fc1"] + self.p["b_fc1"]
        st["g"] = self.O.gelu(st["u"])

    def mlp_out_partial(self, st):
        st["mlp_out_partial"] = torch.from_numpy(st["g"] @ self.p["w_fc2"])

    def residual2(self, st):
        st["y"] = st["h1"] + st["mlp_out_partial"].numpy() + self.p["b_fc2"]

    # backward
    def mlp_out_grad(self, st):
        dy = st["dy"]
        st["du"] = (dy @ self.p["w_fc2"].T) * self.O.gelu_grad(st["u"])

    def fc1_grad(self, st):
        st["dxn2_partial"] = torch.from_numpy(st["du"] @ self.p["w_fc1"].T)

    def ln2_grad(self, st):
        d, _, _ = self.O.layer_norm_backward(st["dxn2_partial"].numpy(), st["h1"], self.p["ln2_g"], *st["st2"])
        st["dh1"] = st["dy"] + d

    def attn_out_grad(self, st):
        st["do"] = self._split(st["dh1"] @ self.p["w_o"].T)

    def attention_grad(self, st):
        dq, dk, dv = self.O.attention_backward(st["do"], st["q"], st["k"], st["v"], self.causal)
        st["dqkv"] = np.concatenate([a.reshape(a.shape[0], a.shape[1], -1) for a in (dq, dk, dv)], -1)

    def qkv_grad(self, st):
        st["dxn1_partial"] = torch.from_numpy(st["dqkv"] @ self.p["w_qkv"].T)

    def ln1_grad(self, st):
        d, _, _ = self.O.layer_norm_backward(st["dxn1_partial"].numpy(), st["x"], self.p["ln1_g"], *st["st1"])
        st["dx"] = st["dh1"] + d


def _rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    from oracle import tp_oracle as O
    from tensor_transformer_layer_tp_b200.parallel import (LAYER_BACKWARD, LAYER_FORWARD, Collective,
                                                           PartitionShard, combine_loss_triples,
                                                           run_schedule, sum_points)
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    coll = Collective()
    rng = np.random.default_rng(7)              # same draws on every rank
    b, s, h, heads, f, v = 2, 8, 32, 4, 128, 64
    p = {n: rng.normal(0, 0.3, shp) for n, shp in dict(
        w_q=(h, h), w_k=(h, h), w_v=(h, h), w_o=(h, h), w_fc1=(h, f), w_fc2=(f, h)).items()}
    for n, shp in dict(b_q=h, b_k=h, b_v=h, b_o=h, b_fc1=f, b_fc2=h, ln1_b=h, ln2_b=h).items():
        p[n] = rng.normal(0, 0.1, shp)
    p["ln1_g"], p["ln2_g"] = 1 + rng.normal(0, 0.1, h), 1 + rng.normal(0, 0.1, h)
    x, dy = rng.normal(0, 1, (b, s, h)), rng.normal(0, 1, (b, s, h))
    shard = PartitionShard(rank=coll.rank, t=coll.size, hidden=h, heads=heads, ffn=f, vocab=v)
    pt = {k: torch.from_numpy(a) for k, a in p.items()}
    local = {k: a.numpy() for k, a in shard.slice_params(pt).items()}
    comp = OracleRankCompute(O, shard, local, heads, True)
    st = run_schedule(LAYER_FORWARD, comp, {"x": x}, coll)
    st["dy"] = dy
    run_schedule(LAYER_BACKWARD, comp, st, coll)
    y_ref, cache = O.layer_forward(x, p, heads, True)
    dx_ref, _ = O.layer_backward(dy, cache, p, heads, True)
    ok_y = float(np.max(np.abs(st["y"] - y_ref)))
    ok_dx = float(np.max(np.abs(st["dx"] - dx_ref)))
    # loss across ranks: each rank reduces its own vocabulary rows
    e = rng.normal(0, 1, (v, h))
    xt = rng.normal(0, 1, (b * s, h))
    tgt = rng.integers(0, v, b * s)
    rows = shard.vocab_rows
    z = xt @ e[rows].T
    m = z.max(1)
    ssum = np.exp(z - m[:, None]).sum(1)
    mine = (tgt >= rows.start) & (tgt < rows.stop)
    zt = np.where(mine, z[np.arange(b * s), np.clip(tgt - rows.start, 0, z.shape[1] - 1)], 0.0)
    loss, tok, lse = combine_loss_triples(torch.from_numpy(m), torch.from_numpy(ssum),
                                          torch.from_numpy(zt), coll)
    loss_ref, tok_ref, _ = O.cross_entropy(xt, e, tgt)
    q.put((coll.rank, ok_y, ok_dx, abs(float(loss) - loss_ref), float(np.max(np.abs(tok.numpy() - tok_ref))),
           sum_points(LAYER_FORWARD) + sum_points(LAYER_BACKWARD), list(shard.head_range)))
    dist.destroy_process_group()


def test_two_ranks_reach_the_unpartitioned_layer_and_loss():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(180)
        assert pr.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ey, edx, eloss, etok, sums, heads in got:
        assert ey < 1e-12 and edx < 1e-12, (ey, edx)
        assert eloss < 1e-12 and etok < 1e-12
        assert len(sums) == 4                       # 2 per module, 4 per layer
        assert heads == [2 * rank, 2 * rank + 1]


def test_partition_shard_ownership():
    from tensor_transformer_layer_tp_b200.parallel import PartitionShard
    sh = PartitionShard(rank=3, t=8, hidden=3072, heads=32, ffn=12288, vocab=50304)
    assert list(sh.head_range) == [12, 13, 14, 15]
    assert sh.hidden_cols == slice(1152, 1536)
    assert sh.ffn_cols == slice(4608, 6144)
    assert sh.vocab_rows == slice(18864, 25152)
    with pytest.raises(ValueError):
        PartitionShard(rank=0, t=3, hidden=3072, heads=32, ffn=12288)


def test_rank_segments_cut_at_the_sum_points():
    """The rank-local calls' three segments per pass are the local steps
    between the schedule's two sum points."""
    from tensor_transformer_layer_tp_b200 import parallel as P
    assert len(P.sum_points(P.LAYER_FORWARD)) == 2 and len(P.sum_points(P.LAYER_BACKWARD)) == 2
    assert [len(s) for s in P.RANK_SEGMENTS_FORWARD] == [4, 4, 1]
    assert [len(s) for s in P.RANK_SEGMENTS_BACKWARD] == [2, 4, 1]
    assert P.RANK_SEGMENTS_FORWARD[0][-1] == "attn_out_partial"
    assert P.RANK_SEGMENTS_BACKWARD[2] == ("ln1_grad",)


def test_rank_runner_orders_segments_and_sums(monkeypatch):
    """RankRunner walks segments 0, 1, 2 of each pass with the all-reduce of
    the partial between them, on the same buffers throughout."""
    from tensor_transformer_layer_tp_b200 import binding as B
    from tensor_transformer_layer_tp_b200 import runner as R
    log = []
    monkeypatch.setattr(B, "tp_layer_rank_saved_bytes", lambda dims: 64)
    monkeypatch.setattr(B, "tp_layer_rank_workspace_bytes", lambda dims: 64)
    monkeypatch.setattr(B, "tp_layer_rank_forward",
                        lambda dims, rank, seg, w, x, vl, partial, y, saved, stream=None:
                        log.append(("f", seg, partial.data_ptr(), saved.data_ptr())))
    monkeypatch.setattr(B, "tp_layer_rank_backward",
                        lambda dims, rank, seg, w, x, vl, saved, dy, partial, dx, g, ws, stream=None:
                        log.append(("b", seg, partial.data_ptr(), ws.data_ptr())))
    dims = B.make_dims(2, 1, 8, 64, 1, 256)
    params = {k: torch.zeros(4) for k in R.REPLICATED}
    params.update({k: [torch.zeros(4)] for k in R.PARTITIONED})
    r = R.RankRunner(dims, 1, params, device="cpu")
    sums = lambda t: log.append(("sum", t.data_ptr()))
    x = torch.zeros(1, 8, 64, dtype=torch.bfloat16)
    r.forward(x, sums)
    r.backward(x, x, sums)
    kinds = [e[0] if e[0] == "sum" else e[0] + str(e[1]) for e in log]
    assert kinds == ["f0", "sum", "f1", "sum", "f2", "b0", "sum", "b1", "sum", "b2"]
    assert len({e[2] if e[0] != "sum" else e[1] for e in log}) == 1   # one partial buffer


def test_rank_xent_runner_orders_segments_and_collectives(monkeypatch):
    """RankXentRunner: segment 0, max over ranks of comm[0], segment 1, sum
    over ranks of comm[1:3], segment 2, and the sum of the dX terms."""
    from tensor_transformer_layer_tp_b200 import binding as B
    from tensor_transformer_layer_tp_b200 import runner as R
    log = []
    monkeypatch.setattr(B, "tp_xent_rank_workspace_bytes", lambda *a: 64)
    monkeypatch.setattr(B, "vocab_parallel_xent_rank",
                        lambda t, rank, seg, *a, **k: log.append(f"seg{seg}"))
    r = R.RankXentRunner(4, 2, 16, 8, 64, device="cpu")
    x = torch.zeros(16, 8, dtype=torch.bfloat16)
    r(x, torch.zeros(16, 8), torch.zeros(16, dtype=torch.int32),
      lambda t: log.append(("max", tuple(t.shape))), lambda t: log.append(("sum", tuple(t.shape))))
    assert log == ["seg0", ("max", (16,)), "seg1", ("sum", (2, 16)), "seg2", ("sum", (16, 8))]
