"""tcgen05 GEMM through the C-ABI (tp_gemm): every operand layout, grouped
(column-parallel) and partition-summed (row-parallel + all-reduce) modes,
ragged M/N/K tails, and enough tiles that each persistent CTA handles several
(both TMEM accumulators, many ring wrap-arounds).  Reference: fp64 matmul of
the same bf16 operands."""
import numpy as np
import pytest
import torch

from helpers import assert_close, f64
from tensor_transformer_layer_tp_b200 import binding as B

pytestmark = pytest.mark.gpu


def _operands(groups, m, n, k, a_layout, b_layout, seed):
    g = torch.Generator().manual_seed(seed)
    A = [torch.randn(m, k, generator=g).to(torch.bfloat16) for _ in range(groups)]
    Bm = [torch.randn(k, n, generator=g).to(torch.bfloat16) for _ in range(groups)]
    a_st = [a.t().contiguous() if a_layout else a for a in A]
    b_st = [b.t().contiguous() if b_layout else b for b in Bm]
    return A, Bm, [x.cuda() for x in a_st], [x.cuda() for x in b_st]


@pytest.mark.parametrize("a_layout,b_layout", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("groups,sum_groups", [(1, 0), (3, 0), (3, 1)])
@pytest.mark.parametrize("m,n,k", [(128, 128, 64), (200, 384, 136), (256, 520, 512),
                                   (384, 1152, 512)])
@pytest.mark.parametrize("tile_n,cta_pair", [(0, -1), (128, 0), (256, 0), (128, 1), (256, 1)])
def test_gemm_layouts(a_layout, b_layout, groups, sum_groups, m, n, k, tile_n, cta_pair):
    A, Bm, a_d, b_d = _operands(groups, m, n, k, a_layout, b_layout, seed=m * 7 + n + k)
    nout = 1 if sum_groups else groups
    c = [torch.empty(m, n, dtype=torch.float32, device="cuda") for _ in range(nout)]
    B.tp_gemm(groups, sum_groups, m, n, k, a_d, a_layout, b_d, b_layout, c, 1, tile_n, cta_pair)
    torch.cuda.synchronize()
    B.tp_device_status()
    refs = [f64(a) @ f64(b) for a, b in zip(A, Bm)]
    if sum_groups:
        refs = [sum(refs)]
    for i in range(nout):
        # fp32 output of exact bf16 products: only accumulation-order rounding
        assert_close(f"C[{i}]", c[i], refs[i], tol=1e-5)


@pytest.mark.parametrize("a_layout,b_layout", [(0, 1), (0, 0), (1, 1)])
def test_gemm_many_tiles_bf16_out(a_layout, b_layout):
    # 20 x 8 = 160 tiles of 128x256 > 148 SMs: some CTAs run two tiles
    m, n, k = 2560, 2048, 1024
    A, Bm, a_d, b_d = _operands(1, m, n, k, a_layout, b_layout, seed=11)
    c = [torch.empty(m, n, dtype=torch.bfloat16, device="cuda")]
    B.tp_gemm(1, 0, m, n, k, a_d, a_layout, b_d, b_layout, c, 0)
    B.tp_device_status()
    assert_close("C", c[0], f64(A[0]) @ f64(Bm[0]), tol=1e-2)


def test_gemm_partition_sum_eight_groups():
    # the row-parallel output projection pattern: 8 partitions of K = 384 summed
    m, n, k, groups = 1024, 3072, 384, 8
    A, Bm, a_d, b_d = _operands(groups, m, n, k, 0, 0, seed=5)
    c = [torch.empty(m, n, dtype=torch.float32, device="cuda")]
    B.tp_gemm(groups, 1, m, n, k, a_d, 0, b_d, 0, c, 1)
    B.tp_device_status()
    ref = sum(f64(a) @ f64(b) for a, b in zip(A, Bm))
    assert_close("C", c[0], ref, tol=1e-5)
    # the sum equals the unpartitioned product [A_0 .. A_7] [B_0; ..; B_7]
    full = f64(torch.cat(A, 1)) @ f64(torch.cat(Bm, 0))
    assert np.max(np.abs(ref - full)) <= 1e-9 * np.max(np.abs(full))


@pytest.mark.parametrize("a_layout,b_layout", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("shared", ["a", "b"])
@pytest.mark.parametrize("groups,m,n,k", [(3, 192, 384, 192), (8, 320, 1152, 128),
                                          (8, 384, 192, 256), (3, 200, 200, 72)])
@pytest.mark.parametrize("tile_n,cta_pair", [(0, -1), (128, 0), (256, 1)])
def test_gemm_shared_operand(a_layout, b_layout, shared, groups, m, n, k, tile_n, cta_pair):
    # Groups that share A (B) are tiled as one problem with the groups' N (M)
    # ranges concatenated, so tiles straddle group edges; the 200 x 200 case has
    # extents that are not multiples of 64 and keeps the per-group tiling.
    A, Bm, a_d, b_d = _operands(groups, m, n, k, a_layout, b_layout, seed=groups * 31 + m + n)
    if shared == "a":
        A, a_d = [A[0]] * groups, [a_d[0]] * groups
    else:
        Bm, b_d = [Bm[0]] * groups, [b_d[0]] * groups
    c = [torch.empty(m, n, dtype=torch.float32, device="cuda") for _ in range(groups)]
    B.tp_gemm(groups, 0, m, n, k, a_d, a_layout, b_d, b_layout, c, 1, tile_n, cta_pair)
    torch.cuda.synchronize()
    B.tp_device_status()
    for i in range(groups):
        assert_close(f"C[{i}]", c[i], f64(A[i]) @ f64(Bm[i]), tol=1e-5)


@pytest.mark.parametrize("groups,m,n,k", [(8, 256, 384, 192), (3, 200, 520, 136)])
def test_explicit_partition_sum_matches_fused(groups, m, n, k):
    # The all-reduce of a row-parallel linear two ways: summed inside the GEMM's
    # K-loop (what the layer runs), and per-partition fp32 partials followed by
    # tp_partition_sum with bias and residual.
    A, Bm, a_d, b_d = _operands(groups, m, n, k, 0, 0, seed=groups + m)
    g = torch.Generator().manual_seed(7)
    bias = torch.randn(n, generator=g).to(torch.bfloat16)
    res = torch.randn(m, n, generator=g).to(torch.bfloat16)
    parts = [torch.empty(m, n, dtype=torch.float32, device="cuda") for _ in range(groups)]
    B.tp_gemm(groups, 0, m, n, k, a_d, 0, b_d, 0, parts, 1)
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    B.tp_partition_sum(parts, out, bias.cuda(), res.cuda())
    fused = [torch.empty(m, n, dtype=torch.float32, device="cuda")]
    B.tp_gemm(groups, 1, m, n, k, a_d, 0, b_d, 0, fused, 1)
    torch.cuda.synchronize()
    B.tp_device_status()
    ref = sum(f64(a) @ f64(b) for a, b in zip(A, Bm)) + f64(bias)[None, :] + f64(res)
    assert_close("explicit", out, ref, tol=1e-2)
    assert_close("fused + epilogue", f64(fused[0]) + f64(bias)[None, :] + f64(res), ref, tol=1e-5)


@pytest.mark.parametrize("shared", ["a", "none"])
@pytest.mark.parametrize("groups,m,n,k", [(3, 320, 384, 512), (4, 200, 520, 256), (8, 256, 192, 1024)])
@pytest.mark.parametrize("c_fp32", [0, 1])
def test_gemm_stacked_group_outputs(shared, groups, m, n, k, c_fp32):
    # Group outputs stacked in one [groups][M][N] buffer: with K <= 1024 the
    # epilogue writes them by tensor stores through one map over all groups'
    # rows (row = g * M + m); M = 200 is not a multiple of 32, so a warp's rows
    # could run into the next group and the register stores are used instead.
    # The rows past each group's block must stay untouched either way.
    A, Bm, a_d, b_d = _operands(groups, m, n, k, 0, 0, seed=groups * 7 + m + k)
    if shared == "a":
        A, a_d = [A[0]] * groups, [a_d[0]] * groups
    dt = torch.float32 if c_fp32 else torch.bfloat16
    stacked = torch.full((groups + 1, m, n), 12345.0, dtype=dt, device="cuda")
    c = [stacked[i] for i in range(groups)]
    B.tp_gemm(groups, 0, m, n, k, a_d, 0, b_d, 0, c, c_fp32)
    torch.cuda.synchronize()
    B.tp_device_status()
    for i in range(groups):
        assert_close(f"C[{i}]", c[i], f64(A[i]) @ f64(Bm[i]), tol=1e-5 if c_fp32 else 1e-2)
    assert bool((stacked[groups] == 12345.0).all()), "rows past the last group were written"
