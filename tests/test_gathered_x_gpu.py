"""The grouped GEMM's ways of bringing x rows into the B operand tiles. For f32 x,
tensor copies of the rows gathered into expert order and split into bf16 halves
once after routing (a workspace sized by moe_qmm_id_workspace_bytes_k) and the
loader warps' 16-byte copies, which split f32 x per tile (the minimum workspace,
or forced through moe_qmm_test_x_copies), give the same bits. For 16-bit x the
k-aware workspace holds the tile-major f16 image of the B operand (bf16 x scaled
per token by a power of two), read with one bulk copy per k-tile, and the
minimum workspace or the hook keeps the loader copies; the two compute in f16
and bf16 respectively, so each is checked against the oracle. Every output is
checked element by element against the oracle. Cases span every weight format,
bf16 / f16 / f32 x, 64- and 256-pair tiles, partial tiles, a ragged last k-tile,
a ragged last row block, out-of-range ids, a gated output and an expert bias."""

import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import check_full, check_full_bias, check_full_glu, run, run_bias, run_glu
from workloads import make_problem
from workloads.gen import (DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_MXFP4, FMT_NVFP4,
                           expert_bias)
from workloads.torch_io import to_device

pytestmark = pytest.mark.gpu


def _ways(P, runner, **kw):
    """Outputs of the default x tiles (k-aware workspace), of the minimum workspace
    and of forced loader copies with the k-aware workspace; and that workspace."""
    dev = to_device(P)
    ws_k = M.new_workspace(P.m, P.n_expert_used, P.num_experts, k=P.k, x_dtype=dev["x"].dtype)
    ws_m = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    outs = [runner(P, path="grouped", dev=dev, workspace=ws_k, **kw),
            runner(P, path="grouped", dev=dev, workspace=ws_m, **kw)]
    L = M.lib()
    assert L.moe_qmm_test_x_copies(1) == 0
    try:
        outs.append(runner(P, path="grouped", dev=dev, workspace=ws_k, **kw))
    finally:
        assert L.moe_qmm_test_x_copies(0) == 0
    torch.cuda.synchronize()
    return outs, ws_k


def _same_bits(outs, P=None, check=None):
    """f32 x: every way gives the default's bits. 16-bit x: each way within the
    oracle's tolerance (check(P, out) -> (violations, ratio, info))."""
    if P is not None and P.x_dtype != DT_F32:
        for i, o in enumerate(outs):
            nviol, ratio, info = check(P, o)
            assert nviol == 0, f"x-tile way {i}: {nviol} outside tolerance ({ratio:.3g}, {info})"
        return
    ref = outs[0].view(torch.uint8)
    for i, o in enumerate(outs[1:], 1):
        assert torch.equal(ref, o.view(torch.uint8)), f"x-tile way {i} differs from the default"


CASES = [
    # fmt, bits, gs, xd, od, m, topk, E, k, n
    (FMT_AFFINE, 4, 64, DT_BF16, DT_F32, 120, 4, 8, 2048, 192),    # 64-pair tiles, partial tiles
    (FMT_AFFINE, 4, 32, DT_F16, DT_BF16, 900, 2, 6, 320, 136),     # 256-pair tiles, ragged k-tile and row block
    (FMT_AFFINE, 8, 64, DT_F32, DT_F32, 200, 2, 4, 448, 128),      # f32 x: gathered halves vs per-tile split
    (FMT_AFFINE, 6, 64, DT_BF16, DT_BF16, 300, 2, 5, 384, 64),
    (FMT_CODEBOOK, 4, 32, DT_BF16, DT_F32, 700, 2, 4, 512, 96),
    (FMT_CODEBOOK, 3, 32, DT_F16, DT_F32, 500, 2, 5, 256, 128),
    (FMT_NVFP4, 4, 16, DT_BF16, DT_F32, 640, 2, 4, 1024, 256),
    (FMT_NVFP4, 4, 16, DT_F32, DT_BF16, 150, 4, 6, 192, 80),
    (FMT_MXFP4, 4, 32, DT_BF16, DT_F32, 1100, 2, 8, 384, 136),
    (FMT_AFFINE, 4, 64, DT_F32, DT_F32, 3, 1, 2, 512, 128),        # a 3-pair tile of gathered f32 rows
    (FMT_NVFP4, 4, 16, DT_F32, DT_F32, 700, 2, 4, 512, 128),       # 128-pair tiles of gathered f32 rows
]


@pytest.mark.parametrize("fmt,bits,gs,xd,od,m,topk,E,k,n", CASES)
def test_x_tile_ways_bit_identical_and_match_oracle(fmt, bits, gs, xd, od, m, topk, E, k, n):
    P = make_problem("x-tiles", seed=8800 + m + k + n, fmt=fmt, bits=bits, group_size=gs, x_dtype=xd,
                     out_dtype=od, m=m, k=k, n=n, n_expert_used=topk, num_experts=E)
    outs, ws = _ways(P, run)
    assert M.poll_error(ws) == 0
    _same_bits(outs, P, check_full)
    nviol, ratio, info = check_full(P, outs[0])
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


def test_x_tiles_out_of_range_ids():
    P = make_problem("x-tiles-bad", seed=8900, fmt=FMT_AFFINE, bits=4, group_size=64, x_dtype=DT_BF16,
                     out_dtype=DT_F32, m=400, k=512, n=128, n_expert_used=2, num_experts=4)
    ids = P.ids.copy()
    ids[3, 1] = P.num_experts
    ids[399, 0] = 0xFFFFFFFF
    P = P.with_ids(ids)
    outs, ws = _ways(P, run)
    assert M.poll_error(ws) == 5
    _same_bits(outs, P, check_full)
    nviol, ratio, info = check_full(P, outs[0])
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


@pytest.mark.parametrize("xd", [DT_BF16, DT_F32])
def test_x_tiles_gated_and_bias(xd):
    P = make_problem("x-tiles-glu", seed=8950, fmt=FMT_AFFINE, bits=4, group_size=64, x_dtype=xd,
                     out_dtype=DT_F32, m=600, k=768, n=256, n_expert_used=2, num_experts=4)
    outs, _ = _ways(P, run_glu, act="silu")
    _same_bits(outs, P, lambda P, o: check_full_glu(P, "silu", o))
    nviol, ratio, info = check_full_glu(P, "silu", outs[0])
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"
    bias = expert_bias(8951, P.num_experts, P.n, DT_F32)
    outs, _ = _ways(P, lambda P, **kw: run_bias(P, bias, DT_F32, **kw))
    _same_bits(outs, P, lambda P, o: check_full_bias(P, o, bias, DT_F32))
    nviol, ratio, info = check_full_bias(P, outs[0], bias, DT_F32)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"
