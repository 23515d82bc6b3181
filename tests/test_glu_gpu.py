"""Fused gate+up projection with the activation in the epilogue (moe_qmm_id_glu:
out = act(gate) * up, gate rows [0, n/2), up rows [n/2, n) of each expert) against
the oracle and its glu step, element by element, on every kernel that takes a
gated output: the one-token decode kernel, the generic decode kernel with routing
fused in or read from the routing prologue, and the grouped GEMM with 64-, 128-,
256-pair tiles (one expert over two); SiLU and both GELU forms; with and without an expert
bias; ragged n; rows of out-of-range ids stay zero."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import check_full_glu, check_sampled_glu, run_glu
from workloads import config_problem, make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4, expert_bias

pytestmark = pytest.mark.gpu

CASES = [
    # name, problem kwargs, path, activation, bias dtype (None: no bias)
    ("one-token", dict(fmt=FMT_AFFINE, bits=4, group_size=64, m=1, k=704, n=96, n_expert_used=8,
                       num_experts=12, x_dtype=DT_BF16, out_dtype=DT_F32), "auto", "silu", None),
    ("one-token-bias", dict(fmt=FMT_AFFINE, bits=4, group_size=32, m=1, k=512, n=200, n_expert_used=6,
                            num_experts=9, x_dtype=DT_F16, out_dtype=DT_BF16), "auto", "gelu_tanh", DT_BF16),
    ("one-token-ragged", dict(fmt=FMT_AFFINE, bits=4, group_size=64, m=1, k=256, n=38, n_expert_used=5,
                              num_experts=7, x_dtype=DT_F32, out_dtype=DT_F32), "auto", "gelu_erf", DT_F32),
    ("fused-affine4", dict(fmt=FMT_AFFINE, bits=4, group_size=32, m=4, k=448, n=200, n_expert_used=4,
                           num_experts=6, x_dtype=DT_F16, out_dtype=DT_BF16), "decode", "gelu_erf", None),
    ("fused-nvfp4", dict(fmt=FMT_NVFP4, bits=4, group_size=16, m=5, k=256, n=72, n_expert_used=3,
                         num_experts=7, x_dtype=DT_F32, out_dtype=DT_F32), "decode", "gelu_tanh", DT_F16),
    ("fused-affine6", dict(fmt=FMT_AFFINE, bits=6, group_size=64, m=3, k=320, n=54, n_expert_used=4,
                           num_experts=5, x_dtype=DT_BF16, out_dtype=DT_F16), "decode", "silu", None),
    ("routed-cb3", dict(fmt=FMT_CODEBOOK, bits=3, group_size=32, m=40, k=320, n=64, n_expert_used=4,
                        num_experts=9, x_dtype=DT_F16, out_dtype=DT_F32), "decode", "silu", DT_F32),
    ("routed-affine8", dict(fmt=FMT_AFFINE, bits=8, group_size=32, m=30, k=256, n=90, n_expert_used=3,
                            num_experts=6, x_dtype=DT_BF16, out_dtype=DT_F32), "decode", "gelu_tanh", None),
    ("grouped-64", dict(fmt=FMT_CODEBOOK, bits=3, group_size=32, m=48, k=448, n=200, n_expert_used=4,
                        num_experts=12, x_dtype=DT_F16, out_dtype=DT_F16), "grouped", "silu", DT_F16),
    ("grouped-128-f32x", dict(fmt=FMT_AFFINE, bits=4, group_size=32, m=300, k=256, n=300, n_expert_used=2,
                              num_experts=4, x_dtype=DT_F32, out_dtype=DT_F32), "grouped", "gelu_erf", None),
    ("grouped-256", dict(fmt=FMT_AFFINE, bits=6, group_size=64, m=400, k=512, n=192, n_expert_used=4,
                         num_experts=8, x_dtype=DT_BF16, out_dtype=DT_F32), "grouped", "gelu_erf", DT_BF16),
    ("grouped-256x2", dict(fmt=FMT_NVFP4, bits=4, group_size=16, m=700, k=256, n=160, n_expert_used=2,
                         num_experts=4, x_dtype=DT_BF16, out_dtype=DT_BF16), "grouped", "gelu_tanh", DT_F32),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_glu_matches_oracle(case):
    name, kw, path, act, bdt = case
    P = make_problem(name, seed=7100 + len(name), scale_range=(0.005, 0.03), **kw)
    bias = expert_bias(7200 + len(name), P.num_experts, P.n, bdt, sigma=0.3) if bdt is not None else None
    out = run_glu(P, act, path=path, bias=bias, bias_dtype=bdt if bdt is not None else DT_F32)
    torch.cuda.synchronize()
    assert out.shape == (P.m, P.n_expert_used, P.n // 2)
    nviol, ratio, info = check_full_glu(P, act, out, bias, bdt if bdt is not None else DT_F32)
    assert nviol == 0, f"{name}: {nviol} outside tolerance ({ratio:.3g}, {info})"


@pytest.mark.parametrize("act", ["silu", "gelu_tanh", "gelu_erf"])
def test_decode_gate_up_config(act):
    """The decode gate/up shape (E=128, top-8, k=2816, n=1408 = gate 704 + up 704),
    full output, one-token kernel."""
    P = config_problem("decode_gate_up")
    out = run_glu(P, act)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full_glu(P, act, out)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


def test_prefill_config_sampled():
    """The prefill shape (NVFP4, m=4096, top-8, k=4096, n=1536) as a fused gate+up
    projection on the grouped GEMM with 256-pair tiles: sampled outputs."""
    P = config_problem("prefill")
    out = run_glu(P, "silu", path="grouped")
    torch.cuda.synchronize()
    rng = np.random.default_rng(7300)
    pairs = rng.integers(0, P.R, 3000).astype(np.uint32)
    cols = rng.integers(0, P.n // 2, 3000).astype(np.uint32)
    nviol, ratio, info = check_sampled_glu(P, "silu", out, pairs, cols)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


@pytest.mark.parametrize("path", ["auto", "decode", "grouped"])
@pytest.mark.parametrize("m", [1, 30])
def test_glu_out_of_range_rows_stay_zero(path, m):
    P = make_problem("glu-bad", fmt=FMT_AFFINE, bits=4, group_size=32, m=m, k=256, n=64,
                     n_expert_used=3, num_experts=5, x_dtype=DT_BF16, out_dtype=DT_F32, seed=7400 + m)
    ids = P.ids.copy()
    ids[0, 1] = P.num_experts
    if m > 9:
        ids[9, 0] = 0xFFFFFFFF
    P = P.with_ids(ids)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    out = torch.full((P.m, P.n_expert_used, P.n // 2), float("nan"), device="cuda")
    run_glu(P, "silu", path=path, out=out, workspace=ws)
    assert M.poll_error(ws) == 5
    assert torch.all(out[0, 1] == 0)
    if m > 9:
        assert torch.all(out[9, 0] == 0)
    nviol, ratio, info = check_full_glu(P, "silu", out)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


def test_odd_n_is_rejected():
    P = make_problem("glu-odd", fmt=FMT_AFFINE, bits=4, group_size=32, m=2, k=64, n=33, n_expert_used=2,
                     num_experts=3, x_dtype=DT_F32, out_dtype=DT_F32, seed=7500)
    with pytest.raises(ValueError):
        run_glu(P, "silu")
