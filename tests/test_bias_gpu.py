"""Per-expert output bias (moe_qmm_id_bias) against the oracle plus its bias
step, element by element, on every kernel path: the one-token decode kernel,
the TMA-staged and generic decode kernels with routing fused in, the routed
decode kernel, and the grouped GEMM with 64- and 256-pair tiles (one expert over two); bias in
f32, bf16 and f16; rows of out-of-range ids stay zero."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import check_full_bias, run_bias, to_device
from workloads import config_problem, make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4, expert_bias

pytestmark = pytest.mark.gpu

CASES = [
    # name, problem kwargs, path, bias dtype
    ("one-token", dict(fmt=FMT_AFFINE, bits=4, group_size=64, m=1, k=704, n=96, n_expert_used=8,
                       num_experts=12, x_dtype=DT_BF16, out_dtype=DT_F32), "auto", DT_F32),
    ("fused-tma", dict(fmt=FMT_AFFINE, bits=4, group_size=32, m=4, k=448, n=200, n_expert_used=4,
                       num_experts=6, x_dtype=DT_F16, out_dtype=DT_BF16), "decode", DT_BF16),
    ("fused-generic", dict(fmt=FMT_NVFP4, bits=4, group_size=16, m=5, k=256, n=72, n_expert_used=3,
                           num_experts=7, x_dtype=DT_F32, out_dtype=DT_F32), "decode", DT_F16),
    ("routed-gemv", dict(fmt=FMT_CODEBOOK, bits=3, group_size=32, m=40, k=320, n=64, n_expert_used=4,
                         num_experts=9, x_dtype=DT_F16, out_dtype=DT_F32), "decode", DT_F32),
    ("grouped-64", dict(fmt=FMT_CODEBOOK, bits=3, group_size=32, m=48, k=448, n=200, n_expert_used=4,
                        num_experts=12, x_dtype=DT_F16, out_dtype=DT_F16), "grouped", DT_F16),
    ("grouped-256", dict(fmt=FMT_AFFINE, bits=6, group_size=64, m=400, k=512, n=192, n_expert_used=4,
                         num_experts=8, x_dtype=DT_BF16, out_dtype=DT_F32), "grouped", DT_BF16),
    ("grouped-256x2", dict(fmt=FMT_NVFP4, bits=4, group_size=16, m=700, k=256, n=160, n_expert_used=2,
                         num_experts=4, x_dtype=DT_BF16, out_dtype=DT_BF16), "grouped", DT_F32),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_bias_matches_oracle(case):
    name, kw, path, bdt = case
    P = make_problem(name, seed=6100 + len(name), scale_range=(0.005, 0.03), **kw)
    bias = expert_bias(6200 + len(name), P.num_experts, P.n, bdt)
    out = run_bias(P, bias, bdt, path=path)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full_bias(P, out, bias, bdt)
    assert nviol == 0, f"{name}: {nviol} outside tolerance ({ratio:.3g}, {info})"


@pytest.mark.parametrize("path", ["auto", "decode", "grouped"])
def test_bias_out_of_range_rows_stay_zero(path):
    P = make_problem("bias-bad", fmt=FMT_AFFINE, bits=4, group_size=32, m=30, k=256, n=64,
                     n_expert_used=3, num_experts=5, x_dtype=DT_BF16, out_dtype=DT_F32, seed=6300)
    ids = P.ids.copy()
    ids[3, 1] = P.num_experts
    ids[9, 0] = 0xFFFFFFFF
    P = P.with_ids(ids)
    bias = expert_bias(6301, P.num_experts, P.n, DT_F32)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    out = torch.full((P.m, P.n_expert_used, P.n), float("nan"), device="cuda")
    run_bias(P, bias, DT_F32, path=path, out=out, workspace=ws)
    assert M.poll_error(ws) == 5
    assert torch.all(out[3, 1] == 0) and torch.all(out[9, 0] == 0)
    nviol, ratio, info = check_full_bias(P, out, bias, DT_F32)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


def test_decode_config_with_bias():
    P = config_problem("decode_gate_up")
    bias = expert_bias(6400, P.num_experts, P.n, DT_BF16)
    out = run_bias(P, bias, DT_BF16)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full_bias(P, out, bias, DT_BF16)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"
