"""moe_qmm_plan (moe_expert_routed_b200.Plan): a projection bound once and run on
new x / ids gives the oracle's results on every path, with an expert bias and a
gated output, and with the one-token kernel's launch flags; a plan keeps working
across calls with different ids and x."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import TORCH_OUT, bias_tensor, check_full, check_full_bias, check_full_glu
from workloads import config_problem, make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4, expert_bias
from workloads.torch_io import to_device

pytestmark = pytest.mark.gpu

_XT = {DT_F32: torch.float32, DT_BF16: torch.bfloat16, DT_F16: torch.float16}


def _plan(P, dev, **kw):
    return M.Plan(dev["packed"], dev["scales"], dev["aux"], m=P.m, k=P.k, n=P.n, group_size=P.group_size,
                  bits=P.bits, fmt=P.fmt, n_expert_used=P.n_expert_used, num_experts=P.num_experts,
                  x_dtype=_XT[P.x_dtype], out_dtype=TORCH_OUT[P.out_dtype], **kw)


@pytest.mark.parametrize("name,kw,path", [
    ("one-token", dict(fmt=FMT_AFFINE, bits=4, group_size=64, m=1, k=704, n=96, n_expert_used=8,
                       num_experts=12, x_dtype=DT_BF16, out_dtype=DT_F32), "auto"),
    ("fused", dict(fmt=FMT_NVFP4, bits=4, group_size=16, m=5, k=256, n=72, n_expert_used=3,
                   num_experts=7, x_dtype=DT_F32, out_dtype=DT_F32), "decode"),
    ("grouped", dict(fmt=FMT_CODEBOOK, bits=3, group_size=32, m=48, k=448, n=200, n_expert_used=4,
                     num_experts=12, x_dtype=DT_F16, out_dtype=DT_F16), "grouped"),
])
def test_plan_matches_oracle_across_calls(name, kw, path):
    P = make_problem(name, seed=8100 + len(name), scale_range=(0.005, 0.03), **kw)
    dev = to_device(P)
    plan = _plan(P, dev, path=path)
    out = torch.empty(plan.shape, dtype=TORCH_OUT[P.out_dtype], device="cuda")
    rng = np.random.default_rng(8200)
    for _ in range(3):
        plan(dev["x"], dev["ids"], out)
        torch.cuda.synchronize()
        nviol, ratio, info = check_full(P, out)
        assert nviol == 0, f"{name}: {nviol} outside tolerance ({ratio:.3g}, {info})"
        # new ids and x for the next call through the same plan
        ids = np.stack([rng.permutation(P.num_experts)[:P.n_expert_used] for _ in range(P.m)]).astype(np.uint32)
        P = P.with_ids(ids).with_x(P.x[rng.permutation(P.m)])
        dev = dict(dev, **{k: v for k, v in to_device(P).items() if k in ("x", "ids")})


def test_plan_bias_and_gated_output():
    P = make_problem("plan-glu", fmt=FMT_AFFINE, bits=6, group_size=64, m=400, k=512, n=192,
                     n_expert_used=4, num_experts=8, x_dtype=DT_BF16, out_dtype=DT_F32, seed=8300,
                     scale_range=(0.005, 0.03))
    dev = to_device(P)
    bias = expert_bias(8301, P.num_experts, P.n, DT_BF16, sigma=0.3)
    bt = bias_tensor(bias, DT_BF16)
    plan = _plan(P, dev, expert_bias=bt)
    out = torch.empty(plan.shape, device="cuda")
    plan(dev["x"], dev["ids"], out)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full_bias(P, out, bias, DT_BF16)
    assert nviol == 0, f"bias: {nviol} outside tolerance ({ratio:.3g}, {info})"
    gplan = _plan(P, dev, expert_bias=bt, act="gelu_tanh")
    gout = torch.empty(gplan.shape, device="cuda")
    assert gplan.shape == (P.m, P.n_expert_used, P.n // 2)
    gplan(dev["x"], dev["ids"], gout)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full_glu(P, "gelu_tanh", gout, bias, DT_BF16)
    assert nviol == 0, f"glu: {nviol} outside tolerance ({ratio:.3g}, {info})"


def test_plan_decode_step_with_launch_flags():
    Ps = [config_problem("decode_gate_up"), config_problem("decode_down")]
    devs = [to_device(P) for P in Ps]
    plans = [_plan(Ps[0], devs[0], launch="pdl"), _plan(Ps[1], devs[1], launch="early_weights")]
    outs = [torch.full(p.shape, float("nan"), device="cuda") for p in plans]
    st = torch.cuda.current_stream()
    for _ in range(5):
        for i in range(2):
            plans[i](devs[i]["x"], devs[i]["ids"], outs[i], st)
    torch.cuda.synchronize()
    for i, P in enumerate(Ps):
        nviol, ratio, info = check_full(P, outs[i])
        assert nviol == 0, f"{P.name}: {nviol} outside tolerance ({ratio:.3g}, {info})"
