"""MXFP4 weights (E2M1 codes, one E8M0 scale per 32 values) against the oracle,
element by element, on the CUDA-core paths that compute them: routing fused in
(one token and several), routing read from the prologue, a gated output, an
expert bias and pointer-table weights; the grouped path reports the format as
unsupported and the automatic path falls back to the routed kernel."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import check_full, check_full_bias, check_full_glu, run, run_bias, run_glu
from workloads import make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_MXFP4, expert_bias

pytestmark = pytest.mark.gpu


def _problem(name, seed, **kw):
    base = dict(fmt=FMT_MXFP4, bits=4, group_size=32, x_dtype=DT_BF16, out_dtype=DT_F32)
    base.update(kw)
    return make_problem(name, seed=seed, **base)


@pytest.mark.parametrize("m,topk,E,k,n,xd,od,path", [
    (1, 8, 16, 2816, 96, DT_BF16, DT_F32, "auto"),     # one token, routing fused in
    (4, 4, 9, 512, 72, DT_F16, DT_BF16, "decode"),      # several tokens
    (3, 2, 5, 96, 40, DT_F32, DT_F16, "decode"),        # three 32-value blocks per row
    (40, 4, 12, 1024, 64, DT_BF16, DT_F32, "decode"),   # routed: prologue + per-expert kernel
    (300, 2, 8, 512, 48, DT_BF16, DT_F32, "auto"),      # large call: routed (no grouped MXFP4)
])
def test_mxfp4_matches_oracle(m, topk, E, k, n, xd, od, path):
    P = _problem("mxfp4", 9600 + m + k, m=m, k=k, n=n, n_expert_used=topk, num_experts=E, x_dtype=xd,
                 out_dtype=od)
    out = run(P, path)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


def test_mxfp4_grouped_path_unsupported():
    P = _problem("mxfp4-grouped", 9700, m=100, k=256, n=64, n_expert_used=2, num_experts=4)
    with pytest.raises(M.MoeError) as exc:
        run(P, "grouped")
    assert exc.value.status == 2


def test_mxfp4_gated_output_and_bias():
    P = _problem("mxfp4-glu", 9800, m=6, k=512, n=80, n_expert_used=4, num_experts=10)
    bias = expert_bias(9801, P.num_experts, P.n, DT_F32, sigma=0.3)
    out = run_glu(P, "silu", path="decode", bias=bias, bias_dtype=DT_F32)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full_glu(P, "silu", out, bias, DT_F32)
    assert nviol == 0, f"glu: {nviol} outside tolerance ({ratio:.3g}, {info})"
    out = run_bias(P, bias, DT_F32, path="decode")
    torch.cuda.synchronize()
    nviol, ratio, info = check_full_bias(P, out, bias, DT_F32)
    assert nviol == 0, f"bias: {nviol} outside tolerance ({ratio:.3g}, {info})"


def test_mxfp4_pointer_tables():
    P = _problem("mxfp4-ptrs", 9900, m=5, k=256, n=40, n_expert_used=3, num_experts=6)
    packed = [torch.from_numpy(np.ascontiguousarray(P.packed[e])).cuda() for e in range(P.num_experts)]
    scales = [torch.from_numpy(np.ascontiguousarray(P.scales[e])).cuda() for e in range(P.num_experts)]
    pp = torch.tensor([t.data_ptr() for t in packed], dtype=torch.int64, device="cuda")
    sp = torch.tensor([t.data_ptr() for t in scales], dtype=torch.int64, device="cuda")
    from workloads.torch_io import to_device
    dev = to_device(P)
    out = torch.empty((P.m, P.n_expert_used, P.n), device="cuda")
    M.qmm_id_ptrs(dev["x"], dev["ids"], pp, sp, None, None, n=P.n, group_size=32, bits=4, fmt=FMT_MXFP4,
                  num_experts=P.num_experts, out=out, path="decode")
    torch.cuda.synchronize()
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"ptrs: {nviol} outside tolerance ({ratio:.3g}, {info})"
