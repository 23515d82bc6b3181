"""MXFP4 weights (E2M1 codes, one E8M0 scale per 32 values) against the oracle,
element by element: on the CUDA-core paths (routing fused in for one token and
several, routing read from the prologue, a gated output, an expert bias and
pointer-table weights) and on the tcgen05 grouped GEMM with bf16 and f32 x
(single-term A: e2m1 * 2^e is exact in bf16), in 64-pair and 256-pair tiles,
with a ragged last row block, a gated output, a bias and pointer tables. With
f16 x the grouped path reports the format as unsupported (e2m1 * 2^e can leave
the f16 range) and the automatic path uses the routed CUDA-core kernel."""

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
    (300, 2, 8, 512, 48, DT_F16, DT_F32, "auto"),       # large call, f16 x: routed CUDA-core kernel
])
def test_mxfp4_matches_oracle(m, topk, E, k, n, xd, od, path):
    P = _problem("mxfp4", 9600 + m + k, m=m, k=k, n=n, n_expert_used=topk, num_experts=E, x_dtype=xd,
                 out_dtype=od)
    out = run(P, path)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


def test_mxfp4_grouped_path_f16_x_unsupported():
    P = _problem("mxfp4-grouped", 9700, m=100, k=256, n=64, n_expert_used=2, num_experts=4, x_dtype=DT_F16)
    with pytest.raises(M.MoeError) as exc:
        run(P, "grouped")
    assert exc.value.status == 2


@pytest.mark.parametrize("m,topk,E,k,n,xd,od", [
    (100, 2, 4, 256, 64, DT_BF16, DT_F32),      # 64-pair tiles
    (60, 4, 6, 512, 200, DT_BF16, DT_BF16),     # ragged last 128-row block
    (1200, 2, 8, 384, 136, DT_BF16, DT_BF16),   # ~300 pairs per expert: 256-pair tiles and a second tile
    (90, 2, 5, 320, 96, DT_F32, DT_F32),        # f32 x as two bf16 halves
])
def test_mxfp4_grouped_matches_oracle(m, topk, E, k, n, xd, od):
    P = _problem("mxfp4-gemm", 9750 + m + n, m=m, k=k, n=n, n_expert_used=topk, num_experts=E, x_dtype=xd,
                 out_dtype=od)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    out = run(P, "grouped", workspace=ws)
    assert M.poll_error(ws) == 0
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


def test_mxfp4_grouped_gated_bias_and_pointer_tables():
    P = _problem("mxfp4-gemm-glu", 9760, m=80, k=256, n=144, n_expert_used=2, num_experts=4)
    bias = expert_bias(9761, P.num_experts, P.n, DT_F32, sigma=0.3)
    out = run_glu(P, "gelu_tanh", path="grouped", bias=bias, bias_dtype=DT_F32)
    torch.cuda.synchronize()
    nviol, ratio, info = check_full_glu(P, "gelu_tanh", out, bias, DT_F32)
    assert nviol == 0, f"glu: {nviol} outside tolerance ({ratio:.3g}, {info})"
    packed = [torch.from_numpy(np.ascontiguousarray(P.packed[e])).cuda() for e in range(P.num_experts)]
    scales = [torch.from_numpy(np.ascontiguousarray(P.scales[e])).cuda() for e in range(P.num_experts)]
    pp = torch.tensor([t.data_ptr() for t in packed], dtype=torch.int64, device="cuda")
    sp = torch.tensor([t.data_ptr() for t in scales], dtype=torch.int64, device="cuda")
    from workloads.torch_io import to_device
    dev = to_device(P)
    out = torch.empty((P.m, P.n_expert_used, P.n), device="cuda")
    M.qmm_id_ptrs(dev["x"], dev["ids"], pp, sp, None, None, n=P.n, group_size=32, bits=4, fmt=FMT_MXFP4,
                  num_experts=P.num_experts, out=out, path="grouped")
    torch.cuda.synchronize()
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"ptrs: {nviol} outside tolerance ({ratio:.3g}, {info})"


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
