"""W4A4 (NVFP4 activations) on the GPU against the oracle.

- The quantisation kernel against the oracle's, bit for bit: E4M3 block scales,
  per-token scales, E2M1 codes (the sign of a zero code is not compared: +0 and
  -0 are the same value) and x^ (the exact product rounded once to f32), for f32,
  bf16 and f16 x, with zero tokens and blocks, a dominant value whose neighbours'
  scales underflow, and magnitudes spread over many binades.
- moe_qmm_id_w4a4 element by element against the oracle on x^ (the operation's
  tolerance) on the one-token decode kernel, the several-token decode path, the
  routed path and the grouped GEMM (16- and 256-pair tiles), with NVFP4 and affine
  weights, and the workspace check.
- The block-scaled MMA (NVFP4 weights, k a multiple of 256): against the oracle,
  and against the bf16-operand GEMM (forced through moe_qmm_test_x_copies), with
  partial tiles, a ragged last row block, bf16 output and out-of-range ids.
"""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
import oracle
from tests.gpu_util import check_full
from workloads import make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_NVFP4, bf16_bits
from workloads.torch_io import to_device

pytestmark = pytest.mark.gpu


def _x(rng, m, k, xd):
    xf = (rng.standard_normal((m, k)) * np.exp(rng.uniform(-8, 8, (m, 1)))).astype(np.float32)
    xf[1 % m, 16:48] = 0.0
    if m > 3:
        xf[3] = 0.0
        xf[2] = rng.standard_normal(k).astype(np.float32) * 1e-2
        xf[2, 5] = 300.0  # 3e4 times the rest: other blocks' scales underflow
    if xd == DT_F32:
        return xf
    if xd == DT_BF16:
        return bf16_bits(xf)
    return xf.astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("xd", [DT_F32, DT_BF16, DT_F16])
@pytest.mark.parametrize("m,k,offset", [(1, 2816, 0), (7, 512, 0), (64, 4096, 0), (5, 256, 1)])
def test_quantize_matches_oracle(xd, m, k, offset):
    rng = np.random.default_rng(1000 + m + k + xd)
    xb = _x(rng, m, k, xd)
    dt = {DT_F32: torch.float32, DT_BF16: torch.bfloat16, DT_F16: torch.float16}[xd]
    xt = torch.from_numpy(xb.view(np.float32) if xd == DT_F32 else xb.view(np.int16)).view(dt).cuda()
    if offset:
        # x one element off a 16-byte boundary: the kernel's element-wise loads
        big = torch.zeros(m * k + offset, dtype=dt, device="cuda")
        big[offset:] = xt.reshape(-1)
        xt = big[offset:].view(m, k)
        assert xt.data_ptr() % 16 != 0
    codes, scales, g, xhat = M.quantize_act_nvfp4(xt)
    torch.cuda.synchronize()
    o_codes, o_scales, o_g, o_xhat = oracle.quantize_act_nvfp4(xb, xd, m, k)
    np.testing.assert_array_equal(g.cpu().numpy().view(np.uint32), o_g.view(np.uint32))
    np.testing.assert_array_equal(scales.cpu().numpy(), o_scales)
    gc = codes.cpu().numpy()
    q = np.stack([gc & 15, gc >> 4], axis=2).reshape(m, k)
    oq = np.stack([o_codes & 15, o_codes >> 4], axis=2).reshape(m, k)
    np.testing.assert_array_equal(q & 7, oq & 7)
    nz = (oq & 7) != 0
    np.testing.assert_array_equal((q >> 3)[nz], (oq >> 3)[nz])
    np.testing.assert_array_equal(xhat.cpu().numpy(), o_xhat.astype(np.float32))


@pytest.mark.parametrize("name,fmt,bits,gs,m,topk,E,k,n,xd,od,path", [
    ("one-token", FMT_NVFP4, 4, 16, 1, 8, 16, 1024, 96, DT_BF16, DT_F32, "auto"),
    ("decode", FMT_NVFP4, 4, 16, 5, 4, 9, 512, 72, DT_F16, DT_BF16, "decode"),
    ("routed", FMT_NVFP4, 4, 16, 40, 4, 12, 1024, 64, DT_BF16, DT_F32, "decode"),
    ("grouped-64", FMT_NVFP4, 4, 16, 100, 2, 4, 256, 64, DT_BF16, DT_F32, "grouped"),
    ("grouped-256", FMT_NVFP4, 4, 16, 1200, 2, 8, 384, 136, DT_F32, DT_BF16, "grouped"),
    ("affine-auto", FMT_AFFINE, 4, 64, 300, 2, 8, 512, 48, DT_BF16, DT_F32, "auto"),
])
def test_w4a4_matches_oracle(name, fmt, bits, gs, m, topk, E, k, n, xd, od, path):
    P = make_problem(f"w4a4-{name}", seed=6100 + m + k, fmt=fmt, bits=bits, group_size=gs, m=m, k=k, n=n,
                     n_expert_used=topk, num_experts=E, x_dtype=xd, out_dtype=od)
    d = to_device(P)
    out = M.qmm_id_w4a4(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], n=P.n, group_size=P.group_size,
                        bits=P.bits, fmt=P.fmt, num_experts=P.num_experts,
                        out_dtype={DT_F32: torch.float32, DT_BF16: torch.bfloat16}[od], path=path)
    torch.cuda.synchronize()
    Q = oracle.w4a4_problem(P)
    nviol, ratio, info = check_full(Q, out)
    assert nviol == 0, f"{name}: {nviol} outside tolerance ({ratio:.3g}, {info})"


def test_w4a4_workspace_check():
    P = make_problem("w4a4-ws", seed=6200, fmt=FMT_NVFP4, bits=4, group_size=16, m=4, k=256, n=32,
                     n_expert_used=2, num_experts=4, x_dtype=DT_BF16, out_dtype=DT_F32)
    d = to_device(P)
    small = torch.zeros(M.workspace_bytes(P.m, 2, 4), dtype=torch.uint8, device="cuda")
    with pytest.raises(M.MoeError) as exc:
        M.qmm_id_w4a4(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], n=P.n, group_size=16, bits=4,
                      fmt=FMT_NVFP4, num_experts=4, workspace=small)
    assert exc.value.status == 3


@pytest.mark.parametrize("m,topk,E,k,n,od", [
    (600, 2, 8, 1024, 200, DT_BF16),   # 150 pairs per expert: a full and a partial 128-pair tile
    (90, 4, 6, 512, 128, DT_F32),      # 60 pairs per expert
    (2000, 8, 16, 2048, 384, DT_BF16), # 1000 pairs per expert, several k-tiles of 256
])
def test_w4a4_block_scaled_mma(m, topk, E, k, n, od):
    P = make_problem("w4a4-mma", seed=6300 + m + k, fmt=FMT_NVFP4, bits=4, group_size=16, m=m, k=k, n=n,
                     n_expert_used=topk, num_experts=E, x_dtype=DT_BF16, out_dtype=od)
    ids = P.ids.copy()
    ids[1, 0] = P.num_experts          # an out-of-range id: zero row and the error word
    P = P.with_ids(ids)
    d = to_device(P)
    odt = {DT_F32: torch.float32, DT_BF16: torch.bfloat16}[od]
    ws = torch.zeros(M.workspace_bytes_w4a4(P.m, P.k, P.n_expert_used, P.num_experts), dtype=torch.uint8,
                     device="cuda")
    kw = dict(n=P.n, group_size=16, bits=4, fmt=FMT_NVFP4, num_experts=P.num_experts, out_dtype=odt, path="grouped")
    out = M.qmm_id_w4a4(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], workspace=ws, **kw)
    torch.cuda.synchronize()
    assert M.poll_error(ws) == 5     # the error word at the start, as for moe_qmm_id
    Q = oracle.w4a4_problem(P)
    nviol, ratio, info = check_full(Q, out)
    assert nviol == 0, f"block-scaled: {nviol} outside tolerance ({ratio:.3g}, {info})"
    L = M.lib()
    assert L.moe_qmm_test_x_copies(1) == 0
    try:
        ref = M.qmm_id_w4a4(d["x"], d["ids"], d["packed"], d["scales"], d["aux"], **kw)
    finally:
        assert L.moe_qmm_test_x_copies(0) == 0
    torch.cuda.synchronize()
    nviol, ratio, info = check_full(Q, ref)
    assert nviol == 0, f"bf16 operand: {nviol} outside tolerance ({ratio:.3g}, {info})"
