"""Failure detection on the GPU without a fault: the test hook
moe_qmm_test_inject_wait_timeout makes one bounded wait per CTA wait on a
barrier that nothing completes, with a 2 ms limit. The kernel must give up,
let its own copies and MMAs in flight complete (their waits keep the full 1 s
limit), free its tensor memory and exit; moe_qmm_id_poll_error must report
MOE_ERR_TIMEOUT; and the next, normal call on the same stream and workspace
must match the oracle."""

import ctypes

import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import check_full, run, to_device
from workloads import config_problem, make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = 6


def inject(limit_ns: int):
    fn = M.lib().moe_qmm_test_inject_wait_timeout
    fn.argtypes = [ctypes.c_uint64]
    fn.restype = ctypes.c_int
    assert fn(limit_ns) == M.MOE_OK


def problems():
    yield "grouped", make_problem("timeout-nvfp4", fmt=FMT_NVFP4, bits=4, group_size=16, m=96, k=512,
                                  n=320, n_expert_used=4, num_experts=8, x_dtype=DT_BF16,
                                  out_dtype=DT_BF16, seed=61)
    yield "grouped", make_problem("timeout-codebook", fmt=FMT_CODEBOOK, bits=3, group_size=32, m=64,
                                  k=320, n=256, n_expert_used=2, num_experts=4, x_dtype=DT_F16,
                                  out_dtype=DT_F32, seed=62, scale_range=(0.01, 0.05))
    yield "auto", config_problem("decode_gate_up")  # the one-token decode kernel
    # 256-pair tiles
    yield "grouped", make_problem("timeout-pair", fmt=FMT_AFFINE, bits=4, group_size=64, m=512, k=512,
                                  n=384, n_expert_used=2, num_experts=8, x_dtype=DT_BF16,
                                  out_dtype=DT_F32, seed=63)


@pytest.mark.parametrize("case", list(range(4)))
def test_wait_timeout_is_reported_and_the_next_call_is_exact(case):
    path, P = list(problems())[case]
    dev = to_device(P)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    assert M.poll_error(ws) == M.MOE_OK
    inject(2_000_000)
    try:
        run(P, path, dev=dev, workspace=ws)
        torch.cuda.synchronize()
    finally:
        inject(0)
    assert M.poll_error(ws) == MOE_ERR_TIMEOUT
    assert M.poll_error(ws) == M.MOE_OK  # read and cleared
    out = run(P, path, dev=dev, workspace=ws)
    assert M.poll_error(ws) == M.MOE_OK
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"{P.name}: {nviol} outside tolerance ({ratio:.3g}, {info})"
