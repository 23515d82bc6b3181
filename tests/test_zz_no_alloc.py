"""moe_qmm_id_noalloc, the entry point for callers that cannot allocate device
memory (its routing scratch is a fixed array inside the library).

Each case is computed once through moe_qmm_id with its own workspace, then twice
in a row through moe_qmm_id_noalloc (the second call finds the first call's
contents in the shared scratch), and both results are compared with the first
under the per-element tolerance the parity tests use, and with the CPU oracle.
Cases run one after the other, so later ones also start from an earlier,
differently sized call's leftovers. Further checks: the calls change neither
torch's allocated bytes nor the device's free memory, and out-of-range ids are
reported through moe_qmm_id_noalloc_poll_error."""

import ctypes

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import TORCH_OUT, check_full, compare, out_to_f64, run, to_device
from workloads import config_problem, make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4

pytestmark = pytest.mark.gpu


def noalloc_fn():
    fn = M.lib().moe_qmm_id_noalloc
    u32 = ctypes.c_uint32
    fn.argtypes = [ctypes.c_void_p] * 6 + [u32] * 5 + [ctypes.c_int, u32, u32, ctypes.c_int,
                                                      ctypes.c_int, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def poll_fn():
    fn = M.lib().moe_qmm_id_noalloc_poll_error
    fn.argtypes = [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def call_noalloc(P, dev, out):
    return noalloc_fn()(dev["x"].data_ptr(), dev["ids"].data_ptr(), dev["packed"].data_ptr(),
                        dev["scales"].data_ptr(), dev["aux"].data_ptr(), out.data_ptr(), P.m, P.k,
                        P.n, P.group_size, P.bits, P.fmt, P.n_expert_used, P.num_experts, P.x_dtype,
                        P.out_dtype, torch.cuda.current_stream().cuda_stream)


def cases():
    yield make_problem("grouped-codebook", fmt=FMT_CODEBOOK, bits=3, group_size=32, m=48, k=448,
                       n=200, n_expert_used=4, num_experts=12, x_dtype=DT_F16, out_dtype=DT_F32,
                       seed=41, scale_range=(0.01, 0.05))
    yield config_problem("decode_gate_up")
    yield make_problem("grouped-nvfp4-zipf", fmt=FMT_NVFP4, bits=4, group_size=16, m=900, k=256,
                       n=160, n_expert_used=2, num_experts=8, x_dtype=DT_BF16, out_dtype=DT_BF16,
                       seed=42, ids="zipf", zipf_s=1.5)
    yield make_problem("grouped-affine6", fmt=FMT_AFFINE, bits=6, group_size=64, m=64, k=512,
                       n=256, n_expert_used=8, num_experts=16, x_dtype=DT_F32, out_dtype=DT_F32,
                       seed=43, ids="zipf")


def test_noalloc_matches_moe_qmm_id_two_calls_in_a_row():
    for P in cases():
        dev = to_device(P)
        ref = run(P, "auto", dev=dev)
        torch.cuda.synchronize()
        ref64 = out_to_f64(ref)
        pairs = np.repeat(np.arange(P.R), P.n)
        cols = np.tile(np.arange(P.n), P.R)
        for call in range(2):
            out = torch.full((P.m, P.n_expert_used, P.n), float("nan"),
                             dtype=TORCH_OUT[P.out_dtype], device="cuda")
            assert call_noalloc(P, dev, out) == M.MOE_OK, P.name
            torch.cuda.synchronize()
            nviol, ratio, info = compare(P, out_to_f64(out).reshape(-1), ref64.reshape(-1), pairs,
                                         cols)
            assert nviol == 0, f"{P.name} call {call}: {nviol} outside tolerance ({ratio:.3g}, {info})"
            nviol, ratio, info = check_full(P, out)
            assert nviol == 0, f"{P.name} call {call} vs oracle: {nviol} outside tolerance ({ratio:.3g}, {info})"
        assert poll_fn()(torch.cuda.current_stream().cuda_stream) == M.MOE_OK, P.name


def test_noalloc_allocates_nothing():
    # warm up (module and kernels loaded, scratch address looked up), then the same
    # calls again with every tensor already allocated: neither torch's allocator nor
    # the device's free memory may move
    probs = list(cases())
    devs = [to_device(P) for P in probs]
    outs = [torch.empty((P.m, P.n_expert_used, P.n), dtype=TORCH_OUT[P.out_dtype], device="cuda")
            for P in probs]
    for P, dev, out in zip(probs, devs, outs):
        assert call_noalloc(P, dev, out) == M.MOE_OK
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        for P, dev, out in zip(probs, devs, outs):
            assert call_noalloc(P, dev, out) == M.MOE_OK
    assert poll_fn()(torch.cuda.current_stream().cuda_stream) == M.MOE_OK
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_reports_out_of_range_ids():
    P = make_problem("noalloc-bad-id", fmt=FMT_AFFINE, bits=4, group_size=32, m=40, k=256, n=96,
                     n_expert_used=2, num_experts=8, x_dtype=DT_BF16, out_dtype=DT_F32, seed=44)
    ids = P.ids.copy()
    ids[3, 1] = P.num_experts + 5
    P = P.with_ids(ids)
    dev = to_device(P)
    poll = poll_fn()
    st = torch.cuda.current_stream().cuda_stream
    assert poll(st) == M.MOE_OK  # leaves a clear error word
    out = torch.full((P.m, P.n_expert_used, P.n), 7.0, dtype=torch.float32, device="cuda")
    assert call_noalloc(P, dev, out) == M.MOE_OK
    assert poll(st) == 5  # MOE_ERR_BAD_EXPERT_ID
    assert poll(st) == M.MOE_OK  # read and cleared
    assert torch.count_nonzero(out[3, 1]).item() == 0
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 250,000 routings over 256 experts need more than MOE_NOALLOC_SCRATCH_BYTES of scratch
    assert M.workspace_bytes(31250, 8, 256) > (1 << 20)
    fn = noalloc_fn()
    st = fn(16, 16, 16, 16, 16, 16, 31250, 2816, 1408, 64, 4, 0, 8, 256, 1, 0, None)
    assert st == 3  # MOE_ERR_WORKSPACE_TOO_SMALL, before any CUDA work
    st = fn(16, 16, 16, 16, 16, 16, 0, 2816, 1408, 64, 4, 0, 8, 256, 1, 0, None)
    assert st == 1  # invalid arguments are still reported as such
