"""Pointer-table weights (moe_qmm_id_ptrs): each expert's packed rows, scales and
biases in buffers of their own, at assorted alignments, against the oracle on
the contiguous copy of the same bytes, element by element, on the CUDA-core and
grouped-GEMM paths; experts with a null entry leave their pairs' rows untouched;
buffers a path cannot read skip the expert and are reported."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import TORCH_OUT, compare, out_to_f64, to_device
import oracle
from workloads import make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4

pytestmark = pytest.mark.gpu

SENTINEL = 7.0


def _own_buffers(arr: torch.Tensor, offsets, keep):
    """Per-expert copies of arr[e] at byte offset offsets[e] inside a buffer of their
    own; returns (tensors kept alive, int64 address table; 0 where not keep[e])."""
    flat = arr.reshape(arr.shape[0], -1).view(torch.uint8)
    bufs, addrs = [], []
    for e in range(arr.shape[0]):
        if not keep[e]:
            addrs.append(0)
            continue
        nb = flat[e].numel()
        b = torch.zeros(nb + 64, dtype=torch.uint8, device="cuda")
        b[offsets[e]:offsets[e] + nb] = flat[e]
        bufs.append(b)
        addrs.append(b.data_ptr() + offsets[e])
    return bufs, torch.tensor(addrs, dtype=torch.int64, device="cuda")


def _run(P, null_experts=(), scale_offset=None, path="auto", seed=0, code_align=1, code_offsets=None):
    dev = to_device(P)
    E = P.num_experts
    keep = [e not in null_experts for e in range(E)]
    rng = np.random.default_rng(seed)
    w_off = code_offsets or [code_align * int(rng.integers(0, 16 // code_align + 1)) for _ in range(E)]
    s_step = 1 if P.fmt == FMT_NVFP4 else 2
    s_off = [scale_offset if scale_offset is not None else s_step * int(rng.integers(0, 8)) for _ in range(E)]
    keep_bufs, packed_t = _own_buffers(dev["packed"].reshape(E, P.n, -1), w_off, keep)
    sb, scale_t = _own_buffers(dev["scales"].reshape(E, P.n, -1), s_off, keep)
    keep_bufs += sb
    bias_t, aux = None, dev["aux"]
    if P.fmt == FMT_AFFINE:
        bb, bias_t = _own_buffers(dev["aux"].reshape(E, P.n, -1), [2 * (e % 8) for e in range(E)], keep)
        keep_bufs += bb
        aux = None
    out = torch.full((P.m, P.n_expert_used, P.n), SENTINEL, dtype=TORCH_OUT[P.out_dtype], device="cuda")
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    M.qmm_id_ptrs(dev["x"], dev["ids"], packed_t, scale_t, bias_t, aux, n=P.n, group_size=P.group_size,
                  bits=P.bits, fmt=P.fmt, num_experts=E, out=out, workspace=ws, path=path)
    status = M.poll_error(ws)
    return out, status


CASES = [
    ("affine4-fused", dict(fmt=FMT_AFFINE, bits=4, group_size=32, m=6, k=256, n=96, n_expert_used=4,
                           num_experts=9, x_dtype=DT_BF16, out_dtype=DT_F32)),
    ("codebook3-routed", dict(fmt=FMT_CODEBOOK, bits=3, group_size=32, m=50, k=320, n=64, n_expert_used=3,
                              num_experts=7, x_dtype=DT_F16, out_dtype=DT_F16)),
    ("nvfp4-routed", dict(fmt=FMT_NVFP4, bits=4, group_size=16, m=40, k=256, n=80, n_expert_used=2,
                          num_experts=6, x_dtype=DT_F32, out_dtype=DT_BF16)),
    ("affine6-one-token", dict(fmt=FMT_AFFINE, bits=6, group_size=64, m=1, k=512, n=128, n_expert_used=8,
                               num_experts=12, x_dtype=DT_BF16, out_dtype=DT_F32)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("nulls", [(), (1, 4)])
def test_pointer_tables_match_oracle(case, nulls):
    name, kw = case
    P = make_problem(name, seed=7100 + len(name), scale_range=(0.005, 0.03), **kw)
    # code buffers at any byte offset: the CUDA-core path (AUTO would take the grouped
    # GEMM for the larger cases, which needs aligned code rows)
    out, status = _run(P, null_experts=nulls, seed=len(name), path="decode")
    assert status == 0
    ref, _ = oracle.qmm_id(P)
    got = out_to_f64(out)
    ids = P.ids.reshape(-1)
    held = np.array([int(e) not in nulls for e in ids])
    assert np.all(got[~held] == SENTINEL), "rows of experts held elsewhere must be untouched"
    pairs = np.repeat(np.arange(P.R)[held], P.n)
    cols = np.tile(np.arange(P.n), int(held.sum()))
    nviol, ratio, info = compare(P, got[held].reshape(-1), ref[held].reshape(-1), pairs, cols)
    assert nviol == 0, f"{name}: {nviol} outside tolerance ({ratio:.3g}, {info})"


def test_misaligned_scales_skip_the_expert_and_report():
    P = make_problem("misaligned", fmt=FMT_CODEBOOK, bits=3, group_size=32, m=4, k=256, n=64,
                     n_expert_used=2, num_experts=5, x_dtype=DT_F16, out_dtype=DT_F32, seed=7200)
    out, status = _run(P, scale_offset=1)  # f16 scales at odd addresses
    assert status == 7
    assert torch.all(out == SENTINEL)


GROUPED = [
    ("affine4-grouped", dict(fmt=FMT_AFFINE, bits=4, group_size=32, m=200, k=256, n=160, n_expert_used=4,
                             num_experts=6, x_dtype=DT_BF16, out_dtype=DT_F32)),
    ("codebook3-grouped", dict(fmt=FMT_CODEBOOK, bits=3, group_size=32, m=48, k=448, n=200, n_expert_used=4,
                               num_experts=12, x_dtype=DT_F16, out_dtype=DT_F32)),
    ("nvfp4-grouped", dict(fmt=FMT_NVFP4, bits=4, group_size=16, m=700, k=256, n=160, n_expert_used=2,
                           num_experts=4, x_dtype=DT_BF16, out_dtype=DT_BF16)),
]


@pytest.mark.parametrize("case", GROUPED, ids=lambda c: c[0])
def test_pointer_tables_grouped(case):
    name, kw = case
    P = make_problem(name, seed=7400 + len(name), scale_range=(0.005, 0.03), **kw)
    nulls = (1,)
    align = 4 if P.fmt == FMT_CODEBOOK else 8
    out, status = _run(P, null_experts=nulls, path="grouped", seed=len(name), code_align=align)
    assert status == 0
    ref, _ = oracle.qmm_id(P)
    got = out_to_f64(out)
    held = np.array([int(e) not in nulls for e in P.ids.reshape(-1)])
    assert np.all(got[~held] == SENTINEL)
    pairs = np.repeat(np.arange(P.R)[held], P.n)
    cols = np.tile(np.arange(P.n), int(held.sum()))
    nviol, ratio, info = compare(P, got[held].reshape(-1), ref[held].reshape(-1), pairs, cols)
    assert nviol == 0, f"{name}: {nviol} outside tolerance ({ratio:.3g}, {info})"


def test_grouped_path_skips_unaligned_code_buffers():
    P = make_problem("grouped-unaligned", fmt=FMT_AFFINE, bits=4, group_size=32, m=64, k=256, n=64,
                     n_expert_used=2, num_experts=4, x_dtype=DT_BF16, out_dtype=DT_F32, seed=7300)
    offs = [3, 0, 16, 8]  # expert 0's code rows at an odd address
    out, status = _run(P, path="grouped", scale_offset=2, code_offsets=offs)
    assert status == 7
    got = out_to_f64(out)
    ids = P.ids.reshape(-1)
    skipped = ids == 0
    assert np.all(got[skipped] == SENTINEL)
    ref, _ = oracle.qmm_id(P)
    pairs = np.repeat(np.arange(P.R)[~skipped], P.n)
    cols = np.tile(np.arange(P.n), int((~skipped).sum()))
    nviol, ratio, info = compare(P, got[~skipped].reshape(-1), ref[~skipped].reshape(-1), pairs, cols)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"
    # the CUDA-core path reads the same buffers
    out2, status2 = _run(P, path="decode", scale_offset=2, code_offsets=offs)
    assert status2 == 0
    ref_all = ref.reshape(-1)
    pairs = np.repeat(np.arange(P.R), P.n)
    cols = np.tile(np.arange(P.n), P.R)
    nviol, ratio, info = compare(P, out_to_f64(out2).reshape(-1), ref_all, pairs, cols)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"
