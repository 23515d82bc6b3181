"""CUDA path vs the CPU oracle, element by element, at sizes the oracle finishes
in seconds: every storage format, x / out type and kernel path, tiles spanning
several k-tiles with ragged tails, and the edge cases (experts with 0 or 1 pairs,
duplicate ids, out-of-range ids, unaligned rows, tiny n)."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import check_full, check_sampled, run, to_device
from workloads import config_problem, make_problem
from workloads.gen import (
    DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4, distinct_uniform_ids, zipf_ids,
)

pytestmark = pytest.mark.gpu


def assert_ok(res, what=""):
    nviol, ratio, info = res
    assert nviol == 0, f"{what}: {nviol} elements outside tolerance (worst err/bound {ratio:.3g}, {info})"


@pytest.mark.parametrize("path", ["auto", "decode", "grouped"])
def test_tiny_config(path):
    P = config_problem("tiny")
    out = run(P, path)
    torch.cuda.synchronize()
    assert_ok(check_full(P, out), f"tiny/{path}")


FORMAT_CASES = [
    # fmt, bits, gs, x_dtype, out_dtype
    (FMT_AFFINE, 4, 32, DT_BF16, DT_F32),
    (FMT_AFFINE, 4, 64, DT_F32, DT_BF16),
    (FMT_AFFINE, 6, 32, DT_F32, DT_F32),
    (FMT_AFFINE, 6, 64, DT_BF16, DT_F16),
    (FMT_AFFINE, 8, 32, DT_F16, DT_F32),
    (FMT_CODEBOOK, 3, 32, DT_F16, DT_F32),
    (FMT_CODEBOOK, 3, 16, DT_BF16, DT_BF16),
    (FMT_CODEBOOK, 2, 32, DT_F16, DT_F32),
    (FMT_CODEBOOK, 4, 64, DT_F32, DT_F32),
    (FMT_NVFP4, 4, 16, DT_BF16, DT_BF16),
    (FMT_NVFP4, 4, 16, DT_F16, DT_F32),
    (FMT_NVFP4, 4, 16, DT_F32, DT_F32),
]


def _mid(fmt, bits, gs, xd, od, m=40, topk=4, E=12, k=448, n=200, seed=0, ids="uniform"):
    return make_problem(f"mid-{fmt}-{bits}", fmt=fmt, bits=bits, group_size=gs, m=m, k=k, n=n,
                        n_expert_used=topk, num_experts=E, x_dtype=xd, out_dtype=od,
                        seed=1000 + seed + 10 * bits + fmt, scale_range=(0.005, 0.03), ids=ids)


@pytest.mark.parametrize("case", FORMAT_CASES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("path", ["decode", "grouped"])
def test_formats_both_paths(case, path):
    fmt, bits, gs, xd, od = case
    P = _mid(fmt, bits, gs, xd, od)
    out = run(P, path)
    torch.cuda.synchronize()
    assert_ok(check_full(P, out), f"{case}/{path}")


@pytest.mark.parametrize("case", FORMAT_CASES, ids=lambda c: "-".join(map(str, c)))
def test_formats_fused_decode(case):
    fmt, bits, gs, xd, od = case
    P = _mid(fmt, bits, gs, xd, od, m=5, topk=3, E=9, k=448, n=77)
    out = run(P, "auto")
    torch.cuda.synchronize()
    assert_ok(check_full(P, out), f"{case}/fused")


@pytest.mark.parametrize("path", ["decode", "grouped"])
def test_large_tiles_and_hot_expert(path):
    # R >= 96 * E selects 256-row tiles; Zipf popularity gives one expert ~1000 rows
    P = make_problem("hot", fmt=FMT_NVFP4, bits=4, group_size=16, m=1500, k=256, n=160,
                     n_expert_used=2, num_experts=8, x_dtype=DT_BF16, out_dtype=DT_BF16, seed=31,
                     ids="zipf", zipf_s=1.5)
    out = run(P, path)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    pairs = rng.integers(0, P.R, 4000)
    cols = rng.integers(0, P.n, 4000)
    assert_ok(check_sampled(P, out, pairs, cols), f"hot/{path}")
    # whole rows of the hottest expert's last tile
    e0 = np.bincount(P.ids.reshape(-1), minlength=P.num_experts).argmax()
    last = np.nonzero(P.ids.reshape(-1) == e0)[0][-40:]
    assert_ok(check_sampled(P, out, np.repeat(last, P.n), np.tile(np.arange(P.n), last.size)),
              "hot/last-tile")


@pytest.mark.parametrize("path", ["decode", "grouped"])
def test_sparse_experts_zero_and_one_pair(path):
    P = make_problem("sparse", fmt=FMT_AFFINE, bits=4, group_size=32, m=36, k=256, n=130,
                     n_expert_used=2, num_experts=200, x_dtype=DT_BF16, out_dtype=DT_F32, seed=32)
    out = run(P, path)
    torch.cuda.synchronize()
    assert_ok(check_full(P, out), f"sparse/{path}")


@pytest.mark.parametrize("path", ["auto", "decode", "grouped"])
def test_duplicate_and_out_of_range_ids(path):
    P = _mid(FMT_AFFINE, 4, 32, DT_BF16, DT_F32, m=30, topk=3)
    ids = P.ids.copy()
    ids[0, 1] = ids[0, 0]                # duplicate expert inside a token
    ids[4, :] = ids[4, 0]
    ids[7, 2] = P.num_experts            # out of range
    ids[11, 0] = 0xFFFFFFFF
    P = P.with_ids(ids)
    dev = to_device(P)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    out = torch.full((P.m, P.n_expert_used, P.n), float("nan"), device="cuda")
    run(P, path, dev=dev, out=out, workspace=ws)
    assert M.poll_error(ws) == 5
    assert M.poll_error(ws) == 0        # cleared
    assert_ok(check_full(P, out), f"dup-bad/{path}")


def test_fused_decode_out_of_range_ids():
    P = _mid(FMT_AFFINE, 4, 32, DT_BF16, DT_F32, m=4, topk=4, E=6)
    ids = P.ids.copy()
    ids[2, 3] = 1000
    P = P.with_ids(ids)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    out = torch.full((P.m, P.n_expert_used, P.n), float("nan"), device="cuda")
    run(P, "auto", out=out, workspace=ws)
    assert M.poll_error(ws) == 5
    assert_ok(check_full(P, out), "fused-bad")


@pytest.mark.parametrize("k,gs,fmt,bits", [(200, 40, FMT_AFFINE, 4), (100, 20, FMT_AFFINE, 6),
                                           (90, 30, FMT_CODEBOOK, 3), (52, 4, FMT_AFFINE, 8),
                                           (80, 16, FMT_NVFP4, 4)])
@pytest.mark.parametrize("m,topk", [(3, 2), (50, 3)])
def test_unaligned_rows_take_the_gemv(k, gs, fmt, bits, m, topk):
    P = make_problem("unaligned", fmt=fmt, bits=bits, group_size=gs, m=m, k=k, n=45,
                     n_expert_used=topk, num_experts=7, x_dtype=DT_F32, out_dtype=DT_F32, seed=33)
    out = run(P, "auto")
    torch.cuda.synchronize()
    assert_ok(check_full(P, out), f"unaligned k={k}")


def test_ragged_k_is_unsupported_not_wrong():
    # k % group_size != 0 is valid storage (ceil groups) that this library does not implement
    P = make_problem("ragged", fmt=FMT_AFFINE, bits=4, group_size=32, m=2, k=100, n=16,
                     n_expert_used=2, num_experts=4, x_dtype=DT_F32, out_dtype=DT_F32, seed=35)
    with pytest.raises(M.MoeError) as ei:
        run(P, "auto")
    assert ei.value.status == 2


@pytest.mark.parametrize("n", [1, 31, 129])
@pytest.mark.parametrize("path", ["auto", "grouped"])
def test_small_and_ragged_n(n, path):
    P = make_problem("n", fmt=FMT_CODEBOOK, bits=3, group_size=32, m=20, k=320, n=n,
                     n_expert_used=4, num_experts=5, x_dtype=DT_F16, out_dtype=DT_F32, seed=34)
    out = run(P, path)
    torch.cuda.synchronize()
    assert_ok(check_full(P, out), f"n={n}/{path}")


@pytest.mark.parametrize("proj", ["decode_gate_up", "decode_down"])
@pytest.mark.parametrize("m", [1, 2, 3, 4, 8, 9, 16, 17, 33])
def test_decode_sweep(proj, m):
    P = config_problem(proj, m=m, seed=7000 + m)
    out = run(P, "auto")
    torch.cuda.synchronize()
    if m == 1:
        assert_ok(check_full(P, out), f"{proj} m=1")
    else:
        rng = np.random.default_rng(m)
        pairs = np.concatenate([np.repeat(np.arange(P.R), 8), rng.integers(0, P.R, 2000)])
        cols = np.concatenate([rng.integers(0, P.n, 8 * P.R), rng.integers(0, P.n, 2000)])
        assert_ok(check_sampled(P, out, pairs, cols), f"{proj} m={m}")


def test_paths_agree_and_reruns_bit_identical():
    P = _mid(FMT_AFFINE, 6, 64, DT_F32, DT_F32, m=64, topk=8, E=16, k=512, n=256, ids="zipf")
    dev = to_device(P)
    a = run(P, "grouped", dev=dev)
    b = run(P, "grouped", dev=dev)
    c = run(P, "decode", dev=dev)
    d = run(P, "decode", dev=dev)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(c, d)
    assert_ok(check_full(P, a), "zipf/grouped")
    assert_ok(check_full(P, c), "zipf/decode")
