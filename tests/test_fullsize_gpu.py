"""Full-size workloads in the launch configuration the benchmark times (path
"auto", the workspace sized by moe_qmm_id_workspace_bytes_k, so that f32 x takes
the gathered rows and 16-bit x with 256-pair tiles the f16 image of B), checked
against the oracle on sampled outputs (the oracle computes them one by one) and on
properties that hold at any size; the minimum workspace (loader copies of x) and
W4A4 on the prefill workload (the block-scaled MMA) as well."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
import oracle
from tests.gpu_util import check_sampled, run, to_device
from workloads import config_problem

pytestmark = pytest.mark.gpu

FULL = ["decode_gate_up", "decode_down", "canvas", "prefill", "skewed"]


@pytest.fixture(scope="module", params=FULL)
def problem(request):
    P = config_problem(request.param)
    dev = to_device(P)
    return P, dev


def _bench_workspace(P, dev):
    """The workspace the benchmark gives a call: room for the grouped path's x pre-pass."""
    return M.new_workspace(P.m, P.n_expert_used, P.num_experts, k=P.k, x_dtype=dev["x"].dtype)


def test_sampled_parity(problem):
    P, dev = problem
    ws = _bench_workspace(P, dev)
    out = run(P, "auto", dev=dev, workspace=ws)
    assert M.poll_error(ws) == 0
    rng = np.random.default_rng(17)
    ns = 3000
    # random elements, whole rows of a few pairs, and the last rows/cols (ragged tiles)
    pairs = np.concatenate([rng.integers(0, P.R, ns), np.repeat(rng.integers(0, P.R, 3), P.n),
                            np.full(64, P.R - 1)])
    cols = np.concatenate([rng.integers(0, P.n, ns), np.tile(np.arange(P.n), 3),
                           np.arange(P.n - 64, P.n)])
    nviol, ratio, info = check_sampled(P, out, pairs, cols)
    assert nviol == 0, f"{P.name}: {nviol} violations, worst err/bound {ratio:.3g} {info}"
    assert torch.isfinite(out.float()).all()


def test_slot_permutation_permutes_output(problem):
    P, dev = problem
    out = run(P, "auto", dev=dev)
    perm = np.random.default_rng(5).permutation(P.n_expert_used)
    dev2 = dict(dev)
    dev2["ids"] = dev["ids"][:, torch.from_numpy(perm).cuda()].contiguous()
    out2 = run(P.with_ids(P.ids[:, perm]), "auto", dev=dev2)
    torch.cuda.synchronize()
    assert torch.equal(out2, out[:, torch.from_numpy(perm).cuda(), :])


def test_rerun_bit_identical(problem):
    P, dev = problem
    a = run(P, "auto", dev=dev)
    b = run(P, "auto", dev=dev)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def _tile_class_sample(P):
    """(pairs, cols) covering each kind of tile the grouped GEMM forms, in full
    output rows: every pair of the hottest and of the coldest expert (all
    columns for the coldest; for the hottest, all columns of the pairs at each
    64-pair boundary inside the expert, 0, 63, 64, 127, 128, ..., and the
    first, middle and last column of every 128-row block for the others), pairs
    256..319 of an expert with more than 256 pairs (the start of its second
    256-pair tile), and the last 128-column block of every pair at a tile
    boundary. The tile list runs over the experts' pairs in ascending pair index
    (metrale helpers_b.rs, launch_grouped_gemm: expert_offsets / sorted_token_ids)."""
    ids = P.ids.reshape(-1).astype(np.int64)
    order = np.argsort(ids, kind="stable")
    counts = np.bincount(ids, minlength=P.num_experts)
    starts = np.concatenate(([0], np.cumsum(counts)))
    used = np.nonzero(counts)[0]
    hot = int(used[np.argmax(counts[used])])
    cold = int(used[np.argmin(counts[used])])
    pairs, cols = [], []

    def full_rows(ps):
        ps = np.asarray(ps, dtype=np.int64)
        pairs.append(np.repeat(ps, P.n))
        cols.append(np.tile(np.arange(P.n), ps.size))

    def some_cols(ps, cs):
        ps = np.asarray(ps, dtype=np.int64)
        pairs.append(np.repeat(ps, cs.size))
        cols.append(np.tile(cs, ps.size))

    hot_pairs = order[starts[hot]:starts[hot + 1]]
    cold_pairs = order[starts[cold]:starts[cold + 1]]
    full_rows(cold_pairs)
    pos = sorted({q for b in range(0, hot_pairs.size, 64) for q in (b, b + 63) if q < hot_pairs.size}
                 | {hot_pairs.size - 1})
    full_rows(hot_pairs[pos])
    blocks = np.arange(0, P.n, 128)
    some_cols(hot_pairs, np.unique(np.concatenate([blocks, blocks + 64, np.minimum(blocks + 127, P.n - 1)])))
    big = np.nonzero(counts > 256)[0]
    if big.size:
        e = int(big[0])
        full_rows(order[starts[e] + 256:starts[e] + min(320, counts[e])])
    # last column block of the first and last pair of every expert
    edge = np.unique(np.concatenate([order[starts[used]], order[starts[used + 1] - 1]]))
    some_cols(edge, np.arange(max(0, P.n - 128), P.n))
    return np.concatenate(pairs), np.concatenate(cols)


@pytest.mark.parametrize("name", ["canvas", "prefill", "skewed"])
def test_every_tile_class(name):
    P = config_problem(name)
    dev = to_device(P)
    ws = _bench_workspace(P, dev)
    out = run(P, "auto", dev=dev, workspace=ws)
    assert M.poll_error(ws) == 0
    pairs, cols = _tile_class_sample(P)
    nviol, ratio, info = check_sampled(P, out, pairs, cols)
    assert nviol == 0, f"{P.name}: {nviol} of {pairs.size} violations, worst err/bound {ratio:.3g} {info}"


@pytest.mark.parametrize("name", ["prefill", "skewed"])
def test_sampled_parity_minimum_workspace(name):
    """The minimum workspace: the loader warps copy x rows themselves (f32 x split per
    tile by the dequantisers)."""
    P = config_problem(name)
    dev = to_device(P)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    out = run(P, "auto", dev=dev, workspace=ws)
    assert M.poll_error(ws) == 0
    rng = np.random.default_rng(23)
    pairs = np.concatenate([rng.integers(0, P.R, 1500), np.full(64, P.R - 1)])
    cols = np.concatenate([rng.integers(0, P.n, 1500), np.arange(P.n - 64, P.n)])
    nviol, ratio, info = check_sampled(P, out, pairs, cols)
    assert nviol == 0, f"{P.name}: {nviol} violations, worst err/bound {ratio:.3g} {info}"


def test_w4a4_prefill_sampled():
    """W4A4 on the prefill workload as the benchmark runs it (NVFP4 weights: the
    block-scaled MMA on the codes of both operands), against the oracle's operation
    on its own quantisation of x, on sampled outputs, whole rows and the last rows."""
    P = config_problem("prefill")
    dev = to_device(P)
    ws = torch.zeros(M.workspace_bytes_w4a4(P.m, P.k, P.n_expert_used, P.num_experts), dtype=torch.uint8,
                     device="cuda")
    out = M.qmm_id_w4a4(dev["x"], dev["ids"], dev["packed"], dev["scales"], dev["aux"], n=P.n,
                        group_size=P.group_size, bits=P.bits, fmt=P.fmt, num_experts=P.num_experts,
                        out_dtype=torch.bfloat16, workspace=ws)
    assert M.poll_error(ws) == 0
    Q = oracle.w4a4_problem(P)
    rng = np.random.default_rng(29)
    pairs = np.concatenate([rng.integers(0, P.R, 2000), np.repeat(rng.integers(0, P.R, 2), P.n),
                            np.full(64, P.R - 1)])
    cols = np.concatenate([rng.integers(0, P.n, 2000), np.tile(np.arange(P.n), 2), np.arange(P.n - 64, P.n)])
    nviol, ratio, info = check_sampled(Q, out, pairs, cols)
    assert nviol == 0, f"W4A4 prefill: {nviol} violations, worst err/bound {ratio:.3g} {info}"
