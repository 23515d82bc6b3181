"""Full-size workloads in the launch configuration the benchmark times (path
"auto"), checked against the oracle on sampled outputs (the oracle computes them
one by one) and on properties that hold at any size."""

import numpy as np
import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import check_sampled, run, to_device
from workloads import config_problem

pytestmark = pytest.mark.gpu

FULL = ["decode_gate_up", "decode_down", "canvas", "prefill", "skewed"]


@pytest.fixture(scope="module", params=FULL)
def problem(request):
    P = config_problem(request.param)
    dev = to_device(P)
    return P, dev


def test_sampled_parity(problem):
    P, dev = problem
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
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
