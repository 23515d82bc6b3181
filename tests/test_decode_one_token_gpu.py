"""The one-token decode kernel (x planes in registers, rows of all pairs split
evenly over the SMs) against the oracle, element by element: row ranges that
straddle pairs, lanes with idle units, groups of 32 to 256 codes, odd group
counts, the widest rows it takes and the first one it does not (handled by
the TMA-staged decode kernel), every x / out type, scale rows that cannot be
bulk-copied, and duplicate and out-of-range ids."""

import pytest
import torch

import moe_expert_routed_b200 as M
from tests.gpu_util import check_full, run, to_device
from workloads import make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE

pytestmark = pytest.mark.gpu

CASES = [
    # k, n, group_size, n_expert_used, num_experts, x_dtype, out_dtype
    (224, 40, 32, 6, 9, DT_F32, DT_BF16),     # 7 units per row: 8 lanes per row, one idle
    (96, 13, 32, 3, 5, DT_F16, DT_F16),       # n not a multiple of 8: scale rows read one by one
    (704, 88, 64, 8, 16, DT_BF16, DT_F32),    # 22 units: 8 lanes x 3 units
    (1024, 24, 128, 2, 3, DT_BF16, DT_F32),   # one group spans 4 units
    (3072, 64, 128, 8, 16, DT_BF16, DT_F32),  # 96 units: the widest row of the kernel
    (3104, 32, 32, 4, 6, DT_F32, DT_F32),     # 97 units: handled by the other decode kernel
    (2816, 1, 64, 8, 12, DT_BF16, DT_F32),    # one row per pair
    (1024, 48, 256, 4, 6, DT_BF16, DT_F32),   # groups of 256
    (4096, 24, 256, 3, 4, DT_F16, DT_F32),    # 128 units: handled by the other decode kernel
    (96, 5, 32, 6, 9, DT_BF16, DT_F32),       # 4 lanes per row: 8 rows at once step over whole pairs
    (224, 3, 32, 8, 10, DT_F16, DT_F32),      # 8 lanes per row, pairs of 3 rows
    (1408, 7, 64, 8, 12, DT_BF16, DT_F32),    # 32 lanes per row, 4 rows per pass over pairs of 7
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"k{c[0]}-n{c[1]}-g{c[2]}-t{c[3]}")
def test_one_token_shapes(case):
    k, n, gs, topk, E, xd, od = case
    P = make_problem("one-token", fmt=FMT_AFFINE, bits=4, group_size=gs, m=1, k=k, n=n,
                     n_expert_used=topk, num_experts=E, x_dtype=xd, out_dtype=od,
                     seed=5100 + k + n, scale_range=(0.002, 0.01))
    out = run(P, "auto")
    torch.cuda.synchronize()
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"{case}: {nviol} outside tolerance ({ratio:.3g}, {info})"


def test_one_token_duplicate_and_out_of_range_ids():
    P = make_problem("one-token-bad", fmt=FMT_AFFINE, bits=4, group_size=64, m=1, k=704, n=96,
                     n_expert_used=8, num_experts=10, x_dtype=DT_BF16, out_dtype=DT_F32,
                     seed=5200, scale_range=(0.002, 0.01))
    ids = P.ids.copy()
    ids[0, 1] = ids[0, 0]
    ids[0, 3] = P.num_experts
    ids[0, 7] = 0xFFFFFFFF
    P = P.with_ids(ids)
    dev = to_device(P)
    ws = M.new_workspace(P.m, P.n_expert_used, P.num_experts)
    out = torch.full((P.m, P.n_expert_used, P.n), float("nan"), device="cuda")
    run(P, "auto", dev=dev, out=out, workspace=ws)
    assert M.poll_error(ws) == 5
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"
    assert torch.all(out[0, 3] == 0) and torch.all(out[0, 7] == 0)
