"""3-bit codebook rows on the grouped GEMM, against the oracle element by element.
Rows that are a multiple of 8 bytes (with n even) reach shared memory as tensor
copies of two-row "super-rows" (the even rows' window of the k-tile, then the odd
rows'); other rows by the loader warps' 4-byte copies. Cases: the canvas row
width (1128 bytes, 282 words), a window that runs past the row's end in the last
k-tile, rows of an odd number of words and an odd n (both copied by the loaders),
f32 x, 64- and 256-pair tiles."""

import pytest
import torch

from tests.gpu_util import check_full, run
from workloads import make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_CODEBOOK

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,topk,E,k,n,xd,od", [
    (64, 4, 4, 2816, 256, DT_F16, DT_F32),     # 1128-byte rows (super-rows of 2256 bytes)
    (48, 2, 3, 320, 128, DT_F16, DT_BF16),     # 128-byte rows; the last window runs past the row
    (40, 2, 3, 288, 96, DT_F16, DT_F32),       # 29 words = 116 bytes: loader copies
    (40, 2, 3, 320, 129, DT_BF16, DT_F32),     # odd n: loader copies
    (50, 2, 4, 640, 192, DT_F32, DT_F32),      # f32 x
    (700, 2, 4, 960, 160, DT_F16, DT_F32),     # 256-pair tiles, ragged last row block
])
def test_cb3_grouped_matches_oracle(m, topk, E, k, n, xd, od):
    P = make_problem("cb3-staging", seed=7700 + k + n + m, fmt=FMT_CODEBOOK, bits=3, group_size=32, x_dtype=xd,
                     out_dtype=od, m=m, k=k, n=n, n_expert_used=topk, num_experts=E, scale_range=(0.01, 0.05))
    out = run(P, "grouped")
    torch.cuda.synchronize()
    nviol, ratio, info = check_full(P, out)
    assert nviol == 0, f"{nviol} outside tolerance ({ratio:.3g}, {info})"
