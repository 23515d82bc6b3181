"""The oracle's MXFP4 storage (spark_model helpers_a.rs: native-MXFP4 routed experts
with one E8M0 scale per 32 values, [N, K/32]; E2M1 codes two per byte as for
NVFP4), pinned to things other than itself:

* all 256 E8M0 bytes against torch's float8_e8m0fnu cast and 2^(b - 127), with
  0xFF the NaN;
* row size k/2 and the nibble order through hand-packed one-hot rows;
* a hand-built problem with constant codes and per-block power-of-two scales
  against its closed form e2m1(c) * sum_g 2^(t_g) X_g;
* random problems against the vectorised NumPy restatement.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from tests import numpy_ref as R
from workloads import make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_MXFP4


def test_e8m0_every_byte():
    b = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(b).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = np.array([oracle.e8m0_to_double(int(v)) for v in b])
    assert np.isnan(got[255]) and np.isnan(want[255])
    np.testing.assert_array_equal(got[:255], want[:255])
    np.testing.assert_array_equal(got[:255], np.ldexp(1.0, b[:255].astype(np.int64) - 127))


def test_row_bytes_and_nibble_order():
    assert oracle.row_bytes(FMT_MXFP4, 4, 4096) == 2048
    assert oracle.row_bytes(FMT_MXFP4, 4, 2816) == 1408
    for j in (0, 1, 30, 31, 33, 63):
        codes = np.zeros(64, np.int64)
        codes[j] = 0xB
        row = R.pack_codes(codes[None], FMT_MXFP4, 4)[0]
        assert row[j // 2] == (0xB << (4 * (j & 1)))
        assert [oracle.code(row, FMT_MXFP4, 4, i) for i in range(64)] == list(codes)


@pytest.mark.parametrize("c", [1, 3, 7, 9, 15])
def test_constant_codes_closed_form(c):
    P = make_problem("mx-const", fmt=FMT_MXFP4, bits=4, group_size=32, m=3, k=128, n=5, n_expert_used=2,
                     num_experts=3, x_dtype=DT_F32, out_dtype=DT_F32, seed=9100 + c)
    P.packed[...] = c | (c << 4)
    rng = np.random.default_rng(9200 + c)
    t = rng.integers(-6, 3, size=P.scales.shape)
    P.scales[...] = (127 + t).astype(np.uint8)
    out, bad = oracle.qmm_id(P)
    assert bad == 0
    e2m1 = {1: 0.5, 3: 1.5, 7: 6.0, 9: -0.5, 15: -6.0}[c]
    X = P.x.astype(np.float64).reshape(P.m, 4, 32).sum(axis=2)      # block sums of x
    ids = P.ids.reshape(-1)
    for p in range(P.R):
        tok = p // P.n_expert_used
        want = e2m1 * (np.ldexp(1.0, t[ids[p]]) * X[tok]).sum(axis=1)   # [n]
        np.testing.assert_allclose(out[p], want, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("seed,xd", [(9301, DT_F32), (9302, DT_BF16), (9303, DT_F16)])
def test_random_against_numpy(seed, xd):
    P = make_problem("mx-rand", fmt=FMT_MXFP4, bits=4, group_size=32, m=4, k=256, n=24, n_expert_used=3,
                     num_experts=6, x_dtype=xd, out_dtype=DT_F32, seed=seed)
    out, _ = oracle.qmm_id(P)
    W = R.dequant_dense(P)
    X = R.x_f64(P)
    ids = P.ids.reshape(-1)
    want = np.einsum("pnk,pk->pn", W[ids], X[np.arange(P.R) // P.n_expert_used])
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_generator_scales_are_plausible_block_exponents():
    P = make_problem("mx-gen", fmt=FMT_MXFP4, bits=4, group_size=32, m=1, k=4096, n=64, n_expert_used=1,
                     num_experts=2, x_dtype=DT_F32, out_dtype=DT_F32, seed=9400)
    e = P.scales.astype(np.int64) - 127
    # amax of 32 draws of N(0, 0.02^2) lies between ~0.03 and ~0.1: exponents -8 .. -6
    assert e.min() >= -10 and e.max() <= -5
    assert not math.isnan(oracle.expert_max_abs_weight(P, 0))


def test_invalid_group_size_rejected():
    P = make_problem("mx-bad", fmt=FMT_MXFP4, bits=4, group_size=32, m=1, k=64, n=2, n_expert_used=1,
                     num_experts=1, x_dtype=DT_F32, out_dtype=DT_F32, seed=9500)
    P.group_size = 16
    with pytest.raises(ValueError):
        oracle.qmm_id(P)
