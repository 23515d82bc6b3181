"""Pins of the oracle's max |w| over one expert's dequantised weights (the max|w_e|
of the stated tolerance, 1e-2 * ||x|| * max|w_e| / sqrt(k); mlx-native
quantized_matmul_id.rs, module documentation, for the dequantised weights it
ranges over).

* Hand-built experts whose largest |w| sits at a known place: the last group of
  the last row, on a row whose length k is not a multiple of the group size,
  with larger codes planted in the padding past k (which must be ignored) and in
  another expert (which must not be read). The expected value is written out
  from the format's closed form, not computed by any dequantiser.
* Random problems of every format against the vectorised NumPy restatement.
"""

import numpy as np
import pytest

import oracle
from tests import numpy_ref as R
from workloads import make_problem
from workloads.gen import (
    DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_MXFP4, FMT_NVFP4, bf16_bits, e4m3_bits, f16_bits,
)

FORMATS = [
    (FMT_AFFINE, 4, 32), (FMT_AFFINE, 6, 64), (FMT_AFFINE, 8, 32),
    (FMT_CODEBOOK, 2, 32), (FMT_CODEBOOK, 3, 32), (FMT_CODEBOOK, 4, 64),
    (FMT_NVFP4, 4, 16), (FMT_MXFP4, 4, 32),
]


def _problem(fmt, bits, gs, k, seed, n=6, E=3):
    return make_problem("maxabs", fmt=fmt, bits=bits, group_size=gs, m=2, k=k, n=n, n_expert_used=2,
                        num_experts=E, x_dtype=DT_F32, out_dtype=DT_F32, seed=seed)


@pytest.mark.parametrize("fmt,bits,gs", FORMATS)
@pytest.mark.parametrize("ragged", [False, True])
def test_random_problems_match_numpy(fmt, bits, gs, ragged):
    k = 4 * gs + (gs // 2 if ragged and fmt not in (FMT_NVFP4, FMT_MXFP4) else 0)
    if ragged and fmt in (FMT_NVFP4, FMT_MXFP4):
        k = 4 * gs + 6  # even, not a multiple of the block
    P = _problem(fmt, bits, gs, k, seed=500 + 10 * fmt + bits + (1000 if ragged else 0))
    for e in range(P.num_experts):
        want = float(np.abs(R.dequant_expert(P, e)).max())
        assert oracle.expert_max_abs_weight(P, e) == want


def _plant(P, codes_e, scales_e, e):
    """Replace expert e's codes (k values per row, padding codes set to the largest
    code) and scales."""
    full = np.full((P.n, P.row_bytes * 8), (1 << P.bits) - 1, np.int64)  # padding: largest code
    full[:, :P.k] = codes_e
    per_row = P.row_bytes * 8 // P.bits if not (P.fmt == FMT_AFFINE and P.bits == 6) else P.row_bytes // 3 * 4
    if P.fmt == FMT_CODEBOOK and P.bits == 3:
        per_row = P.row_bytes // 4 * 10
    P.packed[e] = R.pack_codes(full[:, :per_row], P.fmt, P.bits)
    P.scales[e] = scales_e


@pytest.mark.parametrize("fmt,bits,gs", FORMATS)
def test_planted_max_in_last_group_of_ragged_row(fmt, bits, gs):
    # k not a multiple of the group size, and (except for the 4-bit float formats, whose
    # rows hold exactly k codes) not a multiple of the codes per word: padding codes exist
    ragged_k = 3 * gs + (gs // 2 + 1 if fmt not in (FMT_NVFP4, FMT_MXFP4) else 4)
    P = _problem(fmt, bits, gs, ragged_k, seed=700 + 10 * fmt + bits, n=5, E=3)
    G = P.groups
    e = 1
    top = (1 << bits) - 1
    codes = np.zeros((P.n, P.k), np.int64)
    # the planted element: last row, last valid position, one below the largest code
    codes[P.n - 1, P.k - 1] = top - 1
    if fmt == FMT_AFFINE:
        # s = 2^-4 everywhere, bias 0, except the last group of the last row: s = 2^-1
        s = np.full((P.n, G), 2.0 ** -4, np.float32)
        s[P.n - 1, G - 1] = 0.5
        _plant(P, codes, bf16_bits(s), e)
        P.aux[e] = bf16_bits(np.zeros((P.n, G), np.float32))
        want = (top - 1) * 0.5
    elif fmt == FMT_CODEBOOK:
        cb = np.arange(1 << bits, dtype=np.float32) * 0.25  # cb[c] = c/4, code 0 -> 0
        P.aux[...] = f16_bits(cb)
        s = np.full((P.n, G), 2.0 ** -4, np.float32)
        s[P.n - 1, G - 1] = 2.0
        _plant(P, codes, f16_bits(s), e)
        want = (top - 1) * 0.25 * 2.0
    elif fmt == FMT_NVFP4:
        s = np.full((P.n, G), 2.0 ** -3, np.float32)
        s[P.n - 1, G - 1] = 4.0
        _plant(P, codes, e4m3_bits(s), e)
        P.aux[e] = np.float32(0.5)
        want = 4.0 * 4.0 * 0.5  # code 14 = -4 in E2M1: |w| = 4 * 4 * scale2
    else:  # MXFP4
        s = np.full((P.n, G), 127 - 3, np.uint8)
        s[P.n - 1, G - 1] = 127 + 2
        _plant(P, codes, s, e)
        want = 4.0 * 4.0  # |e2m1(14)| * 2^2
    # the next expert holds larger weights (largest code, the large scale everywhere);
    # they must not be read
    P.packed[e + 1][...] = 0xFF
    P.scales[e + 1][...] = P.scales[e][P.n - 1, G - 1]
    if fmt == FMT_AFFINE:
        P.aux[e + 1][...] = 0
    if fmt == FMT_NVFP4:
        P.aux[e + 1] = P.aux[e]
    assert float(np.abs(R.dequant_expert(P, e + 1)).max()) > want
    got = oracle.expert_max_abs_weight(P, e)
    assert got == want, (got, want)
    # the restatement agrees (so the planted value is the true max)
    assert float(np.abs(R.dequant_expert(P, e)).max()) == want


def test_out_of_range_expert_is_rejected():
    P = _problem(FMT_AFFINE, 4, 32, 128, seed=901)
    assert oracle.expert_max_abs_weight(P, P.num_experts) == -1.0
