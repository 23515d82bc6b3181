"""Pins of the CPU oracle against facts it does not compute itself.

* decoders: exhaustive bit patterns against torch / numpy dtype casts and the
  OCP tables in tests/golden;
* rounding to bf16 / f16: against torch / numpy casts;
* storage sizes: the row sizes the workloads fix (1408, 352, 1128, 2048, 1536 B);
* code extraction: codes packed word-wise (tests/numpy_ref.py) come back bit by bit;
* whole operation: hand-built small-integer weights against a dense matmul,
  closed forms for constant codes, the vectorised NumPy restatement on random
  inputs, permutation invariance, out-of-range ids;
* routing: counts / offsets / stable permutation / tile list against
  numpy.bincount and a stable argsort.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from tests import numpy_ref as R
from workloads import config_problem, make_problem, storage_row_bytes
from workloads.gen import (
    DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4, Problem, bf16_bits, f16_bits,
    e4m3_bits, lloyd_max_normal,
)


def same_float(a, b):
    return (math.isnan(a) and math.isnan(b)) or (a == b and math.copysign(1, a) == math.copysign(1, b))


# ----------------------------------------------------------------- decoders

def test_bf16_decoder_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = R.bf16_to_f64(bits)
    L = oracle.lib()
    for b in range(1 << 16):
        assert same_float(L.oracle_bf16_to_double(b), float(ref[b])), hex(b)


def test_f16_decoder_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = R.f16_to_f64(bits)
    L = oracle.lib()
    for b in range(1 << 16):
        assert same_float(L.oracle_f16_to_double(b), float(ref[b])), hex(b)


def test_e4m3_decoder_exhaustive_and_specials():
    ref = R.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    for b in range(256):
        assert same_float(oracle.e4m3_to_double(b), float(ref[b])), hex(b)
    for line in R.golden_lines("e4m3_special.txt"):
        h, v = line.split()
        assert same_float(oracle.e4m3_to_double(int(h, 16)), float(v)), line


def test_e2m1_decoder_matches_ocp_table():
    for c in range(16):
        assert same_float(oracle.e2m1_to_double(c), float(R.E2M1_TABLE[c])), c
    if hasattr(torch, "float4_e2m1fn_x2"):
        try:
            t = torch.arange(256, dtype=torch.uint8).view(torch.float4_e2m1fn_x2)
            _ = t.to(torch.float32)
        except Exception:
            return  # this torch build has the dtype but no conversion kernel


# ----------------------------------------------------------------- rounding

def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-38).astype(np.float32),   # bf16 subnormals
        (rng.standard_normal(2000) * 1e38).astype(np.float32),
        np.array([0.0, -0.0, 3.3895314e38, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], np.float32),
    ]).astype(np.float64)
    ref = bf16_bits(vals.astype(np.float32))
    got = oracle.round_out(vals, DT_BF16)
    np.testing.assert_array_equal(got, ref)


def test_round_to_f16_matches_numpy():
    rng = np.random.default_rng(12)
    vals = np.concatenate([
        rng.standard_normal(20000), rng.standard_normal(2000) * 1e-6,
        rng.standard_normal(2000) * 7e4, np.array([0.0, -0.0, 65504.0, 65520.0, 1 + 2 ** -11]),
    ])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = oracle.round_out(vals, DT_F16)
    np.testing.assert_array_equal(got, ref)


def test_scalar_rounding_helpers_match_the_casts():
    # the scalar entry points are the same RNE casts as the array one
    rng = np.random.default_rng(13)
    vals = np.concatenate([rng.standard_normal(500), rng.standard_normal(50) * 1e-39,
                           np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1 + 2 ** -11, 65504.0])])
    bf = np.array([oracle.double_to_bf16(v) for v in vals], dtype=np.uint16)
    np.testing.assert_array_equal(bf, bf16_bits(vals.astype(np.float32)))
    with np.errstate(over="ignore"):
        f16 = vals.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(np.array([oracle.double_to_f16(v) for v in vals], dtype=np.uint16), f16)


# ---------------------------------------------------------------- storage

@pytest.mark.parametrize("fmt,bits,k,expect", [
    (FMT_AFFINE, 4, 2816, 1408), (FMT_AFFINE, 4, 704, 352), (FMT_AFFINE, 4, 256, 128),
    (FMT_AFFINE, 6, 2048, 1536), (FMT_AFFINE, 8, 100, 100), (FMT_AFFINE, 6, 5, 6),
    (FMT_CODEBOOK, 3, 2816, 1128), (FMT_CODEBOOK, 3, 10, 4), (FMT_CODEBOOK, 3, 11, 8),
    (FMT_NVFP4, 4, 4096, 2048),
])
def test_row_bytes(fmt, bits, k, expect):
    assert oracle.row_bytes(fmt, bits, k) == expect
    assert storage_row_bytes(fmt, bits, k) == expect


FORMATS = [(FMT_AFFINE, 4), (FMT_AFFINE, 6), (FMT_AFFINE, 8), (FMT_CODEBOOK, 2),
           (FMT_CODEBOOK, 3), (FMT_CODEBOOK, 4), (FMT_NVFP4, 4)]


@pytest.mark.parametrize("fmt,bits", FORMATS)
def test_code_extraction_roundtrip(fmt, bits):
    rng = np.random.default_rng(bits * 7 + fmt)
    for k in (1, 2, 9, 10, 31, 64, 97):
        if fmt == FMT_NVFP4 and k % 2:
            continue
        codes = rng.integers(0, 1 << bits, size=k)
        row = R.pack_codes(codes[None], fmt, bits)[0]
        assert row.size == storage_row_bytes(fmt, bits, k)
        got = [oracle.code(row, fmt, bits, j) for j in range(k)]
        np.testing.assert_array_equal(got, codes)


@pytest.mark.parametrize("fmt,bits", FORMATS)
def test_one_hot_positions(fmt, bits):
    k = 40
    top = (1 << bits) - 1
    for j in range(k):
        codes = np.zeros(k, np.int64)
        codes[j] = top
        row = R.pack_codes(codes[None], fmt, bits)[0]
        for jj in range(k):
            assert oracle.code(row, fmt, bits, jj) == (top if jj == j else 0)


def test_codebook_3bit_ignores_top_two_bits():
    # 10 codes per u32; bits 30-31 of each word carry no code
    row = np.array([0xC0000000, 0xFFFFFFFF], dtype="<u4").view(np.uint8)
    assert [oracle.code(row, FMT_CODEBOOK, 3, j) for j in range(10)] == [0] * 10
    assert [oracle.code(row, FMT_CODEBOOK, 3, j) for j in range(10, 20)] == [7] * 10


# ------------------------------------------------------------ whole operation

def hand_problem(fmt, bits, codes, scales, aux, x, ids, group_size, x_dtype=DT_F32,
                 num_experts=None):
    E, n, k = codes.shape
    return Problem(name="hand", fmt=fmt, bits=bits, group_size=group_size, m=x.shape[0], k=k, n=n,
                   n_expert_used=ids.shape[1], num_experts=num_experts or E, x_dtype=x_dtype,
                   out_dtype=DT_F32, x=x, ids=ids.astype(np.uint32),
                   packed=R.pack_codes(codes, fmt, bits), scales=scales, aux=aux)


def test_hand_built_affine_integer_weights():
    # weights are small integers: w = c*s + b with s = 1, b = -8 -> w in [-8, 7]
    rng = np.random.default_rng(3)
    E, n, k, gs = 3, 5, 64, 16
    codes = rng.integers(0, 16, size=(E, n, k))
    G = k // gs
    scales = bf16_bits(np.ones((E, n, G), np.float32))
    bias = bf16_bits(np.full((E, n, G), -8.0, np.float32))
    x = rng.integers(-3, 4, size=(2, k)).astype(np.float32)
    ids = np.array([[2, 0], [1, 2]])
    P = hand_problem(FMT_AFFINE, 4, codes, scales, bias, x, ids, gs)
    out, bad = oracle.qmm_id(P, nthreads=2)
    W = codes - 8
    expect = np.stack([W[2] @ x[0], W[0] @ x[0], W[1] @ x[1], W[2] @ x[1]])
    assert bad == 0
    np.testing.assert_array_equal(out, expect)


def test_hand_built_codebook_and_nvfp4():
    rng = np.random.default_rng(4)
    E, n, k = 2, 3, 48
    x = rng.integers(-2, 3, size=(1, k)).astype(np.float32)
    ids = np.array([[1, 0]])
    # codebook: centroids are small integers, scale 2 (exact)
    cb = np.array([-3, -1, 0, 2, 5, 7, -2, 4], np.float32)
    codes = rng.integers(0, 8, size=(E, n, k))
    P = hand_problem(FMT_CODEBOOK, 3, codes, f16_bits(np.full((E, n, k // 32 + 1), 2.0, np.float32)),
                     f16_bits(cb), x, ids, 32)
    out, _ = oracle.qmm_id(P, nthreads=1)
    W = cb[codes] * 2.0
    np.testing.assert_array_equal(out, np.stack([W[1] @ x[0], W[0] @ x[0]]))
    # NVFP4: block scales 2 and 0.5 alternate, scale2 = 4
    codes = rng.integers(0, 16, size=(E, n, k))
    s = np.where(np.arange(k // 16) % 2 == 0, 2.0, 0.5).astype(np.float32)
    sc = e4m3_bits(np.broadcast_to(s, (E, n, k // 16)).copy())
    P = hand_problem(FMT_NVFP4, 4, codes, sc, np.full((E,), 4.0, np.float32), x, ids, 16)
    out, _ = oracle.qmm_id(P, nthreads=1)
    W = R.E2M1_TABLE[codes] * np.repeat(s, 16)[None, None, :] * 4.0
    np.testing.assert_array_equal(out, np.stack([W[1] @ x[0], W[0] @ x[0]]))


@pytest.mark.parametrize("fmt,bits", FORMATS)
def test_closed_form_constant_code(fmt, bits):
    """code = c everywhere: out = sum_g (c*s_g + b_g) * X_g  (affine),
    sum_g cb[c]*s_g*X_g (codebook), e2m1(c)*scale2*sum_g s_g*X_g (NVFP4),
    where X_g is the sum of x over group g."""
    rng = np.random.default_rng(100 + 10 * fmt + bits)
    E, n, k = 2, 4, 96
    gs = 16 if fmt == FMT_NVFP4 else 32
    G = k // gs
    x = rng.standard_normal((3, k)).astype(np.float32)
    ids = np.array([[0, 1], [1, 1], [1, 0]])
    Xg = x.reshape(3, G, gs).astype(np.float64).sum(-1)
    for c in (0, 1, (1 << bits) - 1):
        codes = np.full((E, n, k), c)
        if fmt == FMT_AFFINE:
            s = bf16_bits(rng.uniform(0.01, 0.1, (E, n, G)).astype(np.float32))
            b = bf16_bits(rng.normal(0, 0.1, (E, n, G)).astype(np.float32))
            P = hand_problem(fmt, bits, codes, s, b, x, ids, gs)
            w = c * R.bf16_to_f64(s) + R.bf16_to_f64(b)          # [E, n, G]
        elif fmt == FMT_CODEBOOK:
            cb = f16_bits(rng.standard_normal(1 << bits).astype(np.float32))
            s = f16_bits(rng.uniform(0.01, 0.1, (E, n, G)).astype(np.float32))
            P = hand_problem(fmt, bits, codes, s, cb, x, ids, gs)
            w = R.f16_to_f64(cb)[c] * R.f16_to_f64(s)
        else:
            s = e4m3_bits(rng.uniform(0.1, 4, (E, n, G)).astype(np.float32))
            s2 = np.array([0.5, 0.25], np.float32)
            P = hand_problem(fmt, bits, codes, s, s2, x, ids, gs)
            w = R.E2M1_TABLE[c] * R.e4m3_to_f64(s) * s2[:, None, None]
        out, _ = oracle.qmm_id(P, nthreads=1)
        flat = ids.reshape(-1)
        expect = np.stack([w[e] @ Xg[p // 2] for p, e in enumerate(flat)])
        np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("fmt,bits,x_dtype", [
    (FMT_AFFINE, 4, DT_F32), (FMT_AFFINE, 6, DT_BF16), (FMT_AFFINE, 8, DT_F16),
    (FMT_CODEBOOK, 3, DT_F16), (FMT_CODEBOOK, 2, DT_BF16), (FMT_NVFP4, 4, DT_BF16),
])
def test_random_against_numpy_restatement(fmt, bits, x_dtype):
    gs = 16 if fmt == FMT_NVFP4 else 32
    P = make_problem("rand", fmt=fmt, bits=bits, group_size=gs, m=5, k=160, n=24,
                     n_expert_used=3, num_experts=6, x_dtype=x_dtype, out_dtype=DT_F32,
                     seed=77 + bits)
    out, _ = oracle.qmm_id(P, nthreads=3)
    np.testing.assert_allclose(out, R.reference(P), rtol=1e-11, atol=1e-11)
    pairs = np.array([0, 3, 7, 14, 14])
    cols = np.array([0, 23, 5, 1, 22])
    np.testing.assert_array_equal(oracle.qmm_id_sample(P, pairs, cols, nthreads=2),
                                  out[pairs, cols])


def test_tiny_config_against_numpy_restatement():
    P = config_problem("tiny")
    out, bad = oracle.qmm_id(P)
    assert bad == 0
    np.testing.assert_allclose(out, R.reference(P), rtol=1e-12, atol=1e-12)


def test_permutation_invariance():
    P = config_problem("tiny")
    out, _ = oracle.qmm_id(P)
    rng = np.random.default_rng(5)
    perm = rng.permutation(P.n_expert_used)
    Q = P.with_ids(P.ids[:, perm])
    out2, _ = oracle.qmm_id(Q)
    R_ = P.R
    idx = (np.arange(R_) // P.n_expert_used) * P.n_expert_used + np.tile(perm, P.m)
    np.testing.assert_array_equal(out2, out[idx])


def test_out_of_range_ids_give_zero_rows():
    P = config_problem("tiny")
    ids = P.ids.copy()
    ids[1, 0] = P.num_experts
    ids[3, 1] = 0xFFFFFFFF
    out, bad = oracle.qmm_id(P.with_ids(ids))
    assert bad == 2
    assert not out[2].any() and not out[7].any()
    ref, _ = oracle.qmm_id(P)
    keep = [i for i in range(P.R) if i not in (2, 7)]
    np.testing.assert_array_equal(out[keep], ref[keep])


# ------------------------------------------------------------------ routing

@pytest.mark.parametrize("kind", ["uniform", "zipf", "one", "bad", "single"])
def test_route_against_stable_argsort(kind):
    rng = np.random.default_rng(9)
    E, T = 16, 8
    if kind == "uniform":
        ids = rng.integers(0, E, size=300)
    elif kind == "zipf":
        ids = np.minimum(rng.zipf(1.5, size=500) - 1, E - 1)
    elif kind == "one":
        ids = np.full(77, 5)
    elif kind == "bad":
        ids = rng.integers(0, E + 3, size=200)
    else:
        ids = np.array([3])
    ids = ids.astype(np.uint32)
    counts, offsets, sp, tiles = oracle.route(ids, E, T)
    bucket = np.minimum(ids, E)
    np.testing.assert_array_equal(counts, np.bincount(bucket, minlength=E + 1))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    np.testing.assert_array_equal(sp, np.argsort(bucket, kind="stable"))
    expect = [(e, r0) for e in range(E) for r0 in range(0, int(counts[e]), T)]
    assert [tuple(t) for t in tiles.tolist()] == expect


def test_lloyd_max_generator_matches_published_table():
    pub = np.array([float(v) for v in R.golden_lines("lloyd_max_normal_8.txt")])
    np.testing.assert_allclose(lloyd_max_normal(8), pub, atol=1e-4)
