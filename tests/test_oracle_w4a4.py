"""Pins of the oracle's W4A4 activation quantisation (NVFP4 activations: per token
g = amax / 2688, per 16 values an E4M3 scale, E2M1 codes; the reading is stated in
oracle/oracle.c) and of the matmul on the exact dequantised x^.

- E2M1 rounding against the ties-to-even cases worked out by hand from the OCP
  Microscaling definition (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; even = low code bit 0).
- E4M3 rounding against torch's float8_e4m3fn cast, and saturation at 448.
- Tokens built to be exactly representable (power-of-two g, a block at scale 448,
  a code of magnitude 6 in every block) come back bit for bit: this fixes the 2688,
  the 6 in the block scale, the nibble order and x^.
- Random tokens: every code is the nearest E2M1 value of x / d, each block's largest
  element takes magnitude 6 unless its scale underflowed, zero tokens and blocks give
  zero codes.
- The matmul on x^ (oracle x dtype float64) against the NumPy restatement.
"""

import numpy as np
import pytest
import torch

import oracle
from tests import numpy_ref as R
from workloads import make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_NVFP4, bf16_bits

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@pytest.mark.parametrize("v,code", [
    (0.0, 0), (0.5, 1), (1.0, 2), (1.5, 3), (2.0, 4), (3.0, 5), (4.0, 6), (6.0, 7),
    # midpoints: ties to the even code
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
    # just off the midpoints
    (0.2500001, 1), (0.7499999, 1), (4.9999995, 6), (5.0000005, 7),
    # saturation and sign
    (6.5, 7), (1e30, 7), (-0.75, 10), (-6.0, 15), (-1e30, 15), (-0.1, 8),
])
def test_e2m1_rounding(v, code):
    assert oracle.e2m1_rne(np.float32(v)) == code


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(3)
    v = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000)).astype(np.float32)
    v = np.concatenate([v, np.float32([0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 448.0, 1.0625, 1.1875])])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rne_satfinite(x) for x in v], np.uint8)
    np.testing.assert_array_equal(got, ref)
    assert oracle.e4m3_rne_satfinite(np.float32(449.0)) == 0x7E
    assert oracle.e4m3_rne_satfinite(np.float32(1e20)) == 0x7E


def _representable(rng, k, g_exp):
    """A token x = e2m1(q) * e4m3(s_b) * g with g = 2^g_exp, block 0 at s = 448 and a
    code of magnitude 6 in every block; returns (x f32, codes, scales)."""
    nb = k // 16
    s = rng.integers(0x08, 0x7E, nb).astype(np.uint8)   # normal E4M3 scales
    s[0] = 0x7E                                           # 448: the token's largest block
    q = rng.integers(0, 16, k).astype(np.uint8)
    for b in range(nb):
        q[16 * b + rng.integers(0, 16)] = 7 | (rng.integers(0, 2) << 3)   # +-6 in every block
    sv = np.array([oracle.e4m3_to_double(int(b)) for b in s])
    x = np.array([oracle.e2m1_to_double(int(c)) for c in q]) * np.repeat(sv, 16) * 2.0 ** g_exp
    return x.astype(np.float32), q, s


@pytest.mark.parametrize("g_exp", [-12, -3, 0])
def test_representable_tokens_round_trip(g_exp):
    rng = np.random.default_rng(40 + g_exp)
    m, k = 3, 96
    rows = [_representable(rng, k, g_exp) for _ in range(m)]
    x = np.stack([r[0] for r in rows])
    codes, scales, g, xhat = oracle.quantize_act_nvfp4(x, DT_F32, m, k)
    np.testing.assert_array_equal(g, np.float32(2.0 ** g_exp))
    for t, (xt, q, s) in enumerate(rows):
        np.testing.assert_array_equal(scales[t], s)
        # nibble order: element 2i low, 2i+1 high; -0 and +0 are the same value
        got_q = np.stack([codes[t] & 15, codes[t] >> 4], axis=1).reshape(-1)
        mag = lambda c: np.where((c & 7) == 0, 0, c)
        np.testing.assert_array_equal(mag(got_q), mag(q))
        np.testing.assert_array_equal(xhat[t], xt.astype(np.float64))


@pytest.mark.parametrize("xd", [DT_F32, DT_BF16, DT_F16])
def test_random_tokens_nearest_codes(xd):
    rng = np.random.default_rng(7 + xd)
    m, k = 6, 256
    xf = (rng.standard_normal((m, k)) * np.exp(rng.uniform(-6, 6, (m, 1)))).astype(np.float32)
    xf[2, 32:48] = 0.0                       # an all-zero block
    xf[4] = 0.0                              # an all-zero token
    xf[5, 0] = 1e4                           # a dominant value: other blocks' scales underflow
    if xd == DT_F32:
        x = xf
    elif xd == DT_BF16:
        x = bf16_bits(xf)
    else:
        x = xf.astype(np.float16).view(np.uint16)
    xv = R.x_f64(make_problem_stub(x, xd)).astype(np.float32).reshape(m, k)
    codes, scales, g, xhat = oracle.quantize_act_nvfp4(x, xd, m, k)
    q = np.stack([codes & 15, codes >> 4], axis=2).reshape(m, k)
    for t in range(m):
        a = np.abs(xv[t]).max()
        assert g[t] == np.float32(a) / np.float32(2688.0)
        for b in range(k // 16):
            blk = slice(16 * b, 16 * b + 16)
            sv = np.float32(oracle.e4m3_to_double(int(scales[t, b])))
            d = np.float32(sv * g[t])
            if d == 0:
                assert np.all(q[t, blk] & 7 == 0) and np.all(xhat[t, blk] == 0)
                continue
            r = np.abs(xv[t, blk] / d)
            mag = E2M1[q[t, blk] & 7]
            err = np.abs(np.minimum(r, 6.0) - mag)
            nearest = np.min(np.abs(np.minimum(r, 6.0)[:, None] - E2M1[None, :]), axis=1)
            np.testing.assert_allclose(err, nearest, rtol=0, atol=0)
            assert mag[np.argmax(r)] == 6.0 or sv == np.float32(oracle.e4m3_to_double(0x7E))
            sign = (q[t, blk] >> 3) & 1
            nz = mag > 0
            np.testing.assert_array_equal(sign[nz], (xv[t, blk] < 0)[nz])
    assert np.all(xhat[4] == 0) and g[4] == 0


def make_problem_stub(x, xd):
    class S:
        pass
    s = S()
    s.x, s.x_dtype = x, xd
    return s


def test_w4a4_matmul_on_exact_xhat_matches_numpy():
    P = make_problem("w4a4-pin", seed=91, fmt=FMT_NVFP4, bits=4, group_size=16, m=5, k=128, n=24,
                     n_expert_used=2, num_experts=4, x_dtype=DT_BF16, out_dtype=DT_F32)
    Q = oracle.w4a4_problem(P)
    out, bad = oracle.qmm_id(Q, nthreads=2)
    assert bad == 0
    np.testing.assert_allclose(out, R.reference(Q), rtol=1e-12, atol=1e-12)
    # and it is not the W4A16 result
    assert not np.allclose(out, oracle.qmm_id(P, nthreads=2)[0], rtol=1e-6, atol=0)
