"""The oracle's gated-output step (spark_model helpers_a.rs, MoeLayer: the fused
gate+up kernel with SiLU, or GELU for GeGLU experts), pinned to things other than
itself:

* each activation against an independent library routine: SiLU(g) = g * expit(g),
  GELU(g) = g * Phi(g) with Phi the normal CDF, and the tanh form through the
  identity (1 + tanh u) / 2 = expit(2u);
* the symmetry every g * F(g) activation with F(g) + F(-g) = 1 has:
  act(g) - act(-g) = g (a dropped factor or a wrong sign breaks it);
* the row split and its order: with every gate weight 1 and every up weight 2 the
  result is act(S) * 2S, S = sum_j x_j, which the swapped reading act(2S) * S
  does not give; with expert biases b_g, b_u it becomes act(S + b_g) * (2S + b_u);
* rows of out-of-range ids stay zero.
"""

import math

import numpy as np
import pytest
from scipy.special import expit
from scipy.stats import norm

import oracle
from workloads import make_problem
from workloads.gen import DT_F32, FMT_AFFINE, expert_bias

G = np.concatenate([np.linspace(-12.0, 12.0, 241), [-80.0, -30.0, -1e-3, 0.0, 1e-3, 30.0, 80.0]])


def _acts(code):
    return np.array([oracle.act(code, g) for g in G])


def test_silu_is_g_times_the_logistic_function():
    np.testing.assert_allclose(_acts(oracle.ACT_SILU), G * expit(G), rtol=1e-14, atol=1e-300)


# 1 + erf(.) and 1 + tanh(.) cancel for large negative g: the plain formulas keep an
# absolute error of a few units of 1e-16 there, far below any tolerance that uses them
ATOL = 1e-14


def test_gelu_erf_is_g_times_the_normal_cdf():
    np.testing.assert_allclose(_acts(oracle.ACT_GELU_ERF), G * norm.cdf(G), rtol=1e-13, atol=ATOL)


def test_gelu_tanh_through_the_logistic_identity():
    u = math.sqrt(2.0 / math.pi) * (G + 0.044715 * G ** 3)
    np.testing.assert_allclose(_acts(oracle.ACT_GELU_TANH), G * expit(2.0 * u), rtol=1e-13, atol=ATOL)


def test_tanh_form_stays_close_to_the_exact_gelu():
    # the tanh form is a close approximation of g * Phi(g) (error well below 1e-3)
    assert np.max(np.abs(_acts(oracle.ACT_GELU_TANH) - G * norm.cdf(G))) < 1e-3


@pytest.mark.parametrize("code", [oracle.ACT_SILU, oracle.ACT_GELU_TANH, oracle.ACT_GELU_ERF])
def test_odd_part_is_identity(code):
    pos = G[(G > 0) & (G < 40)]
    d = np.array([oracle.act(code, g) - oracle.act(code, -g) for g in pos])
    np.testing.assert_allclose(d, pos, rtol=1e-12, atol=ATOL)
    assert oracle.act(code, 0.0) == 0.0


def test_unknown_activation_is_nan():
    assert math.isnan(oracle.act(3, 1.0))


def _constant_halves(seed, n=16):
    """Affine problem whose gate rows all dequantise to 1 and up rows to 2."""
    P = make_problem("glu", fmt=FMT_AFFINE, bits=4, group_size=32, m=5, k=96, n=n, n_expert_used=3,
                     num_experts=4, x_dtype=DT_F32, out_dtype=DT_F32, seed=seed)
    P.scales[...] = 0
    P.aux[:, : n // 2, :] = 0x3F80  # bf16 1.0
    P.aux[:, n // 2:, :] = 0x4000  # bf16 2.0
    return P


@pytest.mark.parametrize("code,f", [(oracle.ACT_SILU, lambda g: g * expit(g)),
                                    (oracle.ACT_GELU_ERF, lambda g: g * norm.cdf(g)),
                                    (oracle.ACT_GELU_TANH, lambda g: g * expit(
                                        2.0 * math.sqrt(2.0 / math.pi) * (g + 0.044715 * g ** 3)))])
def test_gate_half_then_up_half(code, f):
    P = _constant_halves(31)
    vals, bad = oracle.qmm_id(P)
    assert bad == 0
    got = oracle.glu(vals, code)
    S = P.x.astype(np.float64).sum(axis=1)[np.arange(P.R) // P.n_expert_used]
    want = (f(S) * 2.0 * S)[:, None] * np.ones((1, P.n // 2))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    swapped = (f(2.0 * S) * S)[:, None]
    assert np.max(np.abs(got - swapped)) > 1e-3


def test_bias_enters_before_the_activation():
    P = _constant_halves(32)
    bias = expert_bias(33, P.num_experts, P.n, DT_F32, sigma=0.5)
    vals, _ = oracle.qmm_id(P)
    oracle.add_expert_bias(vals.reshape(-1), P, bias, DT_F32)
    got = oracle.glu(vals, oracle.ACT_SILU)
    e = P.ids.reshape(-1)
    S = P.x.astype(np.float64).sum(axis=1)[np.arange(P.R) // P.n_expert_used][:, None]
    nh = P.n // 2
    g = S + bias[e, :nh].astype(np.float64)
    u = 2.0 * S + bias[e, nh:].astype(np.float64)
    np.testing.assert_allclose(got, g * expit(g) * u, rtol=1e-12, atol=1e-12)


def test_out_of_range_rows_stay_zero():
    P = _constant_halves(34)
    ids = P.ids.copy()
    ids[1, 2] = P.num_experts
    P = P.with_ids(ids)
    vals, bad = oracle.qmm_id(P)
    assert bad == 1
    got = oracle.glu(vals, oracle.ACT_GELU_TANH)
    assert not got[1 * P.n_expert_used + 2].any()
    assert vals[0].all()  # valid pairs have nonzero gate and up sums
