"""The oracle's per-expert output bias step, pinned to its definition
(turboquant fast_switch_patch.py, the switch layer: y + bias[indices]): with all
weights zero the output is the bias row of each pair's expert, exactly; rows of
out-of-range ids stay zero; sampled outputs get the same bias as the full
output; and against an independent NumPy restatement on small problems."""

import numpy as np

import oracle
from tests import numpy_ref as R
from workloads import make_problem
from workloads.gen import DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, expert_bias


def _decode_bias(bias, dt):
    if dt == DT_F32:
        return bias.astype(np.float64)
    return R.bf16_to_f64(bias) if dt == DT_BF16 else R.f16_to_f64(bias)


def _problem(seed, **kw):
    base = dict(fmt=FMT_AFFINE, bits=4, group_size=32, m=6, k=128, n=24, n_expert_used=3,
                num_experts=5, x_dtype=DT_F32, out_dtype=DT_F32, seed=seed)
    base.update(kw)
    return make_problem("bias", **base)


def test_zero_weights_give_the_bias_row_exactly():
    for dt in (DT_F32, DT_BF16, DT_F16):
        P = _problem(11 + dt)
        P.scales[...] = 0
        P.aux[...] = 0  # affine biases: every weight is 0 * c + 0
        ids = P.ids.copy()
        ids[2, 1] = P.num_experts
        P = P.with_ids(ids)
        bias = expert_bias(21 + dt, P.num_experts, P.n, dt)
        out, bad = oracle.qmm_id(P)
        assert bad == 1 and not out.any()
        oracle.add_expert_bias(out.reshape(-1), P, bias, dt)
        b64 = _decode_bias(bias, dt)
        flat = P.ids.reshape(-1)
        for p in range(P.R):
            want = b64[flat[p]] if flat[p] < P.num_experts else np.zeros(P.n)
            assert np.array_equal(out[p], want), (dt, p)


def test_sampled_points_get_the_same_bias():
    P = _problem(31, fmt=FMT_CODEBOOK, bits=3, x_dtype=DT_F16)
    bias = expert_bias(32, P.num_experts, P.n, DT_BF16)
    full, _ = oracle.qmm_id(P)
    full = oracle.add_expert_bias(full.reshape(-1).copy(), P, bias, DT_BF16)
    rng = np.random.default_rng(33)
    pairs = rng.integers(0, P.R, 300)
    cols = rng.integers(0, P.n, 300)
    vals = oracle.qmm_id_sample(P, pairs, cols)
    oracle.add_expert_bias(vals, P, bias, DT_BF16, pairs=pairs, cols=cols)
    assert np.array_equal(vals, full.reshape(P.R, P.n)[pairs, cols])


def test_against_numpy_restatement():
    P = _problem(41, bits=6, group_size=64, k=256, x_dtype=DT_BF16)
    bias = expert_bias(42, P.num_experts, P.n, DT_F16)
    out, _ = oracle.qmm_id(P)
    out = oracle.add_expert_bias(out.reshape(-1).copy(), P, bias, DT_F16).reshape(P.R, P.n)
    ref = R.reference(P).reshape(P.R, P.n) + _decode_bias(bias, DT_F16)[P.ids.reshape(-1)]
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
