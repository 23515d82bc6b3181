"""Helpers of the GPU parity tests: move a workload to the device, run it through
the C ABI, and compare with the CPU oracle under the per-element tolerance.

Tolerance (the stated bar: max relative error 2e-3, max absolute
1e-2 * |x| * max|w| / sqrt(k)), read per element:
    |y - y_ref| <= atol_t + 2e-3 * |y_ref|,   atol_t = 1e-2 * ||x_t||_2 * max|w_e| / sqrt(k)
with x_t the token's row and max|w_e| the largest |dequantised weight| of the
pair's expert. For bf16 / f16 outputs y_ref is the oracle rounded to that type and
one unit in its last place is added to the bound. Rows of out-of-range ids must
be exactly zero.
"""

from __future__ import annotations

import numpy as np
import torch

import moe_expert_routed_b200 as M
import oracle
from tests import numpy_ref as R
from workloads.gen import DT_BF16, DT_F16, DT_F32
from workloads.torch_io import to_device, x_tensor  # noqa: F401

TORCH_OUT = {DT_F32: torch.float32, DT_BF16: torch.bfloat16, DT_F16: torch.float16}


def run(P, path="auto", dev=None, out=None, workspace=None):
    dev = dev or to_device(P)
    return M.qmm_id(dev["x"], dev["ids"], dev["packed"], dev["scales"], dev["aux"], n=P.n,
                    group_size=P.group_size, bits=P.bits, fmt=P.fmt, num_experts=P.num_experts,
                    out=out, out_dtype=TORCH_OUT[P.out_dtype], workspace=workspace, path=path)


def out_to_f64(out: torch.Tensor) -> np.ndarray:
    return out.detach().float().cpu().numpy().astype(np.float64).reshape(-1, out.shape[-1])


def expert_wmax(P, experts) -> dict:
    return {int(e): float(np.abs(R.dequant_expert(P, int(e))).max()) for e in experts}


def ulp16(v: np.ndarray, dtype: int) -> np.ndarray:
    """Spacing of the 16-bit output type at |v|."""
    a = np.abs(v)
    mbits = 7 if dtype == DT_BF16 else 10
    emin = -126 if dtype == DT_BF16 else -14
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    return np.ldexp(1.0, (e - mbits).astype(np.int64))


def compare(P, got: np.ndarray, ref: np.ndarray, pairs: np.ndarray, cols: np.ndarray):
    """got/ref: values at (pairs[i], cols[i]); ref in double from the oracle.
    Returns (number of violations, worst ratio |err| / bound, details)."""
    ids = P.ids.reshape(-1)[pairs]
    bad_id = ids >= P.num_experts
    X = R.x_f64(P)
    xn = np.linalg.norm(X[pairs // P.n_expert_used], axis=1)
    valid = np.unique(ids[~bad_id])
    wmax = expert_wmax(P, valid)
    wm = np.array([wmax.get(int(e), 0.0) for e in ids])
    atol = 1e-2 * xn * wm / np.sqrt(P.k)
    if P.out_dtype == DT_F32:
        y_ref = ref
        slack = 0.0
    else:
        bits = oracle.round_out(ref, P.out_dtype)
        y_ref = R.bf16_to_f64(bits) if P.out_dtype == DT_BF16 else R.f16_to_f64(bits)
        slack = ulp16(y_ref, P.out_dtype)
    bound = atol + 2e-3 * np.abs(y_ref) + slack
    err = np.abs(got - y_ref)
    viol = (err > bound) & ~bad_id
    viol |= bad_id & (got != 0.0)
    ratio = float(np.max(np.where(bad_id, 0.0, err / np.maximum(bound, 1e-300)))) if got.size else 0.0
    return int(viol.sum()), ratio, dict(max_abs_err=float(err.max()) if err.size else 0.0)


def check_full(P, out: torch.Tensor, nthreads=None):
    """Full-output comparison with the oracle."""
    ref, _ = oracle.qmm_id(P, nthreads=nthreads)
    got = out_to_f64(out)
    pairs = np.repeat(np.arange(P.R), P.n)
    cols = np.tile(np.arange(P.n), P.R)
    return compare(P, got.reshape(-1), ref.reshape(-1), pairs, cols)


def check_sampled(P, out: torch.Tensor, pairs: np.ndarray, cols: np.ndarray, nthreads=None):
    ref = oracle.qmm_id_sample(P, pairs, cols, nthreads=nthreads)
    got = out_to_f64(out)[pairs, cols]
    return compare(P, got, ref, pairs, cols)


def bias_tensor(bias: np.ndarray, bias_dtype: int) -> torch.Tensor:
    """Device tensor of a per-expert bias array from workloads.gen.expert_bias."""
    if bias_dtype == DT_F32:
        return torch.from_numpy(bias).cuda()
    t = torch.from_numpy(bias.view(np.int16)).cuda()
    return t.view(torch.bfloat16 if bias_dtype == DT_BF16 else torch.float16)


def run_bias(P, bias: np.ndarray, bias_dtype: int, path="auto", dev=None, out=None, workspace=None):
    dev = dev or to_device(P)
    return M.qmm_id(dev["x"], dev["ids"], dev["packed"], dev["scales"], dev["aux"], n=P.n,
                    group_size=P.group_size, bits=P.bits, fmt=P.fmt, num_experts=P.num_experts,
                    out=out, out_dtype=TORCH_OUT[P.out_dtype], workspace=workspace, path=path,
                    expert_bias=bias_tensor(bias, bias_dtype))


def check_full_bias(P, out: torch.Tensor, bias: np.ndarray, bias_dtype: int, nthreads=None):
    """Full-output comparison with the oracle plus its per-expert bias step."""
    ref, _ = oracle.qmm_id(P, nthreads=nthreads)
    ref = oracle.add_expert_bias(ref.reshape(-1).copy(), P, bias, bias_dtype)
    got = out_to_f64(out)
    pairs = np.repeat(np.arange(P.R), P.n)
    cols = np.tile(np.arange(P.n), P.R)
    return compare(P, got.reshape(-1), ref, pairs, cols)


# ------------------------------------------------------------ gated (GLU) output
#
# out[p][c] = act(g) * u with g, u the pair's results in gate row c and up row
# n/2 + c (bias included). With Bg, Bu the per-element bounds above for g and u
# (atol_t + 2e-3 |y|), the bound on z = act(g) * u is their first-order
# propagation through |act'| <= 1.2 (SiLU's slope stays below 1.1, GELU's below
# 1.13), the second-order term |act''| <= 0.8 (GELU's curvature peaks at
# 2 * phi(0) = 0.80), the cross term, and the fp32 evaluation of the activation:
# a few ulp relative, plus an absolute 1e-6 |g| |u| where 1 + tanh(.) or
# 1 + erf(.) cancels for negative g. 16-bit outputs add one unit in their last
# place after rounding the oracle's z.
ACT_CODE = {"silu": 0, "gelu_tanh": 1, "gelu_erf": 2}


def run_glu(P, act: str, path="auto", bias=None, bias_dtype=DT_F32, dev=None, out=None, workspace=None):
    dev = dev or to_device(P)
    return M.qmm_id(dev["x"], dev["ids"], dev["packed"], dev["scales"], dev["aux"], n=P.n,
                    group_size=P.group_size, bits=P.bits, fmt=P.fmt, num_experts=P.num_experts,
                    out=out, out_dtype=TORCH_OUT[P.out_dtype], workspace=workspace, path=path,
                    expert_bias=bias_tensor(bias, bias_dtype) if bias is not None else None, act=act)


def compare_glu(P, act: str, got: np.ndarray, g_ref: np.ndarray, u_ref: np.ndarray, pairs: np.ndarray):
    """got/g_ref/u_ref at the same output elements of pairs[i]; refs in double."""
    ids = P.ids.reshape(-1)[pairs]
    bad_id = ids >= P.num_experts
    X = R.x_f64(P)
    xn = np.linalg.norm(X[pairs // P.n_expert_used], axis=1)
    wmax = expert_wmax(P, np.unique(ids[~bad_id]))
    wm = np.array([wmax.get(int(e), 0.0) for e in ids])
    atol = 1e-2 * xn * wm / np.sqrt(P.k)
    bg = atol + 2e-3 * np.abs(g_ref)
    bu = atol + 2e-3 * np.abs(u_ref)
    code = ACT_CODE[act]
    z = oracle.glu_elems(g_ref, u_ref, code)
    ag = np.abs(oracle.glu_elems(g_ref, np.ones_like(g_ref), code))
    if P.out_dtype == DT_F32:
        z_ref, slack = z, 0.0
    else:
        bits = oracle.round_out(z, P.out_dtype)
        z_ref = R.bf16_to_f64(bits) if P.out_dtype == DT_BF16 else R.f16_to_f64(bits)
        slack = ulp16(z_ref, P.out_dtype)
    au = np.abs(u_ref)
    bound = (1.2 * au * bg + ag * bu + 1.2 * bg * bu + 0.4 * bg * bg * (au + bu)
             + 4e-6 * np.abs(z) + 1e-6 * np.abs(g_ref) * au + slack)
    err = np.abs(got - z_ref)
    viol = (err > bound) & ~bad_id
    viol |= bad_id & (got != 0.0)
    ratio = float(np.max(np.where(bad_id, 0.0, err / np.maximum(bound, 1e-300)))) if got.size else 0.0
    return int(viol.sum()), ratio, dict(max_abs_err=float(err.max()) if err.size else 0.0)


def check_full_glu(P, act: str, out: torch.Tensor, bias=None, bias_dtype=DT_F32, nthreads=None):
    """Full gated output against the oracle (plus its bias step) and its glu step."""
    ref, _ = oracle.qmm_id(P, nthreads=nthreads)
    if bias is not None:
        oracle.add_expert_bias(ref.reshape(-1), P, bias, bias_dtype)
    nh = P.n // 2
    got = out_to_f64(out).reshape(P.R, nh)
    pairs = np.repeat(np.arange(P.R), nh)
    return compare_glu(P, act, got.reshape(-1), ref[:, :nh].reshape(-1), ref[:, nh:].reshape(-1), pairs)


def check_sampled_glu(P, act: str, out: torch.Tensor, pairs: np.ndarray, cols: np.ndarray, nthreads=None):
    """Sampled gated outputs (pairs[i], cols[i] < n/2) against the oracle's elements."""
    nh = P.n // 2
    g = oracle.qmm_id_sample(P, pairs, cols, nthreads=nthreads)
    u = oracle.qmm_id_sample(P, pairs, cols + nh, nthreads=nthreads)
    got = out_to_f64(out).reshape(P.R, nh)[pairs, cols]
    return compare_glu(P, act, got, g, u, pairs)
