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
