"""CPU oracle for the expert-routed quantized matmul (ctypes wrapper of oracle.c).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py``. The product package never
imports it.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc into liboracle.so (plain -O2, IEEE double)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
             "-o", _LIB, _SRC, "-lm", "-lpthread"]
        )
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        u8p, u16p, u32p, dp, vp = (ctypes.POINTER(t) for t in
                                   (ctypes.c_uint8, ctypes.c_uint16, ctypes.c_uint32,
                                    ctypes.c_double, ctypes.c_void_p))
        u32, u64, i32 = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_double.restype = ctypes.c_double
        L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_double.restype = ctypes.c_double
        L.oracle_e8m0_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e8m0_to_double.restype = ctypes.c_double
        L.oracle_e2m1_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_to_double.restype = ctypes.c_double
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_double_to_f16.argtypes = [ctypes.c_double]
        L.oracle_double_to_f16.restype = ctypes.c_uint16
        L.oracle_round_out.argtypes = [ctypes.c_void_p, ctypes.c_void_p, u64, i32]
        L.oracle_round_out.restype = None
        L.oracle_row_bytes.argtypes = [i32, i32, u32]
        L.oracle_row_bytes.restype = u64
        L.oracle_code.argtypes = [ctypes.c_void_p, i32, i32, u32]
        L.oracle_code.restype = u32
        common = [u32, u32, u32, u32, u32, i32, u32, u32, i32, i32]
        L.oracle_qmm_id.argtypes = [ctypes.c_void_p] * 6 + common
        L.oracle_qmm_id.restype = ctypes.c_int64
        L.oracle_qmm_id_sample.argtypes = [ctypes.c_void_p] * 7 + [u64, ctypes.c_void_p] + common
        L.oracle_qmm_id_sample.restype = i32
        L.oracle_expert_max_abs_weight.argtypes = [ctypes.c_void_p] * 3 + [u32, u32, u32, u32,
                                                                            u32, i32, u32]
        L.oracle_expert_max_abs_weight.restype = ctypes.c_double
        L.oracle_add_expert_bias.argtypes = [ctypes.c_void_p] * 3 + [u64] + [ctypes.c_void_p] * 2 + [i32, u32, u32]
        L.oracle_add_expert_bias.restype = None
        L.oracle_route.argtypes = [ctypes.c_void_p, u64, u32, u32, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, u64]
        L.oracle_route.restype = ctypes.c_int64
        L.oracle_act.argtypes = [i32, ctypes.c_double]
        L.oracle_act.restype = ctypes.c_double
        L.oracle_glu_elems.argtypes = [ctypes.c_void_p] * 2 + [u64, i32, ctypes.c_void_p]
        L.oracle_glu_elems.restype = None
        L.oracle_e2m1_rne.argtypes = [ctypes.c_float]
        L.oracle_e2m1_rne.restype = ctypes.c_uint8
        L.oracle_e4m3_rne_satfinite.argtypes = [ctypes.c_float]
        L.oracle_e4m3_rne_satfinite.restype = ctypes.c_uint8
        L.oracle_quantize_act_nvfp4.argtypes = [ctypes.c_void_p, i32, u32, u32] + [ctypes.c_void_p] * 4
        L.oracle_quantize_act_nvfp4.restype = i32
        del u8p, u16p, u32p, dp, vp
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1


# ------------------------------------------------------------------ decoders

def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


def f16_to_double(bits: int) -> float:
    return lib().oracle_f16_to_double(int(bits))


def e4m3_to_double(b: int) -> float:
    return lib().oracle_e4m3_to_double(int(b))


def e8m0_to_double(b: int) -> float:
    return lib().oracle_e8m0_to_double(int(b))


def e2m1_to_double(c: int) -> float:
    return lib().oracle_e2m1_to_double(int(c))


def double_to_bf16(v: float) -> int:
    return lib().oracle_double_to_bf16(float(v))


def double_to_f16(v: float) -> int:
    return lib().oracle_double_to_f16(float(v))


def round_out(vals: np.ndarray, out_dtype: int) -> np.ndarray:
    """Round doubles to the output dtype's storage: float32 array, or uint16 bits."""
    vals = np.ascontiguousarray(vals, dtype=np.float64)
    out = np.empty(vals.shape, dtype=np.float32 if out_dtype == 0 else np.uint16)
    lib().oracle_round_out(_ptr(vals), _ptr(out), vals.size, out_dtype)
    return out


def row_bytes(fmt: int, bits: int, k: int) -> int:
    return lib().oracle_row_bytes(fmt, bits, k)


def code(row: np.ndarray, fmt: int, bits: int, j: int) -> int:
    row = np.ascontiguousarray(row, dtype=np.uint8)
    return lib().oracle_code(_ptr(row), fmt, bits, j)


# ------------------------------------------------------------------ operation

def _common(P):
    return [P.m, P.k, P.n, P.group_size, P.bits, P.fmt, P.n_expert_used, P.num_experts,
            P.x_dtype]


def _arrays(P):
    return [np.ascontiguousarray(a) for a in (P.x, P.ids, P.packed, P.scales, P.aux)]


def qmm_id(P, nthreads: int | None = None):
    """Full output, double [m*n_expert_used, n]; returns (out, number of bad ids)."""
    arrs = _arrays(P)
    out = np.empty((P.R, P.n), dtype=np.float64)
    rc = lib().oracle_qmm_id(*[_ptr(a) for a in arrs], _ptr(out), *_common(P),
                             nthreads or default_threads())
    if rc < 0:
        raise ValueError("oracle rejected the problem")
    return out, int(rc)


def qmm_id_sample(P, pairs: np.ndarray, cols: np.ndarray, nthreads: int | None = None):
    """out[pairs[i], cols[i]] in double."""
    arrs = _arrays(P)
    pairs = np.ascontiguousarray(pairs, dtype=np.uint32)
    cols = np.ascontiguousarray(cols, dtype=np.uint32)
    vals = np.empty(pairs.shape, dtype=np.float64)
    rc = lib().oracle_qmm_id_sample(*[_ptr(a) for a in arrs], _ptr(pairs), _ptr(cols),
                                    pairs.size, _ptr(vals), *_common(P),
                                    nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the sample")
    return vals


def add_expert_bias(vals: np.ndarray, P, bias: np.ndarray, bias_dtype: int, pairs=None, cols=None):
    """vals (double, from qmm_id or qmm_id_sample) += bias[ids[p]][col] for valid ids,
    in place; bias [num_experts, n] raw storage (float32, or uint16 bits of bf16/f16)."""
    assert vals.dtype == np.float64 and vals.flags["C_CONTIGUOUS"]
    ids = np.ascontiguousarray(P.ids.reshape(-1), dtype=np.uint32)
    bias = np.ascontiguousarray(bias)
    if pairs is not None:
        pairs = np.ascontiguousarray(pairs, dtype=np.uint32)
        cols = np.ascontiguousarray(cols, dtype=np.uint32)
    lib().oracle_add_expert_bias(_ptr(vals), _ptr(pairs) if pairs is not None else None,
                                 _ptr(cols) if cols is not None else None, vals.size, _ptr(ids),
                                 _ptr(bias), bias_dtype, P.n, P.num_experts)
    return vals


ACT_SILU, ACT_GELU_TANH, ACT_GELU_ERF = 0, 1, 2


def act(code: int, g: float) -> float:
    """Activation of the gated output in double (0 SiLU, 1 GELU tanh form, 2 GELU erf form)."""
    return lib().oracle_act(int(code), float(g))


def glu_elems(gate: np.ndarray, up: np.ndarray, code: int) -> np.ndarray:
    """act(gate) * up elementwise, double."""
    gate = np.ascontiguousarray(gate, dtype=np.float64)
    up = np.ascontiguousarray(up, dtype=np.float64)
    assert gate.shape == up.shape
    out = np.empty(gate.shape, dtype=np.float64)
    lib().oracle_glu_elems(_ptr(gate), _ptr(up), gate.size, int(code), _ptr(out))
    return out


def glu(vals: np.ndarray, code: int) -> np.ndarray:
    """Gated output of full results vals [R, n] (double, bias already added): rows
    [0, n/2) of an expert are the gate, [n/2, n) the up projection; returns
    act(gate) * up, [R, n/2] double."""
    R, n = vals.shape
    assert n % 2 == 0
    nh = n // 2
    return glu_elems(vals[:, :nh], vals[:, nh:], code)


def expert_max_abs_weight(P, e: int) -> float:
    arrs = _arrays(P)
    return lib().oracle_expert_max_abs_weight(_ptr(arrs[2]), _ptr(arrs[3]), _ptr(arrs[4]), e,
                                              P.k, P.n, P.group_size, P.bits, P.fmt,
                                              P.num_experts)


def route(ids: np.ndarray, num_experts: int, tile_rows: int):
    """Reference routing: counts[E+1], offsets[E+2], sorted_pairs[R], tiles[ntiles, 2]."""
    ids = np.ascontiguousarray(ids, dtype=np.uint32).reshape(-1)
    R = ids.size
    counts = np.zeros(num_experts + 1, np.uint32)
    offsets = np.zeros(num_experts + 2, np.uint32)
    sp = np.zeros(max(R, 1), np.uint32)
    max_tiles = R // tile_rows + num_experts + 1
    tiles = np.zeros((max_tiles, 2), np.uint32)
    nt = lib().oracle_route(_ptr(ids), R, num_experts, tile_rows, _ptr(counts), _ptr(offsets),
                            _ptr(sp), _ptr(tiles), max_tiles)
    if nt < 0:
        raise ValueError("tile list overflow")
    return counts, offsets, sp[:R], tiles[:nt]


# ------------------------------------------------- W4A4 (NVFP4 activations)

DT_F64 = 3  # oracle-only x dtype: x given exactly as float64


def e2m1_rne(v: float) -> int:
    """Nearest E2M1 code of the f32 value v (ties to even, saturating at 6)."""
    return int(lib().oracle_e2m1_rne(float(v)))


def e4m3_rne_satfinite(v: float) -> int:
    """Nearest finite E4M3 code of the f32 value v >= 0 (ties to even, saturating at 448)."""
    return int(lib().oracle_e4m3_rne_satfinite(float(v)))


def quantize_act_nvfp4(x: np.ndarray, x_dtype: int, m: int, k: int):
    """Per-token NVFP4 quantisation of x [m, k] (raw storage): returns codes [m, k/2]
    uint8 (element 2i in the low nibble), E4M3 block scales [m, k/16] uint8, the
    per-token f32 scale [m] and the exact dequantised x^ [m, k] float64."""
    x = np.ascontiguousarray(x)
    codes = np.zeros((m, k // 2), np.uint8)
    scales = np.zeros((m, k // 16), np.uint8)
    g = np.zeros(m, np.float32)
    xhat = np.zeros((m, k), np.float64)
    if lib().oracle_quantize_act_nvfp4(_ptr(x), int(x_dtype), m, k, _ptr(codes), _ptr(scales), _ptr(g),
                                       _ptr(xhat)) != 0:
        raise ValueError("k must be a positive multiple of 16")
    return codes, scales, g, xhat


def w4a4_problem(P):
    """The problem the W4A4 operation computes: P with x replaced by its NVFP4
    quantisation x^ (float64, exact)."""
    import dataclasses
    _, _, _, xhat = quantize_act_nvfp4(P.x, P.x_dtype, P.m, P.k)
    return dataclasses.replace(P, x=xhat, x_dtype=DT_F64)
