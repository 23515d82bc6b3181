"""Vectorised NumPy restatement of the operation, used only to pin the oracle.

It differs from the oracle in every step that could hide a mistake:
* codes are unpacked from whole little-endian u32 words / 24-bit triplets with
  array shifts (the word-level form of the packing), not bit by bit;
* bf16 / f16 / E4M3 / E8M0 are decoded by torch / numpy dtype casts, E2M1 by
  the OCP table in tests/golden/e2m1_values.txt;
* the contraction is one ``numpy.einsum`` in float64.
"""

from __future__ import annotations

import os

import numpy as np
import torch

from workloads.gen import FMT_AFFINE, FMT_CODEBOOK, FMT_MXFP4, FMT_NVFP4, DT_F32, DT_BF16

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


E2M1_TABLE = np.array([float(v) for v in golden_lines("e2m1_values.txt")], dtype=np.float64)


def bf16_to_f64(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def f16_to_f64(bits):
    return np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def e4m3_to_f64(b):
    t = torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def e8m0_to_f64(b):
    t = torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint8)).view(torch.float8_e8m0fnu)
    return t.to(torch.float64).numpy()


def unpack_codes(packed: np.ndarray, fmt: int, bits: int, k: int) -> np.ndarray:
    """packed [..., row_bytes] -> codes [..., k] (int64)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    lead = packed.shape[:-1]
    if fmt in (FMT_NVFP4, FMT_MXFP4):
        lo = (packed & 0xF).astype(np.int64)
        hi = (packed >> 4).astype(np.int64)
        codes = np.stack([lo, hi], axis=-1).reshape(*lead, -1)
    elif fmt == FMT_AFFINE and bits == 6:
        t = packed.reshape(*lead, -1, 3).astype(np.int64)
        v = t[..., 0] | (t[..., 1] << 8) | (t[..., 2] << 16)
        sh = 6 * np.arange(4)
        codes = ((v[..., None] >> sh) & 63).reshape(*lead, -1)
    else:
        epw = 32 // bits
        words = packed.view("<u4").astype(np.int64)
        sh = bits * np.arange(epw)
        codes = ((words[..., None] >> sh) & ((1 << bits) - 1)).reshape(*lead, -1)
    return codes[..., :k]


def pack_codes(codes: np.ndarray, fmt: int, bits: int) -> np.ndarray:
    """Inverse of unpack_codes for hand-built tests: codes [..., k] -> packed bytes."""
    codes = np.asarray(codes, dtype=np.int64)
    lead, k = codes.shape[:-1], codes.shape[-1]
    if fmt in (FMT_NVFP4, FMT_MXFP4):
        c = np.zeros((*lead, k + (k & 1)), np.int64)
        c[..., :k] = codes
        c = c.reshape(*lead, -1, 2)
        return (c[..., 0] | (c[..., 1] << 4)).astype(np.uint8)
    if fmt == FMT_AFFINE and bits == 6:
        T = (k + 3) // 4
        c = np.zeros((*lead, 4 * T), np.int64)
        c[..., :k] = codes
        c = c.reshape(*lead, T, 4)
        v = c[..., 0] | (c[..., 1] << 6) | (c[..., 2] << 12) | (c[..., 3] << 18)
        out = np.stack([v & 0xFF, (v >> 8) & 0xFF, (v >> 16) & 0xFF], axis=-1)
        return out.reshape(*lead, 3 * T).astype(np.uint8)
    epw = 32 // bits
    W = (k + epw - 1) // epw
    c = np.zeros((*lead, W * epw), np.int64)
    c[..., :k] = codes
    c = c.reshape(*lead, W, epw)
    words = np.zeros((*lead, W), np.int64)
    for i in range(epw):
        words |= c[..., i] << (bits * i)
    return words.astype("<u4").view(np.uint8).reshape(*lead, 4 * W)


def dequant_dense(P) -> np.ndarray:
    """All experts' weights [E, n, k] in float64."""
    codes = unpack_codes(P.packed, P.fmt, P.bits, P.k)
    g = np.arange(P.k) // P.group_size
    if P.fmt == FMT_AFFINE:
        s = bf16_to_f64(P.scales)[..., g]
        b = bf16_to_f64(P.aux)[..., g]
        return codes * s + b
    if P.fmt == FMT_CODEBOOK:
        cb = f16_to_f64(P.aux)
        s = f16_to_f64(P.scales)[..., g]
        return cb[codes] * s
    if P.fmt == FMT_MXFP4:
        return E2M1_TABLE[codes] * e8m0_to_f64(P.scales)[..., g]
    s = e4m3_to_f64(P.scales)[..., g]
    s2 = P.aux.astype(np.float64)[:, None, None]
    return E2M1_TABLE[codes] * s * s2


def x_f64(P) -> np.ndarray:
    if P.x_dtype == 3:  # exact float64 x (the oracle's W4A4 problems)
        return P.x.astype(np.float64)
    if P.x_dtype == DT_F32:
        return P.x.astype(np.float64)
    if P.x_dtype == DT_BF16:
        return bf16_to_f64(P.x)
    return f16_to_f64(P.x)


def reference(P) -> np.ndarray:
    """out [m*n_expert_used, n] float64; out-of-range ids give zero rows."""
    W = dequant_dense(P)
    X = x_f64(P)
    ids = P.ids.reshape(-1).astype(np.int64)
    tok = np.arange(ids.size) // P.n_expert_used
    ok = ids < P.num_experts
    out = np.zeros((ids.size, P.n))
    out[ok] = np.einsum("pnk,pk->pn", W[ids[ok]], X[tok[ok]])
    return out


def dequant_expert(P, e: int) -> np.ndarray:
    """Weights of one expert [n, k] in float64."""
    codes = unpack_codes(P.packed[e], P.fmt, P.bits, P.k)
    g = np.arange(P.k) // P.group_size
    if P.fmt == FMT_AFFINE:
        return codes * bf16_to_f64(P.scales[e])[:, g] + bf16_to_f64(P.aux[e])[:, g]
    if P.fmt == FMT_CODEBOOK:
        return f16_to_f64(P.aux)[codes] * f16_to_f64(P.scales[e])[:, g]
    if P.fmt == FMT_MXFP4:
        return E2M1_TABLE[codes] * e8m0_to_f64(P.scales[e])[:, g]
    return E2M1_TABLE[codes] * e4m3_to_f64(P.scales[e])[:, g] * float(P.aux[e])
