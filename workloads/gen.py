"""Seeded generators for the expert-routed quantized matmul's inputs.

Every array is drawn from ``numpy.random.Generator(PCG64(seed))`` and stored in
the layout the operation reads:

* ``x``       [m, k]: float32 values (f32) or raw uint16 bit patterns (bf16/f16).
* ``ids``     [m, n_expert_used] uint32 expert indices, distinct within a token.
* ``packed``  [E, n, row_bytes] uint8: uniformly random bytes. Every storage
  format here packs codes into whole bits with no redundancy, so random bytes
  are uniformly random codes (padding bits included, which the operation must
  ignore).
* ``scales``  [E, n, ceil(k/group_size)]: bf16 bits (affine), f16 bits
  (codebook), E4M3 bytes (NVFP4, one per 16 values) or E8M0 bytes (MXFP4, one
  per 32 values).
* ``aux``     affine: bf16 bias bits [E, n, G]; codebook: f16 centroid bits
  [2**bits]; NVFP4: float32 scale2 [E]; MXFP4: one unused float32.

Conversions of freshly drawn float32 values to bf16 / f16 / E4M3 bit patterns
use torch/numpy dtype casts (round to nearest even). Nothing here decodes codes
or computes any product of the operation.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch
from scipy.special import ndtr, ndtri

FMT_AFFINE = 0
FMT_CODEBOOK = 1
FMT_NVFP4 = 2
FMT_MXFP4 = 3
DT_F32 = 0
DT_BF16 = 1
DT_F16 = 2

DT_NAMES = {DT_F32: "f32", DT_BF16: "bf16", DT_F16: "f16"}
FMT_NAMES = {FMT_AFFINE: "affine", FMT_CODEBOOK: "codebook", FMT_NVFP4: "nvfp4", FMT_MXFP4: "mxfp4"}


def storage_row_bytes(fmt: int, bits: int, k: int) -> int:
    """Bytes of one packed weight row (the buffer-size contract of the storage).

    Affine 4/8-bit and codebook codes fill whole u32 words (32 // bits codes per
    word, ceil), affine 6-bit fills 3-byte triplets of 4 codes, NVFP4 packs two
    E2M1 codes per byte. (mlx-native ``quantized_matmul_id.rs``,
    ``expert_weight_bytes``; turboquant ``fast_switch_patch.py`` packing.)
    """
    if fmt == FMT_AFFINE and bits == 6:
        return (k + 3) // 4 * 3
    if fmt in (FMT_AFFINE, FMT_CODEBOOK):
        epw = 32 // bits
        return (k + epw - 1) // epw * 4
    if fmt in (FMT_NVFP4, FMT_MXFP4):
        return k // 2
    raise ValueError(f"unknown format {fmt}")


def n_groups(k: int, group_size: int) -> int:
    return (k + group_size - 1) // group_size


def bf16_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f16_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def e4m3_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def lloyd_max_normal(levels: int, iters: int = 2000) -> np.ndarray:
    """Lloyd–Max reconstruction levels of N(0,1) (Max, 1960) by Lloyd iteration.

    Alternate nearest-neighbour thresholds (midpoints) and centroid conditions
    E[Z | t_{i-1} < Z < t_i] = (phi(t_{i-1}) - phi(t_i)) / (Phi(t_i) - Phi(t_{i-1})).
    Used only to build the codebook input.
    """
    y = np.linspace(-2.0, 2.0, levels)
    phi = lambda t: np.exp(-0.5 * t * t) / np.sqrt(2.0 * np.pi)  # noqa: E731
    for _ in range(iters):
        t = np.concatenate(([-np.inf], 0.5 * (y[1:] + y[:-1]), [np.inf]))
        lo, hi = t[:-1], t[1:]
        num = np.where(np.isfinite(lo), phi(lo), 0.0) - np.where(np.isfinite(hi), phi(hi), 0.0)
        y = num / (ndtr(hi) - ndtr(lo))
    return y


def _gumbel_topk(rng: np.random.Generator, logw: np.ndarray, m: int, topk: int) -> np.ndarray:
    """Sequential draws without replacement, P(next = e) proportional to w_e among the
    experts not yet drawn, for m independent tokens: order by log w + Gumbel noise."""
    e = logw.shape[0]
    keys = logw[None, :] + rng.gumbel(size=(m, e))
    order = np.argsort(-keys, axis=1, kind="stable")[:, :topk]
    return order.astype(np.uint32)


def distinct_uniform_ids(rng: np.random.Generator, m: int, topk: int, num_experts: int) -> np.ndarray:
    return _gumbel_topk(rng, np.zeros(num_experts), m, topk)


def zipf_ids(rng: np.random.Generator, m: int, topk: int, num_experts: int, s: float = 1.1) -> np.ndarray:
    """Expert of popularity rank r (1-based) has weight r**-s and id r-1."""
    ranks = np.arange(1, num_experts + 1, dtype=np.float64)
    return _gumbel_topk(rng, -s * np.log(ranks), m, topk)


@dataclass
class Problem:
    name: str
    fmt: int
    bits: int
    group_size: int
    m: int
    k: int
    n: int
    n_expert_used: int
    num_experts: int
    x_dtype: int
    out_dtype: int
    x: np.ndarray
    ids: np.ndarray
    packed: np.ndarray
    scales: np.ndarray
    aux: np.ndarray
    meta: dict = field(default_factory=dict)

    @property
    def R(self) -> int:
        return self.m * self.n_expert_used

    @property
    def row_bytes(self) -> int:
        return storage_row_bytes(self.fmt, self.bits, self.k)

    @property
    def groups(self) -> int:
        return n_groups(self.k, self.group_size)

    def with_ids(self, ids: np.ndarray) -> "Problem":
        ids = np.ascontiguousarray(ids, dtype=np.uint32).reshape(self.m, self.n_expert_used)
        return Problem(**{**self.__dict__, "ids": ids})

    def with_x(self, x: np.ndarray, m: int | None = None) -> "Problem":
        m = x.shape[0] if m is None else m
        return Problem(**{**self.__dict__, "x": np.ascontiguousarray(x), "m": m})


def expert_bias(seed: int, num_experts: int, n: int, dtype: int, sigma: float = 0.05) -> np.ndarray:
    """Per-expert output bias [num_experts, n], N(0, sigma): float32 for DT_F32, else
    the bf16 / f16 bit patterns as uint16."""
    rng = np.random.Generator(np.random.PCG64(seed))
    b = (rng.standard_normal((num_experts, n)) * sigma).astype(np.float32)
    if dtype == DT_F32:
        return b
    return bf16_bits(b) if dtype == DT_BF16 else f16_bits(b)


def _draw_x(rng, m, k, x_dtype):
    xf = rng.standard_normal((m, k), dtype=np.float32)
    if x_dtype == DT_F32:
        return xf
    if x_dtype == DT_BF16:
        return bf16_bits(xf)
    return f16_bits(xf)


def make_problem(
    name: str,
    *,
    fmt: int,
    bits: int,
    group_size: int,
    m: int,
    k: int,
    n: int,
    n_expert_used: int,
    num_experts: int,
    x_dtype: int,
    out_dtype: int,
    seed: int,
    scale_range: tuple[float, float] = (0.002, 0.01),
    bias: str = "normal",
    bias_sigma: float = 0.01,
    ids: str = "uniform",
    zipf_s: float = 1.1,
    scale2: float = 1.0 / 448.0,
    mx_sigma: float = 0.02,
) -> Problem:
    """Draw one problem instance. Order of draws: ids, x, packed codes, scales, aux."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if ids == "uniform":
        id_arr = distinct_uniform_ids(rng, m, n_expert_used, num_experts)
    elif ids == "zipf":
        id_arr = zipf_ids(rng, m, n_expert_used, num_experts, zipf_s)
    else:
        raise ValueError(ids)
    x = _draw_x(rng, m, k, x_dtype)
    rb = storage_row_bytes(fmt, bits, k)
    packed = rng.integers(0, 256, size=(num_experts, n, rb), dtype=np.uint8)
    G = n_groups(k, group_size)
    if fmt == FMT_AFFINE:
        s = rng.uniform(scale_range[0], scale_range[1], size=(num_experts, n, G)).astype(np.float32)
        sb = bf16_bits(s)
        if bias == "neg8s":
            # bias = -8 * scale, taken from the stored (bf16) scale; exact in bf16
            sf = torch.from_numpy(sb.view(np.int16)).view(torch.bfloat16).float().numpy()
            bb = bf16_bits(-8.0 * sf)
        else:
            bb = bf16_bits(rng.normal(0.0, bias_sigma, size=(num_experts, n, G)).astype(np.float32))
        scales, aux = sb, bb
    elif fmt == FMT_CODEBOOK:
        s = rng.uniform(scale_range[0], scale_range[1], size=(num_experts, n, G)).astype(np.float32)
        scales = f16_bits(s)
        aux = f16_bits(lloyd_max_normal(1 << bits).astype(np.float32))
    elif fmt == FMT_NVFP4:
        if group_size != 16:
            raise ValueError("NVFP4 uses 16-value blocks")
        # amax of 16 fresh |N(0,1)| draws, sampled through its CDF (2*Phi(t)-1)**16
        u = rng.random(size=(num_experts, n, G))
        amax = ndtri(0.5 * (1.0 + u ** (1.0 / 16.0)))
        scales = e4m3_bits((amax / 6.0).astype(np.float32))
        aux = np.full((num_experts,), scale2, dtype=np.float32)
    elif fmt == FMT_MXFP4:
        if group_size != 32:
            raise ValueError("MXFP4 uses 32-value blocks")
        # OCP MX shared exponent of a block of 32 weights ~ N(0, mx_sigma^2):
        # floor(log2(amax)) - 2 (E2M1's largest exponent), biased by 127
        u = rng.random(size=(num_experts, n, G))
        amax = mx_sigma * ndtri(0.5 * (1.0 + u ** (1.0 / 32.0)))
        scales = (np.floor(np.log2(amax)) - 2 + 127).clip(0, 254).astype(np.uint8)
        aux = np.zeros((1,), dtype=np.float32)
    else:
        raise ValueError(fmt)
    return Problem(
        name=name, fmt=fmt, bits=bits, group_size=group_size, m=m, k=k, n=n,
        n_expert_used=n_expert_used, num_experts=num_experts, x_dtype=x_dtype,
        out_dtype=out_dtype, x=x, ids=id_arr, packed=packed, scales=scales, aux=aux,
        meta={"seed": seed, "ids": ids},
    )
