"""The benchmark's algorithmic byte count (the numerator of every roofline
fraction it reports) against the figures written out by hand for each workload:
touched experts' codes + scales (+ biases, or scale2) once, x once, out once.

    decode gate/up  8 x 1408 x (1408 + 88 + 88) + 2816*2 + 8*1408*4      = 17,892,864
    decode down     8 x 2816 x (352 + 22 + 22) + 704*2 + 8*2816*4        =  9,012,608
    canvas          128 x 1408 x (1128 + 176) + 256*2816*2 + 2048*1408*4 + 16 = 247,988,240
    prefill         128 x (1536 x (2048 + 256) + 4) + 4096*4096*2 + 32768*1536*2 = 587,203,072
    skewed          256 x 768 x (1536 + 64 + 64) + 8192*2048*4 + 65536*768*4 = 595,591,168
"""

import types

import numpy as np
import pytest

import bench
from workloads import CONFIGS
from workloads.gen import storage_row_bytes


def _shape(name):
    c = CONFIGS[name]
    k, gs = c["k"], c["group_size"]
    return types.SimpleNamespace(
        fmt=c["fmt"], bits=c["bits"], n=c["n"], k=k, m=c["m"], R=c["m"] * c["n_expert_used"],
        num_experts=c["num_experts"], x_dtype=c["x_dtype"], out_dtype=c["out_dtype"],
        row_bytes=storage_row_bytes(c["fmt"], c["bits"], k), groups=(k + gs - 1) // gs)


@pytest.mark.parametrize("name,touched,want", [
    ("decode_gate_up", 8, 17_892_864),
    ("decode_down", 8, 9_012_608),
    ("canvas", 128, 247_988_240),
    ("prefill", 128, 587_203_072),
    ("skewed", 256, 595_591_168),
])
def test_algorithmic_bytes(name, touched, want):
    P = _shape(name)
    ids = np.arange(touched, dtype=np.uint32)  # which experts are touched is all that counts
    assert bench.alg_bytes(P, ids) == want


def test_out_of_range_ids_touch_no_expert():
    P = _shape("decode_gate_up")
    ids = np.array([0, 1, P.num_experts, 0xFFFFFFFF], dtype=np.uint32)
    two = bench.alg_bytes(P, ids[:2])
    assert bench.alg_bytes(P, ids) == two


def test_grouped_launch_counts():
    """Kernels per grouped call, as the bench reports them (gpu_launches): routing
    histogram, scan and scatter, then the GEMM; f32 x adds the gather of its split
    rows (skewed); bf16 x with 256-pair tiles adds the per-token factor and the f16
    image of B (prefill); canvas (64-pair tiles, f16 x) adds nothing."""
    expect = {"canvas": 4, "prefill": 6, "skewed": 5}
    for name, n in expect.items():
        c = CONFIGS[name]
        P = types.SimpleNamespace(m=c["m"], n_expert_used=c["n_expert_used"], num_experts=c["num_experts"],
                                  k=c["k"], x_dtype=c["x_dtype"])
        assert bench.grouped_launches(P) == n, name
