"""The five synthetic workloads, with the sizes and value distributions of the
pages' configurations, plus the decode m=1..8 sweep.

Seeds: tiny=1, decode=2, canvas=3, prefill=4, skewed=5 (the decode "down"
projection uses seed 2 with a different stream offset).
"""

from __future__ import annotations

from .gen import (
    DT_BF16, DT_F16, DT_F32, FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4, Problem, make_problem,
)

CONFIGS = {
    # 8 experts, top-2, m=4, k=256, n=128, affine 4-bit, group 32, bias = -8*scale
    "tiny": dict(fmt=FMT_AFFINE, bits=4, group_size=32, m=4, k=256, n=128, n_expert_used=2,
                 num_experts=8, x_dtype=DT_F32, out_dtype=DT_F32, seed=1,
                 scale_range=(0.005, 0.02), bias="neg8s"),
    # MoE decode, gate/up projection: 128 experts, top-8, k=2816, n=1408, affine 4-bit g64
    "decode_gate_up": dict(fmt=FMT_AFFINE, bits=4, group_size=64, m=1, k=2816, n=1408,
                           n_expert_used=8, num_experts=128, x_dtype=DT_BF16, out_dtype=DT_F32,
                           seed=2, scale_range=(0.002, 0.01), bias="normal"),
    # MoE decode, down projection: k=704, n=2816
    "decode_down": dict(fmt=FMT_AFFINE, bits=4, group_size=64, m=1, k=704, n=2816,
                        n_expert_used=8, num_experts=128, x_dtype=DT_BF16, out_dtype=DT_F32,
                        seed=2 + (1 << 20), scale_range=(0.002, 0.01), bias="normal"),
    # canvas switch call: 256 tokens x top-8, 3-bit codebook g32, fp16 scales U[0.01,0.05]
    "canvas": dict(fmt=FMT_CODEBOOK, bits=3, group_size=32, m=256, k=2816, n=1408,
                   n_expert_used=8, num_experts=128, x_dtype=DT_F16, out_dtype=DT_F32, seed=3,
                   scale_range=(0.01, 0.05)),
    # prefill grouped GEMM, NVFP4 W4A16, bf16 out
    "prefill": dict(fmt=FMT_NVFP4, bits=4, group_size=16, m=4096, k=4096, n=1536,
                    n_expert_used=8, num_experts=128, x_dtype=DT_BF16, out_dtype=DT_BF16, seed=4),
    # skewed routing: Zipf(1.1) popularity, 6-bit affine g64, f32 x
    "skewed": dict(fmt=FMT_AFFINE, bits=6, group_size=64, m=8192, k=2048, n=768, n_expert_used=8,
                   num_experts=256, x_dtype=DT_F32, out_dtype=DT_F32, seed=5,
                   scale_range=(0.002, 0.01), bias="normal", ids="zipf", zipf_s=1.1),
}


def config_problem(name: str, **overrides) -> Problem:
    """Build a named workload; keyword overrides replace any field (e.g. m, seed)."""
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    return make_problem(name, **cfg)
