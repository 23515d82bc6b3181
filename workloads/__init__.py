"""Seeded synthetic inputs for the expert-routed quantized matmul.

This package only draws random numbers and lays them out in the storage formats
the operation reads (raw bits, packed bytes, id arrays). It contains none of the
operation's arithmetic: no code extraction, no dequantisation, no accumulation.
Both the CPU oracle (``oracle/``) and the CUDA library are fed from here.
"""

from .gen import (  # noqa: F401
    FMT_AFFINE,
    FMT_CODEBOOK,
    FMT_NVFP4,
    FMT_MXFP4,
    DT_F32,
    DT_BF16,
    DT_F16,
    Problem,
    make_problem,
    storage_row_bytes,
    lloyd_max_normal,
    distinct_uniform_ids,
    zipf_ids,
)
from .configs import CONFIGS, config_problem  # noqa: F401
