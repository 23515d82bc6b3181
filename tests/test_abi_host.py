"""Host-side checks of the C ABI (no GPU needed): the library loads and exports
every entry point the header declares, sizes follow the storage contract, and
invalid arguments are rejected before any CUDA call."""

import ctypes
import os
import re

import pytest
import torch

import moe_expert_routed_b200 as M
import oracle
from workloads.gen import FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = "".join(open(os.path.join(ROOT, "include", f)).read()
                  for f in sorted(os.listdir(os.path.join(ROOT, "include"))) if f.endswith(".h"))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_symbols_exported():
    names = declared_functions()
    assert "moe_qmm_id" in names and "moe_qmm_id_route" in names
    L = M.lib()
    for name in names:
        assert hasattr(L, name), name


@pytest.mark.parametrize("fmt,bits,k", [(FMT_AFFINE, 4, 2816), (FMT_AFFINE, 4, 704),
                                        (FMT_AFFINE, 6, 2048), (FMT_AFFINE, 6, 5),
                                        (FMT_AFFINE, 8, 100), (FMT_CODEBOOK, 3, 2816),
                                        (FMT_CODEBOOK, 2, 33), (FMT_CODEBOOK, 4, 7),
                                        (FMT_NVFP4, 4, 4096)])
def test_row_bytes_match_oracle(fmt, bits, k):
    assert M.packed_row_bytes(fmt, bits, k) == oracle.row_bytes(fmt, bits, k)


def test_row_bytes_invalid():
    assert M.packed_row_bytes(FMT_AFFINE, 5, 64) == 0
    assert M.packed_row_bytes(FMT_NVFP4, 4, 63) == 0
    assert M.packed_row_bytes(3, 4, 63) == 0      # MXFP4: two codes per byte, k even
    assert M.packed_row_bytes(3, 4, 2816) == 1408
    assert M.packed_row_bytes(3, 3, 64) == 0
    assert M.packed_row_bytes(FMT_CODEBOOK, 8, 64) == 0


def test_workspace_bytes_grows_with_routings():
    a = M.workspace_bytes(1, 8, 128)
    b = M.workspace_bytes(4096, 8, 128)
    assert 0 < a < b and b % 256 == 0


def test_workspace_bytes_with_gathered_x():
    al = lambda v: (v + 255) // 256 * 256
    base = M.workspace_bytes(512, 8, 64)
    f32 = M.workspace_bytes(512, 8, 64, k=1024, x_dtype=torch.float32)
    assert f32 == base + 512 * 8 * 1024 * 4          # f32 x: two bf16 halves per element
    assert M.workspace_bytes(512, 8, 64, k=1028, x_dtype=torch.float32) == base  # k % 8: no room added
    # 16-bit x with 64-pair tiles (fewer than 96 pairs per expert): no room added
    assert M.workspace_bytes(512, 8, 64, k=1024, x_dtype=torch.bfloat16) == base
    # 256-pair tiles: the f16 image, [R/256 + E + 1 tiles][k/64][256 rows][128 B], and one f32 per token
    big = M.workspace_bytes(2048, 8, 64, k=512, x_dtype=torch.float16)
    assert big == M.workspace_bytes(2048, 8, 64) + (16384 // 256 + 64 + 1) * 8 * 256 * 128 + al(2048 * 4)
    # decode-sized calls: no image
    assert M.workspace_bytes(8, 8, 64, k=1024, x_dtype=torch.bfloat16) == M.workspace_bytes(8, 8, 64)
    assert M.workspace_bytes(16, 8, 64, k=1024, x_dtype=torch.bfloat16) == M.workspace_bytes(16, 8, 64)
    assert M.lib().moe_qmm_id_workspace_bytes_k(512, 1024, 8, 64, 3) == 0         # not a moe_dtype


def test_w4a4_workspace_layout():
    """The W4A4 call's own workspace (rounded up to 256 bytes) comes first, then x^ f32,
    the bf16 values, g, the codes and the scales, each rounded up to 256 bytes."""
    al = lambda v: (v + 255) // 256 * 256
    for m, k, topk, E in [(3, 256, 2, 5), (4096, 4096, 8, 128), (17, 48, 1, 1)]:
        front = al(m * k * 4) + al(m * k * 2) + al(m * 4) + al(m * k // 2) + al(m * k // 16)
        assert M.workspace_bytes_w4a4(m, k, topk, E) == al(M.workspace_bytes(m, topk, E)) + front
    L = M.lib()

    def call(wsb, k=256):
        return L.moe_qmm_id_w4a4(16, 16, 16, 16, 16, 16, 4, k, 128, 16, 4, 2, 2, 8, 0, 0, 4096, wsb, None, 0)
    need = M.workspace_bytes_w4a4(4, 256, 2, 8)
    assert call(need - 1) == 3        # one byte short: rejected before any CUDA call
    assert call(64) == 3
    assert call(need, k=250) == 2     # k not a multiple of the 16-value group: unsupported


def test_x_copies_hook_rejects_other_values():
    L = M.lib()
    assert L.moe_qmm_test_x_copies(2) == 1
    assert L.moe_qmm_test_x_copies(-1) == 1
    assert L.moe_qmm_test_x_copies(0) == 0


def _call(**kw):
    args = dict(x=16, ids=16, packed=16, scales=16, aux=16, out=16, m=4, k=256, n=128, gs=32,
                bits=4, fmt=0, topk=2, E=8, xd=0, od=0, ws=4096, wsb=1 << 20, stream=None, path=0)
    args.update(kw)
    L = M.lib()
    return L.moe_qmm_id_path(args["x"], args["ids"], args["packed"], args["scales"], args["aux"],
                             args["out"], args["m"], args["k"], args["n"], args["gs"], args["bits"],
                             args["fmt"], args["topk"], args["E"], args["xd"], args["od"],
                             args["ws"], args["wsb"], args["stream"], args["path"])


@pytest.mark.parametrize("kw", [dict(m=0), dict(k=0), dict(n=0), dict(gs=0), dict(topk=0),
                                dict(E=0), dict(bits=5), dict(bits=3), dict(fmt=4),
                                dict(fmt=3, gs=16), dict(fmt=3, gs=32, k=255), dict(fmt=3, bits=3),
                                dict(fmt=2, bits=4, gs=32), dict(fmt=2, bits=4, gs=16, k=255),
                                dict(fmt=1, bits=8), dict(x=0), dict(ids=0), dict(packed=0),
                                dict(scales=0), dict(aux=0), dict(out=0), dict(ws=0),
                                dict(xd=3), dict(od=-1), dict(path=7), dict(ws=4097)])
def test_invalid_arguments_rejected_before_cuda(kw):
    # all pointers are fake host addresses: any CUDA call would fail or fault, so a
    # clean MOE_ERR_INVALID_ARGUMENT shows validation came first
    assert _call(**kw) == 1


def test_unsupported_and_workspace_errors_before_cuda():
    assert _call(k=250, gs=32) == 2                  # k % group_size != 0
    assert _call(wsb=64) == 3                        # workspace too small


def test_bias_entry_rejects_before_cuda():
    L = M.lib()

    def call(bias=16, bdt=0, m=4):
        return L.moe_qmm_id_bias(16, 16, 16, 16, 16, bias, 16, m, 256, 128, 32, 4, 0, 2, 8, 0, 0, bdt,
                                 4096, 1 << 20, None, 0)
    assert call(bias=0) == 1          # null bias
    assert call(bdt=3) == 1           # unknown bias dtype
    assert call(m=0) == 1             # the operation's own checks still apply


def test_glu_entry_rejects_before_cuda():
    L = M.lib()

    def call(n=128, act=0, bias=16, bdt=0, m=4, path=0):
        return L.moe_qmm_id_glu(16, 16, 16, 16, 16, bias, 16, m, 256, n, 32, 4, 0, 2, 8, 0, 0, bdt, act,
                                4096, 1 << 20, None, path)
    assert call(n=127) == 1           # gate and up halves need an even n
    assert call(act=3) == 1           # unknown activation
    assert call(act=-1) == 1
    assert call(bdt=3) == 1           # unknown bias dtype with a bias
    assert call(m=0) == 1             # the operation's own checks still apply
    assert call(path=5) == 1          # unknown path
    assert call(bias=0, bdt=3, m=0) == 1  # without a bias its dtype is ignored; m=0 still rejected


def test_plan_validation_before_cuda():
    import ctypes
    L = M.lib()
    buf = ctypes.create_string_buffer(24 * 8)

    def init(m=4, n=128, act=-1, bias=None, bdt=0, path=0, ws=4096, wsb=1 << 20):
        return L.moe_qmm_plan_init(buf, 16, 16, 16, bias, m, 256, n, 32, 4, 0, 2, 8, 0, 0, bdt, act, ws, wsb, path)
    assert init(m=0) == 1                 # the operation's own checks
    assert init(act=3) == 1               # unknown activation
    assert init(act=0, n=127) == 1        # gated output needs an even n
    assert init(bias=16, bdt=4) == 1      # unknown bias dtype
    assert init(path=0x400) == 1          # unknown launch flag
    assert init(ws=None) == 1             # no workspace
    assert init(wsb=16) == 3              # workspace too small
    # a plan that failed to initialise is refused by run (no CUDA call is made)
    assert L.moe_qmm_plan_run(buf, 16, 16, 16, None) == 1
    assert L.moe_qmm_plan_run(None, 16, 16, 16, None) == 1
    assert init() == 0                    # valid: only host-side state is written


def test_pointer_table_entry_rejects_before_cuda():
    L = M.lib()

    def call(packed=16, scales=16, biases=16, fmt=0, bits=4, gs=32, path=0):
        return L.moe_qmm_id_ptrs(16, 16, packed, scales, biases, 16, 16, 4, 256, 128, gs, bits, fmt, 2, 8,
                                 0, 0, 4096, 1 << 20, None, path)
    assert call(packed=0) == 1
    assert call(scales=0) == 1
    assert call(biases=0) == 1                    # affine biases come from the table
    assert call(path=7) == 1                      # unknown path
    assert call(path=0x400) == 1                  # unknown launch flag
    assert call(path=0x100 | 3) == 1              # unknown path under a known flag


def test_route_invalid_arguments():
    L = M.lib()
    assert L.moe_qmm_id_route(16, 0, 8, 8, 64, 16, 16, 16, 16, 16, 4096, 1 << 20, None) == 1
    assert L.moe_qmm_id_route(16, 4, 8, 8, 0, 16, 16, 16, 16, 16, 4096, 1 << 20, None) == 1
    assert L.moe_qmm_id_route(16, 4, 8, 2000, 64, 16, 16, 16, 16, 16, 4096, 1 << 20, None) == 2


def test_status_strings():
    for s in range(8):
        assert M.status_str(s) and M.status_str(s) != "unknown status"


def test_binding_requires_cuda_tensors():
    x = torch.zeros(4, 256)
    ids = torch.zeros(4, 2, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        M.qmm_id(x, ids, x, x, x, n=128, group_size=32, bits=4, fmt=0, num_experts=8)
