"""Expert-routed (MoE) quantized matmul for NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in ``include/moe_qmm.h`` (``libmoe_qmm.so``,
built in-tree by ``moe_expert_routed_b200.build``). The binding checks tensor
shapes, dtypes, devices and buffer lengths, then passes raw device pointers and
the current CUDA stream to the library; every step of the computation runs in
the library's kernels. There is no fallback: if the library is missing or a
tensor is not on a CUDA device, calls raise.

    out = qmm_id(x, ids, packed, scales, aux, n=..., group_size=..., bits=...,
                 fmt=FMT_AFFINE, num_experts=...)
    # for every pair p = token*n_expert_used + slot, e = ids[p]:
    #   out[token, slot, col] = sum_j dequant(W[e, col, j]) * x[token, j]
"""

from __future__ import annotations

import ctypes
import functools
import os

import torch

FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4, FMT_MXFP4 = 0, 1, 2, 3
DT_F32, DT_BF16, DT_F16 = 0, 1, 2
PATH_AUTO, PATH_DECODE, PATH_GROUPED = 0, 1, 2
_PATHS = {"auto": PATH_AUTO, "decode": PATH_DECODE, "grouped": PATH_GROUPED}
ACT_SILU, ACT_GELU_TANH, ACT_GELU_ERF = 0, 1, 2
# launch flags OR-ed into the path argument (programmatic dependent launch)
LAUNCH_PDL, LAUNCH_EARLY_WEIGHTS = 0x100, 0x200
_LAUNCH = {None: 0, "pdl": LAUNCH_PDL, "early_weights": LAUNCH_PDL | LAUNCH_EARLY_WEIGHTS}
ACTS = {"silu": ACT_SILU, "gelu_tanh": ACT_GELU_TANH, "gelu_erf": ACT_GELU_ERF}

MOE_OK = 0
STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARGUMENT", 2: "MOE_ERR_UNSUPPORTED",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_BAD_EXPERT_ID",
    6: "MOE_ERR_TIMEOUT", 7: "MOE_ERR_BAD_EXPERT_POINTER",
}

_TORCH_DT = {torch.float32: DT_F32, torch.bfloat16: DT_BF16, torch.float16: DT_F16}
_DT_TORCH = {v: k for k, v in _TORCH_DT.items()}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_qmm.so")
_lib = None


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({status_str(status)})")


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m moe_expert_routed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, u32, sz, i32 = ctypes.c_void_p, ctypes.c_uint32, ctypes.c_size_t, ctypes.c_int
        L.moe_qmm_id.argtypes = [vp] * 6 + [u32] * 5 + [i32, u32, u32, i32, i32, vp, sz, vp]
        L.moe_qmm_id.restype = i32
        L.moe_qmm_id_path.argtypes = L.moe_qmm_id.argtypes + [i32]
        L.moe_qmm_id_bias.argtypes = [vp] * 7 + [u32] * 5 + [i32, u32, u32, i32, i32, i32, vp, sz, vp, i32]
        L.moe_qmm_id_bias.restype = i32
        L.moe_qmm_id_ptrs.argtypes = [vp] * 7 + [u32] * 5 + [i32, u32, u32, i32, i32, vp, sz, vp, i32]
        L.moe_qmm_id_ptrs.restype = i32
        L.moe_qmm_id_glu.argtypes = [vp] * 7 + [u32] * 5 + [i32, u32, u32, i32, i32, i32, i32, vp, sz, vp, i32]
        L.moe_qmm_id_glu.restype = i32
        L.moe_qmm_plan_init.argtypes = [vp] * 5 + [u32] * 5 + [i32, u32, u32, i32, i32, i32, i32, vp, sz, i32]
        L.moe_qmm_plan_init.restype = i32
        L.moe_qmm_plan_run.argtypes = [vp] * 5
        L.moe_qmm_plan_run.restype = i32
        L.moe_qmm_id_path.restype = i32
        L.moe_qmm_id_workspace_bytes.argtypes = [u32, u32, u32]
        L.moe_qmm_id_workspace_bytes.restype = sz
        L.moe_qmm_id_workspace_bytes_k.argtypes = [u32] * 4 + [i32]
        L.moe_qmm_id_workspace_bytes_k.restype = sz
        L.moe_qmm_test_x_copies.argtypes = [i32]
        L.moe_qmm_id_w4a4.argtypes = L.moe_qmm_id.argtypes + [i32]
        L.moe_qmm_id_w4a4.restype = i32
        L.moe_quantize_act_nvfp4.argtypes = [vp, u32, u32, i32, vp, vp, vp, vp, vp]
        L.moe_quantize_act_nvfp4.restype = i32
        L.moe_qmm_id_workspace_bytes_w4a4.argtypes = [u32] * 4
        L.moe_qmm_id_workspace_bytes_w4a4.restype = sz
        L.moe_qmm_test_x_copies.restype = i32
        L.moe_packed_row_bytes.argtypes = [i32, u32, u32]
        L.moe_packed_row_bytes.restype = sz
        L.moe_qmm_id_route.argtypes = [vp, u32, u32, u32, u32, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_qmm_id_route.restype = i32
        L.moe_qmm_id_poll_error.argtypes = [vp, vp]
        L.moe_qmm_id_poll_error.restype = i32
        L.moe_status_str.argtypes = [i32]
        L.moe_status_str.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_str(status: int) -> str:
    try:
        return lib().moe_status_str(int(status)).decode()
    except Exception:  # library not loadable
        return "?"


@functools.lru_cache(maxsize=256)
def packed_row_bytes(fmt: int, bits: int, k: int) -> int:
    return int(lib().moe_packed_row_bytes(fmt, bits, k))


def workspace_bytes(m: int, n_expert_used: int, num_experts: int, k: int | None = None,
                    x_dtype: torch.dtype | None = None) -> int:
    """moe_qmm_id_workspace_bytes; with k and x_dtype, moe_qmm_id_workspace_bytes_k
    (room for the grouped path's gathered x rows)."""
    if k is None:
        return int(lib().moe_qmm_id_workspace_bytes(m, n_expert_used, num_experts))
    return int(lib().moe_qmm_id_workspace_bytes_k(m, k, n_expert_used, num_experts,
                                                  _TORCH_DT[x_dtype or torch.bfloat16]))


def new_workspace(m: int, n_expert_used: int, num_experts: int, device="cuda", k: int | None = None,
                  x_dtype: torch.dtype | None = None) -> torch.Tensor:
    """Zero-initialised workspace (the device error word must start at zero). With k
    and x_dtype it has room for the gathered x rows of the grouped path; without, it
    is the minimum size (the grouped GEMM then gathers x rows itself)."""
    nbytes = workspace_bytes(m, n_expert_used, num_experts, k, x_dtype)
    if nbytes == 0:
        raise ValueError("sizes overflow the workspace layout")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_dev(t: torch.Tensor, name: str, device):
    if isinstance(t, torch.Tensor) and t.is_cuda and t.device == device and t.is_contiguous():
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"quantized_matmul_id: {name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"quantized_matmul_id: {name} must be on a CUDA device")
    if t.device != device:
        raise ValueError(f"quantized_matmul_id: {name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"quantized_matmul_id: {name} must be contiguous")


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _validate_only(x, ids, packed, scales, aux, *, n, group_size, bits, fmt, num_experts, out,
                   expert_bias, act, launch):
    """qmm_id's argument checks (devices, shapes, dtypes, buffer sizes) without a
    call; returns (m, k, n_expert_used, out_n). out may be None."""
    device = x.device
    for t, name in ((x, "input"), (ids, "ids"), (packed, "weight"), (scales, "scales"),
                    (aux, "aux")):
        _check_dev(t, name, device)
    if x.dim() != 2:
        raise ValueError("quantized_matmul_id: input must be [M, K]")
    if x.dtype not in _TORCH_DT:
        raise ValueError(f"quantized_matmul_id: unsupported input dtype {x.dtype}")
    if ids.dim() != 2 or ids.shape[0] != x.shape[0] or ids.element_size() != 4 or \
            ids.dtype.is_floating_point:
        raise ValueError("quantized_matmul_id: ids must be a [M, n_expert_used] 32-bit integer tensor")
    m, k = x.shape
    n_expert_used = ids.shape[1]
    if fmt not in (FMT_AFFINE, FMT_CODEBOOK, FMT_NVFP4, FMT_MXFP4):
        raise ValueError(f"quantized_matmul_id: unknown format {fmt}")
    if bits not in ({4, 6, 8} if fmt == FMT_AFFINE else {2, 3, 4} if fmt == FMT_CODEBOOK else {4}):
        raise ValueError(f"quantized_matmul_id: unsupported bits value {bits} for format {fmt}")
    if m == 0 or k == 0 or n == 0:
        raise ValueError("quantized_matmul_id: M, K, and N must all be > 0")
    if group_size <= 0:
        raise ValueError("quantized_matmul_id: group_size must be > 0")
    if n_expert_used == 0:
        raise ValueError("quantized_matmul_id: n_expert_used must be > 0")
    if num_experts <= 0:
        raise ValueError("quantized_matmul_id: num_experts must be > 0")
    rb = packed_row_bytes(fmt, bits, k)
    if rb == 0:
        raise ValueError("quantized_matmul_id: invalid format/bits/k combination")
    total_w = rb * n * num_experts
    if _nbytes(packed) < total_w:
        raise ValueError(f"quantized_matmul_id: weight buffer too small: expected at least {total_w} "
                         f"bytes for {num_experts} experts, got {_nbytes(packed)}")
    G = (k + group_size - 1) // group_size
    per_s = {FMT_AFFINE: 2, FMT_CODEBOOK: 2, FMT_NVFP4: 1, FMT_MXFP4: 1}[fmt]
    total_s = num_experts * n * G * per_s
    if _nbytes(scales) < total_s:
        raise ValueError(f"quantized_matmul_id: scales buffer too small: expected at least {total_s} "
                         f"bytes, got {_nbytes(scales)}")
    aux_need = {FMT_AFFINE: total_s, FMT_CODEBOOK: 2 * (1 << bits), FMT_NVFP4: 4 * num_experts,
                FMT_MXFP4: 0}[fmt]
    aux_name = {FMT_AFFINE: "biases", FMT_CODEBOOK: "codebook", FMT_NVFP4: "scale2", FMT_MXFP4: "aux"}[fmt]
    if _nbytes(aux) < aux_need:
        raise ValueError(f"quantized_matmul_id: {aux_name} buffer too small: expected at least "
                         f"{aux_need} bytes, got {_nbytes(aux)}")
    if launch not in _LAUNCH:
        raise ValueError(f"quantized_matmul_id: unknown launch mode {launch!r}")
    if act is not None:
        if act not in ACTS:
            raise ValueError(f"quantized_matmul_id: unknown activation {act!r} (one of {sorted(ACTS)})")
        if n % 2:
            raise ValueError("quantized_matmul_id: a gated output needs an even N (gate and up halves)")
    out_n = n // 2 if act is not None else n
    if out is not None:
        _check_dev(out, "out", device)
        if out.dtype not in _TORCH_DT or out.numel() < m * n_expert_used * out_n:
            raise ValueError("quantized_matmul_id: out must hold [M, n_expert_used, N] f32/bf16/f16 "
                             "(N/2 columns with a gated output)")
    if expert_bias is not None:
        _check_dev(expert_bias, "expert_bias", device)
        if expert_bias.dtype not in _TORCH_DT or expert_bias.numel() < num_experts * n:
            raise ValueError("quantized_matmul_id: expert_bias must hold [num_experts, N] f32/bf16/f16")
    return m, k, n_expert_used, out_n


def qmm_id(x: torch.Tensor, ids: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
           aux: torch.Tensor, *, n: int, group_size: int, bits: int, fmt: int, num_experts: int,
           out: torch.Tensor | None = None, out_dtype: torch.dtype = torch.float32,
           workspace: torch.Tensor | None = None, path: str = "auto",
           expert_bias: torch.Tensor | None = None, act: str | None = None,
           launch: str | None = None) -> torch.Tensor:
    """Expert-routed quantized matmul on the current CUDA stream.

    x [m, k] (f32 / bf16 / f16); ids [m, n_expert_used] int32/uint32; packed, scales,
    aux: raw storage tensors (any dtype, byte lengths checked); returns out
    [m, n_expert_used, n]. Buffer-size checks and their messages follow
    mlx-native quantized_matmul_id.rs (quantized_matmul_id). expert_bias, if given,
    is a [num_experts, n] f32 / bf16 / f16 tensor added to every pair's row of its
    expert (moe_qmm_id_bias). act ("silu", "gelu_tanh" or "gelu_erf") makes it the
    fused gate+up projection (moe_qmm_id_glu): rows [0, n/2) of each expert are the
    gate, rows [n/2, n) the up projection, and out [m, n_expert_used, n/2] holds
    act(gate) * up. launch ("pdl" or "early_weights") sets the C ABI's launch flags
    (MOE_LAUNCH_PDL, plus MOE_LAUNCH_EARLY_WEIGHTS): see include/moe_qmm.h for the
    promise "early_weights" makes about ids and weights.
    """
    device = x.device
    m, k, n_expert_used, out_n = _validate_only(x, ids, packed, scales, aux, n=n, group_size=group_size,
                                                bits=bits, fmt=fmt, num_experts=num_experts, out=out,
                                                expert_bias=expert_bias, act=act, launch=launch)
    path_arg = _PATHS[path] | _LAUNCH[launch]
    if out is None:
        out = torch.empty((m, n_expert_used, out_n), dtype=out_dtype, device=device)
    if workspace is None:
        workspace = new_workspace(m, n_expert_used, num_experts, device, k, x.dtype)
    else:
        _check_dev(workspace, "workspace", device)
    if act is not None:
        st = lib().moe_qmm_id_glu(
            x.data_ptr(), ids.data_ptr(), packed.data_ptr(), scales.data_ptr(), aux.data_ptr(),
            expert_bias.data_ptr() if expert_bias is not None else None, out.data_ptr(), m, k, n,
            group_size, bits, fmt, n_expert_used, num_experts, _TORCH_DT[x.dtype], _TORCH_DT[out.dtype],
            _TORCH_DT[expert_bias.dtype] if expert_bias is not None else 0, ACTS[act],
            workspace.data_ptr(), _nbytes(workspace), _stream_ptr(device), path_arg)
    elif expert_bias is None:
        st = lib().moe_qmm_id_path(
            x.data_ptr(), ids.data_ptr(), packed.data_ptr(), scales.data_ptr(), aux.data_ptr(),
            out.data_ptr(), m, k, n, group_size, bits, fmt, n_expert_used, num_experts,
            _TORCH_DT[x.dtype], _TORCH_DT[out.dtype], workspace.data_ptr(), _nbytes(workspace),
            _stream_ptr(device), path_arg)
    else:
        st = lib().moe_qmm_id_bias(
            x.data_ptr(), ids.data_ptr(), packed.data_ptr(), scales.data_ptr(), aux.data_ptr(),
            expert_bias.data_ptr(), out.data_ptr(), m, k, n, group_size, bits, fmt, n_expert_used,
            num_experts, _TORCH_DT[x.dtype], _TORCH_DT[out.dtype], _TORCH_DT[expert_bias.dtype],
            workspace.data_ptr(), _nbytes(workspace), _stream_ptr(device), path_arg)
    if st != MOE_OK:
        raise MoeError(st, "moe_qmm_id")
    return out


class Plan:
    """moe_qmm_plan: one projection with its weights, sizes, types, workspace, path,
    launch mode, optional expert bias and optional gated output bound once
    (validated like qmm_id); each call passes only x, ids and out. For decode
    loops, where the per-call argument checks of qmm_id cost more host time than
    the kernel takes on the device.

        plan = Plan(packed, scales, aux, m=1, k=..., n=..., group_size=..., bits=..., fmt=...,
                    n_expert_used=8, num_experts=128, x_dtype=torch.bfloat16)
        plan(x, ids, out)          # on the current stream, or stream=<torch.cuda.Stream>
    """

    def __init__(self, packed: torch.Tensor, scales: torch.Tensor, aux: torch.Tensor, *, m: int, k: int,
                 n: int, group_size: int, bits: int, fmt: int, n_expert_used: int, num_experts: int,
                 x_dtype: torch.dtype = torch.bfloat16, out_dtype: torch.dtype = torch.float32,
                 workspace: torch.Tensor | None = None, path: str = "auto", launch: str | None = None,
                 expert_bias: torch.Tensor | None = None, act: str | None = None):
        device = packed.device
        # the same size checks as qmm_id, on a placeholder x of the bound shape
        x0 = torch.empty((m, k), dtype=x_dtype, device=device)
        ids0 = torch.zeros((m, n_expert_used), dtype=torch.int32, device=device)
        out_n = n // 2 if act is not None else n
        out0 = torch.empty((m, n_expert_used, out_n), dtype=out_dtype, device=device)
        if workspace is None:
            workspace = new_workspace(m, n_expert_used, num_experts, device, k, x_dtype)
        _validate_only(x0, ids0, packed, scales, aux, n=n, group_size=group_size, bits=bits, fmt=fmt,
                       num_experts=num_experts, out=out0, expert_bias=expert_bias, act=act, launch=launch)
        self._keep = (packed, scales, aux, workspace, expert_bias)  # buffers the plan points into
        self._buf = ctypes.create_string_buffer(24 * 8)
        self.shape = (m, n_expert_used, out_n)
        self.device = device
        st = lib().moe_qmm_plan_init(
            self._buf, packed.data_ptr(), scales.data_ptr(), aux.data_ptr(),
            expert_bias.data_ptr() if expert_bias is not None else None, m, k, n, group_size, bits, fmt,
            n_expert_used, num_experts, _TORCH_DT[x_dtype], _TORCH_DT[out_dtype],
            _TORCH_DT[expert_bias.dtype] if expert_bias is not None else 0,
            ACTS[act] if act is not None else -1, workspace.data_ptr(), _nbytes(workspace),
            _PATHS[path] | _LAUNCH[launch])
        if st != MOE_OK:
            raise MoeError(st, "moe_qmm_plan_init")
        self._run = lib().moe_qmm_plan_run
        self._ref = ctypes.addressof(self._buf)

    def __call__(self, x: torch.Tensor, ids: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
        """x [m, k], ids [m, n_expert_used], out [m, n_expert_used, n (or n/2)]: contiguous
        tensors on the plan's device of the bound types (not re-checked here)."""
        s = (stream or torch.cuda.current_stream(self.device)).cuda_stream
        st = self._run(self._ref, x.data_ptr(), ids.data_ptr(), out.data_ptr(), s)
        if st != MOE_OK:
            raise MoeError(st, "moe_qmm_plan_run")
        return out


def qmm_id_ptrs(x: torch.Tensor, ids: torch.Tensor, packed_ptrs: torch.Tensor, scale_ptrs: torch.Tensor,
                bias_ptrs: torch.Tensor | None, aux: torch.Tensor | None, *, n: int, group_size: int,
                bits: int, fmt: int, num_experts: int, out: torch.Tensor,
                workspace: torch.Tensor | None = None, path: str = "auto") -> torch.Tensor:
    """moe_qmm_id_ptrs: weights in per-expert buffers named by device tables of
    addresses (int64 tensors of num_experts entries; a 0 packed entry skips the
    expert and leaves its pairs' rows of out untouched). aux: codebook (CODEBOOK) or
    scale2 [num_experts] (NVFP4); bias_ptrs: affine biases."""
    device = x.device
    for t, name in ((x, "input"), (ids, "ids"), (packed_ptrs, "packed_ptrs"), (scale_ptrs, "scale_ptrs"),
                    (out, "out")):
        _check_dev(t, name, device)
    for t, name in ((packed_ptrs, "packed_ptrs"), (scale_ptrs, "scale_ptrs"), (bias_ptrs, "bias_ptrs")):
        if t is not None and (t.element_size() != 8 or t.numel() < num_experts):
            raise ValueError(f"quantized_matmul_id: {name} must hold num_experts 64-bit addresses")
    m, k = x.shape
    n_expert_used = ids.shape[1]
    if workspace is None:
        workspace = new_workspace(m, n_expert_used, num_experts, device, k, x.dtype)
    st = lib().moe_qmm_id_ptrs(
        x.data_ptr(), ids.data_ptr(), packed_ptrs.data_ptr(), scale_ptrs.data_ptr(),
        bias_ptrs.data_ptr() if bias_ptrs is not None else None,
        aux.data_ptr() if aux is not None else None, out.data_ptr(), m, k, n, group_size, bits, fmt,
        n_expert_used, num_experts, _TORCH_DT[x.dtype], _TORCH_DT[out.dtype], workspace.data_ptr(),
        _nbytes(workspace), _stream_ptr(device), _PATHS[path])
    if st != MOE_OK:
        raise MoeError(st, "moe_qmm_id_ptrs")
    return out


def route(ids: torch.Tensor, num_experts: int, tile_rows: int,
          workspace: torch.Tensor | None = None):
    """Routing prologue alone. Returns (counts[E+1], offsets[E+2], sorted_pairs[R],
    tiles[tile_count, 2]) as int32 CUDA tensors (values are unsigned)."""
    if not ids.is_cuda or not ids.is_contiguous() or ids.element_size() != 4:
        raise ValueError("route: ids must be a contiguous 32-bit CUDA tensor")
    device = ids.device
    m, ne = (ids.shape[0], ids.shape[1]) if ids.dim() == 2 else (ids.numel(), 1)
    R = m * ne
    counts = torch.empty(num_experts + 1, dtype=torch.int32, device=device)
    offsets = torch.empty(num_experts + 2, dtype=torch.int32, device=device)
    sp = torch.empty(max(R, 1), dtype=torch.int32, device=device)
    max_tiles = R // tile_rows + num_experts + 1
    tiles = torch.empty((max_tiles, 2), dtype=torch.int32, device=device)
    tc = torch.empty(1, dtype=torch.int32, device=device)
    if workspace is None:
        workspace = new_workspace(m, ne, num_experts, device)
    st = lib().moe_qmm_id_route(ids.data_ptr(), m, ne, num_experts, tile_rows, counts.data_ptr(),
                                offsets.data_ptr(), sp.data_ptr(), tiles.data_ptr(), tc.data_ptr(),
                                workspace.data_ptr(), _nbytes(workspace), _stream_ptr(device))
    if st != MOE_OK:
        raise MoeError(st, "moe_qmm_id_route")
    ntiles = int(tc.item())
    return counts, offsets, sp[:R], tiles[:ntiles]


def poll_error(workspace: torch.Tensor) -> int:
    """Synchronise the current stream, read and clear the device error word."""
    return int(lib().moe_qmm_id_poll_error(workspace.data_ptr(), _stream_ptr(workspace.device)))


def quantize_act_nvfp4(x: torch.Tensor):
    """moe_quantize_act_nvfp4: per-token NVFP4 quantisation of x [m, k] (f32 / bf16 /
    f16, k a multiple of 16) on the current stream. Returns (codes [m, k/2] uint8,
    element 2i in the low nibble; E4M3 scales [m, k/16] uint8; per-token scales [m]
    f32; x^ [m, k] f32)."""
    if x.dim() != 2 or not x.is_cuda or not x.is_contiguous() or x.dtype not in _TORCH_DT:
        raise ValueError("quantize_act_nvfp4: x must be a contiguous 2-D f32/bf16/f16 CUDA tensor")
    m, k = x.shape
    dev = x.device
    codes = torch.empty((m, k // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((m, k // 16), dtype=torch.uint8, device=dev)
    g = torch.empty(m, dtype=torch.float32, device=dev)
    xhat = torch.empty((m, k), dtype=torch.float32, device=dev)
    st = lib().moe_quantize_act_nvfp4(x.data_ptr(), m, k, _TORCH_DT[x.dtype], codes.data_ptr(),
                                      scales.data_ptr(), g.data_ptr(), xhat.data_ptr(), _stream_ptr(dev))
    if st != MOE_OK:
        raise MoeError(st, "moe_quantize_act_nvfp4")
    return codes, scales, g, xhat


def workspace_bytes_w4a4(m: int, k: int, n_expert_used: int, num_experts: int) -> int:
    return int(lib().moe_qmm_id_workspace_bytes_w4a4(m, k, n_expert_used, num_experts))


def qmm_id_w4a4(x: torch.Tensor, ids: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                aux: torch.Tensor, *, n: int, group_size: int, bits: int, fmt: int, num_experts: int,
                out: torch.Tensor | None = None, out_dtype: torch.dtype = torch.float32,
                workspace: torch.Tensor | None = None, path: str = "auto", launch: str | None = None) -> torch.Tensor:
    """moe_qmm_id_w4a4: the operation with x quantised per token to NVFP4 first
    (see moe_quantize_act_nvfp4 in include/moe_qmm.h for the quantisation); the
    other arguments and checks as qmm_id."""
    device = x.device
    m, k, n_expert_used, out_n = _validate_only(x, ids, packed, scales, aux, n=n, group_size=group_size,
                                                bits=bits, fmt=fmt, num_experts=num_experts, out=out,
                                                expert_bias=None, act=None, launch=launch)
    if out is None:
        out = torch.empty((m, n_expert_used, out_n), dtype=out_dtype, device=device)
    if workspace is None:
        nbytes = workspace_bytes_w4a4(m, k, n_expert_used, num_experts)
        if nbytes == 0:
            raise ValueError("sizes overflow the workspace layout")
        workspace = torch.zeros(nbytes, dtype=torch.uint8, device=device)
    else:
        _check_dev(workspace, "workspace", device)
    st = lib().moe_qmm_id_w4a4(
        x.data_ptr(), ids.data_ptr(), packed.data_ptr(), scales.data_ptr(), aux.data_ptr(), out.data_ptr(),
        m, k, n, group_size, bits, fmt, n_expert_used, num_experts, _TORCH_DT[x.dtype], _TORCH_DT[out.dtype],
        workspace.data_ptr(), _nbytes(workspace), _stream_ptr(device), _PATHS[path] | _LAUNCH[launch])
    if st != MOE_OK:
        raise MoeError(st, "moe_qmm_id_w4a4")
    return out
