"""Thin Python binding of the C ABI in ``include/mla.h`` (ctypes).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of ``libmla_b200.so``.  Tensors are torch CUDA tensors (device memory
and streams only); each call enqueues on the current torch stream.  A missing
library raises immediately -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

MLA_BF16, MLA_F32 = 0, 1
STATUS = {
    0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED",
    3: "MLA_ERR_ALIGNMENT", 4: "MLA_ERR_WORKSPACE", 5: "MLA_ERR_CUDA",
    6: "MLA_ERR_DEVICE_TIMEOUT", 7: "MLA_ERR_BOUNDS",
}
EXPORTED = (
    "mla_cache_row_elems", "mla_cache_append_workspace_bytes", "mla_cache_append",
    "mla_absorb_q", "mla_decode_default_splits", "mla_decode_workspace_bytes",
    "mla_decode", "mla_combine", "mla_out_proj", "mla_get_device_status",
    "mla_status_string", "mla_decode_noalloc", "mla_decode_paged", "mla_cache_append_paged",
    "mla_merge_partials", "mla_debug_inject_wait", "mla_cache_fp8_row_bytes",
    "mla_cache_append_fp8", "mla_decode_fp8", "mla_fold_output_weights",
    "mla_out_proj_folded_workspace_bytes", "mla_out_proj_folded", "mla_prefill_workspace_bytes",
    "mla_prefill",
)

PAGE_ROWS = 64   # rows per page of a paged latent cache (one decode work tile)


class MLAError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({msg})")
        self.status = status


class CDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d_c", ctypes.c_int32),
                ("d_r", ctypes.c_int32), ("d_nope", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("cache_capacity", ctypes.c_int64), ("dtype", ctypes.c_int32)]


@dataclass(frozen=True)
class Dims:
    """Problem shape (names as in the header: H heads, d_c latent width,
    d_r decoupled-RoPE width, d_nope / d_v per-head content / value widths)."""
    B: int
    H: int
    d_c: int
    d_r: int
    d_nope: int
    d_v: int
    cache_capacity: int
    dtype: str = "bf16"  # "bf16" | "f32"

    def c(self) -> CDims:
        return CDims(self.B, self.H, self.d_c, self.d_r, self.d_nope, self.d_v,
                     self.cache_capacity, MLA_BF16 if self.dtype == "bf16" else MLA_F32)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def R(self) -> int:
        return self.d_c + self.d_r


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the sm_100a library.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with mla_latent_kv_nope_b200.build.build(); "
            "there is no non-CUDA implementation")
    lib = ctypes.CDLL(path)
    P, I32, I64, SZ, F = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                          ctypes.c_float)
    D = ctypes.POINTER(CDims)
    sig = {
        "mla_cache_row_elems": (I64, [I32, I32]),
        "mla_cache_append_workspace_bytes": (SZ, [D, I32]),
        "mla_cache_append": (ctypes.c_int, [D, I32, P, P, P, F, F, P, P, P, SZ, P]),
        "mla_absorb_q": (ctypes.c_int, [D, P, P, P, P, F, P, P]),
        "mla_decode_default_splits": (ctypes.c_int, [D]),
        "mla_decode_workspace_bytes": (SZ, [D, ctypes.c_int]),
        "mla_decode": (ctypes.c_int, [D, P, P, P, F, ctypes.c_int, P, SZ,
                                      ctypes.POINTER(ctypes.c_int), P]),
        "mla_combine": (ctypes.c_int, [D, P, P, SZ, ctypes.c_int, P, P, P]),
        "mla_out_proj": (ctypes.c_int, [D, P, P, P, P]),
        "mla_get_device_status": (ctypes.c_int, [P]),
        "mla_decode_noalloc": (ctypes.c_int, [D, P, P, P, F, P, P, P]),
        "mla_decode_paged": (ctypes.c_int, [D, P, P, I64, P, I32, P, F, ctypes.c_int, P, SZ,
                                            ctypes.POINTER(ctypes.c_int), P]),
        "mla_cache_append_paged": (ctypes.c_int, [D, I32, P, P, P, F, F, P, I64, P, I32, P, P,
                                                  SZ, P]),
        "mla_merge_partials": (ctypes.c_int, [D, ctypes.c_int, P, P, P, P, P]),
        "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "mla_debug_inject_wait": (ctypes.c_int, [ctypes.c_uint64]),
        "mla_cache_fp8_row_bytes": (I64, [I32, I32]),
        "mla_fold_output_weights": (ctypes.c_int, [D, I32, P, P, P, P]),
        "mla_prefill_workspace_bytes": (SZ, [D, I32, I64]),
        "mla_prefill": (ctypes.c_int, [D, I32, I64, P, P, P, P, P, P, F, F, P, P, P, SZ, P]),
        "mla_out_proj_folded_workspace_bytes": (SZ, [D, I32]),
        "mla_out_proj_folded": (ctypes.c_int, [D, I32, P, P, P, P, SZ, P]),
        "mla_cache_append_fp8": (ctypes.c_int, [D, I32, P, P, P, F, F, P, P, P, P, SZ, P]),
        "mla_decode_fp8": (ctypes.c_int, [D, P, P, P, P, F, ctypes.c_int, P, SZ,
                                          ctypes.POINTER(ctypes.c_int), P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != 0:
        msg = load_library().mla_status_string(status).decode()
        raise MLAError(fn, status, msg)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_cuda:
        raise ValueError(f"{name}: expected CUDA {dtype} {tuple(shape)}, got "
                         f"{t.device} {t.dtype} {tuple(t.shape)}")


def _need_ws(t, name="workspace"):
    """A scratch buffer: any dtype, but device memory and contiguous (the
    library writes it from kernels, so a host tensor must never reach it)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        got = t.device if isinstance(t, torch.Tensor) else type(t).__name__
        raise ValueError(f"{name}: expected a contiguous CUDA tensor, got {got}")


# ---------------------------------------------------------------------------
def cache_row_elems(d_c: int, d_r: int) -> int:
    """Elements of one latent cache row, d_c + d_r (mla_cache_row_elems)."""
    return int(load_library().mla_cache_row_elems(d_c, d_r))


def cache_append_workspace_bytes(dims: Dims, hidden: int) -> int:
    """Bytes of fp32 workspace mla_cache_append needs for this hidden size."""
    return int(load_library().mla_cache_append_workspace_bytes(ctypes.byref(dims.c()), hidden))


def cache_append(dims: Dims, h, W_DKV, gamma, cache, seqlens, workspace, eps=1e-6,
                 rope_base=10000.0, stream=None):
    """mla_cache_append: write row L_b = [RMSNorm(W^DKV h) * gamma || RoPE(W^KR h, L_b)]
    of every sequence and increment L_b (cache [B, capacity, R])."""
    dt = dims.torch_dtype
    hidden = h.shape[-1]
    _need(h, dt, (dims.B, hidden), "h")
    _need(W_DKV, dt, (dims.R, hidden), "W_DKV")
    _need(cache, dt, (dims.B, dims.cache_capacity, dims.R), "cache")
    _need(seqlens, torch.int32, (dims.B,), "seqlens")
    if gamma is not None:
        _need(gamma, torch.float32, (dims.d_c,), "gamma")
    _need_ws(workspace)
    st = load_library().mla_cache_append(
        ctypes.byref(dims.c()), hidden, _ptr(h), _ptr(W_DKV), _ptr(gamma), eps, rope_base,
        _ptr(cache), _ptr(seqlens), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("mla_cache_append", st)


def _need_pages(dims: Dims, pool, block_table):
    if pool.dim() != 3 or pool.shape[1:] != (PAGE_ROWS, dims.R):
        raise ValueError(f"cache_pool must be [num_pages, {PAGE_ROWS}, {dims.R}]")
    _need(pool, dims.torch_dtype, tuple(pool.shape), "cache_pool")
    if block_table.dim() != 2 or block_table.shape[0] != dims.B:
        raise ValueError("block_table must be [B, max_blocks]")
    _need(block_table, torch.int32, tuple(block_table.shape), "block_table")


def cache_append_paged(dims: Dims, h, W_DKV, gamma, cache_pool, block_table, seqlens,
                       workspace, eps=1e-6, rope_base=10000.0, stream=None):
    """mla_cache_append on a paged cache: cache_pool [num_pages, 64, R], block_table
    [B, max_blocks] int32 page ids."""
    dt = dims.torch_dtype
    hidden = h.shape[-1]
    _need(h, dt, (dims.B, hidden), "h")
    _need(W_DKV, dt, (dims.R, hidden), "W_DKV")
    _need_pages(dims, cache_pool, block_table)
    _need(seqlens, torch.int32, (dims.B,), "seqlens")
    if gamma is not None:
        _need(gamma, torch.float32, (dims.d_c,), "gamma")
    _need_ws(workspace)
    st = load_library().mla_cache_append_paged(
        ctypes.byref(dims.c()), hidden, _ptr(h), _ptr(W_DKV), _ptr(gamma), eps, rope_base,
        _ptr(cache_pool), cache_pool.shape[0], _ptr(block_table), block_table.shape[1],
        _ptr(seqlens), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check("mla_cache_append_paged", st)


def decode_paged(dims: Dims, q_cat, cache_pool, block_table, seqlens, softmax_scale, workspace,
                 num_splits=0, stream=None) -> int:
    """mla_decode on a paged cache (see cache_append_paged)."""
    _need(q_cat, dims.torch_dtype, (dims.B, dims.H, dims.R), "q_cat")
    _need_pages(dims, cache_pool, block_table)
    _need(seqlens, torch.int32, (dims.B,), "seqlens")
    _need_ws(workspace)
    used = ctypes.c_int(0)
    st = load_library().mla_decode_paged(
        ctypes.byref(dims.c()), _ptr(q_cat), _ptr(cache_pool), cache_pool.shape[0],
        _ptr(block_table), block_table.shape[1], _ptr(seqlens), float(softmax_scale), num_splits,
        _ptr(workspace), workspace.numel() * workspace.element_size(), ctypes.byref(used),
        _stream(stream))
    _check("mla_decode_paged", st)
    return used.value


def cache_fp8_row_bytes(d_c: int, d_r: int) -> int:
    """Bytes of one FP8 latent cache row: d_c E4M3 codes + d_r bf16 RoPE keys."""
    return int(load_library().mla_cache_fp8_row_bytes(d_c, d_r))


def _need_fp8_cache(dims: Dims, cache, scales):
    rb = dims.d_c + 2 * dims.d_r
    _need(cache, torch.uint8, (dims.B, dims.cache_capacity, rb), "cache_fp8")
    _need(scales, torch.float32, (dims.B, dims.cache_capacity), "scales")


def cache_append_fp8(dims: Dims, h, W_DKV, gamma, cache, scales, seqlens, workspace, eps=1e-6,
                     rope_base=10000.0, stream=None):
    """mla_cache_append_fp8: as cache_append, into an FP8 latent cache
    (cache [B, capacity, d_c + 2 d_r] uint8, scales [B, capacity] fp32)."""
    dt = dims.torch_dtype
    hidden = h.shape[-1]
    _need(h, dt, (dims.B, hidden), "h")
    _need(W_DKV, dt, (dims.R, hidden), "W_DKV")
    _need_fp8_cache(dims, cache, scales)
    _need(seqlens, torch.int32, (dims.B,), "seqlens")
    if gamma is not None:
        _need(gamma, torch.float32, (dims.d_c,), "gamma")
    _need_ws(workspace)
    st = load_library().mla_cache_append_fp8(
        ctypes.byref(dims.c()), hidden, _ptr(h), _ptr(W_DKV), _ptr(gamma), eps, rope_base,
        _ptr(cache), _ptr(scales), _ptr(seqlens), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("mla_cache_append_fp8", st)


def decode_fp8(dims: Dims, q_cat, cache, scales, seqlens, softmax_scale, workspace,
               num_splits=0, stream=None) -> int:
    """mla_decode_fp8: mla_decode over an FP8 latent cache; returns the splits used."""
    _need(q_cat, dims.torch_dtype, (dims.B, dims.H, dims.R), "q_cat")
    _need_fp8_cache(dims, cache, scales)
    _need(seqlens, torch.int32, (dims.B,), "seqlens")
    _need_ws(workspace)
    used = ctypes.c_int(0)
    st = load_library().mla_decode_fp8(ctypes.byref(dims.c()), _ptr(q_cat), _ptr(cache),
                                       _ptr(scales), _ptr(seqlens), float(softmax_scale),
                                       num_splits, _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       ctypes.byref(used), _stream(stream))
    _check("mla_decode_fp8", st)
    return used.value


def absorb_q(dims: Dims, q_nope, q_pe, W_UK, q_pos, q_cat, rope_base=10000.0, stream=None):
    """mla_absorb_q: q_cat[b,i] = [W^UK_i^T q_nope[b,i] ; RoPE(q_pe[b,i], q_pos[b])]
    (no rotation when q_pos is None)."""
    dt = dims.torch_dtype
    _need(q_nope, dt, (dims.B, dims.H, dims.d_nope), "q_nope")
    _need(q_pe, dt, (dims.B, dims.H, dims.d_r), "q_pe")
    _need(W_UK, dt, (dims.H, dims.d_nope, dims.d_c), "W_UK")
    _need(q_cat, dt, (dims.B, dims.H, dims.R), "q_cat")
    if q_pos is not None:
        _need(q_pos, torch.int32, (dims.B,), "q_pos")
    st = load_library().mla_absorb_q(ctypes.byref(dims.c()), _ptr(q_nope), _ptr(q_pe),
                                     _ptr(W_UK), _ptr(q_pos), rope_base, _ptr(q_cat),
                                     _stream(stream))
    _check("mla_absorb_q", st)


def decode_default_splits(dims: Dims) -> int:
    """The split count mla_decode uses on the current device when asked for 0."""
    return int(load_library().mla_decode_default_splits(ctypes.byref(dims.c())))


def decode_workspace_bytes(dims: Dims, num_splits: int = 0) -> int:
    """Bytes of workspace mla_decode needs for this many splits (0 = default)."""
    return int(load_library().mla_decode_workspace_bytes(ctypes.byref(dims.c()), num_splits))


def decode(dims: Dims, q_cat, cache, seqlens, softmax_scale, workspace, num_splits=0,
           stream=None) -> int:
    """mla_decode: split-KV latent attention of q_cat over the cache; writes the
    partials into ``workspace`` and returns the number of splits used."""
    dt = dims.torch_dtype
    _need(q_cat, dt, (dims.B, dims.H, dims.R), "q_cat")
    _need(cache, dt, (dims.B, dims.cache_capacity, dims.R), "cache")
    _need(seqlens, torch.int32, (dims.B,), "seqlens")
    _need_ws(workspace)
    used = ctypes.c_int(0)
    st = load_library().mla_decode(ctypes.byref(dims.c()), _ptr(q_cat), _ptr(cache),
                                   _ptr(seqlens), float(softmax_scale), num_splits,
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   ctypes.byref(used), _stream(stream))
    _check("mla_decode", st)
    return used.value


def combine(dims: Dims, seqlens, workspace, splits_used, o_lat, lse=None, stream=None):
    """mla_combine: log-sum-exp merge of the partials into o_lat [B,H,d_c] fp32 (and
    lse [B,H] fp32 when given)."""
    _need(seqlens, torch.int32, (dims.B,), "seqlens")
    _need_ws(workspace)
    _need(o_lat, torch.float32, (dims.B, dims.H, dims.d_c), "o_lat")
    if lse is not None:
        _need(lse, torch.float32, (dims.B, dims.H), "lse")
    st = load_library().mla_combine(ctypes.byref(dims.c()), _ptr(seqlens), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), splits_used,
                                    _ptr(o_lat), _ptr(lse), _stream(stream))
    _check("mla_combine", st)


def merge_partials(dims: Dims, o_parts, lse_parts, o_lat, lse=None, stream=None):
    """mla_merge_partials: log-sum-exp merge of n per-token-range results,
    o_parts [n,B,H,d_c] fp32 and lse_parts [n,B,H] fp32 (stacked combine
    outputs), into o_lat [B,H,d_c] (and lse [B,H] when given)."""
    n = o_parts.shape[0]
    _need(o_parts, torch.float32, (n, dims.B, dims.H, dims.d_c), "o_parts")
    _need(lse_parts, torch.float32, (n, dims.B, dims.H), "lse_parts")
    _need(o_lat, torch.float32, (dims.B, dims.H, dims.d_c), "o_lat")
    if lse is not None:
        _need(lse, torch.float32, (dims.B, dims.H), "lse")
    st = load_library().mla_merge_partials(ctypes.byref(dims.c()), n, _ptr(o_parts),
                                           _ptr(lse_parts), _ptr(o_lat), _ptr(lse),
                                           _stream(stream))
    _check("mla_merge_partials", st)


def out_proj(dims: Dims, o_lat, W_UV, out, stream=None):
    """mla_out_proj: out[b,i] = W^UV_i o_lat[b,i]."""
    dt = dims.torch_dtype
    _need(o_lat, torch.float32, (dims.B, dims.H, dims.d_c), "o_lat")
    _need(W_UV, dt, (dims.H, dims.d_v, dims.d_c), "W_UV")
    _need(out, dt, (dims.B, dims.H, dims.d_v), "out")
    st = load_library().mla_out_proj(ctypes.byref(dims.c()), _ptr(o_lat), _ptr(W_UV), _ptr(out),
                                     _stream(stream))
    _check("mla_out_proj", st)


def debug_inject_wait(cycles: int) -> None:
    """mla_debug_inject_wait: test hook that makes later bf16 decode launches
    wait ``cycles`` SM cycles on a barrier nothing arrives on and give up
    (MLA_ERR_DEVICE_TIMEOUT in the status word); 0 turns it off."""
    _check("mla_debug_inject_wait", load_library().mla_debug_inject_wait(int(cycles)))


def prefill_workspace_bytes(dims: Dims, T: int, L: int) -> int:
    return int(load_library().mla_prefill_workspace_bytes(ctypes.byref(dims.c()), T, L))


def prefill(dims: Dims, q_nope, q_pe, q_pos, W_UK, W_UV, rows, out, workspace, lse=None,
            softmax_scale: float = 0.0, rope_base: float = 10000.0, stream=None):
    """mla_prefill: materialised causal attention of one sequence's T query
    tokens over its L latent rows [L, d_c + d_r]; out [T, H, d_v] (+ lse [T, H])."""
    T, L = q_nope.shape[0], rows.shape[0]
    dt = dims.torch_dtype
    _need(q_nope, dt, (T, dims.H, dims.d_nope), "q_nope")
    if dims.d_r:
        _need(q_pe, dt, (T, dims.H, dims.d_r), "q_pe")
    _need(q_pos, torch.int32, (T,), "q_pos")
    _need(W_UK, dt, (dims.H, dims.d_nope, dims.d_c), "W_UK")
    _need(W_UV, dt, (dims.H, dims.d_v, dims.d_c), "W_UV")
    _need(rows, dt, (L, dims.R), "rows")
    _need(out, dt, (T, dims.H, dims.d_v), "out")
    if lse is not None:
        _need(lse, torch.float32, (T, dims.H), "lse")
    _need_ws(workspace)
    st = load_library().mla_prefill(
        ctypes.byref(dims.c()), T, L, _ptr(q_nope), _ptr(q_pe) if dims.d_r else None,
        _ptr(q_pos), _ptr(W_UK), _ptr(W_UV), _ptr(rows), softmax_scale, rope_base, _ptr(out),
        _ptr(lse) if lse is not None else None, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("mla_prefill", st)


def fold_output_weights(dims: Dims, W_O, W_UV, W_fold, stream=None):
    """mla_fold_output_weights: W_fold [d_model, H*d_c] with
    W_fold[m, i*d_c + c] = (W^O_i W^UV_i)[m, c]; W_O [d_model, H*d_v]."""
    d_model = W_O.shape[0]
    _need(W_O, dims.torch_dtype, (d_model, dims.H * dims.d_v), "W_O")
    _need(W_UV, dims.torch_dtype, (dims.H, dims.d_v, dims.d_c), "W_UV")
    _need(W_fold, dims.torch_dtype, (d_model, dims.H * dims.d_c), "W_fold")
    st = load_library().mla_fold_output_weights(ctypes.byref(dims.c()), d_model, _ptr(W_O),
                                                _ptr(W_UV), _ptr(W_fold), _stream(stream))
    _check("mla_fold_output_weights", st)


def out_proj_folded_workspace_bytes(dims: Dims, d_model: int) -> int:
    return int(load_library().mla_out_proj_folded_workspace_bytes(ctypes.byref(dims.c()),
                                                                  d_model))


def out_proj_folded(dims: Dims, o_lat, W_fold, u, workspace, stream=None):
    """mla_out_proj_folded: u [B, d_model] = sum_i B_i o_lat[:, i] (bf16)."""
    d_model = W_fold.shape[0]
    _need(o_lat, torch.float32, (dims.B, dims.H, dims.d_c), "o_lat")
    _need(W_fold, dims.torch_dtype, (d_model, dims.H * dims.d_c), "W_fold")
    _need(u, dims.torch_dtype, (dims.B, d_model), "u")
    _need_ws(workspace)
    st = load_library().mla_out_proj_folded(
        ctypes.byref(dims.c()), d_model, _ptr(o_lat), _ptr(W_fold), _ptr(u), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("mla_out_proj_folded", st)


def get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(load_library().mla_get_device_status(_stream(stream)))


# ---------------------------------------------------------------------------
class DecodeStep:
    """One MLA decode layer on the device: owns its workspaces (allocated once
    by the caller side through torch) and runs append -> absorb_q -> decode ->
    combine -> out_proj.  All arithmetic is in the CUDA kernels; this class
    only keeps buffers, pointers and the stream order.

    absorb_q does not depend on the cache append, so with ``overlap`` it runs
    on a second stream forked from the current one and joined before decode.
    ``capture`` records one step (plus any caller work) into a CUDA graph so a
    step is replayed with one launch from the host."""

    def __init__(self, dims: Dims, W_UK, W_UV, W_DKV=None, gamma=None, softmax_scale=None,
                 rope_base=10000.0, eps=1e-6, num_splits=0, device="cuda", overlap=True):
        self.dims = dims
        self.W_UK, self.W_UV, self.W_DKV, self.gamma = W_UK, W_UV, W_DKV, gamma
        # 0 asks the library for the pages' scale 1/sqrt(d_nope + d_r).
        self.scale = 0.0 if softmax_scale is None else float(softmax_scale)
        self.rope_base, self.eps = rope_base, eps
        self.num_splits = num_splits or decode_default_splits(dims)
        ws = decode_workspace_bytes(dims, self.num_splits)
        self.ws = torch.empty(ws // 4, dtype=torch.float32, device=device)
        hidden = W_DKV.shape[1] if W_DKV is not None else 1
        self.ws_append = torch.empty(max(cache_append_workspace_bytes(dims, hidden) // 4, 1),
                                     dtype=torch.float32, device=device)
        dt = dims.torch_dtype
        self.q_cat = torch.empty(dims.B, dims.H, dims.R, dtype=dt, device=device)
        self.o_lat = torch.empty(dims.B, dims.H, dims.d_c, dtype=torch.float32, device=device)
        self.lse = torch.empty(dims.B, dims.H, dtype=torch.float32, device=device)
        self.out = torch.empty(dims.B, dims.H, dims.d_v, dtype=dt, device=device)
        self.splits_used = self.num_splits
        self._side = torch.cuda.Stream(device=device) if overlap else None

    def append(self, h, cache, seqlens, block_table=None, scales=None):
        if scales is not None:
            cache_append_fp8(self.dims, h, self.W_DKV, self.gamma, cache, scales, seqlens,
                             self.ws_append, self.eps, self.rope_base)
        elif block_table is None:
            cache_append(self.dims, h, self.W_DKV, self.gamma, cache, seqlens, self.ws_append,
                         self.eps, self.rope_base)
        else:
            cache_append_paged(self.dims, h, self.W_DKV, self.gamma, cache, block_table,
                               seqlens, self.ws_append, self.eps, self.rope_base)

    def absorb(self, q_nope, q_pe, q_pos):
        """absorb_q into the step's q_cat buffer."""
        absorb_q(self.dims, q_nope, q_pe, self.W_UK, q_pos, self.q_cat, self.rope_base)

    def _attend_latent(self, cache, seqlens, block_table=None, scales=None):
        if scales is not None:
            self.splits_used = decode_fp8(self.dims, self.q_cat, cache, scales, seqlens,
                                          self.scale, self.ws, self.num_splits)
        elif block_table is None:
            self.splits_used = decode(self.dims, self.q_cat, cache, seqlens, self.scale, self.ws,
                                      self.num_splits)
        else:
            self.splits_used = decode_paged(self.dims, self.q_cat, cache, block_table, seqlens,
                                            self.scale, self.ws, self.num_splits)
        combine(self.dims, seqlens, self.ws, self.splits_used, self.o_lat, self.lse)
        out_proj(self.dims, self.o_lat, self.W_UV, self.out)
        return self.out

    def attend(self, q_nope, q_pe, q_pos, cache, seqlens, block_table=None, scales=None):
        self.absorb(q_nope, q_pe, q_pos)
        return self._attend_latent(cache, seqlens, block_table, scales)

    def __call__(self, q_nope, q_pe, q_pos, cache, seqlens, h=None, block_table=None,
                 scales=None):
        """One step.  With ``block_table`` the cache is a paged pool
        [num_pages, 64, R] (see decode_paged); with ``scales`` it is an FP8
        latent cache [B, capacity, d_c + 2 d_r] uint8 with its scale plane
        [B, capacity] (see decode_fp8)."""
        if self._side is None:
            if h is not None:
                self.append(h, cache, seqlens, block_table, scales)
            return self.attend(q_nope, q_pe, q_pos, cache, seqlens, block_table, scales)
        main = torch.cuda.current_stream()
        # Fork: the side stream starts after everything issued so far (the
        # previous step's decode has finished reading q_cat).  absorb_q is
        # launched first: measured in a graph on B200 the pair takes 14.9 us
        # this way and 20.6 us with the append launched first (each alone
        # about 12.3 us).
        self._side.wait_stream(main)
        with torch.cuda.stream(self._side):
            self.absorb(q_nope, q_pe, q_pos)
        if h is not None:
            self.append(h, cache, seqlens, block_table, scales)
        main.wait_stream(self._side)
        return self._attend_latent(cache, seqlens, block_table, scales)

    def host_pipeline(self, host_inputs, host_out, cache, seqlens, after=None,
                      block_table=None, scales=None):
        """Steps fed from pinned host memory with the copies overlapped.

        ``host_inputs`` = (q_nope, q_pe, q_pos[, h]) pinned host tensors,
        ``host_out`` a pinned host tensor shaped like ``self.out``.  Two device
        input sets and two output stages alternate; each is served by one CUDA
        graph that runs a step on set c while a forked copy stream brings the
        next step's inputs into set 1 - c and takes the previous step's
        output from stage 1 - c to ``host_out``.  So every step still copies
        its own inputs in and its result out, but one graph launch per step
        does it.  ``run(n)`` performs n steps, with the first step's inputs
        copied in before and the last result copied out after; ``host_out``
        holds the last step's result once the stream has finished."""
        return _HostPipeline(self, host_inputs, host_out, cache, seqlens, after, block_table,
                             scales)

    def capture(self, q_nope, q_pe, q_pos, cache, seqlens, h=None, before=None, after=None,
                block_table=None, scales=None):
        """Record one step into a CUDA graph; ``before``/``after`` are optional
        callables whose device work is recorded around it.  Replay with
        ``graph.replay()``; inputs are read from the same tensors each time."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            if before is not None:
                before()
            self(q_nope, q_pe, q_pos, cache, seqlens, h=h, block_table=block_table,
                 scales=scales)
            if after is not None:
                after()
        return g


class _HostPipeline:
    """See DecodeStep.host_pipeline."""

    def __init__(self, step, host_inputs, host_out, cache, seqlens, after, block_table, scales):
        for t in (*host_inputs, host_out):
            if t.is_cuda or not t.is_pinned():
                raise ValueError("host_pipeline needs pinned host tensors")
        self.step, self.host_in, self.host_out = step, tuple(host_inputs), host_out
        dev = step.out.device
        self.sets = [[torch.empty_like(t, device=dev) for t in self.host_in] for _ in range(2)]
        self.stages = [torch.empty_like(step.out) for _ in range(2)]
        # Host->device and device->host copies on separate streams, so the two
        # directions overlap each other as well as the step.
        self.in_stream = torch.cuda.Stream(device=dev)
        self.out_stream = torch.cuda.Stream(device=dev)
        self.graphs = []
        # Each graph's step writes its output straight into its own stage (the
        # step's output buffer is pointed at the stage while the graph is
        # recorded), so no device copy sits between the step and the next
        # device->host copy.
        out = step.out
        try:
            for c in range(2):
                step.out = self.stages[c]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    main = torch.cuda.current_stream()
                    self.in_stream.wait_stream(main)
                    self.out_stream.wait_stream(main)
                    with torch.cuda.stream(self.in_stream):
                        for d_t, h_t in zip(self.sets[1 - c], self.host_in):
                            d_t.copy_(h_t, non_blocking=True)
                    with torch.cuda.stream(self.out_stream):
                        self.host_out.copy_(self.stages[1 - c], non_blocking=True)
                    x = self.sets[c]
                    step(x[0], x[1], x[2], cache, seqlens, h=x[3] if len(x) > 3 else None,
                         block_table=block_table, scales=scales)
                    if after is not None:
                        after()
                    main.wait_stream(self.in_stream)
                    main.wait_stream(self.out_stream)
                self.graphs.append(g)
        finally:
            step.out = out

    def run(self, n: int):
        for d_t, h_t in zip(self.sets[0], self.host_in):
            d_t.copy_(h_t, non_blocking=True)
        for k in range(n):
            self.graphs[k % 2].replay()
        if n:
            self.host_out.copy_(self.stages[(n - 1) % 2], non_blocking=True)

    def bytes_per_step(self):
        """(host->device, device->host) bytes each step copies."""
        return (sum(t.numel() * t.element_size() for t in self.host_in),
                self.host_out.numel() * self.host_out.element_size())
