"""ctypes binding of libhga.so: argument marshalling only.

Every function has the name of the C entry point it wraps (include/hga.h) and
takes torch tensors where the C call takes device (or pinned host) pointers.
Each step of the HGA attention computation runs in the library's CUDA
kernels; nothing here computes.  A missing library is an ImportError, a
failing call an HgaError: there is no fallback path.
"""
from __future__ import annotations

import ctypes

import numpy as np
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhga.so")

HGA_OK = 0
STATUS_NAMES = {0: "HGA_OK", 1: "HGA_ERR_INVALID_ARG", 2: "HGA_ERR_SHAPE", 3: "HGA_ERR_UNSUPPORTED",
                4: "HGA_ERR_INDEX", 5: "HGA_ERR_TIMEOUT", 6: "HGA_ERR_CUDA"}
HGA_F32, HGA_BF16 = 0, 1


class HgaError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {detail}")


class hga_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("block", ctypes.c_int), ("S", ctypes.c_int), ("n_hist_blocks", ctypes.c_int),
                ("topk", ctypes.c_int), ("dtype", ctypes.c_int), ("q_block", ctypes.c_int)]


@dataclass(frozen=True)
class Dims:
    B: int
    Hq: int
    Hkv: int
    d: int
    block: int
    S: int
    n_hist_blocks: int
    topk: int
    dtype: str = "bf16"  # "bf16" or "f32"
    q_block: int = 0     # query-block size; 0 = block (one size for history and query blocks)

    @property
    def qb(self) -> int:
        return self.q_block or self.block

    @property
    def nqb(self) -> int:
        return self.S // self.qb

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def c(self) -> hga_dims:
        return hga_dims(self.B, self.Hq, self.Hkv, self.d, self.block, self.S, self.n_hist_blocks, self.topk,
                        HGA_BF16 if self.dtype == "bf16" else HGA_F32, self.q_block)

    def with_history(self, n_hist_blocks: int) -> "Dims":
        return Dims(self.B, self.Hq, self.Hkv, self.d, self.block, self.S, n_hist_blocks, self.topk, self.dtype,
                    self.q_block)


class hga_block_cache(ctypes.Structure):
    _fields_ = [("slot_of_block", ctypes.POINTER(ctypes.c_int32)), ("block_of_slot", ctypes.POINTER(ctypes.c_int32)),
                ("last_use", ctypes.POINTER(ctypes.c_int64)), ("host_capacity_blocks", ctypes.c_int),
                ("pool_slots", ctypes.c_int), ("tick", ctypes.c_int64)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.POINTER(hga_dims)
_C = ctypes.POINTER(hga_block_cache)

# (name, restype, argtypes) for every entry point of include/hga.h and
# include/hga_selftest.h.
_SIGNATURES = [
    ("hga_status_string", ctypes.c_char_p, [_I]),
    ("hga_last_error", ctypes.c_char_p, []),
    ("hga_device_status", _I, [_P]),
    ("hga_block_summaries", _I, [_D, _P, _I, _I, _P, _P]),
    ("hga_segment_summaries", _I, [_D, _P, _I, _P, _P]),
    ("hga_select_topk", _I, [_D, _P, _P, _P, _P, _P]),
    ("hga_attn_fwd", _I, [_D, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P]),
    ("hga_attn_bwd_workspace_size", ctypes.c_size_t, [_D]),
    ("hga_attn_bwd", _I, [_D, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    ("hga_attn_bwd_noalloc", _I, [_D, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    ("hga_attn_bwd_sparse", _I, [_D, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P, _P,
                                 ctypes.c_size_t, _P]),
    ("hga_attn_bwd_preprocess", _I, [_D, _P, _P, _P, ctypes.c_size_t, _P]),
    ("hga_attn_bwd_dkdv", _I, [_D, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _P]),
    ("hga_attn_bwd_dq", _I, [_D, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    ("hga_fetch_blocks", _I, [_D, _P, _P, _I, _P, _P, _P, _P, _I, _P, ctypes.POINTER(ctypes.c_int), _P, _P, _P,
                              _I]),
    ("hga_gather_blocks_mapped", _I, [_D, _P, _P, _I, _P, _P, _P, _I, _P, _P]),
    ("hga_block_cache_reset", _I, [_C]),
    ("hga_block_cache_plan", _I, [_C, _P, _I, _P, _P, ctypes.POINTER(ctypes.c_int)]),
    ("hga_fetch_blocks_cached", _I, [_D, _P, _P, _P, _P, _P, _P, _C, _P, ctypes.POINTER(ctypes.c_int),
                                     ctypes.POINTER(ctypes.c_int), _P, _P, _P, _I]),
    ("hga_cache_segment", _I, [_D, _P, _P, _P, _P, _C, _I, _P]),
    ("hga_remap_idx", _I, [_D, _P, _P, _P, _P]),
    ("hga_attn_uses_tensor_cores", _I, [_D, _I]),
    ("hga_set_forward_heads_per_cta", _I, [_I]),
    ("hga_append_segment", _I, [_D, _P, _P, _I, _P, _P, _P, _C, _P, _P, _I, _P, _P]),
    ("hga_offload_segment", _I, [_D, _P, _P, _P, _P, _I, _I, _P]),
    ("hga_decode_select", _I, [_D, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    ("hga_decode_workspace_size", ctypes.c_size_t, [_D, _I]),
    ("hga_decode_attn", _I, [_D, _I, _I, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    ("hga_selftest_umma", _I, [_I, _P, _P, _P, _P]),
    ("hga_selftest_attn_fwd_stalled", _I, [_D, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P]),
]

_lib = None


def load_library() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python segmented_fine_tuning_b200/build.py`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, res, args in _SIGNATURES:
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(status: int, where: str):
    if status != HGA_OK:
        raise HgaError(status, where, load_library().hga_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return stream


def _expect(t: torch.Tensor, shape, dtype, name: str, device=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype} != {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def hga_status_string(status: int) -> str:
    return load_library().hga_status_string(status).decode()


def hga_device_status(stream=None) -> None:
    _check(load_library().hga_device_status(_stream(stream)), "hga_device_status")


def hga_block_summaries(dims: Dims, k_hist, blk_begin: int, blk_end: int, summ, stream=None) -> None:
    _expect(k_hist, (dims.B, dims.n_hist_blocks * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "k_hist")
    _expect(summ, (dims.B, dims.n_hist_blocks, dims.Hkv, dims.d), torch.float32, "summ")
    _check(load_library().hga_block_summaries(ctypes.byref(dims.c()), _ptr(k_hist), blk_begin, blk_end, _ptr(summ),
                                              _stream(stream)), "hga_block_summaries")


def hga_segment_summaries(dims: Dims, k_seg, at_block: int, summ, stream=None) -> None:
    """dims.n_hist_blocks is the capacity (blocks) of the summ array."""
    _expect(k_seg, (dims.B, dims.S, dims.Hkv, dims.d), dims.torch_dtype, "k_seg")
    _expect(summ, (dims.B, dims.n_hist_blocks, dims.Hkv, dims.d), torch.float32, "summ")
    _check(load_library().hga_segment_summaries(ctypes.byref(dims.c()), _ptr(k_seg), at_block, _ptr(summ),
                                                _stream(stream)), "hga_segment_summaries")


def hga_select_topk(dims: Dims, q_seg, summ, idx, scores=None, stream=None) -> None:
    _expect(q_seg, (dims.B, dims.S, dims.Hq, dims.d), dims.torch_dtype, "q_seg")
    if summ is None or summ.dim() != 4 or summ.shape[1] < dims.n_hist_blocks or \
            tuple(summ.shape[2:]) != (dims.Hkv, dims.d) or summ.shape[0] != dims.B:
        raise ValueError(f"summ: expected [B, >= n_hist_blocks, Hkv, d], got {None if summ is None else tuple(summ.shape)}")
    if summ.dtype != torch.float32 or not summ.is_contiguous() or not summ.is_cuda:
        raise ValueError("summ must be a contiguous fp32 CUDA tensor")
    if dims.B > 1 and summ.shape[1] != dims.n_hist_blocks:
        raise ValueError("with B > 1 the summ array must hold exactly n_hist_blocks blocks")
    _expect(idx, (dims.B, dims.Hkv, dims.nqb, dims.topk), torch.int32, "idx")
    if scores is not None:
        _expect(scores, idx.shape, torch.float32, "scores")
    _check(load_library().hga_select_topk(ctypes.byref(dims.c()), _ptr(q_seg), _ptr(summ), _ptr(idx), _ptr(scores),
                                          _stream(stream)), "hga_select_topk")


def _attn_shapes(dims: Dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx):
    _expect(q, (dims.B, dims.S, dims.Hq, dims.d), dims.torch_dtype, "q")
    _expect(k_seg, (dims.B, dims.S, dims.Hkv, dims.d), dims.torch_dtype, "k_seg")
    _expect(v_seg, (dims.B, dims.S, dims.Hkv, dims.d), dims.torch_dtype, "v_seg")
    if n_kv_blocks > 0:
        _expect(k_hist, (dims.B, n_kv_blocks * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "k_hist")
        _expect(v_hist, (dims.B, n_kv_blocks * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "v_hist")
    _expect(idx, (dims.B, dims.Hkv, dims.nqb, dims.topk), torch.int32, "idx")


def hga_attn_fwd(dims: Dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks: int, idx, o, lse, stream=None) -> None:
    _attn_shapes(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx)
    _expect(o, q.shape, dims.torch_dtype, "o")
    _expect(lse, (dims.B, dims.Hq, dims.S), torch.float32, "lse")
    _check(load_library().hga_attn_fwd(ctypes.byref(dims.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg), _ptr(k_hist),
                                       _ptr(v_hist), n_kv_blocks, _ptr(idx), _ptr(o), _ptr(lse), _stream(stream)),
           "hga_attn_fwd")


def hga_attn_bwd_workspace_size(dims: Dims) -> int:
    return int(load_library().hga_attn_bwd_workspace_size(ctypes.byref(dims.c())))


def hga_attn_bwd(dims: Dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks: int, idx, o, lse, d_o, dq, dk_seg,
                 dv_seg, ws, stream=None) -> None:
    _attn_shapes(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx)
    _expect(o, q.shape, dims.torch_dtype, "o")
    _expect(d_o, q.shape, dims.torch_dtype, "d_o")
    _expect(lse, (dims.B, dims.Hq, dims.S), torch.float32, "lse")
    _expect(dq, q.shape, torch.float32, "dq")
    _expect(dk_seg, k_seg.shape, torch.float32, "dk_seg")
    _expect(dv_seg, v_seg.shape, torch.float32, "dv_seg")
    if not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous CUDA tensor")
    _check(load_library().hga_attn_bwd(ctypes.byref(dims.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg), _ptr(k_hist),
                                       _ptr(v_hist), n_kv_blocks, _ptr(idx), _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq),
                                       _ptr(dk_seg), _ptr(dv_seg), _ptr(ws), ws.numel() * ws.element_size(),
                                       _stream(stream)), "hga_attn_bwd")


def hga_attn_bwd_noalloc(dims: Dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks: int, idx, o, lse, d_o, dq,
                         dk_seg, dv_seg, stream=None) -> None:
    """hga_attn_bwd without a workspace argument, for callers that cannot
    allocate device memory: the library keeps the scratch in a fixed 4 MiB
    array per device (B*Hq*S <= 2**20).  Calls that overlap on the GPU race on
    that array."""
    _attn_shapes(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx)
    _expect(o, q.shape, dims.torch_dtype, "o")
    _expect(d_o, q.shape, dims.torch_dtype, "d_o")
    _expect(lse, (dims.B, dims.Hq, dims.S), torch.float32, "lse")
    _expect(dq, q.shape, torch.float32, "dq")
    _expect(dk_seg, k_seg.shape, torch.float32, "dk_seg")
    _expect(dv_seg, v_seg.shape, torch.float32, "dv_seg")
    _check(load_library().hga_attn_bwd_noalloc(ctypes.byref(dims.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg),
                                               _ptr(k_hist), _ptr(v_hist), n_kv_blocks, _ptr(idx), _ptr(o), _ptr(lse),
                                               _ptr(d_o), _ptr(dq), _ptr(dk_seg), _ptr(dv_seg), _stream(stream)),
           "hga_attn_bwd_noalloc")


def _ws(ws):
    if not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous CUDA tensor")
    return _ptr(ws), ws.numel() * ws.element_size()


def hga_attn_bwd_preprocess(dims: Dims, o, d_o, ws, stream=None) -> None:
    _expect(o, (dims.B, dims.S, dims.Hq, dims.d), dims.torch_dtype, "o")
    _expect(d_o, o.shape, dims.torch_dtype, "d_o")
    wp, wb = _ws(ws)
    _check(load_library().hga_attn_bwd_preprocess(ctypes.byref(dims.c()), _ptr(o), _ptr(d_o), wp, wb,
                                                  _stream(stream)), "hga_attn_bwd_preprocess")


def hga_attn_bwd_dkdv(dims: Dims, q, k_seg, v_seg, lse, d_o, ws, dk_seg, dv_seg, stream=None) -> None:
    _expect(q, (dims.B, dims.S, dims.Hq, dims.d), dims.torch_dtype, "q")
    _expect(k_seg, (dims.B, dims.S, dims.Hkv, dims.d), dims.torch_dtype, "k_seg")
    _expect(v_seg, k_seg.shape, dims.torch_dtype, "v_seg")
    _expect(lse, (dims.B, dims.Hq, dims.S), torch.float32, "lse")
    _expect(d_o, q.shape, dims.torch_dtype, "d_o")
    _expect(dk_seg, k_seg.shape, torch.float32, "dk_seg")
    _expect(dv_seg, k_seg.shape, torch.float32, "dv_seg")
    wp, wb = _ws(ws)
    _check(load_library().hga_attn_bwd_dkdv(ctypes.byref(dims.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg), _ptr(lse),
                                            _ptr(d_o), wp, wb, _ptr(dk_seg), _ptr(dv_seg), _stream(stream)),
           "hga_attn_bwd_dkdv")


def hga_attn_bwd_dq(dims: Dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks: int, idx, lse, d_o, ws, dq,
                    stream=None) -> None:
    _attn_shapes(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx)
    _expect(lse, (dims.B, dims.Hq, dims.S), torch.float32, "lse")
    _expect(d_o, q.shape, dims.torch_dtype, "d_o")
    _expect(dq, q.shape, torch.float32, "dq")
    wp, wb = _ws(ws)
    _check(load_library().hga_attn_bwd_dq(ctypes.byref(dims.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg), _ptr(k_hist),
                                          _ptr(v_hist), n_kv_blocks, _ptr(idx), _ptr(lse), _ptr(d_o), wp, wb, _ptr(dq),
                                          _stream(stream)), "hga_attn_bwd_dq")


def hga_fetch_blocks(dims: Dims, host_k, host_v, host_capacity_blocks: int, idx_dev, host_idx_scratch, pool_k,
                     pool_v, pool_slots: int, idx_pool_dev, compute_stream, copy_stream, done: torch.cuda.Event,
                     timeout_ms: int = 10000) -> int:
    """Returns the number of distinct history blocks fetched into the pool."""
    shape = (dims.B, host_capacity_blocks * dims.block, dims.Hkv, dims.d)
    _expect(host_k, shape, dims.torch_dtype, "host_k", device=False)
    _expect(host_v, shape, dims.torch_dtype, "host_v", device=False)
    if not (host_k.is_pinned() and host_v.is_pinned() and host_idx_scratch.is_pinned()):
        raise ValueError("host tier and idx scratch must be pinned host memory")
    _expect(idx_dev, (dims.B, dims.Hkv, dims.nqb, dims.topk), torch.int32, "idx_dev")
    _expect(host_idx_scratch, idx_dev.shape, torch.int32, "host_idx_scratch", device=False)
    _expect(pool_k, (dims.B, pool_slots * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "pool_k")
    _expect(pool_v, pool_k.shape, dims.torch_dtype, "pool_v")
    _expect(idx_pool_dev, idx_dev.shape, torch.int32, "idx_pool_dev")
    n_unique = ctypes.c_int(0)
    _check(load_library().hga_fetch_blocks(ctypes.byref(dims.c()), _ptr(host_k), _ptr(host_v), host_capacity_blocks,
                                           _ptr(idx_dev), _ptr(host_idx_scratch), _ptr(pool_k), _ptr(pool_v),
                                           pool_slots, _ptr(idx_pool_dev), ctypes.byref(n_unique),
                                           _stream(compute_stream), _stream(copy_stream), done.cuda_event,
                                           timeout_ms), "hga_fetch_blocks")
    return n_unique.value


class BlockCache:
    """Host-side state of one layer's device block cache (hga_block_cache):
    which history block each pool slot holds, and when each slot was last
    needed.  The arrays are numpy buffers kept alive by this object."""

    def __init__(self, host_capacity_blocks: int, pool_slots: int):
        self.slot_of_block = np.full(max(1, host_capacity_blocks), -1, dtype=np.int32)
        self.block_of_slot = np.full(max(1, pool_slots), -1, dtype=np.int32)
        self.last_use = np.full(max(1, pool_slots), -1, dtype=np.int64)
        self.c = hga_block_cache(self.slot_of_block.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                 self.block_of_slot.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                 self.last_use.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                 host_capacity_blocks, pool_slots, 0)
        self.reset()

    @property
    def host_capacity_blocks(self) -> int:
        return self.c.host_capacity_blocks

    @property
    def pool_slots(self) -> int:
        return self.c.pool_slots

    def reset(self) -> None:
        _check(load_library().hga_block_cache_reset(ctypes.byref(self.c)), "hga_block_cache_reset")

    def plan(self, need):
        """(slots for `need`, the blocks to copy) -- see hga_block_cache_plan."""
        need = np.ascontiguousarray(need, dtype=np.int32)
        slot = np.empty(max(1, need.size), dtype=np.int32)
        miss = np.empty(max(1, need.size), dtype=np.int32)
        n_miss = ctypes.c_int(0)
        _check(load_library().hga_block_cache_plan(ctypes.byref(self.c), need.ctypes.data, int(need.size),
                                                   slot.ctypes.data, miss.ctypes.data, ctypes.byref(n_miss)),
               "hga_block_cache_plan")
        return slot[:need.size].copy(), miss[:n_miss.value].copy()


def hga_fetch_blocks_cached(dims: Dims, host_k, host_v, idx_dev, host_idx_scratch, pool_k, pool_v,
                            cache: BlockCache, idx_pool_dev, compute_stream, copy_stream, done: torch.cuda.Event,
                            timeout_ms: int = 10000):
    """Returns (distinct selected blocks, blocks copied by this call)."""
    shape = (dims.B, cache.host_capacity_blocks * dims.block, dims.Hkv, dims.d)
    _expect(host_k, shape, dims.torch_dtype, "host_k", device=False)
    _expect(host_v, shape, dims.torch_dtype, "host_v", device=False)
    if not (host_k.is_pinned() and host_v.is_pinned() and host_idx_scratch.is_pinned()):
        raise ValueError("host tier and idx scratch must be pinned host memory")
    _expect(idx_dev, (dims.B, dims.Hkv, dims.nqb, dims.topk), torch.int32, "idx_dev")
    _expect(host_idx_scratch, idx_dev.shape, torch.int32, "host_idx_scratch", device=False)
    _expect(pool_k, (dims.B, cache.pool_slots * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "pool_k")
    _expect(pool_v, pool_k.shape, dims.torch_dtype, "pool_v")
    _expect(idx_pool_dev, idx_dev.shape, torch.int32, "idx_pool_dev")
    n_unique, n_fetched = ctypes.c_int(0), ctypes.c_int(0)
    _check(load_library().hga_fetch_blocks_cached(ctypes.byref(dims.c()), _ptr(host_k), _ptr(host_v), _ptr(idx_dev),
                                                  _ptr(host_idx_scratch), _ptr(pool_k), _ptr(pool_v),
                                                  ctypes.byref(cache.c), _ptr(idx_pool_dev), ctypes.byref(n_unique),
                                                  ctypes.byref(n_fetched), _stream(compute_stream),
                                                  _stream(copy_stream), done.cuda_event, timeout_ms),
           "hga_fetch_blocks_cached")
    return n_unique.value, n_fetched.value


def hga_cache_segment(dims: Dims, k_seg, v_seg, pool_k, pool_v, cache: BlockCache, at_block: int,
                      stream=None) -> None:
    _expect(k_seg, (dims.B, dims.S, dims.Hkv, dims.d), dims.torch_dtype, "k_seg")
    _expect(v_seg, k_seg.shape, dims.torch_dtype, "v_seg")
    _expect(pool_k, (dims.B, cache.pool_slots * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "pool_k")
    _expect(pool_v, pool_k.shape, dims.torch_dtype, "pool_v")
    _check(load_library().hga_cache_segment(ctypes.byref(dims.c()), _ptr(k_seg), _ptr(v_seg), _ptr(pool_k),
                                            _ptr(pool_v), ctypes.byref(cache.c), at_block, _stream(stream)),
           "hga_cache_segment")


def hga_remap_idx(dims: Dims, idx_dev, slot_of_block_dev, idx_pool_dev, stream=None) -> None:
    _expect(idx_dev, (dims.B, dims.Hkv, dims.nqb, dims.topk), torch.int32, "idx_dev")
    _expect(idx_pool_dev, idx_dev.shape, torch.int32, "idx_pool_dev")
    if dims.n_hist_blocks > 0:
        if (slot_of_block_dev.dtype != torch.int32 or not slot_of_block_dev.is_cuda or
                slot_of_block_dev.numel() < dims.n_hist_blocks or not slot_of_block_dev.is_contiguous()):
            raise ValueError("slot_of_block_dev: contiguous CUDA int32 with at least n_hist_blocks entries")
    _check(load_library().hga_remap_idx(ctypes.byref(dims.c()), _ptr(idx_dev),
                                        _ptr(slot_of_block_dev) if dims.n_hist_blocks > 0 else None,
                                        _ptr(idx_pool_dev), _stream(stream)), "hga_remap_idx")


def hga_offload_segment(dims: Dims, k_seg, v_seg, host_k, host_v, capacity_blocks: int, at_block: int,
                        stream=None) -> None:
    _expect(k_seg, (dims.B, dims.S, dims.Hkv, dims.d), dims.torch_dtype, "k_seg")
    _expect(v_seg, k_seg.shape, dims.torch_dtype, "v_seg")
    shape = (dims.B, capacity_blocks * dims.block, dims.Hkv, dims.d)
    _expect(host_k, shape, dims.torch_dtype, "host_k", device=False)
    _expect(host_v, shape, dims.torch_dtype, "host_v", device=False)
    _check(load_library().hga_offload_segment(ctypes.byref(dims.c()), _ptr(k_seg), _ptr(v_seg), _ptr(host_k),
                                              _ptr(host_v), capacity_blocks, at_block, _stream(stream)),
           "hga_offload_segment")


def hga_selftest_umma(form: int, a, b, d, stream=None) -> None:
    _expect(a, (128, 128), torch.bfloat16, "a")
    _expect(b, (128, 128), torch.bfloat16, "b")
    _expect(d, (128, 128), torch.float32, "d")
    _check(load_library().hga_selftest_umma(form, _ptr(a), _ptr(b), _ptr(d), _stream(stream)), "hga_selftest_umma")


def hga_selftest_attn_fwd_stalled(dims: Dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks: int, idx, o, lse,
                                  stream=None) -> None:
    """The tensor-core forward with its K/V loads withheld (timeout-path self test)."""
    _attn_shapes(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx)
    _expect(o, q.shape, dims.torch_dtype, "o")
    _expect(lse, (dims.B, dims.Hq, dims.S), torch.float32, "lse")
    _check(load_library().hga_selftest_attn_fwd_stalled(ctypes.byref(dims.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg),
                                                        _ptr(k_hist), _ptr(v_hist), n_kv_blocks, _ptr(idx), _ptr(o),
                                                        _ptr(lse), _stream(stream)),
           "hga_selftest_attn_fwd_stalled")


def hga_decode_select(dims: Dims, q_new, summ, idx, scores, ws, stream=None) -> None:
    """Selection for the n_q = q_new.shape[1] new queries of a decode step
    (scores may be None; ws of hga_decode_workspace_size bytes)."""
    nq = q_new.shape[1]
    _expect(q_new, (dims.B, nq, dims.Hq, dims.d), dims.torch_dtype, "q_new")
    if dims.n_hist_blocks > 0:
        if summ.dtype != torch.float32 or not summ.is_cuda or summ.numel() < dims.B * dims.n_hist_blocks * dims.Hkv * dims.d:
            raise ValueError("summ: CUDA fp32 [B, n_hist_blocks, Hkv, d]")
    _expect(idx, (dims.B, dims.Hkv, dims.topk), torch.int32, "idx")
    if scores is not None:
        _expect(scores, idx.shape, torch.float32, "scores")
    _check(load_library().hga_decode_select(ctypes.byref(dims.c()), nq, _ptr(q_new), _ptr(summ), _ptr(idx),
                                            _ptr(scores), _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)), "hga_decode_select")


def hga_decode_workspace_size(dims: Dims, n_q: int) -> int:
    return int(load_library().hga_decode_workspace_size(ctypes.byref(dims.c()), n_q))


def hga_decode_attn(dims: Dims, t0: int, q_new, k_seg, v_seg, k_hist, v_hist, n_kv_blocks: int, idx, o, lse, ws,
                    stream=None) -> None:
    """Attention of the n_q new queries (segment positions t0..) over the
    selected history blocks and the segment prefix; dims.S is the capacity of
    the segment buffer k_seg/v_seg."""
    nq = q_new.shape[1]
    _expect(q_new, (dims.B, nq, dims.Hq, dims.d), dims.torch_dtype, "q_new")
    _expect(k_seg, (dims.B, dims.S, dims.Hkv, dims.d), dims.torch_dtype, "k_seg")
    _expect(v_seg, k_seg.shape, dims.torch_dtype, "v_seg")
    if n_kv_blocks > 0:
        _expect(k_hist, (dims.B, n_kv_blocks * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "k_hist")
        _expect(v_hist, k_hist.shape, dims.torch_dtype, "v_hist")
    _expect(idx, (dims.B, dims.Hkv, dims.topk), torch.int32, "idx")
    _expect(o, q_new.shape, dims.torch_dtype, "o")
    _expect(lse, (dims.B, dims.Hq, nq), torch.float32, "lse")
    _check(load_library().hga_decode_attn(ctypes.byref(dims.c()), nq, t0, _ptr(q_new), _ptr(k_seg), _ptr(v_seg),
                                          _ptr(k_hist), _ptr(v_hist), n_kv_blocks, _ptr(idx), _ptr(o), _ptr(lse),
                                          _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hga_decode_attn")


def hga_append_segment(dims: Dims, k_seg, v_seg, at_block: int, summ, pool_k=None, pool_v=None,
                       cache: "BlockCache | None" = None, host_k=None, host_v=None, tier_capacity_blocks: int = 0,
                       stream=None, copy_stream=None) -> None:
    """A finished segment enters the history in one pass: summaries of its
    blocks (dims.n_hist_blocks = summ's capacity), optionally its K/V into the
    device block cache, optionally the copy to the pinned host tier."""
    _expect(k_seg, (dims.B, dims.S, dims.Hkv, dims.d), dims.torch_dtype, "k_seg")
    _expect(v_seg, k_seg.shape, dims.torch_dtype, "v_seg")
    _expect(summ, (dims.B, dims.n_hist_blocks, dims.Hkv, dims.d), torch.float32, "summ")
    if cache is not None:
        _expect(pool_k, (dims.B, cache.pool_slots * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "pool_k")
        _expect(pool_v, pool_k.shape, dims.torch_dtype, "pool_v")
    if host_k is not None or host_v is not None:
        shape = (dims.B, tier_capacity_blocks * dims.block, dims.Hkv, dims.d)
        _expect(host_k, shape, dims.torch_dtype, "host_k", device=False)
        _expect(host_v, shape, dims.torch_dtype, "host_v", device=False)
        if not (host_k.is_pinned() and host_v.is_pinned()):
            raise ValueError("host tier must be pinned host memory")
    _check(load_library().hga_append_segment(
        ctypes.byref(dims.c()), _ptr(k_seg), _ptr(v_seg), at_block, _ptr(summ),
        _ptr(pool_k) if cache is not None else None, _ptr(pool_v) if cache is not None else None,
        ctypes.byref(cache.c) if cache is not None else None, _ptr(host_k), _ptr(host_v), tier_capacity_blocks,
        _stream(stream), _stream(copy_stream) if copy_stream is not None else None), "hga_append_segment")


def hga_gather_blocks_mapped(dims: Dims, host_k, host_v, host_capacity_blocks: int, idx_dev, pool_k, pool_v,
                             pool_slots: int, idx_pool_dev, stream=None) -> None:
    """The distinct selected blocks copied by the GPU from the mapped pinned
    host tier into a compact pool, idx rewritten to slots; no host wait."""
    shape = (dims.B, host_capacity_blocks * dims.block, dims.Hkv, dims.d)
    _expect(host_k, shape, dims.torch_dtype, "host_k", device=False)
    _expect(host_v, shape, dims.torch_dtype, "host_v", device=False)
    if not (host_k.is_pinned() and host_v.is_pinned()):
        raise ValueError("host tier must be pinned host memory")
    _expect(idx_dev, (dims.B, dims.Hkv, dims.nqb, dims.topk), torch.int32, "idx_dev")
    _expect(pool_k, (dims.B, pool_slots * dims.block, dims.Hkv, dims.d), dims.torch_dtype, "pool_k")
    _expect(pool_v, pool_k.shape, dims.torch_dtype, "pool_v")
    _expect(idx_pool_dev, idx_dev.shape, torch.int32, "idx_pool_dev")
    _check(load_library().hga_gather_blocks_mapped(ctypes.byref(dims.c()), _ptr(host_k), _ptr(host_v),
                                                   host_capacity_blocks, _ptr(idx_dev), _ptr(pool_k), _ptr(pool_v),
                                                   pool_slots, _ptr(idx_pool_dev), _stream(stream)),
           "hga_gather_blocks_mapped")


def hga_attn_bwd_sparse(dims: Dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks: int, idx, o, lse, d_o,
                        qblock_mask, scale: float, dq, dk_seg, dv_seg, ws, stream=None) -> None:
    """SpaCO-style sparse backward: only query blocks with qblock_mask[b, i]
    != 0 propagate gradient, every gradient multiplied by `scale`."""
    _attn_shapes(dims, q, k_seg, v_seg, k_hist, v_hist, n_kv_blocks, idx)
    _expect(qblock_mask, (dims.B, dims.nqb), torch.uint8, "qblock_mask")
    for t, shp, nm in ((dq, q.shape, "dq"), (dk_seg, k_seg.shape, "dk_seg"), (dv_seg, v_seg.shape, "dv_seg")):
        _expect(t, shp, torch.float32, nm)
    _check(load_library().hga_attn_bwd_sparse(ctypes.byref(dims.c()), _ptr(q), _ptr(k_seg), _ptr(v_seg),
                                              _ptr(k_hist), _ptr(v_hist), n_kv_blocks, _ptr(idx), _ptr(o), _ptr(lse),
                                              _ptr(d_o), _ptr(qblock_mask), float(scale), _ptr(dq), _ptr(dk_seg),
                                              _ptr(dv_seg), _ptr(ws), ws.numel() * ws.element_size(),
                                              _stream(stream)), "hga_attn_bwd_sparse")


def spaco_sample_blocks(B: int, n_qblocks: int, k: int, generator: torch.Generator, cap: float | None = None):
    """Host helper for a sparse backward step: k of the n_qblocks query blocks
    of each sequence chosen uniformly without replacement (seeded generator),
    and the correction factor t/k (capped at `cap` when given).  Returns
    (uint8 mask [B, n_qblocks] on the CPU, scale)."""
    if not 1 <= k <= n_qblocks:
        raise ValueError("need 1 <= k <= n_qblocks")
    mask = torch.zeros((B, n_qblocks), dtype=torch.uint8)
    for b in range(B):
        mask[b, torch.randperm(n_qblocks, generator=generator)[:k]] = 1
    scale = n_qblocks / k
    return mask, (min(scale, cap) if cap is not None else scale)


def hga_set_forward_heads_per_cta(heads: int):
    """Query heads per CTA of the tensor-core forward for later calls from this thread: 2, 1, or 0 (automatic)."""
    _check(load_library().hga_set_forward_heads_per_cta(heads), "hga_set_forward_heads_per_cta")


def hga_attn_uses_tensor_cores(dims: Dims, n_kv_blocks: int) -> bool:
    """True when the attention calls run these dims on the tcgen05 kernels."""
    r = load_library().hga_attn_uses_tensor_cores(ctypes.byref(dims.c()), n_kv_blocks)
    if r < 0:
        raise ValueError(f"dims rejected by the library: {load_library().hga_last_error().decode()}")
    return bool(r)
