"""Python binding of the C ABI in ``include/kvcr.h`` (ctypes, marshalling only).

Every function here has the name of the C entry point it calls and only turns
Python / torch arguments into pointers and sizes; all work runs in the
library's CUDA kernels.  The library is the in-tree ``libkvcr.so`` built by
``kv_cache_chunk_ring_b200.build``; importing a function that needs it raises
when it is missing (there is no fallback).  torch is used for device memory
and streams only.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import List, Optional, Sequence, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvcr.so")

KVCR_OK, KVCR_EINVAL, KVCR_ESHAPE, KVCR_ESTATE = 0, -1, -2, -3
KVCR_ECUDA, KVCR_ETIMEOUT, KVCR_ESTORAGE, KVCR_EUNSUPPORTED = -4, -5, -6, -7
KVCR_BF16, KVCR_F32 = 0, 1
KVCR_TILE_EMPTY, KVCR_TILE_PARTIAL, KVCR_TILE_FULL = 0, 1, 2
KVCR_CACHE_FP8_K, KVCR_CACHE_FUSED_FINALIZE = 1, 2
(KVCR_K_APPEND_ROPE, KVCR_K_ROPE_STAGE, KVCR_K_CHUNK_ATTN, KVCR_K_MOBA_ATTN,
 KVCR_K_ATTN_F32, KVCR_K_MOBA_BWD_PREP, KVCR_K_MOBA_BWD_DKDV, KVCR_K_MOBA_BWD_DQ,
 KVCR_K_SET_AUX, KVCR_K_APPEND_BATCH, KVCR_K_QUANT_E4M3, KVCR_K_CHUNK_ATTN_FP8) = range(12)
KERNEL_NAMES = {KVCR_K_APPEND_ROPE: "append_rope", KVCR_K_ROPE_STAGE: "rope_stage",
                KVCR_K_CHUNK_ATTN: "chunk_attn", KVCR_K_MOBA_ATTN: "moba_attn",
                KVCR_K_ATTN_F32: "attn_f32", KVCR_K_MOBA_BWD_PREP: "moba_bwd_prep",
                KVCR_K_MOBA_BWD_DKDV: "moba_bwd_dkdv", KVCR_K_MOBA_BWD_DQ: "moba_bwd_dq",
                KVCR_K_SET_AUX: "set_aux", KVCR_K_APPEND_BATCH: "append_batch",
                KVCR_K_QUANT_E4M3: "quant_e4m3", KVCR_K_CHUNK_ATTN_FP8: "chunk_attn_fp8"}

# every symbol include/kvcr.h declares
EXPORTS = [
    "kv_cache_storage_bytes", "kv_cache_init", "kv_cache_storage_bytes_aux", "kv_cache_init_aux",
    "kv_cache_storage_bytes_ex", "kv_cache_init_ex", "kv_cache_slot_data_fp8",
    "chunk_attention_fwd_fp8", "chunk_attention_fwd_finalize", "kv_cache_export_state",
    "kv_cache_import_state",
    "kv_cache_set_aux", "kv_cache_num_aux", "kv_cache_append_rope", "kv_cache_append_rope_batch",
    "kv_cache_evict",
    "kv_cache_slot_map", "kv_cache_last_append", "kv_cache_num_cached", "kv_cache_slot_data",
    "kv_cache_destroy",
    "chunk_attention_fwd", "chunk_attention_fwd_static_scratch", "moba_attention_fwd",
    "moba_attention_bwd", "moba_attention_bwd_workspace_bytes", "moba_classify_tiles",
    "kvcr_check_status",
    "kvcr_last_error", "kvcr_launch_count", "kvcr_debug_inject", "kvcr_trace_enable",
    "kvcr_trace_reset", "kvcr_trace_read",
]


class KvcrError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"kvcr status {code}: {msg}")
        self.code = code


class KvcrArgError(KvcrError, ValueError):
    """A tensor argument that does not match what the call reads or writes; raised by
    the binding before anything reaches the library (nothing is launched)."""


# Sizes of every live cache handle (handle value -> (T, H, D, dtype code, has RoPE)), so the
# tensor-taking calls can check their arguments against the cache before a launch.
_CACHE_INFO = {}


def _expect(specs) -> None:
    """Raise KvcrArgError unless every (name, tensor, shape, torch dtype) of ``specs`` is a
    contiguous tensor of exactly that shape and dtype, and all of them are CUDA tensors
    on one device.  Shapes, dtypes and layouts are checked before devices, so a
    mismatch is reported the same way on a host without a GPU."""
    for name, t, shape, dtype in specs:
        if t is None:
            raise KvcrArgError(KVCR_EINVAL, f"{name} is required")
        shape = tuple(int(x) for x in shape)
        if tuple(t.shape) != shape:
            raise KvcrArgError(KVCR_ESHAPE, f"{name} has shape {tuple(t.shape)}, expected {shape}")
        if t.dtype != dtype:
            raise KvcrArgError(KVCR_EINVAL, f"{name} has dtype {t.dtype}, expected {dtype}")
        if not t.is_contiguous():
            raise KvcrArgError(KVCR_EINVAL, f"{name} must be contiguous")
    device = specs[0][1].device
    for name, t, _, _ in specs:
        if not t.is_cuda:
            raise KvcrArgError(KVCR_EINVAL, f"{name} must be a CUDA tensor")
        if t.device != device:
            raise KvcrArgError(KVCR_EINVAL, f"{name} is on {t.device}, {specs[0][0]} on {device}")


def _torch_dtype(code: int):
    import torch
    return torch.bfloat16 if code == KVCR_BF16 else torch.float32


def _cache_info(handle):
    key = handle.value if isinstance(handle, ctypes.c_void_p) else handle
    info = _CACHE_INFO.get(key)
    if info is None:
        raise KvcrArgError(KVCR_EINVAL, "unknown or destroyed cache handle")
    return info


def _check_chunk_args(handle, q, k_cur, v_cur, n_frames: int, o, lse) -> None:
    """Tensor arguments of chunk attention against the cache's sizes."""
    import torch
    T, H, D, dt, rope = _cache_info(handle)
    if q is None or q.dim() != 3:
        raise KvcrArgError(KVCR_ESHAPE, "q must be [n_q, heads, head_dim]")
    n_q, n_cur = q.shape[0], n_frames * T
    if rope and n_q != n_cur:
        raise KvcrArgError(KVCR_ESHAPE, f"q has {n_q} rows; with RoPE it must have "
                                        f"n_cur_frames * tokens_per_frame = {n_cur}")
    dt = _torch_dtype(dt)
    specs = [("q", q, (n_q, H, D), dt), ("k_cur", k_cur, (n_cur, H, D), dt),
             ("v_cur", v_cur, (n_cur, H, D), dt), ("o", o, (n_q, H, D), dt)]
    if lse is not None:
        specs.append(("lse", lse, (H, n_q), torch.float32))
    _expect(specs)


def _check_kv(handle, k, v, n_frames: int, what: str) -> None:
    T, H, D, dt, _ = _cache_info(handle)
    if k is None and v is None:
        return                                   # bookkeeping-only call; the library checks
    dt = _torch_dtype(dt)
    _expect([(f"{what} k", k, (n_frames * T, H, D), dt),
             (f"{what} v", v, (n_frames * T, H, D), dt)])


def _check_moba_args(L: int, tensors, lse) -> None:
    """q, k, v, o (and the backward's tensors) all [L, heads, head_dim] in one dtype and
    device; lse fp32 [heads, L]."""
    import torch
    first = tensors[0][1]
    if first is None or first.dim() != 3:
        raise KvcrArgError(KVCR_ESHAPE, f"{tensors[0][0]} must be [L, heads, head_dim]")
    shape = (L, first.shape[1], first.shape[2])
    specs = [(name, t, shape, first.dtype) for name, t in tensors]
    if lse is not None:
        specs.append(("lse", lse, (shape[1], L), torch.float32))
    _expect(specs)


class kvcr_rope(ctypes.Structure):
    _fields_ = [("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("pairs_t", ctypes.c_int),
                ("pairs_h", ctypes.c_int), ("pairs_w", ctypes.c_int), ("base", ctypes.c_double)]


class kvcr_moba_layout(ctypes.Structure):
    _fields_ = [("n_chunks", ctypes.c_int), ("chunk_tokens", ctypes.c_int),
                ("n_bidir_chunks", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded ``libkvcr.so``; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m kv_cache_chunk_ring_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    c_int, c_p, c_sz, c_f = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
    i32p = ctypes.POINTER(ctypes.c_int32)
    sig = {
        "kv_cache_storage_bytes": (c_sz, [c_int] * 7 + [c_int]),
        "kv_cache_init": (c_int, [ctypes.POINTER(c_p), c_int, c_int, c_int, c_int, c_int, c_int,
                                  ctypes.POINTER(kvcr_rope), c_int, c_p, c_sz]),
        "kv_cache_storage_bytes_aux": (c_sz, [c_int] * 8 + [c_int]),
        "kv_cache_init_aux": (c_int, [ctypes.POINTER(c_p), c_int, c_int, c_int, c_int, c_int, c_int,
                                      c_int, ctypes.POINTER(kvcr_rope), c_int, c_p, c_sz]),
        "kv_cache_storage_bytes_ex": (c_sz, [c_int] * 9 + [ctypes.c_uint]),
        "kv_cache_init_ex": (c_int, [ctypes.POINTER(c_p), c_int, c_int, c_int, c_int, c_int, c_int,
                                     c_int, ctypes.POINTER(kvcr_rope), c_int, ctypes.c_uint, c_p,
                                     c_sz]),
        "kv_cache_slot_data_fp8": (c_int, [c_p, c_int, ctypes.POINTER(c_p), ctypes.POINTER(c_p)]),
        "kv_cache_export_state": (c_int, [c_p, c_p, c_sz, ctypes.POINTER(c_sz)]),
        "kv_cache_import_state": (c_int, [c_p, c_p, c_sz]),
        "chunk_attention_fwd_fp8": (c_int, [c_p, c_p, c_int, c_p, c_p, i32p, c_int, c_f, c_p, c_p,
                                            c_p]),
        "chunk_attention_fwd_finalize": (c_int, [c_p, c_p, c_int, c_p, c_p, i32p, c_int, c_f, c_p,
                                                 c_p, c_p]),
        "kv_cache_set_aux": (c_int, [c_p, c_p, c_p, i32p, c_int, c_p]),
        "kv_cache_num_aux": (c_int, [c_p, ctypes.POINTER(c_int)]),
        "kv_cache_append_rope": (c_int, [c_p, c_p, c_p, i32p, c_int, c_p]),
        "kv_cache_append_rope_batch": (c_int, [ctypes.POINTER(c_p), c_int, ctypes.POINTER(c_p),
                                               ctypes.POINTER(c_p), i32p, c_int, c_p]),
        "kv_cache_evict": (c_int, [c_p, c_int, i32p, c_int, ctypes.POINTER(c_int)]),
        "kv_cache_slot_map": (c_int, [c_p, i32p, c_int]),
        "kv_cache_last_append": (c_int, [c_p, i32p, c_int, i32p, c_int, ctypes.POINTER(c_int)]),
        "kv_cache_num_cached": (c_int, [c_p, ctypes.POINTER(c_int)]),
        "kv_cache_slot_data": (c_int, [c_p, c_int, ctypes.POINTER(c_p), ctypes.POINTER(c_p)]),
        "kv_cache_destroy": (None, [c_p]),
        "chunk_attention_fwd": (c_int, [c_p, c_p, c_int, c_p, c_p, i32p, c_int, c_f, c_p, c_p,
                                        c_p]),
        "chunk_attention_fwd_static_scratch": (c_int, [c_p, c_p, c_int, c_p, c_p, i32p, c_int,
                                                       c_f, c_p, c_p, c_p]),
        "moba_attention_fwd": (c_int, [c_p, c_p, c_p, ctypes.POINTER(kvcr_moba_layout), c_int,
                                       c_int, c_int, c_f, c_p, c_p, c_p]),
        "moba_attention_bwd": (c_int, [c_p, c_p, c_p, c_p, c_p, c_p,
                                       ctypes.POINTER(kvcr_moba_layout), c_int, c_int, c_int, c_f,
                                       c_p, c_p, c_p, c_p, c_sz, c_p]),
        "moba_attention_bwd_workspace_bytes": (c_sz, [ctypes.POINTER(kvcr_moba_layout), c_int]),
        "moba_classify_tiles": (c_int, [ctypes.POINTER(kvcr_moba_layout), c_int, c_p, c_sz]),
        "kvcr_check_status": (c_int, [c_p]),
        "kvcr_last_error": (ctypes.c_char_p, []),
        "kvcr_launch_count": (ctypes.c_longlong, []),
        "kvcr_debug_inject": (c_int, [c_int, ctypes.c_longlong]),
        "kvcr_trace_enable": (c_int, [c_int]),
        "kvcr_trace_reset": (c_int, []),
        "kvcr_trace_read": (c_int, [c_int, ctypes.POINTER(ctypes.c_longlong),
                                    ctypes.POINTER(ctypes.c_double)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(rc: int) -> None:
    if rc != KVCR_OK:
        raise KvcrError(rc, lib().kvcr_last_error().decode())


def _i32(seq: Sequence[int]):
    arr = (ctypes.c_int32 * max(1, len(seq)))(*[int(x) for x in seq])
    return arr


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _dtype_code(dtype) -> int:
    import torch
    if dtype in (torch.bfloat16, "bf16", KVCR_BF16):
        return KVCR_BF16
    if dtype in (torch.float32, "f32", KVCR_F32):
        return KVCR_F32
    raise ValueError(f"unsupported dtype {dtype}")


# ---------------------------------------------------------------- C names ---

def kv_cache_storage_bytes(sinks, window, tokens_per_frame, heads, head_dim, chunk_frames,
                           with_rope, dtype) -> int:
    return int(lib().kv_cache_storage_bytes(sinks, window, tokens_per_frame, heads, head_dim,
                                            chunk_frames, int(bool(with_rope)),
                                            _dtype_code(dtype)))


def kv_cache_storage_bytes_aux(sinks, window, aux_frames, tokens_per_frame, heads, head_dim,
                               chunk_frames, with_rope, dtype) -> int:
    return int(lib().kv_cache_storage_bytes_aux(sinks, window, aux_frames, tokens_per_frame, heads,
                                                head_dim, chunk_frames, int(bool(with_rope)),
                                                _dtype_code(dtype)))


def kv_cache_init_aux(sinks, window, aux_frames, tokens_per_frame, heads, head_dim, chunk_frames,
                      rope, dtype, storage) -> ctypes.c_void_p:
    """Create a cache with ``aux_frames`` auxiliary slots over ``storage``."""
    return kv_cache_init_ex(sinks, window, aux_frames, tokens_per_frame, heads, head_dim,
                            chunk_frames, rope, dtype, 0, storage)


def kv_cache_storage_bytes_ex(sinks, window, aux_frames, tokens_per_frame, heads, head_dim,
                              chunk_frames, with_rope, dtype, flags) -> int:
    return int(lib().kv_cache_storage_bytes_ex(sinks, window, aux_frames, tokens_per_frame, heads,
                                               head_dim, chunk_frames, int(bool(with_rope)),
                                               _dtype_code(dtype), int(flags)))


def kv_cache_init_ex(sinks, window, aux_frames, tokens_per_frame, heads, head_dim, chunk_frames,
                     rope, dtype, flags, storage) -> ctypes.c_void_p:
    """Create a cache with ``aux_frames`` auxiliary slots and cache ``flags``
    (KVCR_CACHE_FP8_K) over ``storage``."""
    h = ctypes.c_void_p()
    rp = None
    if rope is not None:
        rp = ctypes.byref(kvcr_rope(rope.grid_h, rope.grid_w, rope.pairs_t, rope.pairs_h,
                                    rope.pairs_w, float(rope.base)))
    ptr = None if storage is None else storage.data_ptr()
    nbytes = 0 if storage is None else storage.numel() * storage.element_size()
    _check(lib().kv_cache_init_ex(ctypes.byref(h), sinks, window, aux_frames, tokens_per_frame,
                                  heads, head_dim, chunk_frames, rp, _dtype_code(dtype),
                                  int(flags), ptr, nbytes))
    _CACHE_INFO[h.value] = (tokens_per_frame, heads, head_dim, _dtype_code(dtype),
                            rope is not None)
    return h


def kv_cache_set_aux(handle, k, v, aux_pos: Optional[Sequence[int]], n_frames: int,
                     stream=None) -> None:
    _check_kv(handle, k, v, n_frames, "kv_cache_set_aux")
    s = None if (k is None and v is None) else _stream(stream)
    pos = None if aux_pos is None else _i32(aux_pos)
    _check(lib().kv_cache_set_aux(handle, _ptr(k), _ptr(v), pos, n_frames, s))


def kv_cache_num_aux(handle) -> int:
    n = ctypes.c_int()
    _check(lib().kv_cache_num_aux(handle, ctypes.byref(n)))
    return n.value


def kv_cache_init(sinks, window, tokens_per_frame, heads, head_dim, chunk_frames, rope, dtype,
                  storage) -> ctypes.c_void_p:
    """Create a cache over ``storage`` (a CUDA tensor, or None for bookkeeping only)."""
    h = ctypes.c_void_p()
    rp = None
    if rope is not None:
        rp = ctypes.byref(kvcr_rope(rope.grid_h, rope.grid_w, rope.pairs_t, rope.pairs_h,
                                    rope.pairs_w, float(rope.base)))
    ptr = None if storage is None else storage.data_ptr()
    nbytes = 0 if storage is None else storage.numel() * storage.element_size()
    _check(lib().kv_cache_init(ctypes.byref(h), sinks, window, tokens_per_frame, heads, head_dim,
                               chunk_frames, rp, _dtype_code(dtype), ptr, nbytes))
    _CACHE_INFO[h.value] = (tokens_per_frame, heads, head_dim, _dtype_code(dtype),
                            rope is not None)
    return h


def kv_cache_append_rope(handle, k, v, frame_idx: Sequence[int], stream=None) -> None:
    n = len(frame_idx)
    _check_kv(handle, k, v, n, "kv_cache_append_rope")
    s = None if (k is None and v is None) else _stream(stream)
    _check(lib().kv_cache_append_rope(handle, _ptr(k), _ptr(v), _i32(frame_idx), n, s))


def kv_cache_append_rope_batch(handles, ks, vs, frame_idx: Sequence[int], stream=None) -> None:
    """One launch appending the same frames to several caches (ks[i], vs[i] for handles[i];
    ks = vs = None for bookkeeping-only caches)."""
    n = len(handles)
    hs = (ctypes.c_void_p * n)(*[h.value if isinstance(h, ctypes.c_void_p) else h for h in handles])
    if ks is None:
        kp = vp = None
        s = None
    else:
        if len(ks) != n or len(vs) != n:
            raise KvcrArgError(KVCR_ESHAPE, "one k and one v per cache")
        specs = []
        for i, h in enumerate(handles):
            T, H, D, dt, _ = _cache_info(h)
            shape = (len(frame_idx) * T, H, D)
            specs += [(f"kv_cache_append_rope_batch[{i}] k", ks[i], shape, _torch_dtype(dt)),
                      (f"kv_cache_append_rope_batch[{i}] v", vs[i], shape, _torch_dtype(dt))]
        _expect(specs)
        kp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in ks])
        vp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in vs])
        s = _stream(stream)
    _check(lib().kv_cache_append_rope_batch(hs, n, kp, vp, _i32(frame_idx), len(frame_idx), s))


def append_batch(caches, ks, vs, frames: Sequence[int], stream=None) -> None:
    """Cache-level wrapper of kv_cache_append_rope_batch."""
    kv_cache_append_rope_batch([c.handle for c in caches], ks, vs, frames, stream)


def kv_cache_evict(handle, keep_recent: int) -> List[int]:
    buf = (ctypes.c_int32 * 64)()
    n = ctypes.c_int()
    _check(lib().kv_cache_evict(handle, keep_recent, buf, 64, ctypes.byref(n)))
    return [int(buf[i]) for i in range(min(n.value, 64))]


def kv_cache_slot_map(handle, n_slots: int) -> List[int]:
    buf = (ctypes.c_int32 * n_slots)()
    _check(lib().kv_cache_slot_map(handle, buf, n_slots))
    return [int(x) for x in buf]


def kv_cache_last_append(handle, n_frames: int) -> Tuple[List[int], List[int]]:
    sl = (ctypes.c_int32 * max(1, n_frames))()
    ev = (ctypes.c_int32 * 64)()
    n = ctypes.c_int()
    _check(lib().kv_cache_last_append(handle, sl, n_frames, ev, 64, ctypes.byref(n)))
    return [int(sl[i]) for i in range(n_frames)], [int(ev[i]) for i in range(min(n.value, 64))]


def kv_cache_num_cached(handle) -> int:
    n = ctypes.c_int()
    _check(lib().kv_cache_num_cached(handle, ctypes.byref(n)))
    return n.value


def kv_cache_slot_data(handle, slot: int) -> Tuple[int, int]:
    """Device addresses (ints) of one slot's K and V."""
    k = ctypes.c_void_p()
    v = ctypes.c_void_p()
    _check(lib().kv_cache_slot_data(handle, slot, ctypes.byref(k), ctypes.byref(v)))
    return int(k.value), int(v.value)


def kv_cache_export_state(handle) -> bytes:
    """The cache's host state (slot table, recency, relabelling, counts) as bytes."""
    n = ctypes.c_size_t()
    _check(lib().kv_cache_export_state(handle, None, 0, ctypes.byref(n)))
    buf = ctypes.create_string_buffer(n.value)
    _check(lib().kv_cache_export_state(handle, buf, n.value, ctypes.byref(n)))
    return buf.raw[:n.value]


def kv_cache_import_state(handle, state: bytes) -> None:
    """Restore a state from kv_cache_export_state into a cache of the same configuration."""
    buf = ctypes.create_string_buffer(bytes(state), len(state))
    _check(lib().kv_cache_import_state(handle, buf, len(state)))


def kv_cache_destroy(handle) -> None:
    _CACHE_INFO.pop(handle.value if isinstance(handle, ctypes.c_void_p) else handle, None)
    lib().kv_cache_destroy(handle)


def chunk_attention_fwd(handle, q, k_cur, v_cur, cur_frame_idx: Sequence[int], o, lse=None,
                        softmax_scale: float = 0.0, stream=None) -> None:
    _check_chunk_args(handle, q, k_cur, v_cur, len(cur_frame_idx), o, lse)
    _check(lib().chunk_attention_fwd(handle, _ptr(q), q.shape[0], _ptr(k_cur), _ptr(v_cur),
                                     _i32(cur_frame_idx), len(cur_frame_idx),
                                     float(softmax_scale), _ptr(o), _ptr(lse), _stream(stream)))


def chunk_attention_fwd_fp8(handle, q, k_cur, v_cur, cur_frame_idx: Sequence[int], o, lse=None,
                            softmax_scale: float = 0.0, stream=None) -> None:
    """chunk_attention_fwd with the QK^T product in e4m3 (cache made with KVCR_CACHE_FP8_K)."""
    _check_chunk_args(handle, q, k_cur, v_cur, len(cur_frame_idx), o, lse)
    _check(lib().chunk_attention_fwd_fp8(handle, _ptr(q), q.shape[0], _ptr(k_cur), _ptr(v_cur),
                                         _i32(cur_frame_idx), len(cur_frame_idx),
                                         float(softmax_scale), _ptr(o), _ptr(lse),
                                         _stream(stream)))


def chunk_attention_fwd_finalize(handle, q, k_cur, v_cur, cur_frame_idx: Sequence[int], o,
                                 lse=None, softmax_scale: float = 0.0, stream=None) -> None:
    """chunk_attention_fwd then the append of k_cur, v_cur, in one pass over K and V (cache
    made with KVCR_CACHE_FUSED_FINALIZE)."""
    _check_chunk_args(handle, q, k_cur, v_cur, len(cur_frame_idx), o, lse)
    _check(lib().chunk_attention_fwd_finalize(handle, _ptr(q), q.shape[0], _ptr(k_cur),
                                              _ptr(v_cur), _i32(cur_frame_idx),
                                              len(cur_frame_idx), float(softmax_scale), _ptr(o),
                                              _ptr(lse), _stream(stream)))


def kv_cache_slot_data_fp8(handle, slot: int) -> Tuple[int, int]:
    """Device addresses (ints) of one slot's e4m3 K codes and block scales."""
    k = ctypes.c_void_p()
    sc = ctypes.c_void_p()
    _check(lib().kv_cache_slot_data_fp8(handle, slot, ctypes.byref(k), ctypes.byref(sc)))
    return int(k.value), int(sc.value)


def chunk_attention_fwd_static_scratch(handle, q, k_cur, v_cur, cur_frame_idx: Sequence[int], o,
                                       lse=None, softmax_scale: float = 0.0,
                                       stream=None) -> None:
    """chunk_attention_fwd staged in the library's fixed device array (allocates nothing)."""
    _check_chunk_args(handle, q, k_cur, v_cur, len(cur_frame_idx), o, lse)
    _check(lib().chunk_attention_fwd_static_scratch(
        handle, _ptr(q), q.shape[0], _ptr(k_cur), _ptr(v_cur), _i32(cur_frame_idx),
        len(cur_frame_idx), float(softmax_scale), _ptr(o), _ptr(lse), _stream(stream)))


def moba_attention_fwd(q, k, v, n_chunks: int, chunk_tokens: int, n_bidir_chunks: int, o,
                       lse=None, softmax_scale: float = 0.0, stream=None) -> None:
    L = (2 * n_chunks + n_bidir_chunks) * chunk_tokens
    _check_moba_args(L, [("q", q), ("k", k), ("v", v), ("o", o)], lse)
    lay = kvcr_moba_layout(n_chunks, chunk_tokens, n_bidir_chunks)
    _check(lib().moba_attention_fwd(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(lay), q.shape[1],
                                    q.shape[2], _dtype_code(q.dtype), float(softmax_scale),
                                    _ptr(o), _ptr(lse), _stream(stream)))


def moba_attention_bwd_workspace_bytes(n_chunks: int, chunk_tokens: int, n_bidir_chunks: int,
                                       heads: int) -> int:
    lay = kvcr_moba_layout(n_chunks, chunk_tokens, n_bidir_chunks)
    return int(lib().moba_attention_bwd_workspace_bytes(ctypes.byref(lay), heads))


def moba_attention_bwd(q, k, v, o, d_o, lse, n_chunks: int, chunk_tokens: int,
                       n_bidir_chunks: int, dq, dk, dv, workspace=None,
                       softmax_scale: float = 0.0, stream=None) -> None:
    """dQ, dK, dV of moba_attention_fwd into dq, dk, dv.  ``workspace`` is a device
    tensor of at least moba_attention_bwd_workspace_bytes() bytes (allocated here
    with torch when omitted)."""
    L = (2 * n_chunks + n_bidir_chunks) * chunk_tokens
    if lse is None:
        raise KvcrArgError(KVCR_EINVAL, "lse (the forward's) is required")
    _check_moba_args(L, [("q", q), ("k", k), ("v", v), ("o", o), ("d_o", d_o), ("dq", dq),
                         ("dk", dk), ("dv", dv)], lse)
    lay = kvcr_moba_layout(n_chunks, chunk_tokens, n_bidir_chunks)
    need = int(lib().moba_attention_bwd_workspace_bytes(ctypes.byref(lay), q.shape[1]))
    if workspace is None:
        import torch
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or workspace.device != q.device or not workspace.is_contiguous():
        raise KvcrArgError(KVCR_EINVAL, "workspace must be a contiguous tensor on q's device")
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().moba_attention_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(d_o), _ptr(lse), ctypes.byref(lay),
        q.shape[1], q.shape[2], _dtype_code(q.dtype), float(softmax_scale), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(workspace), nbytes, _stream(stream)))


def moba_classify_tiles(n_chunks: int, chunk_tokens: int, n_bidir_chunks: int, tile: int = 128):
    import numpy as np
    lay = kvcr_moba_layout(n_chunks, chunk_tokens, n_bidir_chunks)
    L = (2 * n_chunks + n_bidir_chunks) * chunk_tokens
    nt = (L + tile - 1) // tile
    out = np.zeros((nt, nt), dtype=np.uint8)
    _check(lib().moba_classify_tiles(ctypes.byref(lay), tile, out.ctypes.data, out.size))
    return out


def kvcr_check_status(stream=None) -> None:
    _check(lib().kvcr_check_status(_stream(stream)))


def kvcr_launch_count() -> int:
    return int(lib().kvcr_launch_count())


def kvcr_debug_inject(kind: int, wait_ns: int = 0) -> None:
    """Failure-path test hook (see include/kvcr.h); kind 0 turns it off."""
    _check(lib().kvcr_debug_inject(int(kind), int(wait_ns)))


def kvcr_trace_enable(on: bool) -> None:
    _check(lib().kvcr_trace_enable(int(bool(on))))


def kvcr_trace_reset() -> None:
    _check(lib().kvcr_trace_reset())


def kvcr_trace_read(kernel_id: int) -> Tuple[int, float]:
    n = ctypes.c_longlong()
    ms = ctypes.c_double()
    _check(lib().kvcr_trace_read(kernel_id, ctypes.byref(n), ctypes.byref(ms)))
    return int(n.value), float(ms.value)


# ------------------------------------------------------------- convenience ---

class Cache:
    """One layer's KV cache: owns the C handle and keeps its device storage alive."""

    def __init__(self, sinks: int, window: int, tokens_per_frame: int, heads: int, head_dim: int,
                 chunk_frames: int, rope=None, dtype="bf16", device="cuda",
                 bookkeeping_only: bool = False, aux_frames: int = 0, fp8_k: bool = False,
                 fused_finalize: bool = False):
        self.sinks, self.window, self.aux_frames = sinks, window, aux_frames
        self.flags = ((KVCR_CACHE_FP8_K if fp8_k else 0) |
                      (KVCR_CACHE_FUSED_FINALIZE if fused_finalize else 0))
        self.T, self.H, self.D, self.F = tokens_per_frame, heads, head_dim, chunk_frames
        self.rope = rope
        self.dtype_code = _dtype_code(dtype)
        self.storage = None
        if not bookkeeping_only:
            import torch
            nbytes = kv_cache_storage_bytes_ex(sinks, window, aux_frames, tokens_per_frame, heads,
                                               head_dim, chunk_frames, rope is not None,
                                               self.dtype_code, self.flags)
            if nbytes == 0:
                raise KvcrError(KVCR_ESHAPE, "invalid cache sizes")
            self.storage = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.handle = kv_cache_init_ex(sinks, window, aux_frames, tokens_per_frame, heads,
                                       head_dim, chunk_frames, rope, self.dtype_code, self.flags,
                                       self.storage)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            kv_cache_destroy(h)
            self.handle = None

    @property
    def torch_dtype(self):
        import torch
        return torch.bfloat16 if self.dtype_code == KVCR_BF16 else torch.float32

    def append(self, k, v, frames: Sequence[int], stream=None) -> Tuple[List[int], List[int]]:
        kv_cache_append_rope(self.handle, k, v, frames, stream)
        return kv_cache_last_append(self.handle, len(frames))

    def evict(self, keep_recent: int) -> List[int]:
        return kv_cache_evict(self.handle, keep_recent)

    def set_aux(self, k, v, positions: Optional[Sequence[int]] = None, stream=None) -> None:
        """Auxiliary frames for the current chunk (dropped by the next append); k, v
        [n * T, H, D] (None, None on a bookkeeping-only cache with n = len(positions))."""
        if k is not None:
            if k.shape != v.shape or k.shape[0] % self.T or tuple(k.shape[1:]) != (self.H, self.D):
                raise ValueError(f"aux k, v must both be [n * {self.T}, {self.H}, {self.D}]")
            n = k.shape[0] // self.T
            if positions is not None and len(positions) != n:
                raise ValueError("one position per auxiliary frame")
        else:
            n = 0 if positions is None else len(positions)
        kv_cache_set_aux(self.handle, k, v, positions, n, stream)

    def num_aux(self) -> int:
        return kv_cache_num_aux(self.handle)

    def export_state(self) -> bytes:
        """Host state for a checkpoint (save it with a copy of ``self.storage``)."""
        return kv_cache_export_state(self.handle)

    def import_state(self, state: bytes) -> None:
        kv_cache_import_state(self.handle, state)

    def slot_map(self) -> List[int]:
        return kv_cache_slot_map(self.handle, self.sinks + self.window)

    def num_cached(self) -> int:
        return kv_cache_num_cached(self.handle)

    def slot_tensors(self, slot: int):
        """Views (torch) of one slot's K and V, [T, H, D] in the cache dtype."""
        import torch
        kp, vp = kv_cache_slot_data(self.handle, slot)
        esize = 2 if self.dtype_code == KVCR_BF16 else 4
        n = self.T * self.H * self.D
        base = self.storage.data_ptr()
        flat = self.storage.view(self.torch_dtype) if self.storage.numel() % esize == 0 else None
        k = flat[(kp - base) // esize:(kp - base) // esize + n].view(self.T, self.H, self.D)
        v = flat[(vp - base) // esize:(vp - base) // esize + n].view(self.T, self.H, self.D)
        return k, v

    def attention(self, q, k_cur, v_cur, frames: Sequence[int], want_lse: bool = False,
                  out=None, softmax_scale: float = 0.0, stream=None, fp8: bool = False):
        """Chunk attention (``fp8``: the e4m3 QK^T variant, cache made with fp8_k)."""
        import torch
        o = out if out is not None else torch.empty_like(q)
        lse = None
        if want_lse:
            lse = torch.empty((self.H, q.shape[0]), dtype=torch.float32, device=q.device)
        fn = chunk_attention_fwd_fp8 if fp8 else chunk_attention_fwd
        fn(self.handle, q, k_cur, v_cur, frames, o, lse, softmax_scale, stream)
        return o, lse

    def attention_finalize(self, q, k_cur, v_cur, frames: Sequence[int], want_lse: bool = False,
                           out=None, softmax_scale: float = 0.0, stream=None):
        """The chunk's last step: attention, then k_cur, v_cur appended (one pass; cache
        made with fused_finalize).  Returns (o, lse); the append's slots and evictions are
        read with kv_cache_last_append."""
        import torch
        o = out if out is not None else torch.empty_like(q)
        lse = None
        if want_lse:
            lse = torch.empty((self.H, q.shape[0]), dtype=torch.float32, device=q.device)
        chunk_attention_fwd_finalize(self.handle, q, k_cur, v_cur, frames, o, lse, softmax_scale,
                                     stream)
        return o, lse

    def slot_tensors_fp8(self, slot: int):
        """Views (torch) of one slot's e4m3 K codes [T, H, D] (uint8) and block scales
        [ceil(T / 128), H] (fp32)."""
        kp, sp = kv_cache_slot_data_fp8(self.handle, slot)
        base = self.storage.data_ptr()
        n = self.T * self.H * self.D
        nb = (self.T + 127) // 128
        codes = self.storage[kp - base:kp - base + n].view(self.T, self.H, self.D)
        scales = self.storage[sp - base:sp - base + 4 * nb * self.H].view(
            __import__("torch").float32).view(nb, self.H)
        return codes, scales


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
