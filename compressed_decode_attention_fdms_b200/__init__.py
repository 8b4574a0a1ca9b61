"""Python binding of the compact-KV decode-attention library (``include/fdms.h``).

Argument marshalling only: every step of the path runs in the CUDA library
``libfdms.so`` built next to this file (``build.py``). Torch supplies device
memory and streams. There is no fallback: if the library is missing, importing
a function raises.

The functions keep the C names. Tensors are checked for device, dtype, shape
and contiguity, then passed as raw pointers; the stream defaults to torch's
current stream on the cache's device.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfdms.so")

FDMS_OK, FDMS_ERR_INVALID_ARG, FDMS_ERR_OUT_OF_BLOCKS, FDMS_ERR_CUDA, \
    FDMS_ERR_UNSUPPORTED, FDMS_ERR_DEVICE = range(6)
FDMS_KV_BF16, FDMS_KV_FP8_E4M3, FDMS_KV_FP8_E4M3_BLOCK = 0, 1, 2

# every symbol include/fdms.h declares
EXPORTED = (
    "fdms_status_string", "fdms_cache_create", "fdms_cache_destroy", "fdms_append_evict",
    "fdms_decode_attn", "fdms_decode_attn_f32", "fdms_cache_stats", "fdms_cache_read_head",
    "fdms_decode_attn_noalloc", "fdms_decode_layout",
)


class FdmsError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class fdms_config(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int), ("max_batch", ctypes.c_int),
        ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("window", ctypes.c_int),
        ("compact_period", ctypes.c_int), ("max_seq_len", ctypes.c_int),
        ("num_blocks", ctypes.c_longlong), ("kv_dtype", ctypes.c_int),
        ("softmax_scale", ctypes.c_float), ("decode_ctas", ctypes.c_int),
    ]


class fdms_stats(ctypes.Structure):
    _fields_ = [
        ("tokens_appended", ctypes.c_longlong), ("slots_store", ctypes.c_longlong),
        ("slots_ring", ctypes.c_longlong), ("blocks_used", ctypes.c_longlong),
        ("blocks_free", ctypes.c_longlong), ("bytes_compact", ctypes.c_longlong),
        ("bytes_dense_equiv", ctypes.c_longlong), ("bytes_reserved", ctypes.c_longlong),
        ("fp8_saturations", ctypes.c_longlong), ("slots_decoded", ctypes.c_longlong),
        ("decode_calls", ctypes.c_longlong), ("bytes_decoded", ctypes.c_longlong),
        ("error", ctypes.c_int),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class fdms_head_info(ctypes.Structure):
    _fields_ = [("num_tokens", ctypes.c_int), ("resolved", ctypes.c_int),
                ("store_len", ctypes.c_int), ("ring_len", ctypes.c_int)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfdms.so (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"CUDA library not built: {path} (run __graft_entry__.build() or "
                          "python -m compressed_decode_attention_fdms_b200.build)")
    lib = ctypes.CDLL(path)
    P, I, LL, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
    lib.fdms_status_string.restype = ctypes.c_char_p
    lib.fdms_status_string.argtypes = [I]
    lib.fdms_cache_create.restype = I
    lib.fdms_cache_create.argtypes = [ctypes.POINTER(fdms_config), I, P, ctypes.POINTER(P)]
    lib.fdms_cache_destroy.restype = I
    lib.fdms_cache_destroy.argtypes = [P]
    lib.fdms_append_evict.restype = I
    lib.fdms_append_evict.argtypes = [P, I, I, P, I, P, P, P, P, P]
    lib.fdms_decode_attn.restype = I
    lib.fdms_decode_attn.argtypes = [P, I, I, P, P, P]
    lib.fdms_decode_attn_f32.restype = I
    lib.fdms_decode_attn_f32.argtypes = [P, I, I, P, P, P, P]
    lib.fdms_decode_attn_noalloc.restype = I
    lib.fdms_decode_attn_noalloc.argtypes = [P, I, I, P, P, P]
    lib.fdms_decode_layout.restype = I
    lib.fdms_decode_layout.argtypes = [P, I, ctypes.POINTER(I), ctypes.POINTER(I)]
    lib.fdms_cache_stats.restype = I
    lib.fdms_cache_stats.argtypes = [P, ctypes.POINTER(fdms_stats), P]
    lib.fdms_cache_read_head.restype = I
    lib.fdms_cache_read_head.argtypes = [P, I, I, I, I, P, P, P, P, P,
                                         ctypes.POINTER(fdms_head_info), P]
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().fdms_status_string(status).decode()


fdms_status_string = status_string


def _check(status: int, what: str):
    if status != FDMS_OK:
        raise FdmsError(status, what)


def _stream_ptr(stream, device) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


@dataclass
class Cache:
    """Handle of one fdms_cache plus the shape facts the binding checks against."""
    handle: int
    config: fdms_config
    device: int

    @property
    def elt(self) -> int:
        """Bytes per element of a row fdms_cache_read_head returns (a per-block
        FP8 cache returns 2 D bytes per row: codes, or bf16 for staged rows)."""
        return 1 if self.config.kv_dtype == FDMS_KV_FP8_E4M3 else 2

    def __del__(self):
        # destroy explicitly with fdms_cache_destroy; this is only a safety net
        if getattr(self, "handle", None) and _lib is not None:
            try:
                _lib.fdms_cache_destroy(ctypes.c_void_p(self.handle))
            except Exception:
                pass
            self.handle = None


def make_config(num_layers, max_batch, num_q_heads, num_kv_heads, head_dim, window,
                compact_period=1, max_seq_len=8192, num_blocks=0, kv_dtype="bf16",
                softmax_scale=0.0, decode_ctas=0) -> fdms_config:
    dt = {"bf16": FDMS_KV_BF16, "fp8_e4m3": FDMS_KV_FP8_E4M3,
          "fp8_e4m3_block": FDMS_KV_FP8_E4M3_BLOCK}[kv_dtype] \
        if isinstance(kv_dtype, str) else int(kv_dtype)
    return fdms_config(num_layers, max_batch, num_q_heads, num_kv_heads, head_dim, window,
                       compact_period, max_seq_len, num_blocks, dt, softmax_scale, decode_ctas)


def fdms_cache_create(config: fdms_config, device: int = 0, stream=None) -> Cache:
    lib = load_library()
    h = ctypes.c_void_p()
    _check(lib.fdms_cache_create(ctypes.byref(config), device,
                                 ctypes.c_void_p(_stream_ptr(stream, device)), ctypes.byref(h)),
           "fdms_cache_create")
    return Cache(h.value, config, device)


def fdms_cache_destroy(cache: Cache):
    if cache.handle:
        st = load_library().fdms_cache_destroy(ctypes.c_void_p(cache.handle))
        cache.handle = None
        _check(st, "fdms_cache_destroy")


def _dev_tensor(t, dtype, shape, name, device):
    """Device pointer of a tensor after checking what the C ABI assumes."""
    # every property at once on the common path (this runs on every call of a
    # decode step, several times); the checks below name what failed
    if (isinstance(t, torch.Tensor) and t.dtype is dtype and t.is_cuda and t.shape == shape
            and t.is_contiguous() and t.get_device() == device):
        return t.data_ptr()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda or t.get_device() != device:
        raise ValueError(f"{name}: must live on cuda:{device}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.shape != shape:
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return t.data_ptr()


def fdms_append_evict(cache: Cache, layer: int, batch: int, n_new: torch.Tensor, max_new: int,
                      k: torch.Tensor, v: torch.Tensor, keep: torch.Tensor,
                      kv_scale: Optional[torch.Tensor] = None, stream=None):
    c = cache.config
    H, D, dev = c.num_kv_heads, c.head_dim, cache.device
    kv = (batch, max_new, H, D)
    st = load_library().fdms_append_evict(
        cache.handle, layer, batch, _dev_tensor(n_new, torch.int32, (batch,), "n_new", dev),
        max_new, _dev_tensor(k, torch.bfloat16, kv, "k", dev),
        _dev_tensor(v, torch.bfloat16, kv, "v", dev),
        _dev_tensor(keep, torch.uint8, kv[:3], "keep", dev),
        None if kv_scale is None else
        _dev_tensor(kv_scale, torch.float32, (batch, H, 2), "kv_scale", dev),
        _stream_ptr(stream, dev))
    if st != FDMS_OK:
        raise FdmsError(st, "fdms_append_evict")


def fdms_decode_attn(cache: Cache, layer: int, batch: int, q: torch.Tensor, out: torch.Tensor,
                     stream=None):
    c = cache.config
    shape = (batch, c.num_q_heads, c.head_dim)
    dev = cache.device
    st = load_library().fdms_decode_attn(
        cache.handle, layer, batch, _dev_tensor(q, torch.bfloat16, shape, "q", dev),
        _dev_tensor(out, torch.bfloat16, shape, "out", dev), _stream_ptr(stream, dev))
    if st != FDMS_OK:
        raise FdmsError(st, "fdms_decode_attn")


def fdms_decode_attn_f32(cache: Cache, layer: int, batch: int, q: torch.Tensor,
                         out: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None):
    c = cache.config
    shape = (batch, c.num_q_heads, c.head_dim)
    qp = _dev_tensor(q, torch.bfloat16, shape, "q", cache.device)
    op = _dev_tensor(out, torch.float32, shape, "out", cache.device)
    lp = None if lse is None else _dev_tensor(lse, torch.float32, shape[:2], "lse", cache.device)
    _check(load_library().fdms_decode_attn_f32(
        ctypes.c_void_p(cache.handle), layer, batch, ctypes.c_void_p(qp), ctypes.c_void_p(op),
        ctypes.c_void_p(lp), ctypes.c_void_p(_stream_ptr(stream, cache.device))),
        "fdms_decode_attn_f32")


def fdms_decode_attn_noalloc(cache: Cache, layer: int, batch: int, q: torch.Tensor,
                             out: torch.Tensor, stream=None):
    """fdms_decode_attn with its scratch in the library's fixed array (no allocation)."""
    c = cache.config
    shape = (batch, c.num_q_heads, c.head_dim)
    qp = _dev_tensor(q, torch.bfloat16, shape, "q", cache.device)
    op = _dev_tensor(out, torch.bfloat16, shape, "out", cache.device)
    _check(load_library().fdms_decode_attn_noalloc(
        ctypes.c_void_p(cache.handle), layer, batch, ctypes.c_void_p(qp), ctypes.c_void_p(op),
        ctypes.c_void_p(_stream_ptr(stream, cache.device))), "fdms_decode_attn_noalloc")


def fdms_decode_layout(cache: Cache, batch: int) -> dict:
    """How a decode call of `batch` sequences runs: cluster CTAs per head (0 =
    global plan) and the split grid of the plan."""
    cl, sp = ctypes.c_int(), ctypes.c_int()
    _check(load_library().fdms_decode_layout(ctypes.c_void_p(cache.handle), batch,
                                             ctypes.byref(cl), ctypes.byref(sp)),
           "fdms_decode_layout")
    return {"cluster_ctas": cl.value, "split_ctas": sp.value}


def decode_cluster_size(cache: Cache, batch: int) -> int:
    return fdms_decode_layout(cache, batch)["cluster_ctas"]


def fdms_cache_stats(cache: Cache, stream=None) -> dict:
    st = fdms_stats()
    _check(load_library().fdms_cache_stats(ctypes.c_void_p(cache.handle), ctypes.byref(st),
                                           ctypes.c_void_p(_stream_ptr(stream, cache.device))),
           "fdms_cache_stats")
    return st.as_dict()


def fdms_cache_read_head(cache: Cache, layer: int, seq: int, kv_head: int, stream=None) -> dict:
    """One head's store then ring, in position order (host numpy arrays)."""
    import numpy as np
    lib = load_library()
    info = fdms_head_info()
    sp = ctypes.c_void_p(_stream_ptr(stream, cache.device))
    h = ctypes.c_void_p(cache.handle)
    _check(lib.fdms_cache_read_head(h, layer, seq, kv_head, 0, None, None, None, None, None,
                                    ctypes.byref(info), sp), "fdms_cache_read_head")
    n = info.store_len + info.ring_len
    rb = cache.config.head_dim * cache.elt
    pos = np.zeros(max(n, 1), np.int32)
    keep = np.zeros(max(n, 1), np.uint8)
    kb = np.zeros((max(n, 1), rb), np.uint8)
    vb = np.zeros((max(n, 1), rb), np.uint8)
    sc = np.zeros((max(n, 1), 2), np.float32)
    cp = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib.fdms_cache_read_head(h, layer, seq, kv_head, max(n, 1), cp(pos), cp(keep), cp(kb),
                                    cp(vb), cp(sc), ctypes.byref(info), sp),
           "fdms_cache_read_head")
    return {"num_tokens": info.num_tokens, "resolved": info.resolved,
            "store_len": info.store_len, "ring_len": info.ring_len,
            "pos": pos[:n], "keep": keep[:n], "k": kb[:n], "v": vb[:n], "scale": sc[:n]}
