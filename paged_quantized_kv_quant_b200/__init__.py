"""pkvq: attention over a paged, 8-bit-quantized KV cache on B200 (sm_100a).

Thin Python binding of ``libpkvq.so`` (C ABI declared in include/pkvq.h).
This module only marshals arguments: it checks tensor dtypes/devices/shapes,
passes raw device pointers and the current CUDA stream, and turns status codes
into exceptions.  Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and loading fails loudly when
the library has not been built.

Entry points (same names as the C ABI, without the ``pkvq_`` prefix):
  kv_write_quant, decode_workspace_bytes, paged_attn_decode (with the _ex
  options as keyword arguments: sliding_window, query_pos),
  paged_attn_prefill (sliding_window), merge_attn_states, kv_copy_blocks,
  device_status, status_string, version.  ``dcp`` adds the all-gather step
  of sequence-sharded decode (torch.distributed plumbing).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkvq.so")
LIB_CHECKED_PATH = os.path.join(_HERE, "libpkvq_checked.so")

KV_FP8_E4M3 = 0
KV_INT8 = 1
KV_FP8_E5M2 = 2
KV_FP16 = 3
_FP8_FORMATS = (KV_FP8_E4M3, KV_FP8_E5M2)

EXPORTED = (
    "pkvq_kv_write_quant",
    "pkvq_decode_workspace_bytes",
    "pkvq_paged_attn_decode_append",
    "pkvq_paged_attn_decode",
    "pkvq_paged_attn_decode_ex",
    "pkvq_paged_attn_decode_noalloc",
    "pkvq_paged_attn_prefill",
    "pkvq_paged_attn_prefill_ex",
    "pkvq_merge_attn_states",
    "pkvq_kv_copy_blocks",
    "pkvq_status_string",
    "pkvq_device_status",
    "pkvq_version",
    "pkvq_last_error",
)


def elem_bytes(dtype: int) -> int:
    """Bytes per stored cache element of a format (2 for FP16, else 1)."""
    return 2 if dtype == KV_FP16 else 1


class PkvqError(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = ""
        if status == 6:
            detail = ": " + _lib().pkvq_last_error().decode()
        super().__init__(f"{what}: {status_string(status)} (status {status}){detail}")
        self.status = status


class CacheStruct(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("k_cache", ctypes.c_void_p),
        ("v_cache", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("k_scale_tok", ctypes.c_void_p),
        ("v_scale_tok", ctypes.c_void_p),
        ("scale_per_layer", ctypes.c_int32),
    ]


class AttnOpts(ctypes.Structure):
    _fields_ = [
        ("sliding_window", ctypes.c_int32),
        ("query_pos", ctypes.c_void_p),
    ]


_libs = {}


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads libpkvq.so (or another build of it); raises if it is missing."""
    path = path or os.environ.get("PKVQ_LIBRARY", LIB_PATH)
    if path in _libs:
        return _libs[path]
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} not found: build the CUDA library first "
            "(python -m paged_quantized_kv_quant_b200.build)")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.pkvq_kv_write_quant.restype = I32
    lib.pkvq_kv_write_quant.argtypes = [P, P, P, P, I32, P]
    lib.pkvq_decode_workspace_bytes.restype = SZ
    lib.pkvq_decode_workspace_bytes.argtypes = [I32, I32, I32, I32, P]
    lib.pkvq_paged_attn_decode.restype = I32
    lib.pkvq_paged_attn_decode.argtypes = [P, P, P, P, P, I32, P, I32, I32, I32, I32,
                                           ctypes.c_float, P, SZ, P]
    lib.pkvq_paged_attn_decode_noalloc.restype = I32
    lib.pkvq_paged_attn_decode_noalloc.argtypes = [P, P, P, P, P, I32, P, I32, I32, I32, I32,
                                                   ctypes.c_float, P]
    lib.pkvq_paged_attn_decode_ex.restype = I32
    lib.pkvq_paged_attn_decode_ex.argtypes = [P, P, P, P, P, I32, P, I32, I32, I32, I32,
                                              ctypes.c_float, P, P, SZ, P]
    lib.pkvq_paged_attn_decode_append.restype = I32
    lib.pkvq_paged_attn_decode_append.argtypes = [P, P, P, P, P, P, P, I32, P, I32, I32, I32,
                                                  I32, ctypes.c_float, P, P, SZ, P]
    lib.pkvq_paged_attn_prefill.restype = I32
    lib.pkvq_paged_attn_prefill.argtypes = [P, P, P, P, P, P, I32, P, I32, I32, I32,
                                            ctypes.c_float, P, SZ, P]
    lib.pkvq_paged_attn_prefill_ex.restype = I32
    lib.pkvq_paged_attn_prefill_ex.argtypes = [P, P, P, P, P, P, I32, P, I32, I32, I32,
                                               ctypes.c_float, P, P, SZ, P]
    lib.pkvq_merge_attn_states.restype = I32
    lib.pkvq_merge_attn_states.argtypes = [P, P, I32, ctypes.c_int64, I32, P, P, P]
    lib.pkvq_kv_copy_blocks.restype = I32
    lib.pkvq_kv_copy_blocks.argtypes = [P, P, P, I32, P]
    lib.pkvq_status_string.restype = ctypes.c_char_p
    lib.pkvq_status_string.argtypes = [I32]
    lib.pkvq_device_status.restype = I32
    lib.pkvq_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), I32]
    lib.pkvq_version.restype = ctypes.c_char_p
    lib.pkvq_version.argtypes = []
    lib.pkvq_last_error.restype = ctypes.c_char_p
    lib.pkvq_last_error.argtypes = []
    _libs[path] = lib
    return lib


_current = None


def _lib():
    return _current if _current is not None else load_library()


@contextlib.contextmanager
def use_library(path: str):
    """Routes every call of this module to another build of the library
    (e.g. libpkvq_checked.so, built with PKVQ_BOUNDS_CHECK) inside the block."""
    global _current
    prev, _current = _current, load_library(path)
    try:
        yield _current
    finally:
        _current = prev


def status_string(status: int) -> str:
    return _lib().pkvq_status_string(int(status)).decode()


def version() -> str:
    return _lib().pkvq_version().decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise PkvqError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, dtype, name: str, ndim: Optional[int] = None,
          host_ok: bool = False):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not (t.is_cuda or (host_ok and (t.is_pinned() or t.dim() == 1))):
        raise ValueError(f"{name} must be a CUDA tensor" +
                         (" or pinned host memory" if host_ok else ""))
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


@dataclass
class PagedKVCache:
    """Caller-owned paged cache: elements [num_blocks][Hkv][block_size][D x
    elem_bytes] uint8 (E4M3 / E5M2 bits, int8 two's complement, or fp16 bits),
    fp32 scales for the FP8 formats ([Hkv], or [1] with scale_per_layer),
    per-(block, head, token) fp16 scales for INT8."""
    dtype: int
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    k_scale: Optional[torch.Tensor] = None
    v_scale: Optional[torch.Tensor] = None
    k_scale_tok: Optional[torch.Tensor] = None
    v_scale_tok: Optional[torch.Tensor] = None
    scale_per_layer: bool = False

    @staticmethod
    def allocate(dtype: int, num_blocks: int, block_size: int, num_kv_heads: int,
                 head_dim: int = 128, device="cuda", k_scale=None, v_scale=None,
                 scale_per_layer: bool = False, pin_host: bool = False):
        """Zeroed cache on `device`; with device="cpu" and pin_host=True, in
        pinned host memory the GPU can address (a host tier for kv_copy_blocks)."""
        shape = (num_blocks, num_kv_heads, block_size, head_dim * elem_bytes(dtype))

        def zeros(shp, dt):
            t = torch.zeros(shp, dtype=dt, device=device)
            return t.pin_memory() if pin_host else t
        kc, vc = zeros(shape, torch.uint8), zeros(shape, torch.uint8)
        if dtype in _FP8_FORMATS:
            n = 1 if scale_per_layer else num_kv_heads
            ks = torch.as_tensor(k_scale, dtype=torch.float32).reshape(-1)[:n].to(device)
            vs = torch.as_tensor(v_scale, dtype=torch.float32).reshape(-1)[:n].to(device)
            if ks.numel() != n or vs.numel() != n:
                raise ValueError(f"need {n} K and V scales")
            return PagedKVCache(dtype, kc, vc, k_scale=ks.contiguous(), v_scale=vs.contiguous(),
                                scale_per_layer=scale_per_layer)
        if dtype == KV_FP16:
            return PagedKVCache(dtype, kc, vc)
        kst, vst = zeros(shape[:3], torch.float16), zeros(shape[:3], torch.float16)
        return PagedKVCache(dtype, kc, vc, k_scale_tok=kst, v_scale_tok=vst)

    @property
    def num_blocks(self):
        return self.k_cache.shape[0]

    @property
    def num_kv_heads(self):
        return self.k_cache.shape[1]

    @property
    def block_size(self):
        return self.k_cache.shape[2]

    @property
    def head_dim(self):
        return self.k_cache.shape[3] // elem_bytes(self.dtype)

    def struct(self, device_ok: bool = False) -> CacheStruct:
        for name in ("k_cache", "v_cache"):
            _need(getattr(self, name), torch.uint8, name, 4, host_ok=device_ok)
        if self.dtype in _FP8_FORMATS:
            # (a block copy reads no scale: a host tier may keep its own copy)
            _need(self.k_scale, torch.float32, "k_scale", 1, host_ok=device_ok)
            _need(self.v_scale, torch.float32, "v_scale", 1, host_ok=device_ok)
        elif self.dtype == KV_INT8:
            _need(self.k_scale_tok, torch.float16, "k_scale_tok", 3, host_ok=device_ok)
            _need(self.v_scale_tok, torch.float16, "v_scale_tok", 3, host_ok=device_ok)
        nb, hkv, bs, rb = self.k_cache.shape
        return CacheStruct(self.dtype, nb, bs, hkv, rb // elem_bytes(self.dtype),
                           self.k_cache.data_ptr(), self.v_cache.data_ptr(),
                           self.k_scale.data_ptr() if self.k_scale is not None else None,
                           self.v_scale.data_ptr() if self.v_scale is not None else None,
                           self.k_scale_tok.data_ptr() if self.k_scale_tok is not None else None,
                           self.v_scale_tok.data_ptr() if self.v_scale_tok is not None else None,
                           1 if self.scale_per_layer else 0)


def kv_write_quant(cache: PagedKVCache, k: torch.Tensor, v: torch.Tensor,
                   slot_mapping: torch.Tensor, stream=None) -> None:
    """Quantizes fp16 K/V [T][Hkv][D] into the cache slots (negative = skip)."""
    _need(k, torch.float16, "k", 3)
    _need(v, torch.float16, "v", 3)
    _need(slot_mapping, torch.int32, "slot_mapping", 1)
    cs = cache.struct()
    _check(_lib().pkvq_kv_write_quant(ctypes.byref(cs), _ptr(k), _ptr(v), _ptr(slot_mapping),
                                      int(slot_mapping.shape[0]), _stream(stream)),
           "kv_write_quant")


def decode_workspace_bytes(cache: PagedKVCache, batch: int, q_len: int, num_q_heads: int,
                           max_context_len: int) -> int:
    cs = cache.struct()
    return int(_lib().pkvq_decode_workspace_bytes(batch, q_len, num_q_heads, max_context_len,
                                                  ctypes.byref(cs)))


def _opts(sliding_window: int, query_pos: Optional[torch.Tensor]):
    if not sliding_window and query_pos is None:
        return None
    return AttnOpts(int(sliding_window), None if query_pos is None else query_pos.data_ptr())


def paged_attn_decode(cache: PagedKVCache, q: torch.Tensor, block_table: torch.Tensor,
                      context_lens: torch.Tensor, max_context_len: int, softmax_scale: float,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None,
                      sliding_window: int = 0,
                      query_pos: Optional[torch.Tensor] = None) -> torch.Tensor:
    """q fp16 [B][q_len][Hq][D] -> out fp16 [B][q_len][Hq][D] (lse fp32 [B][q_len][Hq]).
    sliding_window > 0 limits every query to its last `sliding_window` keys;
    query_pos (int32 [B][q_len]) gives each query's position among the keys."""
    _need(q, torch.float16, "q", 4)
    _need(block_table, torch.int32, "block_table", 2)
    _need(context_lens, torch.int32, "context_lens", 1)
    B, q_len, Hq, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.float16, "out", 4)
    if lse is not None:
        _need(lse, torch.float32, "lse", 3)
    if query_pos is not None:
        _need(query_pos, torch.int32, "query_pos", 2)
        if tuple(query_pos.shape) != (B, q_len):
            raise ValueError("query_pos must be [batch][q_len]")
    need = decode_workspace_bytes(cache, B, q_len, Hq, max_context_len) if B else 0
    if workspace is None and need:   # contents need not be initialised
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    cs = cache.struct()
    opts = _opts(sliding_window, query_pos)
    _check(_lib().pkvq_paged_attn_decode_ex(
        ctypes.byref(cs), _ptr(q), _ptr(out), _ptr(lse), _ptr(block_table),
        int(block_table.shape[1]), _ptr(context_lens), B, q_len, Hq, int(max_context_len),
        float(softmax_scale), None if opts is None else ctypes.byref(opts), _ptr(workspace),
        wbytes, _stream(stream)), "paged_attn_decode")
    return out


def paged_attn_decode_append(cache: PagedKVCache, k_new: torch.Tensor, v_new: torch.Tensor,
                             q: torch.Tensor, block_table: torch.Tensor,
                             context_lens: torch.Tensor, max_context_len: int,
                             softmax_scale: float, out: Optional[torch.Tensor] = None,
                             lse: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None, stream=None,
                             sliding_window: int = 0) -> torch.Tensor:
    """One decode step with its KV write: k_new / v_new fp16 [B][q_len][Hkv][D]
    are the keys and values of each sequence's last q_len positions; they are
    quantised into the cache (as kv_write_quant) and attention runs as
    paged_attn_decode."""
    _need(q, torch.float16, "q", 4)
    _need(k_new, torch.float16, "k_new", 4)
    _need(v_new, torch.float16, "v_new", 4)
    _need(block_table, torch.int32, "block_table", 2)
    _need(context_lens, torch.int32, "context_lens", 1)
    B, q_len, Hq, D = q.shape
    if tuple(k_new.shape) != (B, q_len, cache.num_kv_heads, D) or k_new.shape != v_new.shape:
        raise ValueError("k_new / v_new must be [batch][q_len][num_kv_heads][head_dim]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.float16, "out", 4)
    if lse is not None:
        _need(lse, torch.float32, "lse", 3)
    need = decode_workspace_bytes(cache, B, q_len, Hq, max_context_len) if B else 0
    if workspace is None and need:   # contents need not be initialised
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    cs = cache.struct()
    opts = _opts(sliding_window, None)
    _check(_lib().pkvq_paged_attn_decode_append(
        ctypes.byref(cs), _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(out), _ptr(lse),
        _ptr(block_table), int(block_table.shape[1]), _ptr(context_lens), B, q_len, Hq,
        int(max_context_len), float(softmax_scale), None if opts is None else ctypes.byref(opts),
        _ptr(workspace), wbytes, _stream(stream)), "paged_attn_decode_append")
    return out


def paged_attn_prefill(cache: PagedKVCache, q: torch.Tensor, cu_seqlens_q: torch.Tensor,
                       block_table: torch.Tensor, context_lens: torch.Tensor, max_q_len: int,
                       softmax_scale: float, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, stream=None,
                       sliding_window: int = 0) -> torch.Tensor:
    """q fp16 [total_q][Hq][D] (packed varlen) -> out fp16 [total_q][Hq][D]."""
    _need(q, torch.float16, "q", 3)
    _need(cu_seqlens_q, torch.int32, "cu_seqlens_q", 1)
    _need(block_table, torch.int32, "block_table", 2)
    _need(context_lens, torch.int32, "context_lens", 1)
    total_q, Hq, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.float16, "out", 3)
    if lse is not None:
        _need(lse, torch.float32, "lse", 2)
    B = int(context_lens.shape[0])
    cs = cache.struct()
    opts = _opts(sliding_window, None)
    _check(_lib().pkvq_paged_attn_prefill_ex(
        ctypes.byref(cs), _ptr(q), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q), _ptr(block_table),
        int(block_table.shape[1]), _ptr(context_lens), B, int(max_q_len), Hq,
        float(softmax_scale), None if opts is None else ctypes.byref(opts), None, 0,
        _stream(stream)), "paged_attn_prefill")
    return out


def merge_attn_states(parts_out: torch.Tensor, parts_lse: torch.Tensor,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      stream=None):
    """parts_out fp16 [R][..., D], parts_lse fp32 [R][...] (results of the same
    queries over disjoint key sets) -> (out fp16 [..., D], lse fp32 [...])."""
    _need(parts_out, torch.float16, "parts_out")
    _need(parts_lse, torch.float32, "parts_lse")
    R, D = int(parts_out.shape[0]), int(parts_out.shape[-1])
    if tuple(parts_lse.shape) != tuple(parts_out.shape[:-1]):
        raise ValueError("parts_lse must match parts_out without its last dimension")
    n = parts_lse.numel() // max(R, 1)
    if out is None:
        out = torch.empty(parts_out.shape[1:], dtype=torch.float16, device=parts_out.device)
    if lse is None:
        lse = torch.empty(parts_lse.shape[1:], dtype=torch.float32, device=parts_out.device)
    _need(out, torch.float16, "out")
    _need(lse, torch.float32, "lse")
    _check(_lib().pkvq_merge_attn_states(_ptr(parts_out), _ptr(parts_lse), R, n, D, _ptr(out),
                                         _ptr(lse), _stream(stream)), "merge_attn_states")
    return out, lse


def kv_copy_blocks(dst: PagedKVCache, src: PagedKVCache, pairs: torch.Tensor,
                   stream=None) -> None:
    """Block pairs[i][0] of src -> block pairs[i][1] of dst (either cache on the
    GPU or in pinned host memory; pairs int32 [n][2] on the GPU)."""
    _need(pairs, torch.int32, "pairs", 2)
    sd, ss = dst.struct(device_ok=True), src.struct(device_ok=True)
    _check(_lib().pkvq_kv_copy_blocks(ctypes.byref(sd), ctypes.byref(ss), _ptr(pairs),
                                      int(pairs.shape[0]), _stream(stream)), "kv_copy_blocks")


def device_status(clear: bool = True) -> int:
    """Device status word (0 = no device-side check fired); synchronizes."""
    v = ctypes.c_uint32(0)
    _check(_lib().pkvq_device_status(ctypes.byref(v), 1 if clear else 0), "device_status")
    return int(v.value)
