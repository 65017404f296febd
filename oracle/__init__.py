"""CPU oracle for paged 8-bit-KV attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path
(``paged_quantized_kv_quant_b200``) never imports it and shares no code with
it; the two meet only through the seeded input generators in ``synth``.

The arithmetic lives in ``pkvq_oracle.c`` (plain C, FP64, one output row at a
time); this module compiles it with gcc and marshals numpy arrays through
ctypes.  Each wrapped routine names the passage of the pages it follows in the
C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkvq_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")

FP8_E4M3 = 0
INT8 = 1
FP8_E5M2 = 2
FP16 = 3


def elem_bytes(dtype: int) -> int:
    """Bytes per stored cache element of a format."""
    return 2 if dtype == FP16 else 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp32 division, no contraction)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-std=c11", "-Wall", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int, ctypes.c_long, ctypes.c_float
        lib.or_half_to_double.restype = ctypes.c_double
        lib.or_half_to_double.argtypes = [ctypes.c_uint16]
        lib.or_float_to_half_rn.restype = ctypes.c_uint16
        lib.or_float_to_half_rn.argtypes = [f32]
        lib.or_e4m3_decode.restype = ctypes.c_double
        lib.or_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.or_e4m3_encode.restype = ctypes.c_uint8
        lib.or_e4m3_encode.argtypes = [f32]
        for name in ("or_half_to_double_n", "or_float_to_half_rn_n",
                     "or_e4m3_decode_n", "or_e4m3_encode_n",
                     "or_e5m2_decode_n", "or_e5m2_encode_n"):
            getattr(lib, name).restype = None
            getattr(lib, name).argtypes = [P, P, i64]
        lib.or_quant_row_fp8.restype = None
        lib.or_quant_row_fp8.argtypes = [P, i32, f32, P, i32]
        lib.or_quant_row_int8.restype = None
        lib.or_quant_row_int8.argtypes = [P, i32, P, P]
        lib.or_kv_write_quant.restype = None
        lib.or_kv_write_quant.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, i32, P, P,
                                          P, P, P, i32]
        lib.or_copy_blocks.restype = None
        lib.or_copy_blocks.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, i32]
        lib.or_paged_attention.restype = i32
        lib.or_paged_attention.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, i32, P, P,
                                           P, i32, P, P, P, i32, i32, f32, i32, P, P, i32,
                                           P, P, i32]
        lib.or_merge_states.restype = None
        lib.or_merge_states.argtypes = [i32, i64, i32, P, P, P, P]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


# ---------------------------------------------------------------- formats --

def half_to_double(bits) -> np.ndarray:
    """fp16 bit patterns (uint16) -> exact float64 values."""
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    _load().or_half_to_double_n(_ptr(b), _ptr(out), b.size)
    return out


def float_to_half_bits(x) -> np.ndarray:
    """fp32 values -> fp16 bit patterns, round to nearest even."""
    f = _c(x, np.float32)
    out = np.empty(f.shape, np.uint16)
    _load().or_float_to_half_rn_n(_ptr(f), _ptr(out), f.size)
    return out


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 (FN) codes -> float64 values (NaN for S.1111.111)."""
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().or_e4m3_decode_n(_ptr(c), _ptr(out), c.size)
    return out


def e4m3_encode(q) -> np.ndarray:
    """fp32 values -> E4M3 codes: nearest-even, saturating to +-448."""
    f = _c(q, np.float32)
    out = np.empty(f.shape, np.uint8)
    _load().or_e4m3_encode_n(_ptr(f), _ptr(out), f.size)
    return out


def e5m2_decode(codes) -> np.ndarray:
    """E5M2 codes -> float64 values (+-inf for S.11111.00, NaN for S.11111.xx)."""
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().or_e5m2_decode_n(_ptr(c), _ptr(out), c.size)
    return out


def e5m2_encode(q) -> np.ndarray:
    """fp32 values -> E5M2 codes: nearest-even, saturating to +-57344."""
    f = _c(q, np.float32)
    out = np.empty(f.shape, np.uint8)
    _load().or_e5m2_encode_n(_ptr(f), _ptr(out), f.size)
    return out


def quant_row_fp8(x_bits, scale: float, e5m2: bool = False) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    out = np.empty(x.shape, np.uint8)
    _load().or_quant_row_fp8(_ptr(x), x.size, ctypes.c_float(scale), _ptr(out), int(e5m2))
    return out


def code_magnitude(dtype: int, codes: np.ndarray) -> np.ndarray:
    """Codes of |x| for stored codes of x (same array shape and dtype): the
    sign bit cleared for E4M3, E5M2 and FP16, |code| for INT8 (-127..127)."""
    if dtype == INT8:
        return np.abs(codes.view(np.int8)).astype(np.int8).view(np.uint8)
    if dtype == FP16:
        return (codes.view(np.uint16) & np.uint16(0x7FFF)).view(np.uint8).reshape(codes.shape)
    return codes & np.uint8(0x7F)


def quant_row_int8(x_bits):
    """One INT8 row: returns (codes int8[D], scale fp16 bits)."""
    x = _c(x_bits, np.uint16)
    codes = np.empty(x.shape, np.int8)
    s = np.zeros(1, np.uint16)
    _load().or_quant_row_int8(_ptr(x), x.size, _ptr(codes), _ptr(s))
    return codes, int(s[0])


# ------------------------------------------------------------------ cache --

class Cache:
    """Host copy of a paged cache: elements [NB][Hkv][bs][D * elem_bytes] as
    bytes (+ INT8 fp16 scales [NB][Hkv][bs]), plus the fp32 scales of the FP8
    formats: one per KV head, or one for all heads when scale_per_layer."""

    def __init__(self, dtype: int, num_blocks: int, block_size: int, Hkv: int, D: int,
                 k_scale=None, v_scale=None, scale_per_layer: bool = False):
        self.dtype, self.num_blocks, self.block_size = dtype, num_blocks, block_size
        self.Hkv, self.D = Hkv, D
        self.scale_per_layer = bool(scale_per_layer)
        shape = (num_blocks, Hkv, block_size, D * elem_bytes(dtype))
        self.k_cache = np.zeros(shape, np.uint8)
        self.v_cache = np.zeros(shape, np.uint8)
        self.k_scale = self.v_scale = None
        self.k_scale_tok = self.v_scale_tok = None
        if dtype in (FP8_E4M3, FP8_E5M2):
            n = 1 if self.scale_per_layer else Hkv
            self.k_scale = _c(k_scale, np.float32).reshape(-1)[:n].copy()
            self.v_scale = _c(v_scale, np.float32).reshape(-1)[:n].copy()
            assert self.k_scale.size == n and self.v_scale.size == n
        elif dtype == INT8:
            self.k_scale_tok = np.zeros(shape[:3], np.uint16)
            self.v_scale_tok = np.zeros(shape[:3], np.uint16)

    def write(self, k_bits, v_bits, slot_mapping):
        """Quantize fp16 K/V [T][Hkv][D] into the slots (negative = skip)."""
        k = _c(k_bits, np.uint16)
        v = _c(v_bits, np.uint16)
        sm = _c(slot_mapping, np.int32)
        assert k.shape == v.shape and k.shape[1:] == (self.Hkv, self.D)
        assert sm.shape == (k.shape[0],)
        _load().or_kv_write_quant(
            self.dtype, self.num_blocks, self.block_size, self.Hkv, self.D,
            _ptr(self.k_cache), _ptr(self.v_cache), _ptr(self.k_scale),
            _ptr(self.v_scale), int(self.scale_per_layer), _ptr(self.k_scale_tok),
            _ptr(self.v_scale_tok), _ptr(k), _ptr(v), _ptr(sm), int(k.shape[0]))


def copy_blocks(src: Cache, dst: Cache, pairs) -> None:
    """Block pairs[i][0] of src becomes block pairs[i][1] of dst (same geometry)."""
    assert (src.dtype, src.block_size, src.Hkv, src.D) == (dst.dtype, dst.block_size,
                                                            dst.Hkv, dst.D)
    pr = _c(pairs, np.int32).reshape(-1, 2)
    assert np.all(pr[:, 0] >= 0) and np.all(pr[:, 0] < src.num_blocks)
    assert np.all(pr[:, 1] >= 0) and np.all(pr[:, 1] < dst.num_blocks)
    _load().or_copy_blocks(src.dtype, src.block_size, src.Hkv, src.D,
                           _ptr(src.k_cache), _ptr(src.v_cache), _ptr(src.k_scale_tok),
                           _ptr(src.v_scale_tok), _ptr(dst.k_cache), _ptr(dst.v_cache),
                           _ptr(dst.k_scale_tok), _ptr(dst.v_scale_tok), _ptr(pr),
                           int(pr.shape[0]))


def merge_states(outs, lses):
    """Combine per-part attention results over disjoint key sets:
    outs float64 [R][n][D], lses [R][n] -> (out [n][D], lse [n])."""
    o = _c(outs, np.float64)
    l = _c(lses, np.float64)
    R, n, D = o.shape
    assert l.shape == (R, n)
    out = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    _load().or_merge_states(R, n, D, _ptr(o), _ptr(l), _ptr(out), _ptr(lse))
    return out, lse


def paged_attention(cache: Cache, q_bits, cu_seqlens_q, context_lens, block_table,
                    softmax_scale: float, rows=None, nthreads: int = 0, window: int = 0,
                    query_pos=None):
    """Exact (FP64) softmax attention of each query row over its visible keys.

    q_bits: fp16 bits [total_q][Hq][D]; cu_seqlens_q [B+1]; context_lens [B];
    block_table [B][max_blocks]; rows: optional int array [n][2] of
    (token index, head) pairs; window > 0: sliding window of that many keys;
    query_pos: optional int32 [total_q], each query's position (default
    context - q_len + t).
    Returns (out float64, lse float64, threads_used); out is [total_q][Hq][D]
    and lse [total_q][Hq] when rows is None, else [n][D] and [n].
    """
    q = _c(q_bits, np.uint16)
    total_q, Hq, D = q.shape
    assert D == cache.D and Hq % cache.Hkv == 0
    cu = _c(cu_seqlens_q, np.int32)
    ctx = _c(context_lens, np.int32)
    bt = _c(block_table, np.int32)
    B = ctx.shape[0]
    assert cu.shape == (B + 1,) and bt.shape[0] == B and int(cu[-1]) == total_q
    if rows is None:
        n = total_q * Hq
        rr = None
        out = np.empty((total_q, Hq, D), np.float64)
        lse = np.empty((total_q, Hq), np.float64)
    else:
        rr = _c(rows, np.int32).reshape(-1, 2)
        n = rr.shape[0]
        out = np.empty((n, D), np.float64)
        lse = np.empty((n,), np.float64)
    qp = None
    if query_pos is not None:
        qp = _c(query_pos, np.int32).reshape(-1)
        assert qp.shape == (total_q,)
    used = _load().or_paged_attention(
        cache.dtype, cache.num_blocks, cache.block_size, cache.Hkv, D,
        _ptr(cache.k_cache), _ptr(cache.v_cache), _ptr(cache.k_scale),
        _ptr(cache.v_scale), int(cache.scale_per_layer), _ptr(cache.k_scale_tok),
        _ptr(cache.v_scale_tok), _ptr(q), Hq, _ptr(cu), _ptr(ctx), _ptr(bt), int(bt.shape[1]),
        B, ctypes.c_float(softmax_scale), int(window), _ptr(qp), _ptr(rr), n, _ptr(out),
        _ptr(lse), int(nthreads))
    return out, lse, used
