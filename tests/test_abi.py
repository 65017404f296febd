"""Host-side checks of the C-ABI library (CPU only: nothing is launched).

The library must load, export every entry point include/pkvq.h declares, and
reject bad arguments with a status before touching the device.
"""
import ctypes
import os
import re

import pytest

import paged_quantized_kv_quant_b200 as pk
from paged_quantized_kv_quant_b200 import build as pkbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkvq.h")


@pytest.fixture(scope="module")
def lib():
    pkbuild.build()
    return pk.load_library()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkvq_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ("pkvq_kv_write_quant", "pkvq_paged_attn_decode", "pkvq_paged_attn_prefill",
              "pkvq_decode_workspace_bytes", "pkvq_status_string"):
        assert n in names
    assert set(names) == set(pk.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for n in declared_symbols():
        assert hasattr(lib, n), n


def test_only_the_c_abi_is_exported(lib):
    out = os.popen(f"nm -D --defined-only {pk.LIB_PATH}").read()
    ours = sorted({l.split()[-1] for l in out.splitlines() if " T " in l and "pkvq" in l})
    assert ours == sorted(declared_symbols())


def test_status_strings_and_version(lib):
    assert pk.status_string(0) == "ok"
    for s in range(1, 7):
        assert pk.status_string(s) not in ("", "unknown status")
    assert pk.status_string(99) == "unknown status"
    assert re.fullmatch(r"\d+\.\d+\.\d+", pk.version())


def _cache(**kw):
    base = dict(dtype=0, num_blocks=4, block_size=16, num_kv_heads=2, head_dim=128,
                k_cache=0x1000, v_cache=0x2000, k_scale=0x3000, v_scale=0x4000,
                k_scale_tok=None, v_scale_tok=None)
    base.update(kw)
    return pk.CacheStruct(**base)


INVALID, UNSUPPORTED, MISALIGNED = 1, 2, 3


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=64), UNSUPPORTED),
    (dict(block_size=8), UNSUPPORTED),
    (dict(dtype=7), UNSUPPORTED),
    (dict(num_blocks=0), INVALID),
    (dict(k_cache=None), INVALID),
    (dict(k_scale=None), INVALID),
    (dict(dtype=1, k_scale_tok=None, v_scale_tok=None), INVALID),
    (dict(k_cache=0x1008), MISALIGNED),
    (dict(num_blocks=1 << 26, num_kv_heads=8), UNSUPPORTED),
])
def test_kv_write_rejects_bad_cache(lib, kw, status):
    c = _cache(**kw)
    rc = lib.pkvq_kv_write_quant(ctypes.byref(c), ctypes.c_void_p(0x5000),
                                 ctypes.c_void_p(0x6000), ctypes.c_void_p(0x7000), 4, None)
    assert rc == status


def test_kv_write_argument_checks(lib):
    c = _cache()
    P = ctypes.c_void_p
    assert lib.pkvq_kv_write_quant(None, P(16), P(16), P(16), 1, None) == INVALID
    assert lib.pkvq_kv_write_quant(ctypes.byref(c), P(16), P(16), P(16), -1, None) == INVALID
    assert lib.pkvq_kv_write_quant(ctypes.byref(c), None, P(16), P(16), 1, None) == INVALID
    assert lib.pkvq_kv_write_quant(ctypes.byref(c), P(18), P(16), P(16), 1, None) == MISALIGNED
    # zero tokens is a no-op even with null data pointers
    assert lib.pkvq_kv_write_quant(ctypes.byref(c), None, None, None, 0, None) == 0


def _decode(lib, c, **kw):
    a = dict(q=0x10000, out=0x20000, lse=None, bt=0x30000, maxb=64, ctx=0x40000, B=2, ql=1,
             Hq=8, maxctx=1024, scale=0.088, ws=None, wsb=0)
    a.update(kw)
    P = ctypes.c_void_p
    return lib.pkvq_paged_attn_decode(ctypes.byref(c), P(a["q"]), P(a["out"]), P(a["lse"]),
                                      P(a["bt"]), a["maxb"], P(a["ctx"]), a["B"], a["ql"],
                                      a["Hq"], a["maxctx"], ctypes.c_float(a["scale"]),
                                      P(a["ws"]), a["wsb"], None)


def test_decode_argument_checks(lib):
    c = _cache()
    assert _decode(lib, c, ql=0) == INVALID
    assert _decode(lib, c, ql=17) == INVALID
    assert _decode(lib, c, Hq=7) == INVALID                   # not a multiple of Hkv
    assert _decode(lib, c, Hq=2 * 17) == UNSUPPORTED          # group 17 > 16
    assert _decode(lib, c, scale=float("nan")) == INVALID
    assert _decode(lib, c, q=None) == INVALID
    assert _decode(lib, c, q=0x10008) == MISALIGNED
    assert _decode(lib, c, maxb=4) == INVALID                 # 4 * 16 < max context
    assert _decode(lib, c, B=0) == 0                          # empty batch: no-op
    assert _decode(lib, _cache(head_dim=96)) == UNSUPPORTED


def test_workspace_query_rejects_bad_shapes(lib):
    c = _cache()
    assert lib.pkvq_decode_workspace_bytes(0, 1, 8, 1024, ctypes.byref(c)) == 0
    assert lib.pkvq_decode_workspace_bytes(2, 1, 7, 1024, ctypes.byref(c)) == 0
    assert lib.pkvq_decode_workspace_bytes(2, 1, 8, 1024, None) == 0


def test_prefill_argument_checks(lib):
    c = _cache()
    P = ctypes.c_void_p

    def call(**kw):
        a = dict(q=0x10000, out=0x20000, cu=0x30000, bt=0x40000, ctx=0x50000, B=1, mq=16, Hq=8,
                 scale=0.088)
        a.update(kw)
        return lib.pkvq_paged_attn_prefill(ctypes.byref(c), P(a["q"]), P(a["out"]), None,
                                           P(a["cu"]), P(a["bt"]), 64, P(a["ctx"]), a["B"],
                                           a["mq"], a["Hq"], ctypes.c_float(a["scale"]), None,
                                           0, None)
    assert call(Hq=9) == INVALID
    assert call(cu=None) == INVALID
    assert call(out=0x20004) == MISALIGNED
    assert call(scale=float("inf")) == INVALID
    assert call(mq=0) == 0
    assert call(B=0) == 0


def test_device_status_rejects_null(lib):
    assert lib.pkvq_device_status(None, 0) == INVALID


# ---- decode plan: routing and workspace size (host only; on a machine
# without a GPU the library assumes 148 SMs) ----

def _ws(lib, batch, q_len, hq, hkv, max_ctx):
    c = _cache(num_kv_heads=hkv)
    return lib.pkvq_decode_workspace_bytes(batch, q_len, hq, max_ctx, ctypes.byref(c))


def test_verify_rows_take_the_tensor_core_plan(lib, monkeypatch):
    # 5 tokens x G = 8 -> 40 rows per KV head (17..128): one CTA for all rows,
    # one CTA per SM, C = max(B, SMs / Hkv) slots per KV head
    monkeypatch.delenv("PKVQ_DECODE_CTAS_PER_SM", raising=False)
    sms, hkv, rows, batch = 148, 4, 40, 6
    C = max(batch, sms // hkv)
    assert _ws(lib, batch, 5, 32, hkv, 524288) == hkv * C * rows * (128 + 2) * 4


def test_row_counts_past_one_tile_use_row_groups(lib, monkeypatch):
    # 16 tokens x G = 16 = 256 rows: past 128, the mma.sync kernel in groups of
    # 16 rows; the workspace holds one 16-row partial per slot and row group
    monkeypatch.setenv("PKVQ_DECODE_CTAS_PER_SM", "2")
    sms, hkv, batch = 148, 2, 1
    groups = 256 // 16
    units = hkv * groups
    C = max(batch, 2 * sms // units)
    assert _ws(lib, batch, 16, 32, hkv, 65536) == units * C * 16 * (128 + 2) * 4


def test_one_slot_per_sequence_needs_no_workspace(lib, monkeypatch):
    # more sequences than the GPU has slots for: every sequence is one split
    monkeypatch.setenv("PKVQ_DECODE_CTAS_PER_SM", "1")
    assert _ws(lib, 4096, 1, 32, 4, 32768) == 0


# ---- the entry points added for the next rows (host-side checks only) ----

def test_decode_ex_and_prefill_ex_option_checks(lib):
    c = _cache()
    P = ctypes.c_void_p
    bad = pk.AttnOpts(-1, None)
    rc = lib.pkvq_paged_attn_decode_ex(ctypes.byref(c), P(0x10000), P(0x20000), None,
                                       P(0x30000), 64, P(0x40000), 2, 1, 8, 1024,
                                       ctypes.c_float(0.088), ctypes.byref(bad), None, 0, None)
    assert rc == INVALID
    qp = pk.AttnOpts(0, 0x50000)
    rc = lib.pkvq_paged_attn_prefill_ex(ctypes.byref(c), P(0x10000), P(0x20000), None,
                                        P(0x30000), P(0x40000), 64, P(0x50000), 1, 16, 8,
                                        ctypes.c_float(0.088), ctypes.byref(qp), None, 0, None)
    assert rc == UNSUPPORTED        # query positions are a decode option
    # a zeroed options struct is the plain call: batch 0 is still a no-op
    z = pk.AttnOpts(0, None)
    rc = lib.pkvq_paged_attn_decode_ex(ctypes.byref(c), P(0x10000), P(0x20000), None,
                                       P(0x30000), 64, P(0x40000), 0, 1, 8, 1024,
                                       ctypes.c_float(0.088), ctypes.byref(z), None, 0, None)
    assert rc == 0


def test_new_formats_are_accepted_and_checked(lib):
    # E5M2 needs its fp32 scales like E4M3; FP16 needs none
    assert lib.pkvq_kv_write_quant(ctypes.byref(_cache(dtype=2, k_scale=None)),
                                   ctypes.c_void_p(16), ctypes.c_void_p(16),
                                   ctypes.c_void_p(16), 1, None) == INVALID
    assert lib.pkvq_decode_workspace_bytes(2, 1, 8, 4096,
                                           ctypes.byref(_cache(dtype=3, k_scale=None,
                                                               v_scale=None))) > 0
    assert lib.pkvq_decode_workspace_bytes(2, 1, 8, 4096, ctypes.byref(_cache(dtype=2))) > 0


def test_merge_argument_checks(lib):
    P = ctypes.c_void_p
    m = lambda **kw: lib.pkvq_merge_attn_states(
        P(kw.get("po", 0x1000)), P(kw.get("pl", 0x2000)), kw.get("R", 2), kw.get("n", 4),
        kw.get("D", 128), P(kw.get("out", 0x3000)), None, None)
    assert m(D=64) == UNSUPPORTED
    assert m(R=0) == INVALID and m(R=65) == INVALID and m(n=-1) == INVALID
    assert m(po=None) == INVALID and m(out=None) == INVALID
    assert m(out=0x3008) == MISALIGNED
    assert m(n=0, po=None) == 0     # no rows: no-op


def test_copy_blocks_argument_checks(lib):
    P = ctypes.c_void_p
    a, b = _cache(), _cache(num_blocks=9)
    assert lib.pkvq_kv_copy_blocks(ctypes.byref(a), ctypes.byref(b), P(0x5000), -1, None) == INVALID
    assert lib.pkvq_kv_copy_blocks(ctypes.byref(a), ctypes.byref(b), None, 3, None) == INVALID
    assert lib.pkvq_kv_copy_blocks(ctypes.byref(a), ctypes.byref(b), None, 0, None) == 0
    for kw in (dict(block_size=32), dict(num_kv_heads=4), dict(dtype=1, k_scale_tok=0x7000,
                                                               v_scale_tok=0x8000)):
        assert lib.pkvq_kv_copy_blocks(ctypes.byref(a), ctypes.byref(_cache(**kw)), P(0x5000),
                                       1, None) == INVALID
