"""pkvq_paged_attn_decode_noalloc: decode for callers that cannot allocate
device memory (an engine whose allocator already owns nearly all of HBM, or a
plugin whose host framework owns every allocation).  Its split-KV scratch is a
fixed array inside the library instead of a caller workspace.

The test calls it through the C ABI twice in a row, on two different shapes
(the second call finds the first call's leftovers in the shared array), and
checks each result against pkvq_paged_attn_decode with a caller-allocated
workspace, within the tolerance the other tests use.  This file is collected
last on purpose.
"""
import ctypes

import pytest
import torch

import paged_quantized_kv_quant_b200 as pk
import synth
from pkvq_testutil import MAX_ABS_TOL, REL_L2_TOL, gpu_cache

pytestmark = pytest.mark.gpu


def _noalloc(cache, q, bt, ctx, max_ctx, scale, out, lse):
    lib = pk.load_library()
    cs = cache.struct()
    B, ql, Hq, _ = q.shape
    return lib.pkvq_paged_attn_decode_noalloc(
        ctypes.byref(cs), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(bt.data_ptr()), int(bt.shape[1]),
        ctypes.c_void_p(ctx.data_ptr()), B, ql, Hq, int(max_ctx), ctypes.c_float(scale),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _compare(a, b):
    a, b = a.double(), b.double()
    assert torch.isfinite(a).all()
    err = float((a - b).abs().max())
    rel = float((a - b).norm() / b.norm())
    assert err <= MAX_ABS_TOL and rel <= REL_L2_TOL, (err, rel)


@pytest.mark.parametrize("order", [0, 1])
def test_noalloc_decode_matches_workspace_decode_twice(order):
    specs = [
        synth.CaseSpec("decode", synth.FP8_E4M3, 32, 4, [8192, 3000, 5000, 17], [1] * 4,
                       seed=40),
        synth.CaseSpec("decode", synth.INT8, 32, 4, [4000, 900], [5, 5], seed=41),
    ]
    if order:
        specs.reverse()
    for spec in specs:              # two calls in a row sharing the library's scratch
        case = synth.make_case(spec)
        cache = gpu_cache(case)
        B, ql = len(spec.context_lens), spec.q_lens[0]
        q = case.q.view(B, ql, spec.num_q_heads, 128).cuda()
        bt, ctx = case.block_table.cuda(), case.context_lens.cuda()
        max_ctx = max(spec.context_lens)
        assert pk.decode_workspace_bytes(cache, B, ql, spec.num_q_heads, max_ctx) > 0
        lse_ref = torch.empty((B, ql, spec.num_q_heads), dtype=torch.float32, device="cuda")
        ref = pk.paged_attn_decode(cache, q, bt, ctx, max_ctx, case.softmax_scale, lse=lse_ref)
        out = torch.full_like(q, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        rc = _noalloc(cache, q, bt, ctx, max_ctx, case.softmax_scale, out, lse)
        assert rc == 0, pk.status_string(rc)
        torch.cuda.synchronize()
        _compare(out, ref)
        assert float((lse - lse_ref).abs().max()) <= 2e-3
    assert pk.device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch(monkeypatch):
    # a split plan with many CTAs per SM needs more than the fixed 8 MiB
    monkeypatch.setenv("PKVQ_DECODE_CTAS_PER_SM", "16")
    spec = synth.CaseSpec("decode", synth.FP8_E4M3, 64, 4, [16384] * 4, [2] * 4, seed=42)
    case = synth.make_case(spec)
    cache = gpu_cache(case)
    q = case.q.view(4, 2, 64, 128).cuda()
    need = pk.decode_workspace_bytes(cache, 4, 2, 64, 16384)
    assert need > (8 << 20)
    out = torch.empty_like(q)
    lse = torch.empty((4, 2, 64), dtype=torch.float32, device="cuda")
    rc = _noalloc(cache, q, case.block_table.cuda(), case.context_lens.cuda(), 16384,
                  case.softmax_scale, out, lse)
    assert rc == 4   # PKVQ_ERR_WORKSPACE_TOO_SMALL, nothing launched
