"""GPU parity of pkvq_paged_attn_decode_append (a decode step that first
writes its new tokens into the cache): the cache afterwards is bit-identical
to pkvq_kv_write_quant of the same tokens, the outputs bit-identical to
pkvq_paged_attn_decode after that write, and within the derived bound of the
oracle."""
import numpy as np
import pytest
import torch

import paged_quantized_kv_quant_b200 as pk
import synth
from pkvq_testutil import (assert_matches_oracle, bits16, gpu_cache, oracle_cache, run_gpu,
                           run_oracle)

pytestmark = pytest.mark.gpu

FP8, INT8, E5M2, FP16 = synth.FP8_E4M3, synth.INT8, synth.FP8_E5M2, synth.FP16

CASES = [
    # dtype, Hq, Hkv, ctx list, q_len, bs, window
    (FP8, 32, 4, [777, 16, 1, 2049], 1, 16, 0),        # split kernel, one split per CTA
    (FP8, 32, 4, [16384, 300, 5000], 1, 16, 0),        # many splits: the last one writes
    (INT8, 8, 2, [300, 6, 2], 2, 32, 0),               # new tokens across a block edge
    (INT8, 16, 4, [64, 65, 33], 3, 16, 0),             # 12 rows
    (E5M2, 16, 2, [513, 4000], 1, 64, 0),
    (FP16, 32, 4, [4000, 5], 1, 16, 0),
    (FP8, 8, 2, [3000, 100, 17], 1, 16, 500),          # sliding window
    (INT8, 32, 4, [999, 17, 5], 5, 16, 0),             # 40 rows: KV write kernel, then tcgen05
    (FP8, 16, 2, [900, 2], 3, 32, 0),                  # 24 rows, q_len > one context
]


def _new_tokens(case):
    """k_new / v_new [B][q_len][Hkv][D] (zeros for positions below 0) and the
    rows of case.k written before the step (all others)."""
    s = case.spec
    B, ql = len(s.context_lens), s.q_lens[0]
    kn = torch.zeros(B, ql, s.num_kv_heads, s.head_dim, dtype=torch.float16)
    vn = torch.zeros_like(kn)
    old = torch.ones(case.k.shape[0], dtype=torch.bool)
    for b, c in enumerate(s.context_lens):
        base = int(case.token_offsets[b])
        for t in range(ql):
            pos = c - ql + t
            if pos >= 0:
                kn[b, t] = case.k[base + pos]
                vn[b, t] = case.v[base + pos]
                old[base + pos] = False
    return kn, vn, old


@pytest.mark.parametrize("dtype,Hq,Hkv,ctx,ql,bs,window", CASES)
def test_decode_append_matches_write_then_decode(dtype, Hq, Hkv, ctx, ql, bs, window):
    spec = synth.CaseSpec("decode", dtype, Hq, Hkv, list(ctx), [ql] * len(ctx), block_size=bs,
                          seed=31, window=window, outlier_frac=0.01)
    case = synth.make_case(spec)
    ref_cache = gpu_cache(case)                       # every token by kv_write_quant
    out_ref, lse_ref = run_gpu(case, ref_cache)
    kn, vn, old = _new_tokens(case)
    cache = gpu_cache(case, write=False)              # the same NaN-poisoned pool
    if old.any():
        pk.kv_write_quant(cache, case.k[old].cuda(), case.v[old].cuda(),
                          case.slot_mapping[old].cuda())
    B = len(ctx)
    q = case.q.view(B, ql, Hq, 128).cuda()
    lse = torch.empty((B, ql, Hq), dtype=torch.float32, device="cuda")
    out = pk.paged_attn_decode_append(cache, kn.cuda(), vn.cuda(), q, case.block_table.cuda(),
                                      case.context_lens.cuda(), max(ctx), case.softmax_scale,
                                      lse=lse, sliding_window=window)
    torch.cuda.synchronize()
    for name in ("k_cache", "v_cache", "k_scale_tok", "v_scale_tok"):
        a, r = getattr(cache, name), getattr(ref_cache, name)
        if a is None:
            continue
        assert torch.equal(a.view(torch.uint8), r.view(torch.uint8)), f"{name} differs"
    out = out.view(-1, Hq, 128).cpu()
    assert torch.equal(out, out_ref)
    assert torch.equal(lse.view(-1, Hq).cpu(), lse_ref)
    oc = oracle_cache(case)
    ref, ref_l = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse.view(-1, Hq).cpu(), ref, ref_l,
                          what=f"append {dtype} {ctx} q{ql} bs{bs} w{window}")
    assert pk.device_status() == 0


def test_decode_append_rejects_query_positions():
    spec = synth.CaseSpec("decode", FP8, 8, 2, [100], [1], seed=1)
    case = synth.make_case(spec)
    cache = gpu_cache(case)
    q = case.q.view(1, 1, 8, 128).cuda()
    kn = torch.zeros(1, 1, 2, 128, dtype=torch.float16, device="cuda")
    bt, cl = case.block_table.cuda(), case.context_lens.cuda()
    qp = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    opts = pk._opts(0, qp)
    import ctypes
    cs = cache.struct()
    out = torch.empty_like(q)
    st = pk._lib().pkvq_paged_attn_decode_append(
        ctypes.byref(cs), kn.data_ptr(), kn.data_ptr(), q.data_ptr(), out.data_ptr(), None,
        bt.data_ptr(), bt.shape[1], cl.data_ptr(), 1, 1, 8, 100, 0.1, ctypes.byref(opts),
        None, 0, None)
    assert st != 0
