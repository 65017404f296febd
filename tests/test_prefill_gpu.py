"""GPU parity of pkvq_paged_attn_prefill (causal, chunked over a cached
prefix, varlen batch) against the FP64 oracle."""
import numpy as np
import pytest
import torch

import paged_quantized_kv_quant_b200 as pk
import synth
from pkvq_testutil import assert_matches_oracle, gpu_cache, oracle_cache, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

FP8, INT8 = synth.FP8_E4M3, synth.INT8

CASES = [
    # dtype, Hq, Hkv, ctx list, q_len list, bs
    (FP8, 8, 1, [300], [300], 16),                 # full causal, ragged
    (FP8, 32, 4, [200, 1000], [200, 37], 16),      # one full, one chunk over a prefix
    (FP8, 8, 8, [129, 64], [129, 1], 16),          # MHA; single-token chunk
    (INT8, 16, 2, [555], [555], 32),
    (INT8, 32, 4, [1100, 70], [300, 70], 64),
    (FP8, 4, 2, [1, 2, 3], [1, 2, 3], 16),         # tiny sequences
    (FP8, 12, 2, [260], [130], 16),                # G = 6: 128 % 6 != 0
    (INT8, 32, 4, [2500], [1024], 16),
    (FP8, 16, 2, [700], [300], 64),                # FP8 with 64-token blocks
    (FP8, 8, 2, [96, 1000], [96, 33], 32),         # FP8 with 32-token blocks
]


@pytest.mark.parametrize("outliers", [0.0, 0.01])
@pytest.mark.parametrize("dtype,Hq,Hkv,ctx,ql,bs", CASES)
def test_prefill_matches_oracle(dtype, Hq, Hkv, ctx, ql, bs, outliers):
    spec = synth.CaseSpec("prefill", dtype, Hq, Hkv, list(ctx), list(ql), block_size=bs,
                          seed=31, outlier_frac=outliers)
    case = synth.make_case(spec)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse, what=f"prefill {dtype} {Hq}/{Hkv} {ctx} {ql} bs{bs}")
    assert pk.device_status() == 0


def test_prefill_first_rows_are_exact_value_rows():
    # token 0 sees one key: the output is that key's dequantised V row
    spec = synth.CaseSpec("prefill", FP8, 8, 2, [64], [64], seed=2)
    case = synth.make_case(spec)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, _ = run_gpu(case, cache)
    ref, _ = run_oracle(case, oc)
    # one fp32 rounding of code * v_scale (exact in FP64), then fp16
    assert np.array_equal(out[0].numpy(), ref[0].astype(np.float32).astype(np.float16))


def test_prefill_large_logits_and_max_on_diagonal():
    spec = synth.CaseSpec("prefill", FP8, 8, 2, [700], [700], seed=3)
    case = synth.make_case(spec)
    # every query's own key aligns with it: the maximum sits on the diagonal
    kq = case.q.float().view(700, 2, 4, 128).mean(2)
    case.k = (0.5 * case.k.float() + 2.0 * kq).to(torch.float16)
    case.q.mul_(20.0)
    case.k_scale = synth.per_head_absmax_scale(case.k)
    case.v_scale = synth.per_head_absmax_scale(case.v)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse, what="diagonal max")


def test_prefill_matches_decode_on_the_last_token():
    # the last query of a prefill chunk and a decode step at the same position
    spec = synth.CaseSpec("prefill", INT8, 16, 4, [900], [100], seed=4)
    case = synth.make_case(spec)
    cache = gpu_cache(case)
    out_p, lse_p = run_gpu(case, cache)
    q_last = case.q[-1:].view(1, 1, 16, 128).cuda()
    out_d = pk.paged_attn_decode(cache, q_last, case.block_table.cuda(),
                                 case.context_lens.cuda(), 900, case.softmax_scale)
    torch.cuda.synchronize()
    d = (out_d.view(16, 128).cpu().float() - out_p[-1].float()).abs().max().item()
    assert d <= 2e-3


# ------------------------------------- E5M2, FP16, layer scale, window --

@pytest.mark.parametrize("dtype,Hq,Hkv,ctx,ql,bs,per_layer,window", [
    (synth.FP8_E5M2, 32, 4, [200, 1000], [200, 37], 16, False, 0),
    (synth.FP8_E5M2, 8, 2, [700], [300], 64, True, 0),
    (synth.FP16, 8, 1, [300], [300], 16, False, 0),
    (synth.FP16, 32, 4, [1100, 70], [300, 70], 32, False, 0),
    (synth.FP16, 12, 2, [260], [130], 64, False, 0),
    (FP8, 32, 4, [2500], [1024], 16, True, 0),
    (FP8, 8, 2, [1000], [1000], 16, False, 100),          # window: loop starts late
    (INT8, 32, 4, [3000], [700], 16, False, 257),
    (synth.FP16, 16, 2, [600, 90], [600, 90], 64, False, 64),
    (synth.FP8_E5M2, 8, 8, [129, 64], [129, 1], 32, False, 1),
    (FP8, 32, 4, [5000], [300], 16, False, 4000),         # window longer than the chunk
])
def test_prefill_new_formats_and_window(dtype, Hq, Hkv, ctx, ql, bs, per_layer, window):
    spec = synth.CaseSpec("prefill", dtype, Hq, Hkv, list(ctx), list(ql), block_size=bs,
                          seed=32, outlier_frac=0.01, scale_per_layer=per_layer, window=window)
    case = synth.make_case(spec)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse,
                          what=f"prefill {dtype} {ctx} {ql} bs{bs} L{per_layer} w{window}")
    assert pk.device_status() == 0
