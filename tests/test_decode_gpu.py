"""GPU parity of pkvq_paged_attn_decode against the FP64 oracle on small and
ragged shapes, covering the numerical bug classes the 1Cat-LLM README lists
for its kernels ("Layer 2": short-chunk causal visibility, missed score
maxima, overflowing score tiles, tail range)."""
import numpy as np
import pytest
import torch

import paged_quantized_kv_quant_b200 as pk
import synth
from pkvq_testutil import (assert_close, assert_codes_equal, assert_matches_oracle, gpu_cache,
                           oracle_cache, run_gpu, run_oracle)

pytestmark = pytest.mark.gpu

FP8, INT8 = synth.FP8_E4M3, synth.INT8

CASES = [
    # dtype, Hq, Hkv, ctx list, q_len, bs
    (FP8, 8, 2, [1024], 1, 16),             # workload 1 shape
    (FP8, 32, 4, [777, 16, 1, 2049], 1, 16),  # ragged tails, one-key context
    (FP8, 4, 4, [100, 35], 1, 16),          # MHA (G = 1)
    (FP8, 16, 1, [513], 1, 32),             # G = 16 -> two row tiles
    (FP8, 8, 4, [300, 129], 1, 64),
    (INT8, 32, 4, [999, 17], 5, 16),        # verify: q_len 5 -> 40 rows, row groups
    (INT8, 8, 2, [5, 6, 300], 5, 16),       # q_len == context: first row sees 1 key
    (INT8, 16, 4, [64, 65], 3, 32),
    (FP8, 8, 1, [4099], 4, 16),             # q_len 4, G 8 -> 32 rows
    (FP8, 32, 4, [16384], 1, 16),           # long: many splits
    (INT8, 8, 2, [20000, 3], 2, 16),
    # splits in proportion to length: one long sequence among very short ones
    (FP8, 8, 2, [65536, 1, 16, 17, 4096, 300], 1, 16),
    (INT8, 16, 2, [3000, 40000, 5], 2, 16),
    # more than 32 sequences: the slot map is scanned in several warp chunks
    (FP8, 8, 2, [(i * 977) % 3001 + 1 for i in range(40)], 1, 16),
    # more than 16 rows per KV head: the tcgen05 kernel, every block size
    (FP8, 16, 2, [1000, 333], 3, 32),       # 24 rows
    (INT8, 8, 1, [2000, 77], 4, 64),        # 32 rows
    (INT8, 16, 2, [3000, 129], 6, 16),      # 48 rows
    (FP8, 32, 4, [2500, 1], 7, 32),         # 56 rows
    (INT8, 16, 2, [1300, 700], 8, 16),      # 64 rows: the last half-lane layout
    (INT8, 16, 2, [1500, 90], 9, 16),       # 72 rows: one thread per row
    (FP8, 9, 1, [700, 33], 2, 16),          # 18 rows (G = 9): near the fewest on tcgen05
    (INT8, 20, 2, [1200, 250], 10, 32),     # 100 rows, two threads' worth of lanes idle
    (FP8, 16, 2, [900], 16, 16),            # 128 rows: one full tile
    (FP8, 32, 2, [500], 16, 16),            # 256 rows: past the tile, mma.sync row groups
]


def _case(dtype, Hq, Hkv, ctx, ql, bs, seed=0, **kw):
    spec = synth.CaseSpec("decode", dtype, Hq, Hkv, list(ctx), [ql] * len(ctx),
                          block_size=bs, seed=seed, **kw)
    return synth.make_case(spec)


@pytest.mark.parametrize("outliers", [0.0, 0.01])
@pytest.mark.parametrize("dtype,Hq,Hkv,ctx,ql,bs", CASES)
def test_decode_matches_oracle(dtype, Hq, Hkv, ctx, ql, bs, outliers):
    case = _case(dtype, Hq, Hkv, ctx, ql, bs, seed=21, outlier_frac=outliers)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    assert_codes_equal(cache, oc, case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse,
                          what=f"decode {dtype} {Hq}/{Hkv} {ctx} q{ql} bs{bs} x8:{outliers}")
    assert pk.device_status() == 0


def test_decode_empty_context_and_q_len_beyond_context():
    # context 0 -> zeros / -inf; q_len 3 over context 2 -> the first row sees nothing
    case = _case(FP8, 8, 2, [0, 2, 40], 3, 16, seed=4)
    case.spec.context_lens = [0, 2, 40]
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert np.all(out[:3].numpy() == 0)
    assert np.all(np.isneginf(lse[:3].numpy()))
    assert np.all(out[3].numpy() == 0) and np.all(np.isneginf(lse[3].numpy()))
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse, what="empty rows")


def test_decode_tensor_core_path_empty_context_and_q_len_beyond_context():
    # 5 tokens x G = 4 = 20 rows: the tcgen05 kernel.  Context 0 -> zeros /
    # -inf; q_len 5 over context 3 -> the first two rows see nothing.
    case = _case(FP8, 8, 2, [0, 3, 40], 5, 16, seed=5)
    case.spec.context_lens = [0, 3, 40]
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert np.all(out[:5].numpy() == 0)
    assert np.all(np.isneginf(lse[:5].numpy()))
    assert np.all(out[5:7].numpy() == 0) and np.all(np.isneginf(lse[5:7].numpy()))
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse, what="empty rows, tcgen05 decode")


def test_decode_max_in_last_tile_and_large_logits():
    case = _case(FP8, 8, 2, [3000, 1500], 1, 16, seed=5)
    # a key at the very end of each context that aligns with every query:
    # the softmax maximum sits in the last (partial) tile
    for s, c in enumerate(case.spec.context_lens):
        j = int(case.token_offsets[s]) + c - 1
        case.k[j] = (case.q[s].float().view(2, 4, 128).mean(1) * 3).to(torch.float16)
    case.q.mul_(40.0)        # logits in the hundreds: scores must not overflow
    case.k_scale = synth.per_head_absmax_scale(case.k)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse, what="peaked")


def test_decode_uniform_logits_mean_of_values():
    case = _case(FP8, 8, 2, [513], 1, 16, seed=6)
    case.q.zero_()
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse, what="uniform")
    assert np.allclose(lse.numpy(), np.log(513), atol=1e-4)


def test_decode_block_table_permutation_is_bitwise_invariant():
    case = _case(INT8, 16, 4, [700, 333], 2, 16, seed=7)
    cache = gpu_cache(case)
    out1, lse1 = run_gpu(case, cache)
    # move every block to a new physical id
    perm = torch.randperm(case.num_blocks, generator=torch.Generator().manual_seed(3))
    moved = pk.PagedKVCache(cache.dtype, torch.empty_like(cache.k_cache),
                            torch.empty_like(cache.v_cache),
                            k_scale_tok=torch.empty_like(cache.k_scale_tok),
                            v_scale_tok=torch.empty_like(cache.v_scale_tok))
    pd = perm.cuda()
    moved.k_cache[pd] = cache.k_cache
    moved.v_cache[pd] = cache.v_cache
    moved.k_scale_tok[pd] = cache.k_scale_tok
    moved.v_scale_tok[pd] = cache.v_scale_tok
    case.block_table = perm[case.block_table.long()].to(torch.int32)
    out2, lse2 = run_gpu(case, moved)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_decode_causal_append_within_tolerance():
    # the same prefix decoded at two context lengths: the shorter run's answer
    # for its last token matches the oracle either way (split plans differ)
    case = _case(FP8, 8, 2, [2000], 1, 16, seed=8)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    for c in (1999, 2000):
        case.spec.context_lens = [c]
        case.context_lens = torch.tensor([c], dtype=torch.int32)
        out, lse = run_gpu(case, cache)
        ref, ref_lse = run_oracle(case, oc)
        assert_matches_oracle(case, oc, out, lse, ref, ref_lse, what=f"ctx {c}")


def test_decode_workspace_too_small_is_rejected():
    case = _case(FP8, 32, 4, [8192], 1, 16, seed=9)
    cache = gpu_cache(case)
    need = pk.decode_workspace_bytes(cache, 1, 1, 32, 8192)
    assert need > 0
    q = case.q.view(1, 1, 32, 128).cuda()
    ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(pk.PkvqError) as e:
        pk.paged_attn_decode(cache, q, case.block_table.cuda(), case.context_lens.cuda(), 8192,
                             case.softmax_scale, workspace=ws)
    assert e.value.status == 4


# ------------------------------------------------ E5M2, FP16, layer scale --

FORMAT_CASES = [
    # dtype, Hq, Hkv, ctx list, q_len, bs, per-layer scale
    (synth.FP8_E5M2, 32, 4, [777, 16, 1, 2049], 1, 16, False),   # mma.sync, 8 rows
    (synth.FP8_E5M2, 16, 1, [513], 1, 32, True),                  # 16 rows, layer scale
    (synth.FP8_E5M2, 32, 4, [999, 17], 5, 64, False),             # tcgen05, 40 rows
    (synth.FP16, 32, 4, [777, 16, 1, 2049], 1, 16, False),
    (synth.FP16, 8, 4, [300, 129], 1, 64, False),
    (synth.FP16, 16, 2, [1000, 333], 3, 32, False),               # tcgen05, 24 rows
    (synth.FP16, 32, 4, [4000, 5, 900], 5, 16, False),            # tcgen05, 40 rows
    (synth.FP16, 32, 4, [20000, 3], 2, 16, False),                # 16 rows, many splits
    (synth.FP8_E4M3, 32, 4, [5000, 77], 1, 16, True),             # E4M3, layer scale
    (synth.FP8_E4M3, 32, 4, [3000, 300], 5, 32, True),            # tcgen05, layer scale
]


@pytest.mark.parametrize("dtype,Hq,Hkv,ctx,ql,bs,per_layer", FORMAT_CASES)
def test_decode_new_formats_match_oracle(dtype, Hq, Hkv, ctx, ql, bs, per_layer):
    case = _case(dtype, Hq, Hkv, ctx, ql, bs, seed=22, outlier_frac=0.01,
                 scale_per_layer=per_layer)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    assert_codes_equal(cache, oc, case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse,
                          what=f"decode fmt {dtype} {Hq}/{Hkv} {ctx} q{ql} bs{bs} L{per_layer}")
    assert pk.device_status() == 0


# ---------------------------------------------------------- sliding window --

WINDOW_CASES = [
    # dtype, Hq, Hkv, ctx list, q_len, bs, window
    (FP8, 8, 2, [3000, 100, 17, 0], 1, 16, 500),       # mma.sync; windows past and inside
    (FP8, 32, 4, [16384, 700], 1, 16, 4096),           # many splits inside the window
    (INT8, 16, 4, [2000, 65], 3, 32, 129),             # 12 rows, window of one row + 1
    (INT8, 32, 4, [5000, 64, 3], 5, 16, 1000),         # tcgen05, 40 rows
    (synth.FP16, 16, 2, [3000], 4, 64, 200),           # tcgen05, FP16
    (FP8, 16, 2, [2000, 300], 10, 16, 150),            # tcgen05, 80 rows
    (synth.FP8_E5M2, 8, 2, [999], 2, 16, 1),           # window 1: each row its own key
]


@pytest.mark.parametrize("dtype,Hq,Hkv,ctx,ql,bs,window", WINDOW_CASES)
def test_decode_sliding_window_matches_oracle(dtype, Hq, Hkv, ctx, ql, bs, window):
    case = _case(dtype, Hq, Hkv, ctx, ql, bs, seed=23, window=window)
    case.spec.context_lens = list(ctx)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    out, lse = run_gpu(case, cache)
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out, lse, ref, ref_lse,
                          what=f"decode window {window} {dtype} {ctx} q{ql} bs{bs}")
    assert pk.device_status() == 0


# ---------------------------------- sequence-sharded decode (query positions) --

@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("dtype,Hq,Hkv,ctx,ql,bs", [
    (FP8, 32, 4, [32768, 5000, 16, 1], 1, 16),          # mma.sync path on every rank
    (INT8, 32, 4, [20000, 3000, 7], 5, 16),             # tcgen05 path, verify rows
    (synth.FP16, 16, 2, [4096, 100], 2, 32),
])
def test_sharded_decode_merged_matches_oracle(world, dtype, Hq, Hkv, ctx, ql, bs):
    # one GPU plays every rank in turn: each decodes its share of every
    # sequence's blocks at its queries' local positions; the merge kernel
    # combines the per-rank (out, lse) pairs
    case = _case(dtype, Hq, Hkv, ctx, ql, bs, seed=24)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    outs, lses = [], []
    for r in range(world):
        sh = synth.dcp_shard(case, world, r)
        o, l = run_gpu(case, cache, block_table=sh.block_table, context_lens=sh.context_lens,
                       query_pos=sh.query_pos)
        outs.append(o)
        lses.append(l)
    out, lse = pk.merge_attn_states(torch.stack(outs).cuda(), torch.stack(lses).cuda())
    torch.cuda.synchronize()
    ref, ref_lse = run_oracle(case, oc)
    assert_matches_oracle(case, oc, out.cpu(), lse.cpu(), ref, ref_lse,
                          what=f"sharded x{world} {dtype} {ctx} q{ql}")
    assert pk.device_status() == 0


def test_decode_workspace_reused_across_shapes():
    # One workspace, never cleared and first filled with NaN patterns, serves
    # calls of different shapes in turn: every partial a call reads it wrote
    # itself.
    ws = torch.full((48 << 20,), 0xFF, dtype=torch.uint8, device="cuda")
    specs = [
        (FP8, 32, 4, [16384, 300, 5000], 1, 16),    # mma.sync, merge kernel
        (INT8, 32, 4, [9000, 17], 5, 16),           # tcgen05, merge kernel
        (FP8, 16, 2, [20000, 4000], 1, 32),         # mma.sync again, other partial sizes
        (INT8, 16, 4, [3000, 12000, 64], 1, 16),
    ]
    for dtype, Hq, Hkv, ctx, ql, bs in specs:
        case = _case(dtype, Hq, Hkv, ctx, ql, bs, seed=25)
        cache = gpu_cache(case)
        B = len(ctx)
        q = case.q.view(B, ql, Hq, 128).cuda()
        bt, cl = case.block_table.cuda(), case.context_lens.cuda()
        assert pk.decode_workspace_bytes(cache, B, ql, Hq, max(ctx)) <= ws.numel()
        shared = pk.paged_attn_decode(cache, q, bt, cl, max(ctx), case.softmax_scale,
                                      workspace=ws)
        fresh = pk.paged_attn_decode(cache, q, bt, cl, max(ctx), case.softmax_scale)
        torch.cuda.synchronize()
        assert torch.equal(shared, fresh)
    assert pk.device_status() == 0
