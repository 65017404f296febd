"""Pins for the CPU oracle: every routine is checked against something other
than itself (library conversions, published format tables, a brute-force
dense attention written with numpy, and invariants of softmax attention).

CPU only; runs with ``-m "not gpu"``.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------- binary16 --

def test_half_to_double_exhaustive_vs_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ours = oracle.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros keep their sign
    assert math.copysign(1.0, ours[0x8000]) == -1.0


def _f32_neighbours(x):
    x = np.asarray(x, np.float32)
    up = np.nextafter(x, np.float32(np.inf))
    dn = np.nextafter(x, np.float32(-np.inf))
    return np.concatenate([x, up, dn])


def test_float_to_half_rn_vs_numpy():
    h = np.arange(0, 0x7c00, dtype=np.uint16).view(np.float16).astype(np.float32)
    mids = ((h[:-1].astype(np.float64) + h[1:].astype(np.float64)) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64),
                          (h[:-1].astype(np.float64) + h[1:]) / 2)  # midpoints exact in fp32
    rng = np.random.default_rng(1)
    rnd = (rng.standard_normal(200000) * np.exp2(rng.integers(-30, 18, 200000))).astype(np.float32)
    xs = np.concatenate([_f32_neighbours(h), _f32_neighbours(mids), rnd,
                         np.float32([65504, 65519.99, 65520, 65536, 1e30, np.inf,
                                     2.0 ** -25, 2.0 ** -24 * 1.5, 2.0 ** -26])])
    xs = np.concatenate([xs, -xs])
    ours = oracle.float_to_half_bits(xs)
    ref = xs.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    nan_bits = oracle.float_to_half_bits(np.float32([np.nan]))
    assert (nan_bits[0] & 0x7c00) == 0x7c00 and (nan_bits[0] & 0x3ff) != 0


# ------------------------------------------------------------------ E4M3 --

def test_e4m3_decode_exhaustive_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decode_golden_spot_values():
    n = 0
    with open(os.path.join(GOLDEN, "e4m3_spot_values.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            code, val = line.split()
            got = oracle.e4m3_decode([int(code, 16)])[0]
            if val == "nan":
                assert math.isnan(got), code
            else:
                assert got == float(val), code
                assert math.copysign(1, got) == math.copysign(1, float(val)), code
            n += 1
    assert n >= 15


def _finite_codes():
    return np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)


def test_e4m3_encode_representables_map_to_themselves():
    codes = _finite_codes()
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_e4m3_encode_midpoints_ties_to_even_and_neighbours():
    pos = np.arange(0, 0x7F, dtype=np.uint8)          # 0 .. 448, ascending
    vals = oracle.e4m3_decode(pos)
    assert np.all(np.diff(vals) > 0)
    lo, hi = pos[:-1], pos[1:]
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)
    even = np.where(lo % 2 == 0, lo, hi)              # the code with an even mantissa
    for sgn in (1, -1):
        s = np.uint8(0x80 if sgn < 0 else 0)
        assert np.array_equal(oracle.e4m3_encode(sgn * mids), even | s)
        up = np.nextafter(mids, np.float32(np.inf)) if sgn > 0 else \
            -np.nextafter(mids, np.float32(np.inf))
        dn = np.nextafter(mids, np.float32(-np.inf)) if sgn > 0 else \
            -np.nextafter(mids, np.float32(-np.inf))
        assert np.array_equal(oracle.e4m3_encode(up), hi | s)
        assert np.array_equal(oracle.e4m3_encode(dn), lo | s)


def test_e4m3_encode_vs_torch_in_range():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(300000) * np.exp2(rng.integers(-14, 9, 300000))).astype(np.float32)
    x = x[np.abs(x) < 464.0]      # below the first value that rounds past 448
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturation_and_specials():
    big = np.float32([448.0, 449.0, 463.99, 464.0, 480.0, 1e6, 3.4e38, np.inf])
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)
    assert oracle.e4m3_encode(np.float32([np.nan]))[0] == 0x7F
    assert oracle.e4m3_encode(-np.float32([np.nan]))[0] == 0xFF
    assert oracle.e4m3_encode(np.float32([0.0]))[0] == 0x00
    assert oracle.e4m3_encode(np.float32([-0.0]))[0] == 0x80
    # below half the smallest subnormal -> signed zero; exactly half -> even (0)
    tiny = np.float32([2.0 ** -11, 2.0 ** -10, np.nextafter(np.float32(2.0 ** -10), 1)])
    assert list(oracle.e4m3_encode(tiny)) == [0x00, 0x00, 0x01]
    assert list(oracle.e4m3_encode(-tiny)) == [0x80, 0x80, 0x81]


def test_quant_row_fp8_is_divide_then_encode():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(128).astype(np.float16)
    for scale in (1.0, 0.125, 0.0123, float(np.float32(4.3) / np.float32(448))):
        sc = np.float32(scale)
        q = x.astype(np.float32) / sc               # numpy fp32 IEEE division
        ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(oracle.quant_row_fp8(x.view(np.uint16), scale), ref)
    assert np.all(oracle.quant_row_fp8(x.view(np.uint16), 0.0) == 0)


# ------------------------------------------------------------------ INT8 --

def _int8_ref(x16):
    """numpy restatement: fp32 absmax/127 -> fp16 -> fp32 divide -> rint -> clip."""
    xf = x16.astype(np.float32)
    s16 = (np.float32(np.abs(xf).max()) / np.float32(127.0)).astype(np.float16)
    s = np.float32(s16)
    if s == 0:
        return np.zeros(x16.shape, np.int8), s16
    return np.clip(np.rint(xf / s), -127, 127).astype(np.int8), s16


def test_int8_rows_vs_numpy():
    rng = np.random.default_rng(4)
    for i in range(300):
        scale = float(np.exp2(rng.integers(-20, 12)))
        x = (rng.standard_normal(128) * scale).astype(np.float16)
        codes, s = oracle.quant_row_int8(x.view(np.uint16))
        rc, rs = _int8_ref(x)
        assert s == int(rs.view(np.uint16)), i
        assert np.array_equal(codes, rc), i


def test_int8_absmax_element_and_ties():
    x = np.zeros(128, np.float16)
    x[7] = -63.5                    # absmax 63.5 -> s = 0.5 exactly
    x[0], x[1], x[2], x[3] = 1.25, 1.75, -1.25, 0.25   # x/s = 2.5, 3.5, -2.5, 0.5
    codes, s = oracle.quant_row_int8(x.view(np.uint16))
    assert s == int(np.float16(0.5).view(np.uint16))
    assert codes[7] == -127
    assert list(codes[:4]) == [2, 4, -2, 0]
    z, sz = oracle.quant_row_int8(np.zeros(128, np.uint16))
    assert sz == 0 and np.all(z == 0)


# ------------------------------------------------------------- attention --

def _dequant_dense(cache, block_table, ctx, s):
    """numpy/torch gather of sequence s's keys/values into dense float64
    [ctx][Hkv][D], decoding codes with torch's own float8 type."""
    bs = cache.block_size
    j = np.arange(ctx)
    blk = block_table[s, j // bs]
    off = j % bs
    kc = cache.k_cache[blk, :, off, :]          # [ctx][Hkv][D]
    vc = cache.v_cache[blk, :, off, :]
    if cache.dtype in (oracle.FP8_E4M3, oracle.FP8_E5M2):
        tdt = torch.float8_e4m3fn if cache.dtype == oracle.FP8_E4M3 else torch.float8_e5m2
        dec = lambda c: torch.from_numpy(np.ascontiguousarray(c)).view(tdt).to(
            torch.float64).numpy()
        ks = np.broadcast_to(cache.k_scale.astype(np.float64), (cache.Hkv,))
        vs = np.broadcast_to(cache.v_scale.astype(np.float64), (cache.Hkv,))
        k = dec(kc) * ks[None, :, None]
        v = dec(vc) * vs[None, :, None]
    elif cache.dtype == oracle.FP16:
        k = np.ascontiguousarray(kc).view(np.float16).astype(np.float64)
        v = np.ascontiguousarray(vc).view(np.float16).astype(np.float64)
    else:
        ks = cache.k_scale_tok[blk, :, off].view(np.float16).astype(np.float64)
        vs = cache.v_scale_tok[blk, :, off].view(np.float16).astype(np.float64)
        k = kc.view(np.int8).astype(np.float64) * ks[:, :, None]
        v = vc.view(np.int8).astype(np.float64) * vs[:, :, None]
    return k, v


def _brute_force(cache, case, window=0):
    """Dense softmax attention with numpy matmuls, one sequence at a time
    (window > 0: each query also ignores keys more than window - 1 behind it)."""
    q = case.q.view(torch.int16).numpy().view(np.float16).astype(np.float64)
    Hq = q.shape[1]
    G = Hq // cache.Hkv
    bt = case.block_table.numpy()
    out = np.zeros(q.shape)
    lse = np.full(q.shape[:2], -np.inf)
    cu = case.cu_seqlens_q.numpy()
    for s, (c, ql) in enumerate(zip(case.spec.context_lens, case.spec.q_lens)):
        if c == 0:
            continue
        k, v = _dequant_dense(cache, bt, c, s)
        kh = np.repeat(k, G, axis=1)             # [c][Hq][D]
        vh = np.repeat(v, G, axis=1)
        qs = q[cu[s]:cu[s + 1]]                  # [ql][Hq][D]
        sc = np.einsum("thd,jhd->htj", qs, kh) * np.float64(case.softmax_scale)
        pos = c - ql + np.arange(ql)
        mask = np.arange(c)[None, :] > pos[:, None]      # [ql][c]
        if window > 0:
            mask |= np.arange(c)[None, :] <= pos[:, None] - window
        if mask.all(axis=1).any():
            raise ValueError("brute force needs every row to see a key")
        sc = np.where(mask[None], -np.inf, sc)
        m = sc.max(-1, keepdims=True)
        p = np.exp(sc - m)
        l = p.sum(-1, keepdims=True)
        o = np.einsum("htj,jhd->thd", p / l, vh)
        out[cu[s]:cu[s + 1]] = o
        lse[cu[s]:cu[s + 1]] = (m[..., 0] + np.log(l[..., 0])).T
    return out, lse


def _build(spec):
    case = synth.make_case(spec)
    cache = oracle.Cache(spec.kv_dtype, case.num_blocks, spec.block_size,
                         spec.num_kv_heads, spec.head_dim,
                         None if case.k_scale is None else case.k_scale.numpy(),
                         None if case.v_scale is None else case.v_scale.numpy(),
                         scale_per_layer=spec.scale_per_layer)
    cache.write(case.k.view(torch.int16).numpy(), case.v.view(torch.int16).numpy(),
                case.slot_mapping.numpy())
    return case, cache


def _run(case, cache, rows=None, **kw):
    return oracle.paged_attention(cache, case.q.view(torch.int16).numpy(),
                                  case.cu_seqlens_q.numpy(), case.context_lens.numpy(),
                                  case.block_table.numpy(), case.softmax_scale, rows=rows,
                                  window=case.spec.window, **kw)


BRUTE_CASES = [
    # kind, dtype, Hq, Hkv, ctx, qlen, D, bs
    ("decode", oracle.FP8_E4M3, 8, 2, [37], [1], 128, 16),
    ("decode", oracle.FP8_E4M3, 4, 4, [1, 17, 40], [1, 1, 1], 8, 4),
    ("decode", oracle.INT8, 16, 2, [33, 5], [5, 5], 128, 16),
    ("prefill", oracle.FP8_E4M3, 8, 1, [19, 40, 7], [19, 12, 1], 8, 4),
    ("prefill", oracle.INT8, 8, 4, [40, 24], [40, 3], 128, 16),
    ("prefill", oracle.FP8_E4M3, 2, 2, [23], [23], 8, 16),
    ("decode", oracle.FP8_E5M2, 8, 2, [37, 3], [2, 2], 128, 16),
    ("prefill", oracle.FP8_E5M2, 8, 4, [40, 24], [40, 3], 16, 8),
    ("decode", oracle.FP16, 16, 2, [33, 5], [5, 5], 128, 16),
    ("prefill", oracle.FP16, 4, 1, [19, 30], [19, 7], 8, 4),
]


@pytest.mark.parametrize("kind,dt,Hq,Hkv,ctx,ql,D,bs", BRUTE_CASES)
@pytest.mark.parametrize("window", [0, 5])
def test_attention_vs_dense_brute_force(kind, dt, Hq, Hkv, ctx, ql, D, bs, window):
    spec = synth.CaseSpec(kind, dt, Hq, Hkv, ctx, ql, head_dim=D, block_size=bs, seed=11,
                          window=window)
    case, cache = _build(spec)
    out, lse, _ = _run(case, cache)
    ref_out, ref_lse = _brute_force(cache, case, window=window)
    assert np.allclose(out, ref_out, rtol=0, atol=1e-12)
    assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_attention_sampled_rows_match_full():
    spec = synth.CaseSpec("prefill", oracle.FP8_E4M3, 8, 2, [30, 21], [30, 9],
                          head_dim=16, block_size=4, seed=5)
    case, cache = _build(spec)
    out, lse, _ = _run(case, cache)
    rows = np.array([[0, 0], [29, 7], [30, 3], [38, 5], [5, 1]], np.int32)
    o2, l2, _ = _run(case, cache, rows=rows)
    for r, (i, h) in enumerate(rows):
        assert np.array_equal(o2[r], out[i, h]) and l2[r] == lse[i, h]


def test_one_key_returns_that_value_row_exactly():
    for dt in (oracle.FP8_E4M3, oracle.INT8):
        spec = synth.CaseSpec("decode", dt, 8, 2, [1], [1], seed=7)
        case, cache = _build(spec)
        out, lse, _ = _run(case, cache)
        _, v = _dequant_dense(cache, case.block_table.numpy(), 1, 0)
        G = 4
        for h in range(8):
            assert np.array_equal(out[0, h], v[0, h // G])
        # lse of a single key is its score
        k, _ = _dequant_dense(cache, case.block_table.numpy(), 1, 0)
        q = case.q.float().double().numpy()
        for h in range(8):
            sc = np.float64(case.softmax_scale) * float(np.dot(q[0, h], k[0, h // G]))
            assert abs(lse[0, h] - sc) < 1e-12


def test_uniform_logits_give_mean_of_visible_values():
    spec = synth.CaseSpec("prefill", oracle.FP8_E4M3, 4, 2, [26], [26], head_dim=16,
                          block_size=4, seed=8)
    case, cache = _build(spec)
    case.q.zero_()
    out, lse, _ = _run(case, cache)
    _, v = _dequant_dense(cache, case.block_table.numpy(), 26, 0)
    for t in range(26):
        for h in range(4):
            assert np.allclose(out[t, h], v[:t + 1, h // 2].mean(0), atol=1e-13, rtol=0)
            assert abs(lse[t, h] - math.log(t + 1)) < 1e-13


def test_causal_append_leaves_earlier_rows_unchanged():
    base = synth.CaseSpec("prefill", oracle.INT8, 4, 2, [33], [33], head_dim=16,
                          block_size=4, seed=9)
    case, cache = _build(base)
    out, lse, _ = _run(case, cache)
    # the same sequence cut after 20 tokens: the first 20 rows must not move
    case20 = synth.make_case(base)
    keep = 20
    case20.spec.context_lens = [keep]
    case20.spec.q_lens = [keep]
    case20.q = case20.q[:keep].clone()
    case20.context_lens = torch.tensor([keep], dtype=torch.int32)
    case20.cu_seqlens_q = torch.tensor([0, keep], dtype=torch.int32)
    o20, l20, _ = _run(case20, cache)
    assert np.array_equal(o20, out[:keep]) and np.array_equal(l20, lse[:keep])


def test_block_table_permutation_invariance():
    spec = synth.CaseSpec("prefill", oracle.FP8_E4M3, 8, 2, [45, 17], [6, 17],
                          head_dim=16, block_size=4, seed=10)
    case, cache = _build(spec)
    out, lse, _ = _run(case, cache)
    # move every block to a new physical id and rewrite the table to match
    rng = np.random.default_rng(0)
    perm = rng.permutation(case.num_blocks)
    moved = oracle.Cache(cache.dtype, cache.num_blocks, cache.block_size, cache.Hkv,
                         cache.D, cache.k_scale, cache.v_scale)
    moved.k_cache[perm] = cache.k_cache
    moved.v_cache[perm] = cache.v_cache
    case.block_table = torch.from_numpy(perm[case.block_table.numpy()].astype(np.int32))
    o2, l2, _ = _run(case, moved)
    assert np.array_equal(o2, out) and np.array_equal(l2, lse)


def test_gqa_equals_mha_with_replicated_kv_heads():
    spec = synth.CaseSpec("prefill", oracle.FP8_E4M3, 8, 2, [21], [21], head_dim=16,
                          block_size=4, seed=12)
    case, cache = _build(spec)
    out, lse, _ = _run(case, cache)
    G = 4
    rep = oracle.Cache(cache.dtype, cache.num_blocks, cache.block_size, 8, cache.D,
                       np.repeat(cache.k_scale, G), np.repeat(cache.v_scale, G))
    rep.k_cache[:] = np.repeat(cache.k_cache, G, axis=1)
    rep.v_cache[:] = np.repeat(cache.v_cache, G, axis=1)
    o2, l2, _ = _run(case, rep)
    assert np.array_equal(o2, out) and np.array_equal(l2, lse)


def test_k_scale_power_of_two_trades_with_softmax_scale():
    spec = synth.CaseSpec("decode", oracle.FP8_E4M3, 8, 2, [50], [3], head_dim=16,
                          block_size=16, seed=13)
    case, cache = _build(spec)
    out, lse, _ = _run(case, cache)
    cache.k_scale = (cache.k_scale * np.float32(4.0)).astype(np.float32)
    case.softmax_scale = case.softmax_scale / 4.0
    o2, l2, _ = _run(case, cache)
    assert np.array_equal(o2, out) and np.array_equal(l2, lse)


def test_empty_rows_give_zero_and_minus_inf():
    # q_len > context: the first query rows see no key at all
    spec = synth.CaseSpec("decode", oracle.FP8_E4M3, 4, 2, [2, 0], [3, 3],
                          head_dim=8, block_size=4, seed=14)
    case, cache = _build(spec)
    out, lse, _ = _run(case, cache)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(out[3:] == 0) and np.all(np.isneginf(lse[3:]))
    assert np.all(np.isfinite(lse[1:3]))


def test_kv_write_skips_negative_slots_and_places_rows():
    spec = synth.CaseSpec("decode", oracle.INT8, 4, 2, [9], [1], head_dim=8,
                          block_size=4, seed=15)
    case = synth.make_case(spec)
    cache = oracle.Cache(oracle.INT8, case.num_blocks, 4, 2, 8)
    sm = case.slot_mapping.numpy().copy()
    sm[3] = -1
    cache.write(case.k.view(torch.int16).numpy(), case.v.view(torch.int16).numpy(), sm)
    kb = case.k.view(torch.int16).numpy().view(np.uint16)
    for i in range(9):
        blk, off = divmod(int(case.slot_mapping[i]), 4)
        for h in range(2):
            codes, s = oracle.quant_row_int8(kb[i, h])
            if i == 3:
                assert np.all(cache.k_cache[blk, h, off] == 0)
                assert cache.k_scale_tok[blk, h, off] == 0
            else:
                assert np.array_equal(cache.k_cache[blk, h, off].view(np.int8), codes)
                assert cache.k_scale_tok[blk, h, off] == s


# ------------------------------------------------------------------ E5M2 --

def test_e5m2_decode_exhaustive_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e5m2_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e5m2).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF}
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # E5M2 is the top byte of an fp16: the same value as the fp16 pattern code << 8
    h = (codes.astype(np.uint16) << 8).view(np.float16).astype(np.float64)
    assert np.array_equal(ours[~nan], h[~nan])
    assert ours[0x7B] == 57344.0 and ours[0x7C] == np.inf and ours[0xFC] == -np.inf
    assert ours[0x01] == 2.0 ** -16 and ours[0x3C] == 1.0


def _e5m2_finite():
    return np.array([c for c in range(256) if (c & 0x7C) != 0x7C], np.uint8)


def test_e5m2_encode_representables_map_to_themselves():
    codes = _e5m2_finite()
    vals = oracle.e5m2_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e5m2_encode(vals), codes)


def test_e5m2_encode_midpoints_ties_to_even_and_neighbours():
    pos = np.arange(0, 0x7C, dtype=np.uint8)          # 0 .. 57344, ascending
    vals = oracle.e5m2_decode(pos)
    assert np.all(np.diff(vals) > 0)
    lo, hi = pos[:-1], pos[1:]
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)
    even = np.where(lo % 2 == 0, lo, hi)
    for sgn in (1, -1):
        s = np.uint8(0x80 if sgn < 0 else 0)
        assert np.array_equal(oracle.e5m2_encode(sgn * mids), even | s)
        up = np.nextafter(mids, np.float32(np.inf))
        dn = np.nextafter(mids, np.float32(-np.inf))
        assert np.array_equal(oracle.e5m2_encode(sgn * up), hi | s)
        assert np.array_equal(oracle.e5m2_encode(sgn * dn), lo | s)


def test_e5m2_encode_vs_torch_in_range():
    rng = np.random.default_rng(21)
    x = (rng.standard_normal(300000) * np.exp2(rng.integers(-20, 16, 300000))).astype(np.float32)
    x = x[np.abs(x) < 61440.0]   # torch's cast overflows to inf from the midpoint up
    ours = oracle.e5m2_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e5m2_encode_saturation_and_specials():
    big = np.float32([57344.0, 57345.0, 61439.0, 61440.0, 65536.0, 1e30, np.inf])
    assert np.all(oracle.e5m2_encode(big) == 0x7B)
    assert np.all(oracle.e5m2_encode(-big) == 0xFB)
    assert oracle.e5m2_encode(np.float32([np.nan]))[0] == 0x7F
    assert oracle.e5m2_encode(-np.float32([np.nan]))[0] == 0xFF
    assert oracle.e5m2_encode(np.float32([-0.0]))[0] == 0x80
    tiny = np.float32([2.0 ** -18, 2.0 ** -17, np.nextafter(np.float32(2.0 ** -17), 1)])
    assert list(oracle.e5m2_encode(tiny)) == [0x00, 0x00, 0x01]


def test_quant_row_e5m2_is_divide_then_encode():
    rng = np.random.default_rng(22)
    x = (rng.standard_normal(128) * 30).astype(np.float16)
    for scale in (1.0, 0.125, 0.0123, float(np.float32(90.0) / np.float32(57344))):
        q = x.astype(np.float32) / np.float32(scale)
        ref = torch.from_numpy(q).to(torch.float8_e5m2).view(torch.uint8).numpy()
        assert np.array_equal(oracle.quant_row_fp8(x.view(np.uint16), scale, e5m2=True), ref)


# ------------------------------------------------- FP16 cache, layer scale --

def test_fp16_cache_stores_the_values_bit_for_bit():
    spec = synth.CaseSpec("decode", oracle.FP16, 4, 2, [9, 4], [1, 1], head_dim=8,
                          block_size=4, seed=23)
    case, cache = _build(spec)
    kb = case.k.view(torch.int16).numpy().view(np.uint16)
    for i in range(13):
        blk, off = divmod(int(case.slot_mapping[i]), 4)
        for h in range(2):
            assert np.array_equal(cache.k_cache[blk, h, off].view(np.uint16), kb[i, h])


def test_per_layer_scale_equals_equal_per_head_scales():
    for dt in (oracle.FP8_E4M3, oracle.FP8_E5M2):
        spec = synth.CaseSpec("decode", dt, 8, 4, [50, 7], [2, 2], head_dim=16,
                              block_size=4, seed=24, scale_per_layer=True)
        case, cache = _build(spec)
        assert cache.k_scale.shape == (1,)
        out, lse, _ = _run(case, cache)
        heads = oracle.Cache(dt, case.num_blocks, 4, 4, 16, np.repeat(cache.k_scale, 4),
                             np.repeat(cache.v_scale, 4))
        heads.write(case.k.view(torch.int16).numpy(), case.v.view(torch.int16).numpy(),
                    case.slot_mapping.numpy())
        assert np.array_equal(heads.k_cache, cache.k_cache)
        o2, l2, _ = _run(case, heads)
        assert np.array_equal(o2, out) and np.array_equal(l2, lse)


# ---------------------------------------------------------- sliding window --

def test_window_covering_the_context_is_full_attention():
    spec = synth.CaseSpec("prefill", oracle.FP8_E4M3, 4, 2, [30, 21], [30, 9], head_dim=16,
                          block_size=4, seed=25)
    case, cache = _build(spec)
    out, lse, _ = _run(case, cache)
    o2, l2, _ = oracle.paged_attention(cache, case.q.view(torch.int16).numpy(),
                                       case.cu_seqlens_q.numpy(), case.context_lens.numpy(),
                                       case.block_table.numpy(), case.softmax_scale,
                                       window=30)
    assert np.array_equal(o2, out) and np.array_equal(l2, lse)


def test_window_of_one_returns_the_own_value_row():
    spec = synth.CaseSpec("prefill", oracle.INT8, 4, 2, [12], [12], head_dim=16,
                          block_size=4, seed=26, window=1)
    case, cache = _build(spec)
    out, _, _ = _run(case, cache)
    _, v = _dequant_dense(cache, case.block_table.numpy(), 12, 0)
    for t in range(12):
        for h in range(4):
            assert np.array_equal(out[t, h], v[t, h // 2])


# ------------------------------------------- query positions, merged parts --

def test_explicit_default_query_positions_change_nothing():
    spec = synth.CaseSpec("decode", oracle.FP8_E4M3, 8, 2, [40, 17], [3, 3], head_dim=16,
                          block_size=4, seed=27)
    case, cache = _build(spec)
    out, lse, _ = _run(case, cache)
    qp = np.array([c - 3 + t for c in (40, 17) for t in range(3)], np.int32)
    o2, l2, _ = _run(case, cache, query_pos=qp)
    assert np.array_equal(o2, out) and np.array_equal(l2, lse)


def test_merge_of_one_part_is_the_identity_and_empty_parts_vanish():
    rng = np.random.default_rng(28)
    o = rng.standard_normal((1, 5, 8))
    l = rng.standard_normal((1, 5))
    mo, ml = oracle.merge_states(o, l)
    assert np.array_equal(mo, o[0]) and np.allclose(ml, l[0], atol=0, rtol=0)
    o2 = np.concatenate([o, rng.standard_normal((1, 5, 8))])
    l2 = np.concatenate([l, np.full((1, 5), -np.inf)])
    mo2, ml2 = oracle.merge_states(o2, l2)
    assert np.array_equal(mo2, o[0]) and np.array_equal(ml2, l[0])
    z, zl = oracle.merge_states(np.ones((2, 3, 4)), np.full((2, 3), -np.inf))
    assert np.all(z == 0) and np.all(np.isneginf(zl))


def test_merge_of_two_parts_by_hand():
    # part weights e^0 and e^ln3 -> 1/4 and 3/4; lse = ln 4
    o = np.array([[[4.0, 0.0]], [[0.0, 8.0]]])
    l = np.array([[0.0], [math.log(3.0)]])
    mo, ml = oracle.merge_states(o, l)
    assert np.allclose(mo, [[1.0, 6.0]], atol=1e-15, rtol=0)
    assert abs(ml[0] - math.log(4.0)) < 1e-15


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("dt", [oracle.FP8_E4M3, oracle.INT8])
def test_sharded_keys_merged_equal_full_attention(world, dt):
    # the decode-context-parallel layout: blocks dealt out over ranks, each
    # rank attends over its own keys at its local query positions
    spec = synth.CaseSpec("decode", dt, 8, 2, [45, 16, 3, 70], [4] * 4, head_dim=16,
                          block_size=4, seed=29)
    case, cache = _build(spec)
    full, full_lse, _ = _run(case, cache)
    outs, lses = [], []
    for r in range(world):
        sh = synth.dcp_shard(case, world, r)
        o, l, _ = oracle.paged_attention(cache, case.q.view(torch.int16).numpy(),
                                         case.cu_seqlens_q.numpy(), sh.context_lens.numpy(),
                                         sh.block_table.numpy(), case.softmax_scale,
                                         query_pos=sh.query_pos.numpy())
        outs.append(o.reshape(-1, 16))
        lses.append(l.reshape(-1))
    mo, ml = oracle.merge_states(np.stack(outs), np.stack(lses))
    assert np.allclose(mo, full.reshape(-1, 16), atol=1e-12, rtol=0)
    assert np.allclose(ml, full_lse.reshape(-1), atol=1e-12, rtol=0)


def test_shard_of_one_rank_is_the_whole_sequence():
    spec = synth.CaseSpec("decode", oracle.FP8_E4M3, 4, 2, [45, 16], [3, 3], head_dim=16,
                          block_size=4, seed=30)
    case = synth.make_case(spec)
    sh = synth.dcp_shard(case, 1, 0)
    assert torch.equal(sh.context_lens, case.context_lens)
    assert torch.equal(sh.block_table[:, :12], case.block_table[:, :12])
    assert sh.query_pos.tolist() == [42, 43, 44, 13, 14, 15]


# ------------------------------------------------------------ block copy --

@pytest.mark.parametrize("dt", [oracle.FP8_E4M3, oracle.INT8, oracle.FP16])
def test_copy_blocks_moves_whole_blocks(dt):
    spec = synth.CaseSpec("decode", dt, 4, 2, [30, 9], [1, 1], head_dim=8, block_size=4,
                          seed=31)
    case, src = _build(spec)
    dst = oracle.Cache(dt, 20, 4, 2, 8, src.k_scale, src.v_scale)
    pairs = np.array([[0, 19], [3, 0], [5, 7], [src.num_blocks - 1, 11]], np.int32)
    oracle.copy_blocks(src, dst, pairs)
    for s_, d_ in pairs:
        assert np.array_equal(dst.k_cache[d_], src.k_cache[s_])
        assert np.array_equal(dst.v_cache[d_], src.v_cache[s_])
        if dt == oracle.INT8:
            assert np.array_equal(dst.k_scale_tok[d_], src.k_scale_tok[s_])
            assert np.array_equal(dst.v_scale_tok[d_], src.v_scale_tok[s_])
    untouched = sorted(set(range(20)) - set(pairs[:, 1].tolist()))
    assert not dst.k_cache[untouched].any()
    # out and back to other ids: attention through the new table is unchanged
    back = oracle.Cache(dt, src.num_blocks, 4, 2, 8, src.k_scale, src.v_scale)
    perm = np.random.default_rng(3).permutation(src.num_blocks).astype(np.int32)
    tier = oracle.Cache(dt, src.num_blocks, 4, 2, 8, src.k_scale, src.v_scale)
    oracle.copy_blocks(src, tier, np.stack([np.arange(src.num_blocks), perm], 1))
    oracle.copy_blocks(tier, back, np.stack([perm, perm], 1))
    out, lse, _ = _run(case, src)
    case.block_table = torch.from_numpy(perm[case.block_table.numpy()])
    o2, l2, _ = _run(case, back)
    assert np.array_equal(o2, out) and np.array_equal(l2, lse)
