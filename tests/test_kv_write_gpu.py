"""GPU parity of pkvq_kv_write_quant against the oracle: codes and INT8 scales
must be bit-identical, exhaustively over fp16 bit patterns."""
import numpy as np
import pytest
import torch

import oracle
import paged_quantized_kv_quant_b200 as pk
import synth
from pkvq_testutil import assert_codes_equal, bits16, gpu_cache, oracle_cache

pytestmark = pytest.mark.gpu


def _all_fp16_rows(finite_only: bool) -> torch.Tensor:
    b = np.arange(65536, dtype=np.uint16)
    if finite_only:
        b = b[(b & 0x7C00) != 0x7C00]
    pad = (-b.size) % 128
    b = np.concatenate([b, np.zeros(pad, np.uint16)])
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.float16).view(-1, 1, 128)


def _write_both(dtype, k, v, slots, num_blocks, bs, Hkv, k_scale=None, v_scale=None):
    cache = pk.PagedKVCache.allocate(dtype, num_blocks, bs, Hkv, 128, k_scale=k_scale,
                                     v_scale=v_scale)
    pk.kv_write_quant(cache, k.cuda(), v.cuda(), slots.cuda())
    torch.cuda.synchronize()
    oc = oracle.Cache(dtype, num_blocks, bs, Hkv, 128,
                      None if k_scale is None else np.asarray(k_scale, np.float32),
                      None if v_scale is None else np.asarray(v_scale, np.float32))
    oc.write(bits16(k), bits16(v), slots.numpy())
    return cache, oc


# Power-of-two scales put every fp16 value exactly on its quotient, so the
# E4M3 / E5M2 rounding midpoints among fp16 values are hit exactly (ties to
# even); 1 +- 2^-22 moves them a fraction of an fp32 ulp off the midpoints,
# where a product with the rounded reciprocal can round the other way; tiny
# and huge scales take the quotient to both ends of the fp32 range.
@pytest.mark.parametrize("dtype", [synth.FP8_E4M3, synth.FP8_E5M2])
@pytest.mark.parametrize("scale", [1.0, 0.125, 0.0123, 4.4 / 448, 3.0e-5, 0.0,
                                   1.0 + 2.0 ** -22, 1.0 - 2.0 ** -22, 1.0e-38, 3.0e37])
def test_fp8_every_fp16_pattern(dtype, scale):
    k = _all_fp16_rows(finite_only=False)                 # includes inf and NaN patterns
    v = torch.flip(k, dims=[0]).contiguous()
    T = k.shape[0]
    slots = torch.randperm(T, generator=torch.Generator().manual_seed(1)).to(torch.int32)
    cache, oc = _write_both(dtype, k, v, slots, T // 16, 16, 1,
                            k_scale=[scale], v_scale=[scale * 2])
    for name in ("k_cache", "v_cache"):
        g = getattr(cache, name).cpu().numpy()
        o = getattr(oc, name)
        assert np.array_equal(g, o), f"{name}: {(g != o).sum()} codes differ"


def test_int8_every_finite_fp16_pattern_and_scales():
    k = _all_fp16_rows(finite_only=True)
    # rows with mixed magnitudes: shuffle so each row has a different absmax
    gen = torch.Generator().manual_seed(2)
    flat = k.view(-1)
    k = flat[torch.randperm(flat.numel(), generator=gen)].view(-1, 1, 128).contiguous()
    v = (k.float() * 0.5).to(torch.float16)
    T = k.shape[0]
    bs = 16
    slots = torch.arange(T, dtype=torch.int32)
    cache, oc = _write_both(synth.INT8, k, v, slots, (T + bs - 1) // bs, bs, 1)
    for name in ("k_cache", "v_cache"):
        assert np.array_equal(getattr(cache, name).cpu().numpy(), getattr(oc, name)), name
    for name in ("k_scale_tok", "v_scale_tok"):
        assert np.array_equal(bits16(getattr(cache, name).cpu()), getattr(oc, name)), name


def test_int8_half_integer_quotients():
    # rows whose absmax is 127 have scale 1: x = k + 1/2 is an exact tie
    # (rint to even); other rows put x / s a hair off the half-integers
    gen = torch.Generator().manual_seed(4)
    half = torch.arange(-127, 127, dtype=torch.float32) + 0.5
    rows = []
    for r in range(64):
        x = half[torch.randint(0, half.numel(), (128,), generator=gen)]
        x[0] = 127.0 if r % 2 == 0 else 127.0 * (1.0 + r * 2.0 ** -11)
        rows.append(x)
    k = torch.stack(rows).to(torch.float16).view(-1, 1, 128)
    v = (-k.float()).to(torch.float16)
    T = k.shape[0]
    slots = torch.arange(T, dtype=torch.int32)
    cache, oc = _write_both(synth.INT8, k, v, slots, T // 16, 16, 1)
    for name in ("k_cache", "v_cache"):
        assert np.array_equal(getattr(cache, name).cpu().numpy(), getattr(oc, name)), name
    for name in ("k_scale_tok", "v_scale_tok"):
        assert np.array_equal(bits16(getattr(cache, name).cpu()), getattr(oc, name)), name


@pytest.mark.parametrize("dtype", [synth.FP8_E4M3, synth.INT8])
@pytest.mark.parametrize("bs", [16, 32, 64])
def test_random_tokens_ragged_and_skipped(dtype, bs):
    spec = synth.CaseSpec("decode", dtype, 8, 4, [37, 1, 300], [1, 1, 1], block_size=bs,
                          outlier_frac=0.02, seed=3)
    case = synth.make_case(spec)
    case.slot_mapping[5] = -1     # a skipped token leaves its slot untouched
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    # the skipped slot still holds the poison fill on the GPU; exclude it
    keep = case.slot_mapping >= 0
    case.slot_mapping = case.slot_mapping[keep]
    assert_codes_equal(cache, oc, case)


def test_int8_rows_of_zeros_and_single_spikes():
    T = 64
    k = torch.zeros((T, 2, 128), dtype=torch.float16)
    for i in range(1, T):
        k[i, i % 2, (7 * i) % 128] = float(np.float16(2.0 ** (i % 30 - 15)))
    k[3, 1] = -k[3, 1] - 1.0
    v = -k
    slots = torch.arange(T, dtype=torch.int32)
    cache, oc = _write_both(synth.INT8, k, v, slots, T // 16, 16, 2)
    for name in ("k_cache", "v_cache"):
        assert np.array_equal(getattr(cache, name).cpu().numpy(), getattr(oc, name)), name
    for name in ("k_scale_tok", "v_scale_tok"):
        assert np.array_equal(bits16(getattr(cache, name).cpu()), getattr(oc, name)), name


def test_zero_tokens_is_a_noop():
    cache = pk.PagedKVCache.allocate(synth.FP8_E4M3, 4, 16, 2, k_scale=[1.0, 1.0],
                                     v_scale=[1.0, 1.0])
    cache.k_cache.fill_(5)
    e = torch.empty((0, 2, 128), dtype=torch.float16, device="cuda")
    pk.kv_write_quant(cache, e, e, torch.empty(0, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert int(cache.k_cache.min()) == 5 and int(cache.k_cache.max()) == 5


def test_device_status_clean_after_writes():
    assert pk.device_status(clear=True) == 0


# ------------------------------------------------ E5M2, FP16, layer scale --

@pytest.mark.parametrize("scale", [1.0, 0.125, 0.0123, 90.0 / 57344, 3.0e-5, 0.0])
def test_e5m2_every_fp16_pattern(scale):
    k = _all_fp16_rows(finite_only=False)                 # includes inf and NaN patterns
    v = torch.flip(k, dims=[0]).contiguous()
    T = k.shape[0]
    slots = torch.randperm(T, generator=torch.Generator().manual_seed(5)).to(torch.int32)
    cache, oc = _write_both(synth.FP8_E5M2, k, v, slots, T // 16, 16, 1,
                            k_scale=[scale], v_scale=[scale * 2])
    for name in ("k_cache", "v_cache"):
        g = getattr(cache, name).cpu().numpy()
        o = getattr(oc, name)
        assert np.array_equal(g, o), f"{name}: {(g != o).sum()} codes differ"


def test_fp16_cache_holds_every_pattern_bit_for_bit():
    k = _all_fp16_rows(finite_only=False)
    v = torch.flip(k, dims=[0]).contiguous()
    T = k.shape[0]
    slots = torch.randperm(T, generator=torch.Generator().manual_seed(6)).to(torch.int32)
    cache, oc = _write_both(synth.FP16, k, v, slots, T // 32, 32, 1)
    for name in ("k_cache", "v_cache"):
        assert np.array_equal(getattr(cache, name).cpu().numpy(), getattr(oc, name)), name


@pytest.mark.parametrize("dtype", [synth.FP8_E4M3, synth.FP8_E5M2])
def test_per_layer_scale_write(dtype):
    spec = synth.CaseSpec("decode", dtype, 8, 4, [300, 7], [1, 1], outlier_frac=0.02,
                          scale_per_layer=True, seed=8)
    case = synth.make_case(spec)
    assert case.k_scale.shape == (1,)
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    assert_codes_equal(cache, oc, case)


@pytest.mark.parametrize("dtype", [synth.FP8_E5M2, synth.FP16])
@pytest.mark.parametrize("bs", [16, 32, 64])
def test_new_formats_ragged_and_skipped(dtype, bs):
    spec = synth.CaseSpec("decode", dtype, 8, 4, [37, 1, 300], [1, 1, 1], block_size=bs,
                          outlier_frac=0.02, seed=9)
    case = synth.make_case(spec)
    case.slot_mapping[5] = -1
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    keep = case.slot_mapping >= 0
    case.slot_mapping = case.slot_mapping[keep]
    assert_codes_equal(cache, oc, case)
