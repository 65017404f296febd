"""Helpers shared by the GPU parity tests: build the same seeded case on the
GPU (through the C ABI) and in the CPU oracle, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_quantized_kv_quant_b200 as pk
import synth

# Output tolerance: fp16 outputs vs the FP64 oracle, FP32 accumulation.
MAX_ABS_TOL = 2e-3
REL_L2_TOL = 1e-3
LSE_TOL = 2e-3

NAN_E4M3 = 0x7F          # an E4M3 NaN code: fills never-written cache slots
NAN_FP16_BITS = 0x7E00


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_cache(case: synth.Case) -> oracle.Cache:
    s = case.spec
    c = oracle.Cache(s.kv_dtype, case.num_blocks, s.block_size, s.num_kv_heads, s.head_dim,
                     None if case.k_scale is None else case.k_scale.numpy(),
                     None if case.v_scale is None else case.v_scale.numpy(),
                     scale_per_layer=s.scale_per_layer)
    c.write(bits16(case.k), bits16(case.v), case.slot_mapping.numpy())
    return c


def gpu_cache(case: synth.Case, poison: bool = True, write: bool = True) -> pk.PagedKVCache:
    """Allocates the cache on the GPU, fills every slot with NaN patterns
    (so that reading a never-written slot would show), then writes all
    cached tokens through pkvq_kv_write_quant."""
    s = case.spec
    cache = pk.PagedKVCache.allocate(s.kv_dtype, case.num_blocks, s.block_size,
                                     s.num_kv_heads, s.head_dim, k_scale=case.k_scale,
                                     v_scale=case.v_scale, scale_per_layer=s.scale_per_layer)
    if poison:
        # 0x7F: a NaN code of E4M3 and E5M2; 0x7F7F: an fp16 NaN
        cache.k_cache.fill_(NAN_E4M3)
        cache.v_cache.fill_(NAN_E4M3)
        if cache.k_scale_tok is not None:
            cache.k_scale_tok.view(torch.int16).fill_(NAN_FP16_BITS)
            cache.v_scale_tok.view(torch.int16).fill_(NAN_FP16_BITS)
    if write and case.k.shape[0]:
        pk.kv_write_quant(cache, case.k.cuda(), case.v.cuda(), case.slot_mapping.cuda())
    return cache


def written_mask(case: synth.Case) -> np.ndarray:
    """[NB][bs] bool: slots that hold a cached token."""
    s = case.spec
    m = np.zeros((case.num_blocks, s.block_size), bool)
    sm = case.slot_mapping.numpy()
    sm = sm[sm >= 0]
    m[sm // s.block_size, sm % s.block_size] = True
    return m


def assert_codes_equal(cache: pk.PagedKVCache, oc: oracle.Cache, case: synth.Case) -> None:
    """Bit-exact comparison of every written slot's codes (and INT8 scales)."""
    m = written_mask(case)
    for name in ("k_cache", "v_cache"):
        g = getattr(cache, name).cpu().numpy()
        o = getattr(oc, name)
        assert g.shape == o.shape, (g.shape, o.shape)
        gw = g.transpose(0, 2, 1, 3)[m]
        ow = o.transpose(0, 2, 1, 3)[m]
        bad = np.nonzero(gw != ow)
        assert gw.shape == ow.shape
        assert bad[0].size == 0, f"{name}: {bad[0].size} codes differ, first at {bad}"
    if case.spec.kv_dtype == synth.INT8:
        for name in ("k_scale_tok", "v_scale_tok"):
            g = bits16(getattr(cache, name).cpu()).transpose(0, 2, 1)[m]
            o = getattr(oc, name).transpose(0, 2, 1)[m]
            assert np.array_equal(g, o), f"{name} differs"


def run_gpu(case: synth.Case, cache: pk.PagedKVCache, want_lse: bool = True,
            block_table=None, context_lens=None, query_pos=None):
    """The case through the C ABI; block_table / context_lens / query_pos
    (decode) replace the case's own, e.g. for one rank's share of the keys."""
    s = case.spec
    dev = "cuda"
    bt = (case.block_table if block_table is None else block_table).to(dev)
    ctx = (case.context_lens if context_lens is None else context_lens).to(dev)
    if s.kind == "decode":
        B = len(s.context_lens)
        ql = s.q_lens[0]
        q = case.q.view(B, ql, s.num_q_heads, s.head_dim).to(dev)
        lse = torch.empty((B, ql, s.num_q_heads), dtype=torch.float32, device=dev) \
            if want_lse else None
        qp = None if query_pos is None else query_pos.view(B, ql).to(dev)
        lens = s.context_lens if context_lens is None else context_lens.tolist()
        out = pk.paged_attn_decode(cache, q, bt, ctx, max(list(lens) + [0]),
                                   case.softmax_scale, lse=lse, sliding_window=s.window,
                                   query_pos=qp)
        out = out.view(-1, s.num_q_heads, s.head_dim)
        lse = None if lse is None else lse.view(-1, s.num_q_heads)
    else:
        q = case.q.to(dev)
        lse = torch.empty((q.shape[0], s.num_q_heads), dtype=torch.float32, device=dev) \
            if want_lse else None
        out = pk.paged_attn_prefill(cache, q, case.cu_seqlens_q.to(dev), bt, ctx,
                                    max(s.q_lens + [0]), case.softmax_scale, lse=lse,
                                    sliding_window=s.window)
    torch.cuda.synchronize()
    return out.cpu(), (None if lse is None else lse.cpu())


def run_oracle(case: synth.Case, oc: oracle.Cache, rows=None):
    return oracle.paged_attention(oc, bits16(case.q), case.cu_seqlens_q.numpy(),
                                  case.context_lens.numpy(), case.block_table.numpy(),
                                  case.softmax_scale, rows=rows, window=case.spec.window)[:2]


def abs_value_oracle(case: synth.Case, oc: oracle.Cache, rows=None) -> np.ndarray:
    """A(r, d) = sum_j P_rj |v_jd| / sum_j P_rj: the oracle's own attention with
    every dequantised V value replaced by its magnitude (same Q, K and
    weights).  It bounds how much rounding the weights or V can move an output
    element.  Magnitudes are taken on the codes: sign bit cleared for the
    floating-point formats, |code| for INT8."""
    a = oracle.Cache(oc.dtype, oc.num_blocks, oc.block_size, oc.Hkv, oc.D,
                     oc.k_scale, oc.v_scale, scale_per_layer=oc.scale_per_layer)
    a.k_cache[:] = oc.k_cache
    if oc.k_scale_tok is not None:
        a.k_scale_tok[:] = oc.k_scale_tok
        a.v_scale_tok[:] = oc.v_scale_tok
    a.v_cache[:] = oracle.code_magnitude(oc.dtype, oc.v_cache)
    return run_oracle(case, a, rows=rows)[0]


def half_ulp16(x: np.ndarray) -> np.ndarray:
    """Half the spacing of fp16 numbers at |x|: the largest error of rounding
    x to fp16 (2^-25 in the subnormal range)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -14)))
    return np.exp2(e - 11.0)


def derived_bound(ref: np.ndarray, a_abs: np.ndarray, v_rounded: bool) -> np.ndarray:
    """Per-element bound of an fp16 output computed with fp16 weights P and
    fp16 values, FP32 state (derivation in the design notes, section 3):
      half an fp16 ulp of the output (its final rounding)
      + 2^-11 * A   (P rounded to fp16: relative error <= 2^-11 per weight)
      + 2^-11 * A   (fp32 scores and exponentials: the weights' relative error
                     from score rounding, allowed one more fp16 unit)
      + 2^-11 * A   (INT8 only: V-hat = fp16(code * scale) rounded once)
    with A = abs_value_oracle(...).  The stated bound 2e-3 applies wherever it
    is the larger one."""
    k = 2.0 + (1.0 if v_rounded else 0.0)
    return np.maximum(MAX_ABS_TOL, half_ulp16(ref) + k * 2.0 ** -11 * a_abs)


def assert_close(out_gpu: torch.Tensor, ref: np.ndarray, lse_gpu=None, lse_ref=None,
                 max_abs=MAX_ABS_TOL, rel_l2=REL_L2_TOL, what="", bound=None):
    """Strict form (bound None): the stated tolerance, max |err| <= 2e-3 and
    relative L2 <= 1e-3 over the tensor.  With `bound` (per element, from
    derived_bound), each element is held to max(2e-3, its derived bound);
    relative L2 stays 1e-3 everywhere."""
    g = out_gpu.double().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    tol = max_abs if bound is None else np.maximum(max_abs, bound)
    over = err - tol
    mx = float(over.max()) if err.size else -1.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref) / den) if den > 0 else float(np.linalg.norm(g))
    at = np.unravel_index(over.argmax(), err.shape) if err.size else None
    assert mx <= 0, f"{what}: |err| {float(err[at]):.3e} above its bound by {mx:.3e} at {at}"
    mx = float(err.max()) if err.size else 0.0
    assert rel <= rel_l2, f"{what}: rel L2 {rel:.3e} > {rel_l2}"
    if lse_gpu is not None and lse_ref is not None:
        lg = lse_gpu.double().numpy()
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lg), fin), f"{what}: lse finiteness differs"
        if fin.any():
            le = float(np.abs(lg[fin] - lse_ref[fin]).max())
            assert le <= LSE_TOL, f"{what}: lse err {le:.3e}"
    return mx, rel


def assert_matches_oracle(case: synth.Case, oc: oracle.Cache, out, lse, ref, ref_lse, what=""):
    """Strict tolerance when no element can need more; otherwise each element
    against max(2e-3, its derived bound)."""
    a_abs = abs_value_oracle(case, oc)
    bound = derived_bound(ref, a_abs, case.spec.kv_dtype == synth.INT8)
    strict = bool(np.all(bound <= MAX_ABS_TOL))
    return assert_close(out, ref, lse, ref_lse, what=what + (" (strict)" if strict else ""),
                        bound=None if strict else bound)
