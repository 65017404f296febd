"""GPU parity of the merge of per-part attention results
(pkvq_merge_attn_states) and of the whole-block copy between cache pools
(pkvq_kv_copy_blocks), against the oracle's merge_states and copy_blocks."""
import numpy as np
import pytest
import torch

import oracle
import paged_quantized_kv_quant_b200 as pk
import synth
from pkvq_testutil import MAX_ABS_TOL, gpu_cache, half_ulp16, oracle_cache, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("parts,rows", [(1, 7), (2, 1000), (3, 33), (8, 64), (33, 50),
                                        (64, 9)])
def test_merge_matches_oracle(parts, rows):
    po, pl = synth.attention_parts(parts, rows, seed=parts)
    out, lse = pk.merge_attn_states(po.cuda(), pl.cuda())
    torch.cuda.synchronize()
    ref, ref_lse = oracle.merge_states(po.double().numpy(), pl.double().numpy())
    g = out.cpu().double().numpy()
    # FP32 weights and sums of fp16 inputs: the output's fp16 rounding plus a
    # few fp32 units of the largest part
    bound = half_ulp16(ref) + 2.0 ** -18 * np.abs(po.double().numpy()).max(0)
    assert np.all(np.abs(g - ref) <= np.maximum(bound, 1e-6)), float(np.abs(g - ref).max())
    fin = np.isfinite(ref_lse)
    gl = lse.cpu().double().numpy()
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.all(g[~fin] == 0)
    assert np.allclose(gl[fin], ref_lse[fin], atol=1e-5, rtol=0)


@pytest.mark.parametrize("dtype", [synth.FP8_E4M3, synth.INT8, synth.FP8_E5M2, synth.FP16])
@pytest.mark.parametrize("host_tier", [False, True])
def test_copy_blocks_out_and_back(dtype, host_tier):
    spec = synth.CaseSpec("decode", dtype, 8, 2, [1000, 77], [1, 1], block_size=16, seed=60)
    case = synth.make_case(spec)
    src = gpu_cache(case)
    oc = oracle_cache(case)
    nb = case.num_blocks
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(1)).to(torch.int32)
    pairs_out = torch.stack([torch.arange(nb, dtype=torch.int32), perm], 1)
    # the tier: device memory, or pinned host memory the GPU addresses directly
    tier = pk.PagedKVCache.allocate(dtype, nb, 16, 2, device="cpu" if host_tier else "cuda",
                                    pin_host=host_tier, k_scale=case.k_scale,
                                    v_scale=case.v_scale)
    pk.kv_copy_blocks(tier, src, pairs_out.cuda())
    torch.cuda.synchronize()
    names = ("k_cache", "v_cache") + (("k_scale_tok", "v_scale_tok")
                                      if dtype == synth.INT8 else ())
    # a copy moves every byte of a block, never-written slots included
    for name in names:   # compared as bits: the poison fill is a NaN pattern
        g = getattr(tier, name).cpu().contiguous().view(torch.uint8)
        assert torch.equal(g[perm.long()], getattr(src, name).cpu().contiguous()
                           .view(torch.uint8)), name
    # and agrees with the oracle's copy on every slot that holds a token
    ot = oracle.Cache(dtype, nb, 16, 2, 128,
                      None if case.k_scale is None else case.k_scale.numpy(),
                      None if case.v_scale is None else case.v_scale.numpy())
    oracle.copy_blocks(oc, ot, pairs_out.numpy())
    sm = case.slot_mapping.numpy()
    blk, off = perm.numpy()[sm // 16], sm % 16       # where each token landed
    for name in names:
        g = getattr(tier, name).cpu().contiguous().view(torch.uint8).numpy()
        o = getattr(ot, name).view(np.uint8).reshape(g.shape)
        assert np.array_equal(g[blk, :, off], o[blk, :, off]), name
    # back into a fresh device pool at the tier's ids: attention through the
    # permuted table equals attention through the original one, bit for bit
    back = pk.PagedKVCache.allocate(dtype, nb, 16, 2, k_scale=case.k_scale,
                                    v_scale=case.v_scale)
    pairs_back = torch.stack([perm, perm], 1)
    pk.kv_copy_blocks(back, tier, pairs_back.cuda())
    out1, lse1 = run_gpu(case, src)
    case.block_table = perm[case.block_table.long()].to(torch.int32)
    out2, lse2 = run_gpu(case, back)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)
    assert pk.device_status() == 0
