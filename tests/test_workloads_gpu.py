"""The five named workloads at full size, in the launch configuration the
benchmark times: KV codes bit-exact over the whole cache; attention outputs
against the FP64 oracle under the stated bound (max |err| <= 2e-3, relative L2
<= 1e-3) on every row of the decode workloads and on dense row sets of the two
prefills (both ends of every 128-row query tile); properties that hold at any
size on all rows."""
import numpy as np
import pytest
import torch

import paged_quantized_kv_quant_b200 as pk
import synth
from pkvq_testutil import (assert_close, assert_codes_equal, gpu_cache, oracle_cache, run_gpu,
                           run_oracle)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _tile_rows(case, every_head_tiles, one_head_tiles, last_tokens, n_random, seed=0):
    """(token, head) rows of a prefill chunk: every head of the first and last
    token of the query tiles in `every_head_tiles`, one random head of the
    first and last token of the tiles in `one_head_tiles`, every head of the
    last `last_tokens` tokens, plus n_random random rows.  A query tile is the
    128 packed rows (128 / G tokens) one CTA owns."""
    s = case.spec
    G = s.num_q_heads // s.num_kv_heads
    tpt = 128 // G
    q_len = s.q_lens[0]
    rng = np.random.default_rng(seed)
    rows = set()
    for t in every_head_tiles:
        for tok in (t * tpt, min(q_len, (t + 1) * tpt) - 1):
            rows.update((tok, h) for h in range(s.num_q_heads))
    for t in one_head_tiles:
        for tok in (t * tpt, min(q_len, (t + 1) * tpt) - 1):
            rows.add((tok, int(rng.integers(s.num_q_heads))))
    for tok in range(q_len - last_tokens, q_len):
        rows.update((tok, h) for h in range(s.num_q_heads))
    target = len(rows) + n_random
    while len(rows) < target:
        rows.add((int(rng.integers(q_len)), int(rng.integers(s.num_q_heads))))
    return np.array(sorted(rows), np.int32)


def _rows_for(n, case):
    """Rows compared with the oracle: all of workloads 1, 2 and 5; for the two
    prefills, the rows that see the fewest and the most keys of every query
    tile, the chunk's last tokens and a random sample (the oracle takes
    minutes per full prefill)."""
    if n in (1, 2, 5):
        return None
    G = case.spec.num_q_heads // case.spec.num_kv_heads
    ntile = (case.spec.q_lens[0] * G + 127) // 128
    if n == 3:       # 8K causal: every head of both ends of all 512 query tiles
        return _tile_rows(case, range(ntile), [], 128, 2048, seed=3)
    # 8K over a 120K prefix: every head at both ends of 32 spread tiles, one
    # head at both ends of every tile
    spread = np.linspace(0, ntile - 1, 32).round().astype(int).tolist()
    return _tile_rows(case, spread, range(ntile), 16, 512, seed=4)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5])
def test_workload_full_size(n):
    case = synth.make_case(synth.workload(n))
    cache = gpu_cache(case)
    oc = oracle_cache(case)
    assert_codes_equal(cache, oc, case)
    out, lse = run_gpu(case, cache)
    assert pk.device_status() == 0
    # properties on every row: finite, and each output lies in the convex hull
    # of the dequantised values, i.e. within the largest |v| of its KV head
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    s = case.spec
    if s.kv_dtype == synth.FP8_E4M3:
        vmax = torch.tensor(oc.v_scale).double() * 448.0
    else:
        vmax = torch.full((s.num_kv_heads,), float(case.v.abs().max()) * 1.01)
    G = s.num_q_heads // s.num_kv_heads
    bound = vmax.repeat_interleave(G).view(1, -1, 1)
    assert (out.double().abs() <= bound + 1e-3).all()
    rr = _rows_for(n, case)
    if rr is None:
        ref, ref_lse = run_oracle(case, oc)
        assert_close(out, ref, lse, ref_lse, what=f"workload {n}, every row")
    else:
        ref, ref_lse = run_oracle(case, oc, rows=rr)
        g = out[rr[:, 0], rr[:, 1]]
        gl = lse[rr[:, 0], rr[:, 1]]
        assert_close(g, ref, gl, ref_lse, what=f"workload {n}, {len(rr)} rows")
