"""The five named workloads at full size, in the launch configuration the
benchmark times: KV codes bit-exact over the whole cache, attention outputs
compared with the FP64 oracle on sampled rows (every row where that is cheap),
plus properties that hold at any size on all rows."""
import numpy as np
import pytest
import torch

import paged_quantized_kv_quant_b200 as pk
import synth
from pkvq_testutil import (assert_close, assert_codes_equal, gpu_cache, oracle_cache, run_gpu,
                           run_oracle)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _sample_rows(case, n, seed=0):
    """(token, head) rows: first and last token of every sequence plus random."""
    s = case.spec
    cu = case.cu_seqlens_q.numpy()
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(len(s.q_lens)):
        if s.q_lens[b] == 0:
            continue
        for tok in (cu[b], cu[b + 1] - 1):
            for h in (0, s.num_q_heads - 1, int(rng.integers(s.num_q_heads))):
                rows.add((int(tok), int(h)))
    if s.kind == "prefill":
        # every head of the first 32 tokens of each chunk: the rows that see the
        # fewest keys, where fp16 rounding is least averaged out
        for b in range(len(s.q_lens)):
            for tok in range(int(cu[b]), min(int(cu[b + 1]), int(cu[b]) + 32)):
                for h in range(s.num_q_heads):
                    rows.add((tok, h))
    total = int(cu[-1])
    while len(rows) < n + (1024 if s.kind == "prefill" else 0):
        rows.add((int(rng.integers(total)), int(rng.integers(s.num_q_heads))))
    return np.array(sorted(rows), np.int32)


@pytest.mark.parametrize("n,rows", [(1, None), (2, None), (3, 384), (4, 96), (5, 40)])
def test_workload_full_size(n, rows):
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
    if rows is None:
        ref, ref_lse = run_oracle(case, oc)
        assert_close(out, ref, lse, ref_lse, what=f"workload {n}")
    else:
        rr = _sample_rows(case, rows)
        ref, ref_lse = run_oracle(case, oc, rows=rr)
        g = out[rr[:, 0], rr[:, 1]]
        gl = lse[rr[:, 0], rr[:, 1]]
        assert_close(g, ref, gl, ref_lse, what=f"workload {n} sampled")
