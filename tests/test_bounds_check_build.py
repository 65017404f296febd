"""The debug build: libpkvq_checked.so, compiled with PKVQ_BOUNDS_CHECK, whose
kernels check every block id and slot against the pool before touching it
and record a violation in the device status word instead of reading or
writing out of bounds.

CPU: the build compiles and exports the same C ABI.  GPU: with in-range
inputs only, the checked build gives bit-identical results to the release
build and a clean status word (the checks cost nothing when nothing is out
of range, and change no arithmetic)."""
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import paged_quantized_kv_quant_b200 as pk
import synth
from paged_quantized_kv_quant_b200 import build as pkbuild
from pkvq_testutil import gpu_cache, run_gpu


@pytest.fixture(scope="module")
def checked_path():
    return pkbuild.build(bounds_check=True)


def test_checked_build_exports_the_same_abi(checked_path):
    assert checked_path == pk.LIB_CHECKED_PATH and os.path.exists(checked_path)
    out = subprocess.run(["nm", "-D", "--defined-only", checked_path], capture_output=True,
                         text=True, check=True).stdout
    names = sorted({l.split()[-1] for l in out.splitlines() if " T " in l and "pkvq" in l})
    assert names == sorted(pk.EXPORTED)


CASES = [
    synth.CaseSpec("decode", synth.FP8_E4M3, 32, 4, [5000, 17, 300], [1] * 3, seed=70),
    synth.CaseSpec("decode", synth.INT8, 32, 4, [3000, 40], [5, 5], seed=71),
    synth.CaseSpec("decode", synth.FP16, 16, 2, [900], [2], block_size=32, seed=72),
    synth.CaseSpec("prefill", synth.FP8_E5M2, 16, 2, [700, 300], [300, 300], seed=73),
]


@pytest.mark.gpu
@pytest.mark.parametrize("spec", CASES, ids=lambda s: f"{s.kind}-{s.kv_dtype}")
def test_checked_build_matches_release_bit_for_bit(checked_path, spec):
    case = synth.make_case(spec)
    cache = gpu_cache(case)
    out_r, lse_r = run_gpu(case, cache)
    assert pk.device_status() == 0
    with pk.use_library(checked_path):
        cache_c = gpu_cache(case)          # written by the checked kv_write too
        assert torch.equal(cache_c.k_cache, cache.k_cache)
        assert torch.equal(cache_c.v_cache, cache.v_cache)
        out_c, lse_c = run_gpu(case, cache_c)
        assert pk.device_status() == 0     # the checked build's own status word
    assert torch.equal(out_r, out_c) and torch.equal(lse_r, lse_c)
    maps = open("/proc/self/maps").read()
    assert re.search(r"libpkvq_checked\.so", maps)
