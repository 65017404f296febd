"""Host-side property test of the decode slot map (split_map.cuh).

A decode launch gives every (row group, KV head) C CTA slots; sequence b gets
max(1, ceil(n_b / bpc)) of them with bpc = split_blocks(...).  If the slots
the sequences need ever exceeded C, some split would have no CTA and its keys
would be silently dropped.  This test compiles a small host program against
the library's own split_blocks (nvcc; no GPU needed) and checks, on many
random batches, that the sum stays within C, that bpc honours its minimum and
granularity, and that every block is covered exactly once."""
import os
import random
import shutil
import subprocess

import pytest

ROOT = os.path.join(os.path.dirname(__file__), "..")
CSRC = os.path.join(ROOT, "paged_quantized_kv_quant_b200", "csrc")
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

DRIVER = r"""
#include "split_map.cuh"
#include <cstdio>
int main() {
    int B, C, minb, gran;
    while (scanf("%d %d %d %d", &B, &C, &minb, &gran) == 4) {
        long long total = 0; int longest = 0;
        static int n[5000];
        for (int i = 0; i < B; ++i) { scanf("%d", &n[i]); total += n[i]; if (n[i] > longest) longest = n[i]; }
        printf("%d\n", pkvq::split_blocks(total, C, B, longest, minb, gran));
    }
    return 0;
}
"""


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    if not os.path.exists(NVCC):
        pytest.skip("nvcc not found")
    d = tmp_path_factory.mktemp("splitmap")
    src = d / "drv.cu"
    src.write_text(DRIVER)
    exe = d / "drv"
    subprocess.run([NVCC, "-std=c++17", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    return str(exe)


def _cases():
    rng = random.Random(7)
    out = []
    for _ in range(400):
        B = rng.choice([1, 2, 3, 8, 31, 32, 33, 64, 200])
        kind = rng.random()
        if kind < 0.3:
            n = [rng.randint(0, 40) for _ in range(B)]          # short, some empty
        elif kind < 0.6:
            n = [rng.choice([0, 1, 16384, 32768, 2048]) for _ in range(B)]
        else:
            n = [rng.randint(0, 70000) for _ in range(B)]
        C = rng.choice([B, B + 1, 2 * B, 37, 111, 148, 296, 444, 1000])
        C = max(C, B)                      # the planner never gives fewer slots than sequences
        gran = rng.choice([1, 1, 2, 4])
        minb = rng.choice([1, 12, 16]) * gran
        out.append((B, C, minb, gran, n))
    return out


def test_slots_fit_and_cover(driver):
    cases = _cases()
    inp = "".join(f"{B} {C} {m} {g} " + " ".join(map(str, n)) + "\n" for B, C, m, g, n in cases)
    res = subprocess.run([driver], input=inp, capture_output=True, text=True, check=True)
    bpcs = [int(x) for x in res.stdout.split()]
    assert len(bpcs) == len(cases)
    for (B, C, minb, gran, n), bpc in zip(cases, bpcs):
        assert bpc >= 1 and bpc % gran == 0
        if C > B:
            assert bpc >= minb
        slots = [max(1, -(-x // bpc)) for x in n]
        assert sum(slots) <= C, (B, C, minb, gran, bpc)
        for x, s in zip(n, slots):
            # the splits [k * bpc, min(n, (k + 1) * bpc)) cover 0..n-1 once
            covered = sum(max(0, min(x, (k + 1) * bpc) - k * bpc) for k in range(s))
            assert covered == x


def test_one_slot_per_sequence_when_c_equals_b(driver):
    inp = "3 3 12 1 5 100 7\n"
    res = subprocess.run([driver], input=inp, capture_output=True, text=True, check=True)
    assert int(res.stdout.split()[0]) == 100
