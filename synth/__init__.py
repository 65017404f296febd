"""Seeded synthetic inputs for paged 8-bit-KV attention.

This module is shared by the tests, the benchmark and the smoke check, and is
the only thing the GPU path and the CPU oracle have in common.  It holds no
attention or quantization arithmetic: it draws fp16 tensors from a seeded
``torch.Generator`` on the CPU, lays sequences out over a block pool through a
random block table, and computes the static per-KV-head calibration scale
(absmax / 448) that a caller hands to an FP8 cache.

Draw order (fixed, so every consumer sees the same bytes for a seed):
Q, K, V, then the outlier channels of K and of V, then the block permutation.

The five named workloads follow the shapes the pages describe: 8K and 131K
prompts and an 8,192-token chunked-prefill budget ("ReVolta" PyPI page,
"Measurements" and the launch flags), two 512K or four 256K contexts in one KV
pool ("ReVolta", first section), 1 + 4 verify positions (MTP4, same page) and
block size 16 (the serving stack's default).  No dataset is used anywhere.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

FP8_E4M3 = 0
INT8 = 1
FP8_E5M2 = 2
FP16 = 3
E4M3_MAX = 448.0
E5M2_MAX = 57344.0
FP8_MAX = {FP8_E4M3: E4M3_MAX, FP8_E5M2: E5M2_MAX}


def elem_bytes(kv_dtype: int) -> int:
    """Bytes per stored cache element."""
    return 2 if kv_dtype == FP16 else 1


@dataclass
class CaseSpec:
    kind: str                    # "decode" (uniform q_len) or "prefill" (varlen)
    kv_dtype: int                # FP8_E4M3 or INT8
    num_q_heads: int
    num_kv_heads: int
    context_lens: List[int]      # cached tokens per sequence, new ones included
    q_lens: List[int]            # new (query) tokens per sequence
    head_dim: int = 128
    block_size: int = 16
    pool_factor: float = 1.25    # pool blocks = ceil(factor * blocks used)
    outlier_frac: float = 0.0    # fraction of (head, d) channels scaled x8
    seed: int = 0
    name: str = ""
    scale_per_layer: bool = False  # FP8: one K and one V scale for all heads
    window: int = 0              # > 0: sliding window of that many keys


@dataclass
class Case:
    spec: CaseSpec
    q: torch.Tensor              # fp16 [total_q][Hq][D]
    k: torch.Tensor              # fp16 [total_tokens][Hkv][D]  (all cached tokens)
    v: torch.Tensor
    slot_mapping: torch.Tensor   # int32 [total_tokens]
    block_table: torch.Tensor    # int32 [B][max_blocks]
    context_lens: torch.Tensor   # int32 [B]
    cu_seqlens_q: torch.Tensor   # int32 [B+1]
    k_scale: Optional[torch.Tensor]  # fp32 [Hkv], or [1] per layer (FP8 only)
    v_scale: Optional[torch.Tensor]
    num_blocks: int
    softmax_scale: float
    token_offsets: torch.Tensor = field(default=None)  # int64 [B+1] into k/v

    @property
    def batch(self) -> int:
        return len(self.spec.context_lens)

    def new_token_rows(self) -> torch.Tensor:
        """Indices into k/v of every sequence's q_len newest tokens."""
        idx = []
        for s, (c, ql) in enumerate(zip(self.spec.context_lens, self.spec.q_lens)):
            base = int(self.token_offsets[s])
            idx.append(torch.arange(base + c - ql, base + c))
        return torch.cat(idx) if idx else torch.zeros(0, dtype=torch.int64)


def _randn_fp16(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.float16)


def _outliers(gen: torch.Generator, t: torch.Tensor, frac: float) -> None:
    """Scale round(frac * Hkv * D) (head, d) channels of t by 8, in place."""
    Hkv, D = t.shape[1], t.shape[2]
    n = int(round(frac * Hkv * D))
    if n <= 0:
        return
    ch = torch.randperm(Hkv * D, generator=gen)[:n]
    flat = t.view(t.shape[0], Hkv * D)
    flat[:, ch] = (flat[:, ch].float() * 8.0).to(torch.float16)


def per_head_absmax_scale(t: torch.Tensor, fmax: float = E4M3_MAX) -> torch.Tensor:
    """Static calibration: fp32 absmax over tokens and d, per KV head, / the
    format's largest finite value (448 for E4M3, 57344 for E5M2)."""
    amax = t.abs().amax(dim=(0, 2)).float()
    return amax / torch.tensor(fmax, dtype=torch.float32)


def per_layer_absmax_scale(t: torch.Tensor, fmax: float = E4M3_MAX) -> torch.Tensor:
    """One scale for all heads: fp32 absmax over everything / fmax, shape [1]."""
    amax = t.abs().amax().float().reshape(1)
    return amax / torch.tensor(fmax, dtype=torch.float32)


def make_case(spec: CaseSpec) -> Case:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(spec.seed)
    B = len(spec.context_lens)
    assert len(spec.q_lens) == B
    Hq, Hkv, D, bs = spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.block_size
    total_q = sum(spec.q_lens)
    total_tok = sum(spec.context_lens)
    q = _randn_fp16(gen, (total_q, Hq, D))
    k = _randn_fp16(gen, (total_tok, Hkv, D))
    v = _randn_fp16(gen, (total_tok, Hkv, D))
    if spec.outlier_frac > 0:
        _outliers(gen, k, spec.outlier_frac)
        _outliers(gen, v, spec.outlier_frac)
    nblk = [(c + bs - 1) // bs for c in spec.context_lens]
    used = sum(nblk)
    num_blocks = max(1, int(math.ceil(spec.pool_factor * used)))
    perm = torch.randperm(num_blocks, generator=gen).to(torch.int32)
    max_blocks = max(1, max(nblk) if nblk else 1)
    block_table = torch.zeros((B, max_blocks), dtype=torch.int32)
    slot_mapping = torch.empty(total_tok, dtype=torch.int32)
    offs = [0]
    p = 0
    for s in range(B):
        c = spec.context_lens[s]
        block_table[s, :nblk[s]] = perm[p:p + nblk[s]]
        p += nblk[s]
        j = torch.arange(c, dtype=torch.int64)
        slot_mapping[offs[-1]:offs[-1] + c] = (
            block_table[s, (j // bs)].to(torch.int64) * bs + j % bs).to(torch.int32)
        offs.append(offs[-1] + c)
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(spec.q_lens, dtype=torch.int32), 0)
    if spec.kv_dtype in FP8_MAX:
        fmax = FP8_MAX[spec.kv_dtype]
        cal = per_layer_absmax_scale if spec.scale_per_layer else per_head_absmax_scale
        n = 1 if spec.scale_per_layer else Hkv
        k_scale = cal(k, fmax) if total_tok else torch.ones(n)
        v_scale = cal(v, fmax) if total_tok else torch.ones(n)
    else:
        k_scale = v_scale = None
    softmax_scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
    return Case(spec=spec, q=q, k=k, v=v, slot_mapping=slot_mapping,
                block_table=block_table,
                context_lens=torch.tensor(spec.context_lens, dtype=torch.int32),
                cu_seqlens_q=cu, k_scale=k_scale, v_scale=v_scale,
                num_blocks=num_blocks, softmax_scale=softmax_scale,
                token_offsets=torch.tensor(offs, dtype=torch.int64))


# --------------------------------------------------------- named workloads --

def workload(n: int, seed: int = 0) -> CaseSpec:
    """The five named workloads, 1-based."""
    if n == 1:   # decode, 1 sequence, GQA 4, ctx 1024, pool = exactly the 64 blocks
        return CaseSpec("decode", FP8_E4M3, 8, 2, [1024], [1], pool_factor=1.0,
                        seed=seed, name="decode_b1_ctx1k_h8kv2_e4m3")
    if n == 2:   # decode batch 8 x 32K, outliers, pool 1.25x
        return CaseSpec("decode", FP8_E4M3, 32, 4, [32768] * 8, [1] * 8,
                        outlier_frac=0.01, seed=seed,
                        name="decode_b8_ctx32k_h32kv4_e4m3")
    if n == 3:   # causal prefill 8K, no prefix
        return CaseSpec("prefill", FP8_E4M3, 32, 4, [8192], [8192], seed=seed,
                        name="prefill_8k_h32kv4_e4m3")
    if n == 4:   # chunked prefill: 8K chunk over a 120K cached prefix
        return CaseSpec("prefill", FP8_E4M3, 32, 4, [131072], [8192], seed=seed,
                        name="chunked_prefill_8k_over_120k_h32kv4_e4m3")
    if n == 5:   # mixed long-context verify, INT8
        return CaseSpec("decode", INT8, 32, 4, [524288] * 2 + [262144] * 4, [5] * 6,
                        seed=seed, name="verify_q5_2x512k_4x256k_h32kv4_int8")
    raise ValueError(n)


def kv_read_bytes(spec: CaseSpec) -> int:
    """Algorithmic KV bytes one attention pass reads: every cached token's K
    and V elements for every KV head, plus the INT8 fp16 per-token scales."""
    tok = sum(spec.context_lens)
    per_tok = 2 * spec.num_kv_heads * spec.head_dim * elem_bytes(spec.kv_dtype)
    if spec.kv_dtype == INT8:
        per_tok += 2 * spec.num_kv_heads * 2
    return tok * per_tok


# ------------------------------------------------- sequence-sharded layout --

@dataclass
class Shard:
    """The keys one rank holds when a batch's cached blocks are dealt out
    over `world` ranks, block j of every sequence to rank j % world (the
    decode-context-parallel layout).  Keys keep their order: local key i of
    sequence s is in local block i // bs."""
    block_table: torch.Tensor    # int32 [B][max local blocks] (physical ids)
    context_lens: torch.Tensor   # int32 [B]: keys this rank holds
    query_pos: torch.Tensor      # int32 [total_q]: each query's position in
                                 # local key coordinates (last visible local key)


def dcp_shard(case: Case, world: int, rank: int) -> Shard:
    """Rank `rank`'s share of the case's blocks and the local positions of
    its queries (how many local keys precede or equal each query's global
    position, minus one)."""
    s = case.spec
    bs = s.block_size
    B = len(s.context_lens)
    tables, lens, qpos = [], [], []
    for b, (c, ql) in enumerate(zip(s.context_lens, s.q_lens)):
        nblk = (c + bs - 1) // bs
        mine = [j for j in range(nblk) if j % world == rank]
        tables.append([int(case.block_table[b, j]) for j in mine])
        # global positions of the local keys, in order
        gpos = [j * bs + o for j in mine for o in range(bs) if j * bs + o < c]
        lens.append(len(gpos))
        g = torch.tensor(gpos, dtype=torch.int64)
        for t in range(ql):
            p = c - ql + t
            qpos.append(int((g <= p).sum()) - 1)
    width = max(1, max((len(t) for t in tables), default=1))
    bt = torch.zeros((B, width), dtype=torch.int32)
    for b, t in enumerate(tables):
        if t:
            bt[b, :len(t)] = torch.tensor(t, dtype=torch.int32)
    return Shard(bt, torch.tensor(lens, dtype=torch.int32),
                 torch.tensor(qpos, dtype=torch.int32))


def useful_flops(spec: CaseSpec) -> int:
    """4 * D * Hq per visible (query, key) pair: QK^T and PV, 2 flops per MAC."""
    pairs = 0
    for c, ql in zip(spec.context_lens, spec.q_lens):
        # query t sees c - ql + t + 1 keys
        pairs += ql * (c - ql) + ql * (ql + 1) // 2
    return 4 * spec.head_dim * spec.num_q_heads * pairs


def attention_parts(parts: int, rows: int, head_dim: int = 128, seed: int = 0,
                    empty_frac: float = 0.2):
    """Per-part attention results over disjoint key sets, as the merge of a
    sequence-sharded decode receives them: outputs fp16 [parts][rows][D]
    ~ N(0,1), lse fp32 [parts][rows] ~ N(0, 3^2); a fraction of (part, row)
    entries saw no key (lse -inf), and the last row saw none in any part."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    out = _randn_fp16(gen, (parts, rows, head_dim))
    lse = torch.randn((parts, rows), generator=gen, dtype=torch.float32) * 3.0
    empty = torch.rand((parts, rows), generator=gen) < empty_frac
    lse[empty] = float("-inf")
    if rows:
        lse[:, -1] = float("-inf")
    return out, lse
