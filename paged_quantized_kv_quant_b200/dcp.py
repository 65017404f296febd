"""Sequence-sharded (decode-context-parallel) decode across ranks.

Source: "ReVolta" PyPI page, "Hardware" and the launch flags (TP4 + DCP2,
``--decode-context-parallel-size 2``): each rank keeps part of every
sequence's KV blocks.  Each rank attends over its own keys with
``paged_attn_decode`` given its queries' local positions (``query_pos``), the
ranks exchange their (output, log-sum-exp) pairs with one all-gather, and
``merge_attn_states`` combines them into the attention over all keys.

This module is plumbing only: the all-gather is ``torch.distributed`` (NCCL
between GPUs; any backend works, the tests use gloo on the CPU) and every
step of the arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def gather_states(out: torch.Tensor, lse: torch.Tensor,
                  group: Optional[dist.ProcessGroup] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gathers every rank's partial result: out [..., D] and lse [...] ->
    ([world, ...same], [world, ...same]), stacked in rank order."""
    world = dist.get_world_size(group)
    outs = [torch.empty_like(out) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(outs, out.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return torch.stack(outs), torch.stack(lses)


def paged_attn_decode_dcp(cache, q: torch.Tensor, block_table: torch.Tensor,
                          context_lens: torch.Tensor, query_pos: torch.Tensor,
                          max_context_len: int, softmax_scale: float,
                          group: Optional[dist.ProcessGroup] = None) -> Tuple[torch.Tensor,
                                                                              torch.Tensor]:
    """Decode over this rank's share of the keys, exchange, merge.

    block_table / context_lens / query_pos describe this rank's keys only
    (local block ids, local key counts, each query's last visible local key).
    Returns the merged output fp16 [B][q_len][Hq][D] and lse fp32 [B][q_len][Hq],
    identical on every rank."""
    from . import merge_attn_states, paged_attn_decode
    B, ql, Hq, _ = q.shape
    lse = torch.empty((B, ql, Hq), dtype=torch.float32, device=q.device)
    out = paged_attn_decode(cache, q, block_table, context_lens, max_context_len,
                            softmax_scale, lse=lse, query_pos=query_pos)
    parts_out, parts_lse = gather_states(out, lse, group)
    return merge_attn_states(parts_out, parts_lse)
