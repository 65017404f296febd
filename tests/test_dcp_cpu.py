"""Sequence-sharded decode on two gloo ranks (CPU only).

Each rank takes its share of every sequence's blocks (block j to rank
j % world, synth.dcp_shard), computes the FP64 oracle's attention over its
own keys at its queries' local positions, and the ranks exchange their
(output, log-sum-exp) pairs with the package's all-gather helper.  Merged
with the oracle's merge_states, the result must equal the oracle's attention
over all keys: this checks the partition, the local positions and the
exchange step that the GPU path uses between its decode and merge kernels."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.join(os.path.dirname(__file__), "..")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _rank_main(rank, world, port, dtype, out):
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    from paged_quantized_kv_quant_b200.dcp import gather_states
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = synth.CaseSpec("decode", dtype, 8, 2, [301, 16, 5, 1000], [5] * 4,
                              seed=50 + rank * 0)   # every rank builds the same case
        case = synth.make_case(spec)
        oc = oracle.Cache(dtype, case.num_blocks, 16, 2, 128,
                          None if case.k_scale is None else case.k_scale.numpy(),
                          None if case.v_scale is None else case.v_scale.numpy())
        oc.write(_bits(case.k), _bits(case.v), case.slot_mapping.numpy())
        sh = synth.dcp_shard(case, world, rank)
        o, l, _ = oracle.paged_attention(oc, _bits(case.q), case.cu_seqlens_q.numpy(),
                                         sh.context_lens.numpy(), sh.block_table.numpy(),
                                         case.softmax_scale, query_pos=sh.query_pos.numpy())
        parts_o, parts_l = gather_states(torch.from_numpy(o), torch.from_numpy(l))
        mo, ml = oracle.merge_states(parts_o.numpy().reshape(world, -1, 128),
                                     parts_l.numpy().reshape(world, -1))
        full, full_lse, _ = oracle.paged_attention(
            oc, _bits(case.q), case.cu_seqlens_q.numpy(), case.context_lens.numpy(),
            case.block_table.numpy(), case.softmax_scale)
        out[rank] = (float(np.abs(mo - full.reshape(-1, 128)).max()),
                     float(np.abs(ml - full_lse.reshape(-1)).max()),
                     int(sh.context_lens.sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype", [0, 1])
def test_two_rank_sharded_decode_merges_to_full_attention(dtype):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, dtype, out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        eo, el, _ = res[rank]
        assert eo < 1e-12 and el < 1e-12
    # the ranks hold disjoint shares that cover every key
    assert res[0][2] + res[1][2] == 301 + 16 + 5 + 1000
