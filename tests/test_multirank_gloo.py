"""N > 1 host path on CPU with the gloo backend (world size 2).

Decode and prefill shard with no exchange step: every sequence's attention depends only
on its own pages.  Each rank computes its share of the sequences with the CPU oracle, the
shares are gathered, and the result must equal the one-rank result exactly.  The
bench's max-over-ranks / sum-over-ranks aggregation is checked on the same group.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_path):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    import oracle
    from workloads import make_case
    case = make_case("shard", 41, 10, 8, 2, 32, 8,
                     lambda r: r.integers(1, 90, size=10).astype(np.int32), dtype="bf16",
                     poison=True)
    kc, vc = case.k_cache.copy(), case.v_cache.copy()
    oracle.kv_write(case.key, case.value, case.slot_mapping, kc, vc)
    mine = np.arange(rank, case.num_seqs, world)
    sel = np.array([(s, h) for s in mine for h in range(case.num_q_heads)], np.int32)
    part = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale,
                         case.dtype, sel=sel)
    gathered = [None] * world
    dist.all_gather_object(gathered, (sel.tolist(), part.tolist()))
    # prefill shards the same way: each rank takes whole sequences (its chunks' q rows,
    # renumbered into its own query_start_loc) and needs no other rank's data
    from workloads import make_prefill_case
    pc = make_prefill_case("shard_pf", 42, [(9, 9), (5, 30), (1, 12), (17, 17), (3, 3)], 8, 2,
                           32, 8, poison=True)
    pk, pv = pc.k_cache.copy(), pc.v_cache.copy()
    oracle.kv_write(pc.key, pc.value, pc.slot_mapping, pk, pv)
    pmine = np.arange(rank, pc.num_seqs, world)
    qsl = pc.query_start_loc
    rows = np.concatenate([np.arange(qsl[s], qsl[s + 1]) for s in pmine])
    my_qsl = np.concatenate([[0], np.cumsum([qsl[s + 1] - qsl[s] for s in pmine])]).astype(np.int32)
    ppart = oracle.prefill(pc.q[rows], pk, pv, pc.block_tables[pmine], pc.context_lens[pmine],
                           my_qsl, pc.scale, pc.dtype)
    pgathered = [None] * world
    dist.all_gather_object(pgathered, (rows.tolist(), ppart.tolist()))
    mx = bench.max_over_ranks(float(rank + 1) * 1.5, world)
    tot = bench.sum_over_ranks(float(rank + 1), world)
    if rank == 0:
        full = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale,
                             case.dtype)
        got = np.full_like(full, np.nan)
        for sel_r, part_r in gathered:
            for (s, h), row in zip(sel_r, part_r):
                got[s, h] = row
        pfull = oracle.prefill(pc.q, pk, pv, pc.block_tables, pc.context_lens, qsl, pc.scale,
                               pc.dtype)
        pgot = np.full_like(pfull, np.nan)
        for rows_r, part_r in pgathered:
            pgot[rows_r] = np.asarray(part_r)
        ok = bool(np.array_equal(got, full)) and bool(np.array_equal(pgot, pfull)) and \
            mx == 1.5 * world and tot == world * (world + 1) / 2
        with open(result_path, "w") as f:
            f.write("ok" if ok else f"mismatch mx={mx} tot={tot}")
    dist.barrier()
    dist.destroy_process_group()


def test_sequence_sharding_matches_single_rank(tmp_path):
    world = 2
    path = str(tmp_path / "result.txt")
    mp.spawn(_worker, args=(world, _free_port(), path), nprocs=world, join=True)
    assert open(path).read() == "ok"
