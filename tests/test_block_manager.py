"""Host block manager (C++ in libpa) against a separate Python model, invariants, the
pages' worked examples, and the logical token streams it produces through the oracle's
cache operations (no GPU)."""
import numpy as np
import pytest

import oracle
import paged_kv_cache_441_b200 as pa
from oracle import oracle_np
from tests.bm_model import Model, NoBlocks
from tests.pins import read_golden


def _invariants(bm, model):
    assert bm.num_free_blocks == len(model.free_ids)
    assert bm.num_free_cpu_blocks == len(model.cpu_free)
    refs = [0] * len(model.ref)
    cpu_refs = [0] * len(model.cpu_ref)
    for sid, (blocks, n) in model.seqs.items():
        assert len(blocks) == -(-n // model.bs)
        assert bm.is_swapped(sid) == (sid in model.on_cpu)
        if model.window:  # every page of the window is held
            lo = max(n - model.window, 0)
            assert all(b is not None for b in blocks[lo // model.bs:])
        for b in blocks:
            if b is None:
                continue
            if sid in model.on_cpu:
                cpu_refs[b] += 1
            else:
                refs[b] += 1
    assert refs == model.ref and cpu_refs == model.cpu_ref
    for b, r in enumerate(model.ref):
        assert bm.refcount(b) == r
    assert abs(bm.usage_ratio - (1 - len(model.free_ids) / len(model.ref))) < 1e-12


def test_pages_worked_examples():
    g = {k: kv for k, kv in read_golden() if k in ("blocks_needed", "pool_tokens")}
    ex = g["blocks_needed"]
    assert pa.blocks_needed(int(ex["seq_len"]), int(ex["block_size"])) == int(ex["expect"])
    pool = g["pool_tokens"]
    nb, bs, cap = int(pool["num_blocks"]), int(pool["block_size"]), int(pool["expect"])
    bm = pa.BlockManager(nb, bs)
    assert bm.can_allocate(cap) and not bm.can_allocate(cap + 1)
    bm.allocate(1, 3200)
    assert bm.num_free_blocks == nb - 7
    bm.allocate(2, cap - 7 * bs)  # the rest of the pool, exactly
    assert bm.num_free_blocks == 0 and bm.usage_ratio == 1.0
    with pytest.raises(pa.PAError):
        bm.allocate(3, 1)
    bm.free(1)
    assert bm.num_free_blocks == 7


def _sharing_group(model, sid):
    """sid and every sequence that shares a block with it (transitively), same pool."""
    cpu = sid in model.on_cpu
    group, todo = {sid}, [sid]
    while todo:
        blocks = set(model.seqs[todo.pop()][0]) - {None}
        for other, (ob, _) in model.seqs.items():
            if other not in group and (other in model.on_cpu) == cpu and blocks & set(ob):
                group.add(other)
                todo.append(other)
    return sorted(group)


@pytest.mark.parametrize("seed,window", [(s, 0) for s in range(6)] +
                         [(6, 1), (7, 5), (8, 16), (9, 33)])
def test_random_operations_match_model(seed, window):
    rng = np.random.default_rng(seed)
    nb, bs = int(rng.integers(8, 64)), int(rng.choice([1, 2, 4, 16]))
    ncpu = int(rng.integers(4, 40))
    bm, model = pa.BlockManager(nb, bs), Model(nb, bs, ncpu, window)
    bm.set_cpu_pool(ncpu)
    bm.set_sliding_window(window)
    next_id = 0
    for step in range(300):
        op = rng.choice(["alloc", "fork", "free", "append", "swap_out", "swap_in"],
                        p=[0.22, 0.18, 0.13, 0.35, 0.06, 0.06])
        on_gpu = [s for s in model.seqs if s not in model.on_cpu]
        on_cpu = [s for s in model.seqs if s in model.on_cpu]
        if op in ("swap_out", "swap_in"):
            pool = on_gpu if op == "swap_out" else on_cpu
            if pool:
                group = _sharing_group(model, int(rng.choice(pool)))
                try:
                    want = model.move(group, op == "swap_out")
                    got = (bm.swap_out if op == "swap_out" else bm.swap_in)(group)
                    assert [tuple(x) for x in got.tolist()] == want
                except NoBlocks:
                    with pytest.raises(pa.PAError):
                        (bm.swap_out if op == "swap_out" else bm.swap_in)(group)
            _invariants(bm, model)
            continue
        live = on_gpu if op in ("fork", "append") else list(model.seqs)
        if op == "alloc":
            n = int(rng.integers(0, 3 * bs + 2))
            try:
                model.allocate(next_id, n)
                bm.allocate(next_id, n)
            except NoBlocks:
                with pytest.raises(pa.PAError):
                    bm.allocate(next_id, n)
            next_id += 1
        elif op == "fork" and live:
            p = int(rng.choice(live))
            model.fork(p, next_id)
            bm.fork(p, next_id)
            next_id += 1
        elif op == "free" and live:
            s = int(rng.choice(live))
            model.free(s)
            bm.free(s)
        elif op == "append" and live:
            ids = [int(x) for x in rng.permutation(live)[: int(rng.integers(1, len(live) + 1))]]
            try:
                slots, pairs = model.append(ids)
                s2, p2 = bm.append_slots(ids)
                assert s2.tolist() == slots and [tuple(x) for x in p2.tolist()] == pairs
                assert len(set(slots)) == len(slots)  # no two writers share a slot
            except NoBlocks:
                with pytest.raises(pa.PAError):
                    bm.append_slots(ids)
        _invariants(bm, model)
        for sid, (blocks, n) in model.seqs.items():
            assert bm.seq_len(sid) == n
            if sid in model.on_cpu:
                with pytest.raises(pa.PAError):
                    bm.block_tables([sid], max(len(blocks), 1))
                continue
            bt, cl = bm.block_tables([sid], max(len(blocks), 1))
            assert bt[0, : len(blocks)].tolist() == [-1 if b is None else b for b in blocks]
            assert cl[0] == n
            for pos in range(n):
                blk = blocks[pos // bs]
                assert bm.slot(sid, pos) == (-1 if blk is None else blk * bs + pos % bs)


def test_errors_change_nothing():
    bm = pa.BlockManager(4, 4)
    bm.allocate(7, 6)  # 2 blocks
    bm.fork(7, 8)
    for bad in (lambda: bm.allocate(7, 1), lambda: bm.fork(7, 8), lambda: bm.fork(99, 1),
                lambda: bm.free(99), lambda: bm.append_slots([7, 7]),
                lambda: bm.append_slots([42]), lambda: bm.block_tables([7], 1)):
        with pytest.raises(pa.PAError):
            bad()
    # 2 free blocks; 7 and 8 share a partial block: 8 appends need a copy each -> 2 blocks
    # for the pair, then every further block boundary needs more: exhaust, state unchanged
    before = (bm.num_free_blocks, bm.seq_len(7), bm.seq_len(8))
    bm.allocate(9, 8)  # takes the last 2 blocks
    with pytest.raises(pa.PAError):
        bm.append_slots([7, 8])  # 7 needs a private copy of the shared block: none left
    assert (bm.seq_len(7), bm.seq_len(8)) == before[1:]
    bm.free(9)
    slots, pairs = bm.append_slots([7, 8])
    assert len(pairs) == 1 and pairs[0, 0] == bm.block_tables([8], 2)[0][0, 1]


def test_parallel_sampling_copy_on_write_counts():
    """64 prompts of 1000 tokens, 8 samples each: the first append copies the shared
    partial block for 7 samples of every group (448 pairs); the 8th writes in place."""
    bs = 16
    bm = pa.BlockManager(64 * (63 + 7) + 10, bs)
    ids = []
    for g in range(64):
        bm.allocate(g * 8, 1000)
        for j in range(1, 8):
            bm.fork(g * 8, g * 8 + j)
        ids += list(range(g * 8, g * 8 + 8))
    assert bm.refcount(bm.block_tables([0], 63)[0][0, 62]) == 8
    slots, pairs = bm.append_slots(ids)
    assert pairs.shape == (448, 2)
    assert len(set(slots.tolist())) == 512 and all(int(s) % bs == 1000 % bs for s in slots)
    slots2, pairs2 = bm.append_slots(ids)
    assert pairs2.shape == (0, 2)


@pytest.mark.parametrize("seed,window", [(0, 0), (1, 0), (2, 0), (3, 6), (4, 20)])
def test_append_slots_cow_reports_the_same_copies_per_sequence(seed, window):
    """Two managers driven by the same operations, one appending with pairs and one with
    the per-sequence copy list: the same slots and the same copies; each listed copy names
    the sequence's last block, the rows filled before the token, and the source the pair
    names; the token's row is the first one not copied."""
    rng = np.random.default_rng(seed)
    nb, bs = int(rng.integers(16, 64)), int(rng.choice([2, 4, 8, 16]))
    a, b = pa.BlockManager(nb, bs), pa.BlockManager(nb, bs)
    a.set_sliding_window(window)
    b.set_sliding_window(window)
    live, next_id, copies = [], 0, 0
    for step in range(400):
        op = rng.choice(["alloc", "fork", "free", "append"], p=[0.2, 0.25, 0.1, 0.45])
        if op == "alloc":
            n = int(rng.integers(1, 3 * bs + 2))
            try:
                a.allocate(next_id, n)
            except pa.PAError:
                with pytest.raises(pa.PAError):
                    b.allocate(next_id, n)
            else:
                b.allocate(next_id, n)
                live.append(next_id)
            next_id += 1
        elif op == "fork" and live:
            p = int(rng.choice(live))
            a.fork(p, next_id)
            b.fork(p, next_id)
            live.append(next_id)
            next_id += 1
        elif op == "free" and live:
            sid = int(rng.choice(live))
            a.free(sid)
            b.free(sid)
            live.remove(sid)
        elif op == "append" and live:
            ids = [int(x) for x in rng.permutation(live)[: int(rng.integers(1, len(live) + 1))]]
            try:
                slots, pairs = a.append_slots(ids)
            except pa.PAError:
                with pytest.raises(pa.PAError):
                    b.append_slots_cow(ids)
                continue
            slots2, cow = b.append_slots_cow(ids)
            assert slots2.tolist() == slots.tolist()
            assert cow.shape == (len(ids), 3) and cow.dtype == np.int32
            width = max(b.seq_len(i) for i in ids) // bs + 1
            bt, cl = b.block_tables(ids, width)
            named = []
            for i, (src, lb, rows) in enumerate(cow.tolist()):
                if src < 0:
                    assert (lb, rows) == (0, 0)
                    continue
                L = int(cl[i])
                assert lb == (L - 1) // bs and rows == (L - 1) % bs and rows > 0
                assert int(slots[i]) == int(bt[i, lb]) * bs + rows  # the row past the copy
                named.append((src, int(bt[i, lb])))
            assert named == [tuple(x) for x in pairs.tolist()]
            copies += len(named)
    assert copies > 0


@pytest.mark.parametrize("window", [0, 5, 8])
def test_logical_token_streams_through_tables(window):
    """Drive the oracle's cache write / block copy with the manager through prompts,
    forks, appends, swaps and frees: every live sequence's K, gathered through its
    table, must equal the tokens it logically holds (under a sliding window: its last
    `window` tokens, with the pages before them given back)."""
    rng = np.random.default_rng(3)
    nb, hkv, bs, d = 96, 2, 4, 8
    bm = pa.BlockManager(nb, bs)
    bm.set_cpu_pool(40)
    bm.set_sliding_window(window)
    model = None
    kc = np.zeros((nb, hkv, bs, d), np.uint16)
    vc = np.zeros_like(kc)
    kh = np.zeros((40, hkv, bs, d), np.uint16)  # host pool
    vh = np.zeros_like(kh)
    swapped = set()
    logical = {}
    next_id, counter = 0, 1

    def tok():
        nonlocal counter
        counter += 1
        return np.full((1, hkv, d), counter % 60000, np.uint16)

    for step in range(160):
        live = [s for s in logical if s not in swapped]
        r = rng.random()
        if r > 0.9 and (live or swapped):
            # swap a whole sharing group out, or a swapped group back in
            out = (not swapped) or (live and rng.random() < 0.5)
            pool = live if out else sorted(swapped)
            seed_id = int(rng.choice(pool))
            group = {seed_id}
            tabs = {}
            for sid in pool:
                L = len(logical[sid])
                if out:
                    tabs[sid] = set(bm.block_tables([sid], max(-(-L // bs), 1))[0][0].tolist()) - {-1}
            if out:
                changed = True
                while changed:
                    changed = False
                    for sid in pool:
                        if sid not in group and any(tabs[sid] & tabs[g] for g in group):
                            group.add(sid)
                            changed = True
            else:
                group = set(swapped)  # bring back everything that is out
            try:
                pairs = (bm.swap_out if out else bm.swap_in)(sorted(group))
            except pa.PAError:
                continue
            for a, b in pairs:
                if out:
                    kh[b], vh[b] = kc[a], vc[a]
                else:
                    kc[b], vc[b] = kh[a], vh[a]
            swapped = (swapped | group) if out else (swapped - group)
        elif r < 0.15 or not live:
            n = int(rng.integers(1, 11))
            if bm.can_allocate(n):
                bm.allocate(next_id, n)
                toks = [tok() for _ in range(n)]
                sm = np.array([bm.slot(next_id, i) for i in range(n)], np.int64)  # -1: skip
                oracle.kv_write(np.concatenate(toks), np.concatenate(toks), sm, kc, vc)
                logical[next_id] = toks
                next_id += 1
        elif r < 0.3:
            p = int(rng.choice(live))
            bm.fork(p, next_id)
            logical[next_id] = list(logical[p])
            next_id += 1
        elif r < 0.4:
            s = int(rng.choice(list(logical)))
            bm.free(s)
            del logical[s]
            swapped.discard(s)
        else:
            ids = [int(x) for x in rng.permutation(live)]
            try:
                slots, pairs = bm.append_slots(ids)
            except pa.PAError:
                continue
            oracle.copy_blocks(kc, vc, pairs)  # copies first, then the new tokens
            toks = [tok() for _ in ids]
            oracle.kv_write(np.concatenate(toks), np.concatenate(toks), slots, kc, vc)
            for s, t in zip(ids, toks):
                logical[s].append(t)
        for s, toks in logical.items():
            if s in swapped:
                continue
            L = len(toks)
            bt, cl = bm.block_tables([s], max(-(-L // bs), 1))
            assert cl[0] == L
            lo = L - window if 0 < window < L else 0
            assert np.all(bt[0, lo // bs:-(-L // bs)] >= 0)  # earlier pages: -1 once given back
            for g in range(hkv):
                got = oracle_np.gather_positions(kc, bt[0], lo, L, g)
                want = np.concatenate([t[:, g] for t in toks[lo:]])
                assert np.array_equal(got, want), (step, s)


def test_closed_manager_refuses_calls():
    bm = pa.BlockManager(8, 16)
    bm.allocate(1, 20)
    bm.close()
    bm.close()  # idempotent
    with pytest.raises(pa.PAError, match="closed"):
        bm.allocate(2, 5)
    with pytest.raises(pa.PAError, match="closed"):
        _ = bm.num_free_blocks
