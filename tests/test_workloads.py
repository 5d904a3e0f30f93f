"""Structure of the seeded synthetic workloads (no GPU)."""
import numpy as np

from workloads import NAN_BITS, make_config
from workloads.gen import make_prefix_cow


def _check_tables(c):
    bs = c.block_size
    need = (c.context_lens.astype(np.int64) + bs - 1) // bs
    used = []
    for s in range(c.num_seqs):
        row = c.block_tables[s]
        assert np.all(row[: need[s]] >= 0) and np.all(row[: need[s]] < c.num_blocks)
        assert np.all(row[need[s]:] == -1)
        used.extend(row[: need[s]].tolist())
    return used, need


def test_tiny_matches_spec():
    c = make_config("tiny")
    assert (c.num_seqs, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size) == (4, 4, 4, 64, 16)
    assert c.dtype == "fp16" and c.scale == 1.0 / 8 and c.num_blocks == 64
    assert c.context_lens.tolist() == [1, 17, 33, 100]
    used, need = _check_tables(c)
    assert need.tolist() == [1, 2, 3, 7]
    assert len(set(used)) == len(used) == 13  # distinct ids carved from one permutation
    # the new token lands at position L-1: L = 17, 33 start a block, L = 100 -> block 6, offset 3
    for s, L in enumerate(c.context_lens):
        blk, off = divmod(int(c.slot_mapping[s]), 16)
        assert blk == c.block_tables[s, (L - 1) // 16] and off == (L - 1) % 16
    assert [int(x) % 16 for x in c.slot_mapping] == [0, 0, 0, 3]


def test_poison_marks_everything_not_read():
    c = make_config("tiny")
    nan = NAN_BITS["fp16"]
    kept = 0
    for s, L in enumerate(c.context_lens):
        for t in range(int(L) - 1):
            blk = c.block_tables[s, t // 16]
            assert np.all(c.k_cache[blk, :, t % 16] != nan)
            kept += 1
    n_nan_rows = int(np.all(c.k_cache == nan, axis=-1).sum())
    assert n_nan_rows == 64 * 4 * 16 - kept * 4


def test_deterministic():
    a, b = make_config("tiny"), make_config("tiny")
    for f in ("q", "k_cache", "v_cache", "key", "value", "block_tables", "slot_mapping"):
        assert np.array_equal(getattr(a, f), getattr(b, f))


def test_prefix_cow_structure():
    c = make_prefix_cow(groups=3, samples=8, max_suffix=40)
    assert c.copy_pairs.shape == (3 * 7, 2)
    assert np.all((c.context_lens >= 1001) & (c.context_lens <= 1041))
    for g in range(3):
        rows = c.block_tables[g * 8:(g + 1) * 8]
        assert np.all(rows[:, :62] == rows[0, :62])  # shared full prefix blocks
        partial = rows[:, 62]
        assert partial[7] == c.copy_pairs[g * 7, 0]  # last sample keeps the original
        assert len(set(partial.tolist())) == 8  # the rest own private copies
    dst = c.copy_pairs[:, 1]
    assert len(set(dst.tolist())) == len(dst) and not set(dst) & set(c.copy_pairs[:, 0])
    assert len(set(c.slot_mapping.tolist())) == len(c.slot_mapping)
    # the per-sample copy list names the same copies, restricted to the prompt's 8 rows
    # of block 62 (the slots past them are the ones the step writes)
    assert c.cow.shape == (24, 3) and c.cow.dtype == np.int32
    named = {(int(s), int(c.block_tables[i, lb])) for i, (s, lb, r) in enumerate(c.cow)
             if s >= 0}
    assert named == {(int(a), int(b)) for a, b in c.copy_pairs}
    assert np.all(c.cow[c.cow[:, 0] >= 0, 1:] == [62, 1000 - 62 * 16])
    assert np.all(c.cow[7::8, 0] == -1)  # the sample that keeps the shared block
    written = {(int(x) // 16, int(x) % 16) for x in c.slot_mapping}
    for i, (s, lb, r) in enumerate(c.cow):
        if s >= 0:
            assert not any((int(c.block_tables[i, lb]), k) in written for k in range(r))


def test_prefill_case_structure():
    """Chunks sit at the end of their contexts, each new token's slot is its position's
    page and offset, pages are distinct across sequences, and poison covers exactly the
    slots that are neither earlier context nor written by the step."""
    from workloads import make_prefill_case
    specs = [(9, 9), (5, 30), (1, 12), (0, 7), (17, 17)]
    c = make_prefill_case("pfs", 3, specs, 8, 2, 32, 8, dtype="fp16")
    bs, qsl = c.block_size, c.query_start_loc
    assert qsl.tolist() == [0, 9, 14, 15, 15, 32] and c.num_tokens == 32
    assert c.context_lens.tolist() == [L for _, L in specs]
    used, need = _check_tables(c)
    assert len(set(used)) == len(used) <= c.num_blocks
    for s, (n, L) in enumerate(specs):
        for i in range(n):
            p = L - n + i
            blk, off = divmod(int(c.slot_mapping[qsl[s] + i]), bs)
            assert blk == c.block_tables[s, p // bs] and off == p % bs
    assert len(set(c.slot_mapping.tolist())) == c.num_tokens
    nan = NAN_BITS["fp16"]
    earlier = {(int(c.block_tables[s, p // bs]), p % bs)
               for s, (n, L) in enumerate(specs) for p in range(L - n)}
    for b in range(c.num_blocks):
        for o in range(bs):
            poisoned = bool(np.all(c.k_cache[b, :, o] == nan))
            assert poisoned == ((b, o) not in earlier), (b, o)


def test_prefill_workloads_shapes():
    from workloads import make_prefill_config
    a = make_prefill_config("prefill_2k_gqa", poison=False)
    assert (a.num_seqs, a.num_tokens, a.num_q_heads, a.num_kv_heads, a.head_dim) == \
        (8, 8 * 2048, 32, 8, 128)
    b = make_prefill_config("prefill_chunk512_gqa", poison=False)
    n = np.diff(b.query_start_loc)
    assert b.num_seqs == 16 and np.all(n == 512)
    assert sorted(set(b.context_lens.tolist())) == sorted({2048 + 128 * (i % 13) for i in range(16)})


def test_window_case_holds_only_the_windows_pages():
    """Under a sliding window the pages wholly before each sequence's window are -1 and
    the pool holds the window pages plus spare; the new token's slot is still L - 1."""
    from workloads import make_case
    W, bs = 20, 8
    c = make_case("win", 5, 6, 4, 2, 32, bs, lambda r: np.array([1, 19, 20, 21, 60, 100],
                                                              np.int32), window=W)
    held = []
    for s, L in enumerate(c.context_lens.tolist()):
        need = -(-L // bs)
        dead = max(L - W, 0) // bs
        row = c.block_tables[s]
        assert np.all(row[:dead] == -1) and np.all(row[dead:need] >= 0)
        assert np.all(row[need:] == -1)
        held.extend(row[dead:need].tolist())
        blk, off = divmod(int(c.slot_mapping[s]), bs)
        assert blk == row[(L - 1) // bs] and off == (L - 1) % bs
    assert len(set(held)) == len(held) <= c.num_blocks
