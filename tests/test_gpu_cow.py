"""Copy-on-write folded into the decode (pa_decode_cow) against the oracle.

Bar: both caches bit-exact against the oracle's filled-rows copy (rows [0, rows) of the
named source into the sequence's own block), its cache write and nothing else; the
output within max-abs 2e-3 (fp16) / 1e-2 (bf16) of the oracle's attention over those
caches, and bit-identical to pa_decode run on them.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_441_b200 as pa
from tests.gpu_util import TOL, DeviceCase, bits, dev, dev16, to_f64
from workloads import make_case, make_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.device_error(0, clear=True)
    yield
    bits_left = pa.device_error(0, clear=True)
    assert bits_left == 0, f"device error word {bits_left:#x} left set"


def _copy_rows(kc, vc, cow, tables):
    """The copies a cow list asks for, on host caches: the oracle's filled-rows copy of
    rows [0, rows) of every kv head of the source block into the sequence's block at the
    logical index."""
    triples = [(int(src), int(tables[s, lb]), int(rows)) for s, (src, lb, rows) in enumerate(cow)
               if src >= 0]
    if triples:
        assert oracle.copy_rows(kc, vc, np.array(triples, np.int64)) == 0


def _cow_list(case, rng, frac=0.7):
    """A random cow list for a case: sources among the blocks no sequence owns, logical
    indices anywhere in each table row (inside the context, before a window), row counts
    0..block_size.  Fixed entries: the first sequence copies a whole page; the second
    copies no rows; an empty context and a context shorter than its table row get a
    block past their last position (a table entry attention never reads) to copy into.
    Mutates case.block_tables for those two."""
    owned = set(case.block_tables[case.block_tables >= 0].tolist())
    free = [b for b in range(case.num_blocks) if b not in owned]
    assert len(free) >= 4
    past = []  # (sequence, logical index) of table entries past the context
    for s in range(case.num_seqs):
        n = -(-int(case.context_lens[s]) // case.block_size)
        if n < case.block_tables.shape[1] and len(past) < 2:
            case.block_tables[s, n] = free.pop()
            past.append((s, n))
    cow = np.full((case.num_seqs, 3), -1, np.int32)
    cow[:, 1:] = 0
    for s in range(case.num_seqs):
        width = int(np.sum(case.block_tables[s] >= 0))
        if width == 0 or rng.random() > frac:
            continue
        cow[s] = (int(rng.choice(free)), int(rng.integers(0, width)),
                  int(rng.integers(0, case.block_size + 1)))
    for s, n in past:
        cow[s] = (free[0], n, case.block_size)
    for s in range(case.num_seqs):
        if (s, int(cow[s, 1])) not in past and int(np.sum(case.block_tables[s] >= 0)):
            cow[s] = (free[1], 0, case.block_size)
            break
    for s in range(case.num_seqs - 1, -1, -1):
        if (s, int(cow[s, 1])) not in past and int(np.sum(case.block_tables[s] >= 0)) > 1:
            cow[s] = (free[2], 1, 0)
            break
    return cow


def _fill_free_blocks(case, seed):
    """Random values in the blocks no sequence owns (the copy sources)."""
    rng = np.random.default_rng(seed)
    owned = set(case.block_tables[case.block_tables >= 0].tolist())
    for b in range(case.num_blocks):
        if b not in owned:
            for c in (case.k_cache, case.v_cache):
                c[b] = rng.integers(0, 0x3F80, size=c[b].shape, dtype=np.uint16)


def _run_cow(case, cow, partition_size, window, fused_write):
    dc = DeviceCase(case)
    if not fused_write:
        pa.kv_write(dc.key, dc.value, dc.slot_mapping, dc.k_cache, dc.v_cache)
    kw = dict(key=dc.key, value=dc.value) if fused_write else {}
    pa.decode_cow(dc.out, dc.q, dc.k_cache, dc.v_cache, dc.block_tables, dc.context_lens,
                  dev(cow), case.scale, max_context_len=case.max_context_len,
                  partition_size=partition_size, sliding_window=window, **kw)
    torch.cuda.synchronize()
    return dc


def _expected(case, cow, fused_write):
    """Caches after the call: the fused write comes after the copies; a separate
    pa_kv_write comes before them."""
    kc, vc = case.k_cache.copy(), case.v_cache.copy()
    if not fused_write:
        oracle.kv_write(case.key, case.value, case.slot_mapping, kc, vc)
    _copy_rows(kc, vc, cow, case.block_tables)
    if fused_write:
        oracle.kv_write(case.key, case.value, case.slot_mapping, kc, vc)
    return kc, vc


@pytest.mark.parametrize("dtype,G,d,bs", [("bf16", 1, 128, 16), ("fp16", 4, 128, 32),
                                          ("bf16", 8, 128, 512), ("fp16", 2, 64, 8),
                                          ("bf16", 8, 64, 16)])
@pytest.mark.parametrize("ps,window", [(0, 0), (64, 0), (64, 100), (0, 300)])
@pytest.mark.parametrize("fused_write", [True, False])
def test_cow_rows_copied_by_their_readers(dtype, G, d, bs, ps, window, fused_write):
    """Ragged contexts (empty, one token, tile and page edges, several partitions), the
    copied block anywhere in the table (before the window, past the context, spanning
    partitions when pages are larger than partitions), row counts from 0 to a whole
    page: every cache row bit-exact and every output against the oracle."""
    hkv = 2
    lens = [0, 1, 15, 16, 17, 64, 65, 200, 700, 1030, 33, 129]
    case = make_case(f"cow{G}", 60 + G, len(lens), hkv * G, hkv, d, bs,
                     lambda r: np.array(lens, np.int32), dtype=dtype, spare=0.5)
    _fill_free_blocks(case, 61 + G)
    rng = np.random.default_rng([G, d, bs, ps, window])
    cow = _cow_list(case, rng)
    dc = _run_cow(case, cow, ps, window, fused_write)
    kc, vc = _expected(case, cow, fused_write)
    assert np.array_equal(bits(dc.k_cache), kc)
    assert np.array_equal(bits(dc.v_cache), vc)
    want = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale,
                         dtype, sliding_window=window)
    err = np.max(np.abs(to_f64(dc.out) - want))
    assert np.isfinite(err) and err <= TOL[dtype], err
    # the same bits as pa_decode over the caches the copies left
    ref = DeviceCase(case)
    ref.k_cache, ref.v_cache = dev16(kc, dtype), dev16(vc, dtype)
    ref.decode(partition_size=ps, sliding_window=window)
    torch.cuda.synchronize()
    assert np.array_equal(bits(dc.out), bits(ref.out))


def _prefix_cow_list(case):
    """The prefix workload's copies as a cow list: each sample with a private copy of
    the prompt's partially filled block copies the prompt's rows of it from the shared
    block; the sample that keeps the shared block copies nothing."""
    bs = case.block_size
    prefix = 1000
    lb, rows = prefix // bs, prefix % bs
    src_of = {int(d): int(s) for s, d in case.copy_pairs}
    cow = np.full((case.num_seqs, 3), -1, np.int32)
    cow[:, 1:] = 0
    for s in range(case.num_seqs):
        dst = int(case.block_tables[s, lb])
        if dst in src_of:
            cow[s] = (src_of[dst], lb, rows)
    assert int(np.sum(cow[:, 0] >= 0)) == case.copy_pairs.shape[0]
    return cow


def test_prefix_step_with_the_copies_folded_in():
    """The prefix-sharing workload at full size (64 groups x 8 samples, 1000-token shared
    prompt): the step as cache write + pa_decode_cow leaves both caches bit-identical to
    the three-launch step (block copies, cache write, decode) and gives the same output
    bits; every output against the oracle."""
    case = make_config("prefix_cow")
    cow = _prefix_cow_list(case)
    ref = DeviceCase(case)
    ref.step()
    dc = _run_cow(case, cow, 0, 0, fused_write=False)
    assert np.array_equal(bits(dc.k_cache), bits(ref.k_cache))
    assert np.array_equal(bits(dc.v_cache), bits(ref.v_cache))
    assert np.array_equal(bits(dc.out), bits(ref.out))
    want, kc, vc = oracle.step(case)
    assert np.array_equal(bits(dc.k_cache), kc) and np.array_equal(bits(dc.v_cache), vc)
    err = np.max(np.abs(to_f64(dc.out) - want))
    assert np.isfinite(err) and err <= TOL[case.dtype], err


def test_cow_bad_entries_are_flagged_and_skipped():
    """A source or logical index out of range, or a row count above the page, sets the
    pair bit; a table entry out of range at the copied index sets the block-id bit.  The
    copy of that sequence is skipped, the others are done, and the context stays usable."""
    lens = [40, 100, 7, 300]
    case = make_case("cowbad", 71, len(lens), 8, 2, 128, 16,
                     lambda r: np.array(lens, np.int32), dtype="bf16", spare=0.5)
    _fill_free_blocks(case, 72)
    good = _cow_list(case, np.random.default_rng(73), frac=1.0)
    for s, bad in ((1, (case.num_blocks, 0, 4)), (2, (int(good[2, 0]), 999, 4)),
                   (3, (int(good[3, 0]), 1, 17))):
        cow = good.copy()
        cow[s] = bad
        dc = _run_cow(case, cow, 64, 0, fused_write=True)
        assert pa.device_error(0, clear=True) == pa.DEVERR["pair"], s
        skip = cow.copy()
        skip[s] = (-1, 0, 0)
        kc, vc = _expected(case, skip, fused_write=True)
        assert np.array_equal(bits(dc.k_cache), kc) and np.array_equal(bits(dc.v_cache), vc)
    bt = case.block_tables.copy()
    bt[0, 0] = case.num_blocks + 5
    dc = DeviceCase(case)
    dc.block_tables = dev(bt)
    cow = good.copy()
    cow[0] = (int(good[0, 0]), 0, 16)
    pa.decode_cow(dc.out, dc.q, dc.k_cache, dc.v_cache, dc.block_tables, dc.context_lens,
                  dev(cow), case.scale, partition_size=64)
    torch.cuda.synchronize()
    assert pa.device_error(0, clear=True) & pa.DEVERR["block_id"]
    # still usable: a clean call matches the oracle
    dc = _run_cow(case, good, 64, 0, fused_write=True)
    kc, vc = _expected(case, good, fused_write=True)
    want = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale,
                         "bf16")
    assert np.max(np.abs(to_f64(dc.out) - want)) <= TOL["bf16"]


def test_cow_refuses_the_balanced_and_dynamic_splits():
    lens = [40, 3000]
    case = make_case("cowsplit", 74, len(lens), 8, 2, 128, 16,
                     lambda r: np.array(lens, np.int32), dtype="bf16", spare=0.5)
    dc = DeviceCase(case)
    cow = dev(np.array([[-1, 0, 0]] * 2, np.int32))
    for ps in (pa.PARTITION_BALANCED, pa.PARTITION_DYNAMIC):
        ws = torch.zeros(pa.decode_workspace_bytes(2, 8, 2, 128, 16,
                                                   case.max_blocks_per_seq, 0, ps),
                         dtype=torch.uint8, device="cuda")
        with pytest.raises(pa.PAError, match="unsupported"):
            pa.decode_cow(dc.out, dc.q, dc.k_cache, dc.v_cache, dc.block_tables,
                          dc.context_lens, cow, case.scale, partition_size=ps, workspace=ws)
