"""CUDA path vs the fp64 CPU oracle, element by element, through the C ABI.

Bar: cache write and block copy bit-exact; attention within max-abs 2e-3 (fp16) /
1e-2 (bf16) of the unrounded oracle.  Every output element is compared, for the
small cases and for the five full-size workloads, which run in the launch
configuration the benchmark times.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_441_b200 as pa
from tests.gpu_util import TOL, DeviceCase, bits, dev, dev16, to_f64
from tests.pins import _rand_bits, _tables_for, build_pool
from workloads import NAN_BITS, make_case, make_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.device_error(0, clear=True)
    yield
    bits_left = pa.device_error(0, clear=True)
    assert bits_left == 0, f"device error word {bits_left:#x} left set"


def _check_step(case, partition_size=0, sel=None, full=False, check_cache=True):
    dc = DeviceCase(case)
    out = dc.step(partition_size=partition_size)
    torch.cuda.synchronize()
    ref, kc_ref, vc_ref = oracle.step(case, sel=None if full else sel)
    got = to_f64(out)
    if full:
        err = np.max(np.abs(got - ref))
    else:
        got_sel = got[sel[:, 0], sel[:, 1]]
        err = np.max(np.abs(got_sel - ref))
    assert np.isfinite(err) and err <= TOL[case.dtype], f"{case.name}: max abs err {err}"
    if check_cache:
        # blocks touched by the step (copy destinations and written slots) bit-exact
        touched = set((case.slot_mapping[case.slot_mapping >= 0] // case.block_size).tolist())
        touched |= set(case.copy_pairs[:, 1].tolist())
        idx = np.array(sorted(touched), np.int64)
        it = dev(idx)
        assert np.array_equal(bits(dc.k_cache.index_select(0, it)), kc_ref[idx])
        assert np.array_equal(bits(dc.v_cache.index_select(0, it)), vc_ref[idx])
    return err, dc


# ----------------------------------------------------------------------------- small cases

def test_tiny_full():
    case = make_config("tiny")
    err, dc = _check_step(case, full=True)
    _, kc_ref, vc_ref = oracle.step(case)
    assert np.array_equal(bits(dc.k_cache), kc_ref)  # whole pool, NaN poison included
    assert np.array_equal(bits(dc.v_cache), vc_ref)


def _rand_case(seed, dtype, B, hq, hkv, d, bs, lens, spare=3):
    rng = np.random.default_rng(seed)
    lens = [int(x) for x in lens]
    return make_case(f"rand{seed}", seed, B, hq, hkv, d, bs, lambda r: np.array(lens, np.int32),
                     dtype=dtype, spare=0.25)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_every_kernel_variant(dtype, d, G, bs):
    """All (dtype, head_dim, group, box) instantiations on ragged lengths spanning
    several tiles and partitions, single pass and split-K."""
    hkv = 2
    rng = np.random.default_rng([d, G, bs, 1 if dtype == "bf16" else 2])
    lens = [1, 15, 16, 17, 63, 64, 65, 130, 333, int(rng.integers(1, 700))]
    case = _rand_case(7, dtype, len(lens), hkv * G, hkv, d, bs, lens)
    for ps in (-2, -1, 0, 64, 192):
        _check_step(case, partition_size=ps, full=True)


def test_len1_bit_exact():
    """A one-token context returns that token's V bit for bit (both compute paths)."""
    for dtype in ("bf16", "fp16"):
        for hq, hkv in ((4, 4), (8, 2), (16, 2)):
            case = _rand_case(3, dtype, 5, hq, hkv, 128, 16, [1] * 5)
            dc = DeviceCase(case)
            out = dc.step()
            G = hq // hkv
            want = np.repeat(case.value, G, axis=1)  # the written token is the only one
            assert np.array_equal(bits(out), want), (dtype, hq, hkv)


def test_permutation_bit_identical():
    """The GPU reduction order depends only on logical positions: the same logical
    K/V under two physical permutations gives bit-identical outputs."""
    rng = np.random.default_rng(5)
    lens = [700, 33, 1500, 260]
    B, hq, hkv, d, bs = 4, 8, 2, 128, 16
    Ks = [_rand_bits(rng, (L, hkv, d)) for L in lens]
    Vs = [_rand_bits(rng, (L, hkv, d)) for L in lens]
    q = dev16(_rand_bits(rng, (B, hq, d)), "bf16")
    outs = []
    for trial in range(2):
        nb = sum(-(-L // bs) for L in lens) + 7 * (trial + 1)
        tabs = _tables_for(rng, lens, bs, nb)
        kc, vc, bt = build_pool(Ks, Vs, tabs, nb, bs)
        for ps in (-1, 128):
            out = torch.empty_like(q)
            pa.decode(out, q, dev16(kc, "bf16"), dev16(vc, "bf16"), dev(bt),
                      dev(np.array(lens, np.int32)), 1 / math.sqrt(d), partition_size=ps)
            outs.append((ps, bits(out)))
    assert np.array_equal(outs[0][1], outs[2][1]) and np.array_equal(outs[1][1], outs[3][1])


def test_block_size_invariance():
    """The same logical K/V stored at block sizes 8..512 gives the oracle's answer."""
    rng = np.random.default_rng(6)
    lens = [1000, 17, 513]
    B, hq, hkv, d = 3, 16, 2, 128
    Ks = [_rand_bits(rng, (L, hkv, d)) for L in lens]
    Vs = [_rand_bits(rng, (L, hkv, d)) for L in lens]
    qn = _rand_bits(rng, (B, hq, d))
    ref = None
    for bs in (8, 16, 32, 64, 128, 256, 512):
        nb = sum(-(-L // bs) for L in lens) + 2
        tabs = _tables_for(rng, lens, bs, nb)
        kc, vc, bt = build_pool(Ks, Vs, tabs, nb, bs)
        if ref is None:
            ref = oracle.decode(qn, kc, vc, bt, np.array(lens, np.int32), 0.088, "bf16")
        out = torch.empty(B, hq, d, dtype=torch.bfloat16, device="cuda")
        pa.decode(out, dev16(qn, "bf16"), dev16(kc, "bf16"), dev16(vc, "bf16"), dev(bt),
                  dev(np.array(lens, np.int32)), 0.088)
        err = np.max(np.abs(to_f64(out) - ref))
        assert err <= TOL["bf16"], (bs, err)


def test_identical_keys_mean_of_v():
    rng = np.random.default_rng(8)
    L, hkv, d, bs = 999, 1, 128, 16
    K = np.repeat(_rand_bits(rng, (1, hkv, d)), L, axis=0)
    V = _rand_bits(rng, (L, hkv, d))
    nb = -(-L // bs) + 1
    tabs = _tables_for(rng, [L], bs, nb)
    kc, vc, bt = build_pool([K], [V], tabs, nb, bs)
    for hq in (1, 8):
        q = _rand_bits(rng, (1, hq, d))
        out = torch.empty(1, hq, d, dtype=torch.bfloat16, device="cuda")
        pa.decode(out, dev16(q, "bf16"), dev16(kc, "bf16"), dev16(vc, "bf16"), dev(bt),
                  dev(np.array([L], np.int32)), 0.1)
        want = V[:, 0].view(np.uint16).astype(np.uint32) << 16
        want = want.view(np.float32).astype(np.float64).mean(axis=0)
        assert np.max(np.abs(to_f64(out)[0] - want)) <= TOL["bf16"]


def test_shared_prefix_same_output():
    """Sequences whose tables point at the same prefix blocks, same length and q,
    give identical outputs."""
    rng = np.random.default_rng(9)
    L, hkv, d, bs = 300, 2, 128, 16
    K = _rand_bits(rng, (L, hkv, d))
    V = _rand_bits(rng, (L, hkv, d))
    nb = 40
    tab = _tables_for(rng, [L], bs, nb)[0]
    kc, vc, _ = build_pool([K], [V], [tab], nb, bs)
    bt = np.stack([tab] * 3)
    q = np.repeat(_rand_bits(rng, (1, 8, d)), 3, axis=0)
    out = torch.empty(3, 8, d, dtype=torch.bfloat16, device="cuda")
    pa.decode(out, dev16(q, "bf16"), dev16(kc, "bf16"), dev16(vc, "bf16"), dev(bt),
              dev(np.array([L] * 3, np.int32)), 0.1)
    b = bits(out)
    assert np.array_equal(b[0], b[1]) and np.array_equal(b[0], b[2])


def test_zero_length_and_unread_table_entries():
    """L = 0 gives zeros; table entries past ceil(L/bs) hold out-of-range ids and are
    never read (no error bit)."""
    case = _rand_case(10, "bf16", 4, 8, 2, 128, 16, [0, 5, 16, 40])
    bt = case.block_tables.copy()
    bt[bt < 0] = 10**6
    case.block_tables = bt
    case.slot_mapping[0] = -1  # nothing to write for the empty sequence
    err, dc = _check_step(case, full=True)
    assert np.all(to_f64(dc.out)[0] == 0.0)


@pytest.mark.parametrize("seed", [31, 32, 33])
def test_balanced_split_ragged_and_empty(seed):
    """Default (balanced) split on ragged lengths with empty sequences in between and
    segments cut at arbitrary tiles; fewer tiles than warps; one long sequence."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 400, size=40)
    lens[rng.integers(0, 40, size=8)] = 0
    lens[5] = 1
    for hq, hkv, d, bs in ((8, 8, 128, 16), (32, 4, 128, 8), (16, 2, 64, 32)):
        case = _rand_case(seed, "bf16", len(lens), hq, hkv, d, bs, lens)
        case.slot_mapping[case.context_lens == 0] = -1
        _check_step(case, partition_size=-1, full=True)
    few = _rand_case(seed, "bf16", 3, 8, 2, 128, 16, [0, 3, 20])
    few.slot_mapping[0] = -1
    _check_step(few, partition_size=-1, full=True)
    one = _rand_case(seed, "bf16", 2, 8, 1, 128, 16, [70001, 5])
    _check_step(one, partition_size=-1, full=True)


@pytest.mark.parametrize("B", [100, 128, 129])
def test_second_partitions_longest_first(B):
    """Two partitions per context (partitions of 64, contexts up to 128) and at most 128
    contexts: the second partitions are taken longest first.  Ties in their length,
    contexts without one, empty contexts and one-token second partitions must all land on
    the right outputs (129 contexts keep the plain order)."""
    rng = np.random.default_rng(B)
    lens = rng.integers(0, 129, size=B)
    lens[:10] = [0, 1, 64, 65, 65, 65, 128, 128, 100, 100]
    for G in (1, 4):
        case = _rand_case(B, "bf16", B, 2 * G, 2, 128, 16, lens)
        case.slot_mapping[case.context_lens == 0] = -1
        _check_step(case, partition_size=64, full=True)


def test_table_width_bound():
    """Contexts exactly filling the table width (the largest the table allows)."""
    case = _rand_case(11, "bf16", 3, 8, 8, 128, 32, [32 * 20, 32 * 20, 1])
    _check_step(case, full=True)
    _check_step(case, partition_size=64, full=True)


def test_kv_write_strided_fused_qkv():
    """key/value as column slices of a fused [T, (Hq + 2 Hkv) d] projection."""
    rng = np.random.default_rng(12)
    T, hq, hkv, d, bs, nb = 37, 8, 2, 128, 16, 20
    qkv = dev16(_rand_bits(rng, (T, (hq + 2 * hkv) * d)), "bf16")
    key = qkv[:, hq * d:(hq + hkv) * d].view(T, hkv, d)
    val = qkv[:, (hq + hkv) * d:].view(T, hkv, d)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[4] = -1
    kc0 = _rand_bits(rng, (nb, hkv, bs, d))
    vc0 = _rand_bits(rng, (nb, hkv, bs, d))
    kc, vc = dev16(kc0, "bf16"), dev16(vc0, "bf16")
    pa.kv_write(key, val, dev(slots), kc, vc)
    kr, vr = kc0.copy(), vc0.copy()
    oracle.kv_write(bits(key), bits(val), slots, kr, vr)
    assert np.array_equal(bits(kc), kr) and np.array_equal(bits(vc), vr)


def test_copy_blocks_bit_exact():
    rng = np.random.default_rng(13)
    for nb, hkv, bs, d in ((50, 8, 16, 128), (12, 1, 512, 128), (30, 4, 8, 64)):
        kc0 = _rand_bits(rng, (nb, hkv, bs, d))
        vc0 = _rand_bits(rng, (nb, hkv, bs, d))
        ids = rng.permutation(nb)
        pairs = np.stack([ids[:5], ids[5:10]], axis=1).astype(np.int64)
        kc, vc = dev16(kc0, "bf16"), dev16(vc0, "bf16")
        pa.copy_blocks(kc, vc, dev(pairs))
        kr, vr = kc0.copy(), vc0.copy()
        oracle.copy_blocks(kr, vr, pairs)
        assert np.array_equal(bits(kc), kr) and np.array_equal(bits(vc), vr)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("G,d,bs", [(1, 128, 16), (2, 64, 8), (4, 128, 32), (8, 128, 512),
                                    (8, 64, 16)])
def test_decode_append_equals_write_then_decode(dtype, G, d, bs):
    """The fused step gives the same cache and, bit for bit, the same output as the
    cache write followed by decode (and both match the oracle)."""
    hkv = 2
    lens = [1, 15, 16, 17, 200, 1030, 2100, 33]
    case = _rand_case(40 + G, dtype, len(lens), hkv * G, hkv, d, bs, lens)
    want, _, _ = oracle.step(case)
    for ps in (0, 256, -2):
        ref = DeviceCase(case)
        ref.step(partition_size=ps)
        fused = DeviceCase(case)
        pa.decode_append(fused.out, fused.q, fused.key, fused.value, fused.k_cache,
                         fused.v_cache, fused.block_tables, fused.context_lens, case.scale,
                         max_context_len=case.max_context_len, partition_size=ps)
        torch.cuda.synchronize()
        if ps != pa.PARTITION_DYNAMIC:  # the dynamic split's sums vary in the last bits
            assert np.array_equal(bits(fused.out), bits(ref.out)), (ps, "output differs")
        assert np.array_equal(bits(fused.k_cache), bits(ref.k_cache))
        assert np.array_equal(bits(fused.v_cache), bits(ref.v_cache))
        assert np.max(np.abs(to_f64(fused.out) - want)) <= TOL[dtype], ps


# ------------------------------------------------------------------------ dynamic split

def test_dynamic_split_reuses_its_workspace():
    """Consecutive dynamic-split calls on one workspace, with fixed- and balanced-split
    calls in between: each leaves the counters at zero for the next (no error bit) and
    each result is within the bar; a unit with an empty context, units with one CTA and
    units with many in the same call."""
    lens = [0, 1, 17, 5000, 40000, 300, 12000, 2]
    case = _rand_case(31, "bf16", len(lens), 16, 2, 128, 16, lens)
    dc = DeviceCase(case)
    dc.step(partition_size=-2)
    want, _, _ = oracle.step(case)
    need = max(pa.decode_workspace_bytes(case.num_seqs, case.num_q_heads, case.num_kv_heads,
                                         case.head_dim, case.block_size,
                                         case.max_blocks_per_seq, case.max_context_len, ps)
               for ps in (-2, -1, 256))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    # the other splits share the workspace between dynamic calls and leave its counters be
    for ps in (-2, 256, -2, -1, -2):
        dc.out.fill_(float("nan"))
        dc.decode(partition_size=ps, workspace=ws)
        torch.cuda.synchronize()
        assert np.max(np.abs(to_f64(dc.out) - want)) <= TOL["bf16"], ps
        assert pa.device_error(0) == 0, ps
        assert torch.count_nonzero(ws[:pa.WORKSPACE_ZERO_BYTES]) == 0, ps


@pytest.mark.parametrize("fill", [0xFF, 0x01])
def test_dynamic_split_flags_a_workspace_that_was_not_zeroed(fill):
    """Counters that do not start at zero (-1 or a large count in every word) end the
    claims without forming an address and set the workspace error bit; the call
    leaves the counters zero, so the next call is clean and correct."""
    lens = [3000, 9000, 20000, 64]
    case = _rand_case(32, "bf16", len(lens), 8, 1, 128, 16, lens)
    dc = DeviceCase(case)
    dc.step(partition_size=-2)
    want, _, _ = oracle.step(case)
    need = pa.decode_workspace_bytes(case.num_seqs, case.num_q_heads, case.num_kv_heads,
                                     case.head_dim, case.block_size, case.max_blocks_per_seq,
                                     case.max_context_len, -2)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ws[:pa.WORKSPACE_ZERO_BYTES] = fill
    dc.decode(partition_size=-2, workspace=ws)
    assert pa.device_error(0) == pa.DEVERR["workspace"]
    dc.decode(partition_size=-2, workspace=ws)
    torch.cuda.synchronize()
    assert pa.device_error(0) == 0
    assert np.max(np.abs(to_f64(dc.out) - want)) <= TOL["bf16"]


# ------------------------------------------------------------------------ error handling

def test_device_errors_are_flagged_not_fatal():
    """Bad block ids, slots, pairs and over-long contexts set the sticky error word;
    the bad item is skipped and the context stays usable."""
    case = _rand_case(14, "bf16", 3, 8, 2, 128, 16, [40, 100, 7])
    dc = DeviceCase(case)
    dc.step()
    assert pa.device_error(0) == 0
    bt = case.block_tables.copy()
    bt[1, 2] = case.num_blocks + 3
    dc.block_tables = dev(bt)
    dc.decode()
    assert pa.device_error(0) == pa.DEVERR["block_id"]
    bad_slots = dev(np.array([case.num_blocks * 16 + 1, -1, 0], np.int64))
    pa.kv_write(dc.key, dc.value, bad_slots, dc.k_cache, dc.v_cache)
    assert pa.device_error(0) == pa.DEVERR["slot"]
    pa.copy_blocks(dc.k_cache, dc.v_cache, dev(np.array([[0, -5]], np.int64)))
    assert pa.device_error(0) == pa.DEVERR["pair"]
    dc.block_tables = dev(case.block_tables)
    dc.context_lens = dev(np.array([40, 100, 10**6], np.int32))
    dc.decode(max_context_len=100)
    assert pa.device_error(0) & pa.DEVERR["context"]
    # still usable: a clean run matches the oracle again
    _check_step(case, full=True)


def test_host_rejects_bad_arguments():
    case = _rand_case(15, "bf16", 2, 8, 2, 128, 16, [10, 200])
    dc = DeviceCase(case)
    q6 = dc.q[:, :6].contiguous()
    with pytest.raises(pa.PAError, match="unsupported"):  # refused by the library itself
        pa.decode(torch.empty_like(q6), q6, dc.k_cache, dc.v_cache, dc.block_tables,
                  dc.context_lens, 0.1)  # 6 q heads over 2 kv heads: group 3 not supported
    with pytest.raises(pa.PAError, match="contiguous"):  # refused by the binding
        pa.decode(dc.out[:, :6], dc.q[:, :6], dc.k_cache, dc.v_cache, dc.block_tables,
                  dc.context_lens, 0.1)
    with pytest.raises(pa.PAError, match="expected torch.int32"):
        pa.decode(dc.out, dc.q, dc.k_cache, dc.v_cache, dc.block_tables.long(),
                  dc.context_lens, 0.1)
    with pytest.raises(pa.PAError, match="device"):  # a host tensor never reaches a kernel
        pa.decode(dc.out, dc.q, dc.k_cache, dc.v_cache, dc.block_tables.cpu(),
                  dc.context_lens, 0.1)
    with pytest.raises(pa.PAError):  # workspace too small for the split it needs
        pa.decode(dc.out, dc.q, dc.k_cache, dc.v_cache, dc.block_tables, dc.context_lens, 0.1,
                  partition_size=64, max_context_len=0,
                  workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))


# ------------------------------------------------------------------- full-size workloads

# (workload, builder overrides, partition_size): 0 is the library's choice (the launch
# configuration the benchmark times); 512 is the long-context workload's literal
# "context partitions of 512 tokens"; -1 the balanced split.
FULL = [("llama2_7b", {}, 0), ("gqa_llama3_8b", {"block_size": 16}, 0),
        ("gqa_llama3_8b", {"block_size": 32}, 0), ("long_8_1", {"block_size": 16}, 0),
        ("long_8_1", {"block_size": 512}, 0), ("long_32_8", {"block_size": 16}, 0),
        ("long_32_8", {"block_size": 512}, 0), ("prefix_cow", {}, 0),
        ("long_8_1", {"block_size": 16}, 512), ("long_32_8", {"block_size": 512}, 512),
        ("gqa_llama3_8b", {"block_size": 16}, -1),
        ("long_8_1", {"block_size": 16}, -2), ("long_8_1", {"block_size": 512}, -2),
        ("long_32_8", {"block_size": 16}, -2), ("long_32_8", {"block_size": 512}, -2)]


@pytest.mark.parametrize("name,kw,ps", FULL,
                         ids=[f"{n}-bs{kw.get('block_size', 16)}-ps{ps}" for n, kw, ps in FULL])
def test_full_size(name, kw, ps):
    """Every (sequence, q head) output of the workload against the oracle."""
    case = make_config(name, **kw)
    err, dc = _check_step(case, partition_size=ps, full=True)
    out = dc.out
    assert torch.isfinite(out.float()).all(), "non-finite output somewhere"
    if name == "prefix_cow":
        # samples that share a group and length see the same prefix blocks: equal q
        # would give equal outputs; check the copied blocks' first 8 slots equal the source
        src, dst = case.copy_pairs[0]
        kc = bits(dc.k_cache[int(dst), :, :8])
        assert np.array_equal(kc, case.k_cache[int(src), :, :8])
    del dc
    torch.cuda.empty_cache()
