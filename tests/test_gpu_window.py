"""Sliding-window decode on the GPU vs the fp64 oracle (window read: each query attends
to the last W tokens of its context; the block manager's sliding_window setting in the
dynamic-memory blog's BlockSpaceManager example).

Table entries of pages wholly before each window are set to -1, as the block manager
leaves them after giving those blocks back: reading one would set the device error
word, which the fixture checks after every test.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_441_b200 as pa
from tests.gpu_util import TOL, DeviceCase, bits, to_f64
from workloads import make_case, make_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.device_error(0, clear=True)
    yield
    bits_left = pa.device_error(0, clear=True)
    assert bits_left == 0, f"device error word {bits_left:#x} left set"


def _recycle(case, window):
    """Table entries of pages wholly before each sequence's window -> -1."""
    bt = case.block_tables.copy()
    for s, L in enumerate(case.context_lens.tolist()):
        lo = L - window if 0 < window < L else 0
        bt[s, :lo // case.block_size] = -1
    case.block_tables = bt
    return case


def _case(seed, dtype, hq, hkv, d, bs, lens, window):
    lens = [int(x) for x in lens]
    case = make_case(f"win{seed}", seed, len(lens), hq, hkv, d, bs,
                     lambda r: np.array(lens, np.int32), dtype=dtype, spare=0.25)
    return _recycle(case, window)


def _oracle(case, window, sel=None):
    kc, vc = case.k_cache.copy(), case.v_cache.copy()
    oracle.kv_write(case.key, case.value, case.slot_mapping, kc, vc)
    out, bad = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale,
                             case.dtype, sel=sel, return_bad=True, sliding_window=window)
    assert bad == 0
    return out


def _check(case, window, ps, sel=None):
    dc = DeviceCase(case)
    out = dc.step(partition_size=ps, sliding_window=window)
    torch.cuda.synchronize()
    ref = _oracle(case, window, sel)
    got = to_f64(out)
    if sel is not None:
        got = got[sel[:, 0], sel[:, 1]]
    err = np.max(np.abs(got - ref))
    assert np.isfinite(err) and err <= TOL[case.dtype], (window, ps, err)
    return dc


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("G,d", [(1, 128), (2, 64), (4, 128), (8, 64), (8, 128)])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_window_every_kernel_variant(dtype, G, d, bs):
    """Every compute path and box height: windows that start inside a tile, on a tile or
    page boundary, and windows longer than some contexts; single pass, fixed partitions
    and the balanced split."""
    hkv = 2
    lens = [1, 15, 16, 17, 40, 63, 64, 65, 130, 333, 700]
    for window in (1, 9, 16, 17, 100, 333):
        case = _case(11 + window, dtype, hkv * G, hkv, d, bs, lens, window)
        for ps in (-2, -1, 0, 64, 192):
            _check(case, window, ps)


def test_window_covering_every_context_is_plain_decode():
    """A window at least as long as every context gives the plain result bit for bit."""
    lens = [5, 100, 1000, 3000]
    case = make_case("wplain", 5, len(lens), 16, 4, 128, 16,
                     lambda r: np.array(lens, np.int32), spare=0.25)
    for ps in (-1, 0, 256):
        a = DeviceCase(case).step(partition_size=ps)
        b = DeviceCase(case).step(partition_size=ps, sliding_window=3000)
        torch.cuda.synchronize()
        assert np.array_equal(bits(a), bits(b)), ps


def test_window_of_one_is_last_value_bit_exact():
    """W = 1: the output is the new token's V exactly, on both compute paths."""
    for hq, hkv in ((4, 4), (16, 2)):
        case = _case(6, "bf16", hq, hkv, 128, 16, [1, 2, 17, 500, 4097], 1)
        out = DeviceCase(case).step(sliding_window=1)
        want = np.repeat(case.value, hq // hkv, axis=1)
        assert np.array_equal(bits(out), want), (hq, hkv)


@pytest.mark.parametrize("G,d,bs", [(1, 128, 16), (4, 128, 8), (8, 128, 32)])
def test_decode_append_with_window(G, d, bs):
    """The fused cache write + windowed decode equals kv_write + windowed decode."""
    hkv = 2
    lens = [1, 16, 17, 200, 1030, 2100, 5000]
    window = 1000
    case = _case(50 + G, "bf16", hkv * G, hkv, d, bs, lens, window)
    for ps in (0, 256):
        ref = DeviceCase(case)
        ref.step(partition_size=ps, sliding_window=window)
        fused = DeviceCase(case)
        pa.decode_append(fused.out, fused.q, fused.key, fused.value, fused.k_cache,
                         fused.v_cache, fused.block_tables, fused.context_lens, case.scale,
                         max_context_len=case.max_context_len, partition_size=ps,
                         sliding_window=window)
        torch.cuda.synchronize()
        assert np.array_equal(bits(fused.out), bits(ref.out)), ps
        assert np.array_equal(bits(fused.k_cache), bits(ref.k_cache))
    want = _oracle(case, window)
    assert np.max(np.abs(to_f64(fused.out) - want)) <= TOL["bf16"]


@pytest.mark.parametrize("window", [1000, 4096, 4111])
def test_window_long_contexts(window):
    """Long contexts (the long-context workload's shape, 32/8 heads) with windows of a
    few thousand tokens: only the window's pages are read, in every split; every
    output compared."""
    case = _recycle(make_config("long_32_8", block_size=16, num_seqs=4), window)
    for ps in (-2, -1, 0, 512):
        _check(case, window, ps)


def test_window_rejects_negative():
    case = _case(7, "bf16", 8, 8, 128, 16, [10, 20], 0)
    dc = DeviceCase(case)
    with pytest.raises(pa.PAError):
        pa.decode(dc.out, dc.q, dc.k_cache, dc.v_cache, dc.block_tables, dc.context_lens,
                  case.scale, sliding_window=-1)


@pytest.mark.parametrize("ps", [0, -1])
def test_window_workload_full_size(ps):
    """The benchmark's sliding-window workload (64 sequences, lengths 8K-32K, W = 4096,
    only the windows' pages held), in the launch configuration the benchmark times,
    every output compared; plus the fused step's cache write."""
    case = make_config("window_4096_gqa")
    dc = _check(case, case.window, ps)
    if ps == 0:
        fused = DeviceCase(case)
        pa.decode_append(fused.out, fused.q, fused.key, fused.value, fused.k_cache,
                         fused.v_cache, fused.block_tables, fused.context_lens, case.scale,
                         max_context_len=case.max_context_len, sliding_window=case.window)
        torch.cuda.synchronize()
        assert np.array_equal(bits(fused.out), bits(dc.out))


@pytest.mark.parametrize("B", [60, 129])
def test_window_second_partitions_longest_first(B):
    """Two partitions per window (W = 100, partitions of 64): with at most 128 contexts the
    second partitions are taken longest first.  Ties, contexts shorter than one partition
    and long contexts whose window starts inside a page."""
    rng = np.random.default_rng(B + 7)
    lens = rng.integers(1, 400, size=B)
    lens[:6] = [1, 64, 65, 100, 101, 399]
    case = _case(B, "bf16", 8, 2, 128, 16, lens, 100)
    _check(case, 100, 64)
