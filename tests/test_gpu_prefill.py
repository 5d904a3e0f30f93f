"""Multi-query (prefill / chunked prefill) attention on the tcgen05 tensor cores vs the
fp64 oracle, through the C ABI.  Same bar as decode: max-abs 1e-2 (bf16) / 2e-3
(fp16) against the unrounded oracle; the cache write of the chunk bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_441_b200 as pa
from tests.gpu_util import TOL, bits, dev, dev16, to_f64
from workloads import make_prefill_case, make_prefill_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.device_error(0, clear=True)
    yield
    bits_left = pa.device_error(0, clear=True)
    assert bits_left == 0, f"device error word {bits_left:#x} left set"


def _recycle(case, window):
    """Table entries of pages wholly before the first query's window -> -1."""
    if window > 0:
        n = np.diff(case.query_start_loc)
        for s, L in enumerate(case.context_lens.tolist()):
            lo = max(0, L - int(n[s]) - window + 1)
            case.block_tables[s, :lo // case.block_size] = -1
    return case


def _run(case, window=0):
    dt = case.dtype
    kc, vc = dev16(case.k_cache, dt), dev16(case.v_cache, dt)
    pa.kv_write(dev16(case.key, dt), dev16(case.value, dt), dev(case.slot_mapping), kc, vc)
    q = dev16(case.q, dt)
    out = torch.full_like(q, float("nan"))
    pa.prefill(out, q, kc, vc, dev(case.block_tables), dev(case.context_lens),
               dev(case.query_start_loc), case.scale, sliding_window=window)
    torch.cuda.synchronize()
    return out, kc, vc


def _oracle(case, window=0, sel=None):
    kc, vc = case.k_cache.copy(), case.v_cache.copy()
    oracle.kv_write(case.key, case.value, case.slot_mapping, kc, vc)
    out, bad = oracle.prefill(case.q, kc, vc, case.block_tables, case.context_lens,
                              case.query_start_loc, case.scale, case.dtype, sliding_window=window,
                              sel=sel, return_bad=True)
    assert bad == 0
    return out, kc, vc


def _check(case, window=0, sel=None):
    out, kc, vc = _run(case, window)
    ref, kc_ref, vc_ref = _oracle(case, window, sel)
    got = to_f64(out)
    if sel is not None:
        got = got[sel[:, 0], sel[:, 1]]
    err = np.max(np.abs(got - ref))
    assert np.isfinite(err) and err <= TOL[case.dtype], (case.name, window, err)
    return out, kc, vc, kc_ref, vc_ref


SPECS = [(1, 1), (5, 5), (127, 127), (128, 128), (129, 129), (300, 300), (17, 200),
         (64, 1000), (1, 77), (0, 40), (40, 40)]


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [8, 16, 128, 512])
def test_prefill_every_kernel_variant(dtype, d, G, bs):
    """Whole prompts at and around the 128-row / 128-key tile edges, chunks after longer
    contexts, one-token chunks and an empty chunk, for every (dtype, head_dim, group,
    box) instance; plus the chunk's cache write bit-exact."""
    case = make_prefill_case("pf", 100 + d + G + bs, SPECS, 2 * G, 2, d, bs, dtype=dtype)
    out, kc, vc, kc_ref, vc_ref = _check(case)
    assert np.array_equal(bits(kc), kc_ref) and np.array_equal(bits(vc), vc_ref)


@pytest.mark.parametrize("window", [1, 50, 128, 129, 1000])
@pytest.mark.parametrize("G,bs", [(1, 16), (4, 8), (8, 128)])
def test_prefill_sliding_window(window, G, bs):
    """Windows shorter and longer than the tiles, with the pages before each chunk's
    first window given back (-1): never read."""
    case = _recycle(make_prefill_case("pfw", 200 + window + G, SPECS, 2 * G, 2, 128, bs),
                    window)
    _check(case, window)


def test_prefill_one_token_chunks_match_decode():
    """A batch of one-token chunks is a decode step: same result as pa_decode within
    the bar (both against the oracle), on both tensor-core and SIMT decode paths."""
    specs = [(1, L) for L in (1, 9, 200, 1500)]
    for hq, hkv in ((8, 8), (32, 8)):
        case = make_prefill_case("pf1", 7, specs, hq, hkv, 128, 16)
        out, kc, vc, _, _ = _check(case)
        dec = torch.empty_like(out)
        pa.decode(dec, dev16(case.q, "bf16"), kc, vc, dev(case.block_tables),
                  dev(case.context_lens), case.scale)
        torch.cuda.synchronize()
        assert np.max(np.abs(to_f64(dec) - to_f64(out))) <= 2 * TOL["bf16"]


def test_prefill_many_short_prompts():
    """66,000 one- to three-token prompts (8 query heads on 1 kv head): the launch's bound
    on tile pairs exceeds the grid's y limit, so the kernel takes the layout with the pair
    in blockIdx.x and the kv head in blockIdx.y; every output against the oracle.  Among
    34M outputs some reach magnitudes of 4 and more, where half a bf16 step (2^-6) is
    itself above the 1e-2 bar, so each output may differ from the exact value by the larger
    of the bar and half a bf16 step of that value (rounding the exact result gives the same
    worst case)."""
    specs = [(1, 1 + (i % 3)) for i in range(66000)]
    case = make_prefill_case("many", 5, specs, 8, 1, 64, 16)
    out, kc, vc = _run(case)
    ref, _, _ = _oracle(case)
    got = to_f64(out)
    mag = np.maximum(np.abs(ref), 2.0 ** -126)
    half_step = np.exp2(np.floor(np.log2(mag)) - 8)  # half the bf16 spacing at |ref|
    bound = np.maximum(TOL[case.dtype], half_step)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)) and np.all(err <= bound), float(np.max(err - bound))


@pytest.mark.parametrize("name", ["prefill_2k_gqa", "prefill_chunk512_gqa"])
def test_prefill_workloads_full_size(name):
    """The benchmark's prefill workloads at full size, every (token, head) output."""
    case = make_prefill_config(name)
    _check(case)


def test_prefill_errors_flagged():
    """A chunk longer than its context and an out-of-range table entry set their
    error bits; the other sequences are still computed."""
    case = make_prefill_case("pfe", 9, [(10, 10), (20, 40), (5, 5)], 8, 2, 128, 16)
    ref, _, _ = _oracle(case)
    bad = case.context_lens.copy()
    bad[2] = 4  # n = 5 > L = 4
    dt = case.dtype
    kc, vc = dev16(case.k_cache, dt), dev16(case.v_cache, dt)
    pa.kv_write(dev16(case.key, dt), dev16(case.value, dt), dev(case.slot_mapping), kc, vc)
    q = dev16(case.q, dt)
    out = torch.zeros_like(q)
    pa.prefill(out, q, kc, vc, dev(case.block_tables), dev(bad), dev(case.query_start_loc),
               case.scale)
    assert pa.device_error(0) & pa.DEVERR["context"]
    got = to_f64(out)
    assert np.max(np.abs(got[:30] - ref[:30])) <= TOL["bf16"]
    bt = case.block_tables.copy()
    bt[1, 0] = case.num_blocks + 7
    pa.prefill(out, q, kc, vc, dev(bt), dev(case.context_lens), dev(case.query_start_loc),
               case.scale)
    assert pa.device_error(0) & pa.DEVERR["block_id"]
    with pytest.raises(pa.PAError):
        pa.prefill(out, q, kc, vc, dev(bt), dev(case.context_lens), dev(case.query_start_loc),
                   case.scale, sliding_window=-3)
