"""Decode launched from a host-side plan (pa_decode_planned) against the full-grid launch.

Each unit of the plan computes what the same (sequence, partition) CTA of the full grid
computes, and the merge combines the partitions in their index order, so the outputs
must be bit-identical to pa_decode (pa_decode_append with the new tokens), which the
parity tests compare with the oracle; one small case is compared with the oracle here
as well."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_441_b200 as pa
from tests.gpu_util import TOL, DeviceCase, bits, dev, to_f64
from workloads import make_case, make_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_error_word():
    pa.device_error(0, clear=True)
    yield
    bits_left = pa.device_error(0, clear=True)
    assert bits_left == 0, f"device error word {bits_left:#x} left set"


def _both(case, ps, fused, host_lens=None):
    """(full-grid DeviceCase, planned DeviceCase) after the same step."""
    ref, got = DeviceCase(case), DeviceCase(case)
    hl = case.context_lens.astype(np.int32) if host_lens is None else host_lens
    mcl = case.max_context_len
    if fused:
        pa.decode_append(ref.out, ref.q, ref.key, ref.value, ref.k_cache, ref.v_cache,
                         ref.block_tables, ref.context_lens, case.scale, max_context_len=mcl,
                         partition_size=ps)
        pa.decode_planned(got.out, got.q, got.k_cache, got.v_cache, got.block_tables,
                          got.context_lens, hl, case.scale, key=got.key, value=got.value,
                          max_context_len=mcl, partition_size=ps)
    else:
        for d in (ref, got):
            pa.kv_write(d.key, d.value, d.slot_mapping, d.k_cache, d.v_cache)
        ref.decode(partition_size=ps)
        pa.decode_planned(got.out, got.q, got.k_cache, got.v_cache, got.block_tables,
                          got.context_lens, hl, case.scale, max_context_len=mcl,
                          partition_size=ps)
    torch.cuda.synchronize()
    return ref, got


@pytest.mark.parametrize("dtype,d,G,bs", [("bf16", 128, 1, 16), ("fp16", 128, 4, 32),
                                          ("bf16", 128, 8, 512), ("fp16", 64, 2, 8),
                                          ("bf16", 64, 8, 16)])
@pytest.mark.parametrize("ps", [0, 64, 192])
@pytest.mark.parametrize("fused", [True, False])
def test_planned_equals_full_grid(dtype, d, G, bs, ps, fused):
    """Ragged contexts -- empty, one token, tile, page and partition edges, several
    partitions -- in every kernel shape, with and without the fused cache write."""
    hkv = 2
    lens = [0, 1, 15, 16, 17, 63, 64, 65, 191, 192, 193, 700, 1030, 2100, 33, 0]
    case = make_case(f"plan{G}", 80 + G, len(lens), hkv * G, hkv, d, bs,
                     lambda r: np.array(lens, np.int32), dtype=dtype)
    ref, got = _both(case, ps, fused)
    assert np.array_equal(bits(got.out), bits(ref.out))
    assert np.array_equal(bits(got.k_cache), bits(ref.k_cache))
    assert np.array_equal(bits(got.v_cache), bits(ref.v_cache))


def test_planned_against_the_oracle():
    lens = [5, 300, 0, 1024, 1025, 77]
    case = make_case("plan_oracle", 90, len(lens), 16, 4, 128, 16,
                     lambda r: np.array(lens, np.int32), dtype="bf16")
    _, got = _both(case, 256, True)
    want, kc, vc = oracle.step(case)
    err = np.max(np.abs(to_f64(got.out) - want))
    assert np.isfinite(err) and err <= TOL["bf16"], err
    assert np.array_equal(bits(got.k_cache), kc) and np.array_equal(bits(got.v_cache), vc)


@pytest.mark.parametrize("name,kw", [("llama2_7b", {}), ("gqa_llama3_8b", {"block_size": 16}),
                                     ("long_8_1", {"block_size": 512}),
                                     ("long_32_8", {"block_size": 16})])
def test_planned_full_size_workloads(name, kw):
    """The benchmark's workloads at full size, at the library's default split (the
    launch configuration the benchmark times), with the fused cache write."""
    case = make_config(name, **kw)
    ref, got = _both(case, 0, True)
    assert np.array_equal(bits(got.out), bits(ref.out))
    assert np.array_equal(bits(got.k_cache), bits(ref.k_cache))
    del ref, got
    torch.cuda.empty_cache()


def test_plan_too_large_runs_the_full_grid():
    """More units than the plan holds (600 contexts x 8 partitions): the call launches
    the full grid instead, with the same results."""
    rng = np.random.default_rng(91)
    lens = rng.integers(450, 520, size=600).astype(np.int32)
    case = make_case("plan_big", 91, 600, 8, 8, 64, 16, lambda r: lens, dtype="bf16",
                     poison=False)
    ref, got = _both(case, 64, True)
    assert np.array_equal(bits(got.out), bits(ref.out))


def test_plan_from_wrong_host_lengths_is_flagged():
    """Host lengths that need fewer partitions than the device's: the context error bit
    is set (the partition the plan left out is not computed)."""
    lens = [100, 700, 40]
    case = make_case("plan_bad", 92, len(lens), 8, 2, 128, 16,
                     lambda r: np.array(lens, np.int32), dtype="bf16")
    host = np.array([100, 200, 40], np.int32)  # 700 tokens need 3 partitions of 256
    _both(case, 256, False, host_lens=host)
    assert pa.device_error(0, clear=True) & pa.DEVERR["context"]
    with pytest.raises(pa.PAError, match="host_context_lens"):
        d = DeviceCase(case)
        pa.decode_planned(d.out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                          np.zeros(2, np.int32), case.scale)
    with pytest.raises(pa.PAError, match="host memory"):
        d = DeviceCase(case)
        pa.decode_planned(d.out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                          d.context_lens, case.scale)
