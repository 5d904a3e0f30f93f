"""pa_decode_static_scratch: decode for callers that cannot allocate device memory.

Such callers (an engine that handed all free HBM to its KV-cache pool and offers no
allocator, or code that must not run cudaMalloc inside its decode loop) cannot pass
pa_decode a workspace.  This entry point keeps the split-K partials in the library's
own fixed scratch array instead.  The test calls it through the C ABI several times
in a row, on different inputs that all need several partitions, and checks each
output bit for bit against pa_decode with a caller workspace (the same kernels on
the same plan; within the bf16 bar for the dynamic split, whose sums vary in the
last bits) and against the fp64 oracle within the bf16 bar; a later call must not
be disturbed by what an earlier one left in the shared array, and the dynamic
split's counters, kept at its start, must read zero at each call.  It also checks
that sizes over the fixed limit are refused before any launch, for the fixed and
the balanced split.  This file sorts last so that a stop-at-first-
failure run has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_441_b200 as pa
from tests.gpu_util import TOL, bits, dev, dev16, to_f64
from workloads import make_case

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _inputs(seed, lens, hq=16, hkv=4, d=128, bs=16):
    case = make_case(f"noalloc{seed}", seed, len(lens), hq, hkv, d, bs,
                     lambda r: np.asarray(lens, np.int32), dtype="bf16", poison=True)
    t = dict(q=dev16(case.q, "bf16"), kc=dev16(case.k_cache, "bf16"),
             vc=dev16(case.v_cache, "bf16"), key=dev16(case.key, "bf16"),
             val=dev16(case.value, "bf16"), sm=dev(case.slot_mapping), bt=dev(case.block_tables),
             cl=dev(case.context_lens))
    pa.kv_write(t["key"], t["val"], t["sm"], t["kc"], t["vc"])
    return case, t


def _c_static(case, t, out, partition_size):
    lib = pa.load()
    P = ctypes.c_void_p
    st = lib.pa_decode_static_scratch(
        P(out.data_ptr()), P(t["q"].data_ptr()), P(t["kc"].data_ptr()), P(t["vc"].data_ptr()),
        P(t["bt"].data_ptr()), P(t["cl"].data_ptr()), case.num_seqs, case.num_q_heads,
        case.num_kv_heads, case.head_dim, case.block_size, case.num_blocks,
        case.max_blocks_per_seq, ctypes.c_float(case.scale), case.max_context_len, 0,
        partition_size, 1, P(torch.cuda.current_stream().cuda_stream))
    return st


def test_static_scratch_matches_workspace_path_twice():
    runs = [(21, [3000, 17, 1290, 640, 2048], 128), (22, [700, 2500, 64, 1999], 256),
            (24, [900, 0, 4100, 33], -1), (26, [5000, 1, 2600, 700], -2),
            (27, [3100, 64, 9000, 20], -2)]
    for seed, lens, ps in runs:
        case, t = _inputs(seed, lens)
        need = pa.decode_workspace_bytes(case.num_seqs, case.num_q_heads, case.num_kv_heads,
                                         case.head_dim, case.block_size, case.max_blocks_per_seq,
                                         case.max_context_len, ps)
        assert 0 < need <= pa.STATIC_SCRATCH_BYTES  # really exercises the scratch
        got = torch.empty_like(t["q"])
        assert _c_static(case, t, got, ps) == 0
        want = torch.empty_like(t["q"])
        pa.decode(want, t["q"], t["kc"], t["vc"], t["bt"], t["cl"], case.scale,
                  max_context_len=case.max_context_len, partition_size=ps)
        torch.cuda.synchronize()
        if ps == pa.PARTITION_DYNAMIC:
            # the dynamic split's sums vary in the last bits from call to call; its
            # counters live at the start of the scratch and each call leaves them zero
            assert np.max(np.abs(to_f64(got) - to_f64(want))) <= TOL["bf16"], seed
        else:
            assert np.array_equal(bits(got), bits(want)), seed
        ref, _, _ = oracle.step(case)
        err = np.max(np.abs(to_f64(got) - ref))
        assert err <= TOL["bf16"], (seed, err)
    assert pa.device_error(0) == 0


def test_static_scratch_refuses_sizes_over_the_limit():
    case, t = _inputs(23, [32768] * 8, hq=8, hkv=1)
    need = pa.decode_workspace_bytes(case.num_seqs, case.num_q_heads, case.num_kv_heads,
                                     case.head_dim, case.block_size, case.max_blocks_per_seq,
                                     case.max_context_len, 64)
    assert need > pa.STATIC_SCRATCH_BYTES
    out = torch.zeros_like(t["q"])
    assert _c_static(case, t, out, 64) == 1  # PA_ERR_INVALID_ARG, nothing launched
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.float()) == 0


def test_static_scratch_refuses_balanced_split_over_the_limit():
    """The balanced split sizes its partial results by the GPU's SM count and the
    group size: a group of 8 at head_dim 128 needs more than the fixed array."""
    case, t = _inputs(25, [5000, 7000, 300, 9000], hq=16, hkv=2)
    need = pa.decode_workspace_bytes(case.num_seqs, case.num_q_heads, case.num_kv_heads,
                                     case.head_dim, case.block_size, case.max_blocks_per_seq,
                                     case.max_context_len, -1)
    assert need > pa.STATIC_SCRATCH_BYTES
    out = torch.zeros_like(t["q"])
    assert _c_static(case, t, out, -1) == 1  # PA_ERR_INVALID_ARG, nothing launched
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.float()) == 0
