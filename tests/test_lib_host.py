"""The C-ABI library loads, exports every entry point its header declares, and its
host-only entry points behave (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import paged_kv_cache_441_b200 as pa
from paged_kv_cache_441_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return pa.load()


def header_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names |= set(re.findall(
                r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(pa_[a-z_0-9]+)\s*\(", src, flags=re.M))
    return sorted(names)


def test_header_declares_the_calls():
    names = header_functions()
    for n in ("pa_kv_write", "pa_decode", "pa_copy_blocks", "pa_get_device_error"):
        assert n in names
    assert set(names) == set(pa.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_status_strings_and_version(lib):
    assert pa.version() == 201
    for code in range(7):
        assert lib.pa_status_str(code) != b"unknown status"
    assert lib.pa_status_str(77) == b"unknown status"


def test_workspace_plan(lib):
    warps = 148 * 3 * 4  # no device here: sized for 148 SMs x 3 CTAs x 4 warps
    # Llama-2-7B-shaped step (2048 sequence x kv-head pairs): fixed 1024-token partitions
    B, hq, hkv, d, bs, W = 64, 32, 32, 128, 16, 126
    assert pa.decode_partition_tokens(B, hq, hkv, d, bs, W, 2011) == 1024
    assert pa.decode_workspace_bytes(B, hq, hkv, d, bs, W, 2011) >= B * hq * 2 * (d + 2) * 4
    # short contexts: one pass, no workspace
    assert pa.decode_partition_tokens(B, hq, hkv, d, bs, W, 300) == 320
    assert pa.decode_workspace_bytes(B, hq, hkv, d, bs, W, 300) == 0
    assert pa.decode_partition_tokens(B, hq, hkv, d, bs, W, 1257) == 1280
    # few sequence x kv-head pairs (8 x 1): 2048-token partitions
    assert pa.decode_partition_tokens(8, 8, 1, d, bs, 8192, 131072) == 2048
    assert pa.decode_workspace_bytes(8, 8, 1, d, bs, 8192, 131072) >= 8 * 8 * 64 * (d + 2) * 4
    # forced balanced split: two records per warp, independent of the lengths
    need = pa.decode_workspace_bytes(8, 8, 1, d, bs, 8192, 131072, -1)
    assert need >= 2 * warps * 8 * (d + 2) * 4 + 9 * 4
    assert need == pa.decode_workspace_bytes(8, 8, 1, d, bs, 8192, 0, -1)
    # forced balanced split for the large batch, forced fixed split for the small one
    assert pa.decode_partition_tokens(B, hq, hkv, d, bs, W, 2011, -1) == 0
    assert pa.decode_workspace_bytes(B, hq, hkv, d, bs, W, 2011, -1) >= 2 * warps * (d + 2) * 4
    assert pa.decode_partition_tokens(8, 8, 1, d, bs, 8192, 131072, 512) == 512
    assert pa.decode_workspace_bytes(B, hq, hkv, d, bs, W, 0, 128) >= B * hq * 16 * (d + 2) * 4
    # dynamic split: the counters (zeroed by the caller once), the units' first CTAs and
    # one record per resident CTA (148 SMs x 3), independent of the lengths
    ctas = 148 * 3
    assert pa.decode_partition_tokens(8, 8, 1, d, bs, 8192, 131072, -2) == 0
    need = pa.decode_workspace_bytes(8, 8, 1, d, bs, 8192, 131072, -2)
    assert need % 256 == 0 and need >= pa.WORKSPACE_ZERO_BYTES + ctas * 8 * (d + 2) * 4
    assert need == pa.decode_workspace_bytes(8, 8, 1, d, bs, 8192, 0, -2)
    # ... and more units than resident CTAs fall back to the fixed split
    assert pa.decode_partition_tokens(B, hq, hkv, d, bs, W, 2011, -2) == 1024
    assert pa.decode_workspace_bytes(B, hq, hkv, d, bs, W, 2011, -2) == pa.decode_workspace_bytes(
        B, hq, hkv, d, bs, W, 2011)
    # sliding window: the tiles of a context span at most W + 15 tokens, whatever L is
    assert pa.decode_partition_tokens(8, 8, 1, d, bs, 8192, 131072, 0, 1000) == 1024
    assert pa.decode_workspace_bytes(8, 8, 1, d, bs, 8192, 131072, 0, 1000) == 0
    assert pa.decode_partition_tokens(8, 8, 1, d, bs, 8192, 131072, 0, 4096) == 2048
    ws3 = pa.decode_workspace_bytes(8, 8, 1, d, bs, 8192, 131072, 0, 4096)
    assert 8 * 8 * 3 * (d + 2) * 4 <= ws3 < 8 * 8 * 4 * (d + 2) * 4 + 1024  # 3 partitions
    assert pa.decode_workspace_bytes(8, 8, 1, d, bs, 8192, 100, 0, 4096) == 0  # bound by L


def _decode_args(**over):
    a = dict(out=16, q=16, kc=16, vc=16, bt=16, cl=16, B=2, hq=8, hkv=2, d=128, bs=16, nb=10,
             W=4, scale=0.1, mcl=0, win=0, ps=0, ws=None, wsb=0, dt=1, stream=None)
    a.update(over)
    return a


def _call_decode(lib, a):
    P = ctypes.c_void_p
    return lib.pa_decode(P(a["out"]), P(a["q"]), P(a["kc"]), P(a["vc"]), P(a["bt"]), P(a["cl"]),
                         a["B"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["W"], a["scale"],
                         a["mcl"], a["win"], a["ps"], a["ws"], a["wsb"], a["dt"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(d=96), 2), (dict(hq=6), 2), (dict(hq=7), 1), (dict(bs=24), 2), (dict(bs=4), 2),
    (dict(bs=1024), 2), (dict(q=0), 1), (dict(q=24), 1), (dict(out=8), 1), (dict(ps=100), 1),
    (dict(scale=float("inf")), 1), (dict(dt=5), 1), (dict(nb=0), 1), (dict(W=0), 1),
    (dict(ps=-2), 1), (dict(ps=-1), 1),  # balanced and dynamic splits need a workspace
    (dict(ps=-3), 1),
    (dict(mcl=-1), 1), (dict(B=-1), 1), (dict(hkv=0), 1), (dict(win=-1), 1),
    (dict(ps=64, W=100), 1),  # needs a workspace, none given
])
def test_decode_rejects_before_launch(lib, over, code):
    # every case is refused by host checks, so no CUDA call is made
    assert _call_decode(lib, _decode_args(**over)) == code


def _call_decode_cow(lib, a, key=None, value=None, cow=16, ks=256, vs=256):
    P = ctypes.c_void_p
    return lib.pa_decode_cow(P(a["out"]), P(a["q"]), P(key) if key else None,
                             P(value) if value else None, ks, vs, P(a["kc"]), P(a["vc"]),
                             P(a["bt"]), P(a["cl"]), P(cow) if cow else None, a["B"], a["hq"],
                             a["hkv"], a["d"], a["bs"], a["nb"], a["W"], a["scale"], a["mcl"],
                             a["win"], a["ps"], a["ws"], a["wsb"], a["dt"], a["stream"])


@pytest.mark.parametrize("over,extra,code", [
    ({}, dict(cow=None), 1),                      # no copy list
    ({}, dict(cow=2), 1),                         # misaligned copy list
    ({}, dict(key=16), 1),                        # key without value
    ({}, dict(key=8, value=16), 1),               # misaligned key
    ({}, dict(key=16, value=16, ks=100), 1),      # token stride not a multiple of 8
    ({}, dict(key=16, value=16, vs=128), 1),      # token stride below Hkv * d
    # the balanced and dynamic splits do not take copies (a workspace is given)
    (dict(ps=-1, ws=256, wsb=1 << 40), {}, 2),
    (dict(ps=-2, ws=256, wsb=1 << 40), {}, 2),
    (dict(d=96), {}, 2),                          # the checks of pa_decode apply too
])
def test_decode_cow_rejects_before_launch(lib, over, extra, code):
    assert _call_decode_cow(lib, _decode_args(**over), **extra) == code


def test_decode_planned_rejects_before_launch(lib):
    a = _decode_args()
    P = ctypes.c_void_p
    host = (ctypes.c_int32 * 2)(10, 20)

    def call(key=None, value=None, hl=host, ks=256, vs=256, **over):
        b = dict(a, **over)
        return lib.pa_decode_planned(P(b["out"]), P(b["q"]), P(key) if key else None,
                                     P(value) if value else None, ks, vs, P(b["kc"]),
                                     P(b["vc"]), P(b["bt"]), P(b["cl"]),
                                     ctypes.cast(hl, P) if hl is not None else None, b["B"],
                                     b["hq"], b["hkv"], b["d"], b["bs"], b["nb"], b["W"],
                                     b["scale"], b["mcl"], b["win"], b["ps"], b["ws"], b["wsb"],
                                     b["dt"], b["stream"])
    assert call(hl=None) == 1              # no host lengths
    assert call(key=16) == 1               # key without value
    assert call(key=8, value=16) == 1      # misaligned key
    assert call(key=16, value=16, ks=100) == 1
    assert call(d=96) == 2                 # the checks of pa_decode apply too
    assert call(hl=None, B=0, out=0, q=0) == 0  # nothing to do


def test_zero_sized_calls_are_noops(lib):
    P = ctypes.c_void_p
    assert _call_decode(lib, _decode_args(B=0, out=0, q=0)) == 0
    assert lib.pa_kv_write(None, None, None, 0, 2, 128, 256, 256, None, None, 10, 16, 1, None) == 0
    assert lib.pa_copy_blocks(None, None, None, 0, 2, 16, 128, 10, 1, None) == 0


def test_kv_write_and_copy_reject(lib):
    P = ctypes.c_void_p
    # misaligned key, stride too small, odd head_dim
    assert lib.pa_kv_write(P(8), P(16), P(16), 1, 2, 128, 256, 256, P(16), P(16), 10, 16, 1, None) == 1
    assert lib.pa_kv_write(P(16), P(16), P(16), 1, 2, 128, 128, 256, P(16), P(16), 10, 16, 1, None) == 1
    assert lib.pa_kv_write(P(16), P(16), P(16), 1, 2, 12, 24, 24, P(16), P(16), 10, 16, 1, None) == 1
    assert lib.pa_copy_blocks(P(16), P(16), None, 3, 2, 16, 128, 10, 1, None) == 1
    assert lib.pa_copy_blocks(P(16), P(16), P(8), 3, 2, 16, 128, 0, 1, None) == 1


def _call_prefill(lib, **over):
    a = dict(out=16, q=16, kc=16, vc=16, bt=16, cl=16, qsl=16, B=2, T=10, hq=8, hkv=2, d=128,
             bs=16, nb=10, W=4, scale=0.1, win=0, dt=1, stream=None)
    a.update(over)
    P = ctypes.c_void_p
    return lib.pa_prefill(P(a["out"]), P(a["q"]), P(a["kc"]), P(a["vc"]), P(a["bt"]), P(a["cl"]),
                          P(a["qsl"]), a["B"], a["T"], a["hq"], a["hkv"], a["d"], a["bs"],
                          a["nb"], a["W"], a["scale"], a["win"], a["dt"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(d=96), 2), (dict(hq=6), 2), (dict(hq=7), 1), (dict(hq=32), 2), (dict(bs=24), 2),
    (dict(bs=1024), 2), (dict(q=0), 1), (dict(q=24), 1), (dict(qsl=0), 1), (dict(qsl=2), 1),
    (dict(win=-1), 1), (dict(scale=float("nan")), 1), (dict(scale=0.0), 1),
    (dict(scale=-0.1), 1), (dict(dt=7), 1), (dict(T=-1), 1),
    (dict(B=0), 0), (dict(T=0), 0),
])
def test_prefill_rejects_before_launch(lib, over, code):
    # every case is settled by host checks (or has nothing to do): no CUDA call is made
    assert _call_prefill(lib, **over) == code


def test_kv_write_refuses_oversized_call(lib):
    # 2^28 tokens x 8 heads x 16 chunks = 2^35 chunks: refused before any launch
    P = ctypes.c_void_p
    st = lib.pa_kv_write(P(16), P(16), P(16), 1 << 28, 8, 128, 1024, 1024, P(16), P(16), 1 << 20,
                         16, 1, None)
    assert st == 2  # PA_ERR_UNSUPPORTED


def _attend_bound(W, bs, mcl, win):
    """Most tokens one context's partitions must cover: the table's capacity, cut by the
    max_context_len hint and, under a window, by the window plus the tile it starts in."""
    bound = W * bs
    if 0 < mcl < bound:
        bound = mcl
    if win > 0:
        bound = min(bound, win + 15)
    return max(bound, 1)


@settings(max_examples=400, derandomize=True, deadline=None)
@given(B=st.integers(1, 600), G=st.sampled_from([1, 2, 4, 8]), hkv=st.integers(1, 16),
       d=st.sampled_from([64, 128]), bs=st.sampled_from([8, 16, 32, 64, 128, 256, 512]),
       W=st.integers(1, 4096), mcl=st.integers(0, 300000), win=st.integers(0, 70000),
       ps=st.sampled_from([0, 0, 64, 128, 512, 1024, 4096]))
def test_workspace_plan_invariants(lib, B, G, hkv, d, bs, W, mcl, win, ps):
    """The fixed split covers every token a context may attend, a single pass needs no
    workspace, and a split's workspace holds one (d + 2)-float record per (sequence, q
    head, partition), 256-byte aligned; a longer hint or window never shrinks it."""
    hq = G * hkv
    P = pa.decode_partition_tokens(B, hq, hkv, d, bs, W, mcl, ps, win)
    ws = pa.decode_workspace_bytes(B, hq, hkv, d, bs, W, mcl, ps, win)
    bound = _attend_bound(W, bs, mcl, win)
    assert P > 0 and P % 64 == 0
    if ps > 0:
        assert P == ps
    parts = -(-bound // P)
    if parts == 1:
        assert ws == 0
    else:
        assert ws % 256 == 0 and ws >= B * hq * parts * (d + 2) * 4
    if ps > 0:  # monotone in the hint and the window (the automatic size may switch)
        if mcl > 0:  # a hint of 0 means the table's capacity, which may exceed mcl + 4096
            assert ws <= pa.decode_workspace_bytes(B, hq, hkv, d, bs, W, mcl + 4096, ps, win)
        if win > 0:
            assert ws <= pa.decode_workspace_bytes(B, hq, hkv, d, bs, W, mcl, ps, win + 4096)


@settings(max_examples=300, derandomize=True, deadline=None)
@given(B=st.integers(1, 300), G=st.sampled_from([1, 2, 4, 8]), hkv=st.integers(1, 8),
       bs=st.sampled_from([8, 16, 64, 512]), W=st.integers(1, 600),
       ps=st.sampled_from([0, 64, 256, 1024]), win=st.sampled_from([0, 0, 0, 300]),
       mcl_extra=st.integers(-1, 200), seed=st.integers(0, 2**31 - 1))
def test_planned_units(lib, B, G, hkv, bs, W, ps, win, mcl_extra, seed):
    """The host plan of pa_decode_planned: when it is used, every (sequence, partition)
    unit a context needs appears exactly once with its partition count.  Leaving out at
    least 30% of the grid: full partitions first in partition-major order, then the last
    partitions by decreasing length; leaving out less: partition 0 of every sequence in
    order, then each later partition index by decreasing length.  Not used under a window
    or when the grid has no empty row."""
    rng = np.random.default_rng(seed)
    cap = W * bs
    lens = np.minimum(rng.integers(0, cap + 1, size=B), cap).astype(np.int32)
    if rng.random() < 0.3:
        lens[rng.integers(0, B)] = 0
    mcl = 0 if mcl_extra < 0 else int(lens.max()) + mcl_extra
    hq = G * hkv
    units = pa.decode_planned_units(lens, hq, hkv, 128, bs, W, mcl, win, ps)
    P = pa.decode_partition_tokens(B, hq, hkv, 128, bs, W, mcl, ps, win)
    bound = _attend_bound(W, bs, mcl, win)
    parts = -(-bound // P)
    need = [max(1, -(-min(int(L), bound) // P)) for L in lens]
    need = [min(n, parts) for n in need]
    fits = parts <= 255 and sum(need) <= 4096
    if win > 0 or not fits or sum(need) == B * parts:
        assert units.size == 0
        return
    assert units.size == sum(need)
    su, pu, nu = units >> 16, (units >> 8) & 0xFF, units & 0xFF
    seen = sorted(zip(su.tolist(), pu.tolist()))
    assert seen == sorted((s, p) for s in range(B) for p in range(need[s]))
    assert all(int(nu[i]) == need[int(su[i])] for i in range(units.size))
    size = np.array([min(P, int(lens[s]) - int(p) * P) for s, p in zip(su, pu)])
    if 10 * sum(need) <= 7 * B * parts:  # longest first
        full = size == P
        k = int(full.sum())
        assert full[:k].all() and not full[k:].any()  # full partitions first
        fp = list(zip(pu[:k].tolist(), su[:k].tolist()))
        assert fp == sorted(fp)                       # partition-major, then sequence
        assert np.all(np.diff(size[k:]) <= 0)         # the rest by decreasing length
    else:  # the full grid's order without its empty rows
        assert np.all(np.diff(pu.astype(np.int64)) >= 0)
        assert su[pu == 0].tolist() == list(range(B))
        for p in range(1, parts):
            assert np.all(np.diff(size[pu == p]) <= 0)


def test_planned_units_on_the_benchmark_workloads(lib):
    """GQA (lognormal lengths) and the long contexts are planned longest first, the
    Llama-2 step (75% of its grid rows real) in the grid's order; windowed calls and
    one-partition contexts keep the full grid."""
    from workloads import make_config
    for name, kw, planned in (("gqa_llama3_8b", {"block_size": 16}, True),
                              ("long_8_1", {"block_size": 512}, True),
                              ("llama2_7b", {}, True), ("prefix_cow", {}, False)):
        c = make_config(name, poison=False, **kw)
        u = pa.decode_planned_units(c.context_lens, c.num_q_heads, c.num_kv_heads, c.head_dim,
                                    c.block_size, c.max_blocks_per_seq, c.max_context_len)
        assert (u.size > 0) == planned, name
        w = pa.decode_planned_units(c.context_lens, c.num_q_heads, c.num_kv_heads, c.head_dim,
                                    c.block_size, c.max_blocks_per_seq, c.max_context_len,
                                    sliding_window=4096)
        assert w.size == 0
    assert pa.decode_planned_units(np.zeros(0, np.int32), 8, 2, 128, 16, 4).size == 0
    with pytest.raises(pa.PAError):
        pa.decode_planned_units(np.ones(3, np.int32), 6, 2, 128, 16, 4)  # group 3
