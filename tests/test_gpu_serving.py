"""A small serving loop on the GPU driven by the host block manager: prompts, parallel
samples (forks), decode steps with copy-on-write and cache writes, frees and new
arrivals.  Every step's attention is compared with the oracle on a host mirror of the
caches; the device caches must equal the mirror bit for bit.  With cow=True the step is
one call: the manager's per-sequence copy list and the new tokens go to pa_decode_cow,
which copies, writes and attends."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_441_b200 as pa
from tests.gpu_util import TOL, bits, dev, dev16, to_f64
from tests.pins import _rand_bits

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_swap_blocks_device_and_pinned_host():
    rng = np.random.default_rng(60)
    nb, ncpu, hkv, bs, d = 50, 30, 8, 16, 128
    kd0 = _rand_bits(rng, (nb, hkv, bs, d))
    vd0 = _rand_bits(rng, (nb, hkv, bs, d))
    kd, vd = dev16(kd0, "bf16"), dev16(vd0, "bf16")
    kh = torch.zeros(ncpu, hkv, bs, d, dtype=torch.bfloat16, pin_memory=True)
    vh = torch.zeros_like(kh).pin_memory()
    gpu = rng.permutation(nb)[:12]
    cpu = rng.permutation(ncpu)[:12]
    pa.swap_blocks(kh, vh, kd, vd, dev(np.stack([gpu, cpu], 1).astype(np.int64)))  # out
    torch.cuda.synchronize()
    assert np.array_equal(bits(kh)[cpu], kd0[gpu]) and np.array_equal(bits(vh)[cpu], vd0[gpu])
    kd.zero_()
    vd.zero_()
    back = rng.permutation(nb)[:12]
    pa.swap_blocks(kd, vd, kh, vh, dev(np.stack([cpu, back], 1).astype(np.int64)))  # in
    torch.cuda.synchronize()
    assert np.array_equal(bits(kd)[back], kd0[gpu]) and np.array_equal(bits(vd)[back], vd0[gpu])
    assert pa.device_error(0) == 0
    pageable = torch.zeros(ncpu, hkv, bs, d, dtype=torch.bfloat16)  # not mapped: refused
    with pytest.raises(pa.PAError):
        pa.swap_blocks(pageable, pageable, kd, vd, dev(np.array([[0, 0]], np.int64)))
    pa.swap_blocks(kh, vh, kd, vd, dev(np.array([[0, ncpu]], np.int64)))  # bad host id
    assert pa.device_error(0) == pa.DEVERR["pair"]


@pytest.mark.parametrize("hq,hkv,bs,fused,preempt,window,cow",
                         [(16, 4, 16, False, False, 0, False), (8, 8, 32, True, False, 0, False),
                          (32, 4, 16, True, False, 0, False), (16, 2, 16, True, True, 0, False),
                          (8, 8, 32, False, False, 37, False),
                          (16, 4, 16, True, True, 100, False),
                          (16, 4, 16, True, False, 0, True), (8, 8, 32, True, True, 37, True)])
def test_block_manager_serving_loop(hq, hkv, bs, fused, preempt, window, cow):
    rng = np.random.default_rng(hq * 100 + bs + window)
    nb, d, width, ncpu = 700, 128, 64, 300
    scale = 1 / math.sqrt(d)
    bm = pa.BlockManager(nb, bs)
    bm.set_cpu_pool(ncpu)
    bm.set_sliding_window(window)  # 0: whole contexts
    kc_h = np.full((nb, hkv, bs, d), 0x7FC0, np.uint16)  # NaN where nothing was written
    vc_h = kc_h.copy()
    kc, vc = dev16(kc_h, "bf16"), dev16(vc_h, "bf16")
    kh_h = np.zeros((ncpu, hkv, bs, d), np.uint16)  # host pool mirror and the pinned pool
    vh_h = kh_h.copy()
    kh = torch.zeros(ncpu, hkv, bs, d, dtype=torch.bfloat16, pin_memory=True)
    vh = torch.zeros_like(kh).pin_memory()
    live, next_id, parked = [], 0, []

    def write(ids_tokens_slots):
        key = np.concatenate([k for k, _, _ in ids_tokens_slots])
        val = np.concatenate([v for _, v, _ in ids_tokens_slots])
        sm = np.array([s for _, _, s in ids_tokens_slots], np.int64)
        oracle.kv_write(key, val, sm, kc_h, vc_h)
        pa.kv_write(dev16(key, "bf16"), dev16(val, "bf16"), dev(sm), kc, vc)

    def new_prompt():
        nonlocal next_id
        n = int(rng.integers(20, 400))
        bm.allocate(next_id, n)
        rows = [(_rand_bits(rng, (1, hkv, d)), _rand_bits(rng, (1, hkv, d)), bm.slot(next_id, i))
                for i in range(n)]
        write(rows)
        live.append(next_id)
        next_id += 1
        return next_id - 1

    for _ in range(6):
        p = new_prompt()
        for _ in range(int(rng.integers(0, 4))):
            bm.fork(p, next_id)
            live.append(next_id)
            next_id += 1

    for step in range(10):
        if preempt and step == 2:  # preempt the first prompt and its samples
            group = [s for s in live if bm.block_tables([s], width)[0][0, 0]
                     == bm.block_tables([live[0]], width)[0][0, 0]]
            pairs = bm.swap_out(group)
            for g_blk, c_blk in pairs:
                kh_h[c_blk], vh_h[c_blk] = kc_h[g_blk], vc_h[g_blk]
            pa.swap_blocks(kh, vh, kc, vc, dev(pairs))
            live = [s for s in live if s not in group]
            parked = group
        if preempt and step == 6:  # and bring it back into (other) GPU blocks
            pairs = bm.swap_in(parked)
            for c_blk, g_blk in pairs:
                kc_h[g_blk], vc_h[g_blk] = kh_h[c_blk], vh_h[c_blk]
            pa.swap_blocks(kc, vc, kh, vh, dev(pairs))
            live += parked
            parked = []
        if step % 4 == 3:  # one request ends, one arrives
            bm.free(live.pop(int(rng.integers(0, len(live)))))
            new_prompt()
        if cow:
            slots, cowl = bm.append_slots_cow(live)
            pairs = np.zeros((0, 2), np.int64)
        else:
            slots, pairs = bm.append_slots(live)
        if pairs.shape[0]:
            oracle.copy_blocks(kc_h, vc_h, pairs)
            pa.copy_blocks(kc, vc, dev(pairs))
        key = _rand_bits(rng, (len(live), hkv, d))
        val = _rand_bits(rng, (len(live), hkv, d))
        bt, cl = bm.block_tables(live, width)
        if cow:  # the mirror: the oracle's copy of the listed rows, then the write
            triples = [(src, int(bt[i, lb]), nrows)
                       for i, (src, lb, nrows) in enumerate(cowl.tolist()) if src >= 0]
            if triples:
                assert oracle.copy_rows(kc_h, vc_h, np.array(triples, np.int64)) == 0
        oracle.kv_write(key, val, slots, kc_h, vc_h)
        q = _rand_bits(rng, (len(live), hq, d))
        out = torch.empty(len(live), hq, d, dtype=torch.bfloat16, device="cuda")
        if cow:  # copies, cache write and attention in one call
            pa.decode_cow(out, dev16(q, "bf16"), kc, vc, dev(bt), dev(cl), dev(cowl), scale,
                          key=dev16(key, "bf16"), value=dev16(val, "bf16"),
                          max_context_len=int(cl.max()), partition_size=128,
                          sliding_window=window)
        elif fused:  # cache write fused into the decode
            pa.decode_append(out, dev16(q, "bf16"), dev16(key, "bf16"), dev16(val, "bf16"), kc,
                             vc, dev(bt), dev(cl), scale, max_context_len=int(cl.max()),
                             sliding_window=window)
        else:
            pa.kv_write(dev16(key, "bf16"), dev16(val, "bf16"), dev(slots), kc, vc)
            pa.decode(out, dev16(q, "bf16"), kc, vc, dev(bt), dev(cl), scale,
                      max_context_len=int(cl.max()), partition_size=128,
                      sliding_window=window)
        want, bad = oracle.decode(q, kc_h, vc_h, bt, cl, scale, "bf16", return_bad=True,
                                  sliding_window=window)
        assert bad == 0
        err = np.max(np.abs(to_f64(out) - want))
        assert np.isfinite(err) and err <= TOL["bf16"], (step, err)
    torch.cuda.synchronize()
    assert pa.device_error(0) == 0
    assert np.array_equal(bits(kc), kc_h) and np.array_equal(bits(vc), vc_h)


@pytest.mark.parametrize("window", [0, 50])
def test_engine_loop_prefill_then_decode(window):
    """The block manager drives a whole engine loop on the GPU: prompts arrive and are
    prefilled (whole, or in two chunks), then every live sequence decodes step by step;
    under a sliding window the manager gives back the blocks that fall out of it.  Every
    attention output is checked against the oracle, and the device cache against a host
    mirror."""
    rng = np.random.default_rng(900 + window)
    nb, bs, hq, hkv, d, width = 400, 16, 16, 4, 128, 64
    scale = 1 / math.sqrt(d)
    bm = pa.BlockManager(nb, bs)
    bm.set_sliding_window(window)
    kc_h = np.full((nb, hkv, bs, d), 0x7FC0, np.uint16)
    vc_h = kc_h.copy()
    kc, vc = dev16(kc_h, "bf16"), dev16(vc_h, "bf16")
    live, next_id = [], 0

    def write(key, val, slots):
        oracle.kv_write(key, val, slots, kc_h, vc_h)
        pa.kv_write(dev16(key, "bf16"), dev16(val, "bf16"), dev(slots), kc, vc)

    def prefill_check(sids, chunk_lo, chunk_hi, ctx):
        """Chunk [chunk_lo[i], chunk_hi[i]) of each listed sequence, contexts ctx[i]."""
        n = [h - l for l, h in zip(chunk_lo, chunk_hi)]
        qsl = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
        q = _rand_bits(rng, (int(qsl[-1]), hq, d))
        bt, _ = bm.block_tables(sids, width)
        cl = np.array(ctx, np.int32)
        out = torch.empty(int(qsl[-1]), hq, d, dtype=torch.bfloat16, device="cuda")
        pa.prefill(out, dev16(q, "bf16"), kc, vc, dev(bt), dev(cl), dev(qsl), scale,
                   sliding_window=window)
        want, bad = oracle.prefill(q, kc_h, vc_h, bt, cl, qsl, scale, "bf16",
                                   sliding_window=window, return_bad=True)
        assert bad == 0
        err = np.max(np.abs(to_f64(out) - want))
        assert np.isfinite(err) and err <= TOL["bf16"], err

    def arrive(chunked):
        nonlocal next_id
        n = int(rng.integers(40, 300))
        sid = next_id
        next_id += 1
        bm.allocate(sid, n)
        slots = np.array([bm.slot(sid, i) for i in range(n)], np.int64)
        write(_rand_bits(rng, (n, hkv, d)), _rand_bits(rng, (n, hkv, d)), slots)
        if chunked:  # the first part, then the rest on top of it
            n1 = int(rng.integers(1, n))
            prefill_check([sid], [0], [n1], [n1])
            prefill_check([sid], [n1], [n], [n])
        else:
            prefill_check([sid], [0], [n], [n])
        live.append(sid)

    for k in range(4):
        arrive(chunked=(k % 2 == 1))
    for step in range(12):
        if step % 5 == 4:
            bm.free(live.pop(0))
            arrive(chunked=True)
        slots, pairs = bm.append_slots(live)
        assert pairs.shape[0] == 0  # no sharing in this loop
        key = _rand_bits(rng, (len(live), hkv, d))
        val = _rand_bits(rng, (len(live), hkv, d))
        write(key, val, slots)
        bt, cl = bm.block_tables(live, width)
        q = _rand_bits(rng, (len(live), hq, d))
        out = torch.empty(len(live), hq, d, dtype=torch.bfloat16, device="cuda")
        pa.decode(out, dev16(q, "bf16"), kc, vc, dev(bt), dev(cl), scale,
                  max_context_len=int(cl.max()), sliding_window=window)
        want, bad = oracle.decode(q, kc_h, vc_h, bt, cl, scale, "bf16", return_bad=True,
                                  sliding_window=window)
        assert bad == 0
        err = np.max(np.abs(to_f64(out) - want))
        assert np.isfinite(err) and err <= TOL["bf16"], (step, err)
        if window:  # blocks wholly before every window have gone back to the pool
            held = sum(int((bt[i] >= 0).sum()) for i in range(len(live)))
            need = sum(-(-int(L) // bs) - max(int(L) - window, 0) // bs for L in cl)
            assert held == need
    torch.cuda.synchronize()
    assert pa.device_error(0) == 0
    assert np.array_equal(bits(kc), kc_h) and np.array_equal(bits(vc), vc_h)
