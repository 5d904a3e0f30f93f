"""A small serving loop on the GPU driven by the host block manager: prompts, parallel
samples (forks), decode steps with copy-on-write and cache writes, frees and new
arrivals.  Every step's attention is compared with the oracle on a host mirror of the
caches; the device caches must equal the mirror bit for bit."""
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


@pytest.mark.parametrize("hq,hkv,bs,fused,preempt,window", [(16, 4, 16, False, False, 0),
                                                            (8, 8, 32, True, False, 0),
                                                            (32, 4, 16, True, False, 0),
                                                            (16, 2, 16, True, True, 0),
                                                            (8, 8, 32, False, False, 37),
                                                            (16, 4, 16, True, True, 100)])
def test_block_manager_serving_loop(hq, hkv, bs, fused, preempt, window):
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
        slots, pairs = bm.append_slots(live)
        if pairs.shape[0]:
            oracle.copy_blocks(kc_h, vc_h, pairs)
            pa.copy_blocks(kc, vc, dev(pairs))
        key = _rand_bits(rng, (len(live), hkv, d))
        val = _rand_bits(rng, (len(live), hkv, d))
        oracle.kv_write(key, val, slots, kc_h, vc_h)
        bt, cl = bm.block_tables(live, width)
        q = _rand_bits(rng, (len(live), hq, d))
        out = torch.empty(len(live), hq, d, dtype=torch.bfloat16, device="cuda")
        if fused:  # cache write fused into the decode
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
