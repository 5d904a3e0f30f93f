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


@pytest.mark.parametrize("hq,hkv,bs,fused", [(16, 4, 16, False), (8, 8, 32, True),
                                             (32, 4, 16, True)])
def test_block_manager_serving_loop(hq, hkv, bs, fused):
    rng = np.random.default_rng(hq * 100 + bs)
    nb, d, width = 700, 128, 64
    scale = 1 / math.sqrt(d)
    bm = pa.BlockManager(nb, bs)
    kc_h = np.full((nb, hkv, bs, d), 0x7FC0, np.uint16)  # NaN where nothing was written
    vc_h = kc_h.copy()
    kc, vc = dev16(kc_h, "bf16"), dev16(vc_h, "bf16")
    live, next_id = [], 0

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
                             vc, dev(bt), dev(cl), scale, max_context_len=int(cl.max()))
        else:
            pa.kv_write(dev16(key, "bf16"), dev16(val, "bf16"), dev(slots), kc, vc)
            pa.decode(out, dev16(q, "bf16"), kc, vc, dev(bt), dev(cl), scale,
                      max_context_len=int(cl.max()), partition_size=128)
        want = oracle.decode(q, kc_h, vc_h, bt, cl, scale, "bf16")
        err = np.max(np.abs(to_f64(out) - want))
        assert np.isfinite(err) and err <= TOL["bf16"], (step, err)
    torch.cuda.synchronize()
    assert pa.device_error(0) == 0
    assert np.array_equal(bits(kc), kc_h) and np.array_equal(bits(vc), vc_h)
