"""Checks that tie the C oracle to facts fixed outside itself.

Each ``pin_*`` takes a loaded oracle library (ctypes handle) and raises
``AssertionError`` when the oracle disagrees with:

* closed forms (two tokens, one token, identical keys, zero length);
* a library routine on the contiguous layout (torch fp64 scaled-dot-product
  attention on K/V that were built contiguous first and only then scattered into
  pages);
* invariants the pages state (paging leaves the attention unchanged: any block
  size, any physical permutation, shared prefix blocks);
* the worked examples the pages print (``tests/golden/pages_examples.txt``);
* exact library conversions of the 16-bit formats (numpy float16, torch bfloat16);
* the independent numpy statement in ``oracle/oracle_np.py``;
* for the sliding window: the last token's V exactly at W = 1, and torch fp64
  attention on the last W contiguous rows;
* for multi-query (prefill) attention: torch fp64 attention with its causal path or
  a tril/triu mask on the contiguous K/V, and the one-token chunk equal to decode.

The same functions run against deliberately broken copies of the oracle in
``test_oracle_mutants.py``, which checks that each plausible mistake trips a pin.
"""
from __future__ import annotations

import math
import os

import numpy as np

import oracle
from oracle import oracle_np
from workloads import bits_to_f32, make_config, round_to_bits

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "pages_examples.txt")


def read_golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, *kv = line.split()
            rows.append((kind, dict(x.split("=", 1) for x in kv)))
    return rows


def _scatter_pages(contig, table, nb, bs, fill):
    """contig: [L, Hkv, d] per sequence -> writes pages into a [nb, Hkv, bs, d] pool.

    Pads the sequence to whole pages, reshapes to [pages, bs, Hkv, d] and assigns
    page j to physical block table[j]."""
    L, hkv, d = contig.shape
    npg = -(-L // bs)
    pad = np.full((npg * bs, hkv, d), fill, np.uint16)
    pad[:L] = contig
    pages = pad.reshape(npg, bs, hkv, d).transpose(0, 2, 1, 3)
    return [(int(table[j]), pages[j]) for j in range(npg)]


def build_pool(Ks, Vs, tables, nb, bs, fill=0x7FC0):
    hkv, d = Ks[0].shape[1], Ks[0].shape[2]
    kc = np.full((nb, hkv, bs, d), fill, np.uint16)
    vc = np.full((nb, hkv, bs, d), fill, np.uint16)
    for K, V, tab in zip(Ks, Vs, tables):
        for blk, page in _scatter_pages(K, tab, nb, bs, fill):
            kc[blk] = page
        for blk, page in _scatter_pages(V, tab, nb, bs, fill):
            vc[blk] = page
    width = max(len(t) for t in tables)
    bt = np.full((len(tables), width), -1, np.int32)
    for s, t in enumerate(tables):
        bt[s, :len(t)] = t
    return kc, vc, bt


def _rand_bits(rng, shape, dtype="bf16"):
    return round_to_bits(rng.standard_normal(shape).astype(np.float32), dtype)


def _tables_for(rng, lens, bs, nb):
    perm = rng.permutation(nb)
    out, pos = [], 0
    for L in lens:
        n = -(-L // bs)
        out.append(perm[pos:pos + n].astype(np.int32))
        pos += n
    return out


# ----------------------------------------------------------------------------- closed forms

def pin_two_token(lib):
    """out = sigma(z0 - z1) v0 + sigma(z1 - z0) v1 with hand-picked exact values,
    the two tokens in separate physical pages stored in reverse order; plus a second
    query head sharing the kv head (GQA mapping)."""
    q = np.array([[1.0, 0.5, -1.0, 2.0], [0.25, -2.0, 1.5, 0.0]], np.float32)
    k = np.array([[0.5, 1.0, 0.0, -0.25], [-1.0, 0.25, 0.5, 1.0]], np.float32)
    v = np.array([[1.0, 2.0, 3.0, 4.0], [-2.0, 0.5, 0.0, 8.0]], np.float32)
    scale = 0.5
    kc = np.full((8, 1, 1, 4), 0x7FC0, np.uint16)
    vc = np.full((8, 1, 1, 4), 0x7FC0, np.uint16)
    kc[5, 0, 0] = round_to_bits(k[0], "bf16")
    kc[2, 0, 0] = round_to_bits(k[1], "bf16")
    vc[5, 0, 0] = round_to_bits(v[0], "bf16")
    vc[2, 0, 0] = round_to_bits(v[1], "bf16")
    bt = np.array([[5, 2]], np.int32)
    qb = round_to_bits(q, "bf16").reshape(1, 2, 4)
    out = oracle.decode(qb, kc, vc, bt, np.array([2], np.int32), scale, "bf16", lib=lib)
    for h in range(2):
        z0 = scale * float(np.dot(q[h].astype(np.float64), k[0]))
        z1 = scale * float(np.dot(q[h].astype(np.float64), k[1]))
        a = 1.0 / (1.0 + math.exp(-(z0 - z1)))
        b = 1.0 / (1.0 + math.exp(-(z1 - z0)))
        want = a * v[0].astype(np.float64) + b * v[1].astype(np.float64)
        assert np.max(np.abs(out[0, h] - want)) < 1e-14, (h, out[0, h], want)


def pin_len1_exact(lib):
    """A context of one token returns that token's V exactly."""
    rng = np.random.default_rng(11)
    for dtype in ("bf16", "fp16"):
        B, hq, hkv, d, bs, nb = 6, 4, 2, 32, 8, 16
        Ks = [_rand_bits(rng, (1, hkv, d), dtype) for _ in range(B)]
        Vs = [_rand_bits(rng, (1, hkv, d), dtype) for _ in range(B)]
        tabs = _tables_for(rng, [1] * B, bs, nb)
        kc, vc, bt = build_pool(Ks, Vs, tabs, nb, bs)
        q = _rand_bits(rng, (B, hq, d), dtype)
        out = oracle.decode(q, kc, vc, bt, np.ones(B, np.int32), 0.125, dtype, lib=lib)
        G = hq // hkv
        for s in range(B):
            for h in range(hq):
                want = bits_to_f32(Vs[s][0, h // G], dtype).astype(np.float64)
                assert np.array_equal(out[s, h], want), (dtype, s, h)


def pin_identical_keys(lib):
    """All keys equal -> uniform weights -> the mean of V."""
    rng = np.random.default_rng(12)
    L, hkv, d, bs, nb = 37, 1, 16, 8, 9
    krow = _rand_bits(rng, (1, hkv, d))
    K = np.repeat(krow, L, axis=0)
    V = _rand_bits(rng, (L, hkv, d))
    tabs = _tables_for(rng, [L], bs, nb)
    kc, vc, bt = build_pool([K], [V], tabs, nb, bs)
    q = _rand_bits(rng, (1, 1, d))
    out = oracle.decode(q, kc, vc, bt, np.array([L], np.int32), 0.25, "bf16", lib=lib)
    want = bits_to_f32(V[:, 0], "bf16").astype(np.float64).mean(axis=0)
    assert np.max(np.abs(out[0, 0] - want)) < 1e-13


def pin_zero_len(lib):
    """Context length 0 -> all-zero output, no table entry read."""
    rng = np.random.default_rng(13)
    kc = _rand_bits(rng, (4, 1, 8, 16))
    vc = _rand_bits(rng, (4, 1, 8, 16))
    bt = np.array([[99]], np.int32)  # never read
    out, bad = oracle.decode(_rand_bits(rng, (1, 2, 16)), kc, vc, bt, np.array([0], np.int32),
                             0.25, "bf16", lib=lib, return_bad=True)
    assert bad == 0 and np.all(out == 0.0)


# ------------------------------------------------------- library routine on contiguous K/V

def pin_paged_vs_sdpa(lib):
    """Paged result == torch fp64 scaled-dot-product attention on the contiguous K/V
    the pages were cut from (GQA: kv head h // G)."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(14)
    for dtype, (B, hq, hkv, d, bs) in (("bf16", (3, 4, 2, 16, 4)), ("fp16", (4, 8, 1, 24, 8)),
                                       ("bf16", (2, 6, 6, 8, 16))):
        lens = [int(x) for x in rng.integers(1, 40, size=B)]
        nb = sum(-(-L // bs) for L in lens) + 5
        Ks = [_rand_bits(rng, (L, hkv, d), dtype) for L in lens]
        Vs = [_rand_bits(rng, (L, hkv, d), dtype) for L in lens]
        tabs = _tables_for(rng, lens, bs, nb)
        kc, vc, bt = build_pool(Ks, Vs, tabs, nb, bs)
        q = _rand_bits(rng, (B, hq, d), dtype)
        scale = 1.0 / math.sqrt(d)
        out = oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), scale, dtype, lib=lib)
        G = hq // hkv
        for s in range(B):
            qt = torch.from_numpy(bits_to_f32(q[s], dtype).astype(np.float64))[None, :, None, :]
            kt = torch.from_numpy(bits_to_f32(Ks[s], dtype).astype(np.float64))  # [L, hkv, d]
            vt = torch.from_numpy(bits_to_f32(Vs[s], dtype).astype(np.float64))
            kt = kt.permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
            vt = vt.permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
            ref = F.scaled_dot_product_attention(qt, kt, vt, scale=scale)[0, :, 0, :].numpy()
            assert np.max(np.abs(out[s] - ref)) < 1e-12, (dtype, s)


# -------------------------------------------------------------------- paging invariants

def pin_block_size_and_permutation(lib):
    """Same logical K/V at block sizes 1..64 and under two physical permutations give
    the same result (the paged result does not depend on where pages live)."""
    rng = np.random.default_rng(15)
    B, hq, hkv, d = 3, 4, 2, 16
    lens = [45, 64, 3]
    Ks = [_rand_bits(rng, (L, hkv, d)) for L in lens]
    Vs = [_rand_bits(rng, (L, hkv, d)) for L in lens]
    q = _rand_bits(rng, (B, hq, d))
    ref = None
    for bs in (1, 2, 8, 16, 64):
        for trial in range(2):
            nb = sum(-(-L // bs) for L in lens) + 3 + trial
            tabs = _tables_for(rng, lens, bs, nb)
            kc, vc, bt = build_pool(Ks, Vs, tabs, nb, bs)
            out = oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), 0.3, "bf16", lib=lib)
            if ref is None:
                ref = out
            assert np.max(np.abs(out - ref)) < 1e-13, (bs, trial)


def pin_shared_prefix(lib):
    """Sequences whose tables point at the same prefix blocks (or at private copies
    of them) and have the same length give the same output for the same q."""
    rng = np.random.default_rng(16)
    hkv, d, bs, L = 2, 16, 8, 30
    K = _rand_bits(rng, (L, hkv, d))
    V = _rand_bits(rng, (L, hkv, d))
    nb = 16
    tab_shared = np.array([3, 9, 0, 12], np.int32)
    tab_copy = np.array([3, 9, 0, 7], np.int32)  # last page a private copy
    kc, vc, _ = build_pool([K, K], [V, V], [tab_shared, tab_copy], nb, bs)
    bt = np.stack([tab_shared, tab_shared, tab_copy])
    q1 = _rand_bits(rng, (1, 4, d))
    q = np.repeat(q1, 3, axis=0)
    out = oracle.decode(q, kc, vc, bt, np.array([L, L, L], np.int32), 0.25, "bf16", lib=lib)
    assert np.array_equal(out[0], out[1]) and np.array_equal(out[0], out[2])


# --------------------------------------------------------------- worked examples of pages

def pin_golden_examples(lib):
    rng = np.random.default_rng(17)
    for kind, kv in read_golden():
        if kind == "blocks_needed":
            # A 3200-token sequence at block size 512 reads exactly 7 table entries:
            # entry 6 must be valid, entry 7 is never touched.
            L, bs, n = int(kv["seq_len"]), int(kv["block_size"]), int(kv["expect"])
            nb, d = n + 1, 4
            kc = _rand_bits(rng, (nb, 1, bs, d))
            vc = _rand_bits(rng, (nb, 1, bs, d))
            q = _rand_bits(rng, (1, 1, d))
            cl = np.array([L], np.int32)
            bt = np.array([list(range(n)) + [10**6]], np.int32)
            _, bad = oracle.decode(q, kc, vc, bt, cl, 0.5, "bf16", lib=lib, return_bad=True)
            assert bad == 0, "read past the needed blocks"
            bt2 = bt.copy()
            bt2[0, n - 1] = 10**6
            _, bad = oracle.decode(q, kc, vc, bt2, cl, 0.5, "bf16", lib=lib, return_bad=True)
            assert bad == 1, "did not read the last needed block"
        elif kind == "pool_tokens":
            # A pool of 1024 blocks x 512 tokens has slots 0 .. 524287.
            nb, bs, n = int(kv["num_blocks"]), int(kv["block_size"]), int(kv["expect"])
            kc = np.zeros((nb, 1, bs, 2), np.uint16)
            vc = np.zeros((nb, 1, bs, 2), np.uint16)
            key = np.full((3, 1, 2), 0x3F80, np.uint16)
            sm = np.array([n - 1, n, 0], np.int64)
            bad = oracle.kv_write(key, key, sm, kc, vc, lib=lib)
            assert bad == 1
            assert kc[nb - 1, 0, bs - 1, 0] == 0x3F80 and kc[0, 0, 0, 0] == 0x3F80
            assert int((kc != 0).sum()) == 4
    # Request A -> pages 1, 5, 9; request B -> pages 2, 3: attention over
    # concat(K_page1, K_page5, K_page9) equals attention over those rows directly.
    tabs = {kv["seq"]: [int(x) for x in kv["pages"].split(",")]
            for kind, kv in read_golden() if kind == "page_table"}
    bs, d, nb = 2, 8, 10
    kc = _rand_bits(rng, (nb, 1, bs, d))
    vc = _rand_bits(rng, (nb, 1, bs, d))
    q = _rand_bits(rng, (2, 1, d))
    bt = np.full((2, 3), -1, np.int32)
    bt[0, :3] = tabs["A"]
    bt[1, :2] = tabs["B"]
    lens = np.array([6, 4], np.int32)
    out = oracle.decode(q, kc, vc, bt, lens, 0.5, "bf16", lib=lib)
    for s, name in enumerate(("A", "B")):
        K = np.concatenate([bits_to_f32(kc[p, 0], "bf16") for p in tabs[name]]).astype(np.float64)
        V = np.concatenate([bits_to_f32(vc[p, 0], "bf16") for p in tabs[name]]).astype(np.float64)
        z = 0.5 * (K @ bits_to_f32(q[s, 0], "bf16").astype(np.float64))
        w = np.exp(z - z.max())
        want = (w / w.sum()) @ V
        assert np.max(np.abs(out[s, 0] - want)) < 1e-13, name


# ----------------------------------------------------------------- exact 16-bit widening

def pin_widening(lib):
    """Every fp16 / bf16 bit pattern widens like numpy float16 / torch bfloat16."""
    import torch
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    d = 64
    n = 65536 // d
    for dtype in ("fp16", "bf16"):
        vc = pats.reshape(n, 1, 1, d).copy()
        kc = np.zeros_like(vc)
        bt = np.arange(n, dtype=np.int32).reshape(n, 1)
        q = np.zeros((n, 1, d), np.uint16)
        out = oracle.decode(q, kc, vc, bt, np.ones(n, np.int32), 1.0, dtype, lib=lib)
        if dtype == "fp16":
            want = pats.view(np.float16).astype(np.float64)
        else:
            want = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).to(
                torch.float64).numpy()
        np.testing.assert_array_equal(out.reshape(-1), want)


# ------------------------------------------------------------ second statement (numpy)

def pin_c_vs_numpy(lib):
    cases = [make_config("tiny")]
    rng = np.random.default_rng(18)
    for dtype, (B, hq, hkv, d, bs) in (("bf16", (5, 8, 2, 32, 8)), ("fp16", (3, 4, 4, 16, 4))):
        lens = [int(x) for x in rng.integers(0, 50, size=B)]
        nb = sum(-(-L // bs) for L in lens) + 4
        Ks = [_rand_bits(rng, (L, hkv, d), dtype) for L in lens]
        Vs = [_rand_bits(rng, (L, hkv, d), dtype) for L in lens]
        tabs = _tables_for(rng, lens, bs, nb)
        tabs = [t if len(t) else np.array([0], np.int32) for t in tabs]
        Ks = [k if k.shape[0] else np.zeros((1, hkv, d), np.uint16) for k in Ks]
        Vs = [v if v.shape[0] else np.zeros((1, hkv, d), np.uint16) for v in Vs]
        kc, vc, bt = build_pool(Ks, Vs, tabs, nb, bs)
        q = _rand_bits(rng, (B, hq, d), dtype)
        cases.append((q, kc, vc, bt, np.array(lens, np.int32), 0.2, dtype))
    for c in cases:
        if isinstance(c, tuple):
            q, kc, vc, bt, cl, scale, dtype = c
        else:
            kc, vc = c.k_cache.copy(), c.v_cache.copy()
            oracle.kv_write(c.key, c.value, c.slot_mapping, kc, vc, lib=lib)
            q, bt, cl, scale, dtype = c.q, c.block_tables, c.context_lens, c.scale, c.dtype
        a = oracle.decode(q, kc, vc, bt, cl, scale, dtype, lib=lib)
        b = oracle_np.decode(q, kc, vc, bt, cl, scale, dtype)
        assert np.max(np.abs(a - b)) < 1e-12


# ------------------------------------------------------------- cache write / block copy

def pin_kv_write(lib):
    rng = np.random.default_rng(19)
    nb, hkv, bs, d = 6, 2, 4, 8
    # slots 0..nb*bs-1 in order fill the pool like a reshape of the token stream
    T = nb * bs
    key = _rand_bits(rng, (T, hkv, d))
    val = _rand_bits(rng, (T, hkv, d))
    kc = np.zeros((nb, hkv, bs, d), np.uint16)
    vc = np.zeros((nb, hkv, bs, d), np.uint16)
    assert oracle.kv_write(key, val, np.arange(T), kc, vc, lib=lib) == 0
    assert np.array_equal(kc, key.reshape(nb, bs, hkv, d).transpose(0, 2, 1, 3))
    assert np.array_equal(vc, val.reshape(nb, bs, hkv, d).transpose(0, 2, 1, 3))
    # a shuffled slot map with skips and one out-of-range slot, vs the numpy statement
    sm = rng.permutation(T).astype(np.int64)[:10]
    sm[3] = -1
    sm[7] = T + 5
    key2 = _rand_bits(rng, (10, hkv, d))
    val2 = _rand_bits(rng, (10, hkv, d))
    kc_c, vc_c = kc.copy(), vc.copy()
    bad = oracle.kv_write(key2, val2, sm, kc_c, vc_c, lib=lib)
    assert bad == 1
    kc_n, vc_n = kc.copy(), vc.copy()
    sm_n = sm.copy()
    sm_n[7] = -1
    oracle_np.kv_write(key2, val2, sm_n, kc_n, vc_n)
    assert np.array_equal(kc_c, kc_n) and np.array_equal(vc_c, vc_n)


def pin_copy_blocks(lib):
    rng = np.random.default_rng(20)
    nb, hkv, bs, d = 10, 2, 4, 8
    kc = _rand_bits(rng, (nb, hkv, bs, d))
    vc = _rand_bits(rng, (nb, hkv, bs, d))
    pairs = np.array([[1, 4], [2, 7], [1, 9], [3, 99]], np.int64)
    kc_c, vc_c = kc.copy(), vc.copy()
    assert oracle.copy_blocks(kc_c, vc_c, pairs, lib=lib) == 1
    for s, t in ((1, 4), (2, 7), (1, 9)):
        assert np.array_equal(kc_c[t], kc[s]) and np.array_equal(vc_c[t], vc[s])
    for b in (0, 1, 2, 3, 5, 6, 8):
        assert np.array_equal(kc_c[b], kc[b]) and np.array_equal(vc_c[b], vc[b])


def pin_copy_rows(lib):
    """The filled-rows copy: the listed rows of every head come from the source, the rest
    of the destination and every other block keep their values, bad triples are skipped
    and counted; a whole block's rows equal the block copy; the C and numpy statements
    agree."""
    rng = np.random.default_rng(21)
    nb, hkv, bs, d = 10, 3, 4, 8
    kc = _rand_bits(rng, (nb, hkv, bs, d))
    vc = _rand_bits(rng, (nb, hkv, bs, d))
    triples = np.array([[1, 4, 3], [2, 7, 0], [5, 9, 4], [3, 99, 1], [3, 6, 5]], np.int64)
    kc_c, vc_c = kc.copy(), vc.copy()
    assert oracle.copy_rows(kc_c, vc_c, triples, lib=lib) == 2
    for h in range(hkv):
        for r in range(bs):
            src = kc[1] if r < 3 else kc[4]
            assert np.array_equal(kc_c[4, h, r], src[h, r])
            assert np.array_equal(vc_c[4, h, r], (vc[1] if r < 3 else vc[4])[h, r])
    assert np.array_equal(kc_c[9], kc[5]) and np.array_equal(vc_c[9], vc[5])
    for b in (0, 1, 2, 3, 5, 6, 7, 8):
        assert np.array_equal(kc_c[b], kc[b]) and np.array_equal(vc_c[b], vc[b])
    kb, vb = kc.copy(), vc.copy()
    oracle.copy_blocks(kb, vb, np.array([[5, 9]], np.int64), lib=lib)
    assert np.array_equal(kb[9], kc_c[9]) and np.array_equal(vb[9], vc_c[9])
    kn, vn = kc.copy(), vc.copy()
    oracle_np.copy_rows(kn, vn, triples[[0, 1, 2]])
    assert np.array_equal(kn, kc_c) and np.array_equal(vn, vc_c)


# ------------------------------------------------------------------ sliding window

def _recycle_before(tables, lens, bs, window):
    """Table entries of pages wholly before each sequence's window -> -1 (returned to the
    pool): page j is unused once (j + 1) * bs <= L - window."""
    out = []
    for t, L in zip(tables, lens):
        t = t.copy()
        lo = L - window if 0 < window < L else 0
        t[:lo // bs] = -1
        out.append(t)
    return out


def pin_window_last_token(lib):
    """A window of one token returns the last token's V exactly, whatever the length and
    whatever the (recycled, -1) table entries before it hold."""
    rng = np.random.default_rng(21)
    for dtype in ("bf16", "fp16"):
        hq, hkv, d, bs = 4, 2, 16, 8
        lens = [1, 7, 8, 9, 16, 17, 37]
        B = len(lens)
        nb = sum(-(-L // bs) for L in lens) + 2
        Ks = [_rand_bits(rng, (L, hkv, d), dtype) for L in lens]
        Vs = [_rand_bits(rng, (L, hkv, d), dtype) for L in lens]
        tabs = _tables_for(rng, lens, bs, nb)
        kc, vc, _ = build_pool(Ks, Vs, tabs, nb, bs)
        _, _, bt = build_pool(Ks, Vs, _recycle_before(tabs, lens, bs, 1), nb, bs)
        q = _rand_bits(rng, (B, hq, d), dtype)
        out, bad = oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), 0.25, dtype, lib=lib,
                                 return_bad=True, sliding_window=1)
        assert bad == 0
        G = hq // hkv
        for s, L in enumerate(lens):
            for h in range(hq):
                want = bits_to_f32(Vs[s][L - 1, h // G], dtype).astype(np.float64)
                assert np.array_equal(out[s, h], want), (dtype, s, h)


def pin_window_vs_sdpa(lib):
    """Windowed paged result == torch fp64 scaled-dot-product attention on the last W
    rows of the contiguous K/V, with the pages before the window recycled (-1); a
    window at least as long as the context is the plain result."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(22)
    hq, hkv, d, bs = 4, 2, 16, 4
    lens = [1, 5, 12, 13, 30, 41]
    B = len(lens)
    nb = sum(-(-L // bs) for L in lens) + 3
    Ks = [_rand_bits(rng, (L, hkv, d)) for L in lens]
    Vs = [_rand_bits(rng, (L, hkv, d)) for L in lens]
    tabs = _tables_for(rng, lens, bs, nb)
    kc, vc, bt_full = build_pool(Ks, Vs, tabs, nb, bs)
    q = _rand_bits(rng, (B, hq, d))
    cl = np.array(lens, np.int32)
    G = hq // hkv
    plain = oracle.decode(q, kc, vc, bt_full, cl, 0.3, "bf16", lib=lib)
    for W in (2, 3, 4, 9, 12, 40, 41, 100):
        _, _, bt = build_pool(Ks, Vs, _recycle_before(tabs, lens, bs, W), nb, bs)
        out, bad = oracle.decode(q, kc, vc, bt, cl, 0.3, "bf16", lib=lib, return_bad=True,
                                 sliding_window=W)
        assert bad == 0, W
        for s, L in enumerate(lens):
            lo = max(0, L - W)
            qt = torch.from_numpy(bits_to_f32(q[s], "bf16").astype(np.float64))[None, :, None, :]
            kt = torch.from_numpy(bits_to_f32(Ks[s][lo:], "bf16").astype(np.float64))
            vt = torch.from_numpy(bits_to_f32(Vs[s][lo:], "bf16").astype(np.float64))
            kt = kt.permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
            vt = vt.permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
            ref = F.scaled_dot_product_attention(qt, kt, vt, scale=0.3)[0, :, 0, :].numpy()
            assert np.max(np.abs(out[s] - ref)) < 1e-12, (W, s)
            if W >= L:
                assert np.array_equal(out[s], plain[s]), (W, s)
        npv = oracle_np.decode(q, kc, vc, bt, cl, 0.3, "bf16", sliding_window=W)
        assert np.max(np.abs(out - npv)) < 1e-12, W


# ------------------------------------------------------------- multi-query (prefill)

def _prefill_case(rng, specs, hq, hkv, d, bs, dtype="bf16"):
    """specs: [(n, L)] per sequence -> contiguous K/V, pool, tables, q, qsl."""
    lens = [L for _, L in specs]
    nb = sum(-(-L // bs) for L in lens) + 3
    Ks = [_rand_bits(rng, (L, hkv, d), dtype) for L in lens]
    Vs = [_rand_bits(rng, (L, hkv, d), dtype) for L in lens]
    tabs = _tables_for(rng, lens, bs, nb)
    kc, vc, bt = build_pool(Ks, Vs, tabs, nb, bs)
    qsl = np.concatenate([[0], np.cumsum([n for n, _ in specs])]).astype(np.int32)
    q = _rand_bits(rng, (int(qsl[-1]), hq, d), dtype)
    return Ks, Vs, tabs, kc, vc, bt, q, qsl, np.array(lens, np.int32)


def pin_prefill_vs_sdpa(lib):
    """Causal multi-query attention == torch fp64 scaled-dot-product attention on the
    contiguous K/V: torch's own causal path when the chunk is the whole context, a
    lower-triangular mask aligned to the last query (torch.tril) for a chunk that
    follows earlier context, and that mask cut to the last W keys (torch.triu) under a
    sliding window, with the pages before the first query's window given back (-1)."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(23)
    hq, hkv, d, bs = 4, 2, 16, 4
    specs = [(9, 9), (5, 13), (1, 7), (17, 17), (3, 30)]
    Ks, Vs, tabs, kc, vc, bt_full, q, qsl, cl = _prefill_case(rng, specs, hq, hkv, d, bs)
    G = hq // hkv
    for W in (0, 1, 3, 7, 100):
        bt = bt_full.copy()
        if W:
            for s, (n, L) in enumerate(specs):
                lo = max(0, L - n - W + 1)
                bt[s, :lo // bs] = -1
        out, bad = oracle.prefill(q, kc, vc, bt, cl, qsl, 0.3, "bf16", sliding_window=W,
                                  lib=lib, return_bad=True)
        assert bad == 0, W
        for s, (n, L) in enumerate(specs):
            a = int(qsl[s])
            qt = torch.from_numpy(bits_to_f32(q[a:a + n], "bf16").astype(np.float64))
            qt = qt.permute(1, 0, 2)[None]  # [1, hq, n, d]
            kt = torch.from_numpy(bits_to_f32(Ks[s], "bf16").astype(np.float64))
            vt = torch.from_numpy(bits_to_f32(Vs[s], "bf16").astype(np.float64))
            kt = kt.permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
            vt = vt.permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
            if W == 0 and n == L:
                ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.3)
            else:
                mask = torch.ones(n, L, dtype=torch.bool).tril(diagonal=L - n)
                if W:
                    mask &= torch.ones(n, L, dtype=torch.bool).triu(diagonal=L - n - W + 1)
                ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.3)
            ref = ref[0].permute(1, 0, 2).numpy()  # [n, hq, d]
            assert np.max(np.abs(out[a:a + n] - ref)) < 1e-12, (W, s)
        npv = oracle_np.prefill(q, kc, vc, bt, cl, qsl, 0.3, "bf16", sliding_window=W)
        assert np.max(np.abs(out - npv)) < 1e-12, W


def pin_prefill_one_token_is_decode(lib):
    """A chunk of one token at the end of its context is the decode step (whose oracle
    the decode pins tie down), with and without a window."""
    rng = np.random.default_rng(24)
    specs = [(1, 1), (1, 8), (1, 9), (1, 40)]
    _, _, _, kc, vc, bt, q, qsl, cl = _prefill_case(rng, specs, 8, 2, 16, 8)
    for W in (0, 5):
        a = oracle.prefill(q, kc, vc, bt, cl, qsl, 0.25, "bf16", sliding_window=W, lib=lib)
        b = oracle.decode(q, kc, vc, bt, cl, 0.25, "bf16", sliding_window=W, lib=lib)
        assert np.array_equal(a, b), W


ALL_PINS = [pin_two_token, pin_len1_exact, pin_identical_keys, pin_zero_len, pin_paged_vs_sdpa,
            pin_block_size_and_permutation, pin_shared_prefix, pin_golden_examples,
            pin_widening, pin_c_vs_numpy, pin_kv_write, pin_copy_blocks, pin_copy_rows,
            pin_window_last_token,
            pin_window_vs_sdpa, pin_prefill_vs_sdpa, pin_prefill_one_token_is_decode]


def run_all(lib):
    """Names of the pins that fail (or crash) for this oracle build."""
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except Exception as e:  # noqa: BLE001 - any failure counts
            failed.append(f"{pin.__name__}: {type(e).__name__}")
    return failed
