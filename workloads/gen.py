"""Seeded generators for paged decode workloads.

Layout produced (the library's layout):

* ``k_cache``, ``v_cache``: ``uint16 [num_blocks, num_kv_heads, block_size, head_dim]``
  holding bf16 or fp16 bit patterns; one (block, kv head) is one contiguous run.
* ``block_tables``: ``int32 [num_seqs, max_blocks_per_seq]``; entry ``j`` of row ``s``
  is the physical block holding logical tokens ``[j*bs, (j+1)*bs)`` of sequence ``s``
  ("Sequence -> [page indices]", page 3 section 3 of the vLLM paged-attention note).
  Entries past ``ceil(L/bs)`` are ``-1``.
* ``context_lens``: ``int32 [num_seqs]``, counting the token appended in this step.
* ``key``/``value``: ``uint16 [T, num_kv_heads, head_dim]`` new tokens, ``slot_mapping``:
  ``int64 [T]`` with ``slot = block * block_size + offset``.
* ``copy_pairs``: ``int64 [P, 2]`` (src, dst) copy-on-write block pairs; ``cow``:
  ``int32 [num_seqs, 3]`` the same copies per sequence (source block, logical block
  index, rows), source ``-1`` for none.

Draw order for a seed: context lengths, the pool permutation, q, K pool, V pool, the
new tokens' key, value.  Values are N(0, 1) in fp32 rounded to nearest-even; an array
of more than 2^24 values takes one key from the seed's stream and draws its chunks of
2^24 values from generators seeded with (key, chunk index), on host threads.

Poisoning (``poison=True``): every cache slot that the decode step must not read
(spare blocks, slots at or past ``L-1`` of each sequence's last block, and slot
``L-1`` itself, which the step's cache write fills) holds NaN, so any over-read or
a missing write shows up as NaN in the result.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

NAN_BITS = {"bf16": 0x7FC0, "fp16": 0x7E00}
_CHUNK = 1 << 24


def round_to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """fp32 -> 16-bit pattern, round to nearest even (finite inputs)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "fp16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        u = x.view(np.uint32)
        r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
        return r.astype(np.uint16)
    raise ValueError(dtype)


def bits_to_f32(b: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit pattern -> fp32 (exact widening)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    if dtype == "fp16":
        return b.view(np.float16).astype(np.float32)
    if dtype == "bf16":
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)
    raise ValueError(dtype)


def _draw(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0, 1) values rounded to `dtype`.  Up to _CHUNK values come from `rng` itself;
    a larger array takes one 63-bit key from `rng` and fills chunk i from a generator
    seeded with (key, i), on host threads, so the values do not depend on the thread
    count."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    if n <= _CHUNK:
        out[:] = round_to_bits(rng.standard_normal(n, dtype=np.float32), dtype)
        return out.reshape(shape)
    key = int(rng.integers(0, 2**63 - 1))

    def fill(i: int) -> None:
        m = min(_CHUNK, n - i)
        sub = np.random.default_rng([key, i // _CHUNK])
        out[i:i + m] = round_to_bits(sub.standard_normal(m, dtype=np.float32), dtype)

    workers = max(1, min(16, os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(fill, range(0, n, _CHUNK)))
    return out.reshape(shape)


@dataclass
class DecodeCase:
    name: str
    dtype: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    context_lens: np.ndarray
    block_tables: np.ndarray
    q: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray
    key: np.ndarray
    value: np.ndarray
    slot_mapping: np.ndarray
    copy_pairs: np.ndarray = field(default_factory=lambda: np.zeros((0, 2), np.int64))
    # the same copies per sequence, for a decode that does them itself: int32 [B, 3] =
    # (source block, logical block index, rows to copy), source -1 for none; empty when
    # the case has no copies
    cow: np.ndarray = field(default_factory=lambda: np.zeros((0, 3), np.int32))
    seed: int = 0
    window: int = 0  # sliding window the decode uses (0 = whole contexts)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def _blocks_needed(lens: np.ndarray, bs: int) -> np.ndarray:
    # Ceil division as on page 2 ("(seq_len + block_size - 1) // block_size").
    return (lens.astype(np.int64) + bs - 1) // bs


def _poison(k_cache, v_cache, tables, lens, bs, dtype):
    """NaN in every slot except positions [0, L-1) of each sequence (in the pages it
    holds: table entries of -1 have no block)."""
    nan = NAN_BITS[dtype]
    nb = k_cache.shape[0]
    keep = np.zeros((nb, bs), dtype=bool)
    for s in range(len(lens)):
        n_keep = max(int(lens[s]) - 1, 0)
        if n_keep == 0:
            continue
        nblk = (n_keep + bs - 1) // bs
        ids = tables[s, :nblk]
        full = ids[:-1]
        keep[full[full >= 0], :] = True
        last = n_keep - (nblk - 1) * bs
        if ids[-1] >= 0:
            keep[ids[-1], :last] = True
    kill = ~keep
    k_cache.transpose(0, 2, 1, 3)[kill] = nan
    v_cache.transpose(0, 2, 1, 3)[kill] = nan


def make_case(name: str, seed: int, num_seqs: int, num_q_heads: int, num_kv_heads: int,
              head_dim: int, block_size: int, lens_fn, dtype: str = "bf16",
              scale: float | None = None, spare: float = 0.10, num_blocks: int | None = None,
              poison: bool = True, window: int = 0) -> DecodeCase:
    """Generic decode-step case: one new token per sequence, written at L-1.

    window > 0: the sequences hold only the pages of their last `window` positions, as
    the block manager leaves them under that sliding window; the table entries of the
    pages before are -1 and the pool is sized for the held pages."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens_fn(rng), dtype=np.int32)
    assert lens.shape == (num_seqs,)
    bs = block_size
    nblk = _blocks_needed(lens, bs)
    dead = (np.maximum(lens.astype(np.int64) - window, 0) // bs if window > 0
            else np.zeros_like(nblk))
    total = int((nblk - dead).sum())
    nb = num_blocks if num_blocks is not None else max(int(math.ceil((1.0 + spare) * total)), 1)
    assert nb >= total
    perm = rng.permutation(nb).astype(np.int32)
    width = max(int(nblk.max()) if num_seqs else 1, 1)
    tables = np.full((num_seqs, width), -1, dtype=np.int32)
    pos = 0
    for s in range(num_seqs):
        n, d0 = int(nblk[s]), int(dead[s])
        tables[s, d0:n] = perm[pos:pos + n - d0]
        pos += n - d0
    q = _draw(rng, (num_seqs, num_q_heads, head_dim), dtype)
    k_cache = _draw(rng, (nb, num_kv_heads, bs, head_dim), dtype)
    v_cache = _draw(rng, (nb, num_kv_heads, bs, head_dim), dtype)
    key = _draw(rng, (num_seqs, num_kv_heads, head_dim), dtype)
    value = _draw(rng, (num_seqs, num_kv_heads, head_dim), dtype)
    slots = np.full(num_seqs, -1, dtype=np.int64)
    for s in range(num_seqs):
        L = int(lens[s])
        if L > 0:
            slots[s] = int(tables[s, (L - 1) // bs]) * bs + (L - 1) % bs
    if poison:
        _poison(k_cache, v_cache, tables, lens, bs, dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return DecodeCase(name, dtype, num_seqs, num_q_heads, num_kv_heads, head_dim, bs, nb,
                      float(scale), lens, tables, q, k_cache, v_cache, key, value, slots,
                      seed=seed, window=window)


def make_prefix_cow(seed: int = 5, groups: int = 64, samples: int = 8, prefix: int = 1000,
                    max_suffix: int = 256, num_q_heads: int = 32, num_kv_heads: int = 8,
                    head_dim: int = 128, block_size: int = 16, dtype: str = "bf16",
                    spare: float = 0.10, poison: bool = True) -> DecodeCase:
    """Parallel sampling over a shared prompt, at the step where the samples diverge.

    Each group's prompt of ``prefix`` tokens sits in shared blocks (reference count
    ``samples``); its last block is partially filled.  Samples ``0..samples-2`` get a
    private copy of that block (``copy_pairs``), the last sample keeps the original;
    ``cow`` names the same copies per sample, restricted to the prompt's rows of the
    block (the rows past them receive the sample's own tokens in this step).
    Each sample then has ``u ~ U{0..max_suffix}`` suffix tokens plus the new token,
    ``L = prefix + u + 1``.  The step is: copy the pairs, write the tokens that land in
    the (copied) partial block plus the new token, decode.  Suffix tokens that land in
    later, private blocks already hold values.
    """
    bs = block_size
    rng = np.random.default_rng(seed)
    nseq = groups * samples
    u = rng.integers(0, max_suffix, endpoint=True, size=nseq)
    lens = (prefix + u + 1).astype(np.int32)
    n_full = prefix // bs
    part_fill = prefix - n_full * bs
    assert part_fill > 0, "prefix must end inside a block"
    n_shared = n_full + 1
    part_end = (n_full + 1) * bs  # first position past the partial block
    fresh = [int(max(0, int(L) - part_end) + bs - 1) // bs for L in lens]
    total = groups * n_shared + groups * (samples - 1) + sum(fresh)
    nb = int(math.ceil((1.0 + spare) * total))
    perm = rng.permutation(nb).astype(np.int32)
    width = int(max(n_shared + f for f in fresh))
    tables = np.full((nseq, width), -1, dtype=np.int32)
    pairs = []
    cow = np.full((nseq, 3), -1, dtype=np.int32)
    cow[:, 1:] = 0
    pos = 0
    for g in range(groups):
        shared = perm[pos:pos + n_shared]
        pos += n_shared
        for j in range(samples):
            s = g * samples + j
            tables[s, :n_shared] = shared
            if j < samples - 1:
                cp = perm[pos]
                pos += 1
                tables[s, n_full] = cp
                pairs.append((int(shared[-1]), int(cp)))
                cow[s] = (int(shared[-1]), n_full, part_fill)  # the prompt's rows of it
            f = fresh[s]
            tables[s, n_shared:n_shared + f] = perm[pos:pos + f]
            pos += f
    q = _draw(rng, (nseq, num_q_heads, head_dim), dtype)
    k_cache = _draw(rng, (nb, num_kv_heads, bs, head_dim), dtype)
    v_cache = _draw(rng, (nb, num_kv_heads, bs, head_dim), dtype)
    write_pos = []
    for s in range(nseq):
        L = int(lens[s])
        ps = list(range(prefix, min(part_end, L)))
        if L - 1 >= part_end:
            ps.append(L - 1)
        write_pos.append(ps)
    T = sum(len(p) for p in write_pos)
    key = _draw(rng, (T, num_kv_heads, head_dim), dtype)
    value = _draw(rng, (T, num_kv_heads, head_dim), dtype)
    slots = np.empty(T, dtype=np.int64)
    t = 0
    for s in range(nseq):
        for p in write_pos[s]:
            slots[t] = int(tables[s, p // bs]) * bs + p % bs
            t += 1
    if poison:
        nan = NAN_BITS[dtype]
        keep = np.zeros((nb, bs), dtype=bool)
        for s in range(nseq):
            L = int(lens[s])
            # positions already in the cache before the step: [0, prefix) in shared
            # blocks, [part_end, L-1) in private blocks
            for p in list(range(0, prefix)) + list(range(part_end, L - 1)):
                keep[tables[s, p // bs], p % bs] = True
        for src, dst in pairs:
            keep[dst, :] = False
        kill = ~keep
        k_cache.transpose(0, 2, 1, 3)[kill] = nan
        v_cache.transpose(0, 2, 1, 3)[kill] = nan
    return DecodeCase("prefix_cow", dtype, nseq, num_q_heads, num_kv_heads, head_dim, bs, nb,
                      1.0 / math.sqrt(head_dim), lens, tables, q, k_cache, v_cache, key, value,
                      slots, copy_pairs=np.asarray(pairs, dtype=np.int64).reshape(-1, 2),
                      cow=cow, seed=seed)


@dataclass
class PrefillCase:
    """A prefill / chunked-prefill step: sequence s has ``context_lens[s]`` tokens once
    its ``n_s`` new tokens (q rows ``query_start_loc[s] .. [s+1]``) are written; the
    step writes the new tokens' key/value at ``slot_mapping`` and attends causally."""
    name: str
    dtype: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    context_lens: np.ndarray     # int32 [B]
    query_start_loc: np.ndarray  # int32 [B + 1]
    block_tables: np.ndarray     # int32 [B, W]
    q: np.ndarray                # uint16 [T, Hq, d]
    k_cache: np.ndarray
    v_cache: np.ndarray
    key: np.ndarray              # uint16 [T, Hkv, d]
    value: np.ndarray
    slot_mapping: np.ndarray     # int64 [T]
    window: int = 0
    seed: int = 0

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_tokens(self) -> int:
        return int(self.query_start_loc[-1])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])


def make_prefill_case(name: str, seed: int, specs, num_q_heads: int, num_kv_heads: int,
                      head_dim: int, block_size: int, dtype: str = "bf16",
                      spare: float = 0.10, window: int = 0, poison: bool = True) -> PrefillCase:
    """specs: [(n_s, L_s)] -- a chunk of n_s new tokens ending a context of L_s tokens
    (n_s == L_s: the whole prompt).  Draw order: the pool permutation, q, K pool, V
    pool, the new tokens' key, value.  With poison, every slot that is neither one of
    the earlier L_s - n_s tokens nor written by the step holds NaN."""
    bs = block_size
    rng = np.random.default_rng(seed)
    ns = np.array([n for n, _ in specs], np.int64)
    lens = np.array([L for _, L in specs], np.int32)
    assert np.all(ns <= lens) and np.all(ns >= 0)
    nblk = _blocks_needed(lens, bs)
    total = int(nblk.sum())
    nb = max(int(math.ceil((1.0 + spare) * total)), 1)
    perm = rng.permutation(nb).astype(np.int32)
    B = len(specs)
    tables = np.full((B, max(int(nblk.max()) if B else 1, 1)), -1, np.int32)
    pos = 0
    for s in range(B):
        tables[s, :nblk[s]] = perm[pos:pos + nblk[s]]
        pos += int(nblk[s])
    qsl = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
    T = int(qsl[-1])
    q = _draw(rng, (T, num_q_heads, head_dim), dtype)
    k_cache = _draw(rng, (nb, num_kv_heads, bs, head_dim), dtype)
    v_cache = _draw(rng, (nb, num_kv_heads, bs, head_dim), dtype)
    key = _draw(rng, (T, num_kv_heads, head_dim), dtype)
    value = _draw(rng, (T, num_kv_heads, head_dim), dtype)
    slots = np.empty(T, np.int64)
    for s in range(B):
        L, n = int(lens[s]), int(ns[s])
        for i in range(n):
            p = L - n + i
            slots[qsl[s] + i] = int(tables[s, p // bs]) * bs + p % bs
    if poison:
        nan = NAN_BITS[dtype]
        keep = np.zeros((nb, bs), dtype=bool)
        for s in range(B):
            for p in range(int(lens[s]) - int(ns[s])):
                keep[tables[s, p // bs], p % bs] = True
        kill = ~keep
        k_cache.transpose(0, 2, 1, 3)[kill] = nan
        v_cache.transpose(0, 2, 1, 3)[kill] = nan
    return PrefillCase(name, dtype, num_q_heads, num_kv_heads, head_dim, bs, nb,
                       1.0 / math.sqrt(head_dim), lens, qsl, tables, q, k_cache, v_cache, key,
                       value, slots, window=window, seed=seed)


PREFILL_CONFIGS = {
    # whole prompts: 8 sequences of 2048 tokens, Llama-3-8B-shaped GQA heads
    "prefill_2k_gqa": lambda **kw: make_prefill_case(
        "prefill_2k_gqa", kw.pop("seed", 7), [(2048, 2048)] * kw.pop("num_seqs", 8), 32, 8, 128,
        kw.pop("block_size", 16), **kw),
    # chunked prefill: 16 sequences each adding a 512-token chunk to 1536..3072 earlier tokens
    "prefill_chunk512_gqa": lambda **kw: make_prefill_case(
        "prefill_chunk512_gqa", kw.pop("seed", 8),
        [(512, 2048 + 128 * (i % 13)) for i in range(kw.pop("num_seqs", 16))], 32, 8, 128,
        kw.pop("block_size", 16), **kw),
}


def make_prefill_config(name: str, **kw) -> PrefillCase:
    return PREFILL_CONFIGS[name](**kw)


def _lens_const(vals):
    return lambda rng: np.asarray(vals, dtype=np.int32)


def _lens_uniform(lo, hi, n):
    return lambda rng: rng.integers(lo, hi, endpoint=True, size=n).astype(np.int32)


def _lens_lognormal(median, sigma, lo, hi, n):
    def f(rng):
        x = np.exp(rng.normal(math.log(median), sigma, size=n))
        return np.clip(np.rint(x), lo, hi).astype(np.int32)
    return f


# name -> builder(**overrides).  Shapes follow the five workloads of the decode study:
# tiny MHA, Llama-2-7B-shaped MHA, Llama-3-8B-shaped GQA, long-context split-K, and
# prefix sharing with copy-on-write.
CONFIGS = {
    "tiny": lambda **kw: make_case("tiny", kw.pop("seed", 0), 4, 4, 4, 64, 16,
                                   _lens_const([1, 17, 33, 100]), dtype="fp16", scale=1.0 / 8,
                                   num_blocks=64, **kw),
    "llama2_7b": lambda num_seqs=64, **kw: make_case(
        "llama2_7b", kw.pop("seed", 1), num_seqs, 32, 32, 128, kw.pop("block_size", 16),
        _lens_uniform(128, 2048, num_seqs), **kw),
    "gqa_llama3_8b": lambda num_seqs=256, **kw: make_case(
        "gqa_llama3_8b", kw.pop("seed", 2), num_seqs, 32, 8, 128, kw.pop("block_size", 16),
        _lens_lognormal(1024, 1.0, 16, 8192, num_seqs), **kw),
    "long_8_1": lambda num_seqs=8, **kw: make_case(
        "long_8_1", kw.pop("seed", 3), num_seqs, 8, 1, 128, kw.pop("block_size", 16),
        _lens_uniform(32768, 131072, num_seqs), **kw),
    "long_32_8": lambda num_seqs=8, **kw: make_case(
        "long_32_8", kw.pop("seed", 3), num_seqs, 32, 8, 128, kw.pop("block_size", 16),
        _lens_uniform(32768, 131072, num_seqs), **kw),
    # sliding-window decode over long contexts: only the last 4096 positions are held
    "window_4096_gqa": lambda num_seqs=64, **kw: make_case(
        "window_4096_gqa", kw.pop("seed", 6), num_seqs, 32, 8, 128, kw.pop("block_size", 16),
        _lens_uniform(8192, 32768, num_seqs), window=kw.pop("window", 4096), **kw),
    "prefix_cow": lambda num_seqs=None, **kw: make_prefix_cow(
        groups=(kw.pop("groups", 64) if num_seqs is None else max(1, num_seqs // 8)), **kw),
}


def make_config(name: str, **kw) -> DecodeCase:
    return CONFIGS[name](**kw)
