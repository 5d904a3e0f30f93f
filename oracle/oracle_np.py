"""Second, independent CPU statement of paged decode attention (numpy, fp64).

TEST INFRASTRUCTURE ONLY.  Written separately from ``pa_oracle.c`` so that the two
pin each other on small inputs.  It follows the same passages of the vLLM
paged-attention pages: the "IO-5 vLLM Paged Attention" note, section 3 (each
sequence owns a list of page indices) and section 4 (K = the pages concatenated in
table order, then softmax(q K^T / sqrt(d_k)) V unchanged).

Here the gather is done with numpy fancy indexing over whole pages, and the softmax
with numpy reductions, instead of the C code's per-token loops.
"""
from __future__ import annotations

import numpy as np


def widen(bits: np.ndarray, dtype: str) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def gather(cache_f64: np.ndarray, table_row: np.ndarray, L: int, kv_head: int) -> np.ndarray:
    """Contiguous [L, d] K (or V) of one sequence and kv head: pages in table order."""
    bs = cache_f64.shape[2]
    npages = -(-L // bs)
    pages = cache_f64[np.asarray(table_row[:npages], dtype=np.int64), kv_head]  # [npages, bs, d]
    return pages.reshape(npages * bs, -1)[:L]


def gather_positions(cache_f64: np.ndarray, table_row: np.ndarray, lo: int, L: int,
                     kv_head: int) -> np.ndarray:
    """[L - lo, d] rows of token positions lo .. L-1: page table_row[t // bs], row t % bs."""
    bs = cache_f64.shape[2]
    t = np.arange(lo, L)
    pages = np.asarray(table_row, dtype=np.int64)[t // bs]
    return cache_f64[pages, kv_head, t % bs]


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, dtype,
           sliding_window: int = 0) -> np.ndarray:
    """sliding_window > 0: each query attends to its last ``sliding_window`` tokens."""
    qf = widen(q, dtype)
    kf = widen(k_cache, dtype)
    vf = widen(v_cache, dtype)
    B, hq, d = qf.shape
    hkv = kf.shape[1]
    G = hq // hkv
    out = np.zeros((B, hq, d), np.float64)
    for s in range(B):
        L = int(context_lens[s])
        if L == 0:
            continue
        lo = L - sliding_window if 0 < sliding_window < L else 0
        for g in range(hkv):
            if lo == 0:
                K = gather(kf, block_tables[s], L, g)
                V = gather(vf, block_tables[s], L, g)
            else:
                K = gather_positions(kf, block_tables[s], lo, L, g)
                V = gather_positions(vf, block_tables[s], lo, L, g)
            Q = qf[s, g * G:(g + 1) * G]  # [G, d]
            z = scale * (Q @ K.T)  # [G, L]
            z = z - z.max(axis=1, keepdims=True)
            w = np.exp(z)
            out[s, g * G:(g + 1) * G] = (w @ V) / w.sum(axis=1, keepdims=True)
    return out


def prefill(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale, dtype,
            sliding_window: int = 0) -> np.ndarray:
    """Causal multi-query attention: per sequence, the chunk Q [n, Hq, d] against the whole
    gathered context K, V [L, d], with the score matrix masked where key t is after the
    query's position L - n + i (or more than sliding_window - 1 before it)."""
    qf = widen(q, dtype)
    kf = widen(k_cache, dtype)
    vf = widen(v_cache, dtype)
    T, hq, d = qf.shape
    hkv = kf.shape[1]
    G = hq // hkv
    out = np.zeros((T, hq, d), np.float64)
    qsl = np.asarray(query_start_loc, dtype=np.int64)
    for s in range(len(qsl) - 1):
        a, b = int(qsl[s]), int(qsl[s + 1])
        n, L = b - a, int(context_lens[s])
        if n == 0:
            continue
        # the earliest position any query of the chunk attends (pages before it are
        # never read: under a window they may have been given back)
        lo = max(0, L - n - sliding_window + 1) if sliding_window > 0 else 0
        pos = np.arange(L - n, L)[:, None]  # [n, 1]
        t = np.arange(lo, L)[None, :]  # [1, L - lo]
        allowed = t <= pos
        if sliding_window > 0:
            allowed &= t > pos - sliding_window
        for g in range(hkv):
            K = gather_positions(kf, block_tables[s], lo, L, g)
            V = gather_positions(vf, block_tables[s], lo, L, g)
            Q = qf[a:b, g * G:(g + 1) * G]  # [n, G, d]
            z = scale * np.einsum("ngd,td->ngt", Q, K)
            z = np.where(allowed[:, None, :], z, -np.inf)
            z = z - z.max(axis=2, keepdims=True)
            w = np.exp(z)
            out[a:b, g * G:(g + 1) * G] = np.einsum("ngt,td->ngd", w, V) / w.sum(axis=2)[..., None]
    return out


def kv_write(key, value, slot_mapping, k_cache, v_cache) -> None:
    bs = k_cache.shape[2]
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        blk, off = divmod(int(slot), bs)
        k_cache[blk, :, off, :] = key[t]
        v_cache[blk, :, off, :] = value[t]


def copy_blocks(k_cache, v_cache, pairs) -> None:
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2):
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]


def copy_rows(k_cache, v_cache, triples) -> None:
    """Copy-on-write of the filled rows: block dst's first ``rows`` slots of every kv head
    take block src's; its other slots keep their values."""
    for src, dst, rows in np.asarray(triples, dtype=np.int64).reshape(-1, 3):
        k_cache[dst, :, :rows] = k_cache[src, :, :rows]
        v_cache[dst, :, :rows] = v_cache[src, :, :rows]
