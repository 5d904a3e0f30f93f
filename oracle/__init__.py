"""CPU oracle for the paged KV-cache decode path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline use it; the library never does.  Two independent statements of the same
definition live here:

* ``pa_oracle.c`` (loaded through ctypes, fp64, optional OpenMP): the reference
  that parity tests compare against;
* ``oracle_np.py`` (numpy fp64): a second, separately written statement that pins
  the C code on small inputs.

Neither imports or links anything of the CUDA library.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build_oracle import build as _build

_lib = None

FP16, BF16 = 0, 1


def _dt(dtype: str) -> int:
    return {"fp16": FP16, "bf16": BF16}[dtype]


def load(path: str | None = None):
    """Load (building if needed) the C oracle; ``path`` selects another build."""
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
        _declare(lib)
        return lib
    if _lib is None:
        _lib = ctypes.CDLL(_build())
        _declare(_lib)
    return _lib


def _declare(lib):
    P = ctypes.c_void_p
    i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.orc_kv_write.argtypes = [P, P, P, i32, i32, i32, i64, i64, P, P, i32, i32]
    lib.orc_kv_write.restype = i32
    lib.orc_copy_blocks.argtypes = [P, P, P, i32, i32, i32, i32, i32]
    lib.orc_copy_blocks.restype = i32
    lib.orc_copy_rows.argtypes = [P, P, P, i32, i32, i32, i32, i32]
    lib.orc_copy_rows.restype = i32
    lib.orc_decode.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, dbl, i32, P,
                               i32, i32]
    lib.orc_decode.restype = i32
    lib.orc_decode_window.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, dbl,
                                      i32, i32, P, i32, i32]
    lib.orc_decode_window.restype = i32
    lib.orc_prefill.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, i32, dbl,
                                i32, i32, P, i32, i32]
    lib.orc_prefill.restype = i32
    lib.orc_max_threads.argtypes = []
    lib.orc_max_threads.restype = i32


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def kv_write(key, value, slot_mapping, k_cache, v_cache, lib=None) -> int:
    """In place on ``k_cache``/``v_cache`` (uint16 [NB, Hkv, bs, d]); returns #bad slots."""
    lib = lib or load()
    key = np.ascontiguousarray(key, np.uint16)
    value = np.ascontiguousarray(value, np.uint16)
    sm = np.ascontiguousarray(slot_mapping, np.int64)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    nb, hkv, bs, d = k_cache.shape
    T = sm.shape[0]
    return lib.orc_kv_write(_p(key), _p(value), _p(sm), T, hkv, d, hkv * d, hkv * d,
                            _p(k_cache), _p(v_cache), nb, bs)


def copy_blocks(k_cache, v_cache, pairs, lib=None) -> int:
    lib = lib or load()
    pairs = np.ascontiguousarray(pairs, np.int64).reshape(-1, 2)
    nb, hkv, bs, d = k_cache.shape
    return lib.orc_copy_blocks(_p(k_cache), _p(v_cache), _p(pairs), pairs.shape[0], hkv, bs, d, nb)


def copy_rows(k_cache, v_cache, triples, lib=None) -> int:
    """In place: for each (src, dst, rows), the first ``rows`` slots of every kv head of block
    dst := block src's (the copy-on-write of a block's filled rows); returns #bad triples."""
    lib = lib or load()
    triples = np.ascontiguousarray(triples, np.int64).reshape(-1, 3)
    nb, hkv, bs, d = k_cache.shape
    return lib.orc_copy_rows(_p(k_cache), _p(v_cache), _p(triples), triples.shape[0], hkv, bs,
                             d, nb)


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, dtype, num_q_heads=None,
           sel=None, nthreads=0, lib=None, return_bad=False, sliding_window=0):
    """fp64 attention output, [B, Hq, d] (or [len(sel), d] for selected (s, h) pairs).
    ``sliding_window`` > 0: each query attends to the last that many tokens only."""
    lib = lib or load()
    q = np.ascontiguousarray(q, np.uint16)
    kc = np.ascontiguousarray(k_cache, np.uint16)
    vc = np.ascontiguousarray(v_cache, np.uint16)
    bt = np.ascontiguousarray(block_tables, np.int32)
    cl = np.ascontiguousarray(context_lens, np.int32)
    B, hq, d = q.shape
    nb, hkv, bs, _ = kc.shape
    if sel is not None:
        sel = np.ascontiguousarray(sel, np.int32).reshape(-1, 2)
        out = np.zeros((sel.shape[0], d), np.float64)
        bad = lib.orc_decode_window(_p(out), _p(q), _p(kc), _p(vc), _p(bt), _p(cl), B, hq, hkv,
                                    d, bs, nb, bt.shape[1], float(scale), _dt(dtype),
                                    int(sliding_window), _p(sel), sel.shape[0], nthreads)
    else:
        out = np.zeros((B, hq, d), np.float64)
        bad = lib.orc_decode_window(_p(out), _p(q), _p(kc), _p(vc), _p(bt), _p(cl), B, hq, hkv,
                                    d, bs, nb, bt.shape[1], float(scale), _dt(dtype),
                                    int(sliding_window), None, 0, nthreads)
    return (out, bad) if return_bad else out


def prefill(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale, dtype,
            sliding_window=0, sel=None, nthreads=0, lib=None, return_bad=False):
    """fp64 causal multi-query attention, [num_tokens, Hq, d] (or [len(sel), d] for the
    selected (token, head) pairs): token i of sequence s sits at position
    context_lens[s] - n_s + i and attends to positions up to its own."""
    lib = lib or load()
    q = np.ascontiguousarray(q, np.uint16)
    kc = np.ascontiguousarray(k_cache, np.uint16)
    vc = np.ascontiguousarray(v_cache, np.uint16)
    bt = np.ascontiguousarray(block_tables, np.int32)
    cl = np.ascontiguousarray(context_lens, np.int32)
    qsl = np.ascontiguousarray(query_start_loc, np.int32)
    T, hq, d = q.shape
    nb, hkv, bs, _ = kc.shape
    if sel is not None:
        sel = np.ascontiguousarray(sel, np.int32).reshape(-1, 2)
        out = np.zeros((sel.shape[0], d), np.float64)
        bad = lib.orc_prefill(_p(out), _p(q), _p(kc), _p(vc), _p(bt), _p(cl), _p(qsl),
                              qsl.shape[0] - 1, T, hq, hkv, d, bs, nb, bt.shape[1], float(scale),
                              _dt(dtype), int(sliding_window), _p(sel), sel.shape[0], nthreads)
    else:
        out = np.zeros((T, hq, d), np.float64)
        bad = lib.orc_prefill(_p(out), _p(q), _p(kc), _p(vc), _p(bt), _p(cl), _p(qsl),
                              qsl.shape[0] - 1, T, hq, hkv, d, bs, nb, bt.shape[1], float(scale),
                              _dt(dtype), int(sliding_window), None, 0, nthreads)
    return (out, bad) if return_bad else out


def max_threads(lib=None) -> int:
    return (lib or load()).orc_max_threads()


def step(case, sel=None, nthreads=0, lib=None):
    """One decode step of a workload case on copies of its caches:
    copy-on-write pairs, cache write, then attention.  Returns (out, k_cache, v_cache)."""
    kc = case.k_cache.copy()
    vc = case.v_cache.copy()
    if case.copy_pairs.shape[0]:
        copy_blocks(kc, vc, case.copy_pairs, lib=lib)
    kv_write(case.key, case.value, case.slot_mapping, kc, vc, lib=lib)
    out = decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale, case.dtype,
                 sel=sel, nthreads=nthreads, lib=lib)
    return out, kc, vc
