"""The Python binding's marshalling and argument checks, on CPU.

A stand-in library records the arguments each entry point receives, so the test can
check what the binding passes (shapes, token strides, pointers, byte counts, dtype
code, stream) and that every malformed call is refused with PAError before anything
reaches the library.  The real library's own checks are covered by the host tests of
libpa and, on the GPU, by the parity tests."""
from __future__ import annotations

import types

import numpy as np
import pytest
import torch

from paged_kv_cache_441_b200 import _lib

STREAM = types.SimpleNamespace(cuda_stream=0x5EED)


class FakeLib:
    """Records (name, args) of every call; answers the size queries with fixed numbers."""

    def __init__(self, workspace_bytes=0):
        self.calls = []
        self.workspace_bytes = workspace_bytes

    def __getattr__(self, name):
        if not name.startswith("pa_"):
            raise AttributeError(name)

        def call(*args):
            self.calls.append((name, args))
            if name == "pa_decode_workspace_bytes":
                return self.workspace_bytes
            if name == "pa_status_str":
                return b"stand-in status"
            return 0
        return call

    def last(self, name):
        got = [a for n, a in self.calls if n == name]
        assert got, f"{name} was not called"
        return got[-1]


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(_lib, "_lib", lib)
    monkeypatch.setattr(_lib, "_DEVICE_TYPE", "cpu")
    return lib


def _v(x):
    """Value of a marshalled argument (ctypes pointer or plain number)."""
    return x.value if hasattr(x, "value") else x


def _decode_args(B=3, hq=8, hkv=2, d=64, nb=10, bs=16, W=5, dtype=torch.bfloat16):
    q = torch.zeros(B, hq, d, dtype=dtype)
    return dict(out=torch.empty_like(q), q=q, k_cache=torch.zeros(nb, hkv, bs, d, dtype=dtype),
                v_cache=torch.zeros(nb, hkv, bs, d, dtype=dtype),
                block_tables=torch.zeros(B, W, dtype=torch.int32),
                context_lens=torch.ones(B, dtype=torch.int32))


def test_decode_marshalling(fake):
    fake.workspace_bytes = 4096
    a = _decode_args()
    ws = torch.empty(1024, dtype=torch.float32)  # 4096 bytes, counted in bytes not elements
    _lib.decode(**a, scale=0.125, max_context_len=77, partition_size=128, workspace=ws,
                stream=STREAM, sliding_window=33)
    args = [_v(x) for x in fake.last("pa_decode")]
    assert args[0] == a["out"].data_ptr() and args[1] == a["q"].data_ptr()
    assert args[4] == a["block_tables"].data_ptr() and args[5] == a["context_lens"].data_ptr()
    assert args[6:13] == [3, 8, 2, 64, 16, 10, 5]  # B, Hq, Hkv, d, bs, NB, W
    assert args[13] == pytest.approx(0.125)
    assert args[14:17] == [77, 33, 128]  # max_context_len, sliding_window, partition_size
    assert args[17] == ws.data_ptr() and args[18] == 4096
    assert args[19] == _lib.PA_BF16 and args[20] == STREAM.cuda_stream
    # the workspace query saw the same plan inputs, in the C argument order
    assert [_v(x) for x in fake.last("pa_decode_workspace_bytes")] == [3, 8, 2, 64, 16, 5, 77,
                                                                       33, 128]


def test_decode_allocates_workspace_when_needed(fake):
    fake.workspace_bytes = 300
    _lib.decode(**_decode_args(dtype=torch.float16), scale=0.1, stream=STREAM)
    args = [_v(x) for x in fake.last("pa_decode")]
    assert args[18] == 300 and args[17] and args[19] == _lib.PA_FP16
    fake.workspace_bytes = 0
    _lib.decode(**_decode_args(), scale=0.1, stream=STREAM)
    args = [_v(x) for x in fake.last("pa_decode")]
    assert args[17] is None and args[18] == 0


def test_kv_write_passes_token_strides(fake):
    T, hkv, d = 4, 2, 64
    qkv = torch.zeros(T, 3 * hkv, d, dtype=torch.bfloat16)  # key and value slices of one row
    key, value = qkv[:, hkv:2 * hkv], qkv[:, 2 * hkv:]
    kc = torch.zeros(6, hkv, 16, d, dtype=torch.bfloat16)
    sm = torch.arange(T, dtype=torch.int64)
    _lib.kv_write(key, value, sm, kc, torch.zeros_like(kc), stream=STREAM)
    args = [_v(x) for x in fake.last("pa_kv_write")]
    assert args[0] == key.data_ptr() and args[1] == value.data_ptr()
    assert args[3:8] == [T, hkv, d, 3 * hkv * d, 3 * hkv * d]
    assert args[10:12] == [6, 16]


def test_decode_append_and_prefill_marshalling(fake):
    a = _decode_args()
    key = torch.zeros(3, 2, 64, dtype=torch.bfloat16)
    _lib.decode_append(a["out"], a["q"], key, torch.zeros_like(key), a["k_cache"], a["v_cache"],
                       a["block_tables"], a["context_lens"], 0.2, stream=STREAM)
    args = [_v(x) for x in fake.last("pa_decode_append")]
    assert args[4:6] == [2 * 64, 2 * 64] and args[10:17] == [3, 8, 2, 64, 16, 10, 5]
    q = torch.zeros(11, 8, 64, dtype=torch.bfloat16)
    qsl = torch.tensor([0, 5, 11], dtype=torch.int32)
    bt = torch.zeros(2, 7, dtype=torch.int32)
    cl = torch.tensor([5, 20], dtype=torch.int32)
    _lib.prefill(torch.empty_like(q), q, a["k_cache"], a["v_cache"], bt, cl, qsl, 0.125,
                 sliding_window=9, stream=STREAM)
    args = [_v(x) for x in fake.last("pa_prefill")]
    assert args[6] == qsl.data_ptr()
    assert args[7:15] == [2, 11, 8, 2, 64, 16, 10, 7]  # B, T, Hq, Hkv, d, bs, NB, W
    assert args[16] == 9


def test_decode_cow_marshalling(fake):
    a = _decode_args()
    cow = torch.tensor([[4, 1, 8], [-1, 0, 0], [7, 0, 16]], dtype=torch.int32)
    _lib.decode_cow(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                    a["context_lens"], cow, 0.2, stream=STREAM)
    args = [_v(x) for x in fake.last("pa_decode_cow")]
    assert args[2] is None and args[3] is None and args[4:6] == [0, 0]  # no cache write
    assert args[10] == cow.data_ptr() and args[11:18] == [3, 8, 2, 64, 16, 10, 5]
    key = torch.zeros(3, 2, 64, dtype=torch.bfloat16)
    _lib.decode_cow(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                    a["context_lens"], cow, 0.2, key=key, value=torch.zeros_like(key),
                    stream=STREAM)
    args = [_v(x) for x in fake.last("pa_decode_cow")]
    assert args[2] == key.data_ptr() and args[4:6] == [2 * 64, 2 * 64]
    with pytest.raises(_lib.PAError, match="together"):
        _lib.decode_cow(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                        a["context_lens"], cow, 0.2, key=key, stream=STREAM)
    with pytest.raises(_lib.PAError, match=r"must be \[3, 3\]"):
        _lib.decode_cow(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                        a["context_lens"], cow[:2], 0.2, stream=STREAM)
    with pytest.raises(_lib.PAError, match="int32"):
        _lib.decode_cow(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                        a["context_lens"], cow.long(), 0.2, stream=STREAM)


def test_decode_planned_marshalling(fake):
    a = _decode_args()
    hl = np.array([3, 40, 17], np.int32)
    _lib.decode_planned(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                        a["context_lens"], hl, 0.2, stream=STREAM)
    args = [_v(x) for x in fake.last("pa_decode_planned")]
    assert args[2] is None and args[3] is None and args[4:6] == [0, 0]
    assert args[10] == hl.ctypes.data and args[11:18] == [3, 8, 2, 64, 16, 10, 5]
    key = torch.zeros(3, 2, 64, dtype=torch.bfloat16)
    _lib.decode_planned(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                        a["context_lens"], torch.from_numpy(hl), 0.2, key=key,
                        value=torch.zeros_like(key), stream=STREAM)
    args = [_v(x) for x in fake.last("pa_decode_planned")]
    assert args[2] == key.data_ptr() and args[4:6] == [2 * 64, 2 * 64]
    with pytest.raises(_lib.PAError, match="int32"):
        _lib.decode_planned(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                            a["context_lens"], hl.astype(np.int64), 0.2, stream=STREAM)
    with pytest.raises(_lib.PAError, match="together"):
        _lib.decode_planned(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                            a["context_lens"], hl, 0.2, value=key, stream=STREAM)


def test_swap_blocks_host_and_device_pools(fake):
    dev_k = torch.zeros(8, 2, 16, 64, dtype=torch.bfloat16)
    host_k = torch.zeros(5, 2, 16, 64, dtype=torch.bfloat16)
    pairs = torch.tensor([[1, 4], [2, 0]], dtype=torch.int64)
    _lib.swap_blocks(host_k, host_k.clone(), dev_k, dev_k.clone(), pairs, stream=STREAM)
    args = [_v(x) for x in fake.last("pa_swap_blocks")]
    assert args[5:11] == [2, 2, 16, 64, 8, 5]  # P, Hkv, bs, d, source NB, destination NB
    with pytest.raises(_lib.PAError, match="differ in shape"):
        _lib.swap_blocks(torch.zeros(5, 2, 8, 64, dtype=torch.bfloat16),
                         torch.zeros(5, 2, 8, 64, dtype=torch.bfloat16), dev_k, dev_k, pairs,
                         stream=STREAM)


REJECTS = {
    "int64 block table": (dict(block_tables=torch.zeros(3, 5, dtype=torch.int64)),
                          "expected torch.int32"),
    "int64 lengths": (dict(context_lens=torch.ones(3, dtype=torch.int64)), "expected torch.int32"),
    "short lengths": (dict(context_lens=torch.ones(2, dtype=torch.int32)), r"must be \[3\]"),
    "table rows": (dict(block_tables=torch.zeros(2, 5, dtype=torch.int32)), "must be"),
    "strided table": (dict(block_tables=torch.zeros(3, 10, dtype=torch.int32)[:, ::2]),
                      "contiguous"),
    "out shape": (dict(out=torch.zeros(3, 4, 64, dtype=torch.bfloat16)), "must both be"),
    "mixed dtypes": (dict(out=torch.zeros(3, 8, 64, dtype=torch.float16)), "expected torch"),
    "float32": (dict(out=torch.zeros(3, 8, 64), q=torch.zeros(3, 8, 64),
                     k_cache=torch.zeros(10, 2, 16, 64), v_cache=torch.zeros(10, 2, 16, 64)),
                "unsupported dtype"),
    "strided q": (dict(q=torch.zeros(3, 16, 64, dtype=torch.bfloat16)[:, ::2],
                       out=torch.zeros(3, 8, 64, dtype=torch.bfloat16)), "contiguous"),
    "v cache shape": (dict(v_cache=torch.zeros(10, 2, 32, 64, dtype=torch.bfloat16)),
                      "must both be"),
    "head_dim": (dict(k_cache=torch.zeros(10, 2, 16, 128, dtype=torch.bfloat16),
                      v_cache=torch.zeros(10, 2, 16, 128, dtype=torch.bfloat16)), "head_dim"),
}


@pytest.mark.parametrize("name", list(REJECTS))
def test_decode_rejects(fake, name):
    over, pattern = REJECTS[name]
    a = {**_decode_args(), **over}
    with pytest.raises(_lib.PAError, match=pattern):
        _lib.decode(**a, scale=0.1, stream=STREAM)
    assert not any(n == "pa_decode" for n, _ in fake.calls)


def test_other_rejects(fake):
    a = _decode_args()
    key = torch.zeros(3, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(_lib.PAError, match="contiguous heads"):  # heads not contiguous
        _lib.kv_write(key.transpose(1, 2).contiguous().transpose(1, 2), key,
                      torch.zeros(3, dtype=torch.int64), a["k_cache"], a["v_cache"], stream=STREAM)
    with pytest.raises(_lib.PAError, match="expected torch.int64"):
        _lib.kv_write(key, key, torch.zeros(3, dtype=torch.int32), a["k_cache"], a["v_cache"],
                      stream=STREAM)
    with pytest.raises(_lib.PAError, match="kv heads"):
        _lib.kv_write(torch.zeros(3, 4, 64, dtype=torch.bfloat16),
                      torch.zeros(3, 4, 64, dtype=torch.bfloat16),
                      torch.zeros(3, dtype=torch.int64), a["k_cache"], a["v_cache"], stream=STREAM)
    with pytest.raises(_lib.PAError, match=r"\[P, 2\]"):
        _lib.copy_blocks(a["k_cache"], a["v_cache"], torch.zeros(4, dtype=torch.int64),
                         stream=STREAM)
    with pytest.raises(_lib.PAError, match="must both be"):  # fused write of the wrong batch
        _lib.decode_append(a["out"], a["q"], key[:2], key[:2], a["k_cache"], a["v_cache"],
                           a["block_tables"], a["context_lens"], 0.1, stream=STREAM)
    q = torch.zeros(11, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(_lib.PAError, match="query_start_loc"):
        _lib.prefill(torch.empty_like(q), q, a["k_cache"], a["v_cache"],
                     torch.zeros(2, 7, dtype=torch.int32), torch.ones(2, dtype=torch.int32),
                     torch.zeros(2, dtype=torch.int32), 0.1, stream=STREAM)
    fake.workspace_bytes = _lib.STATIC_SCRATCH_BYTES + 1
    with pytest.raises(_lib.PAError, match="scratch"):
        _lib.decode_static_scratch(**a, scale=0.1, stream=STREAM)
    assert [n for n, _ in fake.calls if not n.endswith("_bytes")] == []


def test_host_tensors_never_reach_the_library(monkeypatch):
    """With the real device rule (CUDA), host tensors are refused before any call: a host
    pointer handed to a kernel would fault the GPU."""
    lib = FakeLib()
    monkeypatch.setattr(_lib, "_lib", lib)
    a = _decode_args()
    with pytest.raises(_lib.PAError, match="cuda device"):
        _lib.decode(**a, scale=0.1, stream=STREAM)
    with pytest.raises(_lib.PAError, match="cuda device"):
        _lib.copy_blocks(a["k_cache"], a["v_cache"], torch.zeros(1, 2, dtype=torch.int64),
                         stream=STREAM)
    assert lib.calls == []
