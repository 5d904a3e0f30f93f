"""Helpers for the GPU tests: move a workload case to the device and run one step
(copy-on-write pairs, cache write, decode) through the libpa binding."""
from __future__ import annotations

import numpy as np

TOL = {"bf16": 1e-2, "fp16": 2e-3}  # max-abs vs the fp64 oracle (after output rounding)


def torch_dtype(dtype: str):
    import torch
    return {"bf16": torch.bfloat16, "fp16": torch.float16}[dtype]


def dev16(a: np.ndarray, dtype: str, device="cuda"):
    """uint16 bit patterns -> CUDA tensor of the 16-bit float type (same bits)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(
        torch_dtype(dtype))


def dev(a: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bits(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t) -> np.ndarray:
    import torch
    return t.to(torch.float64).cpu().numpy()


class DeviceCase:
    def __init__(self, case, device="cuda"):
        import torch
        self.case = case
        dt = case.dtype
        self.q = dev16(case.q, dt, device)
        self.k_cache = dev16(case.k_cache, dt, device)
        self.v_cache = dev16(case.v_cache, dt, device)
        self.key = dev16(case.key, dt, device)
        self.value = dev16(case.value, dt, device)
        self.slot_mapping = dev(case.slot_mapping.astype(np.int64), device)
        self.block_tables = dev(case.block_tables.astype(np.int32), device)
        self.context_lens = dev(case.context_lens.astype(np.int32), device)
        self.pairs = dev(case.copy_pairs.astype(np.int64).reshape(-1, 2), device)
        self.out = torch.empty_like(self.q)

    def step(self, partition_size=0, max_context_len=None, workspace=None, sliding_window=0):
        import paged_kv_cache_441_b200 as pa
        c = self.case
        if self.pairs.shape[0]:
            pa.copy_blocks(self.k_cache, self.v_cache, self.pairs)
        pa.kv_write(self.key, self.value, self.slot_mapping, self.k_cache, self.v_cache)
        self.decode(partition_size, max_context_len, workspace, sliding_window)
        return self.out

    def decode(self, partition_size=0, max_context_len=None, workspace=None, sliding_window=0):
        import torch
        import paged_kv_cache_441_b200 as pa
        c = self.case
        mcl = c.max_context_len if max_context_len is None else max_context_len
        if workspace is None:
            # all-ones bytes = NaN floats: nothing may be read that this call did not write
            # (except the dynamic split's counters, which must start at zero)
            need = pa.decode_workspace_bytes(c.num_seqs, c.num_q_heads, c.num_kv_heads,
                                             c.head_dim, c.block_size, c.max_blocks_per_seq,
                                             mcl, partition_size, sliding_window)
            workspace = torch.full((max(need, 256),), 255, dtype=torch.uint8, device=self.q.device)
            if partition_size == pa.PARTITION_DYNAMIC:
                workspace[:pa.WORKSPACE_ZERO_BYTES] = 0
        pa.decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables,
                  self.context_lens, c.scale, max_context_len=mcl,
                  partition_size=partition_size, workspace=workspace,
                  sliding_window=sliding_window)
        return self.out
