"""The benchmark's algorithmic-work counts against brute-force enumerations on tiny cases:
decode bytes (K/V of every attended token and kv head, q and out, the table entries of the
attended pages, the lengths) and prefill FLOPs (4 d per attended (query, head, key)), with
and without a sliding window."""
import numpy as np

import bench
from workloads import make_case, make_prefill_case


def _decode_bytes_brute(case):
    eb, total = 2, 0
    pages = set()
    for s, L in enumerate(case.context_lens.tolist()):
        lo = L - case.window if 0 < case.window < L else 0
        for t in range(lo, L):
            total += 2 * case.num_kv_heads * case.head_dim * eb  # K and V of every kv head
            pages.add((s, t // case.block_size))
    total += 2 * case.num_seqs * case.num_q_heads * case.head_dim * eb  # q and out
    total += 4 * case.num_kv_heads * len(pages)  # one table entry per page and kv head
    return total + 4 * case.num_seqs


def test_decode_bytes_match_brute_force():
    lens = [1, 15, 16, 17, 100, 333]
    for window in (0, 1, 20, 64):
        case = make_case("m", 3, len(lens), 8, 2, 64, 16, lambda r: np.array(lens, np.int32),
                         window=window, poison=False)
        assert bench.decode_bytes(case) == _decode_bytes_brute(case), window


def test_prefill_flops_match_brute_force():
    specs = [(5, 5), (3, 40), (1, 7), (17, 17)]
    for window in (0, 1, 4, 10):
        case = make_prefill_case("m", 4, specs, 8, 2, 64, 16, window=window, poison=False)
        qsl = case.query_start_loc
        want = 0
        for s, (n, L) in enumerate(specs):
            for i in range(n):
                p = L - n + i
                keys = [u for u in range(p + 1) if window <= 0 or u > p - window]
                want += 4 * case.head_dim * case.num_q_heads * len(keys)
        assert bench.prefill_flops(case) == want, window
        # the per-sample count used by the CPU baseline agrees on the whole set
        sel = np.array([(t, h) for t in range(int(qsl[-1])) for h in range(case.num_q_heads)])
        assert bench.prefill_sample_flops(case, sel) == want


def test_bf16_peaks_measured_and_fallback(tmp_path, monkeypatch):
    """The prefill roofline's denominators: the measured burst and sustained cuBLAS
    rates when the file has them, the recipe's 1,590 / 1,400 TFLOP/s otherwise."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.bf16_peaks() == ((1590.0, "fallback"), (1400.0, "fallback"))
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"bf16_tflops": 1665.0}')
    assert bench.bf16_peaks() == ((1665.0, "measured"), (1400.0, "fallback"))
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        '{"bf16_tflops": 1665.0, "bf16_tflops_sustained": 1339.0}')
    assert bench.bf16_peaks() == ((1665.0, "measured"), (1339.0, "measured"))


def test_cow_bytes_count_the_named_rows():
    """The folded copies move the named rows of every kv head (read and written, K and
    V) plus one triple per sequence; the separate block copy moves whole blocks."""
    from workloads.gen import make_prefix_cow
    c = make_prefix_cow(groups=2, samples=8, max_suffix=20, num_kv_heads=4, head_dim=64)
    rows = 2 * 7 * 8  # 7 copies per group, 8 prompt rows each
    assert bench.cow_bytes(c) == 2 * 2 * rows * 4 * 64 * 2 + 12 * 16
    assert bench.copy_bytes(c) == 2 * 2 * 14 * 4 * 16 * 64 * 2 + 16 * 14
