"""The benchmark's algorithmic byte counts (bench.py), without a GPU: the
window split of a T-token stream, the bytes of one decode and of one append,
pinned to figures computed independently from the workload definitions."""

import bench
from oracle import quantize as qz
from quantized_decode_attention_head_b200 import workloads


def test_split_lengths_invariants():
    for S, R in [(4, 128), (4, 32), (0, 16), (2, 0)]:
        for T in range(0, 400):
            s, tq, r = bench.split_lengths(T, S, R)
            assert s + tq + r == T and s == min(T, S) and tq % 32 == 0
            if T >= S + R:
                assert R <= r < R + 32
            else:
                assert tq == 0


def test_long_context_decode_bytes():
    """131072 tokens, S = 4, R = 128: 4091 tiles of 2-bit K and V (3072-byte
    records) and a 160-token bf16 window per stream, 8 streams, 4 query
    heads per stream (bf16 q in, fp32 out): 101.22 MB per decode."""
    wl = workloads.CONFIGS["long_128k"]
    rec = [[qz.record_bytes(2, 2, 128)] * 8]
    assert rec[0][0] == 4 * 128 * 2 + 512 + 4 * 128 * 2 + 512
    expect = 8 * (4091 * 3072 + 160 * 128 * 2 * 2 + 4 * 128 * 2 + 4 * 128 * 4)
    assert bench.decode_bytes(wl, rec, 131072) == expect
    assert abs(expect / 1e6 - 101.22) < 0.01


def test_append_bytes_count_the_flush_once_per_tile():
    wl = workloads.CONFIGS["long_128k"]
    rec = [[3072] * 8]
    row = 2 * 128 * 2 * 2  # new K and V rows read, then written to the ring
    flush = 32 * 128 * 2 * 2 + 3072  # 32 bf16 K and V rows read, one record written
    T0 = 131072
    per_step = [bench.append_bytes(wl, rec, T) for T in range(T0, T0 + 64)]
    n_flush = sum(b != 8 * row for b in per_step)
    assert n_flush == 2 and all(b in (8 * row, 8 * (row + flush)) for b in per_step)
    # the flush happens on the append that brings the recent window to R + 32
    for T, b in zip(range(T0, T0 + 64), per_step):
        r_after = bench.split_lengths(T + 1, 4, 128)[2]
        assert (b != 8 * row) == (bench.split_lengths(T, 4, 128)[1] != bench.split_lengths(T + 1, 4, 128)[1])
        assert r_after >= 128
