"""The bench's work counts (host arithmetic, no GPU).

The reported metric divides useful work by time, so the counts themselves are
checked here: visible pairs against a brute-force count of the visibility rule
(j <= p, p - j < W when W > 0, j < S, p = i + q_offset), and the closed forms
of the workloads (the 2B/9B layers at T = S = 8192 and the chunked-prefill
tail of the 9B packed workload).
"""
import numpy as np
import pytest

import bench


def _brute_pairs(T, S, qo, W):
    n = 0
    for i in range(T):
        p = i + qo
        for j in range(S):
            if j <= p and (W == 0 or p - j < W):
                n += 1
    return n


@pytest.mark.parametrize("seed", range(40))
def test_visible_pairs_brute_force(seed):
    rng = np.random.default_rng(seed)
    S = int(rng.integers(1, 90))
    T = int(rng.integers(1, S + 1))
    qo = int(rng.integers(0, S - T + 1))
    W = 0 if rng.random() < 0.3 else int(rng.integers(1, S + 5))
    assert bench.visible_pairs(T, S, qo, W) == _brute_pairs(T, S, qo, W)


def test_layer_closed_forms():
    # global: 8192 * 8193 / 2; local: a 4096-key ramp, then 4096 keys per row
    assert bench.visible_pairs(8192, 8192, 0, 0) == 33_558_528
    assert bench.visible_pairs(8192, 8192, 0, 4096) == 4096 * 4097 // 2 + 4096 * 4096
    assert bench.visible_pairs(8192, 8192, 0, 4096) == 25_167_872
    # 2B pair (B=1, H=8, d=256) and 9B pair (B=2, H=16, d=256), 4 d per visible triple
    assert round(bench.prefill_flops(1, 8192, 8192, 8, 256, 0, 4096) / 1e12, 4) == 0.2062
    assert round(bench.prefill_flops(1, 8192, 8192, 8, 256, 0, 0) / 1e12, 4) == 0.2749
    assert round(bench.prefill_flops(2, 8192, 8192, 16, 256, 0, 4096) / 1e12, 4) == 0.8247
    assert round(bench.prefill_flops(2, 8192, 8192, 16, 256, 0, 0) / 1e12, 4) == 1.0996


def test_chunked_tail_closed_form():
    # T = 1024 queries at the end of S = 8192 keys (q_offset 7168): every row sees
    # p + 1 keys globally (7169 .. 8192) and 4096 keys locally
    assert bench.visible_pairs(1024, 8192, 7168, 0) == sum(range(7169, 8193)) == 7_864_832
    assert bench.visible_pairs(1024, 8192, 7168, 4096) == 1024 * 4096 == 4_194_304
    # the varlen count is the per-sequence sum with q_offset = S - T
    Ts, Ss = [300, 1024], [300, 8192]
    expect = 4.0 * 256 * 16 * (bench.visible_pairs(300, 300, 0, 0) + 7_864_832)
    assert bench.varlen_flops(Ts, Ss, 16, 256, 0) == expect


def test_backward_and_decode_counts():
    f = bench.prefill_flops(1, 1000, 1500, 4, 128, 500, 300)
    assert bench.backward_flops(1, 1000, 1500, 4, 128, 500, 300) == 2.5 * f
    # decode reads min(L, W) rows of K and V per KV head (bf16): 8 KiB per row at Hkv=16, d=128
    lengths = [1000, 5000, 8192]
    assert bench.decode_kv_bytes(lengths, 16, 128, 4096) == (1000 + 4096 + 4096) * 16 * 128 * 4
    assert bench.decode_kv_bytes(lengths, 16, 128, 0) == sum(lengths) * 8192
