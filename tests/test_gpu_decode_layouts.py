"""Decode over a ring-buffer cache (local layers keep only their last R tokens)
and over a paged cache (blocks + block table), through the C ABI, against the
fp64 oracle run on the equivalent linear cache. Slots and blocks the queries
must not read hold NaN, so any stray read shows up as a non-finite output."""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import WORKLOADS, decode_inputs
from parity import check

pytestmark = pytest.mark.gpu
NAN_BF16 = torch.tensor(float("nan"), dtype=torch.bfloat16)


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    g2.load_library()
    yield
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK


def to_ring(lengths, cu, cache, R):
    """(sum L, Hkv, d) linear cache -> (n, R, Hkv, d) rings holding each
    sequence's last R positions at slot p mod R; other slots NaN."""
    n, Hkv, d = len(lengths), cache.shape[1], cache.shape[2]
    ring = NAN_BF16.expand(n, R, Hkv, d).clone()
    for s, L in enumerate(lengths):
        for p in range(max(0, L - R), L):
            ring[s, p % R] = cache[int(cu[s]) + p]
    return ring


def to_paged(lengths, cu, k, v, bs, seed):
    """Linear caches -> shuffled blocks of bs rows plus a block table; unused
    blocks NaN, unused table entries -1."""
    rng = np.random.default_rng(seed)
    nblk = [(L + bs - 1) // bs for L in lengths]
    total = sum(nblk) + 3
    perm = rng.permutation(total)
    Hkv, d = k.shape[1], k.shape[2]
    kb = NAN_BF16.expand(total, bs, Hkv, d).clone()
    vb = NAN_BF16.expand(total, bs, Hkv, d).clone()
    table = -np.ones((len(lengths), max(nblk) + 1), dtype=np.int32)
    nxt = 0
    for s, L in enumerate(lengths):
        for b in range(nblk[s]):
            blk = int(perm[nxt]); nxt += 1
            table[s, b] = blk
            p0, p1 = b * bs, min(L, (b + 1) * bs)
            kb[blk, :p1 - p0] = k[int(cu[s]) + p0:int(cu[s]) + p1]
            vb[blk, :p1 - p0] = v[int(cu[s]) + p0:int(cu[s]) + p1]
    return kb, vb, torch.from_numpy(table)


RING_CASES = [
    # lengths, H, Hkv, d, R, window, alpha
    ([1, 5, 127, 128, 129, 300], 4, 2, 64, 128, 128, 0.125),
    ([1, 5, 127, 128, 129, 300], 4, 2, 64, 128, 100, 0.125),
    ([4095, 4096, 4097, 9000], 8, 4, 256, 4096, 4096, 0.0625),
    ([700, 3000], 4, 2, 128, 1024, 512, 0.09),
]


@pytest.mark.parametrize("case", RING_CASES, ids=[str(i) for i in range(len(RING_CASES))])
def test_ring_decode(case):
    lengths, H, Hkv, d, R, W, a = case
    lengths, cu, q, k, v = decode_inputs(0, 0, 0, H, Hkv, d, seed=80 + RING_CASES.index(case),
                                         lengths=lengths)
    kr, vr = to_ring(lengths, cu, k, R), to_ring(lengths, cu, v, R)
    sl = torch.tensor(lengths, dtype=torch.int32)
    out, lse = g2.decode_ring(q.cuda(), kr.cuda(), vr.cuda(), sl.cuda(), W, query_scale=a)
    torch.cuda.synchronize()
    ro, rl = oracle.decode(q, k, v, cu, query_scale=a, window=W)
    check(out, ro, lse, rl, f"ring {case}")


def test_ring_27b_local_layer():
    """The 27B decode workload's local layer served from 4,096-slot rings."""
    w = WORKLOADS["27b_decode"]
    lengths, cu, q, k, v = decode_inputs(16, w.len_lo, w.len_hi, w.H, w.Hkv, w.d, w.std, 91)
    R = w.window_local
    kr, vr = to_ring(lengths, cu, k, R), to_ring(lengths, cu, v, R)
    sl = torch.tensor(lengths, dtype=torch.int32)
    out, lse = g2.decode_ring(q.cuda(), kr.cuda(), vr.cuda(), sl.cuda(), w.window_local,
                              query_scale=w.query_scale, softcap=w.softcap)
    torch.cuda.synchronize()
    ro, rl = oracle.decode(q, k, v, cu, query_scale=w.query_scale, softcap=w.softcap,
                           window=w.window_local)
    check(out, ro, lse, rl, "27b ring local")


PAGED_CASES = [
    # lengths, H, Hkv, d, block_size, window, alpha
    ([1, 15, 16, 17, 200], 4, 2, 64, 16, 0, 0.125),
    ([1, 15, 16, 17, 200], 4, 2, 64, 16, 20, 0.125),
    ([1000, 2500, 4097], 8, 4, 256, 64, 0, 0.0625),
    ([1000, 2500, 4097], 8, 4, 256, 256, 1024, 0.0625),
    ([3333, 80], 4, 2, 128, 32, 0, 0.09),
]


@pytest.mark.parametrize("case", PAGED_CASES, ids=[str(i) for i in range(len(PAGED_CASES))])
def test_paged_decode(case):
    lengths, H, Hkv, d, bs, W, a = case
    lengths, cu, q, k, v = decode_inputs(0, 0, 0, H, Hkv, d, seed=90 + PAGED_CASES.index(case),
                                         lengths=lengths)
    kb, vb, table = to_paged(lengths, cu, k, v, bs, seed=PAGED_CASES.index(case))
    sl = torch.tensor(lengths, dtype=torch.int32)
    out, lse = g2.decode_paged(q.cuda(), kb.cuda(), vb.cuda(), table.cuda(), sl.cuda(),
                               max(lengths), query_scale=a, window=W)
    torch.cuda.synchronize()
    ro, rl = oracle.decode(q, k, v, cu, query_scale=a, window=W)
    check(out, ro, lse, rl, f"paged {case}")
