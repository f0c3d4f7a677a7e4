"""Chunked prefill over a paged KV cache (block table, blocks >= 128 rows),
through the C ABI, against the fp64 oracle's packed varlen layer on the same
keys and values. Blocks no table entry references hold NaN, so a stray read
shows up as a non-finite output."""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import WORKLOADS, varlen_inputs
from parity import check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    g2.load_library()
    yield
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK


def to_paged(Ss, ck, k, v, bs, seed):
    rng = np.random.default_rng(seed)
    nblk = [(S + bs - 1) // bs for S in Ss]
    total = sum(nblk) + 2
    perm = rng.permutation(total)
    Hkv, d = k.shape[1], k.shape[2]
    kb = torch.full((total, bs, Hkv, d), float("nan")).to(torch.bfloat16)
    vb = torch.full((total, bs, Hkv, d), float("nan")).to(torch.bfloat16)
    table = -np.ones((len(Ss), max(nblk) + 1), dtype=np.int32)
    nxt = 0
    for s, S in enumerate(Ss):
        for b in range(nblk[s]):
            blk = int(perm[nxt]); nxt += 1
            table[s, b] = blk
            p0, p1 = b * bs, min(S, (b + 1) * bs)
            # rows past the sequence end: finite filler (the contract)
            kb[blk] = torch.randn(bs, Hkv, d).to(torch.bfloat16)
            vb[blk] = torch.randn(bs, Hkv, d).to(torch.bfloat16)
            kb[blk, :p1 - p0] = k[int(ck[s]) + p0:int(ck[s]) + p1]
            vb[blk, :p1 - p0] = v[int(ck[s]) + p0:int(ck[s]) + p1]
    return kb, vb, torch.from_numpy(table)


CASES = [
    # (T_s, S_s) list, H, Hkv, d, block_size, window, softcap, alpha
    ([(100, 100), (64, 300), (1, 129), (250, 1000)], 4, 2, 64, 128, 0, 50.0, 0.125),
    ([(100, 100), (64, 300), (1, 129), (250, 1000)], 4, 2, 64, 128, 64, 50.0, 0.125),
    ([(300, 300), (128, 1000), (7, 700)], 2, 1, 256, 256, 0, 50.0, 0.0625),
    ([(300, 300), (128, 1000), (7, 700)], 2, 1, 256, 256, 300, 50.0, 0.0625),
    ([(513, 1500), (90, 90)], 4, 2, 128, 512, 0, 0.0, 0.09),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_paged_prefill(case):
    lens, H, Hkv, d, bs, W, C, a = case
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(0, 0, 0, H, Hkv, d, seed=100 + CASES.index(case),
                                            seq_lens=lens)
    kb, vb, table = to_paged(Ss, ck, k, v, bs, seed=CASES.index(case))
    sl = torch.tensor(Ss, dtype=torch.int32)
    out, lse = g2.prefill_paged(q.cuda(), kb.cuda(), vb.cuda(), cq.cuda(), table.cuda(),
                                sl.cuda(), max(Ts), max(Ss), query_scale=a, softcap=C, window=W)
    torch.cuda.synchronize()
    ro, rl = oracle.varlen(q, k, v, cq, ck, query_scale=a, softcap=C, window=W)
    check(out, ro, lse, rl, f"paged prefill {case}")


def test_paged_prefill_matches_packed_varlen():
    """The 9B ragged workload from 256-row blocks equals the packed varlen
    call bit for bit (same tiles, same arithmetic, only the addressing differs)."""
    w = WORKLOADS["9b_varlen"]
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d,
                                            w.std, w.seed, tail_T=w.tail_T, tail_S=w.tail_S)
    kb, vb, table = to_paged(Ss, ck, k, v, 256, seed=5)
    sl = torch.tensor(Ss, dtype=torch.int32)
    qd, cqd = q.cuda(), cq.cuda()
    o1, l1 = g2.prefill_paged(qd, kb.cuda(), vb.cuda(), cqd, table.cuda(), sl.cuda(), max(Ts),
                              max(Ss), query_scale=w.query_scale, softcap=w.softcap,
                              window=w.window_local)
    o2, l2 = g2.prefill_varlen(qd, k.cuda(), v.cuda(), cqd, ck.cuda(), max(Ts), max(Ss),
                               query_scale=w.query_scale, softcap=w.softcap,
                               window=w.window_local)
    torch.cuda.synchronize()
    assert torch.isfinite(o1.float()).all()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
