"""Packed calls at the kernels' sequence-table limit (1024 sequences).

The forward and gradient kernels rank and prefix-sum the sequences of a launch
in shared memory, up to 1024 of them. These cases fill the table: 1024 short
sequences (some empty, some single-token, chunked tails with T < S), so every
table entry, the scan across its 32 warp-sized blocks and the rank order are
exercised. Forward against the oracle's packed layer; gradients against its
per-sequence gradients (the tolerances of the other gradient tests).
"""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import varlen_inputs
from parity import check
from test_gpu_backward_varlen import _close, _reference

pytestmark = pytest.mark.gpu

NSEQ = 1024


def _pairs(seed):
    rng = np.random.default_rng(seed)
    pairs = []
    for _ in range(NSEQ):
        sk = int(rng.integers(1, 41))
        tq = 0 if rng.random() < 0.1 else int(rng.integers(1, sk + 1))
        pairs.append((tq, sk))
    return pairs


@pytest.mark.parametrize("d,W,cap", [(64, 16, 50.0), (128, 0, 0.0)])
def test_forward_full_sequence_table(d, W, cap):
    pairs = _pairs(11 + d)
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(0, 0, 0, 2, 1, d, 1.0, 21, seq_lens=pairs)
    out, lse = g2.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), max(Ts),
                                 max(Ss), query_scale=d ** -0.5, softcap=cap, window=W)
    torch.cuda.synchronize()
    ro, rl = oracle.varlen(q, k, v, cq, ck, query_scale=d ** -0.5, softcap=cap, window=W)
    check(out, ro, lse, rl, what=f"{NSEQ} sequences d={d}")


@pytest.mark.parametrize("d,W,cap", [(64, 16, 50.0), (128, 0, 0.0)])
def test_backward_full_sequence_table(d, W, cap):
    pairs = _pairs(31 + d)
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(0, 0, 0, 2, 1, d, 1.0, 41, seq_lens=pairs)
    g = torch.Generator().manual_seed(42)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, gd, cqd, ckd = q.cuda(), k.cuda(), v.cuda(), dout.cuda(), cq.cuda(), ck.cuda()
    out, lse = g2.prefill_varlen(qd, kd, vd, cqd, ckd, max(Ts), max(Ss), query_scale=d ** -0.5,
                                 softcap=cap, window=W)
    grads = g2.prefill_varlen_backward(qd, kd, vd, out, lse, gd, cqd, ckd, max(Ts), max(Ss),
                                       query_scale=d ** -0.5, softcap=cap, window=W)
    torch.cuda.synchronize()
    ref = _reference(q, k, v, dout, cq.numpy(), ck.numpy(), d ** -0.5, cap, W)
    _close(grads, ref, f"{NSEQ} sequences d={d}")


def test_zz_device_error_word_clear():
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
