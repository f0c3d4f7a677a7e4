"""Gradients of the packed (varlen) layer against the fp64 oracle.

Each sequence of a packing is a dense layer whose queries are the last T_s of
its S_s positions, so the oracle's dense gradient of every sequence, run on
its own slices, is the reference for the packed rows. Keys of a sequence with
no queries (T_s = 0) get zero gradients. The tolerances are those of the dense
gradient tests: relative L2 <= 1e-2 and max-abs <= 2e-2 of the largest
reference entry, per tensor.
"""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import varlen_inputs
from test_gpu_random_shapes import _varlen_cases

pytestmark = pytest.mark.gpu


def _reference(q, k, v, dout, cq, ck, scale, cap, W):
    dq = np.zeros(q.shape, np.float64)
    dk = np.zeros(k.shape, np.float64)
    dv = np.zeros(v.shape, np.float64)
    for s in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[s]), int(cq[s + 1]), int(ck[s]), int(ck[s + 1])
        if q1 == q0:
            continue
        a, b, c = oracle.attn_bwd(q[q0:q1][None], k[k0:k1][None], v[k0:k1][None],
                                  dout[q0:q1][None], q_offset=(k1 - k0) - (q1 - q0),
                                  query_scale=scale, softcap=cap, window=W)
        dq[q0:q1], dk[k0:k1], dv[k0:k1] = a[0], b[0], c[0]
    return dq, dk, dv


def _close(grads, ref, what):
    for name, a, r in zip(("dq", "dk", "dv"), grads, ref):
        a = a.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all(), (name, what)
        nr = np.linalg.norm(r)
        if nr == 0.0:
            assert np.abs(a).max() == 0.0, (name, what)
            continue
        rel = np.linalg.norm(a - r) / nr
        mx = np.abs(a - r).max() / np.abs(r).max()
        assert rel <= 1e-2 and mx <= 2e-2, (name, what, rel, mx)


def _run(pairs, H, Hkv, d, W, cap, seed, scale=None):
    scale = d ** -0.5 if scale is None else scale
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(0, 0, 0, H, Hkv, d, 1.0, seed, seq_lens=pairs)
    g = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, gd, cqd, ckd = q.cuda(), k.cuda(), v.cuda(), dout.cuda(), cq.cuda(), ck.cuda()
    out, lse = g2.prefill_varlen(qd, kd, vd, cqd, ckd, max(Ts), max(Ss), query_scale=scale,
                                 softcap=cap, window=W)
    nan = float("nan")
    dq = torch.full_like(qd, nan)          # every element must be written
    dk = torch.full_like(kd, nan)
    dv = torch.full_like(vd, nan)
    grads = g2.prefill_varlen_backward(qd, kd, vd, out, lse, gd, cqd, ckd, max(Ts), max(Ss),
                                       query_scale=scale, softcap=cap, window=W, dq=dq, dk=dk,
                                       dv=dv)
    torch.cuda.synchronize()
    ref = _reference(q, k, v, dout, cq.numpy(), ck.numpy(), scale, cap, W)
    return grads, ref


FIXED = [
    # ragged tails, an empty and a single-token sequence, a chunked tail T < S
    ([(200, 300), (0, 77), (1, 1), (64, 64), (129, 400)], 4, 2, 128, 0, 50.0),
    ([(200, 300), (0, 77), (1, 1), (64, 64), (129, 400)], 4, 2, 128, 100, 50.0),
    ([(333, 333), (17, 250), (128, 128)], 2, 1, 64, 0, 50.0),
    ([(333, 333), (17, 250), (128, 128)], 6, 3, 64, 65, 0.0),
    ([(700, 700)], 2, 1, 128, 257, 50.0),
    ([(200, 300), (0, 77), (1, 1), (64, 64), (129, 400)], 4, 2, 256, 100, 50.0),
    ([(333, 333), (17, 250), (33, 33)], 2, 1, 256, 0, 0.0),
]


@pytest.mark.parametrize("case", FIXED, ids=[str(i) for i in range(len(FIXED))])
def test_varlen_backward_fixed(case):
    pairs, H, Hkv, d, W, cap = case
    grads, ref = _run(pairs, H, Hkv, d, W, cap, seed=99)
    _close(grads, ref, case)


RANDOM = ([c for c in _varlen_cases(30, 31337) if c[3] in (64, 128)][:8] +
          [c for c in _varlen_cases(30, 2718) if c[3] == 256][:4])


@pytest.mark.parametrize("case", RANDOM, ids=[str(i) for i in range(len(RANDOM))])
def test_varlen_backward_random(case):
    pairs, H, Hkv, d, W, cap, seed = case
    grads, ref = _run(pairs, H, Hkv, d, W, cap, seed)
    _close(grads, ref, case)


@pytest.mark.parametrize("d", [128, 256])
def test_single_sequence_matches_dense_bitwise(d):
    """One packed sequence runs the same units in the same order as the dense
    call with B = 1 and q_offset = S - T, so the gradients agree bit for bit."""
    T, S, H, Hkv = 300, 520, 4, 2
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(0, 0, 0, H, Hkv, d, 1.0, 5, seq_lens=[(T, S)])
    g = torch.Generator().manual_seed(6)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16).cuda()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kw = dict(query_scale=d ** -0.5, softcap=50.0, window=200)
    out, lse = g2.prefill_varlen(qd, kd, vd, cq.cuda(), ck.cuda(), T, S, **kw)
    a = g2.prefill_varlen_backward(qd, kd, vd, out, lse, dout, cq.cuda(), ck.cuda(), T, S, **kw)
    b = g2.prefill_backward(qd[None], kd[None], vd[None], out[None], lse[None], dout[None],
                            q_offset=S - T, **kw)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y[0])


def test_zz_device_error_word_clear():
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
