"""Seeded random shapes against the fp64 oracle (full tensors).

A fixed generator draws dense, varlen, gradient and decode cases. The ranges are:
* head sizes 64 / 128 / 256, with d = 256 running on CTA pairs;
* 1–3 KV heads with two query heads each, batch 1–3;
* S up to 700, 1 <= T <= S, any valid q_offset;
* no window, or any window size;
* cap 50, 5 or off, several query scales, and a few cases with the cap at 100 (above
  C log2(e) = 95 the forward keeps a running max with the cap on);
* varlen packings with empty and single-token sequences;
* decode from linear, ring (power-of-two slots >= window) and paged (16-256-row
  blocks) caches, with 1-12 sequences of up to 3000 tokens.

Each case is small enough for the oracle to finish in a second or two, and
together they hit ragged tails, windows that start or end inside a tile, and
pair units whose odd CTA has no valid rows. Tolerances are those of the fixed
parity check (`parity.py`) and of the gradient tests.
"""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import prefill_inputs, varlen_inputs
from parity import check

pytestmark = pytest.mark.gpu


def _dense_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        d = int(rng.choice([64, 128, 256]))
        Hkv = int(rng.integers(1, 4))
        B = int(rng.integers(1, 4))
        S = int(rng.integers(1, 701))
        T = int(rng.integers(1, S + 1))
        qo = int(rng.integers(0, S - T + 1))
        W = 0 if rng.random() < 0.35 else int(rng.integers(1, S + 40))
        cap = float(rng.choice([50.0, 50.0, 5.0, 0.0]))
        scale = float(rng.choice([d ** -0.5, 1.0 / 16, 0.3]))
        cases.append((B, T, S, 2 * Hkv, Hkv, d, qo, W, cap, scale, int(rng.integers(0, 1 << 30))))
    return cases


def _with_cap(cases, cap, i_cap):
    return [c[:i_cap] + (cap,) + c[i_cap + 1:] for c in cases]


DENSE = _dense_cases(24, 20261202) + _with_cap(_dense_cases(6, 31337), 100.0, 8)


@pytest.mark.parametrize("case", DENSE, ids=[str(i) for i in range(len(DENSE))])
def test_random_dense(case):
    B, T, S, H, Hkv, d, qo, W, cap, scale, seed = case
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, 1.0, seed)
    out, lse = g2.prefill(q.cuda(), k.cuda(), v.cuda(), q_offset=qo, query_scale=scale,
                          softcap=cap, window=W)
    torch.cuda.synchronize()
    ro, rl = oracle.attn(q, k, v, q_offset=qo, query_scale=scale, softcap=cap, window=W)
    check(out, ro, lse, rl, what=str(case))


def _varlen_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        d = int(rng.choice([64, 128, 256]))
        Hkv = int(rng.integers(1, 3))
        pairs = []
        for _ in range(int(rng.integers(1, 7))):
            Sk = int(rng.integers(1, 501))
            Tq = 0 if rng.random() < 0.15 else int(rng.integers(1, Sk + 1))
            pairs.append((Tq, Sk))
        if sum(t for t, _ in pairs) == 0:
            pairs[0] = (1, pairs[0][1])
        W = 0 if rng.random() < 0.4 else int(rng.integers(1, 520))
        cap = float(rng.choice([50.0, 0.0]))
        cases.append((pairs, 2 * Hkv, Hkv, d, W, cap, int(rng.integers(0, 1 << 30))))
    return cases


VARLEN = _varlen_cases(8, 777) + _with_cap(_varlen_cases(3, 4711), 100.0, 5)


@pytest.mark.parametrize("case", VARLEN, ids=[str(i) for i in range(len(VARLEN))])
def test_random_varlen(case):
    pairs, H, Hkv, d, W, cap, seed = case
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(0, 0, 0, H, Hkv, d, 1.0, seed, seq_lens=pairs)
    out, lse = g2.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), max(Ts),
                                 max(Ss), query_scale=d ** -0.5, softcap=cap, window=W)
    torch.cuda.synchronize()
    ro, rl = oracle.varlen(q, k, v, cq, ck, query_scale=d ** -0.5, softcap=cap, window=W)
    check(out, ro, lse, rl, what=str(case))


BACKWARD = ([c for c in _dense_cases(40, 4242) if c[5] in (64, 128)][:8] +
            [c for c in _dense_cases(40, 9898) if c[5] == 256][:6] +
            _with_cap(_dense_cases(2, 5353), 100.0, 8))


@pytest.mark.parametrize("case", BACKWARD, ids=[str(i) for i in range(len(BACKWARD))])
def test_random_backward(case):
    B, T, S, H, Hkv, d, qo, W, cap, scale, seed = case
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, 1.0, seed)
    g = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = g2.prefill(qd, kd, vd, q_offset=qo, query_scale=scale, softcap=cap, window=W)
    grads = g2.prefill_backward(qd, kd, vd, out, lse, gd, q_offset=qo, query_scale=scale,
                                softcap=cap, window=W)
    torch.cuda.synchronize()
    ref = oracle.attn_bwd(q, k, v, dout, q_offset=qo, query_scale=scale, softcap=cap, window=W)
    for name, a, r in zip(("dq", "dk", "dv"), grads, ref):
        a = a.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all(), name
        nr = np.linalg.norm(r)
        if nr == 0.0:  # no visible pair reaches these gradients
            assert np.abs(a).max() == 0.0, name
            continue
        rel = np.linalg.norm(a - r) / nr
        mx = np.abs(a - r).max() / np.abs(r).max()
        assert rel <= 1e-2 and mx <= 2e-2, (name, case, rel, mx)


def _decode_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        layout = ("linear", "ring", "paged")[i % 3]
        d = int(rng.choice([64, 128, 256]))
        Hkv = int(rng.integers(1, 4))
        lengths = [int(x) for x in rng.integers(1, 3001, size=int(rng.integers(1, 13)))]
        if layout == "ring":
            W = int(rng.integers(1, 2049))
            R = 1 << int(np.ceil(np.log2(W)))  # a power of two >= the window
        else:
            W = 0 if rng.random() < 0.4 else int(rng.integers(1, 3000))
            R = 0
        bs = int(rng.choice([16, 32, 64, 128, 256]))
        cap = float(rng.choice([50.0, 0.0]))
        cases.append((layout, lengths, 2 * Hkv, Hkv, d, W, R, bs, cap, int(rng.integers(0, 1 << 30))))
    return cases


DECODE = _decode_cases(12, 5150)


@pytest.mark.parametrize("case", DECODE, ids=[str(i) for i in range(len(DECODE))])
def test_random_decode(case):
    from test_gpu_decode_layouts import to_paged, to_ring
    from global_soft_capped_b200.inputs import decode_inputs
    layout, lengths, H, Hkv, d, W, R, bs, cap, seed = case
    lengths, cu, q, k, v = decode_inputs(0, 0, 0, H, Hkv, d, seed=seed, lengths=lengths)
    alpha = d ** -0.5
    sl = torch.tensor(lengths, dtype=torch.int32)
    if layout == "linear":
        out, lse = g2.decode(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths),
                             query_scale=alpha, softcap=cap, window=W)
    elif layout == "ring":
        kr, vr = to_ring(lengths, cu, k, R), to_ring(lengths, cu, v, R)
        out, lse = g2.decode_ring(q.cuda(), kr.cuda(), vr.cuda(), sl.cuda(), W,
                                  query_scale=alpha, softcap=cap)
    else:
        kb, vb, table = to_paged(lengths, cu, k, v, bs, seed=seed % 1000)
        out, lse = g2.decode_paged(q.cuda(), kb.cuda(), vb.cuda(), table.cuda(), sl.cuda(),
                                   max(lengths), query_scale=alpha, softcap=cap, window=W)
    torch.cuda.synchronize()
    ro, rl = oracle.decode(q, k, v, cu, query_scale=alpha, softcap=cap, window=W)
    check(out, ro, lse, rl, what=str(case))


def test_zz_device_error_word_clear():
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
