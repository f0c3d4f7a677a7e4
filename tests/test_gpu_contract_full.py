"""The contract workloads against the fp64 oracle over whole tensors, and the
gradients of the 8192-token layers against the oracle at sampled rows and keys.

Forward (Gemma 2 card, "Method", per-layer attention pseudo-code; cap formula
of the "Gemma 2 Guide", section 1): the 2B-shaped pair (B=1, T=S=8192, H=8,
Hkv=4, d=256), the 9B-shaped batched pair (B=2, T=S=8192, H=16, Hkv=8, d=256)
and the 9B-shaped ragged packed call (16 sequences plus the 1024-query tail at
q_offset 7168), local (window 4096) and global layers, in the launch
configuration the benchmark times. Every output row and every log-sum-exp is
compared: max-abs <= 2e-2 and relative L2 <= 5e-3 over the whole out tensor,
max |lse error| <= 1e-3. The GPU outputs are all computed first (module
fixture); the oracle then takes about a minute per 9B layer on 16 host cores.

Gradients (the Guide's derivative of the cap, "Deep Dive" item 1): the
benchmark's 27B-shaped (H=32, Hkv=16, d=128) and 2B-shaped (d=256) layers at
T = S = 8192, and the 27B-shaped packed batch of 8 sequences, against
oracle.attn_bwd_sampled at query rows and keys on both ends, on 64- and
128-row tile edges, around the window edge and at random, with the gradient
tolerance of tests/test_gpu_backward.py (relative L2 <= 1e-2 and
max |delta| <= 2e-2 * max |reference| per gradient over the sample).
"""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import (WORKLOADS, backward_inputs, prefill_inputs,
                                            varlen_backward_inputs, varlen_inputs)
from parity import RECORDS, check

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    g2.load_library()
    yield
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK


def _layers(w):
    return (("local", w.window_local), ("global", 0))


@pytest.fixture(scope="module")
def forward_outputs():
    """GPU outputs of every forward workload (CPU copies), computed before
    any oracle call so that the GPU work is not interleaved with it."""
    res = {}
    for name in ("2b", "9b"):
        w = WORKLOADS[name]
        q, k, v = prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        for layer, window in _layers(w):
            out, lse = g2.prefill(qd, kd, vd, query_scale=w.query_scale, softcap=w.softcap,
                                  window=window)
            torch.cuda.synchronize()
            res[name, layer] = (out.cpu(), lse.cpu())
    w = WORKLOADS["9b_varlen"]
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d,
                                            w.std, w.seed, tail_T=w.tail_T, tail_S=w.tail_S)
    for layer, window in _layers(w):
        out, lse = g2.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(),
                                     max(Ts), max(Ss), query_scale=w.query_scale,
                                     softcap=w.softcap, window=window)
        torch.cuda.synchronize()
        res["9b_varlen", layer] = (out.cpu(), lse.cpu())
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
    return res


@pytest.mark.parametrize("name", ["2b", "9b"])
@pytest.mark.parametrize("layer", ["local", "global"])
def test_prefill_whole_tensor(forward_outputs, name, layer):
    w = WORKLOADS[name]
    window = w.window_local if layer == "local" else 0
    q, k, v = prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    ro, rl = oracle.attn(q, k, v, query_scale=w.query_scale, softcap=w.softcap, window=window)
    out, lse = forward_outputs[name, layer]
    check(out, ro, lse, rl, f"{name} {layer} whole tensor", record=True)


@pytest.mark.parametrize("layer", ["local", "global"])
def test_varlen_whole_tensor(forward_outputs, layer):
    w = WORKLOADS["9b_varlen"]
    window = w.window_local if layer == "local" else 0
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d,
                                            w.std, w.seed, tail_T=w.tail_T, tail_S=w.tail_S)
    assert (Ts[-1], Ss[-1]) == (1024, 8192)  # the chunked-prefill tail, q_offset 7168
    ro, rl = oracle.varlen(q, k, v, cq, ck, query_scale=w.query_scale, softcap=w.softcap,
                           window=window)
    assert np.isfinite(ro).all() and np.isfinite(rl).all()  # every sequence computed
    out, lse = forward_outputs["9b_varlen", layer]
    check(out, ro, lse, rl, f"9b_varlen {layer} whole tensor", record=True)
    # the tail alone, so that its rows are not averaged away by the rest
    t0 = int(cq[-2])
    check(out[t0:], ro[t0:], lse[:, t0:], rl[:, t0:], f"9b_varlen {layer} tail (q_offset 7168)",
          record=True)


# ---------------------------------------------------------------------------
# gradients at full size, sampled
# ---------------------------------------------------------------------------
def _grad_check(got, ref, what):
    msgs = []
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        a = np.asarray(a, dtype=np.float64)
        assert np.isfinite(a).all(), (what, name)
        rel = np.linalg.norm(a - r) / max(np.linalg.norm(r), 1e-30)
        mx = np.abs(a - r).max() / max(np.abs(r).max(), 1e-30)
        assert rel <= GRAD_REL_L2 and mx <= GRAD_MAX_REL, (what, name, rel, mx)
        msgs.append(f"{name} rel_l2 {rel:.2e} max/max|ref| {mx:.2e}")
    RECORDS.append(f"{what}: " + ", ".join(msgs))


def _query_positions(T, q_offset, window, rng, n_random=6):
    pos = {0, 1, 63, 64, 65, 127, 128, 129, T // 2, T - 2, T - 1}
    if window:
        # rows whose absolute position is just below, at and past the window edge
        pos |= {window - 2 - q_offset, window - 1 - q_offset, window - q_offset,
                window + 1 - q_offset}
    pos |= set(int(x) for x in rng.integers(0, T, n_random))
    return sorted(p for p in pos if 0 <= p < T)


def _key_positions(S, T, q_offset, window, rng, n_random=6):
    pos = {0, 1, 31, 32, 33, 63, 64, 127, 128, 129, S // 2, S - 2, S - 1, q_offset}
    if window:
        # keys the last query rows just keep or just lose from their window
        last = q_offset + T - 1
        pos |= {last - window, last - window + 1, last - window + 2, window - 1, window}
    pos |= set(int(x) for x in rng.integers(0, S, n_random))
    return sorted(p for p in pos if 0 <= p < S)


@pytest.mark.parametrize("name", ["27b_backward", "2b_backward"])
@pytest.mark.parametrize("layer", ["local", "global"])
def test_backward_full_size_sampled(name, layer):
    """The benchmark's gradient call (forward, then g2attn_prefill_backward) at
    T = S = 8192 against the oracle at edge and random rows and keys. Keys
    are taken from two KV heads (the oracle needs the softmax statistics of
    every row of the heads it samples keys from)."""
    w = WORKLOADS[name]
    window = w.window_local if layer == "local" else 0
    q, k, v, dout = backward_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = g2.prefill(qd, kd, vd, query_scale=w.query_scale, softcap=w.softcap,
                          window=window)
    dq, dk, dv = g2.prefill_backward(qd, kd, vd, out, lse, gd, query_scale=w.query_scale,
                                     softcap=w.softcap, window=window)
    torch.cuda.synchronize()
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    rng = np.random.default_rng(w.seed + (0 if window else 1))
    groups = sorted(set(int(x) for x in rng.choice(w.Hkv, 2, replace=False)))
    rows = [(0, i, int(h)) for i in _query_positions(w.T, 0, window, rng)
            for h in rng.choice(w.H, 4, replace=False)]
    keys = [(0, j, g) for j in _key_positions(w.S, w.T, 0, window, rng) for g in groups]
    ref = oracle.attn_bwd_sampled(q, k, v, dout, rows, keys, query_scale=w.query_scale,
                                  softcap=w.softcap, window=window)
    got = (torch.stack([dq[b, i, h] for b, i, h in rows]).double().numpy(),
           torch.stack([dk[b, j, g] for b, j, g in keys]).double().numpy(),
           torch.stack([dv[b, j, g] for b, j, g in keys]).double().numpy())
    _grad_check(got, ref, f"{name} {layer} ({len(rows)} dq rows, {len(keys)} keys)")


@pytest.mark.parametrize("layer", ["local", "global"])
def test_varlen_backward_full_size_sampled(layer):
    """The benchmark's packed gradient call (8 sequences of 512-8192 tokens,
    27B-shaped) against the oracle at sampled rows and keys of every sequence."""
    w = WORKLOADS["27b_varlen_backward"]
    window = w.window_local if layer == "local" else 0
    Ts, Ss, cq, ck, q, k, v, dout = varlen_backward_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H,
                                                           w.Hkv, w.d, w.std, w.seed)
    qd, kd, vd, gd, cqd, ckd = q.cuda(), k.cuda(), v.cuda(), dout.cuda(), cq.cuda(), ck.cuda()
    out, lse = g2.prefill_varlen(qd, kd, vd, cqd, ckd, max(Ts), max(Ss),
                                 query_scale=w.query_scale, softcap=w.softcap, window=window)
    dq, dk, dv = g2.prefill_varlen_backward(qd, kd, vd, out, lse, gd, cqd, ckd, max(Ts), max(Ss),
                                            query_scale=w.query_scale, softcap=w.softcap,
                                            window=window)
    torch.cuda.synchronize()
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    rng = np.random.default_rng(70 + (0 if window else 1))
    got, ref = ([], [], []), ([], [], [])
    for s, (t, sl) in enumerate(zip(Ts, Ss)):
        q0, k0, qo = int(cq[s]), int(ck[s]), sl - t
        g = int(rng.integers(0, w.Hkv))
        rows = [(0, i, int(rng.integers(0, w.H))) for i in _query_positions(t, qo, window, rng, 2)]
        keys = [(0, j, g) for j in _key_positions(sl, t, qo, window, rng, 2)]
        r = oracle.attn_bwd_sampled(q[q0:q0 + t][None], k[k0:k0 + sl][None], v[k0:k0 + sl][None],
                                    dout[q0:q0 + t][None], rows, keys, q_offset=qo,
                                    query_scale=w.query_scale, softcap=w.softcap, window=window)
        got[0].append(torch.stack([dq[q0 + i, h] for _, i, h in rows]).double().numpy())
        got[1].append(torch.stack([dk[k0 + j, g_] for _, j, g_ in keys]).double().numpy())
        got[2].append(torch.stack([dv[k0 + j, g_] for _, j, g_ in keys]).double().numpy())
        for lst, x in zip(ref, r):
            lst.append(x)
    _grad_check([np.concatenate(x) for x in got], [np.concatenate(x) for x in ref],
                f"27b_varlen_backward {layer} ({len(Ts)} sequences)")
