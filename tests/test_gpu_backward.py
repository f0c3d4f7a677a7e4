"""Gradients (g2attn_prefill_backward) against the fp64 oracle's attn_bwd.

Tolerance per gradient tensor: relative L2 error <= 1e-2 and
max |delta| <= 2e-2 * max |reference|. Derivation: the gradients are returned
in bf16 (half an ulp is 2^-9 = 1.95e-3 relative per element), and the
kernels round P and dS to bf16 before the accumulating UMMAs (2^-9 relative
each, fp32 accumulation). Those roundings alone give relative L2 errors of
about 2-3e-3, which is what the kernels show; the bar leaves a factor of ~4.

The forward's own outputs (out, lse) feed the backward, as in training; the
oracle recomputes everything from q, k, v and dout in fp64.
"""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import prefill_inputs

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_REL = 2e-2


def _dout(B, T, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, T, H, d, generator=g).to(torch.bfloat16)


def _run(B, T, S, H, Hkv, d, q_offset, window, cap, scale, seed=31):
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, 1.0, seed)
    dout = _dout(B, T, H, d, seed + 1)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = g2.prefill(qd, kd, vd, q_offset=q_offset, query_scale=scale, softcap=cap,
                          window=window)
    grads = g2.prefill_backward(qd, kd, vd, out, lse, gd, q_offset=q_offset, query_scale=scale,
                                softcap=cap, window=window)
    torch.cuda.synchronize()
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
    return (q, k, v, dout), grads


def _check(grads, ref):
    for name, a, r in zip(("dq", "dk", "dv"), grads, ref):
        a = a.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all(), name
        rel = np.linalg.norm(a - r) / max(np.linalg.norm(r), 1e-30)
        mx = np.abs(a - r).max() / max(np.abs(r).max(), 1e-30)
        assert rel <= REL_L2 and mx <= MAX_REL, (name, rel, mx)


CASES = [
    # B, T, S, H, Hkv, d, q_offset, window, cap, query_scale
    (1, 128, 128, 2, 1, 128, 0, 0, 50.0, 128 ** -0.5),
    (1, 200, 300, 4, 2, 128, 100, 70, 50.0, 144 ** -0.5),     # ragged, window, chunked
    (2, 130, 130, 4, 2, 64, 0, 0, 50.0, 0.125),               # batch, ragged tail
    (1, 77, 500, 2, 1, 128, 423, 0, 0.0, 128 ** -0.5),        # no cap
    (1, 256, 256, 4, 2, 64, 0, 64, 5.0, 1.0),                 # logits past the cap
    (1, 1, 129, 2, 1, 128, 128, 0, 50.0, 128 ** -0.5),        # a single query
    (1, 64, 1000, 2, 1, 64, 936, 32, 50.0, 0.125),            # keys no query sees: zero grads
    (1, 300, 300, 2, 1, 128, 0, 129, 50.0, 128 ** -0.5),      # window across a tile edge
    # d = 256: 32-row column tiles, the dk/dv kernel in two d-halves
    (1, 200, 300, 4, 2, 256, 100, 70, 50.0, 1 / 16),          # ragged, window, chunked
    (2, 130, 130, 2, 1, 256, 0, 0, 50.0, 1 / 16),             # batch, ragged tail
    (1, 77, 500, 2, 1, 256, 423, 0, 0.0, 1 / 16),             # no cap
    (1, 256, 256, 2, 1, 256, 0, 64, 5.0, 1.0),                # logits past the cap
    (1, 64, 1000, 2, 1, 256, 936, 32, 50.0, 1 / 16),          # keys no query sees: zero grads
    (1, 1, 33, 2, 1, 256, 32, 0, 50.0, 1 / 16),               # a single query
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_backward_matches_oracle(case):
    B, T, S, H, Hkv, d, qo, W, cap, scale = case
    (q, k, v, dout), grads = _run(B, T, S, H, Hkv, d, qo, W, cap, scale)
    ref = oracle.attn_bwd(q, k, v, dout, q_offset=qo, query_scale=scale, softcap=cap, window=W)
    _check(grads, ref)
    if qo > 0 and W > 0:
        # keys before the first query's window get exactly zero gradients
        first = max(0, qo - W + 1)
        assert torch.count_nonzero(grads[1][:, :first]).item() == 0
        assert torch.count_nonzero(grads[2][:, :first]).item() == 0


@pytest.mark.parametrize("layer", ["local", "global"])
def test_27b_shaped_backward(layer):
    """27B head layout (H=32, Hkv=16, d=128, query_scale 144^-1/2) at T = S = 1024."""
    W = 256 if layer == "local" else 0
    (q, k, v, dout), grads = _run(1, 1024, 1024, 32, 16, 128, 0, W, 50.0, 144 ** -0.5, seed=3)
    ref = oracle.attn_bwd(q, k, v, dout, query_scale=144 ** -0.5, softcap=50.0, window=W)
    _check(grads, ref)


@pytest.mark.parametrize("layer", ["local", "global"])
def test_2b_shaped_backward(layer):
    """2B head layout (H=8, Hkv=4, d=256, query_scale 1/16) at T = S = 1024."""
    W = 256 if layer == "local" else 0
    (q, k, v, dout), grads = _run(1, 1024, 1024, 8, 4, 256, 0, W, 50.0, 1 / 16, seed=5)
    ref = oracle.attn_bwd(q, k, v, dout, query_scale=1 / 16, softcap=50.0, window=W)
    _check(grads, ref)


@pytest.mark.parametrize("shape", ["27b", "2b"])
@pytest.mark.parametrize("layer", ["local", "global"])
def test_full_size_value_gradient_invariant(layer, shape):
    """At full size (T = S = 8192, 27B and 2B head layouts): the softmax weights of each
    row sum to one, so the value gradients of KV head g add up to the upstream
    gradients of all rows of its two query heads. Also: two runs agree bitwise
    (no atomics anywhere)."""
    W = 4096 if layer == "local" else 0
    if shape == "27b":
        B, T, S, H, Hkv, d, alpha = 1, 8192, 8192, 32, 16, 128, 144 ** -0.5
    else:
        B, T, S, H, Hkv, d, alpha = 1, 8192, 8192, 8, 4, 256, 1 / 16
    q, k, v = (t.cuda() for t in prefill_inputs(B, T, S, H, Hkv, d, 1.0, 3))
    dout = _dout(B, T, H, d, 4).cuda()
    out, lse = g2.prefill(q, k, v, query_scale=alpha, softcap=50.0, window=W)
    ws = g2.backward_workspace(B, T, H)
    dq, dk, dv = g2.prefill_backward(q, k, v, out, lse, dout, query_scale=alpha,
                                     softcap=50.0, window=W, workspace=ws)
    dq2, dk2, dv2 = g2.prefill_backward(q, k, v, out, lse, dout, query_scale=alpha,
                                        softcap=50.0, window=W, workspace=ws)
    torch.cuda.synchronize()
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
    lhs = dv.double().sum(dim=1)                               # (B, Hkv, d)
    rhs = dout.double().view(B, T, Hkv, 2, d).sum(dim=(1, 3))  # (B, Hkv, d)
    err = (lhs - rhs).abs().max().item() / rhs.abs().max().item()
    assert err < 1e-2, err
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
