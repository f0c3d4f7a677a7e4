"""Pins of the oracle's gradients (oracle.attn_bwd) to something other than itself.

The pages print the forward (Gemma 2 card, "Method", per-layer attention
pseudo-code) and the derivative of the soft-cap ("Gemma 2 Guide", Deep Dive
item 1: d/dx C tanh(x/C) = 1 - tanh^2(x/C)); the gradients follow from them by
the chain rule. Each pin below checks the oracle's analytic gradients against
an independent route:

* central finite differences of a plain NumPy fp64 forward written here;
* torch fp64 autograd of a separate plain PyTorch forward (GQA, window,
  q_offset, cap);
* with the cap off: autograd through torch's scaled_dot_product_attention
  (a library routine) with a boolean mask and repeated KV heads;
* invariants of the softmax: sum_j dv_j = sum of dout over the group's rows
  (weights sum to 1), sum_j dk_j = 0 without the cap (softmax gradients sum to
  0 over a row), zero upstream gradient gives zero gradients, and a cap far
  above every logit matches the cap switched off.
"""
import numpy as np
import pytest
import torch

import oracle
from global_soft_capped_b200.inputs import prefill_inputs


def _f64(t):
    return t.to(torch.float64).numpy()


def _np_forward(q, k, v, q_offset, scale, cap, window):
    """Plain fp64 forward: out (B,T,H,d) from float64 arrays."""
    B, T, H, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    kk = np.repeat(k, H // Hkv, axis=2)
    vv = np.repeat(v, H // Hkv, axis=2)
    x = np.einsum("bihc,bjhc->bhij", q * scale, kk)
    s = cap * np.tanh(x / cap) if cap > 0 else x
    p = np.arange(T)[:, None] + q_offset
    j = np.arange(S)[None, :]
    vis = (j <= p) & ((window == 0) | (p - j < window))
    s = np.where(vis[None, None], s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    w = np.exp(s)
    w /= w.sum(axis=-1, keepdims=True)
    return np.einsum("bhij,bjhc->bihc", w, vv)


def _torch_forward(q, k, v, q_offset, scale, cap, window):
    B, T, H, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    kk = k.repeat_interleave(H // Hkv, dim=2)
    vv = v.repeat_interleave(H // Hkv, dim=2)
    x = torch.einsum("bihc,bjhc->bhij", q * scale, kk)
    s = cap * torch.tanh(x / cap) if cap > 0 else x
    p = torch.arange(T)[:, None] + q_offset
    j = torch.arange(S)[None, :]
    vis = (j <= p) & ((p - j < window) if window > 0 else torch.ones_like(j, dtype=torch.bool))
    s = s.masked_fill(~vis[None, None], float("-inf"))
    w = torch.softmax(s, dim=-1)
    return torch.einsum("bhij,bjhc->bihc", w, vv)


def _inputs(B, T, S, H, Hkv, d, std, seed):
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, std=std, seed=seed)
    g = torch.Generator().manual_seed(seed + 1000)
    dout = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16)
    return q, k, v, dout


@pytest.mark.parametrize("cap,window,q_offset", [(50.0, 0, 0), (2.0, 3, 2), (0.0, 4, 1)])
def test_finite_differences(cap, window, q_offset):
    """Analytic gradients equal central differences of a NumPy forward."""
    B, T, S, H, Hkv, d = 1, 5, 7, 2, 1, 4
    q, k, v, dout = _inputs(B, T, S, H, Hkv, d, std=1.5, seed=21)
    scale = 0.7
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, q_offset=q_offset, query_scale=scale,
                                 softcap=cap, window=window)
    Q, K, V, G = _f64(q), _f64(k), _f64(v), _f64(dout)

    def loss(Q_, K_, V_):
        return float((_np_forward(Q_, K_, V_, q_offset, scale, cap, window) * G).sum())

    eps = 1e-6
    for name, X, grad in (("q", Q, dq), ("k", K, dk), ("v", V, dv)):
        fd = np.zeros_like(X)
        it = np.nditer(X, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args_p = {"q": (Xp, K, V), "k": (Q, Xp, V), "v": (Q, K, Xp)}[name]
            args_m = {"q": (Xm, K, V), "k": (Q, Xm, V), "v": (Q, K, Xm)}[name]
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-7, err_msg=name)


@pytest.mark.parametrize("cap,window,q_offset,H,Hkv", [
    (50.0, 0, 0, 4, 2), (50.0, 7, 3, 4, 2), (5.0, 5, 0, 8, 4), (3.0, 1, 4, 2, 1)])
def test_torch_autograd(cap, window, q_offset, H, Hkv):
    """Analytic gradients equal fp64 autograd of a plain PyTorch forward."""
    B, T, S, d = 2, 23, 27, 16
    q, k, v, dout = _inputs(B, T, S, H, Hkv, d, std=2.0, seed=5)
    scale = 0.5
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, q_offset=q_offset, query_scale=scale,
                                 softcap=cap, window=window)
    Q = q.to(torch.float64).requires_grad_()
    K = k.to(torch.float64).requires_grad_()
    V = v.to(torch.float64).requires_grad_()
    out = _torch_forward(Q, K, V, q_offset, scale, cap, window)
    (out * dout.to(torch.float64)).sum().backward()
    for name, mine, ref in (("q", dq, Q.grad), ("k", dk, K.grad), ("v", dv, V.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12, err_msg=name)


def test_no_cap_matches_sdpa_autograd():
    """Cap off: gradients of torch's scaled_dot_product_attention (fp64)."""
    B, T, S, H, Hkv, d = 1, 19, 30, 4, 2, 8
    q_offset, window, scale = S - T, 6, 0.3
    q, k, v, dout = _inputs(B, T, S, H, Hkv, d, std=1.0, seed=8)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, q_offset=q_offset, query_scale=scale,
                                 softcap=0.0, window=window)
    Q = q.to(torch.float64).requires_grad_()
    K = k.to(torch.float64).requires_grad_()
    V = v.to(torch.float64).requires_grad_()
    p = torch.arange(T)[:, None] + q_offset
    j = torch.arange(S)[None, :]
    mask = (j <= p) & (p - j < window)
    out = torch.nn.functional.scaled_dot_product_attention(
        Q.transpose(1, 2), K.repeat_interleave(H // Hkv, dim=2).transpose(1, 2),
        V.repeat_interleave(H // Hkv, dim=2).transpose(1, 2), attn_mask=mask, scale=scale)
    (out.transpose(1, 2) * dout.to(torch.float64)).sum().backward()
    np.testing.assert_allclose(dq, Q.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, K.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, V.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_invariants():
    B, T, S, H, Hkv, d = 2, 31, 31, 4, 2, 8
    q, k, v, dout = _inputs(B, T, S, H, Hkv, d, std=1.0, seed=3)
    G = _f64(dout)
    for cap in (50.0, 0.0):
        dq, dk, dv = oracle.attn_bwd(q, k, v, dout, query_scale=0.4, softcap=cap, window=9)
        # weights of each row sum to 1: the value gradients of a KV head add
        # up to the upstream gradients of all rows of its query heads
        for g in range(Hkv):
            lhs = dv[:, :, g, :].sum(axis=1)
            rhs = G[:, :, 2 * g:2 * g + 2, :].sum(axis=(1, 2))
            np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-11)
        if cap == 0.0:
            # softmax gradients sum to zero over a row: so do the key gradients
            np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-11)
    zero = torch.zeros_like(dout)
    for t in oracle.attn_bwd(q, k, v, zero, query_scale=0.4, softcap=50.0, window=9):
        assert np.all(t == 0.0)


def test_cap_far_above_logits_equals_cap_off():
    B, T, S, H, Hkv, d = 1, 17, 17, 2, 1, 16
    q, k, v, dout = _inputs(B, T, S, H, Hkv, d, std=1.0, seed=4)
    a = oracle.attn_bwd(q, k, v, dout, query_scale=0.25, softcap=1e9, window=5)
    b = oracle.attn_bwd(q, k, v, dout, query_scale=0.25, softcap=0.0, window=5)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-9, atol=1e-12)


def test_saturated_cap_stops_query_and_key_gradients():
    """Logits far past the cap (|x| / C in the hundreds): 1 - tanh^2 is ~0 for
    every pair, so dq and dk vanish, while dv (which does not pass through the
    cap) is O(1): with C = 1 the capped logits stay in (-1, 1) and the weights
    stay spread. Without the cap factor dq would be ~query_scale * |ds| * |k|."""
    B, T, S, H, Hkv, d = 1, 9, 9, 2, 1, 8
    q, k, v, dout = _inputs(B, T, S, H, Hkv, d, std=1.0, seed=6)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, query_scale=400.0, softcap=1.0, window=0)
    assert np.abs(dv).max() > 1.0
    assert np.abs(dq).max() < 1e-5 and np.abs(dk).max() < 1e-5


def _edge_places(B, T, S, H, Hkv, q_offset, window, rng, n_random=6):
    """Query rows and keys at both ends, around the diagonal and the window
    edge, plus random ones."""
    rows = set()
    for i in {0, 1, T // 2, T - 2, T - 1} | set(int(x) for x in rng.integers(0, T, n_random)):
        if 0 <= i < T:
            rows.add((int(rng.integers(0, B)), i, int(rng.integers(0, H))))
    keys = set()
    js = {0, 1, q_offset, q_offset + 1, S - 2, S - 1} | set(int(x) for x in rng.integers(0, S, n_random))
    if window:
        js |= {q_offset + window - 1 - T // 2, S - window, S - window + 1}
    for j in js:
        if 0 <= j < S:
            keys.add((int(rng.integers(0, B)), j, int(rng.integers(0, Hkv))))
    return sorted(rows), sorted(keys)


@pytest.mark.parametrize("cap,window,q_offset,H,Hkv", [
    (50.0, 0, 0, 4, 2), (2.0, 6, 3, 4, 2), (0.0, 5, 9, 2, 1), (4.0, 1, 2, 8, 4)])
def test_sampled_gradients_match_autograd(cap, window, q_offset, H, Hkv):
    """attn_bwd_sampled at chosen rows and keys equals fp64 autograd of the
    plain PyTorch forward above, entry by entry."""
    B, T, S, d = 2, 21, 30, 16
    q, k, v, dout = _inputs(B, T, S, H, Hkv, d, std=2.0, seed=11)
    scale = 0.45
    rows, keys = _edge_places(B, T, S, H, Hkv, q_offset, window, np.random.default_rng(1))
    dq, dk, dv = oracle.attn_bwd_sampled(q, k, v, dout, rows, keys, q_offset=q_offset,
                                         query_scale=scale, softcap=cap, window=window)
    Q = q.to(torch.float64).requires_grad_()
    K = k.to(torch.float64).requires_grad_()
    V = v.to(torch.float64).requires_grad_()
    out = _torch_forward(Q, K, V, q_offset, scale, cap, window)
    (out * dout.to(torch.float64)).sum().backward()
    ref_q = np.stack([Q.grad[b, i, h].numpy() for b, i, h in rows])
    ref_k = np.stack([K.grad[b, j, g].numpy() for b, j, g in keys])
    ref_v = np.stack([V.grad[b, j, g].numpy() for b, j, g in keys])
    np.testing.assert_allclose(dq, ref_q, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, ref_k, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, ref_v, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("cap,window,q_offset", [(50.0, 0, 0), (50.0, 9, 12), (0.0, 4, 3)])
def test_sampled_gradients_equal_full_gradients(cap, window, q_offset):
    """Every row and every key through attn_bwd_sampled equals attn_bwd (the
    finite-difference and autograd pinned routine) to rounding."""
    B, T, S, H, Hkv, d = 2, 33, 45, 4, 2, 8
    q, k, v, dout = _inputs(B, T, S, H, Hkv, d, std=1.5, seed=12)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, q_offset=q_offset, query_scale=0.6,
                                 softcap=cap, window=window)
    rows = [(b, i, h) for b in range(B) for i in range(T) for h in range(H)]
    keys = [(b, j, g) for b in range(B) for j in range(S) for g in range(Hkv)]
    sq, sk, sv = oracle.attn_bwd_sampled(q, k, v, dout, rows, keys, q_offset=q_offset,
                                         query_scale=0.6, softcap=cap, window=window)
    np.testing.assert_allclose(sq, dq.reshape(-1, d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(sk, dk.reshape(-1, d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(sv, dv.reshape(-1, d), rtol=0, atol=1e-12)


def test_sampled_gradients_reject_out_of_range_places():
    q, k, v, dout = _inputs(1, 4, 6, 2, 1, 8, std=1.0, seed=2)
    with pytest.raises(ValueError):
        oracle.attn_bwd_sampled(q, k, v, dout, [(0, 4, 0)], [(0, 0, 0)])
    with pytest.raises(ValueError):
        oracle.attn_bwd_sampled(q, k, v, dout, [(0, 0, 0)], [(0, 0, 1)])
