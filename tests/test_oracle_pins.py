"""Pins for the fp64 oracle, each independent of the oracle's own code.

The pages print no worked numeric example for the attention layer, so the
oracle is pinned by: brute force written a different way (dense matrices and
the triangular -inf masks of the "Gemma 2 Guide" PyTorch layer), closed forms
(zero keys give the mean of the visible values and lse = ln(count)), the
pages' own arithmetic (the 9B token-state count of the Guide's "Deep Dive"
item 2), invariants (|capped logit| <= 50, weights sum to 1), special cases
that reduce to a library routine (no cap = torch scaled_dot_product_attention
in fp64), window >= S = global, and GQA = MHA with repeated KV heads.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from global_soft_capped_b200.inputs import decode_inputs, prefill_inputs, varlen_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(t):
    return t.to(torch.float64).numpy()


def brute(q, k, v, q_offset, alpha, C, W):
    """Dense fp64 restatement: full (B,H,T,S) score matrix and the triangular
    -inf masks of the Guide's PyTorch layer ("End-to-End Implementation"):
    triu(-inf, diagonal=1) for the future, tril(-inf, diagonal=-W) for keys W
    or more places back. q_offset shifts the query rows (row i sits at q_offset+i)."""
    B, T, H, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    G = H // Hkv
    qd = torch.from_numpy(f64(q)).permute(0, 2, 1, 3) * alpha           # (B,H,T,d)
    kd = torch.from_numpy(f64(k)).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vd = torch.from_numpy(f64(v)).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    scores = qd @ kd.transpose(-1, -2)                                  # (B,H,T,S)
    if C > 0:
        scores = C * torch.tanh(scores / C)
    full = torch.full((q_offset + T, S), float("-inf"), dtype=torch.float64)
    mask = torch.triu(full, diagonal=1)
    if W > 0:
        mask = mask + torch.tril(full, diagonal=-W)
    scores = scores + mask[q_offset:q_offset + T]
    probs = torch.softmax(scores, dim=-1)
    out = (probs @ vd).permute(0, 2, 1, 3)
    lse = torch.logsumexp(scores, dim=-1)
    return out.numpy(), lse.numpy()


CASES = [
    # B, T, S, H, Hkv, d, q_offset, alpha, C, W, std
    (1, 16, 16, 4, 2, 8, 0, 0.35, 50.0, 4, 1.0),
    (2, 9, 23, 4, 2, 16, 14, 0.25, 50.0, 0, 1.0),
    (1, 13, 40, 2, 1, 8, 27, 1.0, 50.0, 7, 3.0),     # logits past the cap
    (1, 33, 33, 6, 3, 8, 0, 0.5, 5.0, 1, 1.0),       # window 1: only the diagonal
    (2, 5, 64, 8, 2, 4, 59, 0.7, 50.0, 63, 1.5),      # group of 4 heads
    (1, 24, 24, 2, 2, 8, 0, 0.3, 0.0, 9, 1.0),       # no cap
]


@pytest.mark.parametrize("case", CASES)
def test_oracle_matches_brute_force(case):
    B, T, S, H, Hkv, d, qo, a, C, W, std = case
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, std=std, seed=hash(case) % 1000)
    out, lse = oracle.attn(q, k, v, q_offset=qo, query_scale=a, softcap=C, window=W)
    bo, bl = brute(q, k, v, qo, a, C, W)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("W", [0, 1, 5, 16, 64])
@pytest.mark.parametrize("C", [50.0, 0.5, 0.0])
def test_zero_keys_closed_form(W, C):
    """K = 0 makes every logit 0 (capped or not): out_i is the plain mean of the
    visible values and lse_i = ln(count_i), count_i = min(p+1, W) (p+1 if global).
    A small cap (0.5) also pins the order cap-then-mask: capping a masked -inf
    first would give masked keys weight exp(-0.5) instead of 0."""
    B, T, S, H, Hkv, d, qo = 1, 20, 37, 4, 2, 8, 17
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, seed=7)
    k = torch.zeros_like(k)
    out, lse = oracle.attn(q, k, v, q_offset=qo, query_scale=0.9, softcap=C, window=W)
    vd = f64(v)
    for i in range(T):
        p = i + qo
        lo = max(0, p - W + 1) if W > 0 else 0
        count = p - lo + 1
        mean = vd[0, lo:p + 1].mean(axis=0)                            # (Hkv, d)
        for h in range(H):
            np.testing.assert_allclose(out[0, i, h], mean[h // 2], rtol=0, atol=1e-13)
            assert abs(lse[0, h, i] - math.log(count)) < 1e-13


def test_token_state_count_matches_guide_arithmetic():
    """The Guide's "Deep Dive" item 2: a 42-layer 9B at an 8,192 context holds
    21*8192 + 21*4096 = 258,048 token states (all-global: 344,064). The last
    query of an 8,192 sequence sees count = exp(lse) keys when K = 0: 8,192 on a
    global layer and 4,096 on a local layer with window 4,096."""
    g = json.load(open(os.path.join(GOLDEN, "kv_token_states_9b.json")))
    S = g["context"]
    lengths, cu, q, k, v = decode_inputs(1, S, S, 2, 1, 8, seed=3)
    k = torch.zeros_like(k)
    _, lse_g = oracle.decode(q, k, v, cu, window=0)
    _, lse_l = oracle.decode(q, k, v, cu, window=g["window"])
    n_global = round(math.exp(lse_g[0, 0]))
    n_local = round(math.exp(lse_l[0, 0]))
    assert (n_global, n_local) == (S, g["window"])
    assert g["local_layers"] * n_local + g["global_layers"] * n_global == \
        g["interleaved_token_states"]
    assert g["layers"] * n_global == g["all_global_token_states"]


def test_window_pattern_matches_guide_demo():
    """Visible keys of the Guide's demo local layer (seq_len 16, window 4),
    stored as text, recovered from the oracle's weights with K = 0 and one-hot
    values v_j = e_j (out_i is then the weight row of query i)."""
    lines = [ln.strip() for ln in open(os.path.join(GOLDEN, "window_mask_s16_w4.txt"))
             if ln.strip() and not ln.startswith("#")]
    expect = np.array([[c == "1" for c in ln] for ln in lines])
    S = 16
    q = torch.randn(1, S, 1, S).to(torch.bfloat16)
    k = torch.zeros(1, S, 1, S, dtype=torch.bfloat16)
    v = torch.eye(S, dtype=torch.bfloat16).reshape(1, S, 1, S)
    out, _ = oracle.attn(q, k, v, softcap=50.0, window=4)
    assert np.array_equal(out[0, :, 0, :] > 0, expect)


@pytest.mark.parametrize("alpha", [0.2, 3.0, 40.0])
def test_cap_bound_and_weights_sum_to_one(alpha):
    """|capped logit| <= 50 (the Guide, section 1: scores can never exceed +-50;
    the card: soft-cap to (-50, 50)); every weight row sums to 1; masked keys
    carry weight exactly 0."""
    B, T, S, H, Hkv, d, qo, W = 1, 12, 30, 4, 2, 32, 18, 10
    q, k, _ = prefill_inputs(B, T, S, H, Hkv, d, std=2.0, seed=11)
    big = 0
    for i in range(T):
        for h in range(H):
            s, w = oracle.row_detail(q, k, 0, i, h, q_offset=qo, query_scale=alpha,
                                     softcap=50.0, window=W)
            vis = np.isfinite(s)
            p = i + qo
            assert vis.sum() == min(p + 1, W)
            assert np.all(np.abs(s[vis]) <= 50.0)
            big += int(np.sum(np.abs(s[vis]) > 45.0))
            assert abs(w.sum() - 1.0) < 1e-12
            assert np.all(w[~vis] == 0.0)
    if alpha >= 40.0:
        assert big > 0  # the cap was really exercised


@pytest.mark.parametrize("W", [0, 6])
def test_no_cap_equals_torch_sdpa(W):
    """softcap = 0 (and a cap of 1e12) reduce to plain scaled masked softmax
    attention: torch's scaled_dot_product_attention in fp64 on the CPU, with a
    boolean mask and scale = query_scale; lse against torch.logsumexp."""
    B, T, S, H, Hkv, d, qo, a = 2, 11, 19, 4, 2, 16, 8, 0.3
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, seed=5)
    qd = torch.from_numpy(f64(q)).permute(0, 2, 1, 3)
    kd = torch.from_numpy(f64(k)).repeat_interleave(2, dim=2).permute(0, 2, 1, 3)
    vd = torch.from_numpy(f64(v)).repeat_interleave(2, dim=2).permute(0, 2, 1, 3)
    pos = torch.arange(T)[:, None] + qo
    j = torch.arange(S)[None, :]
    allowed = (j <= pos) & ((pos - j < W) if W > 0 else torch.ones_like(j, dtype=torch.bool))
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=allowed,
                                                           scale=a).permute(0, 2, 1, 3)
    scores = (qd @ kd.transpose(-1, -2)) * a
    ref_lse = torch.logsumexp(scores.masked_fill(~allowed, float("-inf")), dim=-1)
    for C in (0.0, 1e12):
        out, lse = oracle.attn(q, k, v, q_offset=qo, query_scale=a, softcap=C, window=W)
        np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-11)


def test_wide_window_is_global():
    """A window that reaches past every row's first key is the global layer, bit for bit."""
    B, T, S, H, Hkv, d, qo = 1, 10, 25, 4, 2, 8, 15
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, seed=9)
    g_out, g_lse = oracle.attn(q, k, v, q_offset=qo, window=0)
    for W in (qo + T, S, S + 7, 10 ** 6):
        o, l = oracle.attn(q, k, v, q_offset=qo, window=W)
        assert np.array_equal(o, g_out) and np.array_equal(l, g_lse)
    o, _ = oracle.attn(q, k, v, q_offset=qo, window=qo + T - 1)
    assert not np.array_equal(o, g_out)  # one key short of global on the last row


def test_gqa_equals_repeated_kv_heads():
    """Two query heads per KV head (the card: num_groups = 2; heads 2g and 2g+1
    share KV head g) equals multi-head attention with each KV head repeated."""
    B, T, S, H, Hkv, d = 2, 14, 14, 8, 4, 16
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, seed=13)
    o1, l1 = oracle.attn(q, k, v, query_scale=0.4, window=5)
    o2, l2 = oracle.attn(q, k.repeat_interleave(2, dim=2), v.repeat_interleave(2, dim=2),
                         query_scale=0.4, window=5)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # the pairing matters: swapping the KV heads changes the result
    o3, _ = oracle.attn(q, k.flip(2), v.flip(2), query_scale=0.4, window=5)
    assert not np.allclose(o1, o3)


def test_single_visible_key_and_window_one():
    """A row that sees one key copies that key's value exactly (weight 1)."""
    B, T, S, H, Hkv, d = 1, 12, 12, 4, 2, 8
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, std=2.0, seed=17)
    out, lse = oracle.attn(q, k, v, query_scale=2.0, window=1)
    vd = f64(v)
    for i in range(T):
        for h in range(H):
            assert np.array_equal(out[0, i, h], vd[0, i, h // 2])
            s, _ = oracle.row_detail(q, k, 0, i, h, query_scale=2.0, window=1)
            assert lse[0, h, i] == s[i]
    out0, _ = oracle.attn(q, k, v, query_scale=2.0, window=0)
    for h in range(H):
        assert np.array_equal(out0[0, 0, h], vd[0, 0, h // 2])


@pytest.mark.parametrize("C", [0.0, 5.0, 50.0])
def test_equal_logits_give_uniform_weights(C):
    """All keys equal => all logits of a row equal (capped or not) => the output
    is the mean of the visible values, whatever the cap."""
    B, T, S, H, Hkv, d, W = 1, 9, 9, 2, 1, 8, 4
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, seed=19)
    k = k[:, :1].expand(B, S, Hkv, d).contiguous()
    out, _ = oracle.attn(q, k, v, query_scale=3.0, softcap=C, window=W)
    vd = f64(v)
    for i in range(T):
        lo = max(0, i - W + 1)
        np.testing.assert_allclose(out[0, i, 0], vd[0, lo:i + 1, 0].mean(0), atol=1e-13, rtol=0)


def test_rows_and_decode_and_varlen_agree_with_dense():
    """attn_rows, decode (query at L-1) and varlen (q_offset = S_i - T_i) are the
    dense definition evaluated on the right rows."""
    B, T, S, H, Hkv, d = 2, 7, 19, 4, 2, 8
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, seed=23)
    out, lse = oracle.attn(q, k, v, q_offset=12, window=6)
    rows = [(1, 6, 3), (0, 0, 0), (1, 2, 1)]
    ro, rl = oracle.attn_rows(q, k, v, rows, q_offset=12, window=6)
    for n, (b, i, h) in enumerate(rows):
        assert np.array_equal(ro[n], out[b, i, h]) and rl[n] == lse[b, h, i]

    lengths, cu, qd, kc, vc = decode_inputs(3, 5, 30, H, Hkv, d, seed=29)
    do, dl = oracle.decode(qd, kc, vc, cu, query_scale=0.5, window=8)
    for s_, L in enumerate(lengths):
        k0 = int(cu[s_])
        o, l = oracle.attn(qd[s_][None, None], kc[k0:k0 + L][None], vc[k0:k0 + L][None],
                           q_offset=L - 1, query_scale=0.5, window=8)
        assert np.array_equal(do[s_], o[0, 0]) and np.array_equal(dl[s_], l[0, :, 0])
        # the decode query is the last row of a full prefill of the same cache
        qfull = torch.cat([torch.zeros(L - 1, H, d, dtype=torch.bfloat16), qd[s_][None]])
        of, lf = oracle.attn(qfull[None], kc[k0:k0 + L][None], vc[k0:k0 + L][None],
                             query_scale=0.5, window=8)
        assert np.array_equal(of[0, -1], do[s_]) and np.array_equal(lf[0, :, -1], dl[s_])

    Ts, Ss, cq, ck, qv, kv, vv = varlen_inputs(0, 0, 0, H, Hkv, d, seed=31,
                                               seq_lens=[(5, 5), (3, 11), (1, 1), (6, 6)])
    vo, vl = oracle.varlen(qv, kv, vv, cq, ck, window=4)
    for s_, (t, s) in enumerate(zip(Ts, Ss)):
        q0, k0 = int(cq[s_]), int(ck[s_])
        o, l = oracle.attn(qv[q0:q0 + t][None], kv[k0:k0 + s][None], vv[k0:k0 + s][None],
                           q_offset=s - t, window=4)
        assert np.array_equal(vo[q0:q0 + t], o[0]) and np.array_equal(vl[:, q0:q0 + t], l[0])


def test_rejects_bad_arguments():
    q, k, v = prefill_inputs(1, 4, 4, 3, 2, 8, seed=1)     # H not a multiple of Hkv
    with pytest.raises(ValueError):
        oracle.attn(q, k, v)
    q, k, v = prefill_inputs(1, 4, 4, 2, 1, 8, seed=1)
    with pytest.raises(ValueError):
        oracle.attn(q, k, v, window=-1)
