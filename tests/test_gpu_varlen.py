"""CUDA packed variable-length prefill against the fp64 oracle, through the C ABI."""
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


def run(Ts, Ss, cq, ck, q, k, v, **kw):
    out, lse = g2.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), max(Ts),
                                 max(Ss), **kw)
    torch.cuda.synchronize()
    return out, lse


CASES = [
    # (T_i, S_i) list, H, Hkv, d, window, softcap, alpha
    ([(5, 5), (3, 11), (1, 1), (70, 70), (64, 200)], 4, 2, 64, 0, 50.0, 0.125),
    ([(130, 130), (1, 300), (65, 129), (200, 200)], 4, 2, 128, 63, 50.0, 0.09),
    ([(300, 300), (128, 1000), (7, 7)], 2, 1, 256, 129, 50.0, 0.0625),
    ([(100, 100), (50, 80)], 2, 1, 256, 0, 0.0, 0.0625),
    ([(1, 1)] * 40 + [(257, 257)], 2, 1, 64, 4, 50.0, 1.0),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_varlen_shapes_full(case):
    lens, H, Hkv, d, W, C, a = case
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(0, 0, 0, H, Hkv, d, seed=60 + CASES.index(case),
                                            seq_lens=lens)
    out, lse = run(Ts, Ss, cq, ck, q, k, v, query_scale=a, softcap=C, window=W)
    ro, rl = oracle.varlen(q, k, v, cq, ck, query_scale=a, softcap=C, window=W)
    check(out, ro, lse, rl, f"varlen {case[1:]}")


@pytest.mark.parametrize("layer", ["local", "global"])
def test_9b_varlen_sampled(layer):
    """The benchmark's packed workload (16 sequences plus a chunked-prefill
    tail): every row finite; sampled rows of every sequence (both ends, the
    middle, 64- and 128-row tile edges, the window edge, one random row)
    against the oracle. The whole tensors are compared in
    tests/test_gpu_contract_full.py."""
    w = WORKLOADS["9b_varlen"]
    window = w.window_local if layer == "local" else 0
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d,
                                            w.std, w.seed, tail_T=w.tail_T, tail_S=w.tail_S)
    out, lse = run(Ts, Ss, cq, ck, q, k, v, query_scale=w.query_scale, softcap=w.softcap,
                   window=window)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    oc, lc = out.cpu(), lse.cpu()
    rng = np.random.default_rng(5)
    go, gl, ro_all, rl_all = [], [], [], []
    for s, (t, sl) in enumerate(zip(Ts, Ss)):
        q0, k0 = int(cq[s]), int(ck[s])
        qo = sl - t
        pos = {0, t - 1, t // 2, int(rng.integers(0, t)), 63, 64, 65, 127, 128, 129}
        if window:  # rows whose absolute position sits around the window edge
            pos |= {window - 2 - qo, window - 1 - qo, window - qo, window + 1 - qo}
        pos = sorted(p for p in pos if 0 <= p < t)
        rows = [(0, i, h) for i in pos for h in range(w.H)]
        ro, rl = oracle.attn_rows(q[q0:q0 + t][None], k[k0:k0 + sl][None], v[k0:k0 + sl][None],
                                  rows, q_offset=sl - t, query_scale=w.query_scale,
                                  softcap=w.softcap, window=window)
        go += [oc[q0 + i, h] for _, i, h in rows]
        gl += [lc[h, q0 + i] for _, i, h in rows]
        ro_all.append(ro)
        rl_all.append(rl)
    check(torch.stack(go), np.concatenate(ro_all), torch.stack(gl), np.concatenate(rl_all),
          f"9b varlen {layer}")


def test_concurrent_launches_on_two_streams_are_independent():
    """Packed launches take their units from a per-launch counter slot chosen
    by the launch's grid id: launches running at the same time on two streams
    must not share units. Each stream's results equal those of the same call
    run alone (bitwise: the units compute the same sums whatever CTA runs
    them), over several rounds of overlapping launches."""
    lens_a = [(700, 700), (1200, 1200), (300, 300), (900, 900)]
    lens_b = [(1000, 1000), (64, 64), (1500, 1500)]
    H, Hkv, d, W = 4, 2, 256, 256
    dev = torch.device("cuda")
    a = varlen_inputs(0, 0, 0, H, Hkv, d, seed=71, seq_lens=lens_a)
    b = varlen_inputs(0, 0, 0, H, Hkv, d, seed=72, seq_lens=lens_b)
    ga = [t.to(dev) for t in a[2:]]
    gb = [t.to(dev) for t in b[2:]]
    kw = dict(query_scale=0.0625, softcap=50.0, window=W)

    def launch(g, Ts, Ss, stream=None):
        cq, ck, q, k, v = g
        return g2.prefill_varlen(q, k, v, cq, ck, max(Ts), max(Ss), stream=stream, **kw)

    ref_a = launch(ga, a[0], a[1])
    ref_b = launch(gb, b[0], b[1])
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(8):
        with torch.cuda.stream(s1):
            oa = launch(ga, a[0], a[1], stream=s1)
        with torch.cuda.stream(s2):
            ob = launch(gb, b[0], b[1], stream=s2)
        torch.cuda.synchronize()
        assert torch.equal(oa[0], ref_a[0]) and torch.equal(oa[1], ref_a[1])
        assert torch.equal(ob[0], ref_b[0]) and torch.equal(ob[1], ref_b[1])
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
