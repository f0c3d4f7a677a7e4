"""Gemma 3-shaped parameter variant of the same kernels (window 1024, no
soft-cap; the research-hub page's Gemma 3 entry) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import WORKLOADS, decode_inputs, prefill_inputs
from parity import check, sample_positions

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    g2.load_library()
    yield
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK


@pytest.mark.parametrize("layer", ["local", "global"])
def test_gemma3_pair_sampled_rows(layer):
    w = WORKLOADS["gemma3_2b"]
    window = w.window_local if layer == "local" else 0
    q, k, v = prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    out, lse = g2.prefill(q.cuda(), k.cuda(), v.cuda(), query_scale=w.query_scale,
                          softcap=w.softcap, window=window)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    pos = sample_positions(w.T, window, 12, seed=w.seed)
    rows = [(0, i, h) for i in pos for h in range(w.H)]
    ro, rl = oracle.attn_rows(q, k, v, rows, query_scale=w.query_scale, softcap=w.softcap,
                              window=window)
    oc, lc = out.cpu(), lse.cpu()
    check(torch.stack([oc[b, i, h] for b, i, h in rows]), ro,
          torch.stack([lc[b, h, i] for b, i, h in rows]), rl, f"gemma3 {layer}")


@pytest.mark.parametrize("d,W", [(64, 1024), (128, 1024), (256, 100), (256, 0)])
def test_no_cap_shapes_full(d, W):
    q, k, v = prefill_inputs(1, 1500, 1500, 4, 2, d, seed=70 + d + W)
    a = d ** -0.5
    out, lse = g2.prefill(q.cuda(), k.cuda(), v.cuda(), query_scale=a, softcap=0.0, window=W)
    torch.cuda.synchronize()
    ro, rl = oracle.attn(q, k, v, query_scale=a, softcap=0.0, window=W)
    check(out, ro, lse, rl, f"no cap d={d} W={W}")


def test_no_cap_decode():
    lengths, cu, q, k, v = decode_inputs(8, 500, 3000, 8, 4, 256, seed=77)
    out, lse = g2.decode(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths),
                         query_scale=1 / 16, softcap=0.0, window=1024)
    torch.cuda.synchronize()
    ro, rl = oracle.decode(q, k, v, cu, query_scale=1 / 16, softcap=0.0, window=1024)
    check(out, ro, lse, rl, "no-cap decode")
