"""CUDA prefill (tcgen05) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import WORKLOADS, prefill_inputs
from parity import check, sample_positions

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    g2.load_library()
    yield
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK


def run(q, k, v, **kw):
    out, lse = g2.prefill(q.cuda(), k.cuda(), v.cuda(), **kw)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("window", [64, 0])
def test_tiny_pair_full(window):
    w = WORKLOADS["tiny"]
    q, k, v = prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    out, lse = run(q, k, v, query_scale=w.query_scale, softcap=w.softcap, window=window)
    ro, rl = oracle.attn(q, k, v, query_scale=w.query_scale, softcap=w.softcap, window=window)
    check(out, ro, lse, rl, f"tiny window={window}")


EDGE = [
    # B, T, S, H, Hkv, d, q_offset, window, softcap, alpha, std
    (1, 1, 1, 2, 1, 64, 0, 0, 50.0, 0.125, 1.0),
    (1, 65, 65, 2, 1, 64, 0, 0, 50.0, 0.125, 1.0),
    (1, 130, 130, 4, 2, 64, 0, 1, 50.0, 0.125, 1.0),
    (2, 200, 300, 4, 2, 128, 100, 63, 50.0, 0.09, 1.0),
    (1, 257, 257, 2, 1, 128, 0, 64, 50.0, 0.09, 1.0),
    (1, 257, 257, 2, 1, 128, 0, 65, 50.0, 0.09, 1.0),
    (1, 300, 300, 2, 1, 256, 0, 127, 50.0, 0.0625, 1.0),
    (1, 300, 300, 2, 1, 256, 0, 128, 50.0, 0.0625, 1.0),
    (1, 300, 300, 2, 1, 256, 0, 129, 50.0, 0.0625, 1.0),
    (1, 130, 1000, 4, 2, 256, 870, 300, 50.0, 0.0625, 1.0),
    (1, 77, 500, 2, 1, 256, 423, 0, 50.0, 0.0625, 1.0),
    (3, 100, 100, 4, 2, 64, 0, 4096, 50.0, 0.125, 1.0),
    (1, 190, 190, 2, 1, 128, 0, 50, 0.0, 0.09, 1.0),      # no cap
    (1, 128, 128, 2, 1, 64, 0, 0, 50.0, 4.0, 1.0),        # logits well past the cap
    (1, 192, 192, 2, 1, 256, 0, 70, 50.0, 0.25, 1.0),
    # cap above C log2(e) = 95, i.e. C > 65.8: running max with the cap on
    (1, 300, 300, 2, 1, 128, 0, 0, 100.0, 0.09, 1.0),     # series range
    (1, 200, 200, 2, 1, 256, 0, 64, 100.0, 4.0, 1.0),     # logits past the series range
    (2, 150, 260, 4, 2, 64, 110, 0, 80.0, 0.5, 1.0),
]


@pytest.mark.parametrize("case", EDGE, ids=[str(i) for i in range(len(EDGE))])
def test_edge_shapes_full(case):
    B, T, S, H, Hkv, d, qo, W, C, a, std = case
    q, k, v = prefill_inputs(B, T, S, H, Hkv, d, std, seed=100 + EDGE.index(case))
    out, lse = run(q, k, v, q_offset=qo, query_scale=a, softcap=C, window=W)
    ro, rl = oracle.attn(q, k, v, q_offset=qo, query_scale=a, softcap=C, window=W)
    check(out, ro, lse, rl, f"edge {case}")


def test_lse_optional_and_explicit_stream():
    q, k, v = prefill_inputs(1, 150, 150, 4, 2, 128, seed=5)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
        out, lse = g2.prefill(qc, kc, vc, query_scale=0.09, window=33, want_lse=False, stream=s)
    s.synchronize()
    assert lse is None
    ro, _ = oracle.attn(q, k, v, query_scale=0.09, window=33)
    check(out, ro, what="no lse")


def test_window_at_least_S_equals_global_bitwise():
    q, k, v = prefill_inputs(1, 300, 300, 4, 2, 64, seed=6)
    og, lg = run(q, k, v, query_scale=0.1, window=0)
    ow, lw = run(q, k, v, query_scale=0.1, window=300)
    assert torch.equal(og, ow) and torch.equal(lg, lw)


@pytest.mark.parametrize("name", ["2b", "9b"])
@pytest.mark.parametrize("layer", ["local", "global"])
def test_full_size_sampled_rows(name, layer):
    """The benchmark's launch configuration at full size: every row is
    finite, and sampled rows (tile edges, window edges, both ends, random)
    match the oracle row by row."""
    w = WORKLOADS[name]
    window = w.window_local if layer == "local" else 0
    q, k, v = prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    out, lse = run(q, k, v, query_scale=w.query_scale, softcap=w.softcap, window=window)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    pos = sample_positions(w.T, window, 12, seed=w.seed)
    rows = [(b, i, h) for b in range(w.B) for i in pos for h in range(w.H)]
    ro, rl = oracle.attn_rows(q, k, v, rows, query_scale=w.query_scale, softcap=w.softcap,
                              window=window)
    oc, lc = out.cpu(), lse.cpu()
    go = torch.stack([oc[b, i, h] for b, i, h in rows])
    gl = torch.stack([lc[b, h, i] for b, i, h in rows])
    check(go, ro, gl, rl, f"{name} {layer} sampled")


@pytest.mark.parametrize("d", [64, 256])
def test_output_only_16_byte_aligned(d):
    """The epilogue stores 32 bytes at a time when out is 32-byte aligned and
    16 bytes otherwise; an output buffer offset by 16 bytes gives the same
    bits as an aligned one."""
    q, k, v = (t.cuda() for t in prefill_inputs(1, 200, 200, 4, 2, d, 1.0, 17))
    ref, lse = g2.prefill(q, k, v, query_scale=d ** -0.5, window=70)
    n = ref.numel()
    buf = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
    out = buf[8:8 + n].view(ref.shape)  # 16-byte aligned, not 32
    assert out.data_ptr() % 32 == 16
    g2.prefill(q, k, v, query_scale=d ** -0.5, window=70, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
