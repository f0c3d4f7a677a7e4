"""CUDA split-KV decode against the fp64 oracle, through the C ABI."""
import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import WORKLOADS, decode_inputs
from parity import check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    g2.load_library()
    yield
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK


def run(lengths, cu, q, k, v, **kw):
    out, lse = g2.decode(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths), **kw)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("layer", ["local", "global"])
def test_27b_decode_full(layer):
    w = WORKLOADS["27b_decode"]
    window = w.window_local if layer == "local" else 0
    lengths, cu, q, k, v = decode_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d,
                                         w.std, w.seed)
    out, lse = run(lengths, cu, q, k, v, query_scale=w.query_scale, softcap=w.softcap,
                   window=window)
    ro, rl = oracle.decode(q, k, v, cu, query_scale=w.query_scale, softcap=w.softcap,
                           window=window)
    check(out, ro, lse, rl, f"27b decode {layer}")


CASES = [
    # lengths, H, Hkv, d, window, softcap, alpha
    ([1, 2, 3, 64, 65], 4, 2, 64, 0, 50.0, 0.125),
    ([1, 17, 4096, 4097, 5000], 8, 4, 128, 4096, 50.0, 0.09),
    ([700, 1, 1500], 4, 2, 256, 100, 50.0, 0.0625),
    ([33, 900], 2, 1, 128, 0, 0.0, 0.09),
    ([513, 1024, 1025], 2, 1, 64, 512, 50.0, 1.0),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_decode_shapes(case):
    lengths, H, Hkv, d, W, C, a = case
    lengths, cu, q, k, v = decode_inputs(0, 0, 0, H, Hkv, d, seed=40 + CASES.index(case),
                                         lengths=lengths)
    out, lse = run(lengths, cu, q, k, v, query_scale=a, softcap=C, window=W)
    ro, rl = oracle.decode(q, k, v, cu, query_scale=a, softcap=C, window=W)
    check(out, ro, lse, rl, f"decode {case}")


def test_decode_is_last_row_of_prefill():
    lengths, cu, q, k, v = decode_inputs(0, 0, 0, 4, 2, 128, seed=47, lengths=[300])
    out, lse = run(lengths, cu, q, k, v, query_scale=0.09, window=100)
    L = lengths[0]
    qf = torch.randn(1, L, 4, 128).to(torch.bfloat16)
    qf[0, -1] = q[0]
    po, pl = g2.prefill(qf.cuda(), k[None].cuda(), v[None].cuda(), query_scale=0.09, window=100)
    torch.cuda.synchronize()
    check(out[0], po[0, -1].double().cpu().numpy(), lse[0],
          pl[0, :, -1].double().cpu().numpy(), "decode vs prefill last row")


def test_cache_longer_than_max_cache_len_is_reported():
    """max_cache_len plans the splits; a sequence longer than it keeps only the
    splits the plan has room for. The call still returns OK (the host cannot
    see the lengths), stays inside its buffers, and the sticky device word
    reports G2ATTN_ERR_CACHE_LEN once. Sequences within the plan are right."""
    lengths, cu, q, k, v = decode_inputs(0, 0, 0, 4, 2, 64, seed=48, lengths=[90, 3000])
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
    out, lse = g2.decode(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), 100, query_scale=0.125)
    torch.cuda.synchronize()
    assert g2.g2attn_get_device_error() == g2.G2ATTN_ERR_CACHE_LEN
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK  # reading clears it
    ro, rl = oracle.decode(q, k, v, cu, query_scale=0.125, seqs=[0])
    check(out[:1], ro, lse[:1], rl, "sequence within the plan")
    # the same call with an honest max_cache_len leaves the word clear
    g2.decode(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths), query_scale=0.125)
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK
