"""g2attn_decode_noalloc: decode for callers that cannot allocate device
memory at call time (a serving loop whose memory another allocator planned up
front, a plug-in handed only input and output pointers, code that must avoid
cudaMalloc's implicit device synchronisation). It keeps its split-KV partials
in the library's static 24 MiB scratch instead of a caller workspace.

Checked through the C ABI on two calls in a row (the second call reuses the
scratch the first one left behind): bit for bit against g2attn_decode, which
runs the same kernels with the same split plan on a caller workspace, and
against the fp64 oracle within the library's tolerance. This file is named
so pytest collects it last, and it passes alone in a fresh process too.
"""
import ctypes

import pytest
import torch

import global_soft_capped_b200 as g2
import oracle
from global_soft_capped_b200.inputs import WORKLOADS, decode_inputs
from parity import check

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def test_noalloc_decode_matches_workspace_decode_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = WORKLOADS["27b_decode"]
    lengths, cu, q_h, k_h, v_h = decode_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d,
                                               w.std, w.seed)
    q, k, v, cu = q_h.cuda(), k_h.cuda(), v_h.cuda(), cu.cuda()
    n, H, d = q.shape
    L = max(lengths)
    assert g2.g2attn_decode_workspace_size(n, H, d, L) <= 24 << 20
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, window in enumerate((w.window_local, 0)):
        ws = torch.empty(g2.g2attn_decode_workspace_size(n, H, d, L), dtype=torch.uint8,
                         device="cuda")
        ref_out, ref_lse = torch.empty_like(q), torch.empty(n, H, device="cuda")
        st = g2.g2attn_decode(_p(q), _p(k), _p(v), _p(cu), _p(ref_out), _p(ref_lse), n,
                              k.shape[0], L, H, w.Hkv, d, w.query_scale, w.softcap, window,
                              _p(ws), ws.numel(), stream)
        assert st == g2.G2ATTN_OK
        out, lse = torch.full_like(q, float("nan")), torch.full((n, H), float("nan"),
                                                                device="cuda")
        st = g2.g2attn_decode_noalloc(_p(q), _p(k), _p(v), _p(cu), _p(out), _p(lse), n,
                                      k.shape[0], L, H, w.Hkv, d, w.query_scale, w.softcap,
                                      window, stream)
        assert st == g2.G2ATTN_OK, f"call {call}: {g2.g2attn_status_string(st)}"
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), f"call {call}: out differs from g2attn_decode"
        assert torch.equal(lse, ref_lse), f"call {call}: lse differs from g2attn_decode"
        ro, rl = oracle.decode(q_h, k_h, v_h, cu.cpu(), query_scale=w.query_scale,
                               softcap=w.softcap, window=window)
        check(out, ro, lse, rl, f"noalloc call {call} against the oracle")
    assert g2.g2attn_get_device_error() == g2.G2ATTN_OK


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    n, H, d, L = 1024, 64, 256, 65536  # needs far more than 24 MiB of partials
    assert g2.g2attn_decode_workspace_size(n, H, d, L) > 24 << 20
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(n + 1, dtype=torch.int32, device="cuda")
    st = g2.g2attn_decode_noalloc(_p(x), _p(x), _p(x), _p(cu), _p(x), None, n, 8, L, H, H // 2,
                                  d, 0.1, 50.0, 0, None)
    assert st == g2.G2ATTN_ERR_WORKSPACE
