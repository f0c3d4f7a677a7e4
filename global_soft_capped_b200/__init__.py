"""libg2attn Python binding: Gemma 2 soft-capped local/global attention on B200.

Two layers:

* The C entry points under their own names (``g2attn_prefill``,
  ``g2attn_prefill_varlen``, ``g2attn_prefill_paged``, ``g2attn_decode_workspace_size``,
  ``g2attn_decode``, ``g2attn_decode_ring``, ``g2attn_decode_paged``,
  ``g2attn_decode_noalloc``, ``g2attn_backward_workspace_size``,
  ``g2attn_prefill_backward``, ``g2attn_varlen_backward_workspace_size``,
  ``g2attn_prefill_varlen_backward``, ``g2attn_status_string``,
  ``g2attn_get_device_error``,
  ``g2attn_selftest_wait_timeout``): plain argument marshalling of integers,
  floats and raw pointers through ctypes, returning the status code.
* Tensor helpers (:func:`prefill`, :func:`prefill_varlen`, :func:`decode`,
  :func:`prefill_backward` and the others below)
  that take torch CUDA tensors, allocate the outputs with torch (memory
  plumbing only) and raise :class:`G2AttnError` on a nonzero status.

Every step of the attention runs in the CUDA kernels of ``libg2attn.so``.
There is no CPU or library fallback: if the shared library is missing the
first call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libg2attn.so")

G2ATTN_OK = 0
G2ATTN_ERR_INVALID_ARG = 1
G2ATTN_ERR_UNSUPPORTED = 2
G2ATTN_ERR_MISALIGNED = 3
G2ATTN_ERR_CUDA = 4
G2ATTN_ERR_DEVICE_TIMEOUT = 5
G2ATTN_ERR_WORKSPACE = 6
G2ATTN_ERR_CACHE_LEN = 7

EXPORTS = (
    "g2attn_prefill",
    "g2attn_prefill_varlen",
    "g2attn_prefill_paged",
    "g2attn_decode_workspace_size",
    "g2attn_decode",
    "g2attn_decode_ring",
    "g2attn_decode_paged",
    "g2attn_decode_noalloc",
    "g2attn_backward_workspace_size",
    "g2attn_prefill_backward",
    "g2attn_varlen_backward_workspace_size",
    "g2attn_prefill_varlen_backward",
    "g2attn_status_string",
    "g2attn_get_device_error",
    "g2attn_selftest_wait_timeout",
)


class G2AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_name(status)} (status {status})")


_lib = None


def load_library():
    """Load libg2attn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libg2attn.so is missing at {LIB_PATH}; build it with "
            "`python -m global_soft_capped_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.g2attn_prefill.argtypes = [P, P, P, P, P] + [I] * 7 + [F, F, I, P]
    lib.g2attn_prefill.restype = I
    lib.g2attn_prefill_varlen.argtypes = [P, P, P, P, P, P, P] + [I] * 8 + [F, F, I, P]
    lib.g2attn_prefill_varlen.restype = I
    lib.g2attn_prefill_paged.argtypes = [P, P, P, P, P, P, P, P] + [I] * 10 + [F, F, I, P]
    lib.g2attn_prefill_paged.restype = I
    lib.g2attn_decode_workspace_size.argtypes = [I, I, I, I]
    lib.g2attn_decode_workspace_size.restype = SZ
    lib.g2attn_decode.argtypes = [P, P, P, P, P, P] + [I] * 6 + [F, F, I, P, SZ, P]
    lib.g2attn_decode.restype = I
    lib.g2attn_decode_ring.argtypes = [P, P, P, P, P, P] + [I] * 6 + [F, F, I, P, SZ, P]
    lib.g2attn_decode_ring.restype = I
    lib.g2attn_decode_paged.argtypes = [P, P, P, P, P, P, P] + [I] * 8 + [F, F, I, P, SZ, P]
    lib.g2attn_decode_paged.restype = I
    lib.g2attn_decode_noalloc.argtypes = [P, P, P, P, P, P] + [I] * 6 + [F, F, I, P]
    lib.g2attn_decode_noalloc.restype = I
    lib.g2attn_backward_workspace_size.argtypes = [I, I, I]
    lib.g2attn_backward_workspace_size.restype = SZ
    lib.g2attn_prefill_backward.argtypes = [P] * 9 + [I] * 7 + [F, F, I, P, SZ, P]
    lib.g2attn_prefill_backward.restype = I
    lib.g2attn_varlen_backward_workspace_size.argtypes = [I, I, I]
    lib.g2attn_varlen_backward_workspace_size.restype = SZ
    lib.g2attn_prefill_varlen_backward.argtypes = [P] * 11 + [I] * 8 + [F, F, I, P, SZ, P]
    lib.g2attn_prefill_varlen_backward.restype = I
    lib.g2attn_status_string.argtypes = [I]
    lib.g2attn_status_string.restype = ctypes.c_char_p
    lib.g2attn_get_device_error.argtypes = []
    lib.g2attn_get_device_error.restype = I
    lib.g2attn_selftest_wait_timeout.argtypes = [I]
    lib.g2attn_selftest_wait_timeout.restype = I
    _lib = lib
    return lib


# ---------------------------------------------------------------------------
# C entry points, same names and argument order as include/g2attn.h
# ---------------------------------------------------------------------------
def g2attn_prefill(q, k, v, out, lse, B, T, S, H, Hkv, d, q_offset, query_scale, softcap,
                   window, stream):
    return load_library().g2attn_prefill(q, k, v, out, lse, B, T, S, H, Hkv, d, q_offset,
                                         query_scale, softcap, window, stream)


def g2attn_prefill_varlen(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q,
                          total_k, max_T, max_S, H, Hkv, d, query_scale, softcap, window, stream):
    return load_library().g2attn_prefill_varlen(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k,
                                                num_seqs, total_q, total_k, max_T, max_S, H, Hkv,
                                                d, query_scale, softcap, window, stream)


def g2attn_prefill_paged(q, k_blocks, v_blocks, out, lse, cu_seqlens_q, block_table, seq_lens_k,
                         num_seqs, total_q, num_blocks, block_size, max_blocks_per_seq, max_T,
                         max_S, H, Hkv, d, query_scale, softcap, window, stream):
    return load_library().g2attn_prefill_paged(q, k_blocks, v_blocks, out, lse, cu_seqlens_q,
                                               block_table, seq_lens_k, num_seqs, total_q,
                                               num_blocks, block_size, max_blocks_per_seq, max_T,
                                               max_S, H, Hkv, d, query_scale, softcap, window,
                                               stream)


def g2attn_backward_workspace_size(B, T, H):
    return load_library().g2attn_backward_workspace_size(B, T, H)


def g2attn_prefill_backward(q, k, v, out, lse, dout, dq, dk, dv, B, T, S, H, Hkv, d, q_offset,
                            query_scale, softcap, window, workspace, workspace_bytes, stream):
    return load_library().g2attn_prefill_backward(q, k, v, out, lse, dout, dq, dk, dv, B, T, S,
                                                  H, Hkv, d, q_offset, query_scale, softcap,
                                                  window, workspace, workspace_bytes, stream)


def g2attn_varlen_backward_workspace_size(num_seqs, total_q, H):
    return load_library().g2attn_varlen_backward_workspace_size(num_seqs, total_q, H)


def g2attn_prefill_varlen_backward(q, k, v, out, lse, dout, dq, dk, dv, cu_seqlens_q,
                                   cu_seqlens_k, num_seqs, total_q, total_k, max_T, max_S, H,
                                   Hkv, d, query_scale, softcap, window, workspace,
                                   workspace_bytes, stream):
    return load_library().g2attn_prefill_varlen_backward(
        q, k, v, out, lse, dout, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q,
        total_k, max_T, max_S, H, Hkv, d, query_scale, softcap, window, workspace,
        workspace_bytes, stream)


def g2attn_decode_workspace_size(num_seqs, H, d, max_cache_len):
    return load_library().g2attn_decode_workspace_size(num_seqs, H, d, max_cache_len)


def g2attn_decode(q, k_cache, v_cache, cu_seqlens_k, out, lse, num_seqs, total_k, max_cache_len,
                  H, Hkv, d, query_scale, softcap, window, workspace, workspace_bytes, stream):
    return load_library().g2attn_decode(q, k_cache, v_cache, cu_seqlens_k, out, lse, num_seqs,
                                        total_k, max_cache_len, H, Hkv, d, query_scale, softcap,
                                        window, workspace, workspace_bytes, stream)


def g2attn_decode_ring(q, k_ring, v_ring, seq_lens, out, lse, num_seqs, ring_size, max_cache_len,
                       H, Hkv, d, query_scale, softcap, window, workspace, workspace_bytes,
                       stream):
    return load_library().g2attn_decode_ring(q, k_ring, v_ring, seq_lens, out, lse, num_seqs,
                                             ring_size, max_cache_len, H, Hkv, d, query_scale,
                                             softcap, window, workspace, workspace_bytes, stream)


def g2attn_decode_paged(q, k_blocks, v_blocks, block_table, seq_lens, out, lse, num_seqs,
                        num_blocks, block_size, max_blocks_per_seq, max_cache_len, H, Hkv, d,
                        query_scale, softcap, window, workspace, workspace_bytes, stream):
    return load_library().g2attn_decode_paged(q, k_blocks, v_blocks, block_table, seq_lens, out,
                                              lse, num_seqs, num_blocks, block_size,
                                              max_blocks_per_seq, max_cache_len, H, Hkv, d,
                                              query_scale, softcap, window, workspace,
                                              workspace_bytes, stream)


def g2attn_decode_noalloc(q, k_cache, v_cache, cu_seqlens_k, out, lse, num_seqs, total_k,
                          max_cache_len, H, Hkv, d, query_scale, softcap, window, stream):
    """Decode with the library's static scratch instead of a caller workspace,
    for callers that cannot allocate device memory at call time."""
    return load_library().g2attn_decode_noalloc(q, k_cache, v_cache, cu_seqlens_k, out, lse,
                                                num_seqs, total_k, max_cache_len, H, Hkv, d,
                                                query_scale, softcap, window, stream)


def g2attn_status_string(status):
    return load_library().g2attn_status_string(status).decode()


def g2attn_get_device_error():
    return load_library().g2attn_get_device_error()


def g2attn_selftest_wait_timeout(timeout_us):
    return load_library().g2attn_selftest_wait_timeout(timeout_us)


def status_name(status: int) -> str:
    try:
        return g2attn_status_string(status)
    except Exception:  # library not loadable: still give a readable message
        return f"status {status}"


# ---------------------------------------------------------------------------
# Tensor helpers (torch allocates; the kernels compute)
# ---------------------------------------------------------------------------
def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_bf16(*ts):
    import torch
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("expected contiguous bf16 CUDA tensors")


def prefill(q, k, v, *, q_offset=0, query_scale=1.0, softcap=50.0, window=0, out=None,
            lse=None, want_lse=True, stream=None):
    """Dense prefill. q (B,T,H,d), k/v (B,S,Hkv,d) -> (out (B,T,H,d), lse (B,H,T) | None)."""
    import torch
    _check_bf16(q, k, v)
    B, T, H, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    st = g2attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, T, S, H, Hkv, d,
                        int(q_offset), float(query_scale), float(softcap), int(window),
                        _stream(stream))
    if st != G2ATTN_OK:
        raise G2AttnError(st, "g2attn_prefill")
    return out, lse


def prefill_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_T, max_S, *, query_scale=1.0,
                   softcap=50.0, window=0, out=None, lse=None, want_lse=True, stream=None):
    """Packed prefill. q (sum T,H,d), k/v (sum S,Hkv,d); cu_seqlens int32 CUDA tensors."""
    import torch
    _check_bf16(q, k, v)
    total_q, H, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    num_seqs = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    st = g2attn_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                               _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), num_seqs, total_q, total_k,
                               int(max_T), int(max_S), H, Hkv, d, float(query_scale),
                               float(softcap), int(window), _stream(stream))
    if st != G2ATTN_OK:
        raise G2AttnError(st, "g2attn_prefill_varlen")
    return out, lse


def backward_workspace(B, T, H, device="cuda"):
    """A device buffer of g2attn_backward_workspace_size(B, T, H) bytes."""
    import torch
    n = g2attn_backward_workspace_size(B, T, H)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def prefill_backward(q, k, v, out, lse, dout, *, q_offset=0, query_scale=1.0, softcap=50.0,
                     window=0, workspace=None, dq=None, dk=None, dv=None, stream=None):
    """Gradients of :func:`prefill`: returns (dq, dk, dv) like q, k, v (bf16)."""
    import torch
    _check_bf16(q, k, v, out, dout)
    B, T, H, d = q.shape
    S, Hkv = k.shape[1], k.shape[2]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = backward_workspace(B, T, H, q.device)
    st = g2attn_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, T, S, H, Hkv, d, int(q_offset),
                                 float(query_scale), float(softcap), int(window), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    if st != G2ATTN_OK:
        raise G2AttnError(st, "g2attn_prefill_backward")
    return dq, dk, dv


def prefill_varlen_backward(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, max_T, max_S,
                            *, query_scale=1.0, softcap=50.0, window=0, workspace=None, dq=None,
                            dk=None, dv=None, stream=None):
    """Gradients of :func:`prefill_varlen`: returns (dq, dk, dv), packed like q, k, v."""
    import torch
    _check_bf16(q, k, v, out, dout)
    total_q, H, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    num_seqs = cu_seqlens_q.numel() - 1
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        n = g2attn_varlen_backward_workspace_size(num_seqs, total_q, H)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    st = g2attn_prefill_varlen_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), num_seqs, total_q, total_k,
        int(max_T), int(max_S), H, Hkv, d, float(query_scale), float(softcap), int(window),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if st != G2ATTN_OK:
        raise G2AttnError(st, "g2attn_prefill_varlen_backward")
    return dq, dk, dv


def decode_workspace(num_seqs, H, d, max_cache_len, device="cuda"):
    import torch
    nbytes = g2attn_decode_workspace_size(num_seqs, H, d, max_cache_len)
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def decode(q, k_cache, v_cache, cu_seqlens_k, max_cache_len, *, query_scale=1.0, softcap=50.0,
           window=0, out=None, lse=None, workspace=None, want_lse=True, stream=None):
    """Decode. q (n,H,d), caches (sum L,Hkv,d), cu_seqlens_k int32 CUDA (n+1)."""
    import torch
    _check_bf16(q, k_cache, v_cache)
    n, H, d = q.shape
    total_k, Hkv = k_cache.shape[0], k_cache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((n, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = decode_workspace(n, H, d, max_cache_len, q.device)
    st = g2attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cu_seqlens_k), _ptr(out),
                       _ptr(lse), n, total_k, int(max_cache_len), H, Hkv, d, float(query_scale),
                       float(softcap), int(window), _ptr(workspace), workspace.numel(),
                       _stream(stream))
    if st != G2ATTN_OK:
        raise G2AttnError(st, "g2attn_decode")
    return out, lse


def decode_ring(q, k_ring, v_ring, seq_lens, window, max_cache_len=None, *, query_scale=1.0,
                softcap=50.0, out=None, lse=None, workspace=None, want_lse=True, stream=None):
    """Decode over ring caches (n, R, Hkv, d); seq_lens int32 CUDA (n,)."""
    import torch
    _check_bf16(q, k_ring, v_ring)
    n, H, d = q.shape
    R, Hkv = k_ring.shape[1], k_ring.shape[2]
    max_cache_len = int(window if max_cache_len is None else max_cache_len)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((n, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = decode_workspace(n, H, d, max_cache_len, q.device)
    st = g2attn_decode_ring(_ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(seq_lens), _ptr(out),
                            _ptr(lse), n, R, max_cache_len, H, Hkv, d, float(query_scale),
                            float(softcap), int(window), _ptr(workspace), workspace.numel(),
                            _stream(stream))
    if st != G2ATTN_OK:
        raise G2AttnError(st, "g2attn_decode_ring")
    return out, lse


def decode_paged(q, k_blocks, v_blocks, block_table, seq_lens, max_cache_len, *,
                 query_scale=1.0, softcap=50.0, window=0, out=None, lse=None, workspace=None,
                 want_lse=True, stream=None):
    """Decode over paged caches (num_blocks, bs, Hkv, d); block_table int32 (n, max_blocks)."""
    import torch
    _check_bf16(q, k_blocks, v_blocks)
    n, H, d = q.shape
    nb, bs, Hkv = k_blocks.shape[0], k_blocks.shape[1], k_blocks.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((n, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = decode_workspace(n, H, d, max_cache_len, q.device)
    st = g2attn_decode_paged(_ptr(q), _ptr(k_blocks), _ptr(v_blocks), _ptr(block_table),
                             _ptr(seq_lens), _ptr(out), _ptr(lse), n, nb, bs,
                             block_table.shape[1], int(max_cache_len), H, Hkv, d,
                             float(query_scale), float(softcap), int(window), _ptr(workspace),
                             workspace.numel(), _stream(stream))
    if st != G2ATTN_OK:
        raise G2AttnError(st, "g2attn_decode_paged")
    return out, lse


def prefill_paged(q, k_blocks, v_blocks, cu_seqlens_q, block_table, seq_lens_k, max_T, max_S, *,
                  query_scale=1.0, softcap=50.0, window=0, out=None, lse=None, want_lse=True,
                  stream=None):
    """Chunked prefill: packed q (sum T,H,d) over paged K/V (num_blocks, bs, Hkv, d)."""
    import torch
    _check_bf16(q, k_blocks, v_blocks)
    total_q, H, d = q.shape
    nb, bs, Hkv = k_blocks.shape[0], k_blocks.shape[1], k_blocks.shape[2]
    num_seqs = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    st = g2attn_prefill_paged(_ptr(q), _ptr(k_blocks), _ptr(v_blocks), _ptr(out), _ptr(lse),
                              _ptr(cu_seqlens_q), _ptr(block_table), _ptr(seq_lens_k), num_seqs,
                              total_q, nb, bs, block_table.shape[1], int(max_T), int(max_S), H,
                              Hkv, d, float(query_scale), float(softcap), int(window),
                              _stream(stream))
    if st != G2ATTN_OK:
        raise G2AttnError(st, "g2attn_prefill_paged")
    return out, lse
