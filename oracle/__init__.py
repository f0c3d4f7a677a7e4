"""fp64 CPU oracle for the Gemma 2 per-layer attention forward.

TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this package. The CUDA library never
calls it, and it shares no code with the CUDA library (its arithmetic lives in
``g2ref.c``, compiled with gcc by :func:`build`).

Functions (each follows the Gemma 2 card's per-layer attention pseudo-code,
"Method" section, with the soft-cap formula of the "Gemma 2 Guide", section 1):

* :func:`attn`        dense layer: q (B,T,H,d), k/v (B,S,Hkv,d) -> out, lse
* :func:`attn_rows`   the same definition for chosen (b, i, h) rows
* :func:`row_detail`  one row's masked capped logits and softmax weights
* :func:`decode`      one query per sequence at position L-1 of its cache
* :func:`varlen`      packed sequences, each a dense layer with q_offset = S_i - T_i
* :func:`attn_bwd`    gradients of the dense layer (dq, dk, dv) for an upstream dout
* :func:`attn_bwd_sampled`  the same gradients at chosen query rows and chosen keys

Parity of every function is pinned by ``tests/test_oracle_pins.py`` (the
gradients by ``tests/test_oracle_backward_pins.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "g2ref.c")
_LIB_DEFAULT = os.path.join(_HERE, "libg2ref.so")
# G2REF_LIB points the oracle at another build of g2ref.c; the mutation tests
# use it to check that the pins reject deliberately broken copies.
_LIB = os.environ.get("G2REF_LIB", _LIB_DEFAULT)
_lib = None


def build(force: bool = False) -> str:
    """Compile g2ref.c into libg2ref.so next to it (gcc, OpenMP, -O2)."""
    if _LIB != _LIB_DEFAULT:
        return _LIB
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "g2ref.h"))):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-o",
               _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P, I64, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double
        lib.g2ref_attn.argtypes = [P, P, P, P, P] + [I64] * 7 + [D, D, I64]
        lib.g2ref_attn.restype = ctypes.c_int
        lib.g2ref_attn_rows.argtypes = [P, P, P, P, P, P, I64] + [I64] * 7 + [D, D, I64]
        lib.g2ref_attn_rows.restype = ctypes.c_int
        lib.g2ref_row_detail.argtypes = [P, P, P, P, I64, I64, I64] + [I64] * 7 + [D, D, I64]
        lib.g2ref_row_detail.restype = ctypes.c_int
        lib.g2ref_attn_bwd.argtypes = [P] * 7 + [I64] * 7 + [D, D, I64]
        lib.g2ref_attn_bwd.restype = ctypes.c_int
        lib.g2ref_attn_bwd_sampled.argtypes = [P] * 5 + [I64, P, I64] + [P] * 3 + [I64] * 7 + [
            D, D, I64]
        lib.g2ref_attn_bwd_sampled.restype = ctypes.c_int
        lib.g2ref_set_threads.argtypes = [ctypes.c_int]
        lib.g2ref_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def set_threads(n: int) -> None:
    _load().g2ref_set_threads(int(n))


def max_threads() -> int:
    return int(_load().g2ref_max_threads())


def _bits(t) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy bits."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16, t.dtype
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def attn(q, k, v, q_offset=0, query_scale=1.0, softcap=50.0, window=0):
    """Dense layer. Returns (out (B,T,H,d) float64, lse (B,H,T) float64)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, T, H, d = qb.shape
    S, Hkv = kb.shape[1], kb.shape[2]
    assert kb.shape == (B, S, Hkv, d) and vb.shape == kb.shape
    out = np.empty((B, T, H, d), np.float64)
    lse = np.empty((B, H, T), np.float64)
    rc = _load().g2ref_attn(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), _ptr(lse),
                            B, T, S, H, Hkv, d, int(q_offset), float(query_scale),
                            float(softcap), int(window))
    if rc != 0:
        raise ValueError("g2ref_attn rejected its arguments")
    return out, lse


def attn_rows(q, k, v, rows, q_offset=0, query_scale=1.0, softcap=50.0, window=0):
    """Rows (n,3) of (b, i, h). Returns (out (n,d), lse (n,)) float64."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, T, H, d = qb.shape
    S, Hkv = kb.shape[1], kb.shape[2]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    out = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().g2ref_attn_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), _ptr(lse),
                                 _ptr(rows), n, B, T, S, H, Hkv, d, int(q_offset),
                                 float(query_scale), float(softcap), int(window))
    if rc != 0:
        raise ValueError("g2ref_attn_rows rejected its arguments")
    return out, lse


def row_detail(q, k, b, i, h, q_offset=0, query_scale=1.0, softcap=50.0, window=0):
    """Masked capped logits s (S,) (-inf where masked) and weights w (S,)."""
    qb, kb = _bits(q), _bits(k)
    B, T, H, d = qb.shape
    S, Hkv = kb.shape[1], kb.shape[2]
    s = np.empty((S,), np.float64)
    w = np.empty((S,), np.float64)
    rc = _load().g2ref_row_detail(_ptr(qb), _ptr(kb), _ptr(s), _ptr(w), b, i, h, B, T, S, H,
                                  Hkv, d, int(q_offset), float(query_scale), float(softcap),
                                  int(window))
    if rc != 0:
        raise ValueError("g2ref_row_detail rejected its arguments")
    return s, w


def attn_bwd(q, k, v, dout, q_offset=0, query_scale=1.0, softcap=50.0, window=0):
    """Gradients of :func:`attn` for the upstream gradient dout (B,T,H,d).

    Returns (dq (B,T,H,d), dk (B,S,Hkv,d), dv (B,S,Hkv,d)) as float64: the
    chain rule through the mix, the softmax, the soft-cap (derivative
    1 - tanh^2, "Gemma 2 Guide", Deep Dive item 1) and the scaled dot product.
    """
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, T, H, d = qb.shape
    S, Hkv = kb.shape[1], kb.shape[2]
    assert kb.shape == (B, S, Hkv, d) and vb.shape == kb.shape and gb.shape == qb.shape
    dq = np.empty((B, T, H, d), np.float64)
    dk = np.empty((B, S, Hkv, d), np.float64)
    dv = np.empty((B, S, Hkv, d), np.float64)
    rc = _load().g2ref_attn_bwd(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gb), _ptr(dq), _ptr(dk),
                                _ptr(dv), B, T, S, H, Hkv, d, int(q_offset), float(query_scale),
                                float(softcap), int(window))
    if rc != 0:
        raise ValueError("g2ref_attn_bwd rejected its arguments")
    return dq, dk, dv


def attn_bwd_sampled(q, k, v, dout, qrows, keys, q_offset=0, query_scale=1.0, softcap=50.0,
                     window=0):
    """Gradients of :func:`attn` at chosen places, for layers too large for
    :func:`attn_bwd`.

    ``qrows`` is (nq, 3) of (b, i, h) and ``keys`` (nk, 3) of (b, j, g), g a
    KV head. Returns (dq (nq,d), dk (nk,d), dv (nk,d)) float64: dq[b,i,h,:],
    and dk[b,j,g,:], dv[b,j,g,:] summed over every row of the group's heads
    that sees key j. Same chain rule as :func:`attn_bwd`; the weights a key
    needs come from the statistics (lse, D) of the rows that see it.
    """
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, T, H, d = qb.shape
    S, Hkv = kb.shape[1], kb.shape[2]
    assert kb.shape == (B, S, Hkv, d) and vb.shape == kb.shape and gb.shape == qb.shape
    qrows = np.ascontiguousarray(np.asarray(qrows, dtype=np.int64).reshape(-1, 3))
    keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64).reshape(-1, 3))
    nq, nk = qrows.shape[0], keys.shape[0]
    dq = np.empty((nq, d), np.float64)
    dk = np.empty((nk, d), np.float64)
    dv = np.empty((nk, d), np.float64)
    rc = _load().g2ref_attn_bwd_sampled(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gb), _ptr(qrows), nq,
                                        _ptr(keys), nk, _ptr(dq), _ptr(dk), _ptr(dv), B, T, S, H,
                                        Hkv, d, int(q_offset), float(query_scale),
                                        float(softcap), int(window))
    if rc != 0:
        raise ValueError("g2ref_attn_bwd_sampled rejected its arguments")
    return dq, dk, dv


def decode(q, k_cache, v_cache, cu_seqlens_k, query_scale=1.0, softcap=50.0, window=0,
           seqs=None):
    """One query per sequence, at position L_s - 1 over its own cache.

    q (n,H,d); caches (sum L,Hkv,d) packed by cu_seqlens_k. Each sequence is a
    dense layer with T = 1, S = L_s and q_offset = L_s - 1. ``seqs`` picks a
    subset. Returns (out (n_sel,H,d), lse (n_sel,H)).
    """
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    cu = np.asarray(cu_seqlens_k, dtype=np.int64)
    n, H, d = qb.shape
    sel = range(n) if seqs is None else list(seqs)
    outs, lses = [], []
    for s_ in sel:
        k0, k1 = int(cu[s_]), int(cu[s_ + 1])
        o, l = attn(qb[s_][None, None], kb[k0:k1][None], vb[k0:k1][None], q_offset=k1 - k0 - 1,
                    query_scale=query_scale, softcap=softcap, window=window)
        outs.append(o[0, 0])
        lses.append(l[0, :, 0])
    return np.stack(outs), np.stack(lses)


def varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, query_scale=1.0, softcap=50.0, window=0,
           seqs=None):
    """Packed sequences; each is a dense layer with q_offset = S_i - T_i.

    q (sum T,H,d), k/v (sum S,Hkv,d). Returns (out (sum T,H,d), lse (H, sum T));
    rows of sequences not in ``seqs`` are left as NaN.
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    total_q, H, d = qb.shape
    out = np.full((total_q, H, d), np.nan)
    lse = np.full((H, total_q), np.nan)
    sel = range(len(cq) - 1) if seqs is None else list(seqs)
    for s_ in sel:
        q0, q1, k0, k1 = int(cq[s_]), int(cq[s_ + 1]), int(ck[s_]), int(ck[s_ + 1])
        if q1 == q0:
            continue
        o, l = attn(qb[q0:q1][None], kb[k0:k1][None], vb[k0:k1][None],
                    q_offset=(k1 - k0) - (q1 - q0), query_scale=query_scale,
                    softcap=softcap, window=window)
        out[q0:q1] = o[0]
        lse[:, q0:q1] = l[0]
    return out, lse
