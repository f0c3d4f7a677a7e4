"""Seeded synthetic inputs for the soft-capped local/global attention workloads.

This module is the one piece shared by the CUDA path's tests and benchmark and
by the CPU oracle's tests. It draws random tensors and lengths and nothing
else: it holds none of the attention arithmetic (no scaling, capping, masking
or softmax), so neither side can inherit the other's mistakes through it.

Recipe (every workload): a CPU ``torch.Generator`` seeded with the workload's
seed draws, in this order, the sequence lengths (if any), then Q, K and V as
fp32 standard normals times ``std``, each rounded to bf16 (round to nearest
even). Shapes follow the per-layer attention statement of the Gemma 2 card
("Gemma 2: Improving Open Language Models at a Practical Size", Method,
attention pseudo-code header): queries (B, T, H, d), keys/values (B, S, K, d)
with K = H / 2. Head counts and head sizes are the 2B / 9B / 27B rows of the
same card ("Paper vs code": 8/4/256, 16/8/256, 32/16/128).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

# --------------------------------------------------------------------------
# Workload table
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" | "decode" | "varlen"
    H: int
    Hkv: int
    d: int
    window_local: int    # window of the local layer; the global layer uses 0
    query_scale: float
    softcap: float
    std: float
    seed: int
    B: int = 1
    T: int = 0
    S: int = 0
    num_seqs: int = 0
    len_lo: int = 0
    len_hi: int = 0
    tail_T: int = 0      # varlen: one extra chunked-prefill entry (T new queries ...)
    tail_S: int = 0      # ... over S keys, q_offset = S - T)
    note: str = field(default="", compare=False)


WORKLOADS = {
    "tiny": Workload(
        "tiny", "prefill", H=4, Hkv=2, d=64, window_local=64, query_scale=1.0,
        softcap=50.0, std=1.5, seed=0, B=1, T=256, S=256,
        note="tiny local+global pair, query_scale 1 so some logits pass the cap"),
    "2b": Workload(
        "2b", "prefill", H=8, Hkv=4, d=256, window_local=4096, query_scale=1.0 / 16,
        softcap=50.0, std=1.0, seed=1, B=1, T=8192, S=8192,
        note="2B-shaped prefill layer pair"),
    "9b": Workload(
        "9b", "prefill", H=16, Hkv=8, d=256, window_local=4096, query_scale=1.0 / 16,
        softcap=50.0, std=1.0, seed=2, B=2, T=8192, S=8192,
        note="9B-shaped batched prefill layer pair"),
    "27b_decode": Workload(
        "27b_decode", "decode", H=32, Hkv=16, d=128, window_local=4096,
        query_scale=144.0 ** -0.5, softcap=50.0, std=1.0, seed=3,
        num_seqs=64, len_lo=1024, len_hi=8192,
        note="27B-shaped decode, one query per sequence"),
    "9b_varlen": Workload(
        "9b_varlen", "varlen", H=16, Hkv=8, d=256, window_local=4096, query_scale=1.0 / 16,
        softcap=50.0, std=1.0, seed=4, num_seqs=16, len_lo=512, len_hi=8192,
        tail_T=1024, tail_S=8192,
        note="9B-shaped ragged packed prefill plus a chunked-prefill tail"),
    # Training-shaped 27B layer pair for the gradients (dout drawn after q, k, v
    # from the same generator, N(0, 1) -> bf16)
    "27b_backward": Workload(
        "27b_backward", "prefill", H=32, Hkv=16, d=128, window_local=4096,
        query_scale=144.0 ** -0.5, softcap=50.0, std=1.0, seed=6, B=1, T=8192, S=8192,
        note="27B-shaped layer pair, forward outputs and upstream gradients for the backward"),
    # Training-shaped 2B layer pair for the gradients at d = 256
    "2b_backward": Workload(
        "2b_backward", "prefill", H=8, Hkv=4, d=256, window_local=4096, query_scale=1.0 / 16,
        softcap=50.0, std=1.0, seed=8, B=1, T=8192, S=8192,
        note="2B-shaped layer pair, forward outputs and upstream gradients for the backward"),
    # Packed training batch of the same 27B shape: 8 self-attention sequences of
    # 512-8192 tokens, dout drawn after q, k, v from the same generator
    "27b_varlen_backward": Workload(
        "27b_varlen_backward", "varlen", H=32, Hkv=16, d=128, window_local=4096,
        query_scale=144.0 ** -0.5, softcap=50.0, std=1.0, seed=7, num_seqs=8, len_lo=512,
        len_hi=8192, note="27B-shaped packed batch, gradients of the packed layer pair"),
    # Gemma 3-shaped parameter variant of the same layer pair (the research-hub
    # page: window 1024, soft-capping replaced by QK-norm, which acts on the
    # inputs upstream of this kernel, so the cap is off here).
    "gemma3_2b": Workload(
        "gemma3_2b", "prefill", H=8, Hkv=4, d=256, window_local=1024, query_scale=1.0 / 16,
        softcap=0.0, std=1.0, seed=5, B=1, T=8192, S=8192,
        note="Gemma 3-shaped prefill layer pair: window 1024, no soft-cap"),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal_bf16(shape, std: float, g: torch.Generator) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def prefill_inputs(B, T, S, H, Hkv, d, std=1.0, seed=0):
    """Dense prefill inputs: q (B,T,H,d), k and v (B,S,Hkv,d), bf16 on the CPU."""
    g = _gen(seed)
    q = _normal_bf16((B, T, H, d), std, g)
    k = _normal_bf16((B, S, Hkv, d), std, g)
    v = _normal_bf16((B, S, Hkv, d), std, g)
    return q, k, v


def _lengths(n, lo, hi, g):
    if n == 0:
        return []
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def decode_inputs(num_seqs, len_lo, len_hi, H, Hkv, d, std=1.0, seed=0, lengths=None):
    """Decode inputs: one query per sequence at position L-1 of its cache.

    Returns (lengths, cu_seqlens_k int32 [n+1], q (n,H,d), k_cache (sum L,Hkv,d),
    v_cache). Cache lengths are integers drawn uniformly from [len_lo, len_hi]
    (both ends included) unless ``lengths`` is given.
    """
    g = _gen(seed)
    if lengths is None:
        lengths = _lengths(num_seqs, len_lo, len_hi, g)
    lengths = [int(x) for x in lengths]
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    q = _normal_bf16((len(lengths), H, d), std, g)
    k = _normal_bf16((cu[-1], Hkv, d), std, g)
    v = _normal_bf16((cu[-1], Hkv, d), std, g)
    return lengths, torch.tensor(cu, dtype=torch.int32), q, k, v


def varlen_inputs(num_seqs, len_lo, len_hi, H, Hkv, d, std=1.0, seed=0,
                  tail_T=0, tail_S=0, seq_lens=None):
    """Packed variable-length prefill inputs.

    ``num_seqs`` self-attention entries with T_i = S_i drawn uniformly from
    [len_lo, len_hi], then (if tail_T > 0) one chunked-prefill entry with
    T = tail_T queries over S = tail_S keys. ``seq_lens`` overrides the draw
    with explicit (T_i, S_i) pairs. Returns (T_list, S_list, cu_seqlens_q,
    cu_seqlens_k, q (sum T,H,d), k (sum S,Hkv,d), v).
    """
    return _varlen_draw(_gen(seed), num_seqs, len_lo, len_hi, H, Hkv, d, std, tail_T, tail_S,
                        seq_lens)


def _varlen_draw(g, num_seqs, len_lo, len_hi, H, Hkv, d, std, tail_T, tail_S, seq_lens):
    if seq_lens is None:
        ls = _lengths(num_seqs, len_lo, len_hi, g)
        Ts, Ss = list(ls), list(ls)
        if tail_T > 0:
            Ts.append(int(tail_T))
            Ss.append(int(tail_S))
    else:
        Ts = [int(t) for t, _ in seq_lens]
        Ss = [int(s) for _, s in seq_lens]
    cq, ck = [0], [0]
    for t, s in zip(Ts, Ss):
        cq.append(cq[-1] + t)
        ck.append(ck[-1] + s)
    q = _normal_bf16((cq[-1], H, d), std, g)
    k = _normal_bf16((ck[-1], Hkv, d), std, g)
    v = _normal_bf16((ck[-1], Hkv, d), std, g)
    return (Ts, Ss, torch.tensor(cq, dtype=torch.int32), torch.tensor(ck, dtype=torch.int32),
            q, k, v)


def varlen_backward_inputs(num_seqs, len_lo, len_hi, H, Hkv, d, std=1.0, seed=0):
    """varlen_inputs (no tail), then the upstream gradient dout (sum T,H,d),
    fp32 standard normals rounded to bf16, from the same generator."""
    g = _gen(seed)
    Ts, Ss, cq, ck, q, k, v = _varlen_draw(g, num_seqs, len_lo, len_hi, H, Hkv, d, std, 0, 0,
                                           None)
    dout = _normal_bf16(tuple(q.shape), 1.0, g)
    return Ts, Ss, cq, ck, q, k, v, dout


def backward_inputs(B, T, S, H, Hkv, d, std=1.0, seed=0):
    """q, k, v as prefill_inputs, then the upstream gradient dout (B,T,H,d),
    fp32 standard normals rounded to bf16, from the same generator."""
    g = _gen(seed)
    q = _normal_bf16((B, T, H, d), std, g)
    k = _normal_bf16((B, S, Hkv, d), std, g)
    v = _normal_bf16((B, S, Hkv, d), std, g)
    dout = _normal_bf16((B, T, H, d), 1.0, g)
    return q, k, v, dout


def workload_inputs(name: str):
    """Inputs of a named workload, drawn from its own seed."""
    w = WORKLOADS[name]
    if w.kind == "prefill":
        return prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    if w.kind == "decode":
        return decode_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d, w.std, w.seed)
    if w.kind == "varlen":
        return varlen_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d, w.std, w.seed,
                             tail_T=w.tail_T, tail_S=w.tail_S)
    raise ValueError(w.kind)
