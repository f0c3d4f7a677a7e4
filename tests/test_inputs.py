"""The seeded input generators (shared by the oracle tests, the GPU parity
tests and the bench): determinism, draw order and the workload recipes.

These hold the properties the tests and the bench rely on: the same seed gives
the same bits; the gradient inputs extend the forward inputs (dout is drawn
after q, k, v from the same generator, so the forward of a gradient workload
sees exactly the forward workload's tensors); lengths stay in their stated
ranges; packed offsets add up.
"""
import numpy as np
import torch

from global_soft_capped_b200 import inputs as gi


def test_same_seed_same_bits_and_seeds_differ():
    a = gi.prefill_inputs(1, 40, 50, 4, 2, 64, 1.0, 7)
    b = gi.prefill_inputs(1, 40, 50, 4, 2, 64, 1.0, 7)
    c = gi.prefill_inputs(1, 40, 50, 4, 2, 64, 1.0, 8)
    for x, y, z in zip(a, b, c):
        assert x.dtype == torch.bfloat16
        assert torch.equal(x, y)
        assert not torch.equal(x, z)
    assert a[0].shape == (1, 40, 4, 64) and a[1].shape == (1, 50, 2, 64)


def test_gradient_inputs_extend_forward_inputs():
    q, k, v = gi.prefill_inputs(2, 33, 70, 4, 2, 64, 1.0, 3)
    q2, k2, v2, dout = gi.backward_inputs(2, 33, 70, 4, 2, 64, 1.0, 3)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    assert dout.shape == q.shape and dout.dtype == torch.bfloat16
    a = gi.varlen_inputs(5, 10, 60, 4, 2, 64, 1.0, 11)
    b = gi.varlen_backward_inputs(5, 10, 60, 4, 2, 64, 1.0, 11)
    for x, y in zip(a, b[:7]):
        if isinstance(x, torch.Tensor):
            assert torch.equal(x, y)
        else:
            assert x == y
    assert b[7].shape == a[4].shape


def test_lengths_and_offsets():
    lengths, cu, q, k, v = gi.decode_inputs(64, 1024, 8192, 4, 2, 64, seed=3)
    assert len(lengths) == 64 and min(lengths) >= 1024 and max(lengths) <= 8192
    assert cu.dtype == torch.int32 and cu[0] == 0 and int(cu[-1]) == sum(lengths)
    assert np.all(np.diff(cu.numpy()) == np.asarray(lengths))
    assert q.shape == (64, 4, 64) and k.shape == (sum(lengths), 2, 64)
    Ts, Ss, cq, ck, q, k, v = gi.varlen_inputs(16, 512, 8192, 4, 2, 64, 1.0, 4,
                                               tail_T=1024, tail_S=8192)
    assert len(Ts) == 17 and Ts[-1] == 1024 and Ss[-1] == 8192
    assert all(512 <= t == s <= 8192 for t, s in zip(Ts[:-1], Ss[:-1]))
    assert int(cq[-1]) == sum(Ts) == q.shape[0] and int(ck[-1]) == sum(Ss) == k.shape[0]


def test_tiny_workload_std():
    w = gi.WORKLOADS["tiny"]
    q, k, v = gi.prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    sd = float(torch.cat([q.flatten(), k.flatten(), v.flatten()]).float().std())
    assert abs(sd - 1.5) < 0.05       # N(0, 1.5) read as a standard deviation
