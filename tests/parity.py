"""Comparison of CUDA outputs with the fp64 oracle.

Tolerances (fixed for this operation): bf16 outputs within max-abs 2e-2 and
relative L2 5e-3 of the oracle over each compared tensor; fp32 log-sum-exp
within 1e-3 absolute.
"""
import numpy as np
import torch

TOL_MAX_ABS = 2e-2
TOL_REL_L2 = 5e-3
TOL_LSE = 1e-3

# Errors of the comparisons a test asks to have reported (record=True); the
# test session prints them in its summary (tests/conftest.py).
RECORDS = []


def to_np(t):
    return t.detach().to(torch.float64).cpu().numpy() if isinstance(t, torch.Tensor) else t


def check(out, ref_out, lse=None, ref_lse=None, what="", record=False):
    o, r = to_np(out), np.asarray(ref_out, dtype=np.float64)
    assert o.shape == r.shape, (what, o.shape, r.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    d = np.abs(o - r)
    max_abs = float(d.max()) if d.size else 0.0
    rel = float(np.linalg.norm(o - r) / max(np.linalg.norm(r), 1e-30))
    msg = f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    assert max_abs <= TOL_MAX_ABS, msg
    assert rel <= TOL_REL_L2, msg
    lse_err = None
    if lse is not None:
        l, rl = to_np(lse), np.asarray(ref_lse, dtype=np.float64)
        assert l.shape == rl.shape, (what, l.shape, rl.shape)
        assert np.all(np.isfinite(l)), f"{what}: non-finite lse"
        lse_err = float(np.abs(l - rl).max())
        assert lse_err <= TOL_LSE, f"{msg} lse_err={lse_err:.3e}"
    if record:
        RECORDS.append(f"{what}: {o.size} values, max_abs {max_abs:.3e}, rel_l2 {rel:.3e}"
                       + (f", lse max {lse_err:.3e}" if lse_err is not None else ""))
    return max_abs, rel, lse_err


def sample_positions(T, window, n_random, seed):
    """Query rows that exercise tile edges, the window edge and both ends."""
    fixed = {0, 1, 2, 63, 64, 65, 127, 128, 129, T // 2, T - 2, T - 1}
    if window:
        fixed |= {window - 2, window - 1, window, window + 1, window + 63, window + 64}
    g = np.random.default_rng(seed)
    fixed |= set(int(x) for x in g.integers(0, T, n_random))
    return sorted(p for p in fixed if 0 <= p < T)
