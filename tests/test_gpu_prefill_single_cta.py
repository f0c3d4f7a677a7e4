"""The single-CTA d = 256 prefill kernel, kept behind G2ATTN_PREFILL_PAIR=0.

d = 256 runs on CTA pairs by default; the library reads the switch once per
process, so the single-CTA kernel is exercised in child processes:

* its parity suites (dense edge shapes, varlen, paged) against the oracle;
* bitwise equality of the two kernels on the same inputs. Both compute every
  logit with the same UMMA K-order and run the same softmax code, so their
  outputs and LSEs must agree exactly, which checks the pair's split of K and
  V over two CTAs element by element.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[2])
import global_soft_capped_b200 as g2
from global_soft_capped_b200.inputs import WORKLOADS, prefill_inputs, varlen_inputs
res = {}
w = WORKLOADS["2b"]
q, k, v = (t.cuda() for t in prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed))
for win in (w.window_local, 0):
    o, l = g2.prefill(q, k, v, query_scale=w.query_scale, softcap=w.softcap, window=win)
    res[f"2b_w{win}_out"] = o.view(torch.int16).cpu().numpy()
    res[f"2b_w{win}_lse"] = l.cpu().numpy()
for (qo, T, S, W) in [(870, 130, 1000, 300), (0, 300, 300, 129), (423, 77, 500, 0)]:
    q, k, v = (t.cuda() for t in prefill_inputs(1, T, S, 4, 2, 256, 1.0, 9))
    o, l = g2.prefill(q, k, v, q_offset=qo, query_scale=0.0625, window=W)
    res[f"T{T}_out"] = o.view(torch.int16).cpu().numpy()
    res[f"T{T}_lse"] = l.cpu().numpy()
Ts, Ss, cq, ck, q, k, v = varlen_inputs(0, 0, 0, 4, 2, 256, 1.0, 13,
                                        seq_lens=[(300, 300), (128, 1000), (7, 7), (1000, 1500)])
o, l = g2.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), max(Ts), max(Ss),
                         query_scale=0.0625, window=129)
res["varlen_out"] = o.view(torch.int16).cpu().numpy()
res["varlen_lse"] = l.cpu().numpy()
np.savez(sys.argv[1], **res)
"""


def _run_child(path, pair):
    env = dict(os.environ, G2ATTN_PREFILL_PAIR="1" if pair else "0")
    subprocess.run([sys.executable, "-c", _CHILD, str(path), ROOT], env=env, check=True,
                   timeout=600)
    return np.load(path)


def test_pair_and_single_cta_kernels_agree_bitwise(tmp_path):
    a = _run_child(tmp_path / "pair.npz", True)
    b = _run_child(tmp_path / "single.npz", False)
    assert sorted(a.files) == sorted(b.files)
    for key in a.files:
        assert np.array_equal(a[key], b[key], equal_nan=True), key


def test_single_cta_parity_suites():
    env = dict(os.environ, G2ATTN_PREFILL_PAIR="0")
    res = subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
         "tests/test_gpu_prefill.py::test_edge_shapes_full",
         "tests/test_gpu_prefill.py::test_tiny_pair_full",
         "tests/test_gpu_varlen.py::test_varlen_shapes_full",
         "tests/test_gpu_prefill_paged.py::test_paged_prefill"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-2000:]
