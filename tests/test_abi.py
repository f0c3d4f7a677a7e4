"""The C ABI library: it loads, exports every entry point include/g2attn.h
declares, and rejects bad arguments on the host before any launch (these
checks run without a GPU: no compute call is made)."""
import ctypes
import os
import re
import subprocess

import pytest

import global_soft_capped_b200 as g2
from global_soft_capped_b200 import build as g2build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "g2attn.h")


@pytest.fixture(scope="module")
def lib():
    g2build.build()
    return g2.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"G2ATTN_API\s+[\w\s\*]*?\b(g2attn_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_symbols() == sorted(g2.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {g2.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (g2attn_\w+)", out))
    assert exported == set(declared_symbols())


def test_status_strings(lib):
    names = {g2.g2attn_status_string(i) for i in range(8)}
    assert len(names) == 8
    assert g2.g2attn_status_string(99) == "unknown status"


def test_workspace_size_is_host_only_and_monotone(lib):
    a = g2.g2attn_decode_workspace_size(64, 32, 128, 8192)
    b = g2.g2attn_decode_workspace_size(64, 32, 128, 16384)
    assert 0 < a < b
    assert g2.g2attn_decode_workspace_size(0, 32, 128, 8192) == 0


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: calls fail before launch


def prefill_args(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=None, B=1, T=64, S=64, H=8, Hkv=4, d=256,
             q_offset=0, query_scale=0.0625, softcap=50.0, window=0, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(B=0), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(T=0), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(q_offset=-1), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(q_offset=1), g2.G2ATTN_ERR_INVALID_ARG),          # q_offset + T > S
    (dict(window=-1), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(softcap=-1.0), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(softcap=float("inf")), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(query_scale=float("nan")), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(H=6), g2.G2ATTN_ERR_UNSUPPORTED),                 # H != 2*Hkv
    (dict(d=96), g2.G2ATTN_ERR_UNSUPPORTED),
    (dict(k=ctypes.c_void_p((1 << 20) + 8)), g2.G2ATTN_ERR_MISALIGNED),
])
def test_prefill_rejects_before_launch(lib, kw, status):
    assert g2.g2attn_prefill(*prefill_args(**kw)) == status


def test_varlen_and_decode_reject_before_launch(lib):
    cu = ctypes.c_void_p(1 << 21)
    base = [FAKE, FAKE, FAKE, FAKE, None, cu, cu, 2, 128, 128, 64, 64, 8, 4, 128, 0.1, 50.0, 0,
            None]
    assert g2.g2attn_prefill_varlen(*base[:5], None, *base[6:]) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(base)
    bad[10] = 100  # max_T > max_S
    assert g2.g2attn_prefill_varlen(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(base)
    bad[7] = 5000  # more sequences than the per-launch table holds
    assert g2.g2attn_prefill_varlen(*bad) == g2.G2ATTN_ERR_UNSUPPORTED

    dec = [FAKE, FAKE, FAKE, cu, FAKE, None, 4, 4096, 1024, 32, 16, 128, 0.083, 50.0, 4096,
           FAKE, 16, None]
    assert g2.g2attn_decode(*dec) == g2.G2ATTN_ERR_WORKSPACE          # 16 bytes is too small
    bad = list(dec)
    bad[15] = None
    assert g2.g2attn_decode(*bad) == g2.G2ATTN_ERR_WORKSPACE
    bad = list(dec)
    bad[11] = 80
    assert g2.g2attn_decode(*bad) == g2.G2ATTN_ERR_UNSUPPORTED
    bad = list(dec)
    bad[6] = 0
    assert g2.g2attn_decode(*bad) == g2.G2ATTN_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(g2, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(g2, "_lib", None)
    with pytest.raises(RuntimeError, match="libg2attn.so is missing"):
        g2.load_library()


def test_ring_and_paged_reject_before_launch(lib):
    cu = ctypes.c_void_p(1 << 21)
    ring = [FAKE, FAKE, FAKE, cu, FAKE, None, 4, 4096, 4096, 32, 16, 128, 0.083, 50.0, 4096,
            FAKE, 1 << 30, None]
    bad = list(ring); bad[7] = 3000          # ring size not a power of two
    assert g2.g2attn_decode_ring(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(ring); bad[14] = 0            # a ring serves local layers only
    assert g2.g2attn_decode_ring(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(ring); bad[14] = 8192         # window larger than the ring
    assert g2.g2attn_decode_ring(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(ring); bad[3] = None
    assert g2.g2attn_decode_ring(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    paged = [FAKE, FAKE, FAKE, cu, cu, FAKE, None, 4, 100, 48, 10, 4096, 32, 16, 128, 0.083,
             50.0, 0, FAKE, 1 << 30, None]
    bad = list(paged); bad[9] = 48           # block size not a power of two
    assert g2.g2attn_decode_paged(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    paged[9] = 64
    bad = list(paged); bad[3] = None         # no block table
    assert g2.g2attn_decode_paged(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(paged); bad[18] = None        # no workspace
    assert g2.g2attn_decode_paged(*bad) == g2.G2ATTN_ERR_WORKSPACE


def test_paged_prefill_rejects_before_launch(lib):
    cu = ctypes.c_void_p(1 << 21)
    base = [FAKE, FAKE, FAKE, FAKE, None, cu, cu, cu, 2, 256, 16, 256, 8, 128, 2048, 8, 4, 256,
            0.0625, 50.0, 0, None]
    bad = list(base); bad[11] = 64           # blocks smaller than a 128-key tile
    assert g2.g2attn_prefill_paged(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(base); bad[11] = 384          # not a power of two
    assert g2.g2attn_prefill_paged(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(base); bad[12] = 4            # table cannot hold max_S keys
    assert g2.g2attn_prefill_paged(*bad) == g2.G2ATTN_ERR_INVALID_ARG
    bad = list(base); bad[6] = None          # no block table
    assert g2.g2attn_prefill_paged(*bad) == g2.G2ATTN_ERR_INVALID_ARG


SCHED_BYTES = 256  # the gradient kernels' unit counters, after the per-row vectors


def test_backward_workspace_size(lib):
    a = g2.g2attn_backward_workspace_size(1, 8192, 32)
    assert a == 2 * 1 * 32 * 8192 * 4 + SCHED_BYTES
    assert g2.g2attn_backward_workspace_size(2, 65, 4) == 2 * 2 * 4 * 128 * 4 + SCHED_BYTES
    assert g2.g2attn_backward_workspace_size(0, 64, 4) == 0


def backward_args(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
             B=1, T=64, S=64, H=8, Hkv=4, d=128, q_offset=0, query_scale=0.0625, softcap=50.0,
             window=0, workspace=FAKE, workspace_bytes=1 << 20, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,status", [
    (dict(lse=None), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(dout=None), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(dk=None), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(q_offset=1), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(softcap=-1.0), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(d=96), g2.G2ATTN_ERR_UNSUPPORTED),
    (dict(H=6), g2.G2ATTN_ERR_UNSUPPORTED),
    (dict(workspace=None), g2.G2ATTN_ERR_WORKSPACE),
    (dict(workspace_bytes=1024), g2.G2ATTN_ERR_WORKSPACE),
    (dict(workspace=ctypes.c_void_p((1 << 20) + 4)), g2.G2ATTN_ERR_MISALIGNED),
    (dict(dq=ctypes.c_void_p((1 << 20) + 8)), g2.G2ATTN_ERR_MISALIGNED),
])
def test_backward_rejects_before_launch(lib, kw, status):
    assert g2.g2attn_prefill_backward(*backward_args(**kw)) == status


def test_varlen_backward_workspace_size(lib):
    wmax = (100 + 64 * 3 + 63) // 64 * 64      # every sequence padded to whole tiles
    head = 2 * 8 * wmax * 4 + 4 * 4                # -lse2, -D, then the prefix wq[4]
    head = (head + SCHED_BYTES - 1) // SCHED_BYTES * SCHED_BYTES
    assert g2.g2attn_varlen_backward_workspace_size(3, 100, 8) == head + SCHED_BYTES
    assert g2.g2attn_varlen_backward_workspace_size(0, 100, 8) == 0
    assert g2.g2attn_varlen_backward_workspace_size(3, 0, 8) == 0


def varlen_backward_args(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
             cu_q=FAKE, cu_k=FAKE, num_seqs=2, total_q=128, total_k=256, max_T=64, max_S=128,
             H=8, Hkv=4, d=128, query_scale=0.0625, softcap=50.0, window=0, workspace=FAKE,
             workspace_bytes=1 << 20, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,status", [
    (dict(cu_q=None), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(cu_k=None), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(lse=None), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(num_seqs=0), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(max_T=129), g2.G2ATTN_ERR_INVALID_ARG),             # above max_S
    (dict(max_S=257), g2.G2ATTN_ERR_INVALID_ARG),             # above total_k
    (dict(window=-2), g2.G2ATTN_ERR_INVALID_ARG),
    (dict(d=32), g2.G2ATTN_ERR_UNSUPPORTED),
    (dict(Hkv=3), g2.G2ATTN_ERR_UNSUPPORTED),
    (dict(num_seqs=1025), g2.G2ATTN_ERR_UNSUPPORTED),         # the kernels' sequence table
    (dict(workspace_bytes=64), g2.G2ATTN_ERR_WORKSPACE),
    (dict(workspace=ctypes.c_void_p((1 << 20) + 4)), g2.G2ATTN_ERR_MISALIGNED),
    (dict(cu_k=ctypes.c_void_p((1 << 20) + 2)), g2.G2ATTN_ERR_MISALIGNED),
])
def test_varlen_backward_rejects_before_launch(lib, kw, status):
    assert g2.g2attn_prefill_varlen_backward(*varlen_backward_args(**kw)) == status


def test_header_is_plain_c_and_links(lib, tmp_path):
    """include/g2attn.h compiles as C99 (no C++ in the interface), and a C
    program that calls every declared entry point links against the library
    (the program is built, not run)."""
    names = declared_symbols()
    calls = "\n".join(f"    (void)&{n};" for n in names)
    src = tmp_path / "use.c"
    src.write_text('#include "g2attn.h"\nint main(void) {\n' + calls + "\n    return 0;\n}\n")
    lib_dir = os.path.dirname(g2.LIB_PATH)
    res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                          str(src), "-L", lib_dir, "-lg2attn", "-o", str(tmp_path / "use")],
                         capture_output=True, text=True)
    if res.returncode != 0 and "cannot find -lg2attn" in res.stderr:
        # the library is named libg2attn.so in-tree; link by path instead
        res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I",
                              os.path.join(ROOT, "include"), str(src), g2.LIB_PATH,
                              "-o", str(tmp_path / "use")], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_binding_argument_counts_match_header(lib):
    """Every ctypes prototype has as many arguments as the header declares
    (a miscounted marshalling list would shift every later argument)."""
    text = open(HEADER).read()
    decls = re.findall(r"G2ATTN_API\s+[\w\s\*]*?\b(g2attn_\w+)\s*\(([^)]*)\)\s*;", text)
    assert sorted(n for n, _ in decls) == sorted(g2.EXPORTS)
    for name, params in decls:
        params = " ".join(params.split())
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(getattr(lib, name).argtypes) == n, name
