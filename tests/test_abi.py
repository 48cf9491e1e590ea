"""The C ABI without a GPU: the library loads, exports what include/*.h
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import glob
import os
import re

import pytest

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b([A-Za-z_][A-Za-z0-9_]*)\s*\(", src):
            name = m.group(1)
            if name.startswith(("topk_", "score_")):
                names.add(name)
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return atk.load_library()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert {"topk_bucketed", "topk_exact", "score_topk", "topk_workspace_bytes",
            "topk_status_string"} <= names
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(5):
        assert atk.topk_status_string(s).startswith("TOPK_")
    assert "unknown" in atk.topk_status_string(99)


def test_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    E = atk.TOPK_EINVAL
    # null pointers
    assert lib.topk_bucketed(None, 1, 8, 1, 1, 1, p, p, None, 0, None) == E
    assert lib.topk_bucketed(p, 1, 8, 1, 1, 1, None, p, None, 0, None) == E
    assert lib.topk_exact(p, 1, 8, 1, None, p, None, 0, None) == E
    assert lib.score_topk(None, 1, 128, p, 8, 0, 1, 1, 1, p, p, None, None, 0, None) == E
    # sizes
    assert lib.topk_bucketed(p, 0, 8, 1, 1, 1, p, p, None, 0, None) == E
    assert lib.topk_bucketed(p, 1, 0, 1, 1, 1, p, p, None, 0, None) == E
    assert lib.topk_bucketed(p, 1, 8, 0, 1, 1, p, p, None, 0, None) == E
    assert lib.topk_bucketed(p, 1, 8, 1, 0, 1, p, p, None, 0, None) == E
    assert lib.topk_bucketed(p, 1, 8, 1, 1, 0, p, p, None, 0, None) == E
    assert lib.topk_bucketed(p, 1, 8, 1, 1, 5, p, p, None, 0, None) == E
    assert lib.topk_bucketed(p, 1, 2 ** 31, 1, 1, 1, p, p, None, 0, None) == E
    # beyond this build
    U = atk.TOPK_EUNSUPPORTED
    assert lib.topk_bucketed(p, 1, 8, 1, 2048, 1, p, p, None, 0, None) == U
    assert lib.topk_bucketed(p, 1, 8, 20000, 4, 1, p, p, None, 0, None) == U
    assert lib.score_topk(p, 1, 64, p, 8, 0, 1, 1, 1, p, p, None, None, 0, None) == U
    assert lib.score_topk(p, 1, 128, p, 8, 0, 1, 3, 1, p, p, None, None, 0, None) == U
    # misaligned bf16 pointers
    q = ctypes.c_void_p(18)
    assert lib.score_topk(q, 1, 128, p, 8, 0, 1, 1, 1, p, p, None, None, 0, None) == E


def test_merge_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    E, U = atk.TOPK_EINVAL, atk.TOPK_EUNSUPPORTED
    offs = (ctypes.c_int64 * 2)(0, 100)
    ok = dict(parts=2, rows=1, m=8, n=200, k=4, b=8, kb=1)

    def call(vals=p, idx=p, offsets=offs, out=p, **kw):
        a = dict(ok, **kw)
        return lib.topk_bucketed_merge(vals, idx, a["parts"], a["rows"], a["m"], offsets, a["n"],
                                       a["k"], a["b"], a["kb"], out, p, None)

    assert call(vals=None) == E
    assert call(idx=None) == E
    assert call(out=None) == E
    assert call(parts=0) == E
    assert call(m=0) == E
    assert call(rows=0) == E
    assert call(kb=5) == E
    assert call(n=0) == E
    assert call(offsets=(ctypes.c_int64 * 2)(0, 200)) == E   # offset beyond the row
    assert call(offsets=(ctypes.c_int64 * 2)(-1, 0)) == E
    assert call(parts=65, offsets=None) == U
    assert call(b=2048) == U
    assert call(k=20000) == U


def test_sampling_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    E = atk.TOPK_EINVAL
    assert lib.topk_sample_rows(None, p, 1, 4, 1.0, p, p, None) == E
    assert lib.topk_sample_rows(p, p, 1, 4, 1.0, None, p, None) == E
    assert lib.topk_sample_rows(p, p, 1, 4, 1.0, p, None, None) == E
    assert lib.topk_sample_rows(p, p, 0, 4, 1.0, p, p, None) == E
    assert lib.topk_sample_rows(p, p, 1, 0, 1.0, p, p, None) == E
    for t in (0.0, -1.0, float("inf"), float("nan"), 1e-45):
        assert lib.topk_sample_rows(p, p, 1, 4, t, p, p, None) == E, t
        assert lib.topk_sample(p, 1, 8, 4, 2, 1, t, p, p, p, p, None, 0, None) == E, t
    assert lib.topk_sample(p, 1, 8, 4, 2, 1, 1.0, None, p, p, p, None, 0, None) == E
    assert lib.topk_sample(None, 1, 8, 4, 2, 1, 1.0, p, p, p, p, None, 0, None) == E
    assert lib.topk_sample_bf16(p, 1, 8, 4, 2, 1, 0.0, p, p, p, p, None, 0, None) == E
    assert lib.topk_sample_bf16(p, 1, 8, 4, 2, 1, 1.0, None, p, p, p, None, 0, None) == E
    assert lib.topk_sample_bf16(None, 1, 8, 4, 2, 1, 1.0, p, p, p, p, None, 0, None) == E


def test_selftest_rejects_bad_limits_on_host(lib):
    E = atk.TOPK_EINVAL
    assert lib.topk_selftest_wait_timeout(0, None) == E
    assert lib.topk_selftest_wait_timeout(999, None) == E
    assert lib.topk_selftest_wait_timeout(3 * 10 ** 9, None) == E


def test_binding_refuses_cpu_tensors(lib):
    import torch

    with pytest.raises(TypeError):
        atk.topk_bucketed(torch.zeros(2, 8), 1, 1, 1)
    with pytest.raises(TypeError):
        atk.topk_exact(torch.zeros(2, 8), 1)
    with pytest.raises(TypeError):
        atk.topk_bucketed_merge(torch.zeros(2, 1, 8), torch.zeros(2, 1, 8, dtype=torch.int32), 16, 4, 8, 1)
