"""Host-side checks (no GPU): the C-ABI library loads and exports every symbol the
header declares; argument validation that needs no device answers correctly;
the workload generator is deterministic."""
import ctypes
import os
import re

import numpy as np
import pytest

import query_union_paged_b200 as qup
from query_union_paged_b200 import build, workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^\s*(?:int|const char\*|void)\s+(qup_\w+)\s*\(", src, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ctypes.CDLL(build.LIB)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"qup_sparse_group", "qup_sparse_prefill_attn", "qup_group_workspace",
            "qup_get_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_workspace_sizes_and_limits(lib):
    ws, cap = qup.group_workspace(32, 8, 2048, 16, 288, 8, 64)
    assert cap == 8 * 2048 * min(4 * 16, 288)
    assert ws >= 32 * 2048 * 9 * 4
    with pytest.raises(qup.QupError):
        qup.group_workspace(32, 8, 2048, 16, 288, 9, 64)      # max_group > 8
    with pytest.raises(qup.QupError):
        qup.group_workspace(32, 8, 2048, 16, 288, 8, 60)      # window % max_group
    with pytest.raises(qup.QupError):
        qup.group_workspace(64, 4, 2048, 16, 288, 4, 64)      # 4 * 16 rows > 32
    with pytest.raises(qup.QupError):
        qup.group_workspace(32, 8, 2048, 16, 10 ** 6, 8, 64)  # bitsets exceed shared memory


def test_error_strings(lib):
    lib.qup_error_string.restype = ctypes.c_char_p
    assert lib.qup_error_string(64) == b"pipeline wait timed out"
    assert lib.qup_error_string(0) == b"ok"


def test_generator_is_deterministic():
    a, b = W.random_small(3), W.random_small(3)
    for k in ("Q", "Kc", "Vc", "topk", "page_table", "q_pos"):
        assert np.array_equal(getattr(a, k), getattr(b, k))
    w = W.gqa_chunk_bf16()
    assert w.topk.shape == (32, 2048, 16) and w.kv_len == 16384 + 2048
    assert np.all(w.topk[0] == w.topk[3]) and not np.all(w.topk[0] == w.topk[4])


def test_bundle_window_out_of_range_is_rejected_before_any_device_work(lib):
    # every buffer pointer is non-null but fake: the argument checks run before the device is touched
    fake = [ctypes.c_void_p(0x1000 + 0x100 * i).value for i in range(len(qup._GROUP_KEYS) + len(qup._BUNDLE_KEYS))]
    for bw, want in ((300, qup.ERR["ARG"]), (-1, qup.ERR["ARG"])):
        cs = qup._Groups(*fake[:len(qup._GROUP_KEYS)], 1 << 20, *fake[len(qup._GROUP_KEYS):], 0, bw)
        qup.load()
        rc = qup._lib.qup_sparse_group(ctypes.c_void_p(0x2000), 32, 8, 2048, 16, 288, 8, 64, ctypes.byref(cs),
                                       ctypes.c_void_p(0x3000), 1 << 30, None)
        assert rc == want, (bw, rc)
        rc = qup._lib.qup_build_bundles(ctypes.byref(cs), 32, 8, 2048, 288, 8, ctypes.c_void_p(0x3000), 1 << 30, None)
        assert rc == want, (bw, rc)


def test_union_support_rejects_bad_arguments_before_any_device_work(lib):
    fake = [ctypes.c_void_p(0x1000 + 0x100 * i).value for i in range(len(qup._GROUP_KEYS) + len(qup._BUNDLE_KEYS))]
    cs = qup._Groups(*fake[:len(qup._GROUP_KEYS)], 1 << 20, *fake[len(qup._GROUP_KEYS):], 0, 0)
    qup.load()
    # max_group 9, a missing workspace and an out-of-range bundle window are all refused on the host
    assert qup._lib.qup_union_support(ctypes.byref(cs), 32, 8, 2048, 288, 9, ctypes.c_void_p(0x3000), 1 << 30,
                                      None) == qup.ERR["ARG"]
    assert qup._lib.qup_union_support(ctypes.byref(cs), 32, 8, 2048, 288, 8, None, 0, None) == qup.ERR["CAPACITY"]
    cs.bundle_window = 512
    assert qup._lib.qup_union_support(ctypes.byref(cs), 32, 8, 2048, 288, 8, ctypes.c_void_p(0x3000), 1 << 30,
                                      None) == qup.ERR["ARG"]
