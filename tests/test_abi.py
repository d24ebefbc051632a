"""Host-side checks (no GPU): the C-ABI library loads and exports every symbol the
header declares; argument validation that needs no device answers correctly;
the workload generator is deterministic."""
import ctypes
import os
import re
import textwrap

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


def _run_without_devices(code: str):
    """Run `code` in a fresh interpreter that sees no CUDA device.  The argument checks below pass
    made-up non-null buffer addresses: with no device visible, a check that stopped answering
    first would end in QUP_ERR_CUDA, never in a kernel launch on those addresses."""
    import subprocess
    import sys
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    prog = f"import sys; sys.path.insert(0, {ROOT!r})\n" + textwrap.dedent(code)
    res = subprocess.run([sys.executable, "-c", prog], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr


_FAKE_GROUPS = """
    import ctypes
    import query_union_paged_b200 as qup
    qup.load()
    fake = [0x1000 + 0x100 * i for i in range(len(qup._GROUP_KEYS) + len(qup._BUNDLE_KEYS))]
    def groups(bw):
        return qup._Groups(*fake[:len(qup._GROUP_KEYS)], 1 << 20, *fake[len(qup._GROUP_KEYS):], 0, bw)
"""


def test_bundle_window_out_of_range_is_rejected_before_any_device_work(lib):
    _run_without_devices(_FAKE_GROUPS + """
    for bw in (300, -1):
        cs = groups(bw)
        rc = qup._lib.qup_sparse_group(ctypes.c_void_p(0x2000), 32, 8, 2048, 16, 288, 8, 64, ctypes.byref(cs),
                                       ctypes.c_void_p(0x3000), 1 << 30, None)
        assert rc == qup.ERR["ARG"], (bw, rc)
        rc = qup._lib.qup_build_bundles(ctypes.byref(cs), 32, 8, 2048, 288, 8, ctypes.c_void_p(0x3000), 1 << 30,
                                        None)
        assert rc == qup.ERR["ARG"], (bw, rc)
""")


def test_union_support_rejects_bad_arguments_before_any_device_work(lib):
    _run_without_devices(_FAKE_GROUPS + """
    cs = groups(0)
    # max_group 9, a missing workspace and an out-of-range bundle window are all refused on the host
    assert qup._lib.qup_union_support(ctypes.byref(cs), 32, 8, 2048, 288, 9, ctypes.c_void_p(0x3000), 1 << 30,
                                      None) == qup.ERR["ARG"]
    assert qup._lib.qup_union_support(ctypes.byref(cs), 32, 8, 2048, 288, 8, None, 0, None) == qup.ERR["CAPACITY"]
    cs.bundle_window = 512
    assert qup._lib.qup_union_support(ctypes.byref(cs), 32, 8, 2048, 288, 8, ctypes.c_void_p(0x3000), 1 << 30,
                                      None) == qup.ERR["ARG"]
""")


def test_checked_mode_argument_and_no_device_answer(lib):
    _run_without_devices(_FAKE_GROUPS + """
    assert qup._lib.qup_set_checked(1) == 0
    cs = groups(0)
    cs.rows_per_group = 32
    # Ksel < 0 with topk given is an argument error in checked mode, found before the device
    rc = qup._lib.qup_sparse_prefill_attn(ctypes.c_void_p(0x10000), 1, ctypes.c_void_p(0x20000),
                                          ctypes.c_void_p(0x30000), 1, None, None, ctypes.c_void_p(0x4000), 288,
                                          288, 64, ctypes.c_void_p(0x5000), -1, ctypes.byref(cs),
                                          ctypes.c_void_p(0x6000), 18432, 32, 8, 2048, 128, 0.088,
                                          ctypes.c_void_p(0x70000), None, None)
    assert rc == qup.ERR["ARG"], rc
    # valid arguments reach the device lookup, which answers that there is no device
    rc = qup._lib.qup_sparse_prefill_attn(ctypes.c_void_p(0x10000), 1, ctypes.c_void_p(0x20000),
                                          ctypes.c_void_p(0x30000), 1, None, None, ctypes.c_void_p(0x4000), 288,
                                          288, 64, ctypes.c_void_p(0x5000), 16, ctypes.byref(cs),
                                          ctypes.c_void_p(0x6000), 18432, 32, 8, 2048, 128, 0.088,
                                          ctypes.c_void_p(0x70000), None, None)
    assert rc == qup.ERR["CUDA"], rc
""")


def test_pivot_select_rejects_bad_arguments_before_any_device_work(lib):
    _run_without_devices("""
    import ctypes
    import query_union_paged_b200 as qup
    qup.load()
    f = qup._lib.qup_pivot_select
    q, k, pos, out = (ctypes.c_void_p(a) for a in (0x10000, 0x20000, 0x30000, 0x40000))
    good = dict(dtype=1, Nq=64, Hkv=2, g=4, d=128, P=100, T=64, G=16, C=32, K=8, refine=1)
    def call(**kw):
        a = dict(good, **kw)
        return f(q, k, a["dtype"], pos, a["Nq"], a["Hkv"], a["g"], a["d"], a["P"], a["T"], a["G"], a["C"],
                 a["K"], a["refine"], out, None)
    for bad in (dict(C=0), dict(C=257), dict(K=33), dict(K=0), dict(d=100), dict(d=1024), dict(P=9000),
                dict(G=0), dict(g=33), dict(dtype=2), dict(refine=2)):
        assert call(**bad) == qup.ERR["ARG"], bad
    # fp32 index vectors need a multiple of 4 only
    assert call(dtype=0, d=100) == qup.ERR["CUDA"]
    # valid arguments reach the device lookup, which answers that there is no device
    assert call() == qup.ERR["CUDA"]
""")
