"""qup_sparse_group_static (grouping with its scratch in the library's own fixed
device array) vs qup_sparse_group (caller workspace): identical groups and
bundles, over two calls in a row with different problems, called through the
C ABI; the second call of each problem changes neither torch's allocated bytes
nor the device's free memory.  Runs alone or after every other test file.
"""
import ctypes

import numpy as np
import pytest

import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

from helpers import assert_bundles_equal, assert_groups_equal, groups_to_host

pytestmark = pytest.mark.gpu

STATIC_LIMIT = 16 << 20  # QUP_STATIC_GROUP_SCRATCH_BYTES


def _lib():
    lib = qup.load()
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.qup_sparse_group_static.argtypes = [P, I, I, I, I, I, I, I, ctypes.POINTER(qup._Groups), P]
    lib.qup_sparse_group_static.restype = I
    return lib


def _static_group_into(out, topk, Hq, Hkv, P, max_group, window):
    Hq_, Nq, K = topk.shape
    cs = out.c_struct()
    rc = _lib().qup_sparse_group_static(ctypes.c_void_p(topk.data_ptr()), Hq, Hkv, Nq, K, P, max_group,
                                        window, ctypes.byref(cs), None)
    assert rc == 0, qup.QupError(rc, "qup_sparse_group_static")
    out._after(cs)
    return out


def _problems():
    rng = np.random.default_rng(77)
    small = rng.integers(-1, 300, size=(8, 500, 11)).astype(np.int32)
    w = W.make("2")
    return [(small, 8, 2, 300, 8, 64), (w.topk, w.Hq, w.Hkv, w.num_logical_pages, 8, 64),
            (small, 8, 2, 300, 4, 8)]


def test_static_scratch_matches_workspace_entry_point_two_calls_in_a_row():
    import torch
    for topk_np, Hq, Hkv, P, mg, win in _problems():
        topk = torch.from_numpy(np.ascontiguousarray(topk_np)).cuda()
        ws_bytes, _ = qup.group_workspace(Hq, Hkv, topk.shape[1], topk.shape[2], P, mg, win)
        assert ws_bytes <= STATIC_LIMIT
        ref = groups_to_host(qup.sparse_group(topk, Hq, Hkv, P, mg, win))
        for call in range(2):
            Hq_, Nq, K = topk.shape
            _, cap = qup.group_workspace(Hq, Hkv, Nq, K, P, mg, win)
            out = qup.alloc_groups(Hq, Hkv, Nq, cap, 0, topk.device)  # outputs only, no workspace
            torch.cuda.synchronize()
            before = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
            _static_group_into(out, topk, Hq, Hkv, P, mg, win)
            torch.cuda.synchronize()
            after = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
            if call == 1:  # the first call may still load the library's module; the second allocates nothing
                assert after == before, (before, after)
            got = groups_to_host(out)
            assert qup.get_error() == 0
            assert_groups_equal(got, ref)
            assert_bundles_equal(got, ref)


def test_static_scratch_rejects_oversize_problem():
    import torch
    Hq, Hkv, Nq, K, P = 32, 8, 8192, 4, 544
    ws_bytes, _ = qup.group_workspace(Hq, Hkv, Nq, K, P, 8, 64)
    assert ws_bytes > STATIC_LIMIT
    topk = torch.zeros((Hq, Nq, K), dtype=torch.int32, device="cuda")
    out = qup.alloc_groups(Hq, Hkv, Nq, 1, 0, topk.device)
    cs = out.c_struct()
    rc = _lib().qup_sparse_group_static(ctypes.c_void_p(topk.data_ptr()), Hq, Hkv, Nq, K, P, 8, 64,
                                        ctypes.byref(cs), None)
    assert rc == qup.ERR["CAPACITY"]
    assert qup.get_error() == 0
