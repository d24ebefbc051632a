"""fp64 CPU oracle for paged sparse-attention prefill with query unions.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may import this package. It shares no code with the
CUDA library in ``query_union_paged_b200``; the two meet only through the seeded
inputs of ``query_union_paged_b200.workloads``, which this package does not
import either (callers pass plain arrays).

The C source (``oracle.c``) states the definitions it follows: per-query sparse
attention over each query's own TopK pages with causal masking inside a page
(PageWeaver, Abstract and Figure 1), and the bounded page-affinity grouping rule
with its logical page visits and masked query-page slots (Figure 2).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16, E4M3 = 0, 1, 2
ERRORS = {0: "ok", 1: "bad argument", 2: "page id out of range", 3: "capacity", 4: "out of memory"}


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (OpenMP) into liboracle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_sparse_attn.argtypes = [P, I, P, P, I, P, P, P, I, I, I, P, I, P, I,
                                               I, I, I, I, D, P, I64, P, P, I]
            lib.oracle_sparse_attn.restype = I
            lib.oracle_group.argtypes = [P, I, I, I, I, I, I, I, P, P, P, P, P, P, I64, P]
            lib.oracle_group.restype = I
            lib.oracle_build_unions.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P, I64, P]
            lib.oracle_build_unions.restype = I
            lib.oracle_bundle.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P, I64, P]
            lib.oracle_bundle.restype = I
            lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_decode.restype = D
            lib.oracle_bf16_decode.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_decode.restype = D
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def e4m3_decode(code: int) -> float:
    return _load().oracle_e4m3_decode(code)


def bf16_decode(bits: int) -> float:
    return _load().oracle_bf16_decode(bits)


def sparse_attn(Q, q_dtype, Kc, Vc, kv_dtype, k_scale, v_scale, page_table, num_logical_pages,
                P_phys, T, topk, q_pos, kv_len, Hq, Hkv, Nq, d, softmax_scale,
                rows=None, nthreads=0, want_lse=False):
    """Per-query sparse attention in fp64.

    rows: None for every row (O is [Nq][Hq][d]) or an int64 array of h'*Nq + i
    (O is [len(rows)][d]). Returns O (and lse, natural log, if want_lse).
    """
    lib = _load()
    topk = _c(topk, np.int32)
    K = topk.shape[-1]
    Q = np.ascontiguousarray(Q)
    Kc = np.ascontiguousarray(Kc)
    Vc = np.ascontiguousarray(Vc)
    page_table = _c(page_table, np.int32)
    q_pos = _c(q_pos, np.int32)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    if rows is None:
        n = Hq * Nq
        O = np.zeros((Nq, Hq, d), np.float64)
        lse = np.zeros((Nq, Hq), np.float64) if want_lse else None
        rows_c = None
    else:
        rows_c = _c(rows, np.int64)
        n = rows_c.size
        O = np.zeros((n, d), np.float64)
        lse = np.zeros((n,), np.float64) if want_lse else None
    rc = lib.oracle_sparse_attn(_ptr(Q), q_dtype, _ptr(Kc), _ptr(Vc), kv_dtype, _ptr(ks), _ptr(vs),
                                _ptr(page_table), num_logical_pages, P_phys, T, _ptr(topk), K,
                                _ptr(q_pos), kv_len, Hq, Hkv, Nq, d, softmax_scale,
                                _ptr(rows_c), n, _ptr(O), _ptr(lse), nthreads)
    if rc:
        raise ValueError(f"oracle_sparse_attn: {ERRORS.get(rc, rc)}")
    return (O, lse) if want_lse else O


def sparse_attn_workload(w, rows=None, nthreads=0, want_lse=False):
    """sparse_attn on a Workload-like object (attributes as in the generator)."""
    return sparse_attn(w.Q, w.q_dtype, w.Kc, w.Vc, w.kv_dtype, w.k_scale, w.v_scale, w.page_table,
                       w.num_logical_pages, w.P_phys, w.T, w.topk, w.q_pos, w.kv_len, w.Hq, w.Hkv,
                       w.Nq, w.d, w.softmax_scale, rows=rows, nthreads=nthreads, want_lse=want_lse)


def union_capacity(Hq, Hkv, Nq, K, P):
    g = Hq // Hkv
    return max(1, Hkv * Nq * min(g * K, P))


def _alloc_groups(Hkv, Nq, cap):
    return dict(n_groups=np.zeros(Hkv, np.int32),
                group_ptr=np.zeros((Hkv, Nq + 1), np.int32),
                members=np.zeros((Hkv, Nq), np.int32),
                union_ptr=np.zeros((Hkv, Nq + 1), np.int32),
                union_pages=np.zeros(cap, np.int32),
                row_mask=np.zeros(cap, np.uint64),
                counters=np.zeros((Hkv, 4), np.int64))


def _trim(out):
    Hkv = out["n_groups"].size
    total = int(out["union_ptr"][Hkv - 1, out["n_groups"][Hkv - 1]]) if Hkv else 0
    out["union_pages"] = out["union_pages"][:total].copy()
    out["row_mask"] = out["row_mask"][:total].copy()
    return out


def group(topk, Hq, Hkv, Nq, num_logical_pages, max_group=8, window=64):
    """The bounded page-affinity grouping rule; returns a dict of arrays.

    counters[h] = (logical page visits, masked row slots, masked query slots, page edges).
    """
    lib = _load()
    topk = _c(topk, np.int32)
    K = topk.shape[-1]
    cap = union_capacity(Hq, Hkv, Nq, K, num_logical_pages)
    out = _alloc_groups(Hkv, Nq, cap)
    rc = lib.oracle_group(_ptr(topk), Hq, Hkv, Nq, K, num_logical_pages, max_group, window,
                          *(_ptr(out[k]) for k in ("n_groups", "group_ptr", "members", "union_ptr",
                                                   "union_pages", "row_mask")),
                          cap, _ptr(out["counters"]))
    if rc:
        raise ValueError(f"oracle_group: {ERRORS.get(rc, rc)}")
    return _trim(out)


def build_unions(topk, Hq, Hkv, Nq, num_logical_pages, partition):
    """Unions, row masks and counters for a given partition.

    partition: list over KV heads of lists of groups (each an ascending list of query IDs).
    """
    lib = _load()
    topk = _c(topk, np.int32)
    K = topk.shape[-1]
    cap = union_capacity(Hq, Hkv, Nq, K, num_logical_pages)
    out = _alloc_groups(Hkv, Nq, cap)
    for h, groups in enumerate(partition):
        out["n_groups"][h] = len(groups)
        pos = 0
        for gi, mem in enumerate(groups):
            out["group_ptr"][h, gi] = pos
            out["members"][h, pos:pos + len(mem)] = mem
            pos += len(mem)
        out["group_ptr"][h, len(groups)] = pos
    rc = lib.oracle_build_unions(_ptr(topk), Hq, Hkv, Nq, K, num_logical_pages,
                                 *(_ptr(out[k]) for k in ("n_groups", "group_ptr", "members",
                                                          "union_ptr", "union_pages", "row_mask")),
                                 cap, _ptr(out["counters"]))
    if rc:
        raise ValueError(f"oracle_build_unions: {ERRORS.get(rc, rc)}")
    return _trim(out)


def bundle(groups, Hq, Hkv, Nq, max_group=8, bundle_window=64):
    """Bundles of the groups (dict as returned by group/build_unions); adds bundle keys."""
    lib = _load()
    g = Hq // Hkv
    cap = max(1, int(groups["union_pages"].size))
    out = dict(n_bundles=np.zeros(Hkv, np.int32), bundle_ptr=np.zeros((Hkv, Nq + 1), np.int32),
               bundle_groups=np.zeros((Hkv, Nq), np.int32), bunion_ptr=np.zeros((Hkv, Nq + 1), np.int32),
               bunion_pages=np.zeros(cap, np.int32), bunion_mask=np.zeros((cap, 4), np.uint32),
               bundle_qid=np.full((Hkv, Nq, 128 // g), -1, np.int32), bcounters=np.zeros((Hkv, 2), np.int64))
    gr = {k: np.ascontiguousarray(groups[k]) for k in ("n_groups", "group_ptr", "members", "union_ptr",
                                                      "union_pages", "row_mask")}
    if gr["union_pages"].size == 0:
        gr["union_pages"] = np.zeros(1, np.int32)
        gr["row_mask"] = np.zeros(1, np.uint64)
    rc = lib.oracle_bundle(Hq, Hkv, Nq, max_group, bundle_window,
                           *(_ptr(gr[k]) for k in ("n_groups", "group_ptr", "members", "union_ptr",
                                                   "union_pages", "row_mask")),
                           *(_ptr(out[k]) for k in ("n_bundles", "bundle_ptr", "bundle_groups", "bunion_ptr",
                                                    "bunion_pages", "bunion_mask", "bundle_qid")),
                           cap, _ptr(out["bcounters"]))
    if rc:
        raise ValueError(f"oracle_bundle: {ERRORS.get(rc, rc)}")
    total = int(out["bunion_ptr"][Hkv - 1, out["n_bundles"][Hkv - 1]]) if Hkv else 0
    out["bunion_pages"] = out["bunion_pages"][:total].copy()
    out["bunion_mask"] = out["bunion_mask"][:total].copy()
    res = dict(groups)
    res.update(out)
    return res
