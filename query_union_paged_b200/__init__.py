"""B200 (sm_100a) paged sparse-attention prefill with page-affine query unions.

Thin Python binding over the C ABI in ``include/query_union_paged.h`` (library
``libqup.so`` built in-tree). Every step of the path runs in the library's
CUDA kernels; this module only marshals arguments. PyTorch is used for device
memory and streams. There is no CPU fallback: if the library is missing the
calls raise.

    groups = sparse_group(topk, Hq, Hkv, num_logical_pages, max_group=8, window=64)
    O = sparse_prefill_attn(Q, K_cache, V_cache, page_table, groups, q_pos, kv_len, ...)
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

import numpy as np

__all__ = ["Groups", "sparse_group", "sparse_prefill_attn", "build_bundles", "groups_from_host", "union_support",
           "Batch", "batch_prepare", "sparse_prefill_attn_batch", "PageItems", "page_major_items", "page_major_attn",
           "get_error", "set_debug", "set_checked", "load",
           "QupError", "F32", "BF16", "E4M3", "ERR"]

F32, BF16, E4M3 = 0, 1, 2
ERR = {"ARG": 1, "CAPACITY": 2, "CUDA": 4, "PAGE_ID": 8, "PHYS_PAGE": 16, "GROUP": 32, "TIMEOUT": 64}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqup.so")
_lib = None


class QupError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_strerror(code)} (code {code})")


_GROUP_KEYS = ("n_groups", "group_ptr", "members", "union_ptr", "union_pages", "row_mask", "counters")
_BUNDLE_KEYS = ("n_bundles", "bundle_ptr", "bundle_groups", "bunion_ptr", "bunion_pages", "bunion_mask",
                "bundle_qid", "bcounters", "bundle_order")


class _Groups(ctypes.Structure):
    _fields_ = ([(k, ctypes.c_void_p) for k in _GROUP_KEYS] + [("cap_union", ctypes.c_int64)] +
                [(k, ctypes.c_void_p) for k in _BUNDLE_KEYS] +
                [("rows_per_group", ctypes.c_int32), ("bundle_window", ctypes.c_int32)])


def load():
    """Load libqup.so (in-tree). Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python -m query_union_paged_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.qup_group_workspace.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(SZ), ctypes.POINTER(I64)]
    lib.qup_sparse_group.argtypes = [P, I, I, I, I, I, I, I, ctypes.POINTER(_Groups), P, SZ, P]
    lib.qup_build_bundles.argtypes = [ctypes.POINTER(_Groups), I, I, I, I, I, P, SZ, P]
    lib.qup_sparse_prefill_attn.argtypes = [P, I, P, P, I, P, P, P, I, I, I, P, I,
                                            ctypes.POINTER(_Groups), P, I, I, I, I, I,
                                            ctypes.c_float, P, P, P]
    lib.qup_get_error.argtypes = [ctypes.POINTER(I), P]
    lib.qup_error_string.argtypes = [I]
    lib.qup_error_string.restype = ctypes.c_char_p
    lib.qup_set_debug.argtypes = [I, I]
    lib.qup_num_sms.argtypes = []
    lib.qup_exp2_poly.argtypes = [P, P, I, P]
    lib.qup_union_support.argtypes = [ctypes.POINTER(_Groups), I, I, I, I, I, P, SZ, P]
    lib.qup_set_checked.argtypes = [I]
    lib.qup_batch_prepare.argtypes = [P, P, I, I, I, I, I, P, P, P, I, P, P, P, P]
    lib.qup_page_major_workspace.argtypes = [I, I, I, I, I, I, ctypes.POINTER(SZ), ctypes.POINTER(I64),
                                             ctypes.POINTER(I64), ctypes.POINTER(ctypes.c_int32)]
    lib.qup_page_major_items.argtypes = [P, I, I, I, I, I, I, ctypes.POINTER(_PageItems), P, SZ, P]
    lib.qup_page_major_attn.argtypes = [P, I, P, P, I, P, P, P, I, I, I, ctypes.POINTER(_PageItems), P, I, I, I, I,
                                        I, ctypes.c_float, P, P, P, P, P]
    lib.qup_pivot_select.argtypes = [P, P, I, P, I, I, I, I, I, I, I, I, I, I, P, P]
    lib.qup_sparse_prefill_attn_batch.argtypes = [P, I, P, P, I, P, P, P, I, I, I, P, I,
                                                  ctypes.POINTER(_Groups), P, P, I, I, I, I,
                                                  ctypes.c_float, P, P, P]
    for fn in ("qup_group_workspace", "qup_sparse_group", "qup_build_bundles", "qup_sparse_prefill_attn",
               "qup_get_error", "qup_set_debug", "qup_num_sms", "qup_exp2_poly", "qup_union_support",
               "qup_set_checked", "qup_batch_prepare", "qup_sparse_prefill_attn_batch", "qup_page_major_workspace",
               "qup_page_major_items", "qup_page_major_attn", "qup_pivot_select"):
        getattr(lib, fn).restype = I
    _lib = lib
    return lib


def _strerror(code: int) -> str:
    try:
        return load().qup_error_string(code).decode()
    except Exception:
        return str(code)


def _check(rc: int, where: str):
    if rc != 0:
        raise QupError(rc, where)


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@dataclasses.dataclass
class Groups:
    """Device output of sparse_group (see qup_groups in the C header): the groups and the
    bundles the attention kernel walks."""
    n_groups: "torch.Tensor"
    group_ptr: "torch.Tensor"
    members: "torch.Tensor"
    union_ptr: "torch.Tensor"
    union_pages: "torch.Tensor"
    row_mask: "torch.Tensor"
    counters: "torch.Tensor"
    n_bundles: "torch.Tensor" = None
    bundle_ptr: "torch.Tensor" = None
    bundle_groups: "torch.Tensor" = None
    bunion_ptr: "torch.Tensor" = None
    bunion_pages: "torch.Tensor" = None
    bunion_mask: "torch.Tensor" = None
    bundle_qid: "torch.Tensor" = None
    bcounters: "torch.Tensor" = None
    bundle_order: "torch.Tensor" = None
    workspace: Optional["torch.Tensor"] = None
    rows_per_group: int = 0
    bundle_window: int = 0

    def c_struct(self) -> _Groups:
        cs = _Groups(*[getattr(self, k).data_ptr() for k in _GROUP_KEYS], self.union_pages.numel(),
                     *[getattr(self, k).data_ptr() for k in _BUNDLE_KEYS], self.rows_per_group,
                     self.bundle_window)
        return cs

    def _after(self, cs: _Groups):
        self.rows_per_group = cs.rows_per_group


def group_workspace(Hq, Hkv, Nq, Ksel, num_logical_pages, max_group=8, window=64):
    lib = load()
    ws = ctypes.c_size_t(0)
    cap = ctypes.c_int64(0)
    _check(lib.qup_group_workspace(Hq, Hkv, Nq, Ksel, num_logical_pages, max_group, window,
                                   ctypes.byref(ws), ctypes.byref(cap)), "qup_group_workspace")
    return ws.value, cap.value


def alloc_groups(Hq, Hkv, Nq, cap, ws_bytes, device) -> Groups:
    import torch
    i32 = dict(dtype=torch.int32, device=device)
    g = Hq // Hkv
    cap = max(int(cap), 1)
    return Groups(n_groups=torch.empty(Hkv, **i32), group_ptr=torch.empty(Hkv, Nq + 1, **i32),
                  members=torch.empty(Hkv, Nq, **i32), union_ptr=torch.empty(Hkv, Nq + 1, **i32),
                  union_pages=torch.empty(cap, **i32),
                  row_mask=torch.empty(cap, dtype=torch.int64, device=device),
                  counters=torch.empty(Hkv, 4, dtype=torch.int64, device=device),
                  n_bundles=torch.empty(Hkv, **i32), bundle_ptr=torch.empty(Hkv, Nq + 1, **i32),
                  bundle_groups=torch.empty(Hkv, Nq, **i32), bunion_ptr=torch.empty(Hkv, Nq + 1, **i32),
                  bunion_pages=torch.empty(cap, **i32), bunion_mask=torch.empty(cap, 4, **i32),
                  bundle_qid=torch.empty(Hkv, max(Nq, 1), 128 // g, **i32),
                  bcounters=torch.empty(Hkv, 2, dtype=torch.int64, device=device),
                  bundle_order=torch.empty(max(Hkv * Nq, 1), **i32),
                  workspace=torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device))


def groups_from_host(d: dict, Hq: int, Hkv: int, num_logical_pages: int, max_group: int = 8,
                     device="cuda", stream=None) -> Groups:
    """Upload a partition held as numpy arrays (keys as the C struct: n_groups .. counters)
    and build its bundles on the device (qup_build_bundles)."""
    import torch
    Hkv_, Np1 = d["group_ptr"].shape
    Nq = Np1 - 1
    ws_bytes, cap = group_workspace(Hq, Hkv, Nq, 1, num_logical_pages, max_group, max_group)
    cap = max(cap, int(d["union_pages"].size), 1)
    gr = alloc_groups(Hq, Hkv, Nq, cap, ws_bytes, device)
    for k in _GROUP_KEYS:
        src = d[k].view("int64") if k == "row_mask" else d[k]
        dst = getattr(gr, k)
        if k in ("union_pages", "row_mask"):
            dst[:src.size].copy_(torch.from_numpy(np.ascontiguousarray(src)))
        else:
            dst.copy_(torch.from_numpy(np.ascontiguousarray(src)))
    build_bundles(gr, Hq, Hkv, Nq, num_logical_pages, max_group, stream=stream)
    return gr


def build_bundles(gr: Groups, Hq: int, Hkv: int, Nq: int, num_logical_pages: int, max_group: int = 8,
                  stream=None) -> Groups:
    lib = load()
    cs = gr.c_struct()
    _check(lib.qup_build_bundles(ctypes.byref(cs), Hq, Hkv, Nq, num_logical_pages, max_group,
                                 _p(gr.workspace), gr.workspace.numel(), _stream_ptr(stream)),
           "qup_build_bundles")
    gr._after(cs)
    return gr


def union_support(gr: Groups, Hq: int, Hkv: int, Nq: int, num_logical_pages: int, max_group: int = 8,
                  stream=None) -> Groups:
    """Every row of a group sees every page of its group's union (qup_union_support); the
    bundles are rebuilt.  Attention on the result uses the group unions as supports."""
    lib = load()
    cs = gr.c_struct()
    _check(lib.qup_union_support(ctypes.byref(cs), Hq, Hkv, Nq, num_logical_pages, max_group,
                                 _p(gr.workspace), gr.workspace.numel(), _stream_ptr(stream)),
           "qup_union_support")
    gr._after(cs)
    return gr


def sparse_group(topk, Hq: int, Hkv: int, num_logical_pages: int, max_group: int = 8,
                 window: int = 64, out: Optional[Groups] = None, stream=None,
                 bundle_window: Optional[int] = None) -> Groups:
    """Page-affinity grouping of the queries of every KV head, then bundling (qup_sparse_group).

    topk: int32 CUDA tensor [Hq][Nq][Ksel], -1 = padding. Returns Groups on the device.
    bundle_window: groups per bundling window (None keeps out's setting; 0 = library default).
    """
    lib = load()
    Hq_, Nq, Ksel = topk.shape
    assert Hq_ == Hq and topk.is_cuda and topk.is_contiguous()
    ws_bytes, cap = group_workspace(Hq, Hkv, Nq, Ksel, num_logical_pages, max_group, window)
    if out is None:
        out = alloc_groups(Hq, Hkv, Nq, cap, ws_bytes, topk.device)
    if bundle_window is not None:
        out.bundle_window = int(bundle_window)
    cs = out.c_struct()
    _check(lib.qup_sparse_group(_p(topk), Hq, Hkv, Nq, Ksel, num_logical_pages, max_group, window,
                                ctypes.byref(cs), _p(out.workspace), out.workspace.numel(),
                                _stream_ptr(stream)), "qup_sparse_group")
    out._after(cs)
    return out


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return E4M3
    raise ValueError(f"unsupported dtype {t.dtype}")


def sparse_prefill_attn(Q, K_cache, V_cache, page_table, groups: Groups, q_pos, kv_len: int,
                        k_scale=None, v_scale=None, topk=None, softmax_scale: Optional[float] = None,
                        out=None, lse=None, num_logical_pages: Optional[int] = None, stream=None):
    """Union attention over the groups (qup_sparse_prefill_attn).

    Q [Nq][Hq][d] bf16/fp32; K_cache, V_cache [P_phys][Hkv][T][d] bf16/fp32/E4M3 (uint8 or
    float8_e4m3fn, with fp32 k_scale/v_scale [Hkv]); page_table int32 [pages]; q_pos int32 [Nq].
    Returns O [Nq][Hq][d] in Q's dtype (and fills lse [Nq][Hq] fp32 if given).
    """
    import torch
    lib = load()
    Nq, Hq, d = Q.shape
    P_phys, Hkv, T, d2 = K_cache.shape
    assert d2 == d and V_cache.shape == K_cache.shape
    for t in (Q, K_cache, V_cache, page_table, q_pos):
        assert t.is_cuda and t.is_contiguous()
    if out is None:
        out = torch.empty_like(Q)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if num_logical_pages is None:
        num_logical_pages = page_table.numel()
    cs = groups.c_struct()
    ksel = topk.shape[-1] if topk is not None else 0
    _check(lib.qup_sparse_prefill_attn(_p(Q), _dtype_code(Q), _p(K_cache), _p(V_cache),
                                       _dtype_code(K_cache), _p(k_scale), _p(v_scale), _p(page_table),
                                       num_logical_pages, P_phys, T, _p(topk), ksel, ctypes.byref(cs),
                                       _p(q_pos), kv_len, Hq, Hkv, Nq, d, float(softmax_scale),
                                       _p(out), _p(lse), _stream_ptr(stream)),
           "qup_sparse_prefill_attn")
    return out


class _PageItems(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in ("n_items", "item_ptr", "item_pages", "item_mask", "item_qid",
                                               "item_slot", "item_order", "row_off")] + \
               [("item_cap", ctypes.c_int64), ("slot_cap", ctypes.c_int64), ("tile_pages", ctypes.c_int32)]


@dataclasses.dataclass
class PageItems:
    """Device arrays of page-major items (see qup_page_items) and the partial-result buffers."""
    arrays: dict
    item_cap: int
    slot_cap: int
    tile_pages: int
    workspace: "torch.Tensor"
    part_o: "torch.Tensor"
    part_lse: "torch.Tensor"

    def c_struct(self) -> _PageItems:
        a = self.arrays
        return _PageItems(*[a[k].data_ptr() for k in ("n_items", "item_ptr", "item_pages", "item_mask", "item_qid",
                                                      "item_slot", "item_order", "row_off")],
                          self.item_cap, self.slot_cap, self.tile_pages)


def page_major_items(topk, Hq: int, Hkv: int, num_logical_pages: int, T: int, out: Optional[PageItems] = None,
                     stream=None) -> PageItems:
    """Page-major items of the TopK rows (qup_page_major_items): tiles of 256 tokens and the
    queries that meet them, with per-row partial slots."""
    import torch
    lib = load()
    Hq_, Nq, Ksel = topk.shape
    ws, icap, scap, tp = ctypes.c_size_t(0), ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int32(0)
    _check(lib.qup_page_major_workspace(Hq, Hkv, Nq, Ksel, num_logical_pages, T, ctypes.byref(ws), ctypes.byref(icap),
                                        ctypes.byref(scap), ctypes.byref(tp)), "qup_page_major_workspace")
    if out is None:
        dev = topk.device
        i32 = dict(dtype=torch.int32, device=dev)
        g = Hq // Hkv
        n = Hkv * icap.value
        arrays = dict(n_items=torch.empty(Hkv, **i32), item_ptr=torch.empty(Hkv, icap.value + 1, **i32),
                      item_pages=torch.empty(n * tp.value, **i32), item_mask=torch.empty(n * tp.value, 4, **i32),
                      item_qid=torch.empty(Hkv, icap.value, 128 // g, **i32), item_slot=torch.empty(n, 128, **i32),
                      item_order=torch.empty(n, **i32),
                      row_off=torch.empty(Hq * Nq + 1, dtype=torch.int64, device=dev))
        out = PageItems(arrays=arrays, item_cap=icap.value, slot_cap=scap.value, tile_pages=tp.value,
                        workspace=torch.empty(max(ws.value, 1), dtype=torch.uint8, device=dev),
                        part_o=torch.empty(scap.value, 128, dtype=torch.float32, device=dev),
                        part_lse=torch.empty(scap.value, dtype=torch.float32, device=dev))
    cs = out.c_struct()
    _check(lib.qup_page_major_items(_p(topk), Hq, Hkv, Nq, Ksel, num_logical_pages, T, ctypes.byref(cs),
                                    _p(out.workspace), out.workspace.numel(), _stream_ptr(stream)),
           "qup_page_major_items")
    out.tile_pages = cs.tile_pages
    return out


def page_major_attn(Q, K_cache, V_cache, page_table, items: PageItems, q_pos, kv_len: int, k_scale=None,
                    v_scale=None, softmax_scale: Optional[float] = None, out=None, lse=None,
                    num_logical_pages: Optional[int] = None, stream=None):
    """Page-major attention over the items (qup_page_major_attn): partial results per row and
    tile, then their merge.  Returns O [Nq][Hq][d] in Q's dtype."""
    import torch
    lib = load()
    Nq, Hq, d = Q.shape
    P_phys, Hkv, T, d2 = K_cache.shape
    if out is None:
        out = torch.empty_like(Q)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if num_logical_pages is None:
        num_logical_pages = page_table.numel()
    cs = items.c_struct()
    _check(lib.qup_page_major_attn(_p(Q), _dtype_code(Q), _p(K_cache), _p(V_cache), _dtype_code(K_cache),
                                   _p(k_scale), _p(v_scale), _p(page_table), num_logical_pages, P_phys, T,
                                   ctypes.byref(cs), _p(q_pos), kv_len, Hq, Hkv, Nq, d, float(softmax_scale),
                                   _p(items.part_o), _p(items.part_lse), _p(out), _p(lse), _stream_ptr(stream)),
           "qup_page_major_attn")
    return out


@dataclasses.dataclass
class Batch:
    """Device arrays of batched requests after batch_prepare (see qup_batch_prepare)."""
    q_ptr: "torch.Tensor"
    page_ptr: "torch.Tensor"
    kv_len: "torch.Tensor"
    topk_global: "torch.Tensor"
    q_end: "torch.Tensor"
    page_len: "torch.Tensor"
    total_pages: int


def batch_prepare(topk, q_pos, q_ptr, page_ptr, kv_len, total_pages: int, T: int, stream=None) -> Batch:
    """Rebase request-local TopK rows and positions to the concatenated page space of a batch
    (qup_batch_prepare).  topk int32 [Hq][Nq][Ksel], q_pos int32 [Nq]; q_ptr, page_ptr int32 [R+1];
    kv_len int32 [R]; all CUDA tensors."""
    import torch
    Hq, Nq, Ksel = topk.shape
    R = q_ptr.numel() - 1
    dev = topk.device
    b = Batch(q_ptr=q_ptr, page_ptr=page_ptr, kv_len=kv_len,
              topk_global=torch.empty_like(topk), q_end=torch.empty(Nq, dtype=torch.int32, device=dev),
              page_len=torch.empty(max(total_pages, 1), dtype=torch.int32, device=dev), total_pages=total_pages)
    _check(load().qup_batch_prepare(_p(topk), _p(q_pos), Hq, Nq, Ksel, T, R, _p(q_ptr), _p(page_ptr), _p(kv_len),
                                    total_pages, _p(b.topk_global), _p(b.q_end), _p(b.page_len),
                                    _stream_ptr(stream)), "qup_batch_prepare")
    return b


def pivot_select(q_idx, page_key, q_pos, g: int, T: int, group_size: int, n_cand: int, K: int,
                 refine: bool = True, out=None, stream=None):
    """Proxy-query page selection (qup_pivot_select): TopK page IDs per (query head, query) for
    sparse_group.  q_idx [Nq][Hkv][d_idx] and page_key [P][Hkv][d_idx] bf16 or fp32 CUDA tensors,
    q_pos int32 [Nq]; returns int32 [Hkv*g][Nq][K] (-1 padded)."""
    import torch
    Nq, Hkv, d = q_idx.shape
    P = page_key.shape[0]
    assert page_key.shape[1:] == (Hkv, d) and page_key.dtype == q_idx.dtype
    if out is None:
        out = torch.empty((Hkv * g, Nq, K), dtype=torch.int32, device=q_idx.device)
    _check(load().qup_pivot_select(_p(q_idx), _p(page_key), _dtype_code(q_idx), _p(q_pos), Nq, Hkv, g, d, P, T,
                                   group_size, n_cand, K, 1 if refine else 0, _p(out), _stream_ptr(stream)),
           "qup_pivot_select")
    return out


def sparse_prefill_attn_batch(Q, K_cache, V_cache, page_table, groups: Groups, batch: Batch, k_scale=None,
                              v_scale=None, softmax_scale: Optional[float] = None, out=None, lse=None,
                              checked_topk: bool = False, stream=None):
    """Union attention over batched requests (qup_sparse_prefill_attn_batch): page_table is the
    concatenated table of batch.total_pages entries; groups come from sparse_group on
    batch.topk_global."""
    import torch
    lib = load()
    Nq, Hq, d = Q.shape
    P_phys, Hkv, T, d2 = K_cache.shape
    assert d2 == d and V_cache.shape == K_cache.shape
    if out is None:
        out = torch.empty_like(Q)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    cs = groups.c_struct()
    tk = batch.topk_global if checked_topk else None
    _check(lib.qup_sparse_prefill_attn_batch(_p(Q), _dtype_code(Q), _p(K_cache), _p(V_cache), _dtype_code(K_cache),
                                             _p(k_scale), _p(v_scale), _p(page_table), batch.total_pages, P_phys, T,
                                             _p(tk), tk.shape[-1] if tk is not None else 0, ctypes.byref(cs),
                                             _p(batch.q_end), _p(batch.page_len), Hq, Hkv, Nq, d,
                                             float(softmax_scale), _p(out), _p(lse), _stream_ptr(stream)),
           "qup_sparse_prefill_attn_batch")
    return out


def exp2_poly(x, out=None, stream=None):
    """2^x by the attention softmax's polynomial exponential (test hook, qup_exp2_poly).
    x: float32 CUDA tensor; returns a tensor of the same shape."""
    import torch
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    if out is None:
        out = torch.empty_like(x)
    _check(load().qup_exp2_poly(_p(x), _p(out), x.numel(), _stream_ptr(stream)), "qup_exp2_poly")
    return out


def get_error(stream=None) -> int:
    """Synchronize the stream, then read and clear the device error word."""
    lib = load()
    code = ctypes.c_int(0)
    _check(lib.qup_get_error(ctypes.byref(code), _stream_ptr(stream)), "qup_get_error")
    return code.value


def set_debug(wait_limit_ms: int = 0, skip_stage: int = -1):
    _check(load().qup_set_debug(wait_limit_ms, skip_stage), "qup_set_debug")


def set_checked(on: bool):
    """Checked mode (qup_set_checked): attention calls given topk first verify every bundle row's
    page mask against its TopK row and raise the GROUP error bit on a mismatch."""
    _check(load().qup_set_checked(1 if on else 0), "qup_set_checked")


def num_sms() -> int:
    return load().qup_num_sms()
