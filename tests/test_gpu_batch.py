"""Batched requests (qup_batch_prepare + qup_sparse_group + qup_sparse_prefill_attn_batch through
the C ABI): several sequences, each with its own page table, cache length, positions and TopK rows,
in one grouping call and one attention call, against the fp64 oracle run on each request alone."""
import numpy as np
import pytest

import oracle
import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

from helpers import check_close, out_to_f64

pytestmark = pytest.mark.gpu


def _batch(ws):
    """Concatenate seeded single-sequence workloads into one batch: queries end to end, physical
    caches end to end (each request's page table rebased to its pages), page tables end to end."""
    q_ptr, page_ptr, phys_base = [0], [0], [0]
    for w in ws:
        q_ptr.append(q_ptr[-1] + w.Nq)
        page_ptr.append(page_ptr[-1] + w.num_logical_pages)
        phys_base.append(phys_base[-1] + w.P_phys)
    cat = lambda k, ax=0: np.ascontiguousarray(np.concatenate([getattr(w, k) for w in ws], axis=ax))
    kmax = max(w.K for w in ws)  # TopK rows padded with -1 to one width
    topk = np.concatenate([np.pad(w.topk, ((0, 0), (0, 0), (0, kmax - w.K)), constant_values=-1) for w in ws],
                          axis=1)
    page_table = np.concatenate([w.page_table + b for w, b in zip(ws, phys_base)]).astype(np.int32)
    ks = vs = None
    if ws[0].kv_dtype == W.DT_E4M3:  # one scale per KV head for the whole cache
        for w in ws[1:]:
            w.k_scale, w.v_scale = ws[0].k_scale, ws[0].v_scale
        ks, vs = ws[0].k_scale, ws[0].v_scale
    return dict(Q=cat("Q"), K=cat("Kc"), V=cat("Vc"), topk=np.ascontiguousarray(topk), q_pos=cat("q_pos"),
                page_table=page_table, q_ptr=np.array(q_ptr, np.int32), page_ptr=np.array(page_ptr, np.int32),
                kv_len=np.array([w.kv_len for w in ws], np.int32), k_scale=ks, v_scale=vs)


def _run(ws, max_group=8, window=64):
    import torch
    w0 = ws[0]
    b = _batch(ws)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    view = (lambda x: x.view(torch.bfloat16)) if w0.kv_dtype == W.DT_BF16 else (lambda x: x)
    Q = t(b["Q"]).view(torch.bfloat16) if w0.q_dtype == W.DT_BF16 else t(b["Q"])
    Kc, Vc = view(t(b["K"])), view(t(b["V"]))
    total_pages = int(b["page_ptr"][-1])
    bt = qup.batch_prepare(t(b["topk"]), t(b["q_pos"]), t(b["q_ptr"]), t(b["page_ptr"]), t(b["kv_len"]),
                           total_pages, w0.T)
    gr = qup.sparse_group(bt.topk_global, w0.Hq, w0.Hkv, total_pages, max_group, window)
    qup.set_checked(True)
    try:
        O = qup.sparse_prefill_attn_batch(Q, Kc, Vc, t(b["page_table"]), gr, bt,
                                          k_scale=None if b["k_scale"] is None else t(b["k_scale"]),
                                          v_scale=None if b["v_scale"] is None else t(b["v_scale"]),
                                          checked_topk=True)
    finally:
        qup.set_checked(False)
    assert qup.get_error() == 0
    return out_to_f64(O), b


def _expected(ws):
    return np.concatenate([oracle.sparse_attn_workload(w) for w in ws], axis=0)


def _with_nan_tail(w):
    """Non-finite bytes past kv_len in the request's last (partly filled) page."""
    fill = w.kv_len % w.T
    if fill:
        last = w.page_table[w.num_logical_pages - 1]
        bad = 0x7FC0 if w.kv_dtype == W.DT_BF16 else 0x7F
        w.Kc[last, :, fill:, :] = bad
        w.Vc[last, :, fill:, :] = bad
    return w


def test_batch_bf16_ragged_requests():
    ws = [_with_nan_tail(W.random_small(70, Nq=100, prefix=960, T=64)),
          _with_nan_tail(W.random_small(71, Nq=37, prefix=200, T=64)),
          _with_nan_tail(W.random_small(72, Nq=150, prefix=1500, T=64, K=9))]
    got, _ = _run(ws)
    check_close(got, _expected(ws), W.DT_BF16, "batch bf16", report=True)


def test_batch_e4m3_ragged_requests():
    ws = [_with_nan_tail(W.random_small(73, Nq=90, prefix=900, T=128, kv_dtype=W.DT_E4M3, Hq=8, Hkv=2)),
          _with_nan_tail(W.random_small(74, Nq=200, prefix=2000, T=128, kv_dtype=W.DT_E4M3, Hq=8, Hkv=2)),
          _with_nan_tail(W.random_small(75, Nq=17, prefix=100, T=128, kv_dtype=W.DT_E4M3, Hq=8, Hkv=2))]
    got, _ = _run(ws, window=128)
    check_close(got, _expected(ws), W.DT_E4M3, "batch e4m3", report=True)


def test_batch_of_one_equals_single_sequence_call():
    import torch
    w = W.random_small(76, Nq=120, prefix=700, T=32)
    got, _ = _run([w])
    from helpers import to_device
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    O = qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"], dev["page_table"], gr, dev["q_pos"], w.kv_len,
                                num_logical_pages=w.num_logical_pages)
    assert qup.get_error() == 0
    assert np.array_equal(got, out_to_f64(O))


def test_batch_local_page_id_out_of_range_is_reported():
    import torch
    ws = [W.random_small(77, Nq=40, prefix=300, T=64), W.random_small(78, Nq=30, prefix=500, T=64)]
    b = _batch(ws)
    b["topk"][0, 5, 1] = ws[0].num_logical_pages  # a page of the next request, not of this one
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    qup.batch_prepare(t(b["topk"]), t(b["q_pos"]), t(b["q_ptr"]), t(b["page_ptr"]), t(b["kv_len"]),
                      int(b["page_ptr"][-1]), ws[0].T)
    assert qup.get_error() & qup.ERR["PAGE_ID"]
