"""Error paths on the GPU: bad inputs set device error bits; a bounded pipeline wait
that runs out (host-side fault injection: one ring stage is never loaded)
returns QUP_ERR_TIMEOUT and leaves the context usable. Nothing here faults,
traps or hangs the GPU: every wait in the kernel has a time limit.
"""
import numpy as np
import pytest

import oracle
import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

from helpers import check_close, out_to_f64, to_device

pytestmark = pytest.mark.gpu


def _call(w, dev, gr, page_table=None):
    return qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"],
                                   dev["page_table"] if page_table is None else page_table, gr,
                                   dev["q_pos"], w.kv_len, k_scale=dev["k_scale"],
                                   v_scale=dev["v_scale"], num_logical_pages=w.num_logical_pages)


def test_bad_physical_page_sets_error_bit():
    w = W.random_small(21)
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    bad = dev["page_table"].clone()
    bad[3] = w.P_phys + 5
    _call(w, dev, gr, bad)
    assert qup.get_error() & qup.ERR["PHYS_PAGE"]


def test_bad_group_sets_error_bit():
    w = W.random_small(22)
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    gr.bundle_qid[0, 0, 0] = w.Nq + 3
    _call(w, dev, gr)
    assert qup.get_error() & qup.ERR["GROUP"]


def test_invalid_arguments_are_rejected_synchronously():
    w = W.random_small(23)
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    import torch
    with pytest.raises(qup.QupError):
        qup.sparse_prefill_attn(dev["Q"][:, :, :64].contiguous(), dev["K"][..., :64].contiguous(),
                                dev["V"][..., :64].contiguous(), dev["page_table"], gr, dev["q_pos"],
                                w.kv_len)
    with pytest.raises(qup.QupError):
        qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 9, 64)
    with pytest.raises(qup.QupError):
        qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 60)
    assert qup.get_error() == 0


def test_timeout_is_reported_and_context_stays_usable():
    w = W.random_small(24, Nq=120)
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    try:
        qup.set_debug(wait_limit_ms=50, skip_stage=2)
        _call(w, dev, gr)
        code = qup.get_error()
    finally:
        qup.set_debug(0, -1)
    assert code & qup.ERR["TIMEOUT"]
    got = out_to_f64(_call(w, dev, gr))
    assert qup.get_error() == 0
    check_close(got, oracle.sparse_attn_workload(w), w.kv_dtype, "after timeout")


def test_checked_mode_validates_row_masks_against_topk():
    """Checked mode: correct masks pass; a mask bit added, a bit removed, or a page dropped from a
    bundle union each raise the GROUP error bit (the attention call itself still runs)."""
    import torch
    w = W.random_small(24, Hq=8, Hkv=2, Nq=120)
    dev = to_device(w)
    qup.set_checked(True)
    try:
        gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
        out = qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"], dev["page_table"], gr, dev["q_pos"], w.kv_len,
                                      topk=dev["topk"], num_logical_pages=w.num_logical_pages)
        assert qup.get_error() == 0
        check_close(out_to_f64(out), oracle.sparse_attn_workload(w), w.kv_dtype, "checked mode")
        n0 = int(gr.bunion_ptr[0, 1] - gr.bunion_ptr[0, 0])
        assert n0 > 1
        e0 = int(gr.bunion_ptr[0, 0])
        masks = gr.bunion_mask[e0:e0 + n0].cpu().numpy().view(np.uint32).copy()
        word = masks[:, 0]
        live = np.bitwise_or.reduce(word)              # rows of word 0 that selected some page
        r = int(np.flatnonzero([(live >> b) & 1 for b in range(32)])[0])
        has = (word >> r) & 1
        assert has.any() and not has.all(), "row r must select some but not all union pages"
        for corrupt in ("add", "remove", "drop_all"):
            m = masks.copy()
            if corrupt == "add":        # row r gets a union page it did not select
                j = int(np.flatnonzero(has == 0)[0])
                m[j, 0] |= np.uint32(1 << r)
            elif corrupt == "remove":   # row r loses one page it selected
                j = int(np.flatnonzero(has == 1)[0])
                m[j, 0] &= np.uint32(~(1 << r) & 0xFFFFFFFF)
            else:                       # row r's pages all left the union
                m[:, 0] &= np.uint32(~(1 << r) & 0xFFFFFFFF)
            m = torch.from_numpy(m.view(np.int32)).cuda()
            gr.bunion_mask[e0:e0 + n0] = m
            _call(w, dev, gr)
            assert qup.get_error() == 0, "checked mode needs topk: without it nothing is checked"
            qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"], dev["page_table"], gr, dev["q_pos"], w.kv_len,
                                    topk=dev["topk"], num_logical_pages=w.num_logical_pages)
            assert qup.get_error() & qup.ERR["GROUP"], corrupt
            gr.bunion_mask[e0:e0 + n0] = torch.from_numpy(masks.view(np.int32)).cuda()
    finally:
        qup.set_checked(False)
