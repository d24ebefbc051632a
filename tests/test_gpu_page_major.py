"""Direct KV-page union (qup_page_major_items + qup_page_major_attn through the C ABI): page-major
items with per-row partial results and their lse merge, against the fp64 oracle (the same per-query
supports as the query-union path), and the structure of the items."""
import numpy as np
import pytest

import oracle
import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

from helpers import check_close, out_to_f64, to_device, workload

pytestmark = pytest.mark.gpu


def _run(w, dev, want_lse=False):
    import torch
    items = qup.page_major_items(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, w.T)
    lse = torch.full((w.Nq, w.Hq), float("nan"), device="cuda") if want_lse else None
    O = qup.page_major_attn(dev["Q"], dev["K"], dev["V"], dev["page_table"], items, dev["q_pos"], w.kv_len,
                            k_scale=dev["k_scale"], v_scale=dev["v_scale"], lse=lse,
                            num_logical_pages=w.num_logical_pages)
    code = qup.get_error()
    assert code == 0, f"device error {code}"
    return out_to_f64(O), lse, items


SMALL = [
    dict(seed=50),
    dict(seed=51, T=128, prefix=900, kv_dtype=W.DT_E4M3),
    dict(seed=52, T=32, prefix=1000),
    dict(seed=53, Hq=8, Hkv=1, T=16, prefix=300, K=12),
    dict(seed=54, q_dtype=W.DT_F32, kv_dtype=W.DT_F32),
    dict(seed=55, Hq=2, Hkv=1, Nq=37, prefix=0, K=3),
]


@pytest.mark.parametrize("kw", SMALL, ids=lambda k: f"s{k['seed']}")
def test_small_full_output_and_lse(kw):
    w = W.random_small(**kw)
    ref, ref_lse = oracle.sparse_attn_workload(w, want_lse=True)
    got, lse, _ = _run(w, to_device(w), want_lse=True)
    check_close(got, ref, w.kv_dtype, f"page-major {w.name}", report=True)
    l = lse.cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(l), fin)
    assert np.max(np.abs(l[fin] - ref_lse[fin]), initial=0.0) < (3e-2 if w.kv_dtype == W.DT_E4M3 else 2e-3)


def test_nan_tail_and_empty_rows():
    w = W.random_small(56, Hq=4, Hkv=2, Nq=77, prefix=1000, T=64)
    last = w.page_table[w.num_logical_pages - 1]
    fill = w.kv_len % w.T
    w.Kc[last, :, fill:, :] = 0x7FC0
    w.Vc[last, :, fill:, :] = 0x7FC0
    w.topk[:, 3, :] = -1  # a query with no pages
    ref = oracle.sparse_attn_workload(w)
    got, _, _ = _run(w, to_device(w))
    check_close(got, ref, w.kv_dtype, "page-major nan tail", report=True)
    assert np.all(got[3] == 0)


def test_items_structure():
    """Every row has one partial slot per tile its own TopK row touches, slots are distinct, and an
    item's row masks are exactly the rows' selections of the tile's pages."""
    w = W.random_small(57, Hq=8, Hkv=2, Nq=150, prefix=700, T=64, K=10)
    _, _, it = _run(w, to_device(w))
    a = {k: v.cpu().numpy() for k, v in it.arrays.items()}
    g, Pt, MQ = w.Hq // w.Hkv, it.tile_pages, 128 // (w.Hq // w.Hkv)
    row_off, slots = a["row_off"], a["item_slot"]
    seen = np.zeros(int(row_off[-1]), np.int64)
    head0 = np.concatenate([[0], np.cumsum(a["n_items"])])
    for h in range(w.Hkv):
        for bi in range(int(a["n_items"][h])):
            fi = head0[h] + bi
            e0 = int(a["item_ptr"][h, bi])
            pages = a["item_pages"][e0:e0 + Pt]
            masks = a["item_mask"][e0:e0 + Pt].view(np.uint32)
            for m, qid in enumerate(a["item_qid"][h, bi]):
                for j in range(g):
                    r = m * g + j
                    row = set(int(x) for x in w.topk[h * g + j, qid]) - {-1} if qid >= 0 else set()
                    bits = [(int(masks[x, r // 32]) >> (r % 32)) & 1 for x in range(Pt)]
                    tile = int(pages[0]) // Pt  # entries past the last page repeat page 0, which no row selects
                    want = [int(int(pages[x]) in row and int(pages[x]) // Pt == tile) for x in range(Pt)]
                    assert bits == want, (h, bi, m, j)
                    s = int(slots[fi, r])
                    if any(bits):
                        seen[s] += 1
                        assert row_off[(h * g + j) * w.Nq + qid] <= s < row_off[(h * g + j) * w.Nq + qid + 1]
                    else:
                        assert s == -1
    assert np.all(seen == 1)
    for hq in range(w.Hq):
        for i in range(w.Nq):
            tiles = {int(x) // Pt for x in w.topk[hq, i] if x >= 0}
            assert row_off[hq * w.Nq + i + 1] - row_off[hq * w.Nq + i] == len(tiles)


@pytest.mark.parametrize("cfg", ["2", "4b"])
def test_full_size_every_element(cfg):
    w = workload(cfg)
    got, _, _ = _run(w, to_device(w))
    check_close(got, oracle.sparse_attn_workload(w), w.kv_dtype, f"page-major {w.name}", report=True)
