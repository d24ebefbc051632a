"""Pins for the fp64 attention oracle, each against something other than itself.

- brute force: a dense NumPy score matrix with a boolean support mask, built
  from the pages' statement of the problem (each query attends to the tokens of
  its own selected pages, causally), on tiny inputs and many seeds;
- TopK = every page reduces to dense causal attention (torch SDPA, float64);
- closed forms: one visible token gives that token's V; constant keys give the
  mean of the visible V; empty support gives zeros and lse = -inf;
- invariance of every output row to a permutation of the queries;
- storage decoders against torch's bfloat16 and float8_e4m3fn conversions.
"""
import numpy as np
import pytest
import torch

import oracle
from query_union_paged_b200 import workloads as W


# ----------------------------------------------------------------- decoders

def test_e4m3_decode_all_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 16, size=4000, dtype=np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_decode(int(b)) for b in bits])
    assert np.array_equal(ref, got)


# ------------------------------------------------------------- brute force

def _decode_np(arr, dtype, scale=None):
    """Independent decode of the stored bytes to float64 (numpy/torch routines)."""
    if dtype == W.DT_F32:
        return arr.astype(np.float64)
    if dtype == W.DT_BF16:
        return (arr.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    x = torch.from_numpy(np.ascontiguousarray(arr)).view(torch.float8_e4m3fn).double().numpy()
    return x * scale.astype(np.float64)[None, :, None, None]


def brute_force(w):
    """Dense [Nq, kv_len] scores with a boolean support mask, softmax, times V."""
    g = w.Hq // w.Hkv
    Q = _decode_np(w.Q, w.q_dtype)
    Kc = _decode_np(w.Kc, w.kv_dtype, w.k_scale)
    Vc = _decode_np(w.Vc, w.kv_dtype, w.v_scale)
    t = np.arange(w.kv_len)
    phys = w.page_table[t // w.T]
    Kl = Kc[phys, :, t % w.T, :]  # [kv_len][Hkv][d]
    Vl = Vc[phys, :, t % w.T, :]
    O = np.zeros((w.Nq, w.Hq, w.d))
    lse = np.full((w.Nq, w.Hq), -np.inf)
    for hq in range(w.Hq):
        h = hq // g
        allowed = np.zeros((w.Nq, w.kv_len), bool)
        for i in range(w.Nq):
            pages = set(int(p) for p in w.topk[hq, i] if p != -1)
            allowed[i] = np.isin(t // w.T, list(pages)) & (t <= w.q_pos[i])
        S = (Q[:, hq, :] @ Kl[:, h, :].T) * w.softmax_scale
        S = np.where(allowed, S, -np.inf)
        mx = S.max(axis=1, keepdims=True)
        has = np.isfinite(mx[:, 0])
        E = np.where(allowed, np.exp(S - np.where(has[:, None], mx, 0.0)), 0.0)
        l = E.sum(axis=1)
        O[has, hq, :] = (E[has] @ Vl[:, h, :]) / l[has, None]
        lse[has, hq] = mx[has, 0] + np.log(l[has])
    return O, lse


def _tiny(seed, Hq, Hkv, T, n_pages, Nq, K, q_dtype, kv_dtype, topk_all=False):
    rng = np.random.default_rng(1000 + seed)
    kv_len = n_pages * T
    d = 128
    page_table = rng.permutation(n_pages).astype(np.int32)
    q_pos = np.sort(rng.choice(kv_len, size=Nq, replace=False)).astype(np.int32)
    rng.shuffle(q_pos)  # query IDs need not be in position order
    if topk_all:
        topk = np.tile(np.arange(n_pages, dtype=np.int32), (Hq, Nq, 1))
    else:
        topk = rng.integers(-1, n_pages, size=(Hq, Nq, K)).astype(np.int32)
        topk[:, :, 0] = (q_pos // T)[None, :]  # own page present
        dup = rng.random((Hq, Nq, K)) < 0.15
        topk = np.where(dup, topk[:, :, :1], topk).astype(np.int32)
    Qf = rng.standard_normal((Nq, Hq, d), dtype=np.float32)
    Q = Qf if q_dtype == W.DT_F32 else W.f32_to_bf16_bits(Qf)
    Kc, ks = W._store_kv(rng, (n_pages, Hkv, T, d), kv_dtype)
    Vc, vs = W._store_kv(rng, (n_pages, Hkv, T, d), kv_dtype)
    return W.Workload(name="tiny", Hq=Hq, Hkv=Hkv, Nq=Nq, d=d, T=T, K=topk.shape[2],
                      num_logical_pages=n_pages, P_phys=n_pages, kv_len=kv_len,
                      q_dtype=q_dtype, kv_dtype=kv_dtype, Q=Q, Kc=Kc, Vc=Vc, k_scale=ks,
                      v_scale=vs, page_table=page_table, topk=topk, q_pos=q_pos)


CASES = [
    # seed, Hq, Hkv, T, pages, Nq, K, q_dtype, kv_dtype
    (0, 1, 1, 64, 8, 40, 4, W.DT_F32, W.DT_F32),
    (1, 2, 1, 32, 16, 30, 3, W.DT_BF16, W.DT_BF16),
    (2, 2, 2, 16, 32, 50, 4, W.DT_BF16, W.DT_E4M3),
    (3, 4, 2, 64, 8, 25, 2, W.DT_BF16, W.DT_BF16),
    (4, 2, 1, 128, 4, 33, 4, W.DT_F32, W.DT_E4M3),
    (5, 1, 1, 16, 24, 64, 1, W.DT_BF16, W.DT_BF16),
    (6, 2, 2, 32, 12, 45, 4, W.DT_F32, W.DT_BF16),
    (7, 4, 1, 64, 6, 20, 3, W.DT_BF16, W.DT_E4M3),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"seed{c[0]}")
def test_oracle_matches_dense_brute_force(case):
    w = _tiny(*case)
    O, lse = oracle.sparse_attn_workload(w, want_lse=True)
    Ob, lseb = brute_force(w)
    assert np.max(np.abs(O - Ob)) < 1e-12
    fin = np.isfinite(lseb)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.max(np.abs(lse[fin] - lseb[fin])) < 1e-12


def test_oracle_row_subset_equals_full():
    w = _tiny(*CASES[2])
    O = oracle.sparse_attn_workload(w)
    rng = np.random.default_rng(3)
    rows = rng.choice(w.Hq * w.Nq, size=17, replace=False).astype(np.int64)
    Os = oracle.sparse_attn_workload(w, rows=rows)
    for n, r in enumerate(rows):
        hq, i = divmod(int(r), w.Nq)
        assert np.array_equal(Os[n], O[i, hq])


@pytest.mark.parametrize("kv_dtype", [W.DT_F32, W.DT_BF16])
def test_topk_all_pages_is_dense_causal_attention(kv_dtype):
    """Selecting every page reduces to dense causal attention (torch SDPA, fp64)."""
    w = _tiny(11, 4, 2, 32, 10, 48, 0, W.DT_F32, kv_dtype, topk_all=True)
    O = oracle.sparse_attn_workload(w)
    g = w.Hq // w.Hkv
    Kc = _decode_np(w.Kc, w.kv_dtype)
    Vc = _decode_np(w.Vc, w.kv_dtype)
    t = np.arange(w.kv_len)
    Kl = torch.from_numpy(Kc[w.page_table[t // w.T], :, t % w.T, :])  # [L][Hkv][d]
    Vl = torch.from_numpy(Vc[w.page_table[t // w.T], :, t % w.T, :])
    q = torch.from_numpy(w.Q.astype(np.float64)).permute(1, 0, 2)  # [Hq][Nq][d]
    k = Kl.permute(1, 0, 2).repeat_interleave(g, dim=0)
    v = Vl.permute(1, 0, 2).repeat_interleave(g, dim=0)
    mask = torch.from_numpy(t[None, :] <= w.q_pos[:, None])  # causal with offset
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                           scale=w.softmax_scale)
    assert np.max(np.abs(O - ref.permute(1, 0, 2).numpy())) < 1e-12


def test_single_visible_token_returns_its_value():
    """Query at offset 0 of its page, only that page selected: O = V of that token."""
    w = _tiny(12, 2, 1, 64, 8, 8, 2, W.DT_BF16, W.DT_BF16)
    w.q_pos[:] = np.arange(8, dtype=np.int32) * 64  # offset 0 of page i
    w.topk[:] = -1
    w.topk[:, :, 0] = np.arange(8, dtype=np.int32)[None, :]
    w.topk[:, :, 1] = np.arange(8, dtype=np.int32)[None, :] + 1  # later pages: causally empty
    w.topk[w.topk >= 8] = -1
    O = oracle.sparse_attn_workload(w)
    Vc = _decode_np(w.Vc, w.kv_dtype)
    for i in range(8):
        assert np.array_equal(O[i, 0], Vc[w.page_table[i], 0, 0])
        assert np.array_equal(O[i, 1], Vc[w.page_table[i], 0, 0])


def test_constant_keys_average_visible_values():
    w = _tiny(13, 2, 2, 32, 6, 12, 3, W.DT_F32, W.DT_F32)
    w.Kc[:] = 0.25
    O = oracle.sparse_attn_workload(w)
    t = np.arange(w.kv_len)
    for hq in range(w.Hq):
        for i in range(w.Nq):
            pages = set(int(p) for p in w.topk[hq, i] if p >= 0)
            vis = t[np.isin(t // w.T, list(pages)) & (t <= w.q_pos[i])]
            vals = w.Vc[w.page_table[vis // w.T], hq, vis % w.T].astype(np.float64)
            assert np.max(np.abs(O[i, hq] - vals.mean(axis=0))) < 1e-12


def test_empty_support_gives_zero_and_neg_inf_lse():
    w = _tiny(14, 1, 1, 64, 4, 6, 2, W.DT_F32, W.DT_F32)
    w.topk[:] = -1
    w.topk[0, 0, 0] = 3
    w.q_pos[0] = 10  # page 3 lies after the query: causally empty
    O, lse = oracle.sparse_attn_workload(w, want_lse=True)
    assert np.all(O == 0) and np.all(np.isneginf(lse))


def test_out_of_range_page_id_is_an_error():
    w = _tiny(15, 1, 1, 64, 4, 6, 2, W.DT_F32, W.DT_F32)
    w.topk[0, 2, 1] = 4
    with pytest.raises(ValueError):
        oracle.sparse_attn_workload(w)


def test_query_permutation_invariance():
    w = _tiny(16, 4, 2, 32, 10, 40, 4, W.DT_BF16, W.DT_BF16)
    O = oracle.sparse_attn_workload(w)
    perm = np.random.default_rng(5).permutation(w.Nq)
    w.Q = w.Q[perm].copy()
    w.q_pos = w.q_pos[perm].copy()
    w.topk = w.topk[:, perm].copy()
    Op = oracle.sparse_attn_workload(w)
    assert np.array_equal(Op, O[perm])


def test_page_order_and_duplicates_do_not_matter():
    w = _tiny(17, 2, 1, 32, 10, 30, 4, W.DT_BF16, W.DT_BF16)
    O = oracle.sparse_attn_workload(w)
    rng = np.random.default_rng(9)
    topk2 = np.concatenate([w.topk, w.topk], axis=2)
    for hq in range(w.Hq):
        for i in range(w.Nq):
            rng.shuffle(topk2[hq, i])
    w.topk = topk2
    assert np.max(np.abs(oracle.sparse_attn_workload(w) - O)) < 1e-13
