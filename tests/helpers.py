"""Shared test utilities: move a seeded workload to the GPU and compare results."""
import dataclasses
import functools

import numpy as np

from query_union_paged_b200 import workloads as W


@functools.lru_cache(maxsize=None)
def workload(cfg: str):
    """The named full-size workload, generated once per test session (callers must not modify it)."""
    return W.make(cfg)


def permute_queries(w, perm, q_pos=None, name_suffix="perm"):
    """The same problem with query IDs renumbered: new query i is old query perm[i] (its Q row, its
    TopK rows and its position move with it).  q_pos, if given, replaces the permuted positions."""
    perm = np.asarray(perm)
    pos = w.q_pos[perm] if q_pos is None else np.asarray(q_pos, np.int32)
    return dataclasses.replace(w, name=f"{w.name}_{name_suffix}", Q=np.ascontiguousarray(w.Q[perm]),
                               topk=np.ascontiguousarray(w.topk[:, perm]),
                               q_pos=np.ascontiguousarray(pos, dtype=np.int32))


def to_device(w, device="cuda"):
    import torch
    d = {}
    Q = torch.from_numpy(np.ascontiguousarray(w.Q)).to(device)
    d["Q"] = Q.view(torch.bfloat16) if w.q_dtype == W.DT_BF16 else Q
    for name, arr in (("K", w.Kc), ("V", w.Vc)):
        t = torch.from_numpy(np.ascontiguousarray(arr)).to(device)
        if w.kv_dtype == W.DT_BF16:
            t = t.view(torch.bfloat16)
        d[name] = t
    d["k_scale"] = None if w.k_scale is None else torch.from_numpy(w.k_scale).to(device)
    d["v_scale"] = None if w.v_scale is None else torch.from_numpy(w.v_scale).to(device)
    d["page_table"] = torch.from_numpy(w.page_table).to(device)
    d["topk"] = torch.from_numpy(w.topk).to(device)
    d["q_pos"] = torch.from_numpy(w.q_pos).to(device)
    return d


def groups_to_host(gr):
    """Device Groups -> dict of numpy arrays trimmed to the used union entries."""
    n_groups = gr.n_groups.cpu().numpy()
    union_ptr = gr.union_ptr.cpu().numpy()
    Hkv = n_groups.size
    total = int(union_ptr[Hkv - 1, n_groups[Hkv - 1]]) if Hkv else 0
    d = dict(n_groups=n_groups, group_ptr=gr.group_ptr.cpu().numpy(),
             members=gr.members.cpu().numpy(), union_ptr=union_ptr,
             union_pages=gr.union_pages[:total].cpu().numpy(),
             row_mask=gr.row_mask[:total].cpu().numpy().view(np.uint64),
             counters=gr.counters.cpu().numpy())
    nb = gr.n_bundles.cpu().numpy()
    bptr = gr.bunion_ptr.cpu().numpy()
    btotal = int(bptr[Hkv - 1, nb[Hkv - 1]]) if Hkv else 0
    d.update(n_bundles=nb, bundle_ptr=gr.bundle_ptr.cpu().numpy(),
             bundle_groups=gr.bundle_groups.cpu().numpy(), bunion_ptr=bptr,
             bunion_pages=gr.bunion_pages[:btotal].cpu().numpy(),
             bunion_mask=gr.bunion_mask[:btotal].cpu().numpy().view(np.uint32),
             bundle_qid=gr.bundle_qid.cpu().numpy(), bcounters=gr.bcounters.cpu().numpy())
    if gr.bundle_order is not None:
        d["bundle_order"] = gr.bundle_order[:int(nb.sum())].cpu().numpy()
    return d


def expected_bundle_order(d):
    """Flat bundle indices sorted by union size, largest first, equal sizes by index (sizes above
    4095 count as 4095), from the bundle CSR of `d`."""
    sizes = []
    for h in range(d["n_bundles"].size):
        p = d["bunion_ptr"][h, :int(d["n_bundles"][h]) + 1].astype(np.int64)
        sizes.append(np.diff(p))
    sizes = np.concatenate(sizes) if sizes else np.zeros(0, np.int64)
    key = np.minimum(sizes, 4095)
    return np.argsort(-key, kind="stable").astype(np.int32)


def assert_groups_equal(got, ref):
    Hkv = ref["n_groups"].size
    assert np.array_equal(got["n_groups"], ref["n_groups"])
    assert np.array_equal(got["counters"], ref["counters"])
    for h in range(Hkv):
        n = int(ref["n_groups"][h])
        assert np.array_equal(got["group_ptr"][h, :n + 1], ref["group_ptr"][h, :n + 1])
        m = int(ref["group_ptr"][h, n])
        assert np.array_equal(got["members"][h, :m], ref["members"][h, :m])
        assert np.array_equal(got["union_ptr"][h, :n + 1], ref["union_ptr"][h, :n + 1])
    assert np.array_equal(got["union_pages"], ref["union_pages"])
    assert np.array_equal(got["row_mask"], ref["row_mask"])


def assert_bundles_equal(got, ref):
    Hkv = ref["n_bundles"].size
    assert np.array_equal(got["n_bundles"], ref["n_bundles"])
    assert np.array_equal(got["bcounters"], ref["bcounters"])
    for h in range(Hkv):
        n = int(ref["n_bundles"][h])
        assert np.array_equal(got["bundle_ptr"][h, :n + 1], ref["bundle_ptr"][h, :n + 1])
        m = int(ref["bundle_ptr"][h, n])
        assert np.array_equal(got["bundle_groups"][h, :m], ref["bundle_groups"][h, :m])
        assert np.array_equal(got["bunion_ptr"][h, :n + 1], ref["bunion_ptr"][h, :n + 1])
        assert np.array_equal(got["bundle_qid"][h, :n], ref["bundle_qid"][h, :n])
    assert np.array_equal(got["bunion_pages"], ref["bunion_pages"])
    assert np.array_equal(got["bunion_mask"], ref["bunion_mask"])
    if "bundle_order" in got:
        assert np.array_equal(got["bundle_order"], expected_bundle_order(ref))


def out_to_f64(O):
    import torch
    return O.float().cpu().numpy().astype(np.float64) if O.dtype != torch.float32 else \
        O.cpu().numpy().astype(np.float64)


# bounds from the arithmetic of each storage type (max abs, mean abs)
TOL = {W.DT_F32: (2e-2, 2e-3), W.DT_BF16: (2e-2, 2e-3), W.DT_E4M3: (6e-2, 6e-3)}


def check_close(got, ref, kv_dtype, what="", report=False):
    err = np.abs(got - ref)
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    tmax, tmean = TOL[kv_dtype]
    if report:  # one parseable line per comparison (shown with pytest -s)
        print(f"PARITY {what} elements={err.size} max_abs={mx:.3e} (bound {tmax}) "
              f"mean_abs={mean:.3e} (bound {tmean})", flush=True)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert mx <= tmax and mean <= tmean, f"{what}: max abs {mx:.3e} (<= {tmax}), mean abs {mean:.3e} (<= {tmean})"
    return mx, mean
