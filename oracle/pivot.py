"""Proxy-query page selection (PIVOT-style), the CPU definition the device selector is checked against.

TEST INFRASTRUCTURE, like the rest of this package: only the tests, the smoke check and the bench's
CPU leg use it, and it shares no code with the CUDA library.

PIVOT (Efficient Query-Group Indexing for Token-Level Sparse Attention, Abstract) replaces the
per-query full-prefix scan of a sparse-attention indexer with one scan per group of nearby queries:
the group's queries are aggregated into one proxy query, the proxy scores every preceding key once
to give a candidate set, and each query then takes its own top-k from the candidates (PIVOT-Refine:
re-scored with the query's own indexer query) or the proxy's top-k (PIVOT-Reuse).  In prefill the
groups are fixed-size runs of consecutive queries.

The readings made here, where the page leaves the step open:
  * the selection unit is a KV page (the TopK pages per query that the grouping call consumes), and
    each page has an indexer key per KV head (an input: how it is pooled from the page's tokens is
    upstream of this step); a score is the dot product of an indexer query with a page key;
  * the proxy query is the mean of the group's indexer queries;
  * a query sees pages p with p * T <= its position; the proxy scans the pages its group's last
    query sees; the candidate set is the proxy's n_cand best pages;
  * order: higher score first, equal scores by lower page ID; rows are padded with -1;
  * one selection per KV head, copied to the g query heads of the KV group (output [Hkv*g][Nq][K]).

Arithmetic is float32 with a fixed order, so that the device, which performs the same IEEE
operations in the same order, reaches bit-identical scores and the same integer decisions:
  proxy[t]  = (sum over the group's queries in order of q[t]) / n        (each + and / rounded)
  score(v, k) = sum over t = 0 .. d-1 of (v[t] * k[t])                   (each * and + rounded)
"""
from __future__ import annotations

import numpy as np


def _score(v: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Scores of one float32 vector against rows of keys: sequential float32 accumulation over t
    (no fused multiply-add, no pairwise summation)."""
    acc = np.zeros(keys.shape[0], np.float32)
    for t in range(v.shape[0]):
        acc = (acc + (keys[:, t] * v[t]).astype(np.float32)).astype(np.float32)
    return acc


def _ranked(pages, scores):
    """Pages ordered by score (higher first), equal scores by page ID (lower first)."""
    return sorted(pages, key=lambda p: (-float(scores[p]), int(p)))


def pivot_select(q_idx, page_key, q_pos, T: int, num_logical_pages: int, group_size: int, n_cand: int,
                 K: int, refine: bool, g: int) -> np.ndarray:
    """TopK page IDs per (query head, query): int32 [Hkv*g][Nq][K], -1 padded.

    q_idx     [Nq][Hkv][d] indexer queries (any float dtype whose values float32 holds exactly)
    page_key  [P][Hkv][d] page indexer keys, P = num_logical_pages
    q_pos     [Nq] token positions
    """
    q = np.asarray(q_idx, np.float32)
    keys_all = np.asarray(page_key, np.float32)
    pos = np.asarray(q_pos, np.int64)
    Nq, Hkv, d = q.shape
    P = int(num_logical_pages)
    out = np.full((Hkv, Nq, K), -1, np.int32)
    for h in range(Hkv):
        keys = keys_all[:, h, :]
        for g0 in range(0, Nq, group_size):
            members = list(range(g0, min(Nq, g0 + group_size)))
            acc = np.zeros(d, np.float32)
            for i in members:
                acc = (acc + q[i, h]).astype(np.float32)
            proxy = (acc / np.float32(len(members))).astype(np.float32)
            lim = min(P, int(max(pos[i] for i in members)) // T + 1)
            if lim <= 0:
                continue
            ps = _score(proxy, keys[:lim])
            cand = _ranked(range(lim), ps)[:n_cand]
            for i in members:
                vis = int(pos[i]) // T
                mine = [p for p in cand if p <= vis]
                if refine and mine:
                    qs = np.zeros(lim, np.float32)
                    qs[mine] = _score(q[i, h], keys[mine])
                    sel = _ranked(mine, qs)[:K]
                else:
                    sel = mine[:K]
                out[h, i, :len(sel)] = sel
    return np.repeat(out, g, axis=0)
