"""Seeded synthetic inputs for paged sparse-attention prefill with query unions.

This module only draws inputs. It holds none of the method's arithmetic: no
scores, no softmax, no grouping. Both the CUDA path and the fp64 oracle are fed
from it, so it is the one piece the two share.

The shapes follow the prefill chunks the PageWeaver page measures (Abstract;
Table 1: 16K-query chunks after 0/16K prefixes, a constructed 64K input, Top16
pages per query, FP8 KV) and the block-union workload of CompactAttention
(Approach: 2D block-sparse masks unioned over query blocks and the heads of a
KV group). Real model captures are not available here; every array below is a
synthetic stand-in whose recipe is stated next to its builder.

Storage layouts (the exact bytes both sides read):
  Q        [Nq][Hq][d]            float32 or bfloat16 bits (uint16)
  K, V     [P_phys][Hkv][T][d]    float32, bfloat16 bits (uint16) or E4M3 bytes (uint8)
  k_scale, v_scale [Hkv] float32  (E4M3 only; value = byte decoded * scale)
  page_table [num_logical_pages] int32  logical page -> physical page
  topk     [Hq][Nq][K] int32      selected logical pages, -1 = padding
  q_pos    [Nq] int32             token position of each query
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

DT_F32, DT_BF16, DT_E4M3 = 0, 1, 2
DTYPE_NAMES = {DT_F32: "f32", DT_BF16: "bf16", DT_E4M3: "e4m3"}


@dataclasses.dataclass
class Workload:
    name: str
    Hq: int
    Hkv: int
    Nq: int
    d: int
    T: int
    K: int
    num_logical_pages: int
    P_phys: int
    kv_len: int
    q_dtype: int
    kv_dtype: int
    Q: np.ndarray
    Kc: np.ndarray
    Vc: np.ndarray
    k_scale: Optional[np.ndarray]
    v_scale: Optional[np.ndarray]
    page_table: np.ndarray
    topk: np.ndarray
    q_pos: np.ndarray
    max_group: int = 8
    window: int = 64
    bundle_window: int = 64

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def softmax_scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    def kv_page_bytes(self) -> int:
        """K+V bytes of one page of one KV head."""
        es = 1 if self.kv_dtype == DT_E4M3 else (2 if self.kv_dtype == DT_BF16 else 4)
        return 2 * self.T * self.d * es

    def describe(self) -> dict:
        return {"workload": self.name, "Hq": self.Hq, "Hkv": self.Hkv, "Nq": self.Nq,
                "d": self.d, "page_tokens": self.T, "topk": self.K,
                "kv_len": self.kv_len, "kv_dtype": DTYPE_NAMES[self.kv_dtype],
                "q_dtype": DTYPE_NAMES[self.q_dtype], "max_group": self.max_group,
                "window": self.window}


# ---------------------------------------------------------------------------
# storage conversions (input preparation only)
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest even) and return the bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((b >> 16) & 1) + np.uint32(0x7FFF)
    return ((b + r) >> 16).astype(np.uint16)


def f32_to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    """Quantise to OCP E4M3 (round to nearest even, saturating at 448) via torch."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).clamp_(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _store_kv(rng, shape, kv_dtype):
    """Draw N(0,1) K or V in fp32 and store it in the requested format."""
    x = rng.standard_normal(shape, dtype=np.float32)
    if kv_dtype == DT_F32:
        return x, None
    if kv_dtype == DT_BF16:
        return f32_to_bf16_bits(x), None
    # E4M3 with one fp32 scale per KV head: scale = amax / 448 over that head's cache
    Hkv = shape[1]
    amax = np.abs(x).reshape(shape[0], Hkv, -1).max(axis=(0, 2)).astype(np.float32)
    scale = (amax / np.float32(448.0)).astype(np.float32)
    q = f32_to_e4m3_bytes(x / scale[None, :, None, None])
    return q, scale


def _store_q(rng, shape, q_dtype):
    x = rng.standard_normal(shape, dtype=np.float32)
    return x if q_dtype == DT_F32 else f32_to_bf16_bits(x)


def _finish(name, rng, Hq, Hkv, Nq, d, T, prefix, q_dtype, kv_dtype, topk,
            max_group=8, window=64, identity_pages=False):
    kv_len = prefix + Nq
    nlp = -(-kv_len // T)  # the last page may be partly filled
    P_phys = nlp
    page_table = (np.arange(nlp, dtype=np.int32) if identity_pages
                  else rng.permutation(nlp).astype(np.int32))
    Q = _store_q(rng, (Nq, Hq, d), q_dtype)
    Kc, ks = _store_kv(rng, (P_phys, Hkv, T, d), kv_dtype)
    Vc, vs = _store_kv(rng, (P_phys, Hkv, T, d), kv_dtype)
    q_pos = (prefix + np.arange(Nq)).astype(np.int32)
    return Workload(name=name, Hq=Hq, Hkv=Hkv, Nq=Nq, d=d, T=T, K=topk.shape[2],
                    num_logical_pages=nlp, P_phys=P_phys, kv_len=kv_len,
                    q_dtype=q_dtype, kv_dtype=kv_dtype, Q=Q, Kc=Kc, Vc=Vc,
                    k_scale=ks, v_scale=vs, page_table=page_table,
                    topk=np.ascontiguousarray(topk, dtype=np.int32), q_pos=q_pos,
                    max_group=max_group, window=window)


def _replicate_kv_groups(sel_kv: np.ndarray, g: int) -> np.ndarray:
    """[Hkv][Nq][K] per-KV-head selection -> [Hq][Nq][K] (same pages for the g Q heads)."""
    return np.repeat(sel_kv, g, axis=0)


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------

def tiny_ref(seed: int = 0, identity_pages: bool = False) -> Workload:
    """1 head, d=128, fp32; 64 pages of 64 tokens; 256 queries at 3840..4095.

    TopK 8 per query: page 0, the query's own page, and 6 distinct pages drawn
    uniformly from the pages strictly between them.
    """
    rng = np.random.default_rng(seed)
    T, prefix, Nq = 64, 3840, 256
    sel = np.empty((1, Nq, 8), np.int32)
    for i in range(Nq):
        own = (prefix + i) // T
        extra = rng.choice(np.arange(1, own), size=6, replace=False)
        sel[0, i] = np.concatenate([[0, own], extra])
    return _finish("tiny_ref_fp32", rng, 1, 1, Nq, 128, T, prefix, DT_F32, DT_F32, sel,
                   identity_pages=identity_pages)


def _community_chunk(name, seed, kv_dtype, T, prefix, Nq, n_comm, comm_size, comm_lo, comm_hi,
                     identity_pages=False, window=64):
    """GQA 32/8 chunk: {sink 0, own page, own-1} + 13 pages from the query's community."""
    rng = np.random.default_rng(seed)
    Hq, Hkv, d, K = 32, 8, 128, 16
    g = Hq // Hkv
    sel = np.empty((Hkv, Nq, K), np.int32)
    own = (prefix + np.arange(Nq)) // T
    for h in range(Hkv):
        pool = rng.choice(np.arange(comm_lo, comm_hi + 1), size=n_comm * comm_size, replace=False)
        comms = pool.reshape(n_comm, comm_size)
        cid = rng.integers(0, n_comm, size=Nq)
        # 13 distinct members of the query's community: the first 13 of a random permutation
        # of its comm_size members (one independent permutation per query)
        keys = rng.random((Nq, comm_size))
        picks = np.take_along_axis(comms[cid], np.argsort(keys, axis=1)[:, :K - 3], axis=1)
        sel[h, :, 0] = 0
        sel[h, :, 1] = own
        sel[h, :, 2] = own - 1
        sel[h, :, 3:] = picks
    q_dtype = DT_BF16
    return _finish(name, rng, Hq, Hkv, Nq, d, T, prefix, q_dtype, kv_dtype,
                   _replicate_kv_groups(sel, g), identity_pages=identity_pages, window=window)


def gqa_chunk_bf16(seed: int = 1, identity_pages: bool = False) -> Workload:
    """32/8 heads, bf16, 16K prefix + 2048-query chunk, 64-token pages, Top16.

    Per KV head: 8 disjoint communities of 15 pages drawn from pages 1..254;
    each query's community is drawn iid, so same-community queries are mostly
    not adjacent. Selection per (KV head, query), replicated to its 4 Q heads.
    """
    return _community_chunk("gqa_chunk_bf16_16k+2k", seed, DT_BF16, 64, 16384, 2048,
                            8, 15, 1, 254, identity_pages)


def gqa_chunk_fp8(seed: int = 2, identity_pages: bool = False) -> Workload:
    """As gqa_chunk_bf16 with E4M3 KV (per-KV-head scale) and 128-token pages.

    Grouping window 128 queries: with E4M3 the attention call outweighs the grouping call, and
    the wider window's tighter groups save more attention time than they cost.
    """
    return _community_chunk("gqa_chunk_fp8_16k+2k", seed, DT_E4M3, 128, 16384, 2048,
                            8, 15, 1, 126, identity_pages, window=128)


def chunk16k_fp8(seed: int = 5, identity_pages: bool = False) -> Workload:
    """A 16K-query chunk after a 16K prefix (the pages' base captures: 16K-query chunks, Top16,
    FP8 KV): 32/8 heads, E4M3 KV (per-KV-head scale), 128-token pages, TopK 16 = {sink, own,
    own-1} + 13 from the query's community (8 disjoint communities of 15 pages in 1..126 per KV
    head, one per query iid).  Grouping window 128, as for the other E4M3 community workloads.
    """
    return _community_chunk("chunk16k_fp8_16k+16k", seed, DT_E4M3, 128, 16384, 16384,
                            8, 15, 1, 126, identity_pages, window=128)


def ctx64k_fp8(mix: str = "b", seed: int = 3, identity_pages: bool = False) -> Workload:
    """32/8 heads, E4M3 KV, 64K prefix + 4096-query chunk, 128-token pages, Top16.

    mix "a" (local): own page + the 15 preceding pages.
    mix "b" (50/50): own page + 7 preceding + 8 drawn from a community of 10.
    mix "c" (community): 16 drawn from a community of 18.
    8 disjoint communities per KV head drawn from pages 0..495, one per query iid.
    Grouping window 128 queries for mixes b and c (as for gqa_chunk_fp8); 64 for the local mix,
    whose queries of one page share their whole selection (no union to tighten).
    """
    rng = np.random.default_rng(seed)
    Hq, Hkv, d, T, prefix, Nq, K = 32, 8, 128, 128, 65536, 4096, 16
    g = Hq // Hkv
    sel = np.empty((Hkv, Nq, K), np.int32)
    csize = {"a": 1, "b": 10, "c": 18}[mix]
    for h in range(Hkv):
        pool = rng.choice(np.arange(0, 496), size=8 * csize, replace=False)
        comms = pool.reshape(8, csize)
        cid = rng.integers(0, 8, size=Nq)
        for i in range(Nq):
            own = (prefix + i) // T
            if mix == "a":
                sel[h, i] = own - np.arange(16)
            elif mix == "b":
                picks = rng.choice(comms[cid[i]], size=8, replace=False)
                sel[h, i] = np.concatenate([own - np.arange(8), picks])
            else:
                sel[h, i] = rng.choice(comms[cid[i]], size=16, replace=False)
    return _finish(f"ctx64k_fp8_mix{mix}", rng, Hq, Hkv, Nq, d, T, prefix, DT_BF16, DT_E4M3,
                   _replicate_kv_groups(sel, g), identity_pages=identity_pages,
                   window=64 if mix == "a" else 128)


def block_union_128k(seed: int = 4, identity_pages: bool = False) -> Workload:
    """32/8 heads, bf16, 128K prefix + 1024-query chunk, 64-token pages.

    A query block is 64 queries (one chunk page b). Per (Q head, block b): the
    band {2047+b, 2048+b} plus each page 0..2046+b with probability 0.1. Every
    query of the block carries its block's row; K = the longest row, padded -1.
    """
    rng = np.random.default_rng(seed)
    Hq, Hkv, d, T, prefix, Nq = 32, 8, 128, 64, 131072, 1024
    nb = Nq // 64
    rows = [[None] * nb for _ in range(Hq)]
    kmax = 0
    for hq in range(Hq):
        for b in range(nb):
            cand = np.arange(0, 2047 + b)
            pick = cand[rng.random(cand.size) < 0.1]
            r = np.concatenate([pick, [2047 + b, 2048 + b]]).astype(np.int32)
            rows[hq][b] = r
            kmax = max(kmax, r.size)
    sel = np.full((Hq, Nq, kmax), -1, np.int32)
    for hq in range(Hq):
        for b in range(nb):
            r = rows[hq][b]
            sel[hq, b * 64:(b + 1) * 64, :r.size] = r
    return _finish("block_union_bf16_128k+1k", rng, Hq, Hkv, Nq, d, T, prefix, DT_BF16, DT_BF16,
                   sel, identity_pages=identity_pages)


def random_small(seed: int, Hq=4, Hkv=2, Nq=100, d=128, T=64, prefix=960, K=6,
                 q_dtype=DT_BF16, kv_dtype=DT_BF16, max_group=8, window=64,
                 dup_frac=0.1, pad_frac=0.1, identity_pages=False) -> Workload:
    """Small random case with duplicates and -1 padding in the TopK rows.

    Pages are drawn uniformly from the query's causal range (0..own page), so
    some rows include future-free pages only; the own page is always present.
    """
    rng = np.random.default_rng(seed)
    sel = np.empty((Hq, Nq, K), np.int32)
    for hq in range(Hq):
        for i in range(Nq):
            own = (prefix + i) // T
            row = rng.integers(0, own + 1, size=K)
            row[0] = own
            dup = rng.random(K) < dup_frac
            row[dup] = row[0]
            pad = rng.random(K) < pad_frac
            pad[0] = False
            row[pad] = -1
            sel[hq, i] = row
    return _finish(f"random_small_s{seed}", rng, Hq, Hkv, Nq, d, T, prefix, q_dtype, kv_dtype,
                   sel, max_group=max_group, window=window, identity_pages=identity_pages)


@dataclasses.dataclass
class IndexerInputs:
    """Inputs of the proxy-query page selector: indexer queries q [Nq][Hkv][d] and page keys
    k [P][Hkv][d] (float32 values that bf16 holds exactly when bf16, plus their bf16 bits),
    positions q_pos [Nq]."""
    q: np.ndarray
    k: np.ndarray
    q_bits: Optional[np.ndarray]
    k_bits: Optional[np.ndarray]
    q_pos: np.ndarray
    T: int
    num_logical_pages: int


def indexer_inputs(seed: int, Nq: int, Hkv: int, d: int, prefix: int, T: int, bf16: bool = True,
                   integer: bool = False, shuffle_positions: bool = False, extra_pages: int = 0) -> IndexerInputs:
    """Seeded indexer queries and page keys: N(0, 1) (or small integers in -3..3, which make every
    score exact and produce ties), for a chunk of Nq queries after `prefix` tokens.  The positions
    are prefix + 0 .. Nq-1, optionally permuted; the page space covers them plus extra_pages."""
    rng = np.random.default_rng(seed)
    P = (prefix + Nq + T - 1) // T + extra_pages
    if integer:
        q = rng.integers(-3, 4, size=(Nq, Hkv, d)).astype(np.float32)
        k = rng.integers(-3, 4, size=(P, Hkv, d)).astype(np.float32)
    else:
        q = rng.standard_normal((Nq, Hkv, d), dtype=np.float32)
        k = rng.standard_normal((P, Hkv, d), dtype=np.float32)
    qb = kb = None
    if bf16:
        qb, kb = f32_to_bf16_bits(q), f32_to_bf16_bits(k)
        q = (qb.astype(np.uint32) << 16).view(np.float32)
        k = (kb.astype(np.uint32) << 16).view(np.float32)
    pos = prefix + np.arange(Nq, dtype=np.int32)
    if shuffle_positions:
        pos = rng.permutation(pos).astype(np.int32)
    return IndexerInputs(q, k, qb, kb, pos, T, P)


CONFIGS = {
    "1": tiny_ref,
    "2": gqa_chunk_bf16,
    "3": gqa_chunk_fp8,
    "4a": lambda **kw: ctx64k_fp8("a", **kw),
    "4b": lambda **kw: ctx64k_fp8("b", **kw),
    "4c": lambda **kw: ctx64k_fp8("c", **kw),
    "5": block_union_128k,
    "6": chunk16k_fp8,
}


def make(config: str, **kw) -> Workload:
    return CONFIGS[config](**kw)
