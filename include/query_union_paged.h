/*
 * query_union_paged.h -- C ABI of the B200 (sm_100a) library for token-level
 * sparse-attention prefill over a paged KV cache with page-affine query unions.
 *
 * Source of the operations: "PageWeaver: KV-Guided Query Unions for Sparse
 * Attention" (Abstract; Figure 1; Figure 2; Figure 3).  Each query attends only
 * to the tokens of its own TopK selected KV pages, causally inside a page.
 * Queries that share pages are gathered into unions of up to max_group queries,
 * so each union page is streamed once and fills tensor-core tiles, while every
 * query keeps exactly its own support and writes its output row at its
 * original query ID (no reordered Q tensor, no cross-page partial outputs).
 *
 * Conventions for every entry point
 *  - Pointers marked "device" are CUDA device pointers owned by the caller; the
 *    library never allocates or frees device memory.  Host pointers are read
 *    during the call only.
 *  - Calls are asynchronous on the given stream (cudaStream_t passed as void*;
 *    NULL = the legacy default stream) and do not synchronize.
 *  - The return value is QUP_OK or a synchronous error (bad argument, capacity,
 *    launch failure).  Errors found on the device (a page ID out of range, a
 *    bad group, a timed-out pipeline wait) are ORed into a per-device error
 *    word, read and cleared by qup_get_error().  No call aborts or traps.
 *
 * Layouts (row-major, innermost last)
 *   Q          [Nq][Hq][d]              bf16 or fp32
 *   K, V cache [P_phys][Hkv][T][d]      bf16, fp32 or FP8 E4M3 (+ fp32 scale per KV head)
 *   page_table [num_logical_pages]      int32, logical page -> physical page
 *   topk       [Hq][Nq][Ksel]           int32 logical page IDs, -1 = padding
 *   q_pos      [Nq]                     int32 token position of each query
 *   O          [Nq][Hq][d]              dtype of Q
 * Token t (logical position) lives in logical page t / T, slot t % T.  Query
 * i with position q_pos[i] attends token t iff the page of t is in its row of
 * topk, t <= q_pos[i] and t < kv_len.  KV head of Q head h' is h' / (Hq/Hkv).
 */
#ifndef QUERY_UNION_PAGED_H
#define QUERY_UNION_PAGED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes and device error bits */
#define QUP_OK 0
#define QUP_ERR_ARG 1          /* null pointer, bad dimension, unsupported dtype or limit */
#define QUP_ERR_CAPACITY 2     /* workspace or union capacity too small */
#define QUP_ERR_CUDA 4         /* a CUDA runtime call or launch failed */
#define QUP_ERR_PAGE_ID 8      /* device: a TopK or union page ID outside [0, num_logical_pages) */
#define QUP_ERR_PHYS_PAGE 16   /* device: a page_table entry outside [0, P_phys) */
#define QUP_ERR_GROUP 32       /* device: a group with no members, too many rows or a bad query ID */
#define QUP_ERR_TIMEOUT 64     /* device: a pipeline wait exceeded its limit; the kernel exited cleanly */

/* dtype codes */
#define QUP_F32 0
#define QUP_BF16 1
#define QUP_E4M3 2

/*
 * Output of qup_sparse_group (every buffer is device memory, caller-allocated;
 * sizes from qup_group_workspace).  For KV head h and group k:
 *   members  [h*Nq + group_ptr[h*(Nq+1)+k] .. h*Nq + group_ptr[h*(Nq+1)+k+1])
 *            query IDs of the group, ascending (at most max_group)
 *   union    [union_ptr[h*(Nq+1)+k] .. union_ptr[h*(Nq+1)+k+1]) indexes
 *            union_pages (sorted distinct logical pages of the group) and
 *            row_mask (bit r = rank*g + j set iff that page is in row
 *            topk[h*g+j][member of that rank]); offsets are absolute, the
 *            regions of the KV heads follow each other in head order.
 *   counters [h*4 + 0..3] = logical page visits (sum of union sizes), masked
 *            row slots, masked query slots, page edges (sum of |S(i)|).
 * (Figure 2: logical page visits and masked query-page slots.)
 *
 * Bundles (the attention kernel's work items; no counterpart on the pages,
 * which share a page between the two CTAs of one Union8 group instead):
 * the groups of one KV head are packed, inside windows of bundle_window
 * groups, into bundles of up to 128 / rows_per_group groups by a greedy on
 * group unions: seeded with the first unbundled group, grown by the group
 * with the smallest (new pages - 2 * pages already shared with the bundle
 * union), ties to the smallest index.  A bundle's query rows are
 * laid out slot by slot: row = slot*rows_per_group + rank*g + j, with
 * rows_per_group = max_group*g rounded up to a power of two (<= 32).
 *   bundle_ptr[h*(Nq+1)+b] .. [+b+1]  indexes bundle_groups[h*Nq + ...]
 *            (group indices within head h, ascending = slot order)
 *   bunion   [bunion_ptr[h*(Nq+1)+b] .. [+b+1]) indexes bunion_pages (sorted
 *            union of the bundle's groups) and bunion_mask[4*entry + w]:
 *            bit (row % 32) of word row/32 set iff the page is in that row's
 *            own TopK row.
 *   bundle_qid[(h*Nq + b)*(128/g) + row/g] = query ID of the row, -1 if the
 *            slot or rank is empty.
 *   bcounters[h*2 + 0..1] = bundle page visits (sum of bundle union sizes:
 *            the pages the attention kernel streams), number of bundles.
 *   bundle_order[0 .. total bundles) = flat bundle indices (f = bundles of
 *            earlier KV heads + b) sorted by union size, largest first, equal
 *            sizes by index: the order in which the attention kernel's CTAs
 *            claim bundles at run time.
 */
typedef struct {
    int32_t* n_groups;     /* [Hkv] */
    int32_t* group_ptr;    /* [Hkv][Nq+1] */
    int32_t* members;      /* [Hkv][Nq] */
    int32_t* union_ptr;    /* [Hkv][Nq+1] */
    int32_t* union_pages;  /* [cap_union] */
    uint64_t* row_mask;    /* [cap_union] */
    int64_t* counters;     /* [Hkv][4] */
    int64_t cap_union;     /* entries available in union_pages/row_mask and in bunion_pages */
    int32_t* n_bundles;    /* [Hkv] */
    int32_t* bundle_ptr;   /* [Hkv][Nq+1] */
    int32_t* bundle_groups;/* [Hkv][Nq] */
    int32_t* bunion_ptr;   /* [Hkv][Nq+1] */
    int32_t* bunion_pages; /* [cap_union] */
    uint32_t* bunion_mask; /* [cap_union][4] */
    int32_t* bundle_qid;   /* [Hkv][Nq][128/g] */
    int64_t* bcounters;    /* [Hkv][2] */
    int32_t* bundle_order; /* [Hkv*Nq] */
    int32_t rows_per_group;/* set by qup_sparse_group / qup_build_bundles */
    int32_t bundle_window; /* groups per bundling window: 0 (default 64) .. 256, else QUP_ERR_ARG */
} qup_groups;

/*
 * Sizes for qup_sparse_group.  Writes the scratch workspace bytes and the
 * union capacity that is always sufficient (Hkv * Nq * min(g*Ksel, pages)).
 * Returns QUP_ERR_ARG for unsupported sizes (window > 256, max_group*g > 32,
 * too many pages for the shared-memory bitsets).
 */
int qup_group_workspace(int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages, int max_group,
                        int window, size_t* ws_bytes, int64_t* cap_union);

/*
 * Bounded page-affinity grouping (Abstract: a GPU search of bounded cost
 * turns selected-page affinity into query-ID lists; Figure 2).  Per KV head h, S(i) is
 * the set of distinct valid pages of the g rows topk[h*g+j][i]; inside fixed
 * windows [w*window, (w+1)*window) of query IDs a group is seeded with the
 * smallest unassigned ID and grown, up to max_group members, by the candidate
 * that adds the fewest pages to the union (ties: smallest ID).  Output as in
 * qup_groups; bit-exact with the CPU reference of the same rule.
 *   topk       device int32 [Hq][Nq][Ksel]; -1 = padding, other IDs must lie
 *              in [0, num_logical_pages) (else QUP_ERR_PAGE_ID, entry ignored)
 *   max_group  1..8 and max_group*(Hq/Hkv) <= 32; window a multiple of
 *              max_group, <= 256 (window == max_group gives fixed consecutive groups)
 *   ws         device scratch of ws_bytes (from qup_group_workspace)
 */
int qup_sparse_group(const int32_t* topk, int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages,
                     int max_group, int window, qup_groups* out, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * qup_sparse_group without a caller workspace (the paper has no counterpart:
 * it is an allocation-free calling form of the same grouping).  For callers
 * that cannot hand over a scratch buffer: a host program holding no device
 * allocator at the call, or a serving loop whose device memory is fixed at
 * start-up.  The scratch lives in a fixed array of QUP_STATIC_GROUP_SCRATCH_BYTES
 * in this library's device image (one per device); nothing is allocated.
 * Arguments, outputs and device errors are those of qup_sparse_group.
 *  - Returns QUP_ERR_CAPACITY when the workspace qup_group_workspace reports
 *    for these sizes exceeds QUP_STATIC_GROUP_SCRATCH_BYTES; nothing is launched.
 *  - The first call on a device looks up the array's device address (a host
 *    query, with that device current); make that first call before capturing
 *    a stream.  The address is cached per device context: after a device reset
 *    (or in another context) the next call looks it up again.
 *  - Every call on one device shares the one array: two calls in flight at the
 *    same time (other streams, other host threads) race on it and corrupt each
 *    other's groups.  Order them on one stream.
 */
#define QUP_STATIC_GROUP_SCRATCH_BYTES (16u << 20)
int qup_sparse_group_static(const int32_t* topk, int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages,
                            int max_group, int window, qup_groups* out, void* stream);

/*
 * Pack the groups in `g` (n_groups .. row_mask filled, for instance by a
 * caller's own partition) into bundles: fills n_bundles .. bcounters and
 * rows_per_group.  max_group bounds the members of every group (1..8,
 * max_group*(Hq/Hkv) <= 32).  qup_sparse_group calls this itself.
 *   ws  device scratch of at least the size qup_group_workspace reports
 */
int qup_build_bundles(qup_groups* g, int Hq, int Hkv, int Nq, int num_logical_pages, int max_group,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * Union as support (CompactAttention: Accelerating Chunked Prefill with
 * Block-Union KV Selection, where each query block attends to the whole union
 * table of its KV group): rewrites the row masks of the groups in `g` so that
 * every row of a group sees every page of the group's union, then rebuilds the
 * bundles (as qup_build_bundles).  qup_sparse_prefill_attn on the result
 * computes attention over the group unions instead of each query's own TopK
 * rows.  The group counters keep describing the original selection.
 *   g, ws, sizes: as for qup_build_bundles; groups of more than 64 rows or
 *   union offsets past cap_union raise QUP_ERR_GROUP on the device.
 */
int qup_union_support(qup_groups* g, int Hq, int Hkv, int Nq, int num_logical_pages, int max_group,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * ID-aware union attention (Abstract; Figure 1; Figure 3).  One persistent
 * kernel: per bundle (up to 128 query rows of one KV head) it gathers the
 * rows of Q by original ID into shared memory, streams each page of the
 * bundle union once through a TMA ring, computes S = Q K^T and O += P V with
 * tcgen05 MMAs into TMEM (P written back to TMEM as the A operand), applies
 * each row's page mask and causal mask with an fp32 online softmax, and
 * writes each row to O[qid][h'][:].
 *   Q, q_dtype        device [Nq][Hq][d]; (QUP_F32 with kv QUP_F32) or
 *                     (QUP_BF16 with kv QUP_BF16 or QUP_E4M3)
 *   K_cache, V_cache  device [P_phys][Hkv][T][d], kv_dtype; 16-byte aligned
 *   k_scale, v_scale  device fp32 [Hkv], > 0, required iff kv_dtype == QUP_E4M3
 *   page_table        device int32 [num_logical_pages]
 *   T                 page tokens: 16, 32, 64 or 128
 *   topk, Ksel        device int32 [Hq][Nq][Ksel] or NULL.  The groups' row
 *                     masks carry each query's support: the kernel computes
 *                     from them alone.  topk is read only in checked mode
 *                     (qup_set_checked), which verifies the masks against it
 *                     first.
 *   groups            output of qup_sparse_group (or qup_build_bundles on
 *                     any partition); the kernel walks its bundles
 *   q_pos, kv_len     device int32 [Nq]; tokens >= kv_len are never attended
 *   d                 must be 128; softmax_scale (finite, > 0) is applied to q.k
 *   O                 device [Nq][Hq][d], dtype of Q; rows of queries that
 *                     are in no group are not written
 *   lse               device fp32 [Nq][Hq] natural-log sum of exponentials of
 *                     the scaled scores, or NULL; empty support gives O = 0,
 *                     lse = -inf
 * The CTAs claim bundles at run time from a device counter; each launch takes
 * the next of 64 counters per device in turn, so at most 64 launches of the
 * attention kernel (this call, the batched and page-major calls) may run at
 * the same time, and a captured CUDA graph holding one must not be replayed
 * while a replay of the same graph is still running.
 */
int qup_sparse_prefill_attn(const void* Q, int q_dtype, const void* K_cache, const void* V_cache,
                            int kv_dtype, const float* k_scale, const float* v_scale,
                            const int32_t* page_table, int num_logical_pages, int P_phys, int T,
                            const int32_t* topk, int Ksel, const qup_groups* groups,
                            const int32_t* q_pos, int kv_len, int Hq, int Hkv, int Nq, int d,
                            float softmax_scale, void* O, float* lse, void* stream);

/*
 * Batched requests (varlen chunks; chunked prefill of several sequences over
 * one paged cache, as in CompactAttention: Approach).  R sequences, each with
 * its own page table, cache length and chunk of queries, go through one
 * grouping call and one attention call.  The requests are laid end to end:
 *   q_ptr     device int32 [R+1], ascending: the queries of request r are the
 *             batch rows q_ptr[r] .. q_ptr[r+1) (rows of Q, O, q_pos, topk)
 *   page_ptr  device int32 [R+1], ascending: request r's logical pages are
 *             page_table[page_ptr[r] .. page_ptr[r+1]) of the concatenated
 *             page table (total_pages = page_ptr[R] entries, into one
 *             physical K/V cache)
 *   kv_len    device int32 [R]: tokens in request r's cache (at most its
 *             pages x T); q_pos and topk hold request-local positions and
 *             request-local logical page IDs (-1 = padding)
 * qup_batch_prepare writes, on the stream:
 *   topk_global device int32 [Hq][Nq][Ksel]: the TopK IDs rebased to the
 *             concatenated page space (page_ptr[r] + local ID; -1 kept), for
 *             qup_sparse_group(topk_global, ..., num_logical_pages = total_pages, ...)
 *   q_end     device int32 [Nq]: page_ptr[r]*T + min(q_pos + 1, kv_len[r]),
 *             the end of the query's visible positions (token slot o of
 *             concatenated page u has position u*T + o)
 *   page_len  device int32 [total_pages]: valid tokens of each page (0..T)
 * Device errors: a local page ID outside its request's pages raises
 * QUP_ERR_PAGE_ID (entry dropped); a row in no request or a kv_len beyond its
 * pages raises QUP_ERR_GROUP (the row attends nothing).  QUP_ERR_ARG for bad
 * sizes, T not in {16, 32, 64, 128}, total_pages*T >= 2^31 or missing
 * pointers.  Each query attends exactly the tokens the one-sequence call
 * would give it inside its own request.
 */
int qup_batch_prepare(const int32_t* topk, const int32_t* q_pos, int Hq, int Nq, int Ksel, int T, int R,
                      const int32_t* q_ptr, const int32_t* page_ptr, const int32_t* kv_len, int total_pages,
                      int32_t* topk_global, int32_t* q_end, int32_t* page_len, void* stream);

/*
 * Proxy-query page selection, the step upstream of qup_sparse_group that
 * produces each query's TopK pages (PIVOT: Efficient Query-Group Indexing for
 * Token-Level Sparse Attention, Abstract: one shared full-prefix scan per
 * group of nearby queries instead of one per query).  Queries are cut into
 * groups of group_size consecutive IDs; per KV head and group the mean of the
 * group's indexer queries (the proxy) scores every page the group's last
 * query can see, and its n_cand best pages are the candidates.  Each query
 * then takes Ksel of the candidates it can see (page p is visible to a query
 * at position q iff p * T <= q): re-scored with its own indexer query
 * (refine = 1, PIVOT-Refine) or in the proxy's order (refine = 0,
 * PIVOT-Reuse).  A score is the dot product of an indexer query with a page's
 * indexer key, computed in float32 with every product and sum rounded in
 * element order (the proxy: queries summed in ID order, then divided by the
 * group size); order = higher score first, equal scores by lower page ID.
 *   q_idx      device [Nq][Hkv][d_idx], dtype QUP_BF16 or QUP_F32, 16-byte aligned
 *   page_key   device [num_logical_pages][Hkv][d_idx], same dtype, 16-byte aligned
 *   q_pos      device int32 [Nq], token positions (>= 0)
 *   g          query heads per KV head (1..32): each KV head's selection is
 *              written to its g query heads
 *   topk       out: device int32 [Hkv*g][Nq][Ksel], -1 padded (the topk of
 *              qup_sparse_group, with num_logical_pages pages)
 * Limits (QUP_ERR_ARG otherwise): d_idx <= 512 and a multiple of 8 (bf16) or
 * 4 (fp32); num_logical_pages <= 8192; 1 <= Ksel <= n_cand <= 256; and one
 * CTA's shared memory must hold num_logical_pages * 8 + n_cand * d_idx *
 * (2 or 4) + 36 * d_idx + 2048 bytes (the candidates' key rows are staged
 * there).  Nothing is allocated; the call is asynchronous on `stream`.
 */
int qup_pivot_select(const void* q_idx, const void* page_key, int dtype, const int32_t* q_pos, int Nq, int Hkv,
                     int g, int d_idx, int num_logical_pages, int T, int group_size, int n_cand, int Ksel,
                     int refine, int32_t* topk, void* stream);

/*
 * qup_sparse_prefill_attn for batched requests: the arguments of
 * qup_sparse_prefill_attn with (q_pos, kv_len) replaced by the q_end and
 * page_len arrays of qup_batch_prepare, page_table the concatenated table of
 * total_pages entries, and groups from qup_sparse_group on topk_global.
 * topk_global is read only in checked mode (and may be NULL).
 */
int qup_sparse_prefill_attn_batch(const void* Q, int q_dtype, const void* K_cache, const void* V_cache,
                                  int kv_dtype, const float* k_scale, const float* v_scale,
                                  const int32_t* page_table, int total_pages, int P_phys, int T,
                                  const int32_t* topk_global, int Ksel, const qup_groups* groups,
                                  const int32_t* q_end, const int32_t* page_len, int Hq, int Hkv, int Nq, int d,
                                  float softmax_scale, void* O, float* lse, void* stream);

/*
 * Direct KV-page union (PageWeaver, Abstract; Figure 5): the page-major
 * alternative to query unions.  Work is organised by KV page instead of by
 * query group: the pages of each KV head are cut into tiles of 256 tokens
 * (tile_pages = 256 / T pages), and an item is one tile with up to 128 / g
 * queries whose page set (over the g Q heads of the KV group) meets it.  Each
 * tile is streamed once per item by the same tensor-core union kernel; every
 * row (query, Q head) keeps its own page mask and gets one partial result per
 * tile its own TopK row touches (O_t / l_t in fp32 and lse_t in log2 units),
 * which a merge then reduces per row by lse.  The result equals
 * qup_sparse_prefill_attn's (the same per-query supports) up to rounding.
 *
 * Sizes (qup_page_major_workspace): ws_bytes of scratch for the item builder,
 * item_cap items per KV head and slot_cap partial slots that always suffice,
 * tile_pages.  QUP_ERR_ARG for unsupported sizes (g > 32, too many pages for
 * the builder's shared-memory bitsets, capacities past 2^31).
 */
typedef struct {
    int32_t* n_items;      /* [Hkv] items of each KV head */
    int32_t* item_ptr;     /* [Hkv][item_cap+1] first union entry of each item (item i: tile_pages entries) */
    int32_t* item_pages;   /* [Hkv*item_cap*tile_pages] logical pages of each item's tile */
    uint32_t* item_mask;   /* [Hkv*item_cap*tile_pages][4] 128-bit row masks, as bunion_mask */
    int32_t* item_qid;     /* [Hkv][item_cap][128/g] query of each query slot, -1 if empty */
    int32_t* item_slot;    /* [Hkv*item_cap][128] partial slot of each row, -1 if the row has none */
    int32_t* item_order;   /* [Hkv*item_cap] order in which the kernel's CTAs claim items */
    int64_t* row_off;      /* [Hq*Nq+1] partial slots of row (h', i) = h'*Nq + i: row_off[..] .. row_off[..+1] */
    int64_t item_cap;      /* items per KV head the arrays hold */
    int64_t slot_cap;      /* partial slots the caller's part_o / part_lse hold */
    int32_t tile_pages;    /* set by qup_page_major_items */
} qup_page_items;

int qup_page_major_workspace(int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages, int T, size_t* ws_bytes,
                             int64_t* item_cap, int64_t* slot_cap, int32_t* tile_pages);

/*
 * Builds the page-major items of topk (device int32 [Hq][Nq][Ksel], -1 =
 * padding) on the stream: five small kernels; a query's place inside the items
 * of a tile comes from an atomic counter (run-to-run order varies, results do
 * not).  Device errors: QUP_ERR_PAGE_ID for IDs out of range (dropped),
 * QUP_ERR_CAPACITY if the items or slots exceed the caps.
 */
int qup_page_major_items(const int32_t* topk, int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages, int T,
                         qup_page_items* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Page-major attention: the union kernel over the items, writing each row's
 * partial results to part_o (device fp32 [slot_cap][d], 16-byte aligned) and
 * part_lse (device fp32 [slot_cap]), then the merge into O [Nq][Hq][d] and lse
 * (fp32 [Nq][Hq] natural log, or NULL).  Other arguments as for
 * qup_sparse_prefill_attn.
 */
int qup_page_major_attn(const void* Q, int q_dtype, const void* K_cache, const void* V_cache, int kv_dtype,
                        const float* k_scale, const float* v_scale, const int32_t* page_table, int num_logical_pages,
                        int P_phys, int T, const qup_page_items* items, const int32_t* q_pos, int kv_len, int Hq,
                        int Hkv, int Nq, int d, float softmax_scale, float* part_o, float* part_lse, void* O,
                        float* lse, void* stream);

/* Synchronizes `stream`, then reads and clears this device's error word. */
int qup_get_error(int* code, void* stream);

/* Static text for a return code or error bit. */
const char* qup_error_string(int code);

/*
 * Pipeline-wait limit and host-side fault injection (for tests of the bounded
 * waits; both reset with wait_limit_ms <= 0 and skip_stage < 0).  With
 * skip_stage >= 0 no CTA of the attention kernel loads that stage of its K
 * and V rings, so the consumers' waits run out after wait_limit_ms,
 * QUP_ERR_TIMEOUT is raised and every CTA exits cleanly.
 */
int qup_set_debug(int wait_limit_ms, int skip_stage);

/*
 * Checked mode (process-wide, off by default; on = nonzero).  While it is on,
 * qup_sparse_prefill_attn given a non-NULL topk first runs one extra kernel on
 * the stream that checks every bundle row against its own TopK row: a mask
 * bit is set exactly for the union pages the row selected (a set: duplicates
 * and -1 dropped), every page of the row is in the bundle union, and rows of
 * empty slots carry no bits.  A mismatch raises QUP_ERR_GROUP (a TopK ID out
 * of range QUP_ERR_PAGE_ID) in the device error word; the attention call
 * still runs.  Ksel < 0 is then QUP_ERR_ARG.  Meant for groups a caller builds
 * itself; qup_sparse_group's groups satisfy it by construction.
 */
int qup_set_checked(int on);

/* Number of SMs the persistent attention kernel is sized for on the current device. */
int qup_num_sms(void);

/*
 * Test hook (no counterpart on the pages): y[i] = 2^x[i] by the polynomial
 * exponential the attention kernel uses for part of its softmax (x clamped to
 * -127, where the result is exactly +0; x must be <= 16).  x and y are device
 * float arrays of n elements; asynchronous on `stream`.  Returns QUP_ERR_ARG
 * for n < 0 or null pointers with n > 0, QUP_ERR_CUDA for a launch failure.
 */
int qup_exp2_poly(const float* x, float* y, int n, void* stream);

#ifdef __cplusplus
}
#endif
#endif
