// internal.h -- declarations shared by the host layer and the kernel files.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

namespace qup {

constexpr int kStepTok = 128;   // union tokens per pipeline step (MMA M of S^T, K of PV)
constexpr int kHeadDim = 128;
constexpr int kMaxPPS = 8;      // pages per 128-token step at T = 16
constexpr int kMaxStages = 16;
// Launch slots of the attention kernel's run-time bundle counter: launches that run at the
// same time must hold different slots (the host hands them out in turn).
constexpr int kWalkSlots = 64;

// Raises a kernel's dynamic shared-memory limit to `smem` once per device context (the
// attribute is a maximum: later launches with less need no call).
cudaError_t ensure_smem_attr(const void* fn, size_t smem);

// Unique ID (over the life of the process) of the CUDA context current on this thread, the
// primary context of the current device being made current first if none is.  Caches of
// device addresses and kernel attributes are keyed on it: a device reset or another context
// gets a new ID, so nothing looked up in an earlier context is reused.  0 on failure.
unsigned long long context_id();

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel of the stream finishes; it calls grid_dep_wait() before it
// reads anything that kernel (or earlier work) produced.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct AttnParams {
    const void* Q;
    const float* k_scale;
    const float* v_scale;
    const int32_t* page_table;
    const int32_t* n_bundles;    // [Hkv]
    const int32_t* union_ptr;    // bundle unions: [Hkv][Nq+1] absolute offsets
    const int32_t* union_pages;  // [cap]
    const uint32_t* row_mask;    // [cap][4] 128-bit row masks
    const int32_t* bundle_qid;   // [Hkv][Nq][128/g]
    const int32_t* bundle_order; // [n_items] flat bundle indices, largest union first
    const int32_t* q_pos;
    const int32_t* q_end;     // batched requests: [Nq] end of each query's visible positions, else null
    const int32_t* page_len;  // batched requests: [num_logical_pages] valid tokens per page, else null
    void* O;
    float* lse;
    unsigned* err;
    long long cap_union;
    int num_logical_pages, P_phys, T, kv_len, Hq, Hkv, Nq, g;
    float scale_log2;  // softmax_scale * log2(e)
    int bstride;       // bundles per KV head in the bundle arrays' layout (Nq for groups)
    // page-major items: every row's partial result (O / l in fp32, log2-domain lse) goes to
    // part_o[slot][d], part_lse[slot], slot = item_slot[flat item][row] (-1: none); null otherwise
    float* part_o;
    float* part_lse;
    const int32_t* item_slot;
    int nsk, nsv;  // slots of the K ring and of the V ring
    unsigned long long wait_limit_ns;
    int dbg_skip_stage;
    int walk_slot;  // 0 .. kWalkSlots-1: this launch's bundle counter
};

// dynamic shared memory of the attention kernel for (element size, K slots, V slots, KV heads),
// and one K or V tile (one ring slot)
size_t attn_smem_bytes(int es, int nsk, int nsv, int Hkv, int g);
size_t attn_tile_bytes(int es);

// tmQ: Q [Nq][Hq][d] bf16 with a box of (64 elements, g heads, 1 query) and 128-byte swizzle
// (read by the bf16 kernel only)
cudaError_t launch_union_attn(int es, int T, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                              const AttnParams& p, int grid, size_t smem, cudaStream_t stream);

// page-major items (page_major.cu): shared memory of the count and fill kernels, the item
// builder (count, scan, clear, fill) and the merge of partial results
size_t page_major_build_smem(int g, int NW);
cudaError_t launch_page_major_build(const int32_t* topk, int Hq, int Hkv, int Nq, int K, int P, int NW, int Pt,
                                    int ntiles, int MQ, long long item_cap, long long slot_cap, int32_t* tile_cnt,
                                    int32_t* tile_fill, int32_t* row_cnt, int64_t* tile_base, int64_t* row_off,
                                    int64_t* totals, int32_t* n_items, int32_t* item_ptr, int32_t* item_pages,
                                    uint32_t* item_mask, int32_t* item_qid, int32_t* item_slot, int32_t* item_order,
                                    unsigned* err, cudaStream_t st);
cudaError_t launch_page_major_merge(const float* part_o, const float* part_lse, const int64_t* row_off, int Hq, int Nq,
                                    int q_bf16, void* O, float* lse, cudaStream_t st);

// checked mode: every bundle row's page mask against its own TopK row (QUP_ERR_GROUP on a mismatch)
cudaError_t launch_check_support(const int32_t* topk, int K, int Hkv, int Nq, int g, int P, const int32_t* n_bundles,
                                 const int32_t* bunion_ptr, const int32_t* bunion_pages,
                                 const uint32_t* bunion_mask, const int32_t* bundle_qid, long long cap,
                                 unsigned* err, int sms, cudaStream_t stream);

// the softmax's polynomial 2^x over n floats (test hook)
cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t stream);

// Pick value of the bundling greedy (groups packed into bundles; execution-level, no counterpart
// on the pages): new pages counted against the pages a candidate already shares with the bundle
// union, new - 2 * shared = 3 * new - 2 * |S(c)|, biased non-negative (exact for windows whose
// universe is below 2^20 pages).  The pick key is (value << 9 | local_id), as for groups, whose
// value is the new page count alone.
constexpr int kBundleKeyBias = 1 << 21;
__host__ __device__ inline unsigned pick_value(int new_pages, int set_size, bool bundle) {
    return bundle ? (unsigned)(3 * new_pages - 2 * set_size + kBundleKeyBias) : (unsigned)new_pages;
}

struct GroupLaunch {
    const int32_t* topk;
    int Hq, Hkv, Nq, K, P, NW, max_group, W, nwin;
    uint32_t* rowbits;
    int32_t* ws_usize;
    int32_t* ws_wtot;
    int32_t* ws_wcnt;
    int32_t* n_groups;
    int32_t* group_ptr;
    int32_t* members;
    int32_t* union_ptr;
    int32_t* union_pages;
    uint64_t* row_mask;
    long long cap;
    int64_t* counters;
    unsigned* err;
    int sms;
};

size_t group_greedy_smem(int W, int NW);
cudaError_t launch_group(const GroupLaunch& a, cudaStream_t stream);

struct BundleLaunch {
    int Hkv, Nq, P, NW, g, RS, slots, WB, nwin;
    const int32_t* n_groups;
    const int32_t* group_ptr;
    const int32_t* members;
    const int32_t* union_ptr;
    const int32_t* union_pages;
    const uint64_t* row_mask;
    uint32_t* gbits;
    int32_t* ws_usize;
    int32_t* ws_wtot;
    int32_t* ws_wcnt;
    int32_t* n_bundles;
    int32_t* bundle_ptr;
    int32_t* bundle_groups;
    int32_t* bunion_ptr;
    int32_t* bunion_pages;
    uint32_t* bunion_mask;
    int32_t* bundle_qid;
    long long cap;
    int64_t* bcounters;
    int32_t* bundle_order;
    unsigned* err;
    int sms;
};

cudaError_t launch_bundles(const BundleLaunch& a, cudaStream_t stream);

// Fused grouping path (group_fused.cu): dynamic shared memory of each kernel,
// and the launches.  wcnt / status are workspace arrays sized for Hkv * Nq
// windows; status, the bundle kernel's `done` word and each kernel's window
// ticket must be zero at launch.
size_t fused_group_smem(int W, int g, int NW);
size_t fused_bundle_smem(int WB, int NW, int Hkv);
cudaError_t launch_group_fused(const GroupLaunch& a, uint32_t* gbits, int32_t* wcnt, uint64_t* status,
                               unsigned* ticket, cudaStream_t stream);
cudaError_t launch_bundles_fused(const BundleLaunch& a, int32_t* wcnt, uint64_t* status, unsigned* done,
                                 unsigned* ticket, cudaStream_t stream);
// group union lists -> group bitsets (a.gbits), for bundles of a caller-given partition
cudaError_t launch_gbits(const BundleLaunch& a, cudaStream_t stream);

}  // namespace qup
