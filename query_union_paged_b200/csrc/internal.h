// internal.h -- declarations shared by the host layer and the kernel files.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace qup {

constexpr int kStepTok = 128;   // union tokens per pipeline step (MMA M of S^T, K of PV)
constexpr int kHeadDim = 128;
constexpr int kMaxPPS = 8;      // pages per step at T = 16
constexpr int kMaxStages = 16;

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
    void* O;
    float* lse;
    unsigned* err;
    long long cap_union;
    int num_logical_pages, P_phys, T, kv_len, Hq, Hkv, Nq, g;
    float scale_log2;  // softmax_scale * log2(e)
    int nsk, nsv;  // slots of the K ring and of the V ring
    unsigned long long wait_limit_ns;
    int dbg_skip_stage;
};

// dynamic shared memory of the attention kernel for (element size, K slots, V slots, KV heads),
// and one K or V tile (one ring slot)
size_t attn_smem_bytes(int es, int nsk, int nsv, int Hkv);
size_t attn_tile_bytes(int es);

cudaError_t launch_union_attn(int es, int T, const CUtensorMap& tmK, const CUtensorMap& tmV,
                              const AttnParams& p, int grid, size_t smem, cudaStream_t stream);

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

}  // namespace qup
