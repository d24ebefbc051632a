// select.h -- the proxy-query page selector's limits and launcher (select.cu), for the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace qup {

// At most kMaxSelCand candidates per group, at most kMaxSelPages logical pages (one CTA's shared
// memory holds all of a group's page keys), index width at most kMaxSelDim.
constexpr int kMaxSelCand = 256;
constexpr int kMaxSelPages = 8192;
constexpr int kMaxSelDim = 512;

// dynamic shared memory of one selector CTA (esize: 2 for bf16, 4 for fp32 index vectors)
size_t pivot_select_smem(int num_logical_pages, int d, int esize, int n_cand);

cudaError_t launch_pivot_select(const void* q_idx, const void* page_key, bool bf16, const int32_t* q_pos, int Nq,
                                int Hkv, int g, int d, int P, int T, int G, int n_cand, int K, bool refine,
                                int32_t* topk, cudaStream_t stream);

}  // namespace qup
