// batch.cu -- batched (varlen) requests: several sequences, each with its own
// page table, cache length and chunk of queries, in one grouping call and one
// attention call.
//
// The requests are laid end to end in one logical page space: the pages of
// request r are the global logical pages page_ptr[r] .. page_ptr[r+1) (the
// caller's per-request page tables concatenated), and its queries are the
// batch rows q_ptr[r] .. q_ptr[r+1).  A query's TopK IDs are local to its
// request; qup_batch_prepare rebases them to global IDs, so the grouping call
// runs unchanged on the whole batch (a group may hold queries of two requests
// only at a window that straddles them; their pages are disjoint, so each
// query still keeps exactly its own support).  Token slot o of global page u
// has global position u * T + o, so a query of request r at local position q
// sees global positions < page_ptr[r] * T + min(q + 1, kv_len[r]) (its q_end),
// and page u holds page_len[u] valid tokens.  The attention kernel reads these
// two arrays instead of one kv_len.
#include <cstdint>

#include "internal.h"
#include "query_union_paged.h"

namespace qup {
namespace {

// index of the segment of a prefix array ptr[0..R] that holds x (ptr ascending), -1 if none
__device__ __forceinline__ int find_segment(const int32_t* ptr, int R, int x) {
    if (R <= 0 || x < ptr[0] || x >= ptr[R]) return -1;
    int lo = 0, hi = R - 1;  // the last r with ptr[r] <= x
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ptr[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__global__ void batch_queries_kernel(const int32_t* __restrict__ topk, const int32_t* __restrict__ q_pos, int Hq,
                                     int Nq, int K, int T, int R, const int32_t* __restrict__ q_ptr,
                                     const int32_t* __restrict__ page_ptr, const int32_t* __restrict__ kv_len,
                                     int32_t* __restrict__ topk_global, int32_t* __restrict__ q_end, unsigned* err) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= Nq) return;
    const int r = find_segment(q_ptr, R, i);
    int base = 0, np = 0, vis = 0;
    if (r < 0) {
        atomicOr(err, QUP_ERR_GROUP);  // a batch row outside every request: it attends nothing
    } else {
        base = page_ptr[r];
        np = page_ptr[r + 1] - base;
        const int len = kv_len[r];
        if (np < 0 || len < 0 || (long long)len > (long long)np * T) {
            atomicOr(err, QUP_ERR_GROUP);
            np = 0;
        } else {
            vis = max(0, min(q_pos[i] + 1, len));
        }
    }
    q_end[i] = base * T + vis;
    for (int h = 0; h < Hq; ++h) {
        const int32_t* src = topk + ((size_t)h * Nq + i) * K;
        int32_t* dst = topk_global + ((size_t)h * Nq + i) * K;
        for (int k = 0; k < K; ++k) {
            const int t = src[k];
            int out = -1;
            if (t != -1) {
                if (t < 0 || t >= np) atomicOr(err, QUP_ERR_PAGE_ID);
                else out = base + t;
            }
            dst[k] = out;
        }
    }
}

__global__ void batch_pages_kernel(int total_pages, int T, int R, const int32_t* __restrict__ page_ptr,
                                   const int32_t* __restrict__ kv_len, int32_t* __restrict__ page_len) {
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= total_pages) return;
    const int r = find_segment(page_ptr, R, u);
    int valid = 0;
    if (r >= 0) valid = max(0, min(T, kv_len[r] - (u - page_ptr[r]) * T));
    page_len[u] = valid;
}

}  // namespace

cudaError_t launch_batch_prepare(const int32_t* topk, const int32_t* q_pos, int Hq, int Nq, int K, int T, int R,
                                 const int32_t* q_ptr, const int32_t* page_ptr, const int32_t* kv_len, int total_pages,
                                 int32_t* topk_global, int32_t* q_end, int32_t* page_len, unsigned* err,
                                 cudaStream_t stream) {
    if (Nq > 0) {
        batch_queries_kernel<<<(Nq + 127) / 128, 128, 0, stream>>>(topk, q_pos, Hq, Nq, K, T, R, q_ptr, page_ptr, kv_len,
                                                                   topk_global, q_end, err);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (total_pages > 0) {
        batch_pages_kernel<<<(total_pages + 255) / 256, 256, 0, stream>>>(total_pages, T, R, page_ptr, kv_len, page_len);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace qup
