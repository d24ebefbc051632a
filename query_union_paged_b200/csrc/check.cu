// check.cu -- checked mode of the attention call: every bundle row's page mask
// must be exactly the set of pages of its own TopK row.
//
// The attention kernel takes each query's support from the bundles' row masks
// (PageWeaver, Figure 2: the union decides which pages are loaded, every
// selected edge of a query is kept and no other).  This kernel checks that
// contract against topk before the attention kernel runs: for each bundle row
// with a query ID, a mask bit is set exactly for the union entries whose page
// is in that row (as a set: duplicates and -1 padding dropped), and the number
// of set bits equals the number of distinct valid pages of the row (so no page
// of the row is missing from the bundle union).  Rows without a query carry no
// bits.  A mismatch raises QUP_ERR_GROUP, a TopK entry outside the page range
// QUP_ERR_PAGE_ID; nothing else is written.
#include <algorithm>
#include <cstdint>

#include "internal.h"
#include "query_union_paged.h"

namespace qup {

namespace {

constexpr int kCheckThreads = 128;  // thread = bundle row

__global__ void __launch_bounds__(kCheckThreads)
    check_support_kernel(const int32_t* __restrict__ topk, int K, int Hkv, int Nq, int g, int P,
                         const int32_t* __restrict__ n_bundles, const int32_t* __restrict__ bunion_ptr,
                         const int32_t* __restrict__ bunion_pages, const uint32_t* __restrict__ bunion_mask,
                         const int32_t* __restrict__ bundle_qid, long long cap, unsigned* err) {
    const int h = blockIdx.y, r = threadIdx.x;
    const int nb = n_bundles[h];
    if (nb < 0 || nb > Nq) {
        if (r == 0) atomicOr(err, QUP_ERR_GROUP);
        return;
    }
    const int MQ = kCheckThreads / g;
    for (int b = blockIdx.x; b < nb; b += gridDim.x) {
        const size_t bp = (size_t)h * (Nq + 1) + b;
        const int ub = bunion_ptr[bp], ue = bunion_ptr[bp + 1];
        if (ub < 0 || ue < ub || (long long)ue > cap) {
            if (r == 0) atomicOr(err, QUP_ERR_GROUP);
            continue;
        }
        const int qid = bundle_qid[((size_t)h * Nq + b) * MQ + r / g];
        unsigned bad = 0;
        if (qid >= Nq || qid < -1) {
            bad |= QUP_ERR_GROUP;
        } else if (qid < 0) {
            for (int e = ub; e < ue; ++e)
                if ((bunion_mask[(size_t)e * 4 + r / 32] >> (r & 31)) & 1u) bad |= QUP_ERR_GROUP;
        } else {
            const int32_t* row = topk + ((size_t)(h * g + r % g) * Nq + qid) * K;
            int distinct = 0;
            for (int k = 0; k < K; ++k) {
                const int t = row[k];
                if (t < 0) continue;
                if (t >= P) {
                    bad |= QUP_ERR_PAGE_ID;
                    continue;
                }
                bool dup = false;
                for (int j = 0; j < k; ++j) dup |= row[j] == t;
                distinct += dup ? 0 : 1;
            }
            int bits = 0;
            for (int e = ub; e < ue; ++e) {
                const bool bit = (bunion_mask[(size_t)e * 4 + r / 32] >> (r & 31)) & 1u;
                if (!bit) {
                    // a page of the row may still be left out only if it is not in the union at all,
                    // which the count below catches; a clear bit for a page of the row is caught here
                    const int u = bunion_pages[e];
                    for (int k = 0; k < K; ++k)
                        if (row[k] == u) bad |= QUP_ERR_GROUP;
                    continue;
                }
                ++bits;
                const int u = bunion_pages[e];
                bool in_row = false;
                for (int k = 0; k < K; ++k) in_row |= row[k] == u;
                if (!in_row || u < 0) bad |= QUP_ERR_GROUP;
            }
            if (bits != distinct) bad |= QUP_ERR_GROUP;
        }
        if (bad) atomicOr(err, bad);
    }
}

}  // namespace

cudaError_t launch_check_support(const int32_t* topk, int K, int Hkv, int Nq, int g, int P, const int32_t* n_bundles,
                                 const int32_t* bunion_ptr, const int32_t* bunion_pages,
                                 const uint32_t* bunion_mask, const int32_t* bundle_qid, long long cap,
                                 unsigned* err, int sms, cudaStream_t stream) {
    if (Nq == 0 || Hkv == 0) return cudaSuccess;
    const int gx = std::min(Nq, std::max(1, 4 * sms / Hkv));
    check_support_kernel<<<dim3(gx, Hkv), kCheckThreads, 0, stream>>>(topk, K, Hkv, Nq, g, P, n_bundles, bunion_ptr,
                                                                     bunion_pages, bunion_mask, bundle_qid, cap, err);
    return cudaGetLastError();
}

}  // namespace qup
