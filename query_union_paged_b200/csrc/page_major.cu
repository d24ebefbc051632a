// page_major.cu -- direct KV-page union (PageWeaver, Abstract; Figure 5: the
// page-major alternative to query unions, which reuses pages across queries
// that are not grouped together and pays a reduction of cross-page partial
// outputs).  Built on the same tcgen05 union kernel as the query-union path:
//
//   items    The pages of each KV head are cut into tiles of kTileTokens tokens
//            (two 128-token steps: one per softmax warpgroup).  An item is a
//            tile and up to 128 / g queries whose page set S(i) (over the g Q
//            heads of the KV group) meets it; every page of the tile is
//            streamed once per item and each row keeps its own page mask.
//   partials The union kernel runs on the items in its partial mode: a row
//            (query, Q head) gets one partial result per tile its own TopK row
//            touches, O_t / l_t in fp32 and lse_t = m_t + log2 l_t, at slot
//            row_off[row] + (rank of the tile among the row's tiles).
//   merge    One warp per row combines its partials: O = sum_t 2^(lse_t - M)
//            O_t / sum_t 2^(lse_t - M), M = max_t lse_t; lse = M + log2 of the
//            denominator.  A row with no partial gets O = 0, lse = -inf.
//
// The item builder runs on the device in five small kernels (count, scan,
// item tiles, clear, fill); queries are placed into a tile's items by a global
// atomic counter, so which item holds a query varies from run to run, while
// every row's partials and their merge order (tile order) do not.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdint>

#include "internal.h"
#include "query_union_paged.h"

namespace qup {
namespace {

constexpr int kPmQueries = 32;  // queries per CTA in the count and fill kernels
constexpr int kPmThreads = 256;

// The row bitsets of kPmQueries queries of KV head h in shared memory:
// rows[(q * g + j) * NW + w], and their union per query uni[q * NW + w].
__device__ void pm_bitsets(const int32_t* __restrict__ topk, int Hq, int Nq, int K, int P, int NW, int g, int h, int q0,
                           int nq, uint32_t* rows, uint32_t* uni, unsigned* err) {
    for (int x = threadIdx.x; x < nq * g * NW; x += blockDim.x) rows[x] = 0u;
    for (int x = threadIdx.x; x < nq * NW; x += blockDim.x) uni[x] = 0u;
    __syncthreads();
    for (int x = threadIdx.x; x < nq * g * K; x += blockDim.x) {
        const int k = x % K, row = x / K, q = row / g, j = row % g;
        const int t = topk[((size_t)(h * g + j) * Nq + q0 + q) * K + k];
        if (t == -1) continue;
        if (t < 0 || t >= P) {
            atomicOr(err, QUP_ERR_PAGE_ID);
            continue;
        }
        atomicOr(&rows[((size_t)q * g + j) * NW + (t >> 5)], 1u << (t & 31));
        atomicOr(&uni[(size_t)q * NW + (t >> 5)], 1u << (t & 31));
    }
    __syncthreads();
}

// the tiles a bitset touches, ascending: calls f(tile) once per tile (pages per tile = Pt)
template <typename F>
__device__ __forceinline__ void for_each_tile(const uint32_t* bits, int NW, int Pt, F f) {
    int last = -1;
    for (int w = 0; w < NW; ++w) {
        uint32_t v = bits[w];
        while (v) {
            const int u = w * 32 + __ffs(v) - 1;
            v &= v - 1;
            const int t = u / Pt;
            if (t != last) {
                f(t);
                last = t;
            }
        }
    }
}

// counts: per (h, tile) the queries that meet it; per row the tiles its own TopK row touches
__global__ void __launch_bounds__(kPmThreads) pm_count_kernel(const int32_t* __restrict__ topk, int Hq, int Hkv,
                                                              int Nq, int K, int P, int NW, int Pt, int ntiles,
                                                              int32_t* __restrict__ tile_cnt,
                                                              int32_t* __restrict__ row_cnt, unsigned* err) {
    extern __shared__ uint32_t pm_smem[];
    const int g = Hq / Hkv, h = blockIdx.y, q0 = blockIdx.x * kPmQueries, nq = min(kPmQueries, Nq - q0);
    uint32_t* rows = pm_smem;
    uint32_t* uni = pm_smem + (size_t)kPmQueries * g * NW;
    pm_bitsets(topk, Hq, Nq, K, P, NW, g, h, q0, nq, rows, uni, err);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int x = warp; x < nq * (g + 1); x += kPmThreads / 32) {
        if (lane != 0) continue;
        if (x < nq) {  // the query's union: one count per tile it meets
            for_each_tile(uni + (size_t)x * NW, NW, Pt, [&](int t) { atomicAdd(&tile_cnt[h * ntiles + t], 1); });
        } else {  // a row of the query: the tiles its own TopK row touches
            const int row = x - nq, q = row / g, j = row % g;
            int c = 0;
            for_each_tile(rows + ((size_t)q * g + j) * NW, NW, Pt, [&](int) { ++c; });
            row_cnt[(size_t)(h * g + j) * Nq + q0 + q] = c;
        }
    }
}

// exclusive scan of n ints by one CTA of 1024 threads (sequential over blocks of 1024)
__device__ long long block_scan(const int32_t* in, int64_t* out_excl, long long n, bool ceil_div, int div) {
    __shared__ long long s_warp[32];
    __shared__ long long s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (long long b0 = 0; b0 < n; b0 += blockDim.x) {
        const long long i = b0 + tid;
        long long v = 0;
        if (i < n) v = ceil_div ? (in[i] + div - 1) / div : in[i];
        long long incl = v;
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            long long wv = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0;
            long long wi = wv;
            for (int o = 1; o < 32; o <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += y;
            }
            if (lane < (int)(blockDim.x >> 5)) s_warp[lane] = wi - wv;
        }
        __syncthreads();
        if (i < n) out_excl[i] = s_carry + s_warp[warp] + incl - v;
        __syncthreads();
        if (tid == blockDim.x - 1) s_carry += s_warp[warp] + incl;
        __syncthreads();
    }
    return s_carry;
}

// item bases per (h, tile) and the per-row slot offsets; n_items per head, head bases, totals
__global__ void __launch_bounds__(1024) pm_scan_kernel(const int32_t* __restrict__ tile_cnt,
                                                       const int32_t* __restrict__ row_cnt, int Hq, int Hkv, int Nq,
                                                       int ntiles, int MQ, int64_t* __restrict__ tile_base,
                                                       int64_t* __restrict__ row_off, int32_t* __restrict__ n_items,
                                                       int64_t* __restrict__ totals, long long item_cap,
                                                       long long slot_cap, unsigned* err) {
    long long acc = 0;
    for (int h = 0; h < Hkv; ++h) {
        const long long n = block_scan(tile_cnt + (size_t)h * ntiles, tile_base + (size_t)h * ntiles, ntiles, true, MQ);
        if (threadIdx.x == 0) {
            n_items[h] = (int32_t)min(n, item_cap);
            totals[2 + h] = acc;  // flat index of the head's first item
        }
        if (n > item_cap && threadIdx.x == 0) atomicOr(err, QUP_ERR_CAPACITY);
        acc += min(n, item_cap);
        __syncthreads();
    }
    const long long nrows = (long long)Hq * Nq;
    const long long slots = block_scan(row_cnt, row_off, nrows, false, 1);
    if (threadIdx.x == 0) {
        row_off[nrows] = slots;
        totals[0] = acc;
        totals[1] = slots;
        if (slots > slot_cap) atomicOr(err, QUP_ERR_CAPACITY);
    }
}

// every item: its tile's pages as its union, cleared query slots, row slots and masks
__global__ void pm_clear_kernel(const int64_t* __restrict__ tile_base, const int32_t* __restrict__ tile_cnt,
                                const int32_t* __restrict__ n_items, const int64_t* __restrict__ totals, int Hkv,
                                int ntiles, int Pt, int P, int MQ, long long item_cap, int32_t* __restrict__ item_ptr,
                                int32_t* __restrict__ item_pages, uint32_t* __restrict__ item_mask,
                                int32_t* __restrict__ item_qid, int32_t* __restrict__ item_slot,
                                int32_t* __restrict__ item_order) {
    const int h = blockIdx.y;
    const long long head0 = totals[2 + h];
    const int ni = n_items[h];
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const long long b = tile_base[(size_t)h * ntiles + t];
        const int cnt = tile_cnt[h * ntiles + t];
        const int nit = (cnt + MQ - 1) / MQ;
        for (int k = 0; k < nit; ++k) {
            const long long bi = b + k;
            if (bi >= ni) break;
            const long long fi = head0 + bi;  // flat item
            for (int x = threadIdx.x; x < Pt; x += blockDim.x) {
                const int u = t * Pt + x;
                item_pages[fi * Pt + x] = u < P ? u : 0;  // past the last page: page 0, selected by no row
                for (int wd = 0; wd < 4; ++wd) item_mask[(fi * Pt + x) * 4 + wd] = 0u;
            }
            for (int x = threadIdx.x; x < MQ; x += blockDim.x) item_qid[((size_t)h * item_cap + bi) * MQ + x] = -1;
            for (int x = threadIdx.x; x < 128; x += blockDim.x) item_slot[fi * 128 + x] = -1;
            if (threadIdx.x == 0) {
                item_ptr[(size_t)h * (item_cap + 1) + bi] = (int32_t)(fi * Pt);
                item_order[fi] = (int32_t)fi;
            }
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        // the union of the head's last item ends where the next item would start
        item_ptr[(size_t)h * (item_cap + 1) + ni] = (int32_t)((head0 + ni) * Pt);
    }
}

// place every (query, tile) of a KV head into an item: query slot, row masks, row slots
__global__ void __launch_bounds__(kPmThreads) pm_fill_kernel(
    const int32_t* __restrict__ topk, int Hq, int Hkv, int Nq, int K, int P, int NW, int Pt, int ntiles, int MQ,
    const int64_t* __restrict__ tile_base, int32_t* __restrict__ tile_fill, const int64_t* __restrict__ row_off,
    const int32_t* __restrict__ n_items, const int64_t* __restrict__ totals, long long item_cap,
    int32_t* __restrict__ item_qid, uint32_t* __restrict__ item_mask, int32_t* __restrict__ item_slot,
    unsigned* err) {
    extern __shared__ uint32_t pm_smem[];
    const int g = Hq / Hkv, h = blockIdx.y, q0 = blockIdx.x * kPmQueries, nq = min(kPmQueries, Nq - q0);
    uint32_t* rows = pm_smem;
    uint32_t* uni = pm_smem + (size_t)kPmQueries * g * NW;
    pm_bitsets(topk, Hq, Nq, K, P, NW, g, h, q0, nq, rows, uni, err);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long head0 = totals[2 + h];
    const int ni = n_items[h];
    for (int q = warp; q < nq; q += kPmThreads / 32) {
        if (lane != 0) continue;
        const int i = q0 + q;
        int rank[32];  // per head of the group: tiles of its own row seen so far (g <= 32)
        for (int j = 0; j < g; ++j) rank[j] = 0;
        for_each_tile(uni + (size_t)q * NW, NW, Pt, [&](int t) {
            const int pos = atomicAdd(&tile_fill[h * ntiles + t], 1);
            const long long bi = tile_base[(size_t)h * ntiles + t] + pos / MQ;
            const int m = pos % MQ;
            if (bi >= ni) return;  // capacity exceeded (reported by the scan)
            const long long fi = head0 + bi;
            item_qid[((size_t)h * item_cap + bi) * MQ + m] = i;
            for (int j = 0; j < g; ++j) {
                const uint32_t* rb = rows + ((size_t)q * g + j) * NW;
                const int r = m * g + j;
                bool any = false;
                for (int x = 0; x < Pt; ++x) {
                    const int u = t * Pt + x;
                    if (u < P && ((rb[u >> 5] >> (u & 31)) & 1u)) {
                        atomicOr(&item_mask[(fi * Pt + x) * 4 + (r >> 5)], 1u << (r & 31));
                        any = true;
                    }
                }
                if (any) item_slot[fi * 128 + r] = (int32_t)(row_off[(size_t)(h * g + j) * Nq + i] + rank[j]++);
            }
        });
    }
}

// one warp per row: merge its partials by lse
__global__ void pm_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                const int64_t* __restrict__ row_off, int Hq, int Nq, int q_bf16, void* __restrict__ O,
                                float* __restrict__ lse) {
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (long long)Hq * Nq) return;
    const int h = (int)(row / Nq), i = (int)(row % Nq);
    const long long s0 = row_off[row], s1 = row_off[row + 1];
    float M = -__int_as_float(0x7f800000);
    for (long long s = s0; s < s1; ++s) M = fmaxf(M, part_lse[s]);
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, den = 0.f;
    if (M > -__int_as_float(0x7f800000)) {
        for (long long s = s0; s < s1; ++s) {
            const float wgt = exp2f(part_lse[s] - M);
            const float4 v = reinterpret_cast<const float4*>(part_o + s * kHeadDim)[lane];
            acc[0] += wgt * v.x;
            acc[1] += wgt * v.y;
            acc[2] += wgt * v.z;
            acc[3] += wgt * v.w;
            den += wgt;
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const size_t oi = ((size_t)i * Hq + h) * kHeadDim + 4 * lane;
    if (q_bf16) {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(O) + oi;
        o[0] = __float2bfloat16_rn(acc[0] * inv);
        o[1] = __float2bfloat16_rn(acc[1] * inv);
        o[2] = __float2bfloat16_rn(acc[2] * inv);
        o[3] = __float2bfloat16_rn(acc[3] * inv);
    } else {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(O) + oi);
        *o = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    }
    if (lse && lane == 0)
        lse[(size_t)i * Hq + h] = den > 0.f ? (M + __log2f(den)) * 0.69314718055994531f : -__int_as_float(0x7f800000);
}

}  // namespace

size_t page_major_build_smem(int g, int NW) { return 4u * (size_t)kPmQueries * (g + 1) * NW; }

cudaError_t launch_page_major_build(const int32_t* topk, int Hq, int Hkv, int Nq, int K, int P, int NW, int Pt,
                                    int ntiles, int MQ, long long item_cap, long long slot_cap, int32_t* tile_cnt,
                                    int32_t* tile_fill, int32_t* row_cnt, int64_t* tile_base, int64_t* row_off,
                                    int64_t* totals, int32_t* n_items, int32_t* item_ptr, int32_t* item_pages,
                                    uint32_t* item_mask, int32_t* item_qid, int32_t* item_slot, int32_t* item_order,
                                    unsigned* err, cudaStream_t st) {
    const int g = Hq / Hkv;
    const size_t smem = page_major_build_smem(g, NW);
    cudaError_t e;
    if ((e = cudaMemsetAsync(tile_cnt, 0, sizeof(int32_t) * (size_t)Hkv * ntiles, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(tile_fill, 0, sizeof(int32_t) * (size_t)Hkv * ntiles, st)) != cudaSuccess) return e;
    if ((e = ensure_smem_attr((const void*)pm_count_kernel, smem)) != cudaSuccess) return e;
    if ((e = ensure_smem_attr((const void*)pm_fill_kernel, smem)) != cudaSuccess) return e;
    const dim3 grid((Nq + kPmQueries - 1) / kPmQueries, Hkv);
    pm_count_kernel<<<grid, kPmThreads, smem, st>>>(topk, Hq, Hkv, Nq, K, P, NW, Pt, ntiles, tile_cnt, row_cnt, err);
    pm_scan_kernel<<<1, 1024, 0, st>>>(tile_cnt, row_cnt, Hq, Hkv, Nq, ntiles, MQ, tile_base, row_off, n_items, totals,
                                       item_cap, slot_cap, err);
    pm_clear_kernel<<<dim3(std::min(ntiles, 1024), Hkv), 128, 0, st>>>(tile_base, tile_cnt, n_items, totals, Hkv,
                                                                       ntiles, Pt, P, MQ, item_cap, item_ptr,
                                                                       item_pages, item_mask, item_qid, item_slot,
                                                                       item_order);
    pm_fill_kernel<<<grid, kPmThreads, smem, st>>>(topk, Hq, Hkv, Nq, K, P, NW, Pt, ntiles, MQ, tile_base, tile_fill,
                                                   row_off, n_items, totals, item_cap, item_qid, item_mask, item_slot,
                                                   err);
    return cudaGetLastError();
}

cudaError_t launch_page_major_merge(const float* part_o, const float* part_lse, const int64_t* row_off, int Hq, int Nq,
                                    int q_bf16, void* O, float* lse, cudaStream_t st) {
    const long long rows = (long long)Hq * Nq;
    if (rows == 0) return cudaSuccess;
    pm_merge_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(part_o, part_lse, row_off, Hq, Nq, q_bf16, O, lse);
    return cudaGetLastError();
}

}  // namespace qup
