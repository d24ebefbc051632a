// select.cu -- proxy-query page selection: the upstream step that produces each
// query's TopK pages for the grouping call (PIVOT: Efficient Query-Group
// Indexing for Token-Level Sparse Attention, Abstract).
//
// Queries are cut into fixed groups of consecutive IDs.  Per (KV head, group)
// one CTA: the group's indexer queries are averaged into a proxy query, the
// proxy scores every page the group's last query can see (one scan for the
// whole group instead of one per query), and a radix select over the (score,
// page) keys takes the n_cand best as the candidate set (sorted for Reuse).  Each query then takes its
// Ksel pages from the candidates it can see: PIVOT-Refine re-scores them with
// its own indexer query, PIVOT-Reuse keeps the proxy's order.  A page is the
// selection unit and has one indexer key per KV head; a score is a dot product.
//
// The arithmetic is float32 with explicitly rounded operations in a fixed
// order (proxy: queries added in ID order, then divided by the group size;
// score: products added in element order), so the ranking, an integer result,
// does not depend on how a compiler would contract or reorder it: order by
// score (higher first), equal scores by page ID (lower first).  Rows are
// padded with -1 and copied to the g query heads of the KV group.
#include <cstdint>

#include "internal.h"
#include "select.h"
#include "query_union_paged.h"

namespace qup {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kCandPerLane = kMaxSelCand / 32;

// element t of a row of bf16 or fp32 values, widened to fp32 (exact)
__device__ __forceinline__ float elem(const void* base, size_t idx, bool bf16) {
    if (bf16) return __uint_as_float((uint32_t)static_cast<const uint16_t*>(base)[idx] << 16);
    return static_cast<const float*>(base)[idx];
}

// v . row, row = d values at base[off ..] (global or shared memory): products and sums rounded one
// by one, in element order.  Four 16-byte loads are in flight at a time.
__device__ __forceinline__ float dot_seq(const float* v, const void* base, size_t off, int d, bool bf16) {
    float acc = 0.f;
    if (bf16) {
        const uint4* r = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off);
        const float4* v4 = reinterpret_cast<const float4*>(v);
#pragma unroll 4
        for (int t0 = 0; t0 < d; t0 += 8) {
            const uint4 w = r[t0 / 8];
            const float4 va = v4[t0 / 4], vb = v4[t0 / 4 + 1];
            acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(w.x << 16), va.x));
            acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(w.x & 0xffff0000u), va.y));
            acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(w.y << 16), va.z));
            acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(w.y & 0xffff0000u), va.w));
            acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(w.z << 16), vb.x));
            acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(w.z & 0xffff0000u), vb.y));
            acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(w.w << 16), vb.z));
            acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(w.w & 0xffff0000u), vb.w));
        }
    } else {
        const float4* r = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
        const float4* v4 = reinterpret_cast<const float4*>(v);
#pragma unroll 4
        for (int t0 = 0; t0 < d; t0 += 4) {
            const float4 w = r[t0 / 4], va = v4[t0 / 4];
            acc = __fadd_rn(acc, __fmul_rn(w.x, va.x));
            acc = __fadd_rn(acc, __fmul_rn(w.y, va.y));
            acc = __fadd_rn(acc, __fmul_rn(w.z, va.z));
            acc = __fadd_rn(acc, __fmul_rn(w.w, va.w));
        }
    }
    return acc;
}

// Sort key of (score, page): larger key = higher score, then lower page.  -0 counts as +0; every
// real key is > 0, so 0 marks an empty entry.
__device__ __forceinline__ uint64_t rank_key(float s, int page) {
    uint32_t u = __float_as_uint(s);
    if ((u << 1) == 0u) u = 0u;
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)ord << 32) | (uint64_t)(0xffffffffu - (uint32_t)page);
}
__device__ __forceinline__ int key_page(uint64_t k) { return (int)(0xffffffffu - (uint32_t)k); }

// 64-bit maximum over the warp
__device__ __forceinline__ uint64_t warp_max64(uint64_t k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, k, o);
        k = y > k ? y : k;
    }
    return k;
}

__global__ void __launch_bounds__(kSelThreads) pivot_select_kernel(
    const void* __restrict__ q_idx, const void* __restrict__ page_key, int bf16i, const int32_t* __restrict__ q_pos,
    int Nq, int Hkv, int g, int d, int P, int T, int G, int n_cand, int K, int refine, int Lpad,
    int32_t* __restrict__ topk) {
    extern __shared__ uint64_t sel_sm[];
    float* proxy = reinterpret_cast<float*>(sel_sm);                  // [d]; d % 4 == 0 keeps what follows
    float* qv = proxy + d;                                            // [kSelWarps][d]   16-byte aligned
    uint64_t* keys = reinterpret_cast<uint64_t*>(qv + (size_t)kSelWarps * d);  // [P] the visible pages' keys
    uint64_t* cand = keys + ((P + 1) & ~1);                           // [Lpad <= kMaxSelCand] the candidates
    uint4* ckey = reinterpret_cast<uint4*>(cand + kMaxSelCand);        // [n_cand][row] their key rows
    __shared__ int hist[256];
    __shared__ unsigned long long s_thr;
    __shared__ int s_rem, s_cnt;
    const bool bf16 = bf16i != 0;
    const int h = blockIdx.y, g0 = blockIdx.x * G, n = min(G, Nq - g0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (n <= 0) return;
    // ---- proxy query: the group's indexer queries added in ID order, then divided by n
    for (int t = tid; t < d; t += kSelThreads) {
        float acc = 0.f;
        for (int i = g0; i < g0 + n; ++i) acc = __fadd_rn(acc, elem(q_idx, ((size_t)i * Hkv + h) * d + t, bf16));
        proxy[t] = __fdiv_rn(acc, (float)n);
    }
    // pages the group's last query can see
    int last = -1;
    for (int i = g0; i < g0 + n; ++i) last = max(last, q_pos[i]);
    const int lim = last < 0 ? 0 : min(P, last / T + 1);
    __syncthreads();
    // ---- one scan of the visible pages by the proxy
    for (int p = tid; p < lim; p += kSelThreads)
        keys[p] = rank_key(dot_seq(proxy, page_key, ((size_t)p * Hkv + h) * d, d, bf16), p);
    const int nc = min(n_cand, lim);  // candidates: the nc largest keys (all distinct: pages are)
    // ---- the nc-th largest key by a radix select, 8 bits at a time from the top: after byte k the
    // threshold's top k+1 bytes are known, and s_rem keys sharing them are still to be taken
    if (tid == 0) {
        s_thr = 0ull;
        s_rem = nc;
        s_cnt = 0;
    }
    __syncthreads();
    for (int byte = 7; byte >= 0 && nc < lim; --byte) {
        hist[tid] = 0;  // kSelThreads == 256 bins
        __syncthreads();
        const unsigned long long pre = s_thr;
        const int sh = 8 * byte;
        for (int p = tid; p < lim; p += kSelThreads) {
            const uint64_t k = keys[p];
            if (byte == 7 || (k >> (sh + 8)) == (pre >> (sh + 8))) atomicAdd(&hist[(k >> sh) & 255u], 1);
        }
        __syncthreads();
        if (warp == 0) {  // lane l holds bins 255-8l .. 248-8l, counted from the top
            int c[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                c[e] = hist[255 - 8 * lane - e];
                tot += c[e];
            }
            int above = tot;  // exclusive prefix over the lanes above this one
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, above, o);
                if (lane >= o) above += y;
            }
            above -= tot;
            const int rem = s_rem;
            int run = above;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (run < rem && run + c[e] >= rem) {
                    s_thr = pre | ((unsigned long long)(255 - 8 * lane - e) << sh);
                    s_rem = rem - run;
                }
                run += c[e];
            }
        }
        __syncthreads();
    }
    // ---- the candidates: every key >= the threshold (all keys when they are at most n_cand)
    {
        const unsigned long long thr = nc < lim ? s_thr : 0ull;
        for (int p = tid; p < lim; p += kSelThreads) {
            const uint64_t k = keys[p];
            if (k >= thr) cand[atomicAdd(&s_cnt, 1)] = k;
        }
    }
    __syncthreads();
    if (!refine) {  // Reuse needs the proxy's order: sort the candidates, descending
        for (int x = nc + tid; x < Lpad; x += kSelThreads) cand[x] = 0ull;
        __syncthreads();
        for (int k = 2; k <= Lpad; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int x = tid; x < Lpad; x += kSelThreads) {
                    const int y = x ^ j;
                    if (y > x) {
                        const uint64_t a = cand[x], b = cand[y];
                        if ((x & k) == 0 ? a < b : a > b) {
                            cand[x] = b;
                            cand[y] = a;
                        }
                    }
                }
                __syncthreads();
            }
        }
    }
    // ---- Refine re-scores the candidates with every query of the group: their key rows are read
    // from global memory once, with coalesced loads, into shared memory (same order as cand)
    const int rowv = d * (bf16 ? 2 : 4) / 16;  // 16-byte chunks per key row
    if (refine) {
        for (int x = tid; x < nc * rowv; x += kSelThreads) {
            const int c = x / rowv, j = x - c * rowv;
            const int pg = key_page(cand[c]);
            ckey[x] = __ldg(reinterpret_cast<const uint4*>(static_cast<const char*>(page_key) +
                                                           ((size_t)pg * Hkv + h) * d * (bf16 ? 2 : 4)) + j);
        }
        __syncthreads();
    }
    // ---- each query's pages: one warp per query
    float* my_q = qv + (size_t)warp * d;
    for (int i = g0 + warp; i < g0 + n; i += kSelWarps) {
        const int vis = q_pos[i] < 0 ? -1 : q_pos[i] / T;  // pages <= vis are visible
        int32_t* row0 = topk + ((size_t)(h * g) * Nq + i) * K;
        int filled = 0;
        if (!refine) {  // Reuse: the visible candidates in the proxy's order
            for (int c0 = 0; c0 < nc && filled < K; c0 += 32) {
                const int c = c0 + lane;
                const int pg = c < nc ? key_page(cand[c]) : -1;
                const bool ok = c < nc && pg <= vis;
                const unsigned bal = __ballot_sync(0xffffffffu, ok);
                const int at = filled + __popc(bal & ((1u << lane) - 1u));
                if (ok && at < K)
                    for (int j = 0; j < g; ++j) row0[(size_t)j * Nq * K + at] = pg;
                filled += __popc(bal);
            }
            filled = min(filled, K);
        } else {  // Refine: the visible candidates re-scored with the query's own indexer query
            for (int t = lane; t < d; t += 32) my_q[t] = elem(q_idx, ((size_t)i * Hkv + h) * d + t, bf16);
            __syncwarp();
            uint64_t mine[kCandPerLane];
#pragma unroll
            for (int e = 0; e < kCandPerLane; ++e) {
                const int c = lane + 32 * e;
                const int pg = c < nc ? key_page(cand[c]) : -1;
                mine[e] = (c < nc && pg <= vis)
                              ? rank_key(dot_seq(my_q, ckey + (size_t)c * rowv, 0, d, bf16), pg)
                              : 0ull;
            }
            for (; filled < K; ++filled) {
                uint64_t best = 0ull;
#pragma unroll
                for (int e = 0; e < kCandPerLane; ++e) best = mine[e] > best ? mine[e] : best;
                best = warp_max64(best);
                if (best == 0ull) break;
#pragma unroll
                for (int e = 0; e < kCandPerLane; ++e)
                    if (mine[e] == best) mine[e] = 0ull;  // keys are distinct (pages are)
                if (lane < g) row0[(size_t)lane * Nq * K + filled] = key_page(best);
            }
            __syncwarp();
        }
        for (int x = filled + lane; x < K; x += 32)
            for (int j = 0; j < g; ++j) row0[(size_t)j * Nq * K + x] = -1;
    }
}

}  // namespace

size_t pivot_select_smem(int num_logical_pages, int d, int esize, int n_cand) {
    return (size_t)d * 4 * (1 + kSelWarps) + (size_t)((num_logical_pages + 1) & ~1) * 8 +
           (size_t)kMaxSelCand * 8 + (size_t)n_cand * d * esize;
}

cudaError_t launch_pivot_select(const void* q_idx, const void* page_key, bool bf16, const int32_t* q_pos, int Nq,
                                int Hkv, int g, int d, int P, int T, int G, int n_cand, int K, bool refine,
                                int32_t* topk, cudaStream_t stream) {
    if (Nq == 0 || Hkv == 0) return cudaSuccess;
    int Lpad = 1;  // the candidates' sort width
    while (Lpad < n_cand) Lpad <<= 1;
    const size_t smem = pivot_select_smem(P, d, bf16 ? 2 : 4, n_cand);
    cudaError_t e = ensure_smem_attr((const void*)pivot_select_kernel, smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((Nq + G - 1) / G, Hkv);
    pivot_select_kernel<<<grid, kSelThreads, smem, stream>>>(q_idx, page_key, bf16 ? 1 : 0, q_pos, Nq, Hkv, g, d, P, T,
                                                             G, n_cand, K, refine ? 1 : 0, Lpad, topk);
    return cudaGetLastError();
}

}  // namespace qup
