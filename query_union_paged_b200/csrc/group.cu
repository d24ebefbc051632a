// group.cu -- bounded page-affinity grouping (PageWeaver, Abstract: a GPU
// search of bounded cost turns selected-page affinity into query-ID lists;
// Figure 2: logical page visits and masked query-page slots).
//
// Three kernels, all deterministic:
//   1. rowbits: one warp per TopK row builds the row's page bitset (duplicates
//      and -1 padding vanish; out-of-range IDs raise QUP_ERR_PAGE_ID).
//   2. greedy:  one CTA per (window, KV head).  The g rows of each query are
//      ORed into S(i) in shared memory; warp 0 then runs the greedy: seed =
//      smallest unassigned query, add the candidate with the fewest pages
//      outside the union (ties to the smallest ID) until max_group members or
//      the window is exhausted.  The argmin is one warp reduction of the
//      packed key (value << 9 | local_id), value = pick_value: the new page
//      count for groups; for bundles (the same kernels run on group unions)
//      new - 2 * shared pages.
//   3. emit:    one CTA per (window, KV head) sums the union sizes of all
//      earlier windows for its absolute offset, then one warp per group
//      writes the sorted union pages and per-page row masks from the bitsets.
#include <algorithm>
#include <cstdint>

#include "ptx.cuh"
#include "internal.h"
#include "query_union_paged.h"

namespace qup {

__global__ void __launch_bounds__(256) grp_rowbits_kernel(const int32_t* __restrict__ topk, int Hq,
                                                           int Hkv, int Nq, int K, int P, int NW,
                                                           uint32_t* __restrict__ rowbits,
                                                           int64_t* __restrict__ counters,
                                                           unsigned* err) {
    extern __shared__ uint32_t sm_rb[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* bits = sm_rb + warp * NW;
    if (blockIdx.x == 0)
        for (int x = threadIdx.x; x < Hkv * 4; x += blockDim.x) counters[x] = 0;
    const int g = Hq / Hkv;
    const long long nrows = (long long)Hq * Nq;
    for (long long row = (long long)blockIdx.x * 8 + warp; row < nrows; row += (long long)gridDim.x * 8) {
        const int hq = (int)(row / Nq), i = (int)(row % Nq);
        for (int w = lane; w < NW; w += 32) bits[w] = 0;
        __syncwarp();
        const int32_t* tr = topk + row * K;
        for (int k = lane; k < K; k += 32) {
            const int p = tr[k];
            if (p == -1) continue;
            if (p < 0 || p >= P) {
                atomicOr(err, QUP_ERR_PAGE_ID);
                continue;
            }
            atomicOr(&bits[p >> 5], 1u << (p & 31));
        }
        __syncwarp();
        const int h = hq / g, j = hq % g;
        uint32_t* dst = rowbits + (((size_t)h * Nq + i) * g + j) * NW;
        for (int w = lane; w < NW; w += 32) dst[w] = bits[w];
        __syncwarp();
    }
}

// Greedy packing of the items of one KV head inside one window.  Items are
// queries (sets = the g TopK rows of the query, ORed) or groups (sets = the
// group union bitset); n_items_dev == nullptr means Nq items per head.
__global__ void __launch_bounds__(128) grp_greedy_kernel(const uint32_t* __restrict__ rowbits, int sets_per_item,
                                                          int Hkv, int Nq, const int32_t* __restrict__ n_items_dev,
                                                          int NW, int max_group, int W,
                                                          int nwin, int32_t* __restrict__ group_ptr,
                                                          int32_t* __restrict__ members,
                                                          int32_t* __restrict__ n_groups,
                                                          int32_t* __restrict__ ws_usize,
                                                          int32_t* __restrict__ ws_wtot,
                                                          int32_t* __restrict__ ws_wcnt,
                                                          int64_t* __restrict__ out_count, int bundle) {
    extern __shared__ uint32_t sm_gr[];
    const int NWp = NW | 1;  // odd row pitch: lanes reading different queries hit different banks
    uint32_t* S = sm_gr;
    uint32_t* U = S + (size_t)W * NWp;
    int* ssize = reinterpret_cast<int*>(U + NWp);
    const int w = blockIdx.x, h = blockIdx.y, g = sets_per_item;
    const int n_items = n_items_dev ? n_items_dev[h] : Nq;
    const int w0 = w * W, nw = max(0, min(W, n_items - w0));
    if (nw == 0) {  // window past the head's last item: contributes nothing
        if (threadIdx.x == 0) {
            const int f = h * nwin + w;
            ws_wtot[f] = 0;
            ws_wcnt[f * 3 + 0] = ws_wcnt[f * 3 + 1] = ws_wcnt[f * 3 + 2] = 0;
            if (w == 0) {
                n_groups[h] = 0;
                group_ptr[(size_t)h * (Nq + 1)] = 0;
                if (out_count) out_count[h * 2 + 1] = 0;
            }
        }
        return;
    }

    for (int idx = threadIdx.x; idx < nw * NW; idx += blockDim.x) {
        const int a = idx / NW, wd = idx % NW;
        const uint32_t* src = rowbits + ((size_t)h * Nq + w0 + a) * g * NW + wd;
        uint32_t v = 0;
        for (int j = 0; j < g; ++j) v |= src[(size_t)j * NW];
        S[a * NWp + wd] = v;
    }
    __syncthreads();
    for (int a = threadIdx.x; a < nw; a += blockDim.x) {
        int c = 0;
        for (int wd = 0; wd < NW; ++wd) c += __popc(S[a * NWp + wd]);
        ssize[a] = c;
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;

    const int lane = threadIdx.x;
    const int CPL = (W + 31) >> 5;  // candidates per lane: lane + 32k
    uint32_t taken = 0;
    for (int k = 0; k < CPL; ++k)
        if (lane + 32 * k >= nw) taken |= 1u << k;
    const int gbase = w * (W / max_group);
    int ngw = 0, mpos = 0, visits = 0, masked_q = 0, edges = 0;
    for (int a = lane; a < nw; a += 32) edges += ssize[a];
    edges = __reduce_add_sync(0xffffffffu, edges);

    while (true) {
        unsigned my = 0xffffffffu;
        for (int k = 0; k < CPL; ++k)
            if (!((taken >> k) & 1u)) my = min(my, (unsigned)(lane + 32 * k));
        const unsigned seed = __reduce_min_sync(0xffffffffu, my);
        if (seed == 0xffffffffu) break;
        unsigned ing = 0;  // bit k: candidate lane + 32 k is in this group
        if ((int)(seed & 31u) == lane) {
            taken |= 1u << (seed >> 5);
            ing |= 1u << (seed >> 5);
        }
        for (int wd = lane; wd < NW; wd += 32) U[wd] = S[seed * NWp + wd];
        __syncwarp();
        int cnt = 1, sum_s = ssize[seed];
        while (cnt < max_group) {
            unsigned key = 0xffffffffu;
            for (int k = 0; k < CPL; ++k) {
                if ((taken >> k) & 1u) continue;
                const int a = lane + 32 * k;
                const uint32_t* sa = S + a * NWp;
                int nc = 0;
                for (int wd = 0; wd < NW; ++wd) nc += __popc(sa[wd] & ~U[wd]);
                key = min(key, (pick_value(nc, ssize[a], bundle != 0) << 9) | (unsigned)a);
            }
            const unsigned best = __reduce_min_sync(0xffffffffu, key);
            if (best == 0xffffffffu) break;
            const int c = (int)(best & 511u);
            if ((c & 31) == lane) {
                taken |= 1u << (c >> 5);
                ing |= 1u << (c >> 5);
            }
            __syncwarp();
            for (int wd = lane; wd < NW; wd += 32) U[wd] |= S[c * NWp + wd];
            __syncwarp();
            ++cnt;
            sum_s += ssize[c];
        }
        int us = 0;
        for (int wd = lane; wd < NW; wd += 32) us += __popc(U[wd]);
        us = __reduce_add_sync(0xffffffffu, us);
        {  // members in ascending local ID (candidate lane + 32 k: k-major, then lane)
            const unsigned lt = (1u << lane) - 1u;
            int base = 0;
            for (int k = 0; k < CPL; ++k) {
                const unsigned bk = __ballot_sync(0xffffffffu, (ing >> k) & 1u);
                if ((ing >> k) & 1u) members[(size_t)h * Nq + w0 + mpos + base + __popc(bk & lt)] = w0 + lane + 32 * k;
                base += __popc(bk);
            }
        }
        if (lane == 0) {
            group_ptr[(size_t)h * (Nq + 1) + gbase + ngw] = w0 + mpos;
            ws_usize[(size_t)h * Nq + gbase + ngw] = us;
        }
        mpos += cnt;
        ++ngw;
        visits += us;
        masked_q += cnt * us - sum_s;
        __syncwarp();
    }
    if (lane == 0) {
        const int f = h * nwin + w;
        ws_wtot[f] = visits;
        ws_wcnt[f * 3 + 0] = visits;
        ws_wcnt[f * 3 + 1] = masked_q;
        ws_wcnt[f * 3 + 2] = edges;
        if (w0 + nw == n_items) {  // the window holding the head's last item
            n_groups[h] = gbase + ngw;
            group_ptr[(size_t)h * (Nq + 1) + gbase + ngw] = w0 + mpos;
            if (out_count) out_count[h * 2 + 1] = gbase + ngw;
        }
    }
}

__global__ void __launch_bounds__(256) grp_emit_kernel(
    const uint32_t* __restrict__ rowbits, int Hq, int Hkv, int Nq, int NW, int max_group, int W,
    int nwin, const int32_t* __restrict__ group_ptr, const int32_t* __restrict__ members,
    const int32_t* __restrict__ ws_usize, const int32_t* __restrict__ ws_wtot,
    const int32_t* __restrict__ ws_wcnt, int32_t* __restrict__ union_ptr,
    int32_t* __restrict__ union_pages, uint64_t* __restrict__ row_mask, long long cap,
    int64_t* __restrict__ counters, unsigned* err) {
    extern __shared__ uint32_t sm_em[];
    __shared__ long long red[8];
    __shared__ long long s_base;
    __shared__ int goff[257];
    __shared__ int s_mem[8][8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w = blockIdx.x, h = blockIdx.y, g = Hq / Hkv;
    const int f = h * nwin + w;

    long long s = 0;
    for (int x = threadIdx.x; x < f; x += blockDim.x) s += ws_wtot[x];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[warp] = s;
    __syncthreads();
    const int w0 = w * W, nw = min(W, Nq - w0);
    const int ngw = (nw + max_group - 1) / max_group;
    const int gbase = w * (W / max_group);
    if (threadIdx.x == 0) {
        long long b = 0;
        for (int x = 0; x < 8; ++x) b += red[x];
        s_base = b;
        int o = 0;
        for (int k = 0; k < ngw; ++k) {
            goff[k] = o;
            union_ptr[(size_t)h * (Nq + 1) + gbase + k] = (int32_t)(b + o);
            o += ws_usize[(size_t)h * Nq + gbase + k];
        }
        goff[ngw] = o;
        if (w == nwin - 1) union_ptr[(size_t)h * (Nq + 1) + gbase + ngw] = (int32_t)(b + o);
        if (b + o > cap) atomicOr(err, QUP_ERR_CAPACITY);
    }
    __syncthreads();
    const long long base = s_base;
    if (base + goff[ngw] > cap) return;

    uint32_t* Uw = sm_em + warp * NW;
    int masked_row = 0;
    for (int k = warp; k < ngw; k += 8) {
        const int gi = gbase + k;
        const int p0 = group_ptr[(size_t)h * (Nq + 1) + gi];
        const int nm = group_ptr[(size_t)h * (Nq + 1) + gi + 1] - p0;
        const int R = nm * g;
        if (lane < nm) s_mem[warp][lane] = members[(size_t)h * Nq + p0 + lane];
        __syncwarp();
        for (int wd = lane; wd < NW; wd += 32) {
            uint32_t u = 0;
            for (int m = 0; m < nm; ++m) {
                const uint32_t* src = rowbits + ((size_t)h * Nq + s_mem[warp][m]) * g * NW + wd;
                for (int j = 0; j < g; ++j) u |= src[(size_t)j * NW];
            }
            Uw[wd] = u;
        }
        __syncwarp();
        const int wpl = (NW + 31) >> 5;
        const int wb = min(NW, lane * wpl), we = min(NW, wb + wpl);
        int c = 0;
        for (int wd = wb; wd < we; ++wd) c += __popc(Uw[wd]);
        int incl = c;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int rank = incl - c;
        const long long out0 = base + goff[k];
        int pop = 0;
        for (int wd = wb; wd < we; ++wd) {
            uint32_t word = Uw[wd];
            if (!word) continue;
            uint32_t rw[32];
#pragma unroll
            for (int r = 0; r < 32; ++r)
                rw[r] = (r < R) ? rowbits[((size_t)h * Nq + s_mem[warp][r / g]) * g * NW +
                                          (size_t)(r % g) * NW + wd]
                                : 0u;
            while (word) {
                const int b = __ffs(word) - 1;
                word &= word - 1;
                uint64_t mk = 0;
#pragma unroll
                for (int r = 0; r < 32; ++r) mk |= (uint64_t)((rw[r] >> b) & 1u) << r;
                union_pages[out0 + rank] = wd * 32 + b;
                row_mask[out0 + rank] = mk;
                pop += __popcll(mk);
                ++rank;
            }
        }
        pop = __reduce_add_sync(0xffffffffu, pop);
        masked_row += ws_usize[(size_t)h * Nq + gi] * R - pop;
        __syncwarp();
    }
    __syncthreads();
    if (lane == 0) red[warp] = masked_row;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long mr = 0;
        for (int x = 0; x < 8; ++x) mr += red[x];
        atomicAdd(reinterpret_cast<unsigned long long*>(&counters[h * 4 + 0]),
                  (unsigned long long)ws_wcnt[f * 3 + 0]);
        atomicAdd(reinterpret_cast<unsigned long long*>(&counters[h * 4 + 1]), (unsigned long long)mr);
        atomicAdd(reinterpret_cast<unsigned long long*>(&counters[h * 4 + 2]),
                  (unsigned long long)ws_wcnt[f * 3 + 1]);
        atomicAdd(reinterpret_cast<unsigned long long*>(&counters[h * 4 + 3]),
                  (unsigned long long)ws_wcnt[f * 3 + 2]);
    }
}

// ------------------------------------------------------------------ bundles

// One warp per group: the group's union list -> its page bitset.
__global__ void __launch_bounds__(256) bnd_gbits_kernel(const int32_t* __restrict__ n_groups,
                                                         const int32_t* __restrict__ union_ptr,
                                                         const int32_t* __restrict__ union_pages, int Hkv,
                                                         int Nq, int P, int NW, uint32_t* __restrict__ gbits,
                                                         int64_t* __restrict__ bcounters, unsigned* err) {
    extern __shared__ uint32_t sm_gb[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* bits = sm_gb + warp * NW;
    if (blockIdx.x == 0)
        for (int x = threadIdx.x; x < Hkv * 2; x += blockDim.x) bcounters[x] = 0;
    const long long total = (long long)Hkv * Nq;
    for (long long it = (long long)blockIdx.x * 8 + warp; it < total; it += (long long)gridDim.x * 8) {
        const int h = (int)(it / Nq), gi = (int)(it % Nq);
        if (gi >= n_groups[h]) continue;  // warp-uniform
        for (int x = lane; x < NW; x += 32) bits[x] = 0;
        __syncwarp();
        const int u0 = union_ptr[(size_t)h * (Nq + 1) + gi], u1 = union_ptr[(size_t)h * (Nq + 1) + gi + 1];
        for (int e = u0 + lane; e < u1; e += 32) {
            const int p = union_pages[e];
            if (p < 0 || p >= P) {
                atomicOr(err, QUP_ERR_PAGE_ID);
                continue;
            }
            atomicOr(&bits[p >> 5], 1u << (p & 31));
        }
        __syncwarp();
        uint32_t* dst = gbits + ((size_t)h * Nq + gi) * NW;
        for (int x = lane; x < NW; x += 32) dst[x] = bits[x];
        __syncwarp();
    }
}

// One CTA per (bundle window, KV head): absolute offsets from the earlier
// windows' totals, then one warp per bundle writes the merged union (sorted,
// from the OR of the group bitsets), the 128-bit row masks (each group's row
// mask placed at its slot) and the row -> query table.
__global__ void __launch_bounds__(256) bnd_emit_kernel(
    const uint32_t* __restrict__ gbits, int Hkv, int Nq, int NW, int g, int RS, int slots, int WB, int nwin,
    const int32_t* __restrict__ group_ptr, const int32_t* __restrict__ members,
    const int32_t* __restrict__ union_ptr, const int32_t* __restrict__ union_pages,
    const uint64_t* __restrict__ row_mask, const int32_t* __restrict__ n_bundles,
    const int32_t* __restrict__ bundle_ptr, const int32_t* __restrict__ bundle_groups,
    const int32_t* __restrict__ ws_usize, const int32_t* __restrict__ ws_wtot, int32_t* __restrict__ bunion_ptr,
    int32_t* __restrict__ bunion_pages, uint32_t* __restrict__ bunion_mask, int32_t* __restrict__ bundle_qid,
    long long cap, int64_t* __restrict__ bcounters, unsigned* err) {
    extern __shared__ uint32_t sm_be[];
    __shared__ long long red[8];
    __shared__ long long s_base;
    __shared__ int goff[257];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w = blockIdx.x, h = blockIdx.y;
    const int f = h * nwin + w;
    const int MQ = 128 / g;
    long long s = 0;
    for (int x = threadIdx.x; x < f; x += blockDim.x) s += ws_wtot[x];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[warp] = s;
    __syncthreads();
    const int nb = n_bundles[h];
    const int bbase = w * (WB / slots);
    const int nbw = max(0, min(WB / slots, nb - bbase));
    if (threadIdx.x == 0) {
        long long b = 0;
        for (int x = 0; x < 8; ++x) b += red[x];
        s_base = b;
        int o = 0;
        for (int k = 0; k < nbw; ++k) {
            goff[k] = o;
            bunion_ptr[(size_t)h * (Nq + 1) + bbase + k] = (int32_t)(b + o);
            o += ws_usize[(size_t)h * Nq + bbase + k];
        }
        goff[nbw] = o;
        if (bbase + nbw == nb && (nbw > 0 || w == 0)) bunion_ptr[(size_t)h * (Nq + 1) + nb] = (int32_t)(b + o);
        if (b + o > cap) atomicOr(err, QUP_ERR_CAPACITY);
        if (o > 0) atomicAdd(reinterpret_cast<unsigned long long*>(&bcounters[h * 2]), (unsigned long long)o);
    }
    __syncthreads();
    const long long base = s_base;
    if (nbw == 0 || base + goff[nbw] > cap) return;
    uint32_t* Uw = sm_be + warp * NW;
    for (int k = warp; k < nbw; k += 8) {
        const int bi = bbase + k;
        const int q0 = bundle_ptr[(size_t)h * (Nq + 1) + bi];
        const int cnt = bundle_ptr[(size_t)h * (Nq + 1) + bi + 1] - q0;
        // row -> query table
        int32_t* qt = bundle_qid + ((size_t)h * Nq + bi) * MQ;
        for (int x = lane; x < MQ; x += 32) qt[x] = -1;
        __syncwarp();
        for (int j = 0; j < cnt; ++j) {
            const int gj = bundle_groups[(size_t)h * Nq + q0 + j];
            const int m0 = group_ptr[(size_t)h * (Nq + 1) + gj], m1 = group_ptr[(size_t)h * (Nq + 1) + gj + 1];
            for (int m = lane; m < m1 - m0; m += 32) qt[j * (RS / g) + m] = members[(size_t)h * Nq + m0 + m];
        }
        // merged union bitset
        for (int wd = lane; wd < NW; wd += 32) {
            uint32_t u = 0;
            for (int j = 0; j < cnt; ++j)
                u |= gbits[((size_t)h * Nq + bundle_groups[(size_t)h * Nq + q0 + j]) * NW + wd];
            Uw[wd] = u;
        }
        __syncwarp();
        const int wpl = (NW + 31) >> 5;
        const int wb = min(NW, lane * wpl), we = min(NW, wb + wpl);
        int c = 0;
        for (int wd = wb; wd < we; ++wd) c += __popc(Uw[wd]);
        int incl = c;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const long long out0 = base + goff[k] + (incl - c);
        // pages, zeroed masks
        {
            long long e = out0;
            for (int wd = wb; wd < we; ++wd) {
                uint32_t word = Uw[wd];
                while (word) {
                    const int b = __ffs(word) - 1;
                    word &= word - 1;
                    bunion_pages[e] = wd * 32 + b;
                    bunion_mask[e * 4 + 0] = bunion_mask[e * 4 + 1] = bunion_mask[e * 4 + 2] =
                        bunion_mask[e * 4 + 3] = 0u;
                    ++e;
                }
            }
        }
        // each slot's row masks: walk the group's sorted union alongside this lane's pages
        for (int j = 0; j < cnt; ++j) {
            const int gj = bundle_groups[(size_t)h * Nq + q0 + j];
            const int u0 = union_ptr[(size_t)h * (Nq + 1) + gj], u1 = union_ptr[(size_t)h * (Nq + 1) + gj + 1];
            int lo = u0, hi = u1;  // first entry with page >= 32 * wb
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (union_pages[mid] < wb * 32) lo = mid + 1;
                else hi = mid;
            }
            int kk = lo;
            long long e = out0;
            const int bit0 = j * RS;
            for (int wd = wb; wd < we; ++wd) {
                uint32_t word = Uw[wd];
                while (word) {
                    const int b = __ffs(word) - 1;
                    word &= word - 1;
                    const int pg = wd * 32 + b;
                    while (kk < u1 && union_pages[kk] < pg) ++kk;
                    if (kk < u1 && union_pages[kk] == pg) {
                        const uint32_t mk = (uint32_t)row_mask[kk] & (RS == 32 ? 0xffffffffu : ((1u << RS) - 1u));
                        bunion_mask[e * 4 + (bit0 >> 5)] |= mk << (bit0 & 31);
                    }
                    ++e;
                }
            }
        }
        __syncwarp();
    }
}

size_t group_greedy_smem(int W, int NW) {
    const int NWp = NW | 1;
    return sizeof(uint32_t) * ((size_t)W * NWp + NWp + W);
}

// One warp per TopK row without shared memory: lane l builds words l, l + 32, ...
// of the row's page bitset while the row's entries are broadcast one by one
// (K <= 64 entries, at most 32 * kRbWords words).
constexpr int kRbWords = 8;
__global__ void __launch_bounds__(256) grp_rowbits_shfl_kernel(const int32_t* __restrict__ topk, int Hq, int Hkv,
                                                                int Nq, int K, int P, int NW,
                                                                uint32_t* __restrict__ rowbits,
                                                                int64_t* __restrict__ counters, unsigned* err) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (blockIdx.x == 0)
        for (int x = threadIdx.x; x < Hkv * 4; x += blockDim.x) counters[x] = 0;
    const int g = Hq / Hkv;
    const long long nrows = (long long)Hq * Nq;
    for (long long row = (long long)blockIdx.x * 8 + warp; row < nrows; row += (long long)gridDim.x * 8) {
        const int hq = (int)(row / Nq), i = (int)(row % Nq);
        const int32_t* tr = topk + row * K;
        uint32_t wb[kRbWords];
#pragma unroll
        for (int x = 0; x < kRbWords; ++x) wb[x] = 0u;
        for (int k0 = 0; k0 < K; k0 += 32) {
            int e = k0 + lane < K ? tr[k0 + lane] : -1;
            if (e != -1 && (e < 0 || e >= P)) {
                atomicOr(err, QUP_ERR_PAGE_ID);
                e = -1;
            }
            const int n = min(32, K - k0);
            for (int t = 0; t < n; ++t) {
                const int pe = __shfl_sync(0xffffffffu, e, t);
                if (pe >= 0 && ((pe >> 5) & 31) == lane) {
                    const int slot = pe >> 10;
#pragma unroll
                    for (int x = 0; x < kRbWords; ++x)
                        if (x == slot) wb[x] |= 1u << (pe & 31);
                }
            }
        }
        const int h = hq / g, j = hq % g;
        uint32_t* dst = rowbits + (((size_t)h * Nq + i) * g + j) * NW;
#pragma unroll
        for (int x = 0; x < kRbWords; ++x)
            if (lane + 32 * x < NW) dst[lane + 32 * x] = wb[x];
    }
}

// ------------------------------------------------------------------ register-resident greedy
// The same greedy as grp_greedy_kernel for windows of at most 64 items whose sets
// fit in NWR words: one warp per (window, KV head), lane l holds the sets of items
// l and l + 32 in registers, so a pick is 2 x NWR and-not/popcounts per lane, one
// warp min-reduction of the packed key (new_pages << 9 | local_id) and a shuffle
// of the winner's set from its owner lane.  Members are kept as a 64-bit mask of
// local IDs; each lane also flags which of its two items joined the current
// group, and two ballots give every member its rank (ascending local ID).
template <int NWR>
__global__ void __launch_bounds__(128) grp_greedy_reg_kernel(const uint32_t* __restrict__ rowbits, int sets_per_item,
                                                              int Hkv, int Nq, const int32_t* __restrict__ n_items_dev,
                                                              int NW, int max_group, int W, int nwin,
                                                              int32_t* __restrict__ group_ptr,
                                                              int32_t* __restrict__ members,
                                                              int32_t* __restrict__ n_groups,
                                                              int32_t* __restrict__ ws_usize,
                                                              int32_t* __restrict__ ws_wtot,
                                                              int32_t* __restrict__ ws_wcnt,
                                                              int64_t* __restrict__ out_count, int bundle) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x * 4 + warp;
    if (item >= nwin * Hkv) return;
    const int h = item / nwin, w = item % nwin, g = sets_per_item;
    const int n_items = n_items_dev ? n_items_dev[h] : Nq;
    const int w0 = w * W, nw = max(0, min(W, n_items - w0));
    if (nw == 0) {  // window past the head's last item: contributes nothing
        if (lane == 0) {
            const int f = h * nwin + w;
            ws_wtot[f] = 0;
            ws_wcnt[f * 3 + 0] = ws_wcnt[f * 3 + 1] = ws_wcnt[f * 3 + 2] = 0;
            if (w == 0) {
                n_groups[h] = 0;
                group_ptr[(size_t)h * (Nq + 1)] = 0;
                if (out_count) out_count[h * 2 + 1] = 0;
            }
        }
        return;
    }
    constexpr unsigned kNone = 0xffffffffu;
    uint32_t s0[NWR], s1[NWR], U[NWR];
#pragma unroll
    for (int x = 0; x < NWR; ++x) s0[x] = s1[x] = 0u;
    const bool v0 = lane < nw, v1 = lane + 32 < nw;
    if (v0) {
        const uint32_t* src = rowbits + ((size_t)h * Nq + w0 + lane) * g * NW;
        for (int j = 0; j < g; ++j)
#pragma unroll
            for (int x = 0; x < NWR; ++x)
                if (x < NW) s0[x] |= src[(size_t)j * NW + x];
    }
    if (v1) {
        const uint32_t* src = rowbits + ((size_t)h * Nq + w0 + lane + 32) * g * NW;
        for (int j = 0; j < g; ++j)
#pragma unroll
            for (int x = 0; x < NWR; ++x)
                if (x < NW) s1[x] |= src[(size_t)j * NW + x];
    }
    int sz0 = 0, sz1 = 0;
#pragma unroll
    for (int x = 0; x < NWR; ++x) {
        sz0 += __popc(s0[x]);
        sz1 += __popc(s1[x]);
    }
    const int edges = __reduce_add_sync(0xffffffffu, sz0 + sz1);  // invalid items hold empty sets
    unsigned taken = (v0 ? 0u : 1u) | (v1 ? 0u : 2u);
    const int gbase = w * (W / max_group);
    int ngw = 0, mpos = 0, visits = 0, masked_q = 0;
    while (true) {
        const unsigned my = !(taken & 1u) ? (unsigned)lane : (!(taken & 2u) ? (unsigned)lane + 32u : kNone);
        const unsigned seed = __reduce_min_sync(0xffffffffu, my);
        if (seed == kNone) break;
        int owner = (int)(seed & 31u), k = (int)(seed >> 5);
        unsigned ing = 0;  // bit k: item lane + 32 k is in this group
        if (lane == owner) {
            taken |= 1u << k;
            ing |= 1u << k;
        }
#pragma unroll
        for (int x = 0; x < NWR; ++x) U[x] = __shfl_sync(0xffffffffu, k ? s1[x] : s0[x], owner);
        int sum_s = __shfl_sync(0xffffffffu, k ? sz1 : sz0, owner);
        int cnt = 1;
        while (cnt < max_group) {
            unsigned key = kNone;
            if (!(taken & 1u)) {
                int nc = 0;
#pragma unroll
                for (int x = 0; x < NWR; ++x) nc += __popc(s0[x] & ~U[x]);
                key = (pick_value(nc, sz0, bundle != 0) << 9) | (unsigned)lane;
            }
            if (!(taken & 2u)) {
                int nc = 0;
#pragma unroll
                for (int x = 0; x < NWR; ++x) nc += __popc(s1[x] & ~U[x]);
                key = min(key, (pick_value(nc, sz1, bundle != 0) << 9) | (unsigned)(lane + 32));
            }
            const unsigned best = __reduce_min_sync(0xffffffffu, key);
            if (best == kNone) break;
            const int c = (int)(best & 511u);
            owner = c & 31;
            k = c >> 5;
            if (lane == owner) {
                taken |= 1u << k;
                ing |= 1u << k;
            }
#pragma unroll
            for (int x = 0; x < NWR; ++x) U[x] |= __shfl_sync(0xffffffffu, k ? s1[x] : s0[x], owner);
            sum_s += __shfl_sync(0xffffffffu, k ? sz1 : sz0, owner);
            ++cnt;
        }
        int us = 0;
#pragma unroll
        for (int x = 0; x < NWR; ++x) us += __popc(U[x]);
        {  // members in ascending local ID: items 0..31 (k = 0) before 32..63 (k = 1)
            const unsigned b0 = __ballot_sync(0xffffffffu, ing & 1u), b1 = __ballot_sync(0xffffffffu, ing & 2u);
            const unsigned lt = (1u << lane) - 1u;
            int32_t* dst = members + (size_t)h * Nq + w0 + mpos;
            if (ing & 1u) dst[__popc(b0 & lt)] = w0 + lane;
            if (ing & 2u) dst[__popc(b0) + __popc(b1 & lt)] = w0 + lane + 32;
        }
        if (lane == 0) {
            group_ptr[(size_t)h * (Nq + 1) + gbase + ngw] = w0 + mpos;
            ws_usize[(size_t)h * Nq + gbase + ngw] = us;
        }
        mpos += cnt;
        ++ngw;
        visits += us;
        masked_q += cnt * us - sum_s;
    }
    if (lane == 0) {
        const int f = h * nwin + w;
        ws_wtot[f] = visits;
        ws_wcnt[f * 3 + 0] = visits;
        ws_wcnt[f * 3 + 1] = masked_q;
        ws_wcnt[f * 3 + 2] = edges;
        if (w0 + nw == n_items) {  // the window holding the head's last item
            n_groups[h] = gbase + ngw;
            group_ptr[(size_t)h * (Nq + 1) + gbase + ngw] = w0 + mpos;
            if (out_count) out_count[h * 2 + 1] = gbase + ngw;
        }
    }
}

// Greedy dispatch: the register kernel when the window holds at most 64 items and a
// set fits in 32 words, else the shared-memory kernel.
static cudaError_t launch_greedy(const uint32_t* sets, int sets_per_item, int Hkv, int Nq, const int32_t* n_items_dev,
                                 int NW, int max_group, int W, int nwin, int32_t* group_ptr, int32_t* members,
                                 int32_t* n_groups, int32_t* ws_usize, int32_t* ws_wtot, int32_t* ws_wcnt,
                                 int64_t* out_count, bool bundle, cudaStream_t stream) {
    if (W <= 64 && NW <= 32) {
        const int items = nwin * Hkv, grid = (items + 3) / 4;
#define QUP_GREEDY_REG(N)                                                                                        \
    grp_greedy_reg_kernel<N><<<grid, 128, 0, stream>>>(sets, sets_per_item, Hkv, Nq, n_items_dev, NW, max_group, \
                                                       W, nwin, group_ptr, members, n_groups, ws_usize, ws_wtot, \
                                                       ws_wcnt, out_count, bundle ? 1 : 0)
        if (NW <= 4) QUP_GREEDY_REG(4);
        else if (NW <= 8) QUP_GREEDY_REG(8);
        else if (NW <= 12) QUP_GREEDY_REG(12);
        else if (NW <= 16) QUP_GREEDY_REG(16);
        else if (NW <= 24) QUP_GREEDY_REG(24);
        else QUP_GREEDY_REG(32);
#undef QUP_GREEDY_REG
        return cudaGetLastError();
    }
    const size_t sm = group_greedy_smem(W, NW);
    cudaError_t e = cudaFuncSetAttribute(grp_greedy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    grp_greedy_kernel<<<dim3(nwin, Hkv), 128, sm, stream>>>(sets, sets_per_item, Hkv, Nq, n_items_dev, NW, max_group,
                                                             W, nwin, group_ptr, members, n_groups, ws_usize, ws_wtot,
                                                             ws_wcnt, out_count, bundle ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_group(const GroupLaunch& a, cudaStream_t stream) {
    const size_t sm1 = sizeof(uint32_t) * 8 * (size_t)a.NW;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(grp_rowbits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm1)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(grp_emit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm1)) != cudaSuccess)
        return e;
    const long long rows = (long long)a.Hq * a.Nq;
    const int grid1 = (int)std::min<long long>((rows + 7) / 8, (long long)a.sms * 8);
    if (a.K <= 64 && a.NW <= 32 * kRbWords)
        grp_rowbits_shfl_kernel<<<grid1, 256, 0, stream>>>(a.topk, a.Hq, a.Hkv, a.Nq, a.K, a.P, a.NW, a.rowbits,
                                                            a.counters, a.err);
    else
        grp_rowbits_kernel<<<grid1, 256, sm1, stream>>>(a.topk, a.Hq, a.Hkv, a.Nq, a.K, a.P, a.NW,
                                                       a.rowbits, a.counters, a.err);
    const dim3 grid2(a.nwin, a.Hkv);
    if ((e = launch_greedy(a.rowbits, a.Hq / a.Hkv, a.Hkv, a.Nq, nullptr, a.NW, a.max_group, a.W, a.nwin,
                           a.group_ptr, a.members, a.n_groups, a.ws_usize, a.ws_wtot, a.ws_wcnt, nullptr, false,
                           stream)) != cudaSuccess)
        return e;
    grp_emit_kernel<<<grid2, 256, sm1, stream>>>(a.rowbits, a.Hq, a.Hkv, a.Nq, a.NW, a.max_group, a.W,
                                                 a.nwin, a.group_ptr, a.members, a.ws_usize, a.ws_wtot,
                                                 a.ws_wcnt, a.union_ptr, a.union_pages, a.row_mask, a.cap,
                                                 a.counters, a.err);
    return cudaGetLastError();
}

// Work order of the attention kernel: the flat bundle indices (KV heads in
// order, then bundles) sorted by union size, largest first, equal sizes by
// index (a stable counting sort; sizes above kOrderBuckets-1 share the top
// bucket).  The attention kernel's CTAs claim bundles in this order at run
// time, so the largest go first and the smallest fill the end.
constexpr int kOrderBuckets = 4096;

__global__ void __launch_bounds__(1024) bnd_order_kernel(const int32_t* __restrict__ n_bundles,
                                                         const int32_t* __restrict__ bunion_ptr, int Hkv, int Nq,
                                                         int32_t* __restrict__ order) {
    __shared__ int cursor[kOrderBuckets];
    __shared__ int warp_sum[32];
    extern __shared__ int head_start[];  // [Hkv + 1] flat index of each KV head's first bundle
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        int acc = 0;
        for (int h = 0; h < Hkv; ++h) {
            head_start[h] = acc;
            const int n = n_bundles[h];
            acc += (n >= 0 && n <= Nq) ? n : 0;  // the attention kernel reports a bad count
        }
        head_start[Hkv] = acc;
    }
    for (int k = tid; k < kOrderBuckets; k += blockDim.x) cursor[k] = 0;
    __syncthreads();
    const int n = head_start[Hkv];
    auto key_of = [&](int h, int bi) {
        const size_t b = (size_t)h * (Nq + 1) + bi;
        const int size = bunion_ptr[b + 1] - bunion_ptr[b];
        return kOrderBuckets - 1 - min(max(size, 0), kOrderBuckets - 1);  // larger union -> smaller key
    };
    for (int h = 0; h < Hkv; ++h)
        for (int bi = tid; bi < head_start[h + 1] - head_start[h]; bi += blockDim.x) atomicAdd(&cursor[key_of(h, bi)], 1);
    __syncthreads();
    // exclusive scan of the histogram: kOrderBuckets / blockDim.x buckets per thread
    constexpr int kPer = kOrderBuckets / 1024;
    int v[kPer], run = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        v[k] = run;
        run += cursor[tid * kPer + k];
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_sum[lane], wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        warp_sum[lane] = wi - w;
    }
    __syncthreads();
    const int base = warp_sum[warp] + incl - run;
#pragma unroll
    for (int k = 0; k < kPer; ++k) cursor[tid * kPer + k] = base + v[k];
    __syncthreads();
    // stable scatter: one warp walks the flat indices in order, 32 at a time
    if (warp == 0) {
        int h = 0;
        for (int f0 = 0; f0 < n; f0 += 32) {
            const int f = f0 + lane;
            const unsigned live = __ballot_sync(0xffffffffu, f < n);
            if (f < n) {
                while (head_start[h + 1] <= f) ++h;
                const int key = key_of(h, f - head_start[h]);
                const unsigned peers = __match_any_sync(live, key);
                const int leader = __ffs(peers) - 1;
                const int rank = __popc(peers & ((1u << lane) - 1u));
                int start = 0;
                if (lane == leader) {
                    start = cursor[key];
                    cursor[key] = start + __popc(peers);
                }
                start = __shfl_sync(live, start, leader);
                order[start + rank] = f;
            }
            __syncwarp();
        }
    }
}

}  // namespace qup

namespace qup {

// Union as support (CompactAttention: Accelerating Chunked Prefill with Block-Union KV
// Selection, where a query block attends to its whole union table): every row of a group sees
// every page of the group's union.  One warp per group sets each union entry's row mask to the
// group's rows (bits 0 .. members * g - 1).
__global__ void __launch_bounds__(256) grp_union_support_kernel(const int32_t* __restrict__ n_groups,
                                                               const int32_t* __restrict__ group_ptr,
                                                               const int32_t* __restrict__ union_ptr,
                                                               uint64_t* __restrict__ row_mask, int Hkv, int Nq,
                                                               int g, long long cap, unsigned* err) {
    const int lane = threadIdx.x & 31;
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long x = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); x < (long long)Hkv * Nq;
         x += nwarps) {
        const int h = (int)(x / Nq), k = (int)(x % Nq);
        if (k >= n_groups[h]) continue;
        const size_t gp = (size_t)h * (Nq + 1) + k;
        const int cnt = group_ptr[gp + 1] - group_ptr[gp];
        const long long e0 = union_ptr[gp], e1 = union_ptr[gp + 1];
        if (cnt < 1 || cnt * g > 64 || e0 < 0 || e1 < e0 || e1 > cap) {
            if (lane == 0) atomicOr(err, QUP_ERR_GROUP);
            continue;
        }
        const int R = cnt * g;
        const uint64_t full = R == 64 ? ~0ull : ((1ull << R) - 1ull);
        for (long long e = e0 + lane; e < e1; e += 32) row_mask[e] = full;
    }
}

cudaError_t launch_union_support(const int32_t* n_groups, const int32_t* group_ptr, const int32_t* union_ptr,
                                 uint64_t* row_mask, int Hkv, int Nq, int g, long long cap, unsigned* err, int sms,
                                 cudaStream_t stream) {
    const long long items = (long long)Hkv * Nq;
    if (items == 0) return cudaSuccess;
    const int grid = (int)std::min<long long>((items + 7) / 8, (long long)sms * 8);
    grp_union_support_kernel<<<grid, 256, 0, stream>>>(n_groups, group_ptr, union_ptr, row_mask, Hkv, Nq, g, cap,
                                                       err);
    return cudaGetLastError();
}

cudaError_t launch_gbits(const BundleLaunch& a, cudaStream_t stream) {
    const size_t smw = sizeof(uint32_t) * 8 * (size_t)a.NW;
    cudaError_t e = cudaFuncSetAttribute(bnd_gbits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smw);
    if (e != cudaSuccess) return e;
    const long long items = (long long)a.Hkv * a.Nq;
    const int grid1 = (int)std::min<long long>((items + 7) / 8, (long long)a.sms * 8);
    bnd_gbits_kernel<<<grid1, 256, smw, stream>>>(a.n_groups, a.union_ptr, a.union_pages, a.Hkv, a.Nq, a.P, a.NW,
                                                  a.gbits, a.bcounters, a.err);
    return cudaGetLastError();
}

cudaError_t launch_bundles(const BundleLaunch& a, cudaStream_t stream) {
    const size_t smw = sizeof(uint32_t) * 8 * (size_t)a.NW;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(bnd_gbits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smw)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(bnd_emit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smw)) !=
        cudaSuccess)
        return e;
    const long long items = (long long)a.Hkv * a.Nq;
    const int grid1 = (int)std::min<long long>((items + 7) / 8, (long long)a.sms * 8);
    bnd_gbits_kernel<<<grid1, 256, smw, stream>>>(a.n_groups, a.union_ptr, a.union_pages, a.Hkv, a.Nq, a.P, a.NW,
                                                  a.gbits, a.bcounters, a.err);
    const dim3 grid2(a.nwin, a.Hkv);
    if ((e = launch_greedy(a.gbits, 1, a.Hkv, a.Nq, a.n_groups, a.NW, a.slots, a.WB, a.nwin, a.bundle_ptr,
                           a.bundle_groups, a.n_bundles, a.ws_usize, a.ws_wtot, a.ws_wcnt, a.bcounters, true, stream)) !=
        cudaSuccess)
        return e;
    bnd_emit_kernel<<<grid2, 256, smw, stream>>>(a.gbits, a.Hkv, a.Nq, a.NW, a.g, a.RS, a.slots, a.WB, a.nwin,
                                                 a.group_ptr, a.members, a.union_ptr, a.union_pages, a.row_mask,
                                                 a.n_bundles, a.bundle_ptr, a.bundle_groups, a.ws_usize, a.ws_wtot,
                                                 a.bunion_ptr, a.bunion_pages, a.bunion_mask, a.bundle_qid, a.cap,
                                                 a.bcounters, a.err);
    bnd_order_kernel<<<1, 1024, sizeof(int) * (a.Hkv + 1), stream>>>(a.n_bundles, a.bunion_ptr, a.Hkv, a.Nq,
                                                                      a.bundle_order);
    return cudaGetLastError();
}

}  // namespace qup
