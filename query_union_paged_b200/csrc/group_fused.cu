// group_fused.cu -- the grouping call in two fused kernels (PageWeaver,
// Abstract: a GPU search of bounded cost turns the affinity of the queries'
// selected pages into query-ID lists; Figure 2: logical page visits and masked
// query-page slots).
//
// Same rule and same outputs as the multi-kernel path in group.cu, with the
// intermediate state kept in shared memory:
//   grp_fused_kernel  one CTA per (query window, KV head): the window's TopK
//                     rows -> per-row page bitsets (one thread per row) ->
//                     per-query sets (OR over the g heads of the KV group) ->
//                     greedy groups (pick: fewest new pages) -> union pages and
//                     row masks of every group, written at offsets found by a
//                     look-back over the earlier windows.  256 threads, or 128
//                     (four CTAs per SM) when the windows outnumber the CTAs.
//   bnd_fused_kernel  one CTA per (window of groups, KV head): the groups'
//                     union bitsets -> greedy bundles of up to `slots` groups
//                     (pick: smallest new - 2 * shared pages, pick_value) ->
//                     bundle unions, 128-bit row masks and the row -> query
//                     table; the CTA that finishes last also sorts the bundles
//                     by union size for the attention kernel.
//
// The greedy runs on sets compacted to the window's own pages: page p of the
// window universe becomes bit rank(p), so |S(c) \ U| is computed over a few
// words however large the page space is.  Compaction is a bijection on the
// universe, so every count, and with it every pick, equals the uncompacted
// greedy's.
//
// Offsets: windows are numbered f = h * nwin + w (the order of the CSR
// outputs).  Each CTA publishes its window's entry count, then walks back over
// the windows before it (decoupled look-back) until it meets one that already
// published its inclusive prefix.  CTAs claim windows from an atomic ticket, in
// increasing f: a window is only ever claimed by a CTA that is running, and
// every window before it was claimed earlier by a running CTA that publishes it
// without waiting on later windows, so the look-back always ends, however many
// of the grid's CTAs the device holds at once (other kernels may share it).
// Each wait is still bounded; a wait that runs out raises QUP_ERR_TIMEOUT.
#include <algorithm>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "query_union_paged.h"

namespace qup {
namespace {

constexpr unsigned kNone = 0xffffffffu;
constexpr int kFusedThreads = 256;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr uint64_t kFlagAgg = 1ull << 62, kFlagIncl = 2ull << 62, kValMask = (1ull << 62) - 1;

// ---------------------------------------------------------------- shared-memory plan
// One window: n <= W items with original sets S[n][NW] (pitch NW), their
// universe and its word prefix counts, compact sets cs[n][NWC] (pitch NWCp),
// and the greedy's output lists.
struct WinSmem {
    uint32_t* S;      // [W][NW]
    uint32_t* UW;     // [NW]
    int* pref;        // [NW + 1]
    uint32_t* cs;     // [W][NWCp]
    uint32_t* Ug;     // [NWCp] greedy union (smem path)
    int* ssize;       // [W]
    int* order;       // [W] items in group order, ascending inside a group
    int* gstart;      // [W + 1]
    int* gus;         // [W] union size of each group
    int* gsum;        // [W] sum of member set sizes of each group
    int* misc;        // [8]: 0 groups, 1 compact words NWC, 7 compact pitch
    int* goff;        // [W + 1] exclusive prefix of gus
    uint32_t* post;   // [kPostWords] block greedy: per-warp best keys and sets, group tallies
};

constexpr int kPostWords = 2 * 8 * (8 + 1) + 2 * 8;  // up to 8 warps, 8-word compact sets

__host__ __device__ inline size_t win_smem_bytes(int W, int NW, int extra_words) {
    const int NWCp = NW | 1;
    size_t words = (size_t)W * NW + NW + (NW + 1) + (size_t)W * NWCp + NWCp + W + W + (W + 1) + W + W + 8 + (W + 1) +
                   kPostWords;
    return 4 * (words + (size_t)extra_words) + 64;
}

__device__ inline WinSmem carve(uint32_t* base, int W, int NW) {
    WinSmem s;
    const int NWCp = NW | 1;
    uint32_t* p = base;
    s.S = p;
    p += (size_t)W * NW;
    s.UW = p;
    p += NW;
    s.pref = reinterpret_cast<int*>(p);
    p += NW + 1;
    s.cs = p;
    p += (size_t)W * NWCp;
    s.Ug = p;
    p += NWCp;
    s.ssize = reinterpret_cast<int*>(p);
    p += W;
    s.order = reinterpret_cast<int*>(p);
    p += W;
    s.gstart = reinterpret_cast<int*>(p);
    p += W + 1;
    s.gus = reinterpret_cast<int*>(p);
    p += W;
    s.gsum = reinterpret_cast<int*>(p);
    p += W;
    s.misc = reinterpret_cast<int*>(p);
    p += 8;
    s.goff = reinterpret_cast<int*>(p);
    p += W + 1;
    s.post = p;
    return s;
}

// 32 x 32 bit matrix held one row per lane (bit k of lane i = element (i, k)) transposed in
// place: afterwards bit i of lane k = element (i, k).  Five block swaps: at width j, the rows
// with bit j clear take the left-hand columns of row i + j into their right-hand half, and
// rows with bit j set take the right-hand columns of row i - j into their left-hand half.
__device__ __forceinline__ void transpose32(uint32_t& x, int lane) {
    const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        const int j = 16 >> i;
        const uint32_t m = masks[i];  // columns k with (k & j) == 0
        const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
        x = (lane & j) ? ((x & ~m) | ((y & ~m) >> j)) : ((x & m) | ((y & m) << j));
    }
}

// Universe, its prefix counts, set sizes and compact sets of items [0, n).
// Whole CTA; ends with the compact sets ready (a barrier inside).
__device__ void compact_window(const WinSmem& s, int n, int NW) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int wd = tid; wd < NW; wd += blockDim.x) s.UW[wd] = 0u;
    __syncthreads();
    // universe words: each thread ORs one word over a run of items, then one atomic per run
    // (atomics of every item on the same few words would serialise)
    const int runs = max(1, (int)blockDim.x / max(NW, 1));
    const int per = (n + runs - 1) / runs;
    for (int x = tid; x < NW * runs; x += blockDim.x) {
        const int wd = x % NW, c = x / NW;
        const int a1 = min(n, (c + 1) * per);
        uint32_t acc = 0u;
        for (int a = c * per; a < a1; ++a) acc |= s.S[(size_t)a * NW + wd];
        if (acc) atomicOr(&s.UW[wd], acc);
    }
    // set sizes: one thread per item
    for (int a = tid; a < n; a += blockDim.x) {
        int c = 0;
        for (int wd = 0; wd < NW; ++wd) c += __popc(s.S[(size_t)a * NW + wd]);
        s.ssize[a] = c;
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of popc(UW) over words
        int carry = 0;
        for (int w0 = 0; w0 < NW; w0 += 32) {
            const int wd = w0 + lane;
            const int c = wd < NW ? __popc(s.UW[wd]) : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (wd < NW) s.pref[wd] = carry + incl - c;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            s.pref[NW] = carry;
            s.misc[1] = (carry + 31) >> 5;  // NWC
            s.misc[7] = NW | 1;             // pitch of the compact sets
        }
    }
    __syncthreads();
    const int NWCp = NW | 1;
    for (int x = tid; x < n * NWCp; x += blockDim.x) s.cs[x] = 0u;
    __syncthreads();
    // compact sets (bit c = the c-th page of the universe): one thread per (item, word); the
    // word's bits land at ranks p0 .. p0 + popc(universe word) - 1, in at most two compact words,
    // so a word costs at most two atomics however many bits it has
    for (int x = tid; x < n * NW; x += blockDim.x) {
        uint32_t v = s.S[x];
        if (!v) continue;
        const int a = x / NW, wd = x - a * NW;
        const uint32_t uw = s.UW[wd];
        const int p0 = s.pref[wd];
        uint64_t acc = 0u;
        while (v) {
            const int b = __ffs(v) - 1;
            v &= v - 1;
            acc |= 1ull << __popc(uw & ((1u << b) - 1u));
        }
        acc <<= (p0 & 31);
        uint32_t* dst = s.cs + (size_t)a * NWCp + (p0 >> 5);
        if ((uint32_t)acc) atomicOr(dst, (uint32_t)acc);
        if ((uint32_t)(acc >> 32)) atomicOr(dst + 1, (uint32_t)(acc >> 32));
    }
    __syncthreads();
}

// Greedy (warp 0) with every set of a window of at most 32 * CPL items in registers:
// lane l holds items l, l + 32, ..., l + 32 * (CPL - 1).  Writes order / gstart / gus / gsum
// and the group count.  The pick key is (value << 9 | local_id), value = pick_value (the new
// page count for groups); ties go to the smallest ID.
template <int NWR, int CPL, bool BUNDLE>
__device__ __noinline__ void greedy_reg(const WinSmem& s, int n, int max_group) {
    constexpr bool bundle = BUNDLE;
    const int lane = threadIdx.x & 31;
    uint32_t sc[CPL][NWR], U[NWR];
    int sz[CPL];
    const int pitch = s.misc[7], NWC = s.misc[1];
    unsigned taken = 0;
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
        const int a = lane + 32 * k;
#pragma unroll
        for (int x = 0; x < NWR; ++x) sc[k][x] = (a < n && x < NWC) ? s.cs[(size_t)a * pitch + x] : 0u;
        sz[k] = a < n ? s.ssize[a] : 0;
        if (a >= n) taken |= 1u << k;
    }
    constexpr unsigned kAll = (1u << CPL) - 1u;
    int ng = 0, pos = 0;
    while (true) {
        const unsigned free_k = ~taken & kAll;
        const unsigned my = free_k ? (unsigned)lane + 32u * (unsigned)(__ffs(free_k) - 1) : kNone;
        const unsigned seed = __reduce_min_sync(0xffffffffu, my);
        if (seed == kNone) break;
        int owner = (int)(seed & 31u), k = (int)(seed >> 5);
        unsigned ing = 0;
        if (lane == owner) {
            taken |= 1u << k;
            ing |= 1u << k;
        }
#pragma unroll
        for (int x = 0; x < NWR; ++x) {
            uint32_t v = sc[0][x];
#pragma unroll
            for (int kk = 1; kk < CPL; ++kk)
                if (k == kk) v = sc[kk][x];
            U[x] = __shfl_sync(0xffffffffu, v, owner);
        }
        int cnt = 1;
        while (cnt < max_group) {
            unsigned bestk = kNone;
#pragma unroll
            for (int kk = 0; kk < CPL; ++kk) {
                int c = 0;
#pragma unroll
                for (int x = 0; x < NWR; ++x) c += __popc(sc[kk][x] & ~U[x]);
                const unsigned key =
                    (taken >> kk) & 1u ? kNone : ((pick_value(c, sz[kk], bundle) << 9) | (unsigned)(lane + 32 * kk));
                bestk = min(bestk, key);
            }
            const unsigned best = __reduce_min_sync(0xffffffffu, bestk);
            if (best == kNone) break;
            const int c = (int)(best & 511u);
            owner = c & 31;
            k = c >> 5;
            if (lane == owner) {
                taken |= 1u << k;
                ing |= 1u << k;
            }
#pragma unroll
            for (int x = 0; x < NWR; ++x) {
                uint32_t v = sc[0][x];
#pragma unroll
                for (int kk = 1; kk < CPL; ++kk)
                    if (k == kk) v = sc[kk][x];
                U[x] |= __shfl_sync(0xffffffffu, v, owner);
            }
            ++cnt;
        }
        int us = 0;
#pragma unroll
        for (int x = 0; x < NWR; ++x) us += __popc(U[x]);
        int mysum = 0;
#pragma unroll
        for (int kk = 0; kk < CPL; ++kk) mysum += (ing >> kk) & 1u ? sz[kk] : 0;
        const int sum_s = __reduce_add_sync(0xffffffffu, mysum);
        // members in ascending ID: item lane + 32 kk ranks after every member of a lower kk
        const unsigned lt = (1u << lane) - 1u;
        int before = 0;
#pragma unroll
        for (int kk = 0; kk < CPL; ++kk) {
            const unsigned bk = __ballot_sync(0xffffffffu, (ing >> kk) & 1u);
            if ((ing >> kk) & 1u) s.order[pos + before + __popc(bk & lt)] = lane + 32 * kk;
            before += __popc(bk);
        }
        if (lane == 0) {
            s.gstart[ng] = pos;
            s.gus[ng] = us;
            s.gsum[ng] = sum_s;
        }
        pos += cnt;
        ++ng;
    }
    if (lane == 0) {
        s.gstart[ng] = pos;
        s.misc[0] = ng;
    }
}

// Greedy (warp 0) for any window (n <= 256) and any compact width: sets and
// the running union stay in shared memory.
__device__ __noinline__ void greedy_smem(const WinSmem& s, int n, int max_group, bool bundle) {
    const int lane = threadIdx.x & 31;
    const int NWC = s.misc[1], pitch = s.misc[7];
    const int CPL = (n + 31) >> 5;
    uint32_t taken = 0;
    for (int k = 0; k < CPL; ++k)
        if (lane + 32 * k >= n) taken |= 1u << k;
    int ng = 0, pos = 0;
    while (true) {
        unsigned my = kNone;
        for (int k = 0; k < CPL; ++k)
            if (!((taken >> k) & 1u)) my = min(my, (unsigned)(lane + 32 * k));
        const unsigned seed = __reduce_min_sync(0xffffffffu, my);
        if (seed == kNone) break;
        unsigned ing = 0;
        if ((int)(seed & 31u) == lane) {
            taken |= 1u << (seed >> 5);
            ing |= 1u << (seed >> 5);
        }
        for (int wd = lane; wd < NWC; wd += 32) s.Ug[wd] = s.cs[(size_t)seed * pitch + wd];
        __syncwarp();
        int cnt = 1, sum_s = s.ssize[seed];
        while (cnt < max_group) {
            unsigned key = kNone;
            for (int k = 0; k < CPL; ++k) {
                if ((taken >> k) & 1u) continue;
                const int a = lane + 32 * k;
                const uint32_t* sa = s.cs + (size_t)a * pitch;
                int nc = 0;
                for (int wd = 0; wd < NWC; ++wd) nc += __popc(sa[wd] & ~s.Ug[wd]);
                key = min(key, (pick_value(nc, s.ssize[a], bundle) << 9) | (unsigned)a);
            }
            const unsigned best = __reduce_min_sync(0xffffffffu, key);
            if (best == kNone) break;
            const int c = (int)(best & 511u);
            if ((c & 31) == lane) {
                taken |= 1u << (c >> 5);
                ing |= 1u << (c >> 5);
            }
            __syncwarp();
            for (int wd = lane; wd < NWC; wd += 32) s.Ug[wd] |= s.cs[(size_t)c * pitch + wd];
            __syncwarp();
            ++cnt;
            sum_s += s.ssize[c];
        }
        int us = 0;
        for (int wd = lane; wd < NWC; wd += 32) us += __popc(s.Ug[wd]);
        us = __reduce_add_sync(0xffffffffu, us);
        const unsigned lt = (1u << lane) - 1u;
        int base = 0;
        for (int k = 0; k < CPL; ++k) {
            const unsigned bk = __ballot_sync(0xffffffffu, (ing >> k) & 1u);
            if ((ing >> k) & 1u) s.order[pos + base + __popc(bk & lt)] = lane + 32 * k;
            base += __popc(bk);
        }
        if (lane == 0) {
            s.gstart[ng] = pos;
            s.gus[ng] = us;
            s.gsum[ng] = sum_s;
        }
        pos += cnt;
        ++ng;
        __syncwarp();
    }
    if (lane == 0) {
        s.gstart[ng] = pos;
        s.misc[0] = ng;
    }
}

// Greedy with the whole CTA for windows of 65..256 items whose compact sets fit
// in NWR words: thread t holds item t's set in registers.  A pick: each thread
// scores its item, each warp's best lane posts its key and set to shared memory
// (double-buffered by pick parity), one barrier, and every thread reduces the
// posted keys and ORs the winner's set into its copy of the running union.
// Same keys (pick_value << 9 | local_id) and so the same picks as greedy_reg.
template <int NWR, bool BUNDLE>
__device__ __noinline__ void greedy_block(const WinSmem& s, int n, int max_group) {
    constexpr bool bundle = BUNDLE;
    uint32_t* post = s.post;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarp = blockDim.x >> 5;
    const int pitch = s.misc[7], NWC = s.misc[1];
    // post[parity][warp] = {key, set words...}
    const int stride = NWR + 1;
    uint32_t sv[NWR], U[NWR];
#pragma unroll
    for (int x = 0; x < NWR; ++x) sv[x] = (tid < n && x < NWC) ? s.cs[(size_t)tid * pitch + x] : 0u;
    const int sz = tid < n ? s.ssize[tid] : 0;
    bool taken = tid >= n;
    int ng = 0, pos = 0, par = 0;
    // block-wide argmin of `key` (kNone when nothing); the winner's set ends in `win`
    auto block_pick = [&](unsigned key, uint32_t (&win)[NWR]) -> unsigned {
        const unsigned wmin = __reduce_min_sync(0xffffffffu, key);
        const unsigned hit = __ballot_sync(0xffffffffu, key == wmin);
        uint32_t* slot = post + (size_t)(par * nwarp + warp) * stride;
        if (lane == __ffs(hit) - 1) {
            slot[0] = wmin;
#pragma unroll
            for (int x = 0; x < NWR; ++x) slot[1 + x] = sv[x];
        }
        __syncthreads();
        unsigned best = kNone;
        int bw = 0;
        for (int w = 0; w < nwarp; ++w) {
            const unsigned k = post[(size_t)(par * nwarp + w) * stride];
            if (k < best) {
                best = k;
                bw = w;
            }
        }
#pragma unroll
        for (int x = 0; x < NWR; ++x) win[x] = post[(size_t)(par * nwarp + bw) * stride + 1 + x];
        par ^= 1;
        return best;
    };
    while (true) {
        uint32_t win[NWR];
        const unsigned seed = block_pick(taken ? kNone : (unsigned)tid, win);
        if (seed == kNone) break;
        bool ing = (int)seed == tid;
        if (ing) taken = true;
#pragma unroll
        for (int x = 0; x < NWR; ++x) U[x] = win[x];
        int cnt = 1;
        while (cnt < max_group) {
            int nc = 0;
#pragma unroll
            for (int x = 0; x < NWR; ++x) nc += __popc(sv[x] & ~U[x]);
            const unsigned best =
                block_pick(taken ? kNone : ((pick_value(nc, sz, bundle) << 9) | (unsigned)tid), win);
            if (best == kNone) break;
            if ((int)(best & 511u) == tid) {
                taken = true;
                ing = true;
            }
#pragma unroll
            for (int x = 0; x < NWR; ++x) U[x] |= win[x];
            ++cnt;
        }
        int us = 0;
#pragma unroll
        for (int x = 0; x < NWR; ++x) us += __popc(U[x]);
        // members in ascending local ID: prefix over the warps' ballots (one more barrier)
        const unsigned bal = __ballot_sync(0xffffffffu, ing);
        int* wcount = reinterpret_cast<int*>(post + (size_t)2 * nwarp * stride);  // [nwarp]
        int* wsum = wcount + nwarp;                                                // [nwarp]
        const int ssum = __reduce_add_sync(0xffffffffu, ing ? sz : 0);
        if (lane == 0) {
            wcount[warp] = __popc(bal);
            wsum[warp] = ssum;
        }
        __syncthreads();
        int before = 0, sum_s = 0;
        for (int w = 0; w < nwarp; ++w) {
            if (w < warp) before += wcount[w];
            sum_s += wsum[w];
        }
        if (ing) s.order[pos + before + __popc(bal & ((1u << lane) - 1u))] = tid;
        if (tid == 0) {
            s.gstart[ng] = pos;
            s.gus[ng] = us;
            s.gsum[ng] = sum_s;
        }
        pos += cnt;
        ++ng;
        __syncthreads();  // wcount / wsum are rewritten by the next group
    }
    if (tid == 0) {
        s.gstart[ng] = pos;
        s.misc[0] = ng;
    }
}

// The greedy on the compact sets: warp 0 for windows of up to 64 items (or wide
// sets), the whole CTA for larger windows of narrow sets; the CTA waits.  The greedy
// functions stay out of line: inlined into the kernel body they compiled to a
// loop several times slower.
template <bool BUNDLE>
__device__ __noinline__ void run_greedy_t(const WinSmem& s, int n, int max_group) {
    const int nwc = s.misc[1];
    // windows of 65..128 items with narrow compact sets: one warp, four items per lane
    const bool reg4 = n > 64 && n <= 128 && nwc <= 16;
    if (!reg4 && n > 64 && n <= (int)blockDim.x && blockDim.x <= 256 && nwc <= 8) {  // the whole CTA
        if (nwc <= 1) greedy_block<1, BUNDLE>(s, n, max_group);
        else if (nwc <= 2) greedy_block<2, BUNDLE>(s, n, max_group);
        else if (nwc <= 4) greedy_block<4, BUNDLE>(s, n, max_group);
        else greedy_block<8, BUNDLE>(s, n, max_group);
        __syncthreads();
        return;
    }
    if (threadIdx.x < 32) {
        const int NWC = s.misc[1];
        if (reg4) {
            if (NWC <= 2) greedy_reg<2, 4, BUNDLE>(s, n, max_group);
            else if (NWC <= 4) greedy_reg<4, 4, BUNDLE>(s, n, max_group);
            else if (NWC <= 6) greedy_reg<6, 4, BUNDLE>(s, n, max_group);
            else if (NWC <= 8) greedy_reg<8, 4, BUNDLE>(s, n, max_group);
            else if (NWC <= 12) greedy_reg<12, 4, BUNDLE>(s, n, max_group);
            else greedy_reg<16, 4, BUNDLE>(s, n, max_group);
        } else if (n <= 64 && NWC <= 32) {
            switch (NWC) {  // exact widths up to 8 words, then 12, 16, 24, 32
                case 0:
                case 1: greedy_reg<1, 2, BUNDLE>(s, n, max_group); break;
                case 2: greedy_reg<2, 2, BUNDLE>(s, n, max_group); break;
                case 3: greedy_reg<3, 2, BUNDLE>(s, n, max_group); break;
                case 4: greedy_reg<4, 2, BUNDLE>(s, n, max_group); break;
                case 5: greedy_reg<5, 2, BUNDLE>(s, n, max_group); break;
                case 6: greedy_reg<6, 2, BUNDLE>(s, n, max_group); break;
                case 7: greedy_reg<7, 2, BUNDLE>(s, n, max_group); break;
                case 8: greedy_reg<8, 2, BUNDLE>(s, n, max_group); break;
                default:
                    if (NWC <= 12) greedy_reg<12, 2, BUNDLE>(s, n, max_group);
                    else if (NWC <= 16) greedy_reg<16, 2, BUNDLE>(s, n, max_group);
                    else if (NWC <= 24) greedy_reg<24, 2, BUNDLE>(s, n, max_group);
                    else greedy_reg<32, 2, BUNDLE>(s, n, max_group);
            }
        } else {
            greedy_smem(s, n, max_group, BUNDLE);
        }
    }
    __syncthreads();
}

// The greedy on the compact sets of a window: groups (bundle = false) or bundles (true).
__device__ __forceinline__ void run_greedy(const WinSmem& s, int n, int max_group, bool bundle) {
    if (bundle)
        run_greedy_t<true>(s, n, max_group);
    else
        run_greedy_t<false>(s, n, max_group);
}

// Decoupled look-back (warp 0): publishes `agg` for item f and returns the sum
// of the aggregates of items [0, f).  status[] holds (flag << 62 | value).
__device__ long long lookback(uint64_t* status, int f, long long agg, unsigned* err, unsigned spin_limit) {
    const int lane = threadIdx.x & 31;
    volatile uint64_t* st = status;
    if (f == 0) {
        __threadfence();
        if (lane == 0) atomicExch(reinterpret_cast<unsigned long long*>(&status[0]),
                                  (unsigned long long)(kFlagIncl | (uint64_t)agg));
        return 0;
    }
    __threadfence();  // what this item wrote before the call is visible before its status
    if (lane == 0) atomicExch(reinterpret_cast<unsigned long long*>(&status[f]),
                              (unsigned long long)(kFlagAgg | (uint64_t)agg));
    long long excl = 0;
    int j = f - 1;  // lanes look at items j - lane
    unsigned spins = 0;
    while (j >= 0) {
        const int idx = j - lane;
        const uint64_t v = idx >= 0 ? st[idx] : (uint64_t)(2ull << 62);  // before item 0: an inclusive zero
        const unsigned not_ready = __ballot_sync(0xffffffffu, (v >> 62) == 0);
        const unsigned incl = __ballot_sync(0xffffffffu, (v >> 62) == 2);
        const int first_incl = incl ? __ffs(incl) - 1 : 32;
        // every lane up to and including the first inclusive one must have published
        const unsigned need = first_incl == 32 ? 0xffffffffu : (0xffffffffu >> (31 - first_incl));
        if (not_ready & need) {
            if (++spins > spin_limit) {
                if (lane == 0) atomicOr(err, QUP_ERR_TIMEOUT);
                break;
            }
            __nanosleep(32);
            continue;
        }
        long long part = (lane <= first_incl && idx >= 0) ? (long long)(v & kValMask) : 0;
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        excl += part;
        if (first_incl < 32) break;
        j -= 32;
    }
    if (lane == 0) atomicExch(reinterpret_cast<unsigned long long*>(&status[f]),
                              (unsigned long long)(kFlagIncl | (uint64_t)(excl + agg)));
    __threadfence();  // and what the earlier items wrote before theirs is visible after this
    return excl;
}


// ---------------------------------------------------------------- groups

// Per window counters, written before the window publishes its look-back
// status: visits, masked row slots, masked query slots, selected page edges.
// The last window of a KV head adds up its head's windows after its look-back
// (which implies every earlier window has published, and so written these).
// NT threads per CTA: 256 (two CTAs per SM), or 128 (four per SM) when the windows outnumber
// the CTAs that fit at 256 threads (the greedy of a window of at most 64 queries is one warp's
// work either way).
template <int NT>
__global__ void __launch_bounds__(NT, 65536 / (NT * 128)) grp_fused_kernel(
    const int32_t* __restrict__ topk, int Hq, int Hkv, int Nq, int K, int P, int NW, int max_group, int W,
    int nwin, int32_t* __restrict__ group_ptr, int32_t* __restrict__ members, int32_t* __restrict__ n_groups,
    int32_t* __restrict__ union_ptr, int32_t* __restrict__ union_pages, uint64_t* __restrict__ row_mask,
    int64_t* __restrict__ counters, uint32_t* __restrict__ gbits, int32_t* __restrict__ wcnt,
    uint64_t* __restrict__ status, unsigned* __restrict__ ticket, long long cap, unsigned* err,
    unsigned spin_limit) {
    extern __shared__ uint32_t sm_f1[];
    const int g = Hq / Hkv;
    uint32_t* rb = sm_f1;  // [W][g][NW] page bitset of every TopK row of the window
    const WinSmem s = carve(sm_f1 + (size_t)W * g * NW, W, NW);
    __shared__ long long s_base;
    constexpr int kWarps = NT / 32;
    __shared__ int s_red[kWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    grid_dep_launch();  // the bundle kernel may take free SMs now; it waits for this grid
    const int items = Hkv * nwin;
    __shared__ int s_f;
    for (;;) {
        if (tid == 0) s_f = (int)atomicAdd(ticket, 1u);  // windows in claim order
        __syncthreads();
        const int f = s_f;
        if (f >= items) break;
        const int h = f / nwin, w = f % nwin;
        const int w0 = w * W, nw = min(W, Nq - w0);
        // ---- TopK rows -> row bitsets (-1 is padding, out-of-range IDs are reported and dropped).
        // One thread per (query, Q head) row owns that row's bitset words: no two threads update
        // one word (rows that select the same pages would otherwise collide on shared-memory
        // atomics), and the row's IDs are read with 16-byte loads when K allows it.
        for (int x = tid; x < nw * g * NW; x += blockDim.x) rb[x] = 0u;
        __syncthreads();
        for (int row = tid; row < nw * g; row += blockDim.x) {
            const int i = row / g, j = row - i * g;
            const int32_t* src = topk + ((size_t)(h * g + j) * Nq + w0 + i) * K;
            uint32_t* dst = rb + ((size_t)i * g + j) * NW;
            auto put = [&](int pg) {
                if (pg == -1) return;
                if (pg < 0 || pg >= P) {
                    atomicOr(err, QUP_ERR_PAGE_ID);
                    return;
                }
                dst[pg >> 5] |= 1u << (pg & 31);
            };
            if ((K & 3) == 0 && (reinterpret_cast<uintptr_t>(topk) & 15) == 0) {
                const int4* s4 = reinterpret_cast<const int4*>(src);
                for (int k0 = 0; k0 < K / 4; k0 += 4) {
                    int4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) v[u] = k0 + u < K / 4 ? s4[k0 + u] : make_int4(-1, -1, -1, -1);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        put(v[u].x);
                        put(v[u].y);
                        put(v[u].z);
                        put(v[u].w);
                    }
                }
            } else {  // 16 loads in flight at a time (the stores to dst could alias src for the compiler)
                for (int k0 = 0; k0 < K; k0 += 16) {
                    int v[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) v[u] = k0 + u < K ? __ldg(src + k0 + u) : -1;
#pragma unroll
                    for (int u = 0; u < 16; ++u) put(v[u]);
                }
            }
        }
        __syncthreads();
        // ---- S(i): union over the g rows of query i; total row bits of the window
        int rbits = 0;
        for (int x = tid; x < nw * NW; x += blockDim.x) {
            const int i = x / NW, wd = x - i * NW;
            uint32_t v = 0;
            for (int j = 0; j < g; ++j) {
                const uint32_t r = rb[((size_t)i * g + j) * NW + wd];
                v |= r;
                rbits += __popc(r);
            }
            s.S[x] = v;
        }
        rbits = __reduce_add_sync(0xffffffffu, rbits);
        if (lane == 0) s_red[warp] = rbits;
        __syncthreads();
        compact_window(s, nw, NW);
        run_greedy(s, nw, max_group, false);
        const int ng = s.misc[0];
        // ---- offsets: group prefix inside the window, window prefix by look-back
        if (warp == 0) {
            int carry = 0;
            for (int k0 = 0; k0 < ng; k0 += 32) {
                const int k = k0 + lane;
                const int c = k < ng ? s.gus[k] : 0;
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (k < ng) s.goff[k] = carry + incl - c;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) s.goff[ng] = carry;
            // window counters first (read by the head's last window after its look-back)
            // masked row slots = sum over groups of |U| x rows - the window's row bits (every
            // row's pages lie in its group's union)
            int mq = 0, ed = 0, mr = 0;
            for (int k = lane; k < ng; k += 32) {
                const int cnt = s.gstart[k + 1] - s.gstart[k];
                mq += cnt * s.gus[k] - s.gsum[k];
                mr += cnt * g * s.gus[k];
            }
            for (int a = lane; a < nw; a += 32) ed += s.ssize[a];
            mq = __reduce_add_sync(0xffffffffu, mq);
            ed = __reduce_add_sync(0xffffffffu, ed);
            mr = __reduce_add_sync(0xffffffffu, mr);
            if (lane == 0) {
                wcnt[f * 4 + 0] = carry;
                int rb_total = 0;
                for (int x = 0; x < kWarps; ++x) rb_total += s_red[x];
                wcnt[f * 4 + 1] = mr - rb_total;
                wcnt[f * 4 + 2] = mq;
                wcnt[f * 4 + 3] = ed;
            }
            const long long base = lookback(status, f, carry, err, spin_limit);
            if (lane == 0) s_base = base;
        }
        __syncthreads();
        const long long base = s_base;
        const int total = s.goff[ng];
        const bool fits = base + total <= cap;
        if (tid == 0 && !fits) atomicOr(err, QUP_ERR_CAPACITY);
        const int gbase = w * (W / max_group);
        // ---- emit: one warp per group; lane r holds row r of the group (row = member rank * g +
        // head; max_group * g <= 32), so the union word is one OR reduction and each page's row
        // mask one ballot
        for (int k = warp; k < ng; k += kWarps) {
            const int m0 = s.gstart[k], cnt = s.gstart[k + 1] - m0, R = cnt * g;
            const int gi = gbase + k;
            for (int m = lane; m < cnt; m += 32) members[(size_t)h * Nq + w0 + m0 + m] = w0 + s.order[m0 + m];
            if (lane == 0) {
                group_ptr[(size_t)h * (Nq + 1) + gi] = w0 + m0;
                union_ptr[(size_t)h * (Nq + 1) + gi] = (int32_t)(base + s.goff[k]);
            }
            const uint32_t* row0 =
                lane < R ? rb + ((size_t)s.order[m0 + lane / g] * g + (lane % g)) * NW : nullptr;
            long long out = base + s.goff[k];
            for (int wd = 0; wd < NW; ++wd) {
                // the 32 x 32 bit block (row = lane, page = bit) transposed: lane b ends with page
                // wd * 32 + b's row mask
                uint32_t x = row0 ? row0[wd] : 0u;
                transpose32(x, lane);
                const uint32_t u = __ballot_sync(0xffffffffu, x != 0u);
                // the group's union bitset (for the bundle pass) and its pages in order
                if (lane == 0) gbits[((size_t)h * Nq + gi) * NW + wd] = u;
                if (fits && x != 0u) {
                    const long long e = out + __popc(u & ((1u << lane) - 1u));
                    union_pages[e] = wd * 32 + lane;
                    row_mask[e] = (uint64_t)x;
                }
                out += __popc(u);
            }
        }
        if (tid == 0) {
            if (w == nwin - 1) {  // the window holding the head's last query
                n_groups[h] = gbase + ng;
                group_ptr[(size_t)h * (Nq + 1) + gbase + ng] = w0 + nw;
                union_ptr[(size_t)h * (Nq + 1) + gbase + ng] = (int32_t)(base + total);
            }
        }
        if (w == nwin - 1 && warp == 0) {
            // counters of the head: every window of it wrote its wcnt before publishing
            // its look-back status, and this window's look-back has seen all of them
            long long c0 = 0, c1 = 0, c2 = 0, c3 = 0;
            for (int x = h * nwin + lane; x <= f; x += 32) {
                const volatile int32_t* wc = wcnt + (size_t)x * 4;
                c0 += wc[0];
                c1 += wc[1];
                c2 += wc[2];
                c3 += wc[3];
            }
            for (int o = 16; o > 0; o >>= 1) {
                c0 += __shfl_xor_sync(0xffffffffu, c0, o);
                c1 += __shfl_xor_sync(0xffffffffu, c1, o);
                c2 += __shfl_xor_sync(0xffffffffu, c2, o);
                c3 += __shfl_xor_sync(0xffffffffu, c3, o);
            }
            if (lane == 0) {
                counters[h * 4 + 0] = c0;
                counters[h * 4 + 1] = c1;
                counters[h * 4 + 2] = c2;
                counters[h * 4 + 3] = c3;
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- bundles

constexpr int kOrderBuckets2 = 4096;

// Counting sort of the flat bundle indices by union size, largest first, equal
// sizes by index (sizes above kOrderBuckets2 - 1 share the top bucket).  Whole
// CTA; `sm` holds kOrderBuckets2 + 64 + Hkv + 1 ints, then room for `kcap`
// ints.  When all keys fit there (and per-warp tables of the keys' range),
// every warp scatters a contiguous chunk; otherwise warp 0 scatters alone.
__device__ void order_bundles(int* sm, int kcap, const int32_t* n_bundles, const int32_t* bunion_ptr, int Hkv,
                              int Nq, int32_t* order) {
    int* cursor = sm;
    int* warp_sum = sm + kOrderBuckets2;
    int* head_start = warp_sum + 64;
    int* keys = head_start + Hkv + 1;
    __shared__ int s_kmin, s_kmax;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x, nwarp = nt >> 5;
    if (warp == 0) {  // head_start = exclusive prefix of the bundle counts (lanes load them at once)
        int carry = 0;
        for (int h0 = 0; h0 < Hkv; h0 += 32) {
            const int h = h0 + lane;
            int c = h < Hkv ? __ldcg(n_bundles + h) : 0;
            c = (c >= 0 && c <= Nq) ? c : 0;  // the attention kernel reports a bad count
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (h < Hkv) head_start[h] = carry + incl - c;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            head_start[Hkv] = carry;
            s_kmin = kOrderBuckets2;
            s_kmax = -1;
        }
    }
    for (int k = tid; k < kOrderBuckets2; k += nt) cursor[k] = 0;
    __syncthreads();
    const int n = head_start[Hkv];
    auto key_of = [&](int f) {
        int h = 0;
        while (head_start[h + 1] <= f) ++h;
        const size_t b = (size_t)h * (Nq + 1) + (f - head_start[h]);
        const int size = __ldcg(bunion_ptr + b + 1) - __ldcg(bunion_ptr + b);
        return kOrderBuckets2 - 1 - min(max(size, 0), kOrderBuckets2 - 1);  // larger union -> smaller key
    };
    const bool cached = n <= kcap;
    int lo = kOrderBuckets2, hi = -1;
    for (int f = tid; f < n; f += nt) {
        const int key = key_of(f);
        if (cached) keys[f] = key;
        atomicAdd(&cursor[key], 1);
        lo = min(lo, key);
        hi = max(hi, key);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
        atomicMin(&s_kmin, lo);
        atomicMax(&s_kmax, hi);
    }
    __syncthreads();
    // exclusive scan of the histogram: each thread owns a contiguous run of buckets
    const int per = kOrderBuckets2 / nt;
    int run = 0;
    for (int k = 0; k < per; ++k) run += cursor[tid * per + k];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < nwarp ? warp_sum[lane] : 0;
        int wi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        if (lane < nwarp) warp_sum[32 + lane] = wi - v;
    }
    __syncthreads();
    int acc = warp_sum[32 + warp] + incl - run;
    for (int k = 0; k < per; ++k) {
        const int c = cursor[tid * per + k];
        cursor[tid * per + k] = acc;
        acc += c;
    }
    __syncthreads();
    const int kmin = s_kmin, R = s_kmax - s_kmin + 1;
    // stable scatter of a chunk: 32 flat indices at a time, equal keys ranked by lane
    auto scatter = [&](int f0, int f1, int* cur, int koff) {
        for (int fb = f0; fb < f1; fb += 32) {
            const int f = fb + lane;
            const unsigned live = __ballot_sync(0xffffffffu, f < f1);
            if (f < f1) {
                const int key = cached ? keys[f] : key_of(f);
                const unsigned peers = __match_any_sync(live, key);
                const int leader = __ffs(peers) - 1;
                const int rank = __popc(peers & ((1u << lane) - 1u));
                int start = 0;
                if (lane == leader) {
                    start = cur[key - koff];
                    cur[key - koff] = start + __popc(peers);
                }
                start = __shfl_sync(live, start, leader);
                order[start + rank] = f;
            }
            __syncwarp();
        }
    };
    if (cached && n > 0 && (size_t)R * nwarp <= (size_t)(kcap - n)) {
        // per-warp cursors: warp w's chunk of equal keys starts after the earlier chunks' ones
        int* tab = keys + n;  // [nwarp][R]
        const int chunk = (n + nwarp - 1) / nwarp;
        for (int x = tid; x < R * nwarp; x += nt) tab[x] = 0;
        __syncthreads();
        const int f0 = min(n, warp * chunk), f1 = min(n, f0 + chunk);
        for (int f = f0 + lane; f < f1; f += 32) atomicAdd(&tab[warp * R + keys[f] - kmin], 1);
        __syncthreads();
        for (int k = tid; k < R; k += nt) {
            int running = cursor[kmin + k];
            for (int w = 0; w < nwarp; ++w) {
                const int c = tab[w * R + k];
                tab[w * R + k] = running;
                running += c;
            }
        }
        __syncthreads();
        scatter(f0, f1, tab + warp * R, kmin);
    } else if (warp == 0) {
        scatter(0, n, cursor, 0);
    }
}

// Bundles: windows of WB groups of one KV head; greedy packs up to `slots`
// page-affine groups into one 128-row work item.  The window counters (bundle
// page visits) and the bundle count of a head are written like the groups'.
__global__ void __launch_bounds__(kFusedThreads, 2) bnd_fused_kernel(
    const uint32_t* __restrict__ gbits, int Hkv, int Nq, int NW, int g, int RS, int slots, int WB, int nwinB,
    const int32_t* __restrict__ n_groups, const int32_t* __restrict__ group_ptr,
    const int32_t* __restrict__ members, const int32_t* __restrict__ union_ptr,
    const int32_t* __restrict__ union_pages, const uint64_t* __restrict__ row_mask,
    int32_t* __restrict__ n_bundles, int32_t* __restrict__ bundle_ptr, int32_t* __restrict__ bundle_groups,
    int32_t* __restrict__ bunion_ptr, int32_t* __restrict__ bunion_pages, uint32_t* __restrict__ bunion_mask,
    int32_t* __restrict__ bundle_qid, int64_t* __restrict__ bcounters, int32_t* __restrict__ bundle_order,
    int32_t* __restrict__ wcnt, uint64_t* __restrict__ status, unsigned* __restrict__ done,
    unsigned* __restrict__ ticket, long long cap, unsigned* err, unsigned spin_limit, int order_kcap, int ecap) {
    extern __shared__ uint32_t sm_f2[];
    const WinSmem s = carve(sm_f2, WB, NW);
    // per warp: the bundle's union bitset and its word prefix counts
    uint32_t* wscr = sm_f2 + (win_smem_bytes(WB, NW, 0) - 64) / 4;
    __shared__ long long s_base;
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t* Ub = wscr + (size_t)warp * (2 * NW + 1);
    int* pw = reinterpret_cast<int*>(Ub + NW);
    // the window's group offsets: member starts and union starts, [WB + 1] each
    int* gp = reinterpret_cast<int*>(wscr + (size_t)kFusedWarps * (2 * NW + 1));
    int* up = gp + WB + 1;
    // the window's group union entries (page, low 32 mask bits) when at most ecap of them
    int* epg = up + WB + 1;
    uint32_t* emk = reinterpret_cast<uint32_t*>(epg + ecap);
    const int MQ = 128 / g, rpg = RS / g;
    grid_dep_launch();  // the attention kernel may start its prologue
    grid_dep_wait();    // the group kernel's outputs are complete and visible
    const int items = Hkv * nwinB;
    __shared__ int s_f;
    for (;;) {
        if (tid == 0) s_f = (int)atomicAdd(ticket, 1u);  // windows in claim order
        __syncthreads();
        const int f = s_f;
        if (f >= items) break;
        const int h = f / nwinB, wbi = f % nwinB;
        int ngh = n_groups[h];
        if (ngh < 0 || ngh > Nq) {
            if (tid == 0) atomicOr(err, QUP_ERR_GROUP);
            ngh = 0;
        }
        const int w0 = wbi * WB, nw = max(0, min(WB, ngh - w0));
        for (int x = tid; x < nw * NW; x += blockDim.x) s.S[x] = gbits[((size_t)h * Nq + w0) * NW + x];
        for (int x = tid; x <= nw; x += blockDim.x) {
            gp[x] = group_ptr[(size_t)h * (Nq + 1) + w0 + x];
            up[x] = union_ptr[(size_t)h * (Nq + 1) + w0 + x];
        }
        __syncthreads();
        const int e_base = nw > 0 ? up[0] : 0, n_ent = nw > 0 ? up[nw] - up[0] : 0;
        const bool ent_smem = n_ent >= 0 && n_ent <= ecap;
        if (ent_smem)
            for (int x = tid; x < n_ent; x += blockDim.x) {
                epg[x] = union_pages[e_base + x];
                emk[x] = (uint32_t)row_mask[e_base + x];
            }
        // (the barriers inside the greedy below order these stores before the emission)
        int ng = 0;
        if (nw > 0) {
            compact_window(s, nw, NW);
            run_greedy(s, nw, slots, true);
            ng = s.misc[0];
        }
        if (warp == 0) {
            int carry = 0;
            for (int k0 = 0; k0 < ng; k0 += 32) {
                const int k = k0 + lane;
                const int c = k < ng ? s.gus[k] : 0;
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (k < ng) s.goff[k] = carry + incl - c;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) {
                s.goff[ng] = carry;
                wcnt[f] = carry;
            }
            const long long base = lookback(status, f, carry, err, spin_limit);
            if (lane == 0) s_base = base;
        }
        __syncthreads();
        const long long base = s_base;
        const int total = ng > 0 ? s.goff[ng] : 0;
        const bool fits = base + total <= cap;
        if (tid == 0 && !fits) atomicOr(err, QUP_ERR_CAPACITY);
        const int bbase = wbi * (WB / slots);
        for (int k = warp; k < ng; k += kFusedWarps) {
            const int b0 = s.gstart[k], cnt = s.gstart[k + 1] - b0;
            const int bi = bbase + k;
            const long long out0 = base + s.goff[k];
            for (int m = lane; m < cnt; m += 32) bundle_groups[(size_t)h * Nq + w0 + b0 + m] = w0 + s.order[b0 + m];
            if (lane == 0) {
                bundle_ptr[(size_t)h * (Nq + 1) + bi] = w0 + b0;
                bunion_ptr[(size_t)h * (Nq + 1) + bi] = (int32_t)out0;
            }
            // row -> query table: slot j holds group j's members, rows_per_group / g queries each
            int32_t* qt = bundle_qid + ((size_t)h * Nq + bi) * MQ;
            for (int x = lane; x < MQ; x += 32) qt[x] = -1;
            __syncwarp();
            for (int x = lane; x < cnt * rpg; x += 32) {  // slot j = x / rpg, member m = x % rpg
                const int j = x / rpg, m = x - j * rpg, a = s.order[b0 + j];
                const int m0 = gp[a], m1 = gp[a + 1];
                if (m < m1 - m0) qt[x] = members[(size_t)h * Nq + m0 + m];
            }
            // bundle union bitset and its word prefix counts
            for (int wd = lane; wd < NW; wd += 32) {
                uint32_t u = 0;
                for (int j = 0; j < cnt; ++j) u |= s.S[(size_t)s.order[b0 + j] * NW + wd];
                Ub[wd] = u;
            }
            __syncwarp();
            int carry = 0;
            for (int x0 = 0; x0 < NW; x0 += 32) {
                const int wd = x0 + lane;
                const int c = wd < NW ? __popc(Ub[wd]) : 0;
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (wd < NW) pw[wd] = carry + incl - c;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            __syncwarp();
            if (fits) {
                // pages in order, masks zeroed
                for (int wd = lane; wd < NW; wd += 32) {
                    uint32_t u = Ub[wd];
                    long long e = out0 + pw[wd];
                    while (u) {
                        const int b = __ffs(u) - 1;
                        u &= u - 1;
                        bunion_pages[e] = wd * 32 + b;
                        reinterpret_cast<uint4*>(bunion_mask)[e] = make_uint4(0u, 0u, 0u, 0u);
                        ++e;
                    }
                }
                __syncwarp();
                // each slot's row masks, placed by the page's rank in the bundle union; the
                // entries of all slots form one flat range so their loads overlap (slot
                // starts are held by lanes 0..cnt-1: at most 32 slots)
                const uint32_t keep = RS == 32 ? 0xffffffffu : ((1u << RS) - 1u);
                if (cnt <= 32) {
                    const int a = lane < cnt ? s.order[b0 + lane] : 0;
                    const int len = lane < cnt ? up[a + 1] - up[a] : 0;
                    int incl = len;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    const int start = incl - len, tot = __shfl_sync(0xffffffffu, incl, 31);
                    const int u0 = lane < cnt ? up[a] : 0;
                    for (int t0 = 0; t0 < tot; t0 += 32) {
                        const int t = t0 + lane;
                        int j = 0;
                        for (int q = 1; q < cnt; ++q) j += __shfl_sync(0xffffffffu, start, q) <= t ? 1 : 0;
                        const int e = __shfl_sync(0xffffffffu, u0, j) + t - __shfl_sync(0xffffffffu, start, j);
                        if (t < tot) {
                            const int pg = ent_smem ? epg[e - e_base] : union_pages[e];
                            const int wd = pg >> 5;
                            if (pg >= 0 && wd < NW) {
                                const int pos = pw[wd] + __popc(Ub[wd] & ((1u << (pg & 31)) - 1u));
                                const uint32_t mk = (ent_smem ? emk[e - e_base] : (uint32_t)row_mask[e]) & keep;
                                const int bit0 = j * RS;
                                if (mk) atomicOr(&bunion_mask[(out0 + pos) * 4 + (bit0 >> 5)], mk << (bit0 & 31));
                            }
                        }
                    }
                } else {
                    for (int j = 0; j < cnt; ++j) {
                        const int a = s.order[b0 + j];
                        const int bit0 = j * RS;
                        for (int e = up[a] + lane; e < up[a + 1]; e += 32) {
                            const int pg = union_pages[e];
                            const int wd = pg >> 5;
                            if (pg < 0 || wd >= NW) continue;
                            const int pos = pw[wd] + __popc(Ub[wd] & ((1u << (pg & 31)) - 1u));
                            const uint32_t mk = (uint32_t)row_mask[e] & keep;
                            if (mk) atomicOr(&bunion_mask[(out0 + pos) * 4 + (bit0 >> 5)], mk << (bit0 & 31));
                        }
                    }
                }
            }
            __syncwarp();
        }
        if (tid == 0) {
            const int last_w = ngh > 0 ? (ngh - 1) / WB : 0;
            if (wbi == last_w) {  // the window holding the head's last group writes the head's ends
                n_bundles[h] = bbase + ng;
                bundle_ptr[(size_t)h * (Nq + 1) + bbase + ng] = w0 + nw;
                bunion_ptr[(size_t)h * (Nq + 1) + bbase + ng] = (int32_t)(base + total);
                bcounters[h * 2 + 1] = bbase + ng;
            }
        }
        if (warp == 0 && wbi == nwinB - 1) {  // page visits of the head: sum of its windows
            long long c0 = 0;
            for (int x = h * nwinB + lane; x <= f; x += 32) c0 += *(volatile int32_t*)(wcnt + x);
            for (int o = 16; o > 0; o >>= 1) c0 += __shfl_xor_sync(0xffffffffu, c0, o);
            if (lane == 0) bcounters[h * 2 + 0] = c0;
        }
        __syncthreads();
    }
    // the last CTA to finish sorts the bundles for the attention kernel
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_last) {
        __threadfence();
        order_bundles(reinterpret_cast<int*>(sm_f2), order_kcap, n_bundles, bunion_ptr, Hkv, Nq, bundle_order);
    }
}

}  // namespace

// ---------------------------------------------------------------- host side

size_t fused_group_smem(int W, int g, int NW) {
    return 4 * (size_t)W * g * NW + win_smem_bytes(W, NW, 0);
}

// order keys cached in shared memory by the sorting CTA (more bundles: read twice)
constexpr int kOrderKeyCap = 8192;
// group union entries of one bundle window kept in shared memory (more: read from global)
constexpr int kBundleEntryCap = 4096;

size_t fused_bundle_smem(int WB, int NW, int Hkv) {
    const size_t a = win_smem_bytes(WB, NW, kFusedWarps * (2 * NW + 1) + 2 * (WB + 1) + 2 * kBundleEntryCap);
    const size_t b = 4 * (size_t)(kOrderBuckets2 + 64 + Hkv + 1 + kOrderKeyCap) + 64;
    return a > b ? a : b;
}

// CTAs that can be resident at once for `kernel` with `smem` bytes: the grid of
// a look-back kernel never exceeds it (every window waited on must be running).
// (cached per device, kernel and shared-memory size)
template <typename Kern>
static int resident_ctas(Kern kernel, size_t smem, int sms, int threads = kFusedThreads) {
    struct Entry {
        int dev;
        const void* fn;
        size_t smem;
        int per_sm;
    };
    static std::mutex mu;
    static Entry table[64];
    static int n = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < n; ++i)
        if (table[i].dev == dev && table[i].fn == (const void*)kernel && table[i].smem == smem)
            return table[i].per_sm * sms;
    int per_sm = 0;
    // the kernels want shared memory, not L1: ask for the largest carveout before counting
    cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    if (n < 64) table[n++] = Entry{dev, (const void*)kernel, smem, per_sm};
    return per_sm * sms;
}

cudaError_t launch_group_fused(const GroupLaunch& a, uint32_t* gbits, int32_t* wcnt, uint64_t* status,
                               unsigned* ticket, cudaStream_t stream) {
    const int g = a.Hq / a.Hkv;
    const size_t smem = fused_group_smem(a.W, g, a.NW);
    const int items = a.Hkv * a.nwin;
    cudaError_t e = ensure_smem_attr((const void*)grp_fused_kernel<256>, smem);
    if (e != cudaSuccess) return e;
    int grid = std::min(items, resident_ctas(grp_fused_kernel<256>, smem, a.sms, 256));
    if (items > grid && a.W <= 64) {  // more windows than CTAs: four smaller CTAs per SM
        e = ensure_smem_attr((const void*)grp_fused_kernel<128>, smem);
        if (e != cudaSuccess) return e;
        grid = std::min(items, resident_ctas(grp_fused_kernel<128>, smem, a.sms, 128));
        grp_fused_kernel<128><<<grid, 128, smem, stream>>>(
            a.topk, a.Hq, a.Hkv, a.Nq, a.K, a.P, a.NW, a.max_group, a.W, a.nwin, a.group_ptr, a.members, a.n_groups,
            a.union_ptr, a.union_pages, a.row_mask, a.counters, gbits, wcnt, status, ticket, a.cap, a.err, 1u << 22);
        return cudaGetLastError();
    }
    grp_fused_kernel<256><<<grid, 256, smem, stream>>>(
        a.topk, a.Hq, a.Hkv, a.Nq, a.K, a.P, a.NW, a.max_group, a.W, a.nwin, a.group_ptr, a.members, a.n_groups,
        a.union_ptr, a.union_pages, a.row_mask, a.counters, gbits, wcnt, status, ticket, a.cap, a.err, 1u << 22);
    return cudaGetLastError();
}

cudaError_t launch_bundles_fused(const BundleLaunch& a, int32_t* wcnt, uint64_t* status, unsigned* done,
                                 unsigned* ticket, cudaStream_t stream) {
    const size_t smem = fused_bundle_smem(a.WB, a.NW, a.Hkv);
    cudaError_t e = ensure_smem_attr((const void*)bnd_fused_kernel, smem);
    if (e != cudaSuccess) return e;
    const int items = a.Hkv * a.nwin;
    const int grid = std::max(1, std::min(items, resident_ctas(bnd_fused_kernel, smem, a.sms)));
    return launch_pdl(bnd_fused_kernel, dim3(grid), dim3(kFusedThreads), smem, stream,
        (const uint32_t*)a.gbits, a.Hkv, a.Nq, a.NW, a.g, a.RS, a.slots, a.WB, a.nwin, a.n_groups, a.group_ptr, a.members,
        a.union_ptr, a.union_pages, a.row_mask, a.n_bundles, a.bundle_ptr, a.bundle_groups, a.bunion_ptr,
        a.bunion_pages, a.bunion_mask, a.bundle_qid, a.bcounters, a.bundle_order, wcnt, status, done, ticket, a.cap, a.err,
        1u << 22, (int)((smem - 64) / 4 - (kOrderBuckets2 + 64 + a.Hkv + 1)), kBundleEntryCap);
}


}  // namespace qup

