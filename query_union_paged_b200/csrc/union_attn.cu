// union_attn.cu -- ID-aware union attention for sm_100a (PageWeaver,
// Abstract; Figure 1; Figure 3), re-designed for tcgen05 + TMEM.
//
// Work item: a bundle of up to 128 query rows (up to 128 / rows_per_group
// page-affine groups of one KV head, see qup_groups); each CTA claims its
// bundles at run time, largest unions first (the walk, below).  Pages of the bundle
// union are streamed once per bundle in steps of 128 tokens (one 128-token
// page, or 128 / T smaller pages) through two TMA rings, one of K tiles and
// one of V tiles.  Step s of a bundle belongs to softmax warpgroup w = s % 2,
// which owns S buffer w and O accumulator w in TMEM:
//      S_w  = Q K^T     M = 128 rows, N = 128 tokens, K = d  (Q and K from shared memory)
//      P_w  = masked online softmax of S_w, written over S_w  (TMEM -> registers -> TMEM)
//      O_w += P_w V     M = 128 rows, N = d, K = 128 tokens   (P from TMEM, V from shared memory)
// Thread = TMEM lane = bundle row in both warpgroups, so a row's running max
// and sum never leave its thread; each warpgroup keeps its own for its steps.
// While one warpgroup computes the exponentials of step s, the other works on
// step s + 1 and the tensor pipe runs the O update of step s - 1 and S of step
// s + 2: the serial chain of one warp (TMEM load, row max, exponentials, P
// store) is hidden behind the other warp of its SM sub-partition.  The
// epilogue merges the two partial results of each row (O_0, O_1 with their
// maxima and sums) and writes the row to O[qid][h'].
// A row's max is only raised when a score exceeds it by more than kTau (log2
// units); O_w and the row sum are rescaled then, which after the first steps
// is rare.  A warp whose 32 rows selected none of a step's pages skips that
// step's exponentials.  Each softmax warp reads the bundle's page numbers and
// its own 32-bit word of every page's row mask straight from the bundle
// arrays, 32 entries at a time, one batch ahead.  On a page that reaches past
// the end of its sequence the scores there become -inf and the PV warp zeroes
// the V rows there (they may hold non-finite bytes).  Two (bf16) or three (E4M3) pairs in eight of the exponentials come
// from a polynomial on the FMA pipe (exp2_poly2), the rest from the MUFU unit.
// E4M3 P goes to a shared-memory tile of the warpgroup (its S buffer is then
// free as soon as the scores are in registers); bf16 and fp32 P go over S.
//
// Q: the bundle's rows, gathered by original query ID (no reordered Q tensor),
// sit in shared memory as the A operand of S in the 128-byte-swizzled K-major
// layout.  bf16: the V producer loads them by TMA (one box of g heads x 64
// elements per query and half of d; empty query slots read zeros from outside
// the tensor) once every S of the previous bundle has completed.  E4M3: the V
// producer bulk-copies the bf16 rows into a stage, and the softmax warpgroups
// quantise each row to E4M3 with its own scale into the operand (each writes
// half of every row).  fp32: the two warpgroups copy the rows from global
// memory, half each.
//
// Warp roles (384 threads; warp w runs on SM sub-partition w % 4):
//   warps 0-3   softmax warpgroup 0 (even steps), warps 4-7 warpgroup 1 (odd
//               steps); both run the epilogue, each for half of the columns.
//   warp 8      K producer: claims the CTA's bundles and publishes them to
//               the other roles; walks each bundle's page list, resolves
//               physical pages (warp-parallel) and TMA-loads the K tiles.
//   warp 10     V producer: the same walk for the V tiles; writes each
//               bundle's header (item and query IDs of its rows) and loads
//               or stages its Q rows.
//   warp 9      S issuer (one elected lane of a warp-uniform loop) and TMEM
//               owner (512 columns): S(s) once K tile s has landed and the O
//               update that last read P from S_w has finished.
//   warp 11     PV issuer: O_w += P_w V once P(s) and V tile s are ready.
// Producers and issuers wait with suspended try_waits, which leave the
// sub-partition's issue slots to the softmax warps, and give registers to
// them (setmaxnreg).
// TMEM columns: O_0 [0,128); O_1 [128,256); S_0 [256,384); S_1 [384,512).
// P_w occupies the first kPCols columns of S_w.
// Operand types: bf16 (kind::f16), fp32 (kind::tf32), FP8 E4M3
// (kind::f8f6f4: K and V straight from the cache, Q quantised per row with
// its own scale, P stored as E4M3 of 2^4 p).  Every MMA consumes 32 bytes of
// its K extent per row, so the descriptor arithmetic is shared.
//
// Every wait is bounded (ptx.cuh); on a timeout the CTA raises an abort flag,
// drains its in-flight TMA loads and MMAs, frees TMEM and exits.  The two
// softmax warpgroups meet only on mbarriers (bounded waits), never on a
// named barrier.
#include <cstdint>
#include <cuda.h>

#include "internal.h"
#include "ptx.cuh"
#include "query_union_paged.h"

namespace qup {

constexpr int kThreads = 384;
constexpr int kRows = 128;
constexpr int kD = kHeadDim;
constexpr int kST = 128;  // tokens per pipeline step
constexpr int kTmemCols = 512;
constexpr int kSoftmaxWarps = 8;
constexpr int kKProducerWarp = 8, kSWarp = 9, kVProducerWarp = 10, kPvWarp = 11;
constexpr uint32_t kColO = 0, kColS = 256;  // O_w at kColO + 128 w, S_w at kColS + 128 w
// Register split: the launch gives every thread kLaunchRegs (384 x 168 = 64,512 of the SM's
// 65,536); the producer and issuer warpgroup gives back down to kOtherRegs and the two softmax
// warpgroups take kSoftmaxRegs: 256 x 208 + 128 x 88 = 64,512, exactly the launch's total.
constexpr int kLaunchRegs = 168, kSoftmaxRegs = 208, kOtherRegs = 88;
static_assert(256 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs, "register split");

template <int ES, int T>
struct Geo {
    static constexpr int PPS = T < kST ? kST / T : 1;   // pages per step
    static constexpr int BOXR = T < 64 ? T : 64;        // token rows per TMA box
    static constexpr int BPP = T / BOXR;                // boxes per page (along tokens)
    static constexpr int kTile = kST * kD * ES;         // one K or V tile of a step
    static constexpr int kChunkElems = 128 / ES;        // elements per 128-byte swizzle row
    static constexpr int kNChunk = kD * ES / 128;       // 128-byte chunks along d
    static constexpr int kChunkBytes = kST * 128;       // one chunk column of a K or V tile
    static constexpr int kQBytes = kRows * kD * ES;     // the Q operand of a bundle
    static constexpr int kQChunkBytes = kRows * 128;    // one chunk column of the Q operand
    static constexpr int kMmaK = 32 / ES;               // K elements per MMA instruction
    static constexpr int kNumMmaS = kD * ES / 32;       // MMAs per S (K = d)
    static constexpr int kNumMmaPV = kST * ES / 32;     // MMAs per O update (K = 128 tokens)
    static constexpr int kPCols = kST * ES / 4;         // TMEM columns of P
    static_assert(kPCols <= 128, "P fits in its S buffer");
    // E4M3: P goes to shared memory (one 16 KB K-major tile per warpgroup), so S_w is free as
    // soon as the softmax has loaded it; the other types write P over S in TMEM
    static constexpr bool kPSmem = ES == 1;
    static constexpr int kPBytes = kRows * kST * ES;    // one warpgroup's P tile in shared memory
    // exponentials on the FMA pipe by a polynomial for pairs (j / 2) % 8 < kPolyPairs of every 16
    // columns, the rest on the MUFU unit (measured on this part per 128-score step of a warp: E4M3
    // pack 809 cycles with 3 pairs, 832 with 2, 1,040 with none; bf16 pack 887 with 2)
    static constexpr int kPolyPairs = ES == 1 ? 3 : 2;
    static_assert(PPS <= kMaxPPS, "pages per step");
    static constexpr uint32_t kFmt = (ES == 2) ? 1u : (ES == 4 ? 2u : 0u);
    static constexpr int kKind = (ES == 2) ? 0 : (ES == 4 ? 1 : 2);
    static constexpr float kTau = ES == 1 ? 4.5f : 8.f;  // lazy-rescale margin (log2 units)
    // E4M3 P is stored as 2^kPLog2 p (p <= 2^kTau, so at most 2^8.5 < 448, E4M3's largest
    // finite value; a P below 2^-10 of its row's max is a subnormal of E4M3); the row sum
    // carries the same factor, which cancels in O / l
    static constexpr float kPLog2 = ES == 1 ? 4.f : 0.f;
};

struct SmemLayout {
    uint32_t kst, vst, q, p, qst, sinfo, mrg, bars, misc, walk, total;
};

// Stage of the next bundle (E4M3: its bf16 Q rows): query slot m holds the g rows of its query,
// 256 bytes each, at m * qstage_stride(g); the 16-byte pad keeps row reads free of bank conflicts.
__host__ __device__ inline uint32_t qstage_stride(int g) { return (uint32_t)g * 256u + 16u; }
constexpr int kSinfoWords = 8;  // bundle header: flat bundle, h, bi, ub, nU, nsteps, ok
constexpr int kWalkRing = 64;    // entries of the walk's shared-memory ring (a power of two)
constexpr int kWalkReaders = 11; // roles that read the walk: softmax warps 0-7, V, S and PV warps
constexpr int kFixedBars = 16;

__host__ __device__ inline SmemLayout smem_layout(int es, int nsk, int nsv, int Hkv, int g) {
    SmemLayout L;
    const uint32_t MQ = (uint32_t)(kRows / g);
    uint32_t off = 0;
    L.kst = off;
    off += (uint32_t)nsk * kST * kD * es;
    L.vst = off;
    off += (uint32_t)nsv * kST * kD * es;
    L.q = off;  // 1024-aligned: every tile above is a multiple of 16 KB
    off += (uint32_t)kRows * kD * es;
    L.p = off;  // E4M3: the two warpgroups' P tiles (1024-aligned)
    if (es == 1) off += 2u * kRows * kST;
    L.qst = off;
    if (es == 1) off += MQ * qstage_stride(g);
    L.sinfo = off;
    off += 4u * (kSinfoWords + MQ);  // header, qid[MQ]
    L.mrg = off;
    off += 2u * kRows * 8u;  // per warpgroup and row: running max and sum (float2)
    off = (off + 7u) & ~7u;
    L.bars = off;
    off += 8u * (2u * (nsk + nsv) + kFixedBars);
    L.misc = off;
    off += 16u + 4u * (uint32_t)(Hkv + 1);
    off = (off + 15u) & ~15u;
    L.walk = off;  // the walk: ring, published count, readers' progress
    off += 4u * (kWalkRing + 1 + kWalkReaders);
    L.total = off + 1024u;  // slack for aligning the dynamic base to 1024
    return L;
}

// barrier block: K ring full/empty, V ring full/empty, then the fixed barriers
struct Bars {
    uint32_t base;
    int nsk, nsv;
    __device__ __forceinline__ uint32_t kfull(int s) const { return base + 8u * s; }
    __device__ __forceinline__ uint32_t kempty(int s) const { return base + 8u * (nsk + s); }
    __device__ __forceinline__ uint32_t vfull(int s) const { return base + 8u * (2 * nsk + s); }
    __device__ __forceinline__ uint32_t vempty(int s) const { return base + 8u * (2 * nsk + nsv + s); }
    __device__ __forceinline__ uint32_t fixed(int i) const { return base + 8u * (2 * (nsk + nsv) + i); }
    __device__ __forceinline__ uint32_t sfull(int w) const { return fixed(w); }       // S_w computed
    __device__ __forceinline__ uint32_t pfull(int w) const { return fixed(2 + w); }   // P_w stored
    __device__ __forceinline__ uint32_t pvdone(int w) const { return fixed(4 + w); }  // O_w += P_w V done
    __device__ __forceinline__ uint32_t qfull() const { return fixed(6); }   // the bundle's Q operand is in place
    __device__ __forceinline__ uint32_t qfree() const { return fixed(7); }   // every S of the bundle completed
    __device__ __forceinline__ uint32_t stfull() const { return fixed(8); }  // header (and E4M3 stage) written
    __device__ __forceinline__ uint32_t stempty() const { return fixed(9); } // header read by every softmax warp
    __device__ __forceinline__ uint32_t ep1() const { return fixed(10); }    // both row states published
    __device__ __forceinline__ uint32_t ep2() const { return fixed(11); }    // both halves of O read
    __device__ __forceinline__ uint32_t sfree(int w) const { return fixed(12 + w); }  // S_w loaded (P in smem)
    __device__ __forceinline__ uint32_t drain() const { return fixed(14); }
    __device__ __forceinline__ uint32_t drain2() const { return fixed(15); }
};

struct Item {
    int h, bi, ub, nU, nsteps;
    bool ok;
};

// Decode flat bundle f; every role calls this and reaches the same verdict.
template <int PPS>
__device__ __forceinline__ Item load_item(const AttnParams& p, const int* nb_prefix, int f) {
    Item it;
    int h = 0;
    while (h + 1 < p.Hkv && nb_prefix[h + 1] <= f) ++h;
    it.h = h;
    it.bi = f - nb_prefix[h];
    const size_t bp = (size_t)h * (p.bstride + 1) + it.bi;
    it.ub = p.union_ptr[bp];
    it.nU = p.union_ptr[bp + 1] - it.ub;
    it.ok = it.ub >= 0 && it.nU >= 0 && (long long)it.ub + it.nU <= p.cap_union;
    if (!it.ok) it.nU = 0;
    it.nsteps = (it.nU + PPS - 1) / PPS;
    return it;
}

// ------------------------------------------------------------------ the walk of bundles
// Bundles are handed out at run time: the K warp of each CTA takes the next position of
// the bundle order (largest unions first) from a counter shared by the whole grid, so a
// CTA on a slower SM simply takes fewer bundles.  It publishes the claimed bundles, in
// order, in a ring in shared memory (-1 ends the walk); every other role reads the
// same sequence from the ring and records how far it has read, and the K warp does not
// overwrite an entry before every reader has read it.
//
// One counter pair per launch slot: [0] claims, [1] CTAs done.  The last CTA to finish
// resets both, so the next launch given the same slot starts from zero; the host hands
// out the slots in turn, so up to kWalkSlots launches may run at once.
__device__ unsigned g_walk_ticket[kWalkSlots][2];

constexpr int kReaderV = 8, kReaderS = 9, kReaderPV = 10;  // walk readers after the softmax warps

struct Walk {
    int* ring;           // [kWalkRing] flat bundle indices, -1: end of the walk
    volatile int* pub;   // entries published so far
    volatile int* prog;  // [kWalkReaders] entries each reader has read
};

// Bounded spin of one thread until cond() holds; false (and the abort flag and
// QUP_ERR_TIMEOUT set) when it runs out, false without an error when another role aborted.
template <class F>
__device__ __forceinline__ bool spin_until(F cond, volatile int* abort_flag, unsigned* err, uint64_t limit_ns) {
    if (cond()) return true;
    const uint64_t t0 = cycles();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (cond()) return true;
        if ((it & 15u) == 0) {
            if (*abort_flag) return false;
            if (cycles() - t0 > limit_ns * kCyclesPerNs) {
                *abort_flag = 1;
                atomicOr(err, QUP_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Entry j of the walk for reader `reader` (warp-collective; lane 0 waits): the flat bundle
// index, -1 at the end of the walk or when the wait gave up.
__device__ __forceinline__ int walk_get(const Walk& wk, int j, int reader, volatile int* abort_flag, unsigned* err,
                                        uint64_t limit_ns, int lane) {
    int f = -1;
    if (lane == 0) {
        if (spin_until([&] { return *wk.pub > j; }, abort_flag, err, limit_ns)) {
            __threadfence_block();
            f = *reinterpret_cast<volatile int*>(wk.ring + (j & (kWalkRing - 1)));
        }
        __threadfence_block();  // the entry is read before the K warp may reuse it
        wk.prog[reader] = j + 1;
    }
    return __shfl_sync(0xffffffffu, f, 0);
}

// K warp, lane 0: claim and publish entry j (once every reader has read entry j - kWalkRing).
// Bad order entries are reported and skipped.  Returns the published value.
__device__ __forceinline__ int walk_publish(const Walk& wk, int j, const AttnParams& p, unsigned* ticket, int n_items,
                                            volatile int* abort_flag, uint64_t limit_ns) {
    int f = -1;
    const bool room = spin_until(
        [&] {
            int lo = 0x7fffffff;
#pragma unroll
            for (int r = 0; r < kWalkReaders; ++r) lo = min(lo, wk.prog[r]);
            return lo > j - kWalkRing;
        },
        abort_flag, p.err, limit_ns);
    __threadfence_block();  // the readers' progress is seen before the entry is rewritten
    if (room) {
        for (;;) {
            const unsigned t = atomicAdd(ticket, 1u);
            if (t >= (unsigned)n_items) break;
            const int ff = p.bundle_order[t];
            if (ff >= 0 && ff < n_items) {
                f = ff;
                break;
            }
            atomicOr(p.err, QUP_ERR_GROUP);
        }
    }
    wk.ring[j & (kWalkRing - 1)] = f;
    __threadfence_block();
    *wk.pub = j + 1;
    return f;
}

// byte offset of 16-byte chunk c of row r inside a K-major SW128 operand tile of `rows` rows
__device__ __forceinline__ uint32_t kmajor_sw128(int r, int c, int rows) {
    return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ bool warp_ok(bool ok) { return __all_sync(0xffffffffu, ok); }

// Valid tokens of logical page u (0..T): tokens past the end of its sequence are never attended
// and may hold any bytes.  One sequence: kv_len; batched requests: the per-page count.
__device__ __forceinline__ int page_valid(const AttnParams& p, int u, int T) {
    return p.page_len ? p.page_len[u] : max(0, min(T, p.kv_len - u * T));
}

template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t* v) {
    if constexpr (N == 8) {
        tmem_st_x8(taddr, v);
    } else if constexpr (N == 16) {
        tmem_st_x16(taddr, v);
    } else {
        static_assert(N % 32 == 0, "stores come in 8, 16 or 32-column pieces");
#pragma unroll
        for (int i = 0; i < N / 32; ++i) tmem_st_x32(taddr + 32u * i, v + 32 * i);
    }
}

template <int ES, int T>
__global__ void __launch_bounds__(kThreads, 1)
    union_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ AttnParams p) {
    using G = Geo<ES, T>;
    constexpr int PPS = G::PPS, BOXR = G::BOXR, BPP = G::BPP;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const SmemLayout L = smem_layout(ES, p.nsk, p.nsv, p.Hkv, p.g);
    const int NSK = p.nsk, NSV = p.nsv;
    const uint32_t sbase = smem_u32(smem);
    const Bars B{sbase + L.bars, NSK, NSV};
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
    int* nb_prefix = reinterpret_cast<int*>(smem + L.misc + 16);
    const Walk wk{reinterpret_cast<int*>(smem + L.walk), reinterpret_cast<volatile int*>(smem + L.walk) + kWalkRing,
                  reinterpret_cast<volatile int*>(smem + L.walk) + kWalkRing + 1};
    unsigned* const ticket = g_walk_ticket[(unsigned)p.walk_slot < (unsigned)kWalkSlots ? p.walk_slot : 0];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t lim = p.wait_limit_ns;
    const int g = p.g, MQ = kRows / g;

    // ---------------------------------------------------------------- setup
    // barriers, TMEM and the tensor maps first; the kernel ahead in the stream may
    // still be running (programmatic launch): its outputs are read after grid_dep_wait
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSK; ++s) {
            mbar_init(B.kfull(s), 1);
            mbar_init(B.kempty(s), 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(B.vfull(s), 1);
            mbar_init(B.vempty(s), 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(B.sfull(w), 1);
            mbar_init(B.pfull(w), 4);  // one arrive per warp of softmax warpgroup w
            mbar_init(B.pvdone(w), 1);
        }
        mbar_init(B.qfull(), ES == 2 ? 1 : kSoftmaxWarps);  // bf16: the TMA transactions; else the softmax warps
        for (int w = 0; w < 2; ++w) mbar_init(B.sfree(w), 4);
        mbar_init(B.qfree(), 1);
        mbar_init(B.stfull(), 1);
        mbar_init(B.stempty(), kSoftmaxWarps);
        mbar_init(B.ep1(), kSoftmaxWarps);
        mbar_init(B.ep2(), kSoftmaxWarps);
        mbar_init(B.drain(), 1);
        mbar_init(B.drain2(), 1);
        fence_mbar_init();
        *abort_flag = 0;
        *wk.pub = 0;
        for (int r = 0; r < kWalkReaders; ++r) wk.prog[r] = 0;
    }
    if (threadIdx.x == kKProducerWarp * 32) prefetch_tensormap(&tmK);
    if (threadIdx.x == kVProducerWarp * 32) {
        prefetch_tensormap(&tmV);
        if constexpr (ES == 2) prefetch_tensormap(&tmQ);
    }
    if (warp == kSWarp) {
        tmem_alloc(smem_u32((const void*)tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    grid_dep_wait();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int h = 0; h < p.Hkv; ++h) {
            nb_prefix[h] = acc;
            int n = p.n_bundles[h];
            if (n < 0 || n > p.bstride) {
                atomicOr(p.err, QUP_ERR_GROUP);
                n = 0;
            }
            acc += n;
        }
        nb_prefix[p.Hkv] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_items = nb_prefix[p.Hkv];

    if (warp >= kSoftmaxWarps) {
        regs_decrease<kOtherRegs>();
        if (warp == kKProducerWarp || warp == kVProducerWarp) {
            // ======================================================== producers (whole warp each)
            // Both walk the same bundles and pages; the K warp fills the K ring, the V warp the V
            // ring, writes each bundle's header and loads (bf16) or stages (E4M3) its Q rows.
            const bool isV = warp == kVProducerWarp;
            const int NR = isV ? NSV : NSK;
            const CUtensorMap* tm = isV ? &tmV : &tmK;
            const uint32_t ring = sbase + (isV ? L.vst : L.kst);
            int gs = 0, n_done = 0;
            bool ok = true;
            for (int j = 0; ok; ++j) {
                // the K warp claims the CTA's next bundle once it has issued every K tile of the
                // previous one; the V warp reads the same entry of the walk
                int f = -1;
                if (!isV) {
                    if (lane == 0) f = walk_publish(wk, j, p, ticket, n_items, abort_flag, lim);
                    f = __shfl_sync(0xffffffffu, f, 0);
                } else {
                    f = walk_get(wk, j, kReaderV, abort_flag, p.err, lim, lane);
                }
                if (f < 0) break;
                const Item it = load_item<PPS>(p, nb_prefix, f);
                if (isV) {
                    // the header, once every softmax warp has read the previous bundle's
                    if (n_done > 0) {
                        int okv = 0;
                        if (lane == 0)
                            okv = mbar_wait_idle(B.stempty(), (n_done - 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT,
                                                 lim);
                        ok = __shfl_sync(0xffffffffu, okv, 0) != 0;
                        if (!ok) break;
                    }
                    int* sinfo = reinterpret_cast<int*>(smem + L.sinfo);
                    int nvalid = 0;
                    for (int m0 = 0; m0 < MQ; m0 += 32) {
                        const int m = m0 + lane;
                        int qid = -1;
                        if (m < MQ) {
                            qid = p.bundle_qid[((size_t)it.h * p.bstride + it.bi) * MQ + m];
                            if (qid >= p.Nq) {
                                atomicOr(p.err, QUP_ERR_GROUP);
                                qid = -1;
                            }
                            qid = max(qid, -1);
                            sinfo[kSinfoWords + m] = qid;
                        }
                        nvalid += __popc(__ballot_sync(0xffffffffu, qid >= 0));
                    }
                    if (lane == 0) {
                        sinfo[0] = f;
                        sinfo[1] = it.h;
                        sinfo[2] = it.bi;
                        sinfo[3] = it.ub;
                        sinfo[4] = it.nU;
                        sinfo[5] = it.nsteps;
                        sinfo[6] = it.ok ? 1 : 0;
                    }
                    __syncwarp();
                    if constexpr (ES == 1) {
                        // the bf16 Q rows, by query ID (the g rows of a query are contiguous in Q)
                        const uint32_t qbytes = (uint32_t)g * kD * 2u;
                        if (lane == 0) mbar_arrive_expect_tx(B.stfull(), (uint32_t)nvalid * qbytes);
                        __syncwarp();
                        for (int m = lane; m < MQ; m += 32) {
                            const int qid = sinfo[kSinfoWords + m];
                            if (qid >= 0)
                                bulk_g2s(sbase + L.qst + (uint32_t)m * qstage_stride(g),
                                         static_cast<const uint16_t*>(p.Q) + ((size_t)qid * p.Hq + (size_t)it.h * g) * kD,
                                         qbytes, B.stfull());
                        }
                    } else {
                        if (lane == 0) mbar_arrive(B.stfull());
                    }
                    if constexpr (ES == 2) {
                        // the Q operand by TMA, once every S of the previous bundle has completed: per
                        // query slot and half of d one box of g rows; an empty slot reads zeros from
                        // outside the tensor
                        if (n_done > 0) {
                            int okv = 0;
                            if (lane == 0)
                                okv = mbar_wait_idle(B.qfree(), (n_done - 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT,
                                                     lim);
                            ok = __shfl_sync(0xffffffffu, okv, 0) != 0;
                            if (!ok) break;
                        }
                        if (lane == 0) mbar_arrive_expect_tx(B.qfull(), (uint32_t)G::kQBytes);
                        __syncwarp();
                        for (int m = lane; m < MQ; m += 32) {
                            const int qid = sinfo[kSinfoWords + m];
                            const int qc = qid >= 0 ? qid : p.Nq;
#pragma unroll
                            for (int kb = 0; kb < 2; ++kb)
                                tma_load_3d(sbase + L.q + (uint32_t)kb * G::kQChunkBytes + (uint32_t)(m * g) * 128u, &tmQ,
                                            B.qfull(), kb * 64, it.h * g, qc);
                        }
                    }
                    ++n_done;
                }
                const int n_ent = it.nsteps * PPS;  // incl. padding of the last step
                for (int e0 = 0; e0 < n_ent && ok; e0 += 32) {
                    const int idx = e0 + lane;
                    int u = 0, phys = p.P_phys;  // P_phys: outside the tensor, TMA fills zeros
                    if (idx < it.nU) {
                        u = p.union_pages[it.ub + idx];
                        if (u < 0 || u >= p.num_logical_pages) {
                            atomicOr(p.err, QUP_ERR_PAGE_ID);
                            u = 0;
                        } else {
                            phys = p.page_table[u];
                            if (phys < 0 || phys >= p.P_phys) {
                                atomicOr(p.err, QUP_ERR_PHYS_PAGE);
                                phys = p.P_phys;
                            }
                        }
                    }
                    const int nst = min(32, n_ent - e0) / PPS;  // 32 is a multiple of PPS
                    for (int k = 0; k < nst; ++k, ++gs) {
                        const int slot = gs % NR;
                        int okv = 0;
                        if (lane == 0)
                            okv = mbar_wait_idle(isV ? B.vempty(slot) : B.kempty(slot), ((gs / NR) & 1) ^ 1,
                                                 abort_flag, p.err, QUP_ERR_TIMEOUT, lim);
                        ok = __shfl_sync(0xffffffffu, okv, 0) != 0;
                        if (!ok) break;
                        const bool issue = lane == 0 && !(p.dbg_skip_stage >= 0 && gs == p.dbg_skip_stage);
                        int ph[PPS];
#pragma unroll
                        for (int q = 0; q < PPS; ++q) ph[q] = __shfl_sync(0xffffffffu, phys, k * PPS + q);
                        if (issue) {
                            const uint32_t fb = isV ? B.vfull(slot) : B.kfull(slot);
                            mbar_arrive_expect_tx(fb, G::kTile);
                            const uint32_t dst = ring + (uint32_t)slot * G::kTile;
#pragma unroll
                            for (int q = 0; q < PPS; ++q) {
#pragma unroll
                                for (int bb = 0; bb < BPP; ++bb) {
#pragma unroll
                                    for (int c = 0; c < G::kNChunk; ++c) {
                                        const uint32_t off =
                                            (uint32_t)c * G::kChunkBytes + (uint32_t)(q * T + bb * BOXR) * 128u;
                                        tma_load_4d(dst + off, tm, fb, c * G::kChunkElems, bb * BOXR, it.h, ph[q]);
                                    }
                                }
                            }
                        }
                        __syncwarp();
                    }
                }
            }
            // every issued load lands before the CTA may exit: the last NR stages of this ring,
            // and the last bundle's staged or loaded Q rows
            if (lane == 0) {
                if (isV && n_done > 0) {
                    if constexpr (ES == 1) mbar_wait_drain(B.stfull(), (n_done - 1) & 1, lim);
                    if constexpr (ES == 2) mbar_wait_drain(B.qfull(), (n_done - 1) & 1, lim);
                }
                for (int i = max(0, gs - NR); i < gs; ++i) {
                    if (p.dbg_skip_stage >= 0 && i == p.dbg_skip_stage) continue;
                    mbar_wait_drain(isV ? B.vfull(i % NR) : B.kfull(i % NR), (i / NR) & 1, lim);
                }
            }
            __syncwarp();
        } else {
            // ======================================================== MMA issuers (whole warp, one elected lane)
            //   S warp:  S_w = Q K^T for step s (w = s % 2): needs the bundle's Q operand, K tile s,
            //            and the O update that last read P from S_w finished; commits S-full(w) and
            //            the K slot, and after the bundle's last S the Q-free barrier.
            //   PV warp: O_w += P_w V: needs P(s) and V tile s; commits PV-done(w) and the V slot.
            // The first O update of each accumulator in a bundle overwrites it; its P is stored
            // after both warpgroups have read the previous bundle's O (the epilogue's barrier).
            const bool isS = warp == kSWarp;
            const uint32_t idesc_s = instr_desc(G::kFmt, 0, 0, kST, kRows);
            const uint32_t idesc_o = instr_desc(G::kFmt, 0, 1, kD, kRows);
            // V as the MN-major B operand (N = d): 128-byte swizzle with 8-row atoms; tf32
            // has only the 128-byte swizzle with 32-byte atoms (layout 1, 4-row atoms)
            constexpr uint32_t vlayout = ES == 4 ? 1u : 2u;
            constexpr uint32_t vsbo = ES == 4 ? 512u : 1024u;
            const uint64_t qdesc = smem_desc(sbase + L.q, 16, 1024, 2);
            int use[2] = {0, 0}, item_no = 0;
            int ks = 0, kph = 0, vs = 0, vph = 0;  // ring slot and phase of the next step
            bool ok = true;
            for (int rnd = 0; ok; ++rnd) {
                const int f = walk_get(wk, rnd, isS ? kReaderS : kReaderPV, abort_flag, p.err, lim, lane);
                if (f < 0) break;
                const Item it = load_item<PPS>(p, nb_prefix, f);
                if (isS) {
                    ok = warp_ok(mbar_wait_idle(B.qfull(), item_no & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                    if (!ok) break;
                    tc_fence_after();
                    for (int s = 0; s < it.nsteps; ++s) {
                        const int w = s & 1, k = use[w];
                        // S_w is free once its previous use has been read: by the softmax (P in
                        // shared memory) or by the O update (P over S in TMEM)
                        ok = warp_ok(mbar_wait_idle(B.kfull(ks), kph, abort_flag, p.err, QUP_ERR_TIMEOUT, lim) &&
                                     (k < 1 || mbar_wait_idle(G::kPSmem ? B.sfree(w) : B.pvdone(w), (k - 1) & 1,
                                                              abort_flag, p.err, QUP_ERR_TIMEOUT, lim)));
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t kdesc = smem_desc(sbase + L.kst + (uint32_t)ks * G::kTile, 16, 1024, 2);
                        if (elect_one_sync()) {
#pragma unroll
                            for (int kk = 0; kk < G::kNumMmaS; ++kk) {
                                const uint32_t koff = ((kk >> 2) * G::kChunkBytes + (kk & 3) * 32) >> 4;
                                const uint32_t qoff = ((kk >> 2) * G::kQChunkBytes + (kk & 3) * 32) >> 4;
                                tc_mma<G::kKind>(tmem + kColS + 128u * w, qdesc + qoff, kdesc + koff, idesc_s, kk > 0);
                            }
                            tc_commit(B.sfull(w));
                            tc_commit(B.kempty(ks));
                        }
                        __syncwarp();
                        ++use[w];
                        if (++ks == NSK) {
                            ks = 0;
                            kph ^= 1;
                        }
                    }
                    if (!ok) break;
                    if (elect_one_sync()) tc_commit(B.qfree());
                    __syncwarp();
                } else {
                    // The bundle's union entries, 32 at a time (lane j: entry cb + j); a page that
                    // reaches past kv_len may hold non-finite bytes there: its V rows past kv_len
                    // are zeroed before the O update reads the tile (P is 0 there, but 0 * NaN is not)
                    int cb = -32, cpg = -1;
                    for (int s = 0; s < it.nsteps; ++s) {
                        const int w = s & 1, k = use[w];
                        const int e0 = s * PPS;
                        if (e0 >= cb + 32) {
                            cb = e0 - (e0 & 31);
                            const int e = cb + lane;
                            cpg = e < it.nU ? p.union_pages[it.ub + e] : -1;
                            if (cpg >= p.num_logical_pages) cpg = -1;
                        }
                        bool tail = false;
#pragma unroll
                        for (int q = 0; q < PPS; ++q) {
                            const int pg = __shfl_sync(0xffffffffu, cpg, e0 - cb + q);
                            tail |= pg >= 0 && page_valid(p, pg, T) < T;
                        }
                        ok = warp_ok(mbar_wait_idle(B.pfull(w), k & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim) &&
                                     mbar_wait_idle(B.vfull(vs), vph, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                        if (!ok) break;
                        if (tail) {
                            uint8_t* vt = smem + L.vst + (uint32_t)vs * G::kTile;
#pragma unroll 1
                            for (int q = 0; q < PPS; ++q) {
                                const int pg = __shfl_sync(0xffffffffu, cpg, e0 - cb + q);
                                const int t0 = pg < 0 ? T : page_valid(p, pg, T);  // first token row past kv_len
                                if (t0 >= T) continue;
                                const int nwords = (T - t0) * G::kNChunk * 8;  // 16-byte words to clear
                                for (int i = lane; i < nwords; i += 32) {
                                    const int row = q * T + t0 + i / (G::kNChunk * 8);
                                    const int rest = i % (G::kNChunk * 8);
                                    *reinterpret_cast<uint4*>(vt + (rest >> 3) * G::kChunkBytes + row * 128 +
                                                              (rest & 7) * 16) = make_uint4(0, 0, 0, 0);
                                }
                            }
                            fence_proxy_async_smem();  // zeroed rows -> the tensor core
                            __syncwarp();
                        }
                        tc_fence_after();
                        const uint64_t vdesc = smem_desc(sbase + L.vst + (uint32_t)vs * G::kTile,
                                                         (uint32_t)G::kChunkBytes, vsbo, vlayout);
                        const uint64_t pdesc = smem_desc(sbase + L.p + (uint32_t)w * G::kPBytes, 16, 1024, 2);
                        if (elect_one_sync()) {
#pragma unroll
                            for (int kk = 0; kk < G::kNumMmaPV; ++kk) {
                                // K step = kMmaK tokens: 32 bytes of each P row, kMmaK rows of V
                                if constexpr (G::kPSmem)
                                    tc_mma<G::kKind>(tmem + kColO + 128u * w, pdesc + ((kk * 32) >> 4),
                                                     vdesc + ((kk * G::kMmaK * 128) >> 4), idesc_o, s >= 2 || kk > 0);
                                else
                                    tc_mma_ts<G::kKind>(tmem + kColO + 128u * w, tmem + kColS + 128u * w + 8u * kk,
                                                        vdesc + ((kk * G::kMmaK * 128) >> 4), idesc_o, s >= 2 || kk > 0);
                            }
                            tc_commit(B.pvdone(w));
                            tc_commit(B.vempty(vs));
                        }
                        __syncwarp();
                        ++use[w];
                        if (++vs == NSV) {
                            vs = 0;
                            vph ^= 1;
                        }
                    }
                }
                ++item_no;
            }
            // every MMA this warp issued completes before TMEM is freed
            const uint32_t dbar = isS ? B.drain() : B.drain2();
            if (elect_one_sync()) tc_commit(dbar);
            __syncwarp();
            mbar_wait_drain(dbar, 0, lim);
            __syncwarp();
        }
    } else {
        regs_increase<kSoftmaxRegs>();
        // ============================================================ softmax / epilogue (warps 0-7)
        const int w = warp >> 2;          // warpgroup: the steps s with s % 2 == w
        const int wq = warp & 3;          // TMEM lane quarter of this warp
        const int r = wq * 32 + lane;     // bundle row == TMEM lane
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const uint32_t colS = kColS + 128u * w, colO = kColO + 128u * w;
        const float kNegInf = -__int_as_float(0x7f800000);
        const float kPosInf = __int_as_float(0x7f800000);
        const int* sinfo = reinterpret_cast<const int*>(smem + L.sinfo);
        float2* mrg = reinterpret_cast<float2*>(smem + L.mrg);  // [2][kRows]
        int use = 0;  // this warpgroup's uses of S_w and O_w so far
        bool ok = true;
        // the row's bundle state: item, query (original ID), Q head, visible positions, score scale
        Item it{};
        int qid = -1, head = 0, vis_end = 0, fl = 0;
        float cs = p.scale_log2, vscale = 1.f;
        float m_used = kNegInf, lsum = 0.f;
        f2 cs2{cs, cs};
        // The bundle's union entries, 32 at a time: lane j holds entry base + j, its logical
        // page (-1 for padding or an entry the producers reject) and this warp's 32-bit word
        // of the page's row mask.  The next 32 are loaded one batch ahead.
        // A page whose tokens reach past the end of its sequence (a tail page) may hold non-finite
        // bytes there: its entry carries a tail flag.
        int cpage = -1, npage = -1;
        uint32_t cmask = 0u, nmask = 0u;
        bool ctail = false, ntail = false;
        int cbase = 0;
        auto fetch = [&](int base, int& pg, uint32_t& mk, bool& tl) {
            const int e = base + lane;
            pg = -1;
            mk = 0u;
            tl = false;
            if (e < it.nU) {
                const int u = p.union_pages[it.ub + e];
                const uint32_t m = p.row_mask[(size_t)(it.ub + e) * 4 + wq];
                if (u >= 0 && u < p.num_logical_pages) {
                    const int ph = p.page_table[u];
                    if (ph >= 0 && ph < p.P_phys) {
                        pg = u;
                        mk = m;
                        tl = page_valid(p, u, T) < T;
                    }
                }
            }
        };
        // Take over the ino-th bundle of this CTA from the header the V warp wrote: its item, this
        // row's query (original ID) and position, the first union entries.  For the non-bf16
        // types both warpgroups write the Q operand (E4M3: quantised per row from the staged bf16
        // rows; fp32: from global memory), half of each row each, once every S of the previous
        // bundle has completed.  Releases the header.
        auto take = [&](int ino) -> bool {
            if (!warp_ok(mbar_wait(B.stfull(), ino & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim))) return false;
            fl = sinfo[0];
            it.h = sinfo[1];
            it.bi = sinfo[2];
            it.ub = sinfo[3];
            it.nU = sinfo[4];
            it.nsteps = sinfo[5];
            it.ok = sinfo[6] != 0;
            qid = sinfo[kSinfoWords + r / g];
            // positions < this end are visible to the query (batched requests: its precomputed end
            // in the global token space); loaded alongside the first union entries
            const int qend = qid < 0 ? 0 : (p.q_end ? p.q_end[qid] : min(p.q_pos[qid] + 1, p.kv_len));
            if (!it.ok && threadIdx.x == 0) atomicOr(p.err, QUP_ERR_GROUP);
            head = it.h * g + (r % g);
            vis_end = qend;  // positions < vis_end are visible
            cs = p.scale_log2;                  // score scale (log2 domain) of this row
            cbase = 0;
            fetch(0, cpage, cmask, ctail);
            fetch(32, npage, nmask, ntail);
            if constexpr (ES == 1) vscale = p.v_scale[it.h];
            if constexpr (ES != 2) {
                // the Q operand, once every S of the previous bundle has completed: each warpgroup
                // writes half of every row's 128-byte chunks
                if (ino > 0 && !warp_ok(mbar_wait(B.qfree(), (ino - 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim)))
                    return false;
                uint8_t* qt = smem + L.q;
                if constexpr (ES == 4) {
                    const size_t row_off = ((size_t)(qid >= 0 ? qid : 0) * p.Hq + head) * kD;
                    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(p.Q) + row_off);
#pragma unroll
                    for (int c = 16 * w; c < 16 * w + 16; ++c) {
                        const uint4 v = qid >= 0 ? src[c] : make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4*>(qt + kmajor_sw128(r, c, kRows)) = v;
                    }
                } else {  // the whole row's amax, then this half: bf16 -> E4M3 with the row's scale amax / 448
                    const uint8_t* row = smem + L.qst + (uint32_t)(r / g) * qstage_stride(g) + (uint32_t)(r % g) * 256u;
                    uint4 raw[16];
                    float amax = 0.f;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        raw[c] = qid >= 0 ? *reinterpret_cast<const uint4*>(row + c * 16) : make_uint4(0, 0, 0, 0);
                        const uint32_t w4[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w4[e] << 16)),
                                                     fabsf(__uint_as_float(w4[e] & 0xffff0000u))));
                    }
                    const float inv = amax > 0.f ? 448.f / amax : 0.f;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {  // 16 bf16 -> 16 E4M3 (one 16-byte chunk)
                        if ((c >> 2) != w) continue;
                        uint32_t qv[4];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint4 v = raw[2 * c + hh];
                            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                            float x[8];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                x[2 * e] = __uint_as_float(w4[e] << 16) * inv;
                                x[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u) * inv;
                            }
                            qv[2 * hh] = pack_e4m3x4(x[0], x[1], x[2], x[3]);
                            qv[2 * hh + 1] = pack_e4m3x4(x[4], x[5], x[6], x[7]);
                        }
                        *reinterpret_cast<uint4*>(qt + kmajor_sw128(r, c, kRows)) = make_uint4(qv[0], qv[1], qv[2], qv[3]);
                    }
                    cs = amax * (1.f / 448.f) * p.k_scale[it.h] * p.scale_log2;
                }
                fence_proxy_async_smem();  // generic-proxy writes of Q -> the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(B.qfull());
            }
            // a Q row of zeros (E4M3 scale 0) keeps a positive score scale: its scores are 0 anyway
            cs = fmaxf(cs, 1e-30f);
            cs2 = f2{cs, cs};
            __syncwarp();
            if (lane == 0) mbar_arrive(B.stempty());
            return true;
        };
        // entry rr of the CTA's walk of bundles: -1 past the end
        auto walk = [&](int rr) -> int { return walk_get(wk, rr, warp, abort_flag, p.err, lim, lane); };
        // exponentials of one step: p = 2^(s*cs - m_used + kPLog2), their sum returned.  P leaves
        // every 16 tokens as it is made (E4M3: one 16-byte chunk of row r of this warpgroup's
        // shared-memory P tile; bf16: 8 TMEM columns over S_w), so no more than a chunk of it is
        // ever held in registers; fp32 P is written over sv and stored by the caller.
        uint32_t sv[kST];
        uint8_t* const ptile = smem + L.p + (uint32_t)w * G::kPBytes;
        auto exps = [&](const int (&lim_q)[PPS], uint32_t s_addr) -> float {
            const float mb = (m_used == kNegInf ? 0.f : m_used) - G::kPLog2;
            f2 part[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
            f2 e_prev{0.f, 0.f};  // E4M3: the first pair of a 4-token word
            uint32_t ck[8];       // the current 16-token chunk of P (bf16: 8 words, E4M3: 4)
#pragma unroll
            for (int q = 0; q < PPS; ++q) {  // one page (T tokens) at a time
                // a page the row did not select gets an infinite offset: 2^-inf = 0
                const float off = lim_q[q] == 0 ? kPosInf : mb;
                const f2 noff{-off, -off};
#pragma unroll
                for (int j = q * T; j < (q + 1) * T; j += 2) {
                    const f2 y = fma2(f2{__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])}, cs2, noff);
                    f2 e;
                    if (((j >> 1) & 7) < G::kPolyPairs) {
                        e = exp2_poly2(y);
                    } else {
                        e.x = ex2(y.x);
                        e.y = ex2(y.y);
                    }
                    part[(j >> 1) & 3] = add2(part[(j >> 1) & 3], e);
                    if constexpr (ES == 2) {
                        ck[(j & 15) >> 1] = pack_bf16x2(e.x, e.y);
                        if ((j & 15) == 14) tmem_st_x8(s_addr + (uint32_t)(j >> 1) - 7u, ck);
                    } else if constexpr (ES == 4) {
                        sv[j] = __float_as_uint(e.x);
                        sv[j + 1] = __float_as_uint(e.y);
                    } else {  // E4M3: four tokens per 32-bit word, four words per chunk
                        if (j & 2)
                            ck[(j & 15) >> 2] = pack_e4m3x4(e_prev.x, e_prev.y, e.x, e.y);
                        else
                            e_prev = e;
                        if ((j & 15) == 14)
                            *reinterpret_cast<uint4*>(ptile + kmajor_sw128(r, j >> 4, kRows)) =
                                make_uint4(ck[0], ck[1], ck[2], ck[3]);
                    }
                }
            }
            const f2 ps = add2(add2(part[0], part[1]), add2(part[2], part[3]));
            return ps.x + ps.y;
        };
        // P of zeros (a warp whose rows selected none of the step's pages)
        auto zero_p = [&](uint32_t s_addr) {
            if constexpr (ES == 1) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(ptile + kmajor_sw128(r, c, kRows)) = make_uint4(0, 0, 0, 0);
            } else {
                uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
                for (int c = 0; c < G::kPCols; c += 8) tmem_st_x8(s_addr + (uint32_t)c, z);
            }
        };

        int rnd = 0, item_no = 0;
        int f = walk(rnd);
        if (f >= 0) ok = take(0);
        while (f >= 0 && ok) {
            m_used = kNegInf;
            lsum = 0.f;
            for (int s = w; s < it.nsteps; s += 2) {
                const int k = use++;
                // this step's pages and mask words (PPS divides 32: a step never spans two batches)
                const int e0 = s * PPS;
                while (e0 >= cbase + 32) {
                    cbase += 32;
                    cpage = npage;
                    cmask = nmask;
                    ctail = ntail;
                    fetch(cbase + 32, npage, nmask, ntail);
                }
                // row r sees token t of page q iff the page is in its own TopK row (its bit of the
                // page's mask) and the token's position is < vis_end; a page that reaches kv_len
                // may hold non-finite bytes past it (a tail step: its scores there become -inf
                // here, its V rows there are zeroed by the PV warp)
                int lim_q[PPS];
                bool live = false, partial = false, tail = false;
#pragma unroll
                for (int q = 0; q < PPS; ++q) {
                    const int pg = __shfl_sync(0xffffffffu, cpage, e0 - cbase + q);
                    const uint32_t mw = __shfl_sync(0xffffffffu, cmask, e0 - cbase + q);
                    const bool mine = pg >= 0 && ((mw >> lane) & 1u);
                    lim_q[q] = mine ? max(0, min(T, vis_end - pg * T)) : 0;
                    live |= lim_q[q] > 0;
                    partial |= lim_q[q] > 0 && lim_q[q] < T;
                    tail |= __shfl_sync(0xffffffffu, ctail, e0 - cbase + q);
                }
                ok = warp_ok(mbar_wait(B.sfull(w), k & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                if (!ok) break;
                tc_fence_after();
                const uint32_t s_addr = tmem + lane_base + colS;
                tmem_ld128_wait(s_addr, sv);
                if constexpr (G::kPSmem) {  // S_w is in registers: the next S may overwrite it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(B.sfree(w));
                }
                const bool warp_live = __any_sync(0xffffffffu, live);
                // Raw scores of unseen tokens (past the row's causal limit or kv_len inside a page
                // it selected) become -inf; pages the row did not select get an infinite offset in
                // the exponent.  cs > 0, so the max of raw scores orders the scaled ones.
                if (warp_live && (tail || __any_sync(0xffffffffu, partial))) {
#pragma unroll
                    for (int j = 0; j < kST; ++j) {
                        const int q = j / T, t = j - q * T;
                        if (t >= lim_q[q]) sv[j] = __float_as_uint(kNegInf);
                    }
                }
                bool need = false;
                float alpha = 1.f;
                if (warp_live) {
                    float mloc = kNegInf;
#pragma unroll
                    for (int q = 0; q < PPS; ++q) {
                        float mx[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
                        for (int j = q * T; j < (q + 1) * T; j += 8) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mx[kk] = max3f(mx[kk], __uint_as_float(sv[j + 2 * kk]), __uint_as_float(sv[j + 2 * kk + 1]));
                        }
                        const float mq = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                        if (lim_q[q] > 0) mloc = fmaxf(mloc, mq * cs);
                    }
                    // lazy running max: raise it only when a score exceeds it by more than kTau
                    need = mloc > m_used + G::kTau;
                    if (need) {
                        alpha = ex2(m_used - mloc);  // 0 when m_used is -inf
                        m_used = mloc;
                        lsum *= alpha;
                    }
                }
                // O_w is rescaled only after its previous update has finished (rare); the first
                // update of O_w in a bundle overwrites it.  The shared-memory P tile (E4M3) is
                // rewritten only after that update has read it.
                const bool rescale = s >= 2 && __any_sync(0xffffffffu, need);
                if (rescale || (G::kPSmem && k >= 1)) {
                    ok = warp_ok(mbar_wait(B.pvdone(w), (k - 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                    if (!ok) break;
                    tc_fence_after();
                }
                if (rescale) {
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t ov[32];
                        tmem_ld32_wait(tmem + lane_base + colO + 32u * c, ov);
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st_x32(tmem + lane_base + colO + 32u * c, ov);
                    }
                }
                // P of this step: over S_w (bf16, fp32) or into row r of this warpgroup's shared-memory
                // P tile (E4M3, K-major, swizzled), as it is made
                if (warp_live) {
                    lsum += exps(lim_q, s_addr);
                    if constexpr (ES == 4) tmem_st_n<kST>(s_addr, sv);
                } else {
                    zero_p(s_addr);
                }
                if constexpr (G::kPSmem) fence_proxy_async_smem();
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(B.pfull(w));
            }
            if (!ok) break;
            const Item it_cur = it;
            const int qid_cur = qid, head_cur = head, f_cur = fl;
            const float vsc = vscale;
            const float lsum_cur = lsum, m_cur = m_used;
            const int k_last = use - 1;
            const int n0 = (it_cur.nsteps + 1) / 2, n1 = it_cur.nsteps / 2;  // steps of each warpgroup
            // The next bundle's header (and Q operand) is taken before this bundle's epilogue, so
            // its first S = Q K^T runs while the epilogue reads O.  Its entry of the walk is read
            // only now: the K warp claims it once this bundle's K tiles are all issued.
            const int rnd2 = rnd + 1;
            const int fn = walk(rnd2);
            if (fn >= 0) ok = take(item_no + 1);
            if (!ok) break;
            // ---- epilogue: merge the two warpgroups' partial rows, O / l -> O[qid][head][:]
            if ((w == 0 ? n0 : n1) > 0)
                ok = warp_ok(mbar_wait(B.pvdone(w), k_last & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
            if (!ok) break;
            mrg[w * kRows + r] = make_float2(m_cur, lsum_cur);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(B.ep1());
            ok = warp_ok(mbar_wait(B.ep1(), item_no & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
            if (!ok) break;
            tc_fence_after();
            const float2 other = mrg[(1 - w) * kRows + r];
            const float m0 = w == 0 ? m_cur : other.x, l0 = w == 0 ? lsum_cur : other.y;
            const float m1 = w == 0 ? other.x : m_cur, l1 = w == 0 ? other.y : lsum_cur;
            const float mm = fmaxf(l0 > 0.f ? m0 : kNegInf, l1 > 0.f ? m1 : kNegInf);
            const float f0 = l0 > 0.f ? ex2(m0 - mm) : 0.f, f1 = l1 > 0.f ? ex2(m1 - mm) : 0.f;
            const float ltot = l0 * f0 + l1 * f1;
            const float inv = ltot > 0.f ? vsc / ltot : 0.f;
            const float a0 = f0 * inv, a1 = f1 * inv;
            const size_t oi = ((size_t)(qid_cur >= 0 ? qid_cur : 0) * p.Hq + head_cur) * kD;
            // page-major items: this row's partial result goes to its slot (none: -1)
            const long long pslot = p.part_o ? p.item_slot[(size_t)f_cur * kRows + r] : -1;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {  // this warpgroup's half of the columns
                const uint32_t col = 64u * w + 32u * c;
                uint32_t o0[32], o1[32];
                if (n0 > 0) {
                    tmem_ld32_wait(tmem + lane_base + kColO + col, o0);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o0[e] = 0u;
                }
                if (n1 > 0) {
                    tmem_ld32_wait(tmem + lane_base + kColO + 128u + col, o1);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o1[e] = 0u;
                }
                float ov[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) ov[e] = __uint_as_float(o0[e]) * a0 + __uint_as_float(o1[e]) * a1;
                if (p.part_o) {
                    if (pslot >= 0) {
                        float4* dst = reinterpret_cast<float4*>(p.part_o + (size_t)pslot * kD + col);
#pragma unroll
                        for (int e = 0; e < 8; ++e) dst[e] = make_float4(ov[4 * e], ov[4 * e + 1], ov[4 * e + 2], ov[4 * e + 3]);
                    }
                } else if (qid_cur >= 0) {
                    if constexpr (ES == 4) {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.O) + oi + col);
#pragma unroll
                        for (int e = 0; e < 8; ++e) dst[e] = make_float4(ov[4 * e], ov[4 * e + 1], ov[4 * e + 2], ov[4 * e + 3]);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.O) + oi + col);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(pack_bf16x2(ov[8 * e], ov[8 * e + 1]), pack_bf16x2(ov[8 * e + 2], ov[8 * e + 3]),
                                                pack_bf16x2(ov[8 * e + 4], ov[8 * e + 5]),
                                                pack_bf16x2(ov[8 * e + 6], ov[8 * e + 7]));
                    }
                }
            }
            if (w == 0 && p.part_o && pslot >= 0)  // log2 domain, merged by the page-major reduction
                p.part_lse[pslot] = ltot > 0.f ? mm + __log2f(ltot) - G::kPLog2 : kNegInf;
            if (w == 0 && !p.part_o && qid_cur >= 0 && p.lse != nullptr)
                p.lse[(size_t)qid_cur * p.Hq + head_cur] =
                    ltot > 0.f ? (mm + __log2f(ltot) - G::kPLog2) * 0.69314718055994531f : kNegInf;
            // neither accumulator is overwritten by the next bundle before both warpgroups read it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(B.ep2());
            ok = warp_ok(mbar_wait(B.ep2(), item_no & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
            if (!ok) break;
            tc_fence_after();
            f = fn;
            rnd = rnd2;
            ++item_no;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kSWarp) tmem_dealloc(tmem, kTmemCols);
    // the last CTA out resets this launch slot's bundle counter (every claim has been made)
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(ticket + 1, 1u) == gridDim.x - 1) {
            atomicExch(ticket, 0u);
            atomicExch(ticket + 1, 0u);
        }
    }
}

size_t attn_smem_bytes(int es, int nsk, int nsv, int Hkv, int g) { return smem_layout(es, nsk, nsv, Hkv, g).total; }

size_t attn_tile_bytes(int es) { return (size_t)kST * kD * es; }

template <int ES, int T>
static cudaError_t launch_t(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                            const AttnParams& p, int grid, size_t smem, cudaStream_t stream) {
    // The register split (setmaxnreg) is sized for kLaunchRegs per thread at launch: a kernel
    // built with another count is not launched (an increase beyond the launch's registers would
    // never be granted).
    static const int regs = [] {
        cudaFuncAttributes a;
        return cudaFuncGetAttributes(&a, (const void*)union_attn_kernel<ES, T>) == cudaSuccess ? a.numRegs : -1;
    }();
    if (regs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    cudaError_t e = ensure_smem_attr((const void*)union_attn_kernel<ES, T>, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(union_attn_kernel<ES, T>, dim3(grid), dim3(kThreads), smem, stream, tmK, tmV, tmQ, p);
}

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const f2 r = exp2_poly2(f2{x[i], i + 1 < n ? x[i + 1] : 0.f});
    y[i] = r.x;
    if (i + 1 < n) y[i + 1] = r.y;
}

cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const int threads = 256, pairs = (n + 1) / 2;
    exp2_poly_kernel<<<(pairs + threads - 1) / threads, threads, 0, stream>>>(x, y, n);
    return cudaGetLastError();
}

cudaError_t launch_union_attn(int es, int T, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                              const AttnParams& p, int grid, size_t smem, cudaStream_t stream) {
    if (es == 2 && T == 16) return launch_t<2, 16>(tmK, tmV, tmQ, p, grid, smem, stream);
    if (es == 2 && T == 32) return launch_t<2, 32>(tmK, tmV, tmQ, p, grid, smem, stream);
    if (es == 2 && T == 64) return launch_t<2, 64>(tmK, tmV, tmQ, p, grid, smem, stream);
    if (es == 2 && T == 128) return launch_t<2, 128>(tmK, tmV, tmQ, p, grid, smem, stream);
    if (es == 1 && T == 64) return launch_t<1, 64>(tmK, tmV, tmQ, p, grid, smem, stream);
    if (es == 1 && T == 128) return launch_t<1, 128>(tmK, tmV, tmQ, p, grid, smem, stream);
    if (es == 4 && T == 32) return launch_t<4, 32>(tmK, tmV, tmQ, p, grid, smem, stream);
    if (es == 4 && T == 64) return launch_t<4, 64>(tmK, tmV, tmQ, p, grid, smem, stream);
    return cudaErrorInvalidValue;
}

}  // namespace qup
