// union_attn.cu -- ID-aware union attention for sm_100a (PageWeaver,
// Abstract; Figure 1; Figure 3), re-designed for tcgen05 + TMEM.
//
// Work item: a bundle of up to 128 query rows (up to 128 / rows_per_group
// page-affine groups of one KV head, see qup_groups).  Pages of the bundle
// union are streamed once per bundle in steps of 128 tokens (one 128-token
// page, or 128 / T smaller pages) through two TMA rings, one of K tiles and
// one of V tiles.  Per step g, with b = g & 1:
//      S_b  = Q K^T     M = 128 rows, N = 128 tokens, K = d  (Q from TMEM, K from smem)
//      P_b  = masked online softmax of S_b, written over S_b  (TMEM -> registers -> TMEM)
//      O   += P_b V     M = 128 rows, N = d, K = 128 tokens   (P from TMEM, V from smem)
// One warpgroup runs the softmax: thread = TMEM lane = bundle row, so the row
// max and the row sum never leave the thread, and each SM sub-partition holds
// one softmax warp (two busy softmax warps on one sub-partition starve each
// other's latency-bound phases).  While it works on step g the tensor pipe
// runs O += P(g-1) V and then S(g+1) = Q K^T: P is written over the S buffer
// it came from, so S(g+2) waits for the O update of step g.
// A row's max is only raised when a score exceeds it by more than kTau (log2
// units); O and the row sum are rescaled then, which after the first steps is
// rare.  A warp whose 32 rows selected none of a step's pages skips that
// step's exponentials.  Each softmax warp reads the bundle's page numbers and
// its own 32-bit word of every page's row mask straight from the bundle
// arrays, 32 entries at a time, one batch ahead; it waits for a V tile only
// on a step whose page reaches kv_len (whose V rows past kv_len it zeroes).
// A quarter of the exponentials come from a polynomial on the FMA pipe
// (exp2_poly2) and the rest from the MUFU unit.
//
// Bundle boundaries: the V warp stages each bundle a few steps ahead (header,
// query IDs and positions, and the bundle's Q rows by original query ID,
// bulk-copied into shared memory); right after a bundle's last P the softmax
// warps move the next bundle's Q rows into the other of two TMEM Q buffers,
// so the next bundle's first S = Q K^T runs during this bundle's epilogue.
//
// Warp roles (256 threads):
//   warps 0-3  softmax / epilogue: thread = TMEM lane = bundle row.  They
//              also move each bundle's Q rows (gathered by original query ID:
//              no reordered Q tensor) into TMEM.
//   warp 4     K producer: walks the bundle's page list, resolves physical
//              pages (warp-parallel) and TMA-loads the K tiles.
//   warp 6     V producer: the same walk for the V tiles; stages each bundle.
//   warp 5     S issuer (one elected lane of a warp-uniform loop) and TMEM
//              owner (512 columns): S(g) once K tile g has landed and the O
//              update of step g - 2 has finished with S_b.
//   warp 7     PV issuer: O += P_b V once P(g) and V tile g are ready.
// The two issuers sit on different SM sub-partitions, each beside one softmax
// warp and no other busy warp; producers and issuers wait with suspended
// try_waits, which leave the sub-partition's issue slots to the softmax.
// TMEM columns: O [0,128); S_0 [128,256); S_1 [256,384); two Q buffers from
// 384 (bf16: 64 columns each, E4M3: 32; fp32 Q stays in shared memory).  P_b
// occupies the first kPCols columns of S_b.
// Operand types: bf16 (kind::f16), fp32 (kind::tf32, Q in shared memory),
// FP8 E4M3 (kind::f8f6f4: K and V straight from the cache, Q quantised per
// row with its own scale, P stored as E4M3 of 2^4 p).  Every MMA consumes 32
// bytes of its K extent per row, so the descriptor arithmetic is shared.
//
// Every wait is bounded (ptx.cuh); on a timeout the CTA raises an abort flag,
// drains its in-flight TMA loads and MMAs, frees TMEM and exits.
#include <cstdint>
#include <cuda.h>

#include "internal.h"
#include "ptx.cuh"
#include "query_union_paged.h"

namespace qup {

constexpr int kThreads = 256;
constexpr int kRows = 128;
constexpr int kD = kHeadDim;
constexpr int kST = 128;  // tokens per pipeline step
constexpr int kTmemCols = 512;
constexpr int kKProducerWarp = 4, kSWarp = 5, kVProducerWarp = 6, kPvWarp = 7;
constexpr uint32_t kColO = 0, kColS = 128, kColQ = 384;

template <int ES, int T>
struct Geo {
    static constexpr int SPP = T > kST ? T / kST : 1;   // steps per page (not used: T <= 128)
    static constexpr int PPS = T < kST ? kST / T : 1;   // pages per step
    static constexpr int BOXR = T < 64 ? T : 64;        // token rows per TMA box
    static constexpr int BPP = T / BOXR;                // boxes per page (along tokens)
    static constexpr int kTile = kST * kD * ES;         // one K or V tile of a step
    static constexpr int kChunkElems = 128 / ES;        // elements per 128-byte swizzle row
    static constexpr int kNChunk = kD * ES / 128;       // 128-byte chunks along d
    static constexpr int kChunkBytes = kST * 128;       // one chunk column of a K or V tile
    static constexpr int kQChunkBytes = kRows * 128;    // one chunk column of a shared-memory Q tile
    static constexpr int kMmaK = 32 / ES;               // K elements per MMA instruction
    static constexpr int kNumMmaS = kD * ES / 32;       // MMAs per S (K = d)
    static constexpr int kNumMmaPV = kST * ES / 32;     // MMAs per O update (K = 128 tokens)
    static constexpr int kPCols = kST * ES / 4;         // TMEM columns of P
    static constexpr bool kQTmem = ES != 4;             // Q as the TMEM A operand (bf16, E4M3)
    static constexpr int kQCols = kD * ES / 4;          // TMEM columns of Q
    static_assert(!kQTmem || kColQ + 2 * kQCols <= kTmemCols, "TMEM budget (two Q buffers)");
    static_assert(kPCols <= 128, "P fits in its S buffer");
    // exponentials on the FMA pipe by a polynomial: pairs (j / 2) % 8 < kPolyPairs of every 16
    // columns; the rest go to the MUFU unit
    static constexpr int kPolyPairs = 2;
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
    uint32_t kst, vst, q, qst, sinfo, bars, misc, total;
};

// Stage of the next bundle (bf16 Q rows): query slot m holds the g rows of its query, 256 bytes
// each, at m * qstage_stride(g); the 16-byte pad keeps row reads free of bank conflicts.
__host__ __device__ inline uint32_t qstage_stride(int g) { return (uint32_t)g * 256u + 16u; }
constexpr int kSinfoWords = 8;  // stage header: flat bundle, h, bi, ub, nU, nsteps, ok

__host__ __device__ inline SmemLayout smem_layout(int es, int nsk, int nsv, int Hkv, int g) {
    SmemLayout L;
    uint32_t off = 0;
    L.kst = off;
    off += (uint32_t)nsk * kST * kD * es;
    L.vst = off;
    off += (uint32_t)nsv * kST * kD * es;
    L.q = off;
    if (es == 4) off += (uint32_t)kRows * kD * es;  // fp32 Q stays in shared memory
    L.qst = off;
    if (es != 4) off += (uint32_t)(kRows / g) * qstage_stride(g);
    L.sinfo = off;
    off += 4u * (kSinfoWords + 2 * kRows);  // header, qid[128 / g], q_pos[128 / g]
    L.bars = off;
    off += 8u * (2u * (nsk + nsv) + 12u);
    L.misc = off;
    off += 16u + 4u * (uint32_t)(Hkv + 1);
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
    __device__ __forceinline__ uint32_t sfull(int i) const { return fixed(i); }
    __device__ __forceinline__ uint32_t pfull(int i) const { return fixed(2 + i); }
    __device__ __forceinline__ uint32_t pvdone(int i) const { return fixed(4 + i); }
    __device__ __forceinline__ uint32_t qfull() const { return fixed(6); }
    __device__ __forceinline__ uint32_t drain() const { return fixed(7); }
    __device__ __forceinline__ uint32_t drain2() const { return fixed(8); }
    __device__ __forceinline__ uint32_t stfull() const { return fixed(9); }
    __device__ __forceinline__ uint32_t stempty() const { return fixed(10); }
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
    const size_t bp = (size_t)h * (p.Nq + 1) + it.bi;
    it.ub = p.union_ptr[bp];
    it.nU = p.union_ptr[bp + 1] - it.ub;
    it.ok = it.ub >= 0 && it.nU >= 0 && (long long)it.ub + it.nU <= p.cap_union;
    if (!it.ok) it.nU = 0;
    it.nsteps = (it.nU + PPS - 1) / PPS;
    return it;
}

// Flat bundle index of this CTA's r-th work item, -1 past the end, -2 for a bad
// order entry (skipped; QUP_ERR_GROUP).  The bundle order (largest unions first)
// is dealt out in a snake: round r gives CTA b the position r*G + b when r is
// even and r*G + G-1-b when r is odd, so each CTA's total work stays near the
// mean.  Positions only grow with r, so the first position past the end ends
// the walk.  Every role calls this and reaches the same verdict.
__device__ __forceinline__ int item_at(const AttnParams& p, int r, int n_items) {
    const long long G = gridDim.x;
    const long long pos = (long long)r * G + ((r & 1) ? G - 1 - blockIdx.x : (long long)blockIdx.x);
    if (pos >= n_items) return -1;
    const int f = p.bundle_order[pos];
    return (f >= 0 && f < n_items) ? f : -2;
}

// byte offset of 16-byte chunk c of row r inside a K-major SW128 operand tile of `rows` rows
__device__ __forceinline__ uint32_t kmajor_sw128(int r, int c, int rows) {
    return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ bool warp_ok(bool ok) { return __all_sync(0xffffffffu, ok); }

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
                      const __grid_constant__ AttnParams p) {
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
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t lim = p.wait_limit_ns;

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
        for (int i = 0; i < 2; ++i) {
            mbar_init(B.sfull(i), 1);
            mbar_init(B.pfull(i), 4);  // one arrive per softmax warp
            mbar_init(B.pvdone(i), 1);
        }
        mbar_init(B.qfull(), 4);
        mbar_init(B.drain(), 1);
        mbar_init(B.drain2(), 1);
        mbar_init(B.stfull(), 1);
        mbar_init(B.stempty(), 4);  // one arrive per softmax warp
        fence_mbar_init();
        *abort_flag = 0;
    }
    if (threadIdx.x == kKProducerWarp * 32) prefetch_tensormap(&tmK);
    if (threadIdx.x == kVProducerWarp * 32) prefetch_tensormap(&tmV);
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
            if (n < 0 || n > p.Nq) {
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

    if (warp == kKProducerWarp || warp == kVProducerWarp) {
        // ============================================================ producers (whole warp each)
        // Both walk the same bundles and pages; the K warp fills the K ring, the V warp the
        // V ring (and stages each bundle for the softmax warps).
        const bool isV = warp == kVProducerWarp;
        const int NR = isV ? NSV : NSK;
        const CUtensorMap* tm = isV ? &tmV : &tmK;
        const uint32_t ring = sbase + (isV ? L.vst : L.kst);
        int gs = 0, n_staged = 0;
        bool ok = true;
        for (int rnd = 0; ok; ++rnd) {
            const int f = item_at(p, rnd, n_items);
            if (f == -1) break;
            if (f < 0) continue;
            const Item it = load_item<PPS>(p, nb_prefix, f);
            if constexpr (ES != 4) {
                // The V warp stages the bundle for the softmax warps (a few steps before they reach
                // it): header, query IDs and positions of its query slots, and its Q rows (bulk
                // copies by original query ID: the g rows of a query are contiguous in Q).
                if (isV) {
                    if (n_staged > 0) {  // the softmax warps have read the previous stage
                        int okv = 0;
                        if (lane == 0)
                            okv = mbar_wait_idle(B.stempty(), (n_staged - 1) & 1, abort_flag, p.err,
                                                 QUP_ERR_TIMEOUT, lim);
                        ok = __shfl_sync(0xffffffffu, okv, 0) != 0;
                        if (!ok) break;
                    }
                    int* sinfo = reinterpret_cast<int*>(smem + L.sinfo);
                    const int MQ = kRows / p.g;
                    int nvalid = 0;
                    for (int m0 = 0; m0 < MQ; m0 += 32) {
                        const int m = m0 + lane;
                        int qid = -1;
                        if (m < MQ) {
                            qid = p.bundle_qid[((size_t)it.h * p.Nq + it.bi) * MQ + m];
                            if (qid >= p.Nq) {
                                atomicOr(p.err, QUP_ERR_GROUP);
                                qid = -1;
                            }
                            qid = max(qid, -1);
                            sinfo[kSinfoWords + m] = qid;
                            sinfo[kSinfoWords + kRows + m] = qid >= 0 ? p.q_pos[qid] : -1;
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
                    const uint32_t qbytes = (uint32_t)p.g * kD * 2u;
                    if (lane == 0) mbar_arrive_expect_tx(B.stfull(), (uint32_t)nvalid * qbytes);
                    __syncwarp();
                    for (int m = lane; m < MQ; m += 32) {
                        const int qid = sinfo[kSinfoWords + m];
                        if (qid >= 0)
                            bulk_g2s(sbase + L.qst + (uint32_t)m * qstage_stride(p.g),
                                     static_cast<const uint16_t*>(p.Q) + ((size_t)qid * p.Hq + (size_t)it.h * p.g) * kD,
                                     qbytes, B.stfull());
                    }
                    ++n_staged;
                }
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
                        okv = mbar_wait_idle(isV ? B.vempty(slot) : B.kempty(slot), ((gs / NR) & 1) ^ 1, abort_flag,
                                        p.err, QUP_ERR_TIMEOUT, lim);
                    ok = __shfl_sync(0xffffffffu, okv, 0) != 0;
                    if (!ok) break;
                    const bool issue = lane == 0 && !(p.dbg_skip_stage >= 0 && blockIdx.x == 0 &&
                                                      gs == p.dbg_skip_stage);
                    int ph[PPS];
#pragma unroll
                    for (int q = 0; q < PPS; ++q) {
                        const int src = k * PPS + q;
                        ph[q] = __shfl_sync(0xffffffffu, phys, src);
                    }
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
        // every issued load lands before the CTA may exit: the last NR stages of this ring, and
        // the last stage of Q rows
        if (lane == 0) {
            if (n_staged > 0) mbar_wait_drain(B.stfull(), (n_staged - 1) & 1, lim);
            for (int i = max(0, gs - NR); i < gs; ++i) {
                if (p.dbg_skip_stage >= 0 && blockIdx.x == 0 && i == p.dbg_skip_stage) continue;
                mbar_wait_drain(isV ? B.vfull(i % NR) : B.kfull(i % NR), (i / NR) & 1, lim);
            }
        }
        __syncwarp();
    } else if (warp == kSWarp || warp == kPvWarp) {
        // ============================================================ MMA issuers (whole warp, one elected lane)
        //   S warp:  S(g) = Q K^T into S_b: needs K tile g, and the O update of step g - 2
        //            (which read P from S_b) finished; commits S-full(b) and the K slot.
        //   PV warp: O += P_b V: needs P(g) and V tile g; commits PV-done(b) and the V slot.
        // The PV warp needs no Q barrier: P(g) of a bundle's first step is written after the
        // softmax warps have finished the previous bundle's epilogue (its reads of O).
        const bool isS = warp == kSWarp;
        const uint32_t idesc_s = instr_desc(G::kFmt, 0, 0, kST, kRows);
        const uint32_t idesc_o = instr_desc(G::kFmt, 0, 1, kD, kRows);
        // V as the MN-major B operand (N = d): 128-byte swizzle with 8-row atoms; tf32
        // has only the 128-byte swizzle with 32-byte atoms (layout 1, 4-row atoms)
        constexpr uint32_t vlayout = ES == 4 ? 1u : 2u;
        constexpr uint32_t vsbo = ES == 4 ? 512u : 1024u;
        const uint32_t qbase = sbase + L.q;
        int gs = 0, item_no = 0;
        int ks = 0, kph = 0, vs = 0, vph = 0;  // ring slot and phase of step gs
        bool ok = true;
        for (int rnd = 0; ok; ++rnd) {
            const int f = item_at(p, rnd, n_items);
            if (f == -1) break;
            if (f < 0) continue;
            const Item it = load_item<PPS>(p, nb_prefix, f);
            if (isS) {
                ok = warp_ok(mbar_wait_idle(B.qfull(), item_no & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                if (!ok) break;
                tc_fence_after();
                for (int s = 0; s < it.nsteps; ++s) {
                    const int g = gs + s, b = g & 1;
                    ok = warp_ok(mbar_wait_idle(B.kfull(ks), kph, abort_flag, p.err, QUP_ERR_TIMEOUT, lim) &&
                                 (g < 2 || mbar_wait_idle(B.pvdone(b), ((g - 2) >> 1) & 1, abort_flag, p.err,
                                                     QUP_ERR_TIMEOUT, lim)));
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t kdesc = smem_desc(sbase + L.kst + (uint32_t)ks * G::kTile, 16, 1024, 2);
                    const uint64_t qdesc = smem_desc(qbase, 16, 1024, 2);
                    if (elect_one_sync()) {
#pragma unroll
                        for (int k = 0; k < G::kNumMmaS; ++k) {
                            const uint32_t koff = ((k >> 2) * G::kChunkBytes + (k & 3) * 32) >> 4;
                            if constexpr (G::kQTmem) {
                                tc_mma_ts<G::kKind>(tmem + kColS + 128u * b,
                                                    tmem + kColQ + (uint32_t)(item_no & 1) * G::kQCols + 8u * k, kdesc + koff,
                                                    idesc_s, k > 0);
                            } else {
                                const uint32_t qoff = ((k >> 2) * G::kQChunkBytes + (k & 3) * 32) >> 4;
                                tc_mma<G::kKind>(tmem + kColS + 128u * b, qdesc + qoff, kdesc + koff, idesc_s, k > 0);
                            }
                        }
                        tc_commit(B.sfull(b));
                        tc_commit(B.kempty(ks));
                    }
                    __syncwarp();
                    if (++ks == NSK) {
                        ks = 0;
                        kph ^= 1;
                    }
                }
            } else {
                for (int s = 0; s < it.nsteps; ++s) {
                    const int g = gs + s, b = g & 1;
                    ok = warp_ok(mbar_wait_idle(B.pfull(b), (g >> 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim) &&
                                 mbar_wait_idle(B.vfull(vs), vph, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t vdesc = smem_desc(sbase + L.vst + (uint32_t)vs * G::kTile,
                                                     (uint32_t)G::kChunkBytes, vsbo, vlayout);
                    if (elect_one_sync()) {
#pragma unroll
                        for (int k = 0; k < G::kNumMmaPV; ++k) {
                            // K step = kMmaK tokens: 8 TMEM columns of P, kMmaK rows of V
                            tc_mma_ts<G::kKind>(tmem + kColO, tmem + kColS + 128u * b + 8u * k,
                                                vdesc + ((k * G::kMmaK * 128) >> 4), idesc_o, s > 0 || k > 0);
                        }
                        tc_commit(B.pvdone(b));
                        tc_commit(B.vempty(vs));
                    }
                    __syncwarp();
                    if (++vs == NSV) {
                        vs = 0;
                        vph ^= 1;
                    }
                }
            }
            gs += it.nsteps;
            ++item_no;
        }
        // every MMA this warp issued completes before TMEM is freed
        const uint32_t dbar = isS ? B.drain() : B.drain2();
        if (elect_one_sync()) tc_commit(dbar);
        __syncwarp();
        mbar_wait_drain(dbar, 0, lim);
        __syncwarp();
    } else {
        // ============================================================ softmax / epilogue (warps 0-3)
        const int r = warp * 32 + lane;  // bundle row == TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float kNegInf = -__int_as_float(0x7f800000);
        const float kPosInf = __int_as_float(0x7f800000);
        const int g = p.g, MQ = kRows / g;
        const int* sinfo = reinterpret_cast<const int*>(smem + L.sinfo);
        int gs = 0, vs = 0, vph = 0;
        bool ok = true;
        // the row's bundle state: item, query (original ID), Q head, visible positions, score scale
        Item it{};
        int qid = -1, head = 0, vis_end = 0;
        float cs = p.scale_log2;
        float m_used = kNegInf, lsum = 0.f;
        f2 cs2{cs, cs};
        // The bundle's union entries, 32 at a time: lane j holds entry base + j, its logical
        // page (-1 for padding or an entry the producers reject) and this warp's 32-bit word
        // of the page's row mask.  The next 32 are loaded one batch ahead.
        int cpage = -1, npage = -1;
        uint32_t cmask = 0u, nmask = 0u;
        int cbase = 0;
        auto fetch = [&](int base, int& pg, uint32_t& mk) {
            const int e = base + lane;
            pg = -1;
            mk = 0u;
            if (e < it.nU) {
                const int u = p.union_pages[it.ub + e];
                const uint32_t m = p.row_mask[(size_t)(it.ub + e) * 4 + warp];
                if (u >= 0 && u < p.num_logical_pages) {
                    const int ph = p.page_table[u];
                    if (ph >= 0 && ph < p.P_phys) {
                        pg = u;
                        mk = m;
                    }
                }
            }
        };
        // Take over flat bundle ff, the ino-th of this CTA: its header and this row's query
        // (bf16 Q: from the stage the V warp filled; fp32 Q: from global memory), the first union
        // entries, and this row of Q by original query ID into the bundle's TMEM Q buffer (fp32:
        // the shared-memory Q tile).  Arrives on the Q barrier (and releases the stage).
        auto take = [&](int ff, int ino) -> bool {
            int qpos = -1;
            if constexpr (ES != 4) {
                if (!warp_ok(mbar_wait(B.stfull(), ino & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim))) return false;
                it.h = sinfo[1];
                it.bi = sinfo[2];
                it.ub = sinfo[3];
                it.nU = sinfo[4];
                it.nsteps = sinfo[5];
                it.ok = sinfo[6] != 0;
                qid = sinfo[kSinfoWords + r / g];
                qpos = sinfo[kSinfoWords + kRows + r / g];
            } else {
                it = load_item<PPS>(p, nb_prefix, ff);
                qid = p.bundle_qid[((size_t)it.h * p.Nq + it.bi) * MQ + r / g];
                if (qid >= p.Nq) {
                    atomicOr(p.err, QUP_ERR_GROUP);
                    qid = -1;
                }
                qid = max(qid, -1);
                qpos = qid >= 0 ? p.q_pos[qid] : -1;
            }
            if (!it.ok && threadIdx.x == 0) atomicOr(p.err, QUP_ERR_GROUP);
            head = it.h * g + (r % g);
            vis_end = min(qpos + 1, p.kv_len);  // positions < vis_end are visible
            cs = p.scale_log2;                  // score scale (log2 domain) of this row
            cbase = 0;
            fetch(0, cpage, cmask);
            fetch(32, npage, nmask);
            const uint32_t qcol = kColQ + (uint32_t)(ino & 1) * G::kQCols;
            if constexpr (ES == 2) {
                const uint8_t* row = smem + L.qst + (uint32_t)(r / g) * qstage_stride(g) + (uint32_t)(r % g) * 256u;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t qv[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v =
                            qid >= 0 ? *reinterpret_cast<const uint4*>(row + half * 128 + c * 16) : make_uint4(0, 0, 0, 0);
                        qv[4 * c] = v.x;
                        qv[4 * c + 1] = v.y;
                        qv[4 * c + 2] = v.z;
                        qv[4 * c + 3] = v.w;
                    }
                    tmem_st_x32(tmem + lane_base + qcol + 32u * half, qv);
                }
            } else if constexpr (ES == 4) {
                uint8_t* qt = smem + L.q;
                const size_t row_off = ((size_t)(qid >= 0 ? qid : 0) * p.Hq + head) * kD;
                const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(p.Q) + row_off);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const uint4 v = qid >= 0 ? src[c] : make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(qt + kmajor_sw128(r, c, kRows)) = v;
                }
                fence_proxy_async_smem();
            } else {  // the whole row: bf16 -> E4M3 with the row's scale amax / 448
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
                uint32_t qv[32];
#pragma unroll
                for (int c = 0; c < 16; ++c) {  // 8 bf16 -> 8 E4M3 (2 columns)
                    const uint32_t w4[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        x[2 * e] = __uint_as_float(w4[e] << 16) * inv;
                        x[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u) * inv;
                    }
                    qv[2 * c] = pack_e4m3x4(x[0], x[1], x[2], x[3]);
                    qv[2 * c + 1] = pack_e4m3x4(x[4], x[5], x[6], x[7]);
                }
                tmem_st_x32(tmem + lane_base + qcol, qv);
                cs = amax * (1.f / 448.f) * p.k_scale[it.h] * p.scale_log2;
            }
            if constexpr (G::kQTmem) tmem_wait_st();
            // a Q row of zeros (E4M3 scale 0) keeps a positive score scale: its scores are 0 anyway
            cs = fmaxf(cs, 1e-30f);
            cs2 = f2{cs, cs};
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(B.qfull());
                if constexpr (ES != 4) mbar_arrive(B.stempty());
            }
            return true;
        };
        // the walk of bundles: -1 past the end; order entries that are bad are reported and skipped
        auto walk = [&](int& rr) -> int {
            int ff = item_at(p, rr, n_items);
            while (ff == -2) {
                if (threadIdx.x == 0) atomicOr(p.err, QUP_ERR_GROUP);
                ff = item_at(p, ++rr, n_items);
            }
            return ff;
        };
        // exponentials of one step: p = 2^(s*cs - m_used + kPLog2) into pk (or sv for fp32),
        // and their sum
        uint32_t sv[kST];
        uint32_t pk[ES == 4 ? 1 : G::kPCols];
        auto exps = [&](const int (&lim)[PPS]) -> float {
            const float mb = (m_used == kNegInf ? 0.f : m_used) - G::kPLog2;
            f2 part[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
            f2 e_prev{0.f, 0.f};  // E4M3: the first pair of a 4-token column
#pragma unroll
            for (int q = 0; q < PPS; ++q) {  // one page (T tokens) at a time
                // a page the row did not select gets an infinite offset: 2^-inf = 0
                const float off = lim[q] == 0 ? kPosInf : mb;
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
                        pk[j / 2] = pack_bf16x2(e.x, e.y);
                    } else if constexpr (ES == 4) {
                        sv[j] = __float_as_uint(e.x);
                        sv[j + 1] = __float_as_uint(e.y);
                    } else {  // E4M3: four tokens per 32-bit column
                        if (j & 2)
                            pk[j / 4] = pack_e4m3x4(e_prev.x, e_prev.y, e.x, e.y);
                        else
                            e_prev = e;
                    }
                }
            }
            const f2 ps = add2(add2(part[0], part[1]), add2(part[2], part[3]));
            return ps.x + ps.y;
        };

        int rnd = 0, item_no = 0;
        int f = walk(rnd);
        if (f >= 0) ok = take(f, 0);
        while (f >= 0 && ok) {
            // the next bundle's flat index: loaded now, used after this bundle's steps
            int rnd2 = rnd + 1;
            const int f2raw = item_at(p, rnd2, n_items);
            m_used = kNegInf;
            lsum = 0.f;
            for (int s = 0; s < it.nsteps; ++s) {
                const int gstep = gs + s, b = gstep & 1, slot = vs;
                const int vphase = vph;
                if (++vs == NSV) {
                    vs = 0;
                    vph ^= 1;
                }
                // this step's pages and mask words (PPS divides 32: a step never spans two batches)
                const int e0 = s * PPS;
                if (e0 >= cbase + 32) {
                    cbase += 32;
                    cpage = npage;
                    cmask = nmask;
                    fetch(cbase + 32, npage, nmask);
                }
                // row r sees token t of page q iff the page is in its own TopK row (its bit of the
                // page's mask) and the token's position is < vis_end; a page that reaches kv_len
                // may hold non-finite bytes past it (a tail step)
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
                    tail |= pg >= 0 && pg * T + T > p.kv_len;
                }
                if (ok) ok = warp_ok(mbar_wait(B.sfull(b), (gstep >> 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                if (ok && tail) ok = warp_ok(mbar_wait(B.vfull(slot), vphase, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                if (!ok) continue;
                tc_fence_after();
                const uint32_t s_addr = tmem + lane_base + kColS + 128u * b;
                tmem_ld128_wait(s_addr, sv);
                if (tail) {  // thread r zeroes V token row r of the step if it lies past kv_len
                    const int q = r / T;
                    const int pg = __shfl_sync(0xffffffffu, cpage, e0 - cbase + q);
                    if (pg >= 0 && pg * T + (r - q * T) >= p.kv_len) {
                        uint8_t* vt = smem + L.vst + (uint32_t)slot * G::kTile;
#pragma unroll
                        for (int c = 0; c < G::kNChunk; ++c)
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                *reinterpret_cast<uint4*>(vt + c * G::kChunkBytes + r * 128 + e * 16) =
                                    make_uint4(0, 0, 0, 0);
                    }
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
                            for (int k = 0; k < 4; ++k)
                                mx[k] = max3f(mx[k], __uint_as_float(sv[j + 2 * k]), __uint_as_float(sv[j + 2 * k + 1]));
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
                    lsum += exps(lim_q);
                } else {
                    if constexpr (ES == 4) {
#pragma unroll
                        for (int j = 0; j < kST; ++j) sv[j] = 0u;
                    } else {
#pragma unroll
                        for (int j = 0; j < G::kPCols; ++j) pk[j] = 0u;
                    }
                }
                // O is rescaled only after every earlier O update has finished (rare)
                if (s > 0 && __any_sync(0xffffffffu, need)) {
                    const int pg = gstep - 1;
                    ok = warp_ok(mbar_wait(B.pvdone(pg & 1), (pg >> 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
                    if (!ok) continue;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t ov[32];
                        tmem_ld32_wait(tmem + lane_base + kColO + 32u * c, ov);
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st_x32(tmem + lane_base + kColO + 32u * c, ov);
                    }
                }
                // P over the S buffer it came from (every column of S is in registers)
                if constexpr (ES == 4) {
                    tmem_st_n<kST>(s_addr, sv);
                } else {
                    tmem_st_n<G::kPCols>(s_addr, pk);
                }
                tmem_wait_st();
                if (tail) fence_proxy_async_smem();  // zeroed V rows -> async proxy
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(B.pfull(b));
            }
            gs += it.nsteps;
            const Item it_cur = it;
            const int qid_cur = qid, head_cur = head;
            const float lsum_cur = lsum, m_cur = m_used;
            // The next bundle takes the other Q buffer before this bundle's epilogue, so its first
            // S = Q K^T runs while the epilogue reads O.
            int f2 = f2raw;
            while (f2 == -2) {
                if (threadIdx.x == 0) atomicOr(p.err, QUP_ERR_GROUP);
                f2 = item_at(p, ++rnd2, n_items);
            }
            if (ok && f2 >= 0) ok = take(f2, item_no + 1);
            // ---- epilogue: O / l -> O[qid][head][:]
            if (ok && it_cur.nsteps > 0) {
                const int last = gs - 1;
                ok = warp_ok(mbar_wait(B.pvdone(last & 1), (last >> 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim));
            }
            if (!ok) break;
            tc_fence_after();
            float vsc = 1.f;
            if constexpr (ES == 1) vsc = p.v_scale[it_cur.h];
            const float inv = lsum_cur > 0.f ? vsc / lsum_cur : 0.f;
            const size_t oi = ((size_t)(qid_cur >= 0 ? qid_cur : 0) * p.Hq + head_cur) * kD;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t ov[32];
                if (it_cur.nsteps > 0) {
                    tmem_ld32_wait(tmem + lane_base + kColO + 32u * c, ov);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = 0u;
                }
                if (qid_cur >= 0) {
                    if constexpr (ES == 4) {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.O) + oi + 32 * c);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                                 __uint_as_float(ov[4 * e + 2]) * inv,
                                                 __uint_as_float(ov[4 * e + 3]) * inv);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.O) + oi + 32 * c);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(
                                pack_bf16x2(__uint_as_float(ov[8 * e]) * inv, __uint_as_float(ov[8 * e + 1]) * inv),
                                pack_bf16x2(__uint_as_float(ov[8 * e + 2]) * inv, __uint_as_float(ov[8 * e + 3]) * inv),
                                pack_bf16x2(__uint_as_float(ov[8 * e + 4]) * inv, __uint_as_float(ov[8 * e + 5]) * inv),
                                pack_bf16x2(__uint_as_float(ov[8 * e + 6]) * inv, __uint_as_float(ov[8 * e + 7]) * inv));
                    }
                }
            }
            if (qid_cur >= 0 && p.lse != nullptr)
                p.lse[(size_t)qid_cur * p.Hq + head_cur] =
                    lsum_cur > 0.f ? (m_cur + __log2f(lsum_cur) - G::kPLog2) * 0.69314718055994531f : kNegInf;
            tc_fence_before();
            f = f2;
            rnd = rnd2;
            ++item_no;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kSWarp) tmem_dealloc(tmem, kTmemCols);
}

size_t attn_smem_bytes(int es, int nsk, int nsv, int Hkv, int g) { return smem_layout(es, nsk, nsv, Hkv, g).total; }

size_t attn_tile_bytes(int es) { return (size_t)kST * kD * es; }

template <int ES, int T>
static cudaError_t launch_t(const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnParams& p, int grid,
                            size_t smem, cudaStream_t stream) {
    cudaError_t e = ensure_smem_attr((const void*)union_attn_kernel<ES, T>, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(union_attn_kernel<ES, T>, dim3(grid), dim3(kThreads), smem, stream, tmK, tmV, p);
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

cudaError_t launch_union_attn(int es, int T, const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnParams& p,
                              int grid, size_t smem, cudaStream_t stream) {
    if (es == 2 && T == 16) return launch_t<2, 16>(tmK, tmV, p, grid, smem, stream);
    if (es == 2 && T == 32) return launch_t<2, 32>(tmK, tmV, p, grid, smem, stream);
    if (es == 2 && T == 64) return launch_t<2, 64>(tmK, tmV, p, grid, smem, stream);
    if (es == 2 && T == 128) return launch_t<2, 128>(tmK, tmV, p, grid, smem, stream);
    if (es == 1 && T == 64) return launch_t<1, 64>(tmK, tmV, p, grid, smem, stream);
    if (es == 1 && T == 128) return launch_t<1, 128>(tmK, tmV, p, grid, smem, stream);
    if (es == 4 && T == 32) return launch_t<4, 32>(tmK, tmV, p, grid, smem, stream);
    if (es == 4 && T == 64) return launch_t<4, 64>(tmK, tmV, p, grid, smem, stream);
    return cudaErrorInvalidValue;
}

}  // namespace qup
