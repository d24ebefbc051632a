// union_attn.cu -- ID-aware union attention for sm_100a (PageWeaver,
// Abstract; Figure 1; Figure 3), re-designed for tcgen05 + TMEM.
//
// One persistent CTA per SM walks (KV head, group) work items.  A group has
// R = members * g query rows (g = Hq / Hkv), at most 32, which is far below
// the M = 128 rows of a tcgen05 MMA, so the two products are computed
// transposed, with the page tokens on the M side:
//      S^T[t][r] = sum_d K[t][d] Q[r][d]          M = 128 tokens, N = R_pad, K = d
//      O^T[d][r] += sum_t V^T[d][t] P^T[t][r]     M = d = 128,    N = R_pad, K = 128 tokens
// A pipeline step covers 128 consecutive union tokens (128 / T union pages).
// Both accumulators live in TMEM: two S^T buffers (double-buffered so the QK^T
// of step s+1 overlaps the softmax of step s) and one O^T.
//
// Warp roles (192 threads):
//   warp 0     producer: loads the union page list, row masks and physical
//              pages (warp-parallel), then TMA-loads each step's K and V
//              tiles into an NS-slot shared-memory ring (Figure 3's KV slots,
//              with mbarrier "ready" and "released" events).
//   warp 1     MMA issuer (one thread) and TMEM owner.
//   warps 2-5  softmax / epilogue (128 threads, thread = one TMEM lane):
//              gather the members' Q rows by original ID into the swizzled
//              Q operand tile, then per step read S^T, apply the row mask
//              (bit r of the union page's mask), the causal mask
//              (pos(t) <= q_pos) and t < kv_len, run the fp32 online softmax
//              (the column max is a warp transpose-reduce plus a 4-warp
//              exchange), rescale O^T in TMEM when a row max grows, and
//              write P^T into the MN-major P operand tile.  The epilogue
//              divides by the row sums and writes each row to O[qid][h'].
//
// Operand element types: bf16 (kind::f16), fp32 (kind::tf32) and FP8 E4M3
// (kind::f8f6f4: K and V straight from the cache; Q is quantised per row
// with its own scale, P is stored as E4M3 of 256 * p).  Every MMA consumes 32
// bytes of its K extent per row, so the descriptor arithmetic is the same for
// all three.
//
// Every wait is bounded (ptx.cuh: mbar_wait); on a timeout the CTA raises an
// abort flag, drains its in-flight TMA loads and MMAs, frees TMEM and exits.
#include <cstdint>
#include <cuda.h>

#include "internal.h"
#include "ptx.cuh"
#include "query_union_paged.h"

namespace qup {

constexpr int kThreads = 192;
constexpr int kD = kHeadDim;
constexpr int kTmemCols = 128;  // S^T buffers at columns [0,32) and [32,64), O^T at [64,96)

struct StageMeta {
    int32_t upage[kMaxPPS];
    uint64_t mask[kMaxPPS];
};

template <int ES>
struct Geo {
    static constexpr int kTile = kStepTok * kD * ES;  // one K or V tile of a step
    static constexpr int kStage = 2 * kTile;
    static constexpr int kChunkElems = 128 / ES;      // elements per 128-byte swizzle row
    static constexpr int kNChunk = kD * ES / 128;     // 128-byte chunks along d
    static constexpr int kChunkBytes = kStepTok * 128;  // one chunk column of a tile
    static constexpr int kMmaK = 32 / ES;             // K elements per MMA instruction
    static constexpr int kNumMma = kD * ES / 32;      // MMAs per S^T (K = d) and per PV (K = 128 tokens)
    static constexpr uint32_t kFmt = (ES == 2) ? 1u : (ES == 4 ? 2u : 0u);
    static constexpr int kKind = (ES == 2) ? 0 : (ES == 4 ? 1 : 2);
};

struct SmemLayout {
    uint32_t stages, q, p, bars, meta, red, bc, qsc, misc;
    uint32_t total;
};

__host__ __device__ inline SmemLayout smem_layout(int es, int r_pad, int n_stages, int Hkv) {
    SmemLayout L;
    uint32_t off = 0;
    L.stages = off;
    off += (uint32_t)n_stages * 2u * kStepTok * kD * es;
    L.q = off;
    off += (uint32_t)r_pad * kD * es;
    off = (off + 1023u) & ~1023u;
    L.p = off;
    off += (uint32_t)kStepTok * r_pad * es;
    off = (off + 1023u) & ~1023u;
    L.bars = off;
    off += 8u * (2u * n_stages + 8u);
    L.meta = off;
    off += (uint32_t)sizeof(StageMeta) * n_stages;
    L.red = off;
    off += 2u * 4u * 32u * 4u;
    L.bc = off;
    off += 4u * 2u * 32u * 4u;
    L.qsc = off;
    off += 32u * 4u;
    L.misc = off;
    off += 16u + 4u * (uint32_t)(Hkv + 1);
    L.total = off + 1024u;  // slack for aligning the dynamic base to 1024
    return L;
}

// barrier indices inside the barrier block
__device__ __forceinline__ uint32_t bar_full(uint32_t b, int s) { return b + 8u * s; }
__device__ __forceinline__ uint32_t bar_empty(uint32_t b, int s, int ns) { return b + 8u * (ns + s); }
__device__ __forceinline__ uint32_t bar_sfull(uint32_t b, int i, int ns) { return b + 8u * (2 * ns + i); }
__device__ __forceinline__ uint32_t bar_sfree(uint32_t b, int i, int ns) { return b + 8u * (2 * ns + 2 + i); }
__device__ __forceinline__ uint32_t bar_pfull(uint32_t b, int ns) { return b + 8u * (2 * ns + 4); }
__device__ __forceinline__ uint32_t bar_pvdone(uint32_t b, int ns) { return b + 8u * (2 * ns + 5); }
__device__ __forceinline__ uint32_t bar_qfull(uint32_t b, int ns) { return b + 8u * (2 * ns + 6); }
__device__ __forceinline__ uint32_t bar_drain(uint32_t b, int ns) { return b + 8u * (2 * ns + 7); }

struct Item {
    int h, nm, ub, nU, nsteps, gp0;
    bool ok;
};

// Decode flat work item f; every role calls this and reaches the same verdict.
__device__ __forceinline__ Item load_item(const AttnParams& p, const int* ng_prefix, int f) {
    Item it;
    int h = 0;
    while (h + 1 < p.Hkv && ng_prefix[h + 1] <= f) ++h;
    const int gi = f - ng_prefix[h];
    const size_t gp = (size_t)h * (p.Nq + 1) + gi;
    it.h = h;
    it.gp0 = p.group_ptr[gp];
    it.nm = p.group_ptr[gp + 1] - it.gp0;
    it.ub = p.union_ptr[gp];
    it.nU = p.union_ptr[gp + 1] - it.ub;
    const int pps = kStepTok / p.T;
    it.ok = it.nm >= 1 && it.nm <= p.max_members && it.gp0 >= 0 && it.gp0 + it.nm <= p.Nq &&
            it.ub >= 0 && it.nU >= 0 && (long long)it.ub + it.nU <= p.cap_union;
    if (!it.ok) it.nU = 0;
    it.nsteps = it.ok ? (it.nU + pps - 1) / pps : 0;
    return it;
}

// byte offset of 16-byte chunk c of row r inside a K-major SW128 operand tile with `rows` rows
__device__ __forceinline__ uint32_t kmajor_sw128(int r, int c, int rows) {
    return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// swizzle the byte offset of an MN-major P tile (row = token, rowbytes = 32/64/128):
// 16-byte units XOR the row bits (32/64/128-byte swizzle), or for 32-bit (tf32)
// operands, whose only MN-major layout is the 128-byte swizzle with 32-byte
// atoms, 32-byte units XOR (row & 3).
template <int ES>
__device__ __forceinline__ uint32_t swz_off(uint32_t off, uint32_t mask) {
    if constexpr (ES == 4) return off ^ (((off >> 7) & 3u) << 5);
    else return off ^ (((off >> 7) & mask) << 4);
}

// After this, lane r of the warp holds the max (or sum) over the warp's 32
// lanes of column r of v (RP = 32 columns), or of column r & 15 (RP = 16).
// A recursive-halving transpose: 31 shuffles instead of 32 x 5.
template <int RP, bool MAX>
__device__ __forceinline__ void transpose_reduce(float (&v)[32], int lane) {
    auto op = [](float a, float b) { return MAX ? fmaxf(a, b) : a + b; };
    if constexpr (RP == 32) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const bool up = lane & 16;
            const float send = up ? v[i] : v[i + 16];
            const float keep = up ? v[i + 16] : v[i];
            v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = op(v[i], __shfl_xor_sync(0xffffffffu, v[i], 16));
    }
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1) {
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const bool up = lane & s;
            const float send = up ? v[i] : v[i + s];
            const float keep = up ? v[i + s] : v[i];
            v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, s));
        }
    }
}

template <int RP>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[32]) {
    if constexpr (RP == 32) {
        tmem_ld32(taddr, v);
    } else {
        tmem_ld16(taddr, v);
#pragma unroll
        for (int r = 16; r < 32; ++r) v[r] = 0u;
    }
}

template <int RP>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&v)[32]) {
    if constexpr (RP == 32) tmem_st32(taddr, v);
    else tmem_st16(taddr, v);
}

// every lane agrees: a failed wait anywhere in the warp fails the warp
__device__ __forceinline__ bool warp_ok(bool ok) { return __all_sync(0xffffffffu, ok); }

template <int ES, int RP>
__global__ void __launch_bounds__(kThreads, 1)
    union_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ AttnParams p) {
    using G = Geo<ES>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const SmemLayout L = smem_layout(ES, RP, p.n_stages, p.Hkv);
    const int NS = p.n_stages;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + L.bars;
    StageMeta* meta = reinterpret_cast<StageMeta*>(smem + L.meta);
    float* red = reinterpret_cast<float*>(smem + L.red);
    float* bc = reinterpret_cast<float*>(smem + L.bc);
    float* qsc = reinterpret_cast<float*>(smem + L.qsc);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
    int* ng_prefix = reinterpret_cast<int*>(smem + L.misc + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t lim = p.wait_limit_ns;

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar_full(bars, s), 1);
            mbar_init(bar_empty(bars, s, NS), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_sfull(bars, i, NS), 1);
            mbar_init(bar_sfree(bars, i, NS), 128);
        }
        mbar_init(bar_pfull(bars, NS), 128);
        mbar_init(bar_pvdone(bars, NS), 1);
        mbar_init(bar_qfull(bars, NS), 128);
        mbar_init(bar_drain(bars, NS), 1);
        fence_mbar_init();
        *abort_flag = 0;
        int acc = 0;
        for (int h = 0; h < p.Hkv; ++h) {
            ng_prefix[h] = acc;
            int n = p.n_groups[h];
            if (n < 0 || n > p.Nq) {
                atomicOr(p.err, QUP_ERR_GROUP);
                n = 0;
            }
            acc += n;
        }
        ng_prefix[p.Hkv] = acc;
    }
    if (threadIdx.x == 32) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    // Q and P operand tiles start zeroed: rows past a group's R must hold finite values
    for (uint32_t o = threadIdx.x * 16u; o < L.bars - L.q; o += kThreads * 16u)
        *reinterpret_cast<uint4*>(smem + L.q + o) = make_uint4(0, 0, 0, 0);
    if (warp == 1) {
        tmem_alloc(smem_u32((const void*)tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_items = ng_prefix[p.Hkv];
    const int pps = kStepTok / p.T;

    if (warp == 0) {
        // ============================================================ producer (whole warp)
        int gs = 0;
        int last_issue[kMaxStages];
#pragma unroll
        for (int s = 0; s < kMaxStages; ++s) last_issue[s] = -1;
        bool ok = true;
        for (int f = blockIdx.x; f < n_items && ok; f += gridDim.x) {
            const Item it = load_item(p, ng_prefix, f);
            const int n_ent = it.nsteps * pps;  // union entries incl. padding of the last step
            for (int c0 = 0; c0 < n_ent && ok; c0 += 32) {
                const int idx = c0 + lane;
                int u = 0, phys = p.P_phys;  // P_phys: out of the tensor, TMA fills zeros
                uint64_t mk = 0;
                if (idx < it.nU) {
                    u = p.union_pages[it.ub + idx];
                    mk = p.row_mask[it.ub + idx];
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
                    if (phys == p.P_phys) mk = 0;
                }
                const int steps_here = min(32, n_ent - c0) / pps;
                for (int sl = 0; sl < steps_here; ++sl, ++gs) {
                    const int slot = gs % NS;
                    int okv = 0;
                    if (lane == 0)
                        okv = mbar_wait(bar_empty(bars, slot, NS), ((gs / NS) & 1) ^ 1, abort_flag, p.err,
                                        QUP_ERR_TIMEOUT, lim);
                    ok = __shfl_sync(0xffffffffu, okv, 0) != 0;
                    if (!ok) break;
                    int up_l[kMaxPPS], ph_l[kMaxPPS];
                    uint64_t mk_l[kMaxPPS];
#pragma unroll
                    for (int q = 0; q < kMaxPPS; ++q) {
                        const int src = (sl * pps + q) & 31;
                        up_l[q] = __shfl_sync(0xffffffffu, u, src);
                        ph_l[q] = __shfl_sync(0xffffffffu, phys, src);
                        mk_l[q] = __shfl_sync(0xffffffffu, mk, src);
                    }
                    if (lane == 0 && !(p.dbg_skip_stage >= 0 && blockIdx.x == 0 && gs == p.dbg_skip_stage)) {
                        StageMeta& m = meta[slot];
                        for (int q = 0; q < pps; ++q) {
                            m.upage[q] = up_l[q];
                            m.mask[q] = mk_l[q];
                        }
                        const uint32_t fb = bar_full(bars, slot);
                        mbar_arrive_expect_tx(fb, G::kStage);
                        const uint32_t kdst = sbase + L.stages + (uint32_t)slot * G::kStage;
                        const uint32_t vdst = kdst + G::kTile;
                        for (int q = 0; q < pps; ++q) {
#pragma unroll
                            for (int c = 0; c < G::kNChunk; ++c) {
                                const uint32_t off = (uint32_t)c * G::kChunkBytes + (uint32_t)(q * p.T) * 128u;
                                tma_load_4d(kdst + off, &tmK, fb, c * G::kChunkElems, 0, it.h, ph_l[q]);
                                tma_load_4d(vdst + off, &tmV, fb, c * G::kChunkElems, 0, it.h, ph_l[q]);
                            }
                        }
                        last_issue[slot] = gs;
                    }
                    __syncwarp();
                }
            }
        }
        // every issued load lands before the CTA may exit
        if (lane == 0) {
            for (int s = 0; s < NS; ++s)
                if (last_issue[s] >= 0) mbar_wait_drain(bar_full(bars, s), (last_issue[s] / NS) & 1, lim);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ============================================================ MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t prow = (uint32_t)RP * ES;  // P row bytes: 32, 64 or 128
            // MN-major operands: 128/64/32-byte swizzle with 8-row atoms; tf32 needs the
            // 128-byte swizzle with 32-byte atoms (layout 1), whose atoms are 4 rows
            constexpr uint32_t playout = ES == 4 ? 1u : (prow == 128 ? 2u : (prow == 64 ? 4u : 6u));
            constexpr uint32_t psbo = ES == 4 ? 4 * prow : 8 * prow;
            constexpr uint32_t vlayout = ES == 4 ? 1u : 2u;
            constexpr uint32_t vsbo = ES == 4 ? 512u : 1024u;
            const uint32_t idesc_s = instr_desc(G::kFmt, 0, 0, RP, 128);
            const uint32_t idesc_o = instr_desc(G::kFmt, 1, 1, RP, 128);
            const uint32_t qbase = sbase + L.q, pbase = sbase + L.p;
            int gs = 0, item_no = 0;
            bool ok = true;
            for (int f = blockIdx.x; f < n_items && ok; f += gridDim.x, ++item_no) {
                const Item it = load_item(p, ng_prefix, f);
                ok = mbar_wait(bar_qfull(bars, NS), item_no & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim);
                if (!ok) break;
                tc_fence_after();
                // S(s) is issued before PV(s-1) so QK^T overlaps the softmax; with a
                // single ring stage S(s) needs the slot PV(s-1) frees, so PV goes first
                const bool pv_first = NS == 1;
                for (int s = 0; s <= it.nsteps && ok; ++s) {
                    for (int half = 0; half < 2 && ok; ++half) {
                        const bool do_s = (half == (pv_first ? 1 : 0)) && s < it.nsteps;
                        const bool do_pv = (half == (pv_first ? 0 : 1)) && s > 0;
                        if (do_s) {
                            const int g = gs + s, slot = g % NS, b = g & 1;
                            ok = mbar_wait(bar_full(bars, slot), (g / NS) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT,
                                           lim) &&
                                 mbar_wait(bar_sfree(bars, b, NS), ((g >> 1) & 1) ^ 1, abort_flag, p.err,
                                           QUP_ERR_TIMEOUT, lim);
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t kbase = sbase + L.stages + (uint32_t)slot * G::kStage;
#pragma unroll
                            for (int k = 0; k < G::kNumMma; ++k) {
                                const uint32_t koff = (uint32_t)(k >> 2) * G::kChunkBytes + (uint32_t)(k & 3) * 32u;
                                const uint32_t qoff = (uint32_t)(k >> 2) * (RP * 128u) + (uint32_t)(k & 3) * 32u;
                                tc_mma<G::kKind>(tmem + (uint32_t)b * 32u, smem_desc(kbase + koff, 16, 1024, 2),
                                                 smem_desc(qbase + qoff, 16, 1024, 2), idesc_s, k > 0);
                            }
                            tc_commit(bar_sfull(bars, b, NS));
                        }
                        if (do_pv) {
                            const int g = gs + s - 1, slot = g % NS;
                            ok = mbar_wait(bar_pfull(bars, NS), g & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim);
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t vbase = sbase + L.stages + (uint32_t)slot * G::kStage + G::kTile;
#pragma unroll
                            for (int k = 0; k < G::kNumMma; ++k) {
                                // K step = kMmaK tokens: kMmaK rows of V (128 B) and of P (prow B)
                                tc_mma<G::kKind>(tmem + 64u,
                                                 smem_desc(vbase + (uint32_t)(k * G::kMmaK) * 128u,
                                                           (uint32_t)G::kChunkBytes, vsbo, vlayout),
                                                 smem_desc(pbase + (uint32_t)(k * G::kMmaK) * prow, 16 * prow,
                                                           psbo, playout),
                                                 idesc_o, (s - 1) > 0 || k > 0);
                            }
                            tc_commit(bar_empty(bars, slot, NS));
                            tc_commit(bar_pvdone(bars, NS));
                        }
                    }
                }
                gs += it.nsteps;
            }
            // every issued MMA completes before TMEM is freed
            tc_commit(bar_drain(bars, NS));
            mbar_wait_drain(bar_drain(bars, NS), 0, lim);
        }
        __syncwarp();
    } else {
        // ============================================================ softmax / epilogue (128 threads)
        const int sw = warp - 2;                 // 0..3
        const int quad = warp & 3;               // TMEM lane quadrant this warp may access
        const int L_tok = quad * 32 + lane;      // step-tile token == S^T lane; O^T lane == feature d
        const int tid = sw * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const float kNegInf = -__int_as_float(0x7f800000);
        constexpr uint32_t prow = (uint32_t)RP * ES;
        constexpr uint32_t pmask = prow == 128 ? 7u : (prow == 64 ? 3u : 1u);
        uint8_t* qtile = smem + L.q;
        uint8_t* ptile = smem + L.p;
        int gs = 0, xphase = 0;  // xphase alternates the two 4-warp exchange buffers
        bool ok = true;
        for (int f = blockIdx.x; f < n_items; f += gridDim.x) {
            const Item it = load_item(p, ng_prefix, f);
            if (!it.ok && tid == 0) atomicOr(p.err, QUP_ERR_GROUP);
            // ---- members (lane m holds member m), positions, Q gather by original ID
            int qid_m = 0, qpos_m = 0;
            bool mem_ok = true;
            if (lane < it.nm) {
                qid_m = p.members[(size_t)it.h * p.Nq + it.gp0 + lane];
                if (qid_m < 0 || qid_m >= p.Nq) {
                    mem_ok = false;
                    qid_m = 0;
                }
                qpos_m = p.q_pos[qid_m];
            }
            if (!warp_ok(mem_ok) && tid == 0) atomicOr(p.err, QUP_ERR_GROUP);
            const int R = it.nm * p.g;
            {
                constexpr int CPR = 8 * ES;    // 16-byte chunks per Q row in shared memory
                constexpr int RPP = 128 / CPR;  // rows per pass
                const int c = tid % CPR;
#pragma unroll 1
                for (int r0 = 0; r0 < RP; r0 += RPP) {
                    const int r = r0 + tid / CPR;
                    const int m = r / p.g, j = r % p.g;
                    const int qid = __shfl_sync(0xffffffffu, qid_m, m & 7);
                    const bool live = r < R;
                    const size_t row_off = ((size_t)qid * p.Hq + (size_t)it.h * p.g + j) * kD;
                    uint4 out = make_uint4(0, 0, 0, 0);
                    if constexpr (ES == 4) {
                        if (live) out = *reinterpret_cast<const uint4*>(static_cast<const float*>(p.Q) + row_off + c * 4);
                    } else if constexpr (ES == 2) {
                        if (live) out = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.Q) + row_off + c * 8);
                    } else {
                        // 16 bf16 -> 16 E4M3 with the row's scale amax / 448
                        float x[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) x[e] = 0.f;
                        if (live) {
                            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.Q) + row_off + c * 16);
                            const uint4 a0 = src[0], a1 = src[1];
                            const uint32_t w[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                x[2 * e] = __uint_as_float(w[e] << 16);
                                x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                            }
                        }
                        float amax = 0.f;
#pragma unroll
                        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
                        for (int o = 1; o < CPR; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                        const float inv = amax > 0.f ? 448.f / amax : 0.f;
                        out.x = pack_e4m3x4(x[0] * inv, x[1] * inv, x[2] * inv, x[3] * inv);
                        out.y = pack_e4m3x4(x[4] * inv, x[5] * inv, x[6] * inv, x[7] * inv);
                        out.z = pack_e4m3x4(x[8] * inv, x[9] * inv, x[10] * inv, x[11] * inv);
                        out.w = pack_e4m3x4(x[12] * inv, x[13] * inv, x[14] * inv, x[15] * inv);
                        if (c == 0) qsc[r] = amax * (1.f / 448.f);
                    }
                    *reinterpret_cast<uint4*>(qtile + kmajor_sw128(r, c, RP)) = out;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(bar_qfull(bars, NS));
            // ---- per-row constants: score scale (log2 domain), causal bound, output row
            float cs[32];
            if constexpr (ES == 1) {
                bar_sync(1, 128);  // qsc written by the gather
                const float ks = p.k_scale[it.h] * p.scale_log2;
#pragma unroll
                for (int r = 0; r < 32; ++r) cs[r] = (r < RP) ? qsc[r] * ks : 0.f;
            } else {
#pragma unroll
                for (int r = 0; r < 32; ++r) cs[r] = p.scale_log2;
            }
            int rpos[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) rpos[r] = __shfl_sync(0xffffffffu, qpos_m, (r / p.g) & 7);
            const uint32_t live_rows = (R >= 32) ? 0xffffffffu : ((1u << R) - 1u);

            float m_lane = kNegInf;  // lane r holds the running max of row r (log2 domain)
            float lpart[32];         // this thread's token partial of each row's sum
#pragma unroll
            for (int r = 0; r < 32; ++r) lpart[r] = 0.f;

            for (int s = 0; s < it.nsteps; ++s, ++gs) {
                const int slot = gs % NS, b = gs & 1;
                if (ok)
                    ok = mbar_wait(bar_full(bars, slot), (gs / NS) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim) &&
                         mbar_wait(bar_sfull(bars, b, NS), (gs >> 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim);
                ok = warp_ok(ok);
                float x[32];
                if (ok) {
                    uint32_t sr[32];
                    tc_fence_after();
                    tmem_ld_cols<RP>(tmem + lane_base + (uint32_t)b * 32u, sr);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(bar_sfree(bars, b, NS));
                    const int ps = L_tok / p.T, o = L_tok - ps * p.T;
                    const int u = meta[slot].upage[ps];
                    const uint64_t mk = meta[slot].mask[ps];
                    const int pos = u * p.T + o;
                    uint32_t valid = (uint32_t)mk & live_rows;
                    if (s * pps + ps >= it.nU) valid = 0;
                    if (pos >= p.kv_len) {
                        valid = 0;
                        // cache slots past kv_len may hold non-finite bytes: zero this V row
                        uint8_t* vt = smem + L.stages + (uint32_t)slot * G::kStage + G::kTile;
                        for (int c = 0; c < G::kNChunk; ++c)
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                *reinterpret_cast<uint4*>(vt + c * G::kChunkBytes + L_tok * 128 + e * 16) =
                                    make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int r = 0; r < 32; ++r) {
                        const bool v = r < RP && ((valid >> r) & 1u) && pos <= rpos[r];
                        x[r] = v ? __uint_as_float(sr[r]) * cs[r] : kNegInf;
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < 32; ++r) x[r] = kNegInf;
                }
                // ---- row max over the step's 128 tokens
                float v[32];
#pragma unroll
                for (int r = 0; r < 32; ++r) v[r] = x[r];
                transpose_reduce<RP, true>(v, lane);
                float* rb = red + (xphase & 1) * 128;
                ++xphase;
                rb[sw * 32 + lane] = v[0];
                ok = bar_and(1, 128, ok);
                if (!ok) break;
                {
                    const float mx = fmaxf(fmaxf(rb[lane], rb[32 + lane]), fmaxf(rb[64 + lane], rb[96 + lane]));
                    const float m_new = fmaxf(m_lane, mx);
                    const float m_safe = (m_new == kNegInf) ? 0.f : m_new;
                    const float alpha = ex2(m_lane - m_safe);
                    m_lane = m_new;
                    bc[sw * 64 + lane] = m_safe;
                    bc[sw * 64 + 32 + lane] = alpha;
                }
                __syncwarp();
                float msafe[32], alpha[32];
#pragma unroll
                for (int r = 0; r < 32; r += 4) {
                    const float4 a = *reinterpret_cast<const float4*>(bc + sw * 64 + r);
                    const float4 c = *reinterpret_cast<const float4*>(bc + sw * 64 + 32 + r);
                    msafe[r] = a.x; msafe[r + 1] = a.y; msafe[r + 2] = a.z; msafe[r + 3] = a.w;
                    alpha[r] = c.x; alpha[r + 1] = c.y; alpha[r + 2] = c.z; alpha[r + 3] = c.w;
                }
                float pv[32];
                bool rescale = false;
#pragma unroll
                for (int r = 0; r < 32; ++r) {
                    pv[r] = ex2(x[r] - msafe[r]);
                    lpart[r] = lpart[r] * alpha[r] + pv[r];
                    if (r < RP) rescale |= alpha[r] != 1.f;
                }
                if (s > 0) {
                    ok = warp_ok(mbar_wait(bar_pvdone(bars, NS), (gs - 1) & 1, abort_flag, p.err,
                                           QUP_ERR_TIMEOUT, lim));
                    if (ok) {
                        tc_fence_after();
                        if (rescale) {  // uniform: alpha comes from the shared exchange
                            uint32_t ov[32];
                            const uint32_t oaddr = tmem + lane_base + 64u;
                            tmem_ld_cols<RP>(oaddr, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int r = 0; r < 32; ++r)
                                ov[r] = __float_as_uint(__uint_as_float(ov[r]) * alpha[r]);
                            tmem_st_cols<RP>(oaddr, ov);
                            tmem_wait_st();
                        }
                    }
                }
                if (ok) {
                    // ---- this token's P^T row into the MN-major operand tile
                    const uint32_t rowoff = (uint32_t)L_tok * prow;
                    if constexpr (ES == 2) {
#pragma unroll
                        for (int c = 0; c < RP / 8; ++c) {
                            uint4 w;
                            w.x = pack_bf16x2(pv[c * 8 + 0], pv[c * 8 + 1]);
                            w.y = pack_bf16x2(pv[c * 8 + 2], pv[c * 8 + 3]);
                            w.z = pack_bf16x2(pv[c * 8 + 4], pv[c * 8 + 5]);
                            w.w = pack_bf16x2(pv[c * 8 + 6], pv[c * 8 + 7]);
                            *reinterpret_cast<uint4*>(ptile + swz_off<ES>(rowoff + c * 16, pmask)) = w;
                        }
                    } else if constexpr (ES == 4) {
#pragma unroll
                        for (int c = 0; c < RP / 4; ++c) {
                            const uint4 w = make_uint4(__float_as_uint(pv[c * 4]), __float_as_uint(pv[c * 4 + 1]),
                                                       __float_as_uint(pv[c * 4 + 2]), __float_as_uint(pv[c * 4 + 3]));
                            *reinterpret_cast<uint4*>(ptile + swz_off<ES>(rowoff + c * 16, pmask)) = w;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < RP / 16; ++c) {
                            const float* q = pv + c * 16;
                            uint4 w;
                            w.x = pack_e4m3x4(q[0] * 256.f, q[1] * 256.f, q[2] * 256.f, q[3] * 256.f);
                            w.y = pack_e4m3x4(q[4] * 256.f, q[5] * 256.f, q[6] * 256.f, q[7] * 256.f);
                            w.z = pack_e4m3x4(q[8] * 256.f, q[9] * 256.f, q[10] * 256.f, q[11] * 256.f);
                            w.w = pack_e4m3x4(q[12] * 256.f, q[13] * 256.f, q[14] * 256.f, q[15] * 256.f);
                            *reinterpret_cast<uint4*>(ptile + swz_off<ES>(rowoff + c * 16, pmask)) = w;
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(bar_pfull(bars, NS));
                }
            }
            // ---- epilogue: row sums, lse, O^T / l -> O[qid][h*g + j][d]
            if (ok && it.nsteps > 0)
                ok = mbar_wait(bar_pvdone(bars, NS), (gs - 1) & 1, abort_flag, p.err, QUP_ERR_TIMEOUT, lim);
            ok = warp_ok(ok);
            transpose_reduce<RP, false>(lpart, lane);
            float* rb = red + (xphase & 1) * 128;
            ++xphase;
            rb[sw * 32 + lane] = lpart[0];
            ok = bar_and(1, 128, ok);
            if (!ok) break;
            {
                const float l = rb[lane] + rb[32 + lane] + rb[64 + lane] + rb[96 + lane];
                bc[sw * 64 + lane] = l > 0.f ? 1.f / l : 0.f;
            }
            if (p.lse != nullptr && sw == 0) {
                // m_lane is in the log2 domain (scores * log2 e); lse is a natural log
                const float l = rb[lane] + rb[32 + lane] + rb[64 + lane] + rb[96 + lane];
                const int qid = __shfl_sync(0xffffffffu, qid_m, (lane / p.g) & 7);
                if (lane < R) {
                    const int j = lane % p.g;
                    p.lse[(size_t)qid * p.Hq + (size_t)it.h * p.g + j] =
                        l > 0.f ? (m_lane + __log2f(l)) * 0.69314718055994531f : kNegInf;
                }
            }
            __syncwarp();
            float vsc = 1.f;
            if constexpr (ES == 1) vsc = p.v_scale[it.h] * (1.f / 256.f);
            uint32_t ov[32];
            if (it.nsteps > 0) {
                tc_fence_after();
                tmem_ld_cols<RP>(tmem + lane_base + 64u, ov);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int r = 0; r < 32; ++r) ov[r] = 0u;
            }
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const int qid = __shfl_sync(0xffffffffu, qid_m, (r / p.g) & 7);
                if (r < R) {
                    const float val = __uint_as_float(ov[r]) * bc[sw * 64 + r] * vsc;
                    const size_t oi = ((size_t)qid * p.Hq + (size_t)it.h * p.g + (r % p.g)) * kD + L_tok;
                    if constexpr (ES == 4) static_cast<float*>(p.O)[oi] = val;
                    else static_cast<uint16_t*>(p.O)[oi] = (uint16_t)(pack_bf16x2(val, 0.f) & 0xffffu);
                }
            }
            tc_fence_before();
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

size_t attn_smem_bytes(int es, int r_pad, int n_stages, int Hkv) {
    return smem_layout(es, r_pad, n_stages, Hkv).total;
}

template <int ES, int RP>
static cudaError_t launch_t(const CUtensorMap& tmK, const CUtensorMap& tmV, const AttnParams& p, int grid,
                            size_t smem, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(union_attn_kernel<ES, RP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    union_attn_kernel<ES, RP><<<grid, kThreads, smem, stream>>>(tmK, tmV, p);
    return cudaGetLastError();
}

cudaError_t launch_union_attn(int es, int r_pad, const CUtensorMap& tmK, const CUtensorMap& tmV,
                              const AttnParams& p, int grid, size_t smem, cudaStream_t stream) {
    if (es == 2 && r_pad == 32) return launch_t<2, 32>(tmK, tmV, p, grid, smem, stream);
    if (es == 2 && r_pad == 16) return launch_t<2, 16>(tmK, tmV, p, grid, smem, stream);
    if (es == 4 && r_pad == 32) return launch_t<4, 32>(tmK, tmV, p, grid, smem, stream);
    if (es == 1 && r_pad == 32) return launch_t<1, 32>(tmK, tmV, p, grid, smem, stream);
    return cudaErrorInvalidValue;
}

}  // namespace qup
