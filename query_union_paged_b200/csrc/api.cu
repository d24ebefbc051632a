// api.cu -- C ABI host layer: argument validation, workspace carving, TMA
// tensor-map encoding, launches and the per-device error word.  Nothing here
// allocates device memory; every buffer comes from the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "select.h"
#include "query_union_paged.h"

namespace qup {
// batch.cu: request-local TopK IDs -> global IDs, per-query visible ends, per-page valid tokens
cudaError_t launch_batch_prepare(const int32_t* topk, const int32_t* q_pos, int Hq, int Nq, int K, int T, int R,
                                 const int32_t* q_ptr, const int32_t* page_ptr, const int32_t* kv_len, int total_pages,
                                 int32_t* topk_global, int32_t* q_end, int32_t* page_len, unsigned* err,
                                 cudaStream_t stream);
// group.cu: every row of each group sees every page of the group's union (row masks set to the
// group's rows)
cudaError_t launch_union_support(const int32_t* n_groups, const int32_t* group_ptr, const int32_t* union_ptr,
                                 uint64_t* row_mask, int Hkv, int Nq, int g, long long cap, unsigned* err, int sms,
                                 cudaStream_t stream);
}  // namespace qup

namespace {

__device__ unsigned g_err_word;  // ORed device error bits, read and cleared by qup_get_error

constexpr int kMaxDevices = 64;

struct DevState {
    unsigned long long ctx = 0;  // context the fields below were looked up in (0: not yet)
    unsigned* err = nullptr;     // device address of g_err_word in that context
    int sms = 0;
    int smem_optin = 0;
};

std::mutex g_mu;
DevState g_dev[kMaxDevices];
std::atomic<int> g_wait_limit_ms{0};  // 0: default
std::atomic<int> g_skip_stage{-1};
std::atomic<int> g_checked{0};  // checked mode: attention validates the row masks against topk
std::atomic<unsigned> g_walk_slot{0};  // the next launch slot of the attention kernel's bundle counter

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int device_state(DevState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QUP_ERR_CUDA;
    const unsigned long long ctx = qup::context_id();
    if (ctx == 0) return QUP_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DevState& s = g_dev[dev];
    if (s.ctx != ctx) {  // first call in this context (a reset or another context starts over)
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return QUP_ERR_CUDA;
        s.err = static_cast<unsigned*>(p);
        if (cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return QUP_ERR_CUDA;
        if (cudaDeviceGetAttribute(&s.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return QUP_ERR_CUDA;
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return QUP_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        s.ctx = ctx;
    }
    *out = &s;
    return QUP_OK;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct GroupWs {
    size_t rowbits, usize, wtot, wcnt, fwcnt, fstatus, total;
};

GroupWs group_ws_layout(int Hq, int Hkv, int Nq, int NW, int nwin) {
    GroupWs w;
    size_t off = 0;
    w.rowbits = off;
    off = align256(off + sizeof(uint32_t) * (size_t)Hq * Nq * NW);
    w.usize = off;
    off = align256(off + sizeof(int32_t) * (size_t)Hkv * Nq);
    w.wtot = off;
    off = align256(off + sizeof(int32_t) * (size_t)Hkv * nwin);
    w.wcnt = off;
    off = align256(off + sizeof(int32_t) * 3 * (size_t)Hkv * nwin);
    // fused path: per-window counters of both kernels, look-back status words of both
    // kernels and the bundle kernel's completion count (windows: at most Nq per head)
    w.fwcnt = off;
    off = align256(off + sizeof(int32_t) * 5 * (size_t)Hkv * std::max(Nq, 1));
    w.fstatus = off;
    off = align256(off + sizeof(uint64_t) * 2 * (size_t)Hkv * std::max(Nq, 1) + 16);  // + done word, 2 tickets
    w.total = off;
    return w;
}

// Bundle geometry: rows per group slot (power of two >= max_group*g), slots
// per 128-row bundle, and the bundling window (a multiple of the slots).
void bundle_geometry(int g, int max_group, int bundle_window, int* RS, int* slots, int* WB) {
    int rs = 1;
    while (rs < max_group * g) rs <<= 1;
    *RS = rs;
    *slots = 128 / rs;
    int wb = bundle_window > 0 ? bundle_window : 64;
    wb = (wb / *slots) * *slots;
    *WB = wb < *slots ? *slots : wb;
}

// The fused kernels keep a whole window in shared memory: they run when it fits.
bool fused_group_ok(int g, int NW, int W, const DevState* ds) {
    return W <= 256 && qup::fused_group_smem(W, g, NW) <= (size_t)ds->smem_optin;
}
bool fused_bundle_ok(int NW, int WB, int Hkv, const DevState* ds) {
    return WB <= 256 && qup::fused_bundle_smem(WB, NW, Hkv) <= (size_t)ds->smem_optin;
}

int check_group_args(int Hq, int Hkv, int Nq, int K, int P, int max_group, int window) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Nq < 0 || K < 0 || P <= 0) return QUP_ERR_ARG;
    const int g = Hq / Hkv;
    if (max_group < 1 || max_group > 8 || max_group * g > 32) return QUP_ERR_ARG;
    if (window < max_group || window % max_group != 0 || window > 256) return QUP_ERR_ARG;
    return QUP_OK;
}

}  // namespace

extern "C" {

int qup_group_workspace(int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages, int max_group, int window,
                        size_t* ws_bytes, int64_t* cap_union) {
    int rc = check_group_args(Hq, Hkv, Nq, Ksel, num_logical_pages, max_group, window);
    if (rc) return rc;
    const int NW = (num_logical_pages + 31) / 32;
    const int g = Hq / Hkv;
    int RS, slots, WB;
    bundle_geometry(g, max_group, 0, &RS, &slots, &WB);
    const int nwin = std::max((Nq + window - 1) / window, (Nq + slots - 1) / slots);
    // the greedy kernels keep a window's bitsets in shared memory (227 KB per CTA)
    if (qup::group_greedy_smem(window, NW) > 227u * 1024u || qup::group_greedy_smem(std::max(WB, 256), NW) > 227u * 1024u ||
        8u * 4u * (size_t)NW > 227u * 1024u)
        return QUP_ERR_ARG;
    const int64_t cap = (int64_t)Hkv * Nq * std::min<int64_t>((int64_t)g * Ksel, num_logical_pages);
    if (cap >= ((int64_t)1 << 31)) return QUP_ERR_ARG;  // union offsets are int32
    (void)nwin;
    if (ws_bytes) *ws_bytes = group_ws_layout(Hq, Hkv, Nq, NW, std::max(Nq, 1)).total;
    if (cap_union) *cap_union = std::max<int64_t>(cap, 1);
    return QUP_OK;
}

}  // extern "C"

namespace {

// gbits_ready: the group bitsets are already in the workspace (written by the fused group
// kernel, which also zeroed the bundle status words: they follow its own, at
// fused_status_offset words into the status region).
// max_groups: an upper bound of the groups of one KV head (Nq for any partition).
int run_bundles(qup_groups* g, int Hq, int Hkv, int Nq, int num_logical_pages, int max_group, void* ws,
                DevState* ds, cudaStream_t st, bool gbits_ready = false, size_t fused_status_offset = 0,
                int max_groups = -1) {
    const int gq = Hq / Hkv;
    int RS, slots, WB;
    bundle_geometry(gq, max_group, g->bundle_window, &RS, &slots, &WB);
    g->rows_per_group = RS;
    if (Nq == 0) {
        if (cudaMemsetAsync(g->n_bundles, 0, sizeof(int32_t) * Hkv, st) != cudaSuccess ||
            cudaMemsetAsync(g->bundle_ptr, 0, sizeof(int32_t) * Hkv, st) != cudaSuccess ||
            cudaMemsetAsync(g->bunion_ptr, 0, sizeof(int32_t) * Hkv, st) != cudaSuccess ||
            cudaMemsetAsync(g->bcounters, 0, sizeof(int64_t) * 2 * Hkv, st) != cudaSuccess)
            return QUP_ERR_CUDA;
        return QUP_OK;
    }
    const int NW = (num_logical_pages + 31) / 32;
    const GroupWs L = group_ws_layout(Hq, Hkv, Nq, NW, std::max(Nq, 1));
    char* base = static_cast<char*>(ws);
    qup::BundleLaunch a;
    a.Hkv = Hkv;
    a.Nq = Nq;
    a.P = num_logical_pages;
    a.NW = NW;
    a.g = gq;
    a.RS = RS;
    a.slots = slots;
    a.WB = WB;
    a.nwin = ((max_groups >= 0 ? std::min(max_groups, Nq) : Nq) + WB - 1) / WB;
    a.n_groups = g->n_groups;
    a.group_ptr = g->group_ptr;
    a.members = g->members;
    a.union_ptr = g->union_ptr;
    a.union_pages = g->union_pages;
    a.row_mask = g->row_mask;
    a.gbits = reinterpret_cast<uint32_t*>(base + L.rowbits);
    a.ws_usize = reinterpret_cast<int32_t*>(base + L.usize);
    a.ws_wtot = reinterpret_cast<int32_t*>(base + L.wtot);
    a.ws_wcnt = reinterpret_cast<int32_t*>(base + L.wcnt);
    a.n_bundles = g->n_bundles;
    a.bundle_ptr = g->bundle_ptr;
    a.bundle_groups = g->bundle_groups;
    a.bunion_ptr = g->bunion_ptr;
    a.bunion_pages = g->bunion_pages;
    a.bunion_mask = g->bunion_mask;
    a.bundle_qid = g->bundle_qid;
    a.cap = g->cap_union;
    a.bcounters = g->bcounters;
    a.bundle_order = g->bundle_order;
    a.err = ds->err;
    a.sms = ds->sms;
    if (fused_bundle_ok(NW, WB, Hkv, ds)) {
        // status words of the bundle windows (after those of the group windows, if any), then
        // the completion count and the two window tickets (group kernel, bundle kernel), all
        // starting at zero
        uint64_t* status = reinterpret_cast<uint64_t*>(base + L.fstatus) + fused_status_offset;
        unsigned* done = reinterpret_cast<unsigned*>(status + (size_t)Hkv * a.nwin);
        int32_t* wcnt = reinterpret_cast<int32_t*>(base + L.fwcnt) + 4 * (size_t)Hkv * std::max(Nq, 1);
        if (!gbits_ready) {
            if (cudaMemsetAsync(status, 0, sizeof(uint64_t) * (size_t)Hkv * a.nwin + 3 * sizeof(unsigned), st) !=
                cudaSuccess)
                return QUP_ERR_CUDA;
        }
        if (!gbits_ready && qup::launch_gbits(a, st) != cudaSuccess) return QUP_ERR_CUDA;
        return qup::launch_bundles_fused(a, wcnt, status, done, done + 2, st) == cudaSuccess ? QUP_OK : QUP_ERR_CUDA;
    }
    return qup::launch_bundles(a, st) == cudaSuccess ? QUP_OK : QUP_ERR_CUDA;
}

bool bundle_fields_ok(const qup_groups* g) {
    return g->n_bundles && g->bundle_ptr && g->bundle_groups && g->bunion_ptr && g->bunion_pages && g->bunion_mask &&
           g->bundle_qid && g->bcounters && g->bundle_order;
}

}  // namespace

extern "C" {

int qup_build_bundles(qup_groups* g, int Hq, int Hkv, int Nq, int num_logical_pages, int max_group, void* ws,
                      size_t ws_bytes, void* stream) {
    size_t need = 0;
    int64_t cap = 0;
    int rc = qup_group_workspace(Hq, Hkv, Nq, 1, num_logical_pages, max_group, max_group, &need, &cap);
    if (rc) return rc;
    if (!g || !g->n_groups || !g->group_ptr || !g->members || !g->union_ptr || !g->union_pages || !g->row_mask ||
        !bundle_fields_ok(g))
        return QUP_ERR_ARG;
    if (g->bundle_window < 0 || g->bundle_window > 256) return QUP_ERR_ARG;
    if (!ws || ws_bytes < need) return QUP_ERR_CAPACITY;
    DevState* ds = nullptr;
    if ((rc = device_state(&ds))) return rc;
    return run_bundles(g, Hq, Hkv, Nq, num_logical_pages, max_group, ws, ds, static_cast<cudaStream_t>(stream));
}

int qup_union_support(qup_groups* g, int Hq, int Hkv, int Nq, int num_logical_pages, int max_group, void* ws,
                      size_t ws_bytes, void* stream) {
    size_t need = 0;
    int64_t cap = 0;
    int rc = qup_group_workspace(Hq, Hkv, Nq, 1, num_logical_pages, max_group, max_group, &need, &cap);
    if (rc) return rc;
    if (!g || !g->n_groups || !g->group_ptr || !g->members || !g->union_ptr || !g->union_pages || !g->row_mask ||
        !bundle_fields_ok(g))
        return QUP_ERR_ARG;
    if (g->bundle_window < 0 || g->bundle_window > 256) return QUP_ERR_ARG;
    if (!ws || ws_bytes < need) return QUP_ERR_CAPACITY;
    DevState* ds = nullptr;
    if ((rc = device_state(&ds))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (qup::launch_union_support(g->n_groups, g->group_ptr, g->union_ptr, g->row_mask, Hkv, Nq, Hq / Hkv,
                                  g->cap_union, ds->err, ds->sms, st) != cudaSuccess)
        return QUP_ERR_CUDA;
    return run_bundles(g, Hq, Hkv, Nq, num_logical_pages, max_group, ws, ds, st);
}

int qup_sparse_group(const int32_t* topk, int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages, int max_group,
                     int window, qup_groups* out, void* ws, size_t ws_bytes, void* stream) {
    size_t need = 0;
    int64_t cap = 0;
    int rc = qup_group_workspace(Hq, Hkv, Nq, Ksel, num_logical_pages, max_group, window, &need, &cap);
    if (rc) return rc;
    if (!out || !out->n_groups || !out->group_ptr || !out->members || !out->union_ptr || !out->union_pages ||
        !out->row_mask || !out->counters || !bundle_fields_ok(out))
        return QUP_ERR_ARG;
    if (out->bundle_window < 0 || out->bundle_window > 256) return QUP_ERR_ARG;
    if ((Nq > 0 && Ksel > 0 && !topk) || (!ws && need > 0)) return QUP_ERR_ARG;
    if (ws_bytes < need) return QUP_ERR_CAPACITY;
    if (out->cap_union < cap) return QUP_ERR_CAPACITY;
    DevState* ds = nullptr;
    if ((rc = device_state(&ds))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (Nq == 0) {  // nothing to group: zero groups, empty unions, zero counters
        if (cudaMemsetAsync(out->n_groups, 0, sizeof(int32_t) * Hkv, st) != cudaSuccess ||
            cudaMemsetAsync(out->group_ptr, 0, sizeof(int32_t) * Hkv, st) != cudaSuccess ||
            cudaMemsetAsync(out->union_ptr, 0, sizeof(int32_t) * Hkv, st) != cudaSuccess ||
            cudaMemsetAsync(out->counters, 0, sizeof(int64_t) * 4 * Hkv, st) != cudaSuccess)
            return QUP_ERR_CUDA;
        return run_bundles(out, Hq, Hkv, Nq, num_logical_pages, max_group, ws, ds, st);
    }
    const int NW = (num_logical_pages + 31) / 32;
    const int nwin = (Nq + window - 1) / window;
    const GroupWs L = group_ws_layout(Hq, Hkv, Nq, NW, std::max(Nq, 1));
    char* base = static_cast<char*>(ws);
    qup::GroupLaunch a;
    a.topk = topk;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Nq = Nq;
    a.K = Ksel;
    a.P = num_logical_pages;
    a.NW = NW;
    a.max_group = max_group;
    a.W = window;
    a.nwin = nwin;
    a.rowbits = reinterpret_cast<uint32_t*>(base + L.rowbits);
    a.ws_usize = reinterpret_cast<int32_t*>(base + L.usize);
    a.ws_wtot = reinterpret_cast<int32_t*>(base + L.wtot);
    a.ws_wcnt = reinterpret_cast<int32_t*>(base + L.wcnt);
    a.n_groups = out->n_groups;
    a.group_ptr = out->group_ptr;
    a.members = out->members;
    a.union_ptr = out->union_ptr;
    a.union_pages = out->union_pages;
    a.row_mask = out->row_mask;
    a.cap = out->cap_union;
    a.counters = out->counters;
    a.err = ds->err;
    a.sms = ds->sms;
    if (Ksel == 0) a.topk = nullptr;
    int RS, slots, WB;
    bundle_geometry(Hq / Hkv, max_group, out->bundle_window, &RS, &slots, &WB);
    if (fused_group_ok(Hq / Hkv, NW, window, ds) && fused_bundle_ok(NW, WB, Hkv, ds)) {
        // one memset zeroes the status words of both kernels and the completion count.  Every
        // window but the last yields window / max_group groups (groups are always filled).
        const int max_groups = std::min(Nq, nwin * ((window + max_group - 1) / max_group));
        const int nwinB = (max_groups + WB - 1) / WB;
        uint64_t* status = reinterpret_cast<uint64_t*>(base + L.fstatus);
        unsigned* done = reinterpret_cast<unsigned*>(status + (size_t)Hkv * (nwin + nwinB));
        if (cudaMemsetAsync(status, 0, sizeof(uint64_t) * (size_t)Hkv * (nwin + nwinB) + 3 * sizeof(unsigned), st) !=
            cudaSuccess)
            return QUP_ERR_CUDA;
        if (qup::launch_group_fused(a, a.rowbits, reinterpret_cast<int32_t*>(base + L.fwcnt), status, done + 1, st) !=
            cudaSuccess)
            return QUP_ERR_CUDA;
        return run_bundles(out, Hq, Hkv, Nq, num_logical_pages, max_group, ws, ds, st, true, (size_t)Hkv * nwin,
                           max_groups);
    }
    if (qup::launch_group(a, st) != cudaSuccess) return QUP_ERR_CUDA;
    return run_bundles(out, Hq, Hkv, Nq, num_logical_pages, max_group, ws, ds, st);
}

}  // extern "C"

namespace {

// The attention kernel's work list: bundles of query unions (qup_groups), or page-major items
// whose rows write partial results.
struct Work {
    const int32_t* n_bundles;
    const int32_t* union_ptr;
    const int32_t* union_pages;
    const uint32_t* row_mask;
    const int32_t* bundle_qid;
    const int32_t* bundle_order;
    long long cap_union;
    int bstride;           // bundles per KV head in the layout of union_ptr and bundle_qid
    float* part_o;         // page-major: partial results, else null
    float* part_lse;
    const int32_t* item_slot;
};

Work work_of(const qup_groups* g, int Nq) {
    Work w;
    w.n_bundles = g->n_bundles;
    w.union_ptr = g->bunion_ptr;
    w.union_pages = g->bunion_pages;
    w.row_mask = g->bunion_mask;
    w.bundle_qid = g->bundle_qid;
    w.bundle_order = g->bundle_order;
    w.cap_union = g->cap_union;
    w.bstride = Nq;
    w.part_o = nullptr;
    w.part_lse = nullptr;
    w.item_slot = nullptr;
    return w;
}

// The attention call for one sequence (q_pos, kv_len) or for batched requests (q_end, page_len),
// on the bundles of `groups` (checked mode may validate them against topk) or on a work list.
int attn_impl(const void* Q, int q_dtype, const void* K_cache, const void* V_cache, int kv_dtype,
              const float* k_scale, const float* v_scale, const int32_t* page_table, int num_logical_pages,
              int P_phys, int T, const int32_t* topk, int Ksel, const qup_groups* groups, const Work* work,
              const int32_t* q_pos, int kv_len, const int32_t* q_end, const int32_t* page_len, int Hq, int Hkv, int Nq,
              int d, float softmax_scale, void* O, float* lse, void* stream) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Nq < 0 || d != qup::kHeadDim) return QUP_ERR_ARG;
    if (!(T == 16 || T == 32 || T == 64 || T == 128)) return QUP_ERR_ARG;
    // supported (dtype, page size) pairs: bf16 16/32/64/128, E4M3 64/128, fp32 32/64
    if (num_logical_pages <= 0 || P_phys <= 0 || kv_len < 0) return QUP_ERR_ARG;
    if (!(std::isfinite(softmax_scale) && softmax_scale > 0.f)) return QUP_ERR_ARG;
    int es;
    if (q_dtype == QUP_F32 && kv_dtype == QUP_F32) es = 4;
    else if (q_dtype == QUP_BF16 && kv_dtype == QUP_BF16) es = 2;
    else if (q_dtype == QUP_BF16 && kv_dtype == QUP_E4M3) es = 1;
    else return QUP_ERR_ARG;
    if (es == 1 && (!k_scale || !v_scale)) return QUP_ERR_ARG;
    if ((es == 1 && T < 64) || (es == 4 && (T < 32 || T > 64))) return QUP_ERR_ARG;
    if (groups && (!bundle_fields_ok(groups) || groups->rows_per_group < 1)) return QUP_ERR_ARG;
    if (!groups && !work) return QUP_ERR_ARG;
    if ((int64_t)num_logical_pages * T >= ((int64_t)1 << 31)) return QUP_ERR_ARG;  // token positions are int32
    if (Nq == 0) return QUP_OK;
    if (!Q || !K_cache || !V_cache || !page_table || !O) return QUP_ERR_ARG;
    if (!q_end && !q_pos) return QUP_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(K_cache) | reinterpret_cast<uintptr_t>(V_cache)) & 15) return QUP_ERR_ARG;
    const Work wk = groups ? work_of(groups, Nq) : *work;
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(wk.row_mask)) & 15) return QUP_ERR_ARG;
    const int g = Hq / Hkv;
    if (128 % g != 0 || (groups && groups->rows_per_group % g != 0)) return QUP_ERR_ARG;
    const bool checked = g_checked.load() != 0 && topk != nullptr && groups != nullptr;
    if (checked && Ksel < 0) return QUP_ERR_ARG;
    DevState* ds = nullptr;
    int rc = device_state(&ds);
    if (rc) return rc;
    if (checked && qup::launch_check_support(topk, Ksel, Hkv, Nq, g, num_logical_pages, groups->n_bundles,
                                             groups->bunion_ptr, groups->bunion_pages, groups->bunion_mask,
                                             groups->bundle_qid, groups->cap_union, ds->err, ds->sms,
                                             static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return QUP_ERR_CUDA;

    // K / V cache tensor maps: dims (d, T, Hkv, P_phys), box (128 bytes of d, T, 1, 1), 128B swizzle
    CUtensorMap tm[2];
    const CUtensorMapDataType dt = es == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                           : (es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8);
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)Hkv, (cuuint64_t)P_phys};
    const cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)T * d * es, (cuuint64_t)Hkv * T * d * es};
    const cuuint32_t box[4] = {(cuuint32_t)(128 / es), (cuuint32_t)std::min(T, 64), 1, 1};  // one 64-token step
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const void* srcs[2] = {K_cache, V_cache};
    for (int i = 0; i < 2; ++i) {
        if (g_encode(&tm[i], dt, 4, const_cast<void*>(srcs[i]), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     // V is an MN-major operand; for tf32 its only layout uses 32-byte swizzle atoms
                     (es == 4 && i == 1) ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QUP_ERR_ARG;
    }
    // Q rows for the bf16 kernel's Q operand: dims (d, Hq, Nq), box (64 elements, g heads, 1 query),
    // 128-byte swizzle (the operand's K-major layout); a query coordinate of Nq reads zeros
    CUtensorMap tmq;
    std::memset(&tmq, 0, sizeof(tmq));
    if (es == 2) {
        const cuuint64_t qdims[3] = {(cuuint64_t)d, (cuuint64_t)Hq, (cuuint64_t)Nq};
        const cuuint64_t qstrides[2] = {(cuuint64_t)d * 2, (cuuint64_t)Hq * d * 2};
        const cuuint32_t qbox[3] = {64, (cuuint32_t)g, 1};
        const cuuint32_t qestr[3] = {1, 1, 1};
        if (g_encode(&tmq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(Q), qdims, qstrides, qbox, qestr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QUP_ERR_ARG;
    }
    // a pipeline step is 128 tokens: as many K and V tiles in flight as shared memory allows,
    // split between the K ring and the V ring (a V slot is held longer: through the softmax)
    int nt = 2 * qup::kMaxStages;
    while (nt >= 2 && qup::attn_smem_bytes(es, nt / 2, nt - nt / 2, Hkv, g) > (size_t)ds->smem_optin) --nt;
    if (nt < 2) return QUP_ERR_ARG;
    const int nsk = nt / 2, nsv = nt - nt / 2;
    const size_t smem = qup::attn_smem_bytes(es, nsk, nsv, Hkv, g);

    qup::AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.Q = Q;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.page_table = page_table;
    p.n_bundles = wk.n_bundles;
    p.union_ptr = wk.union_ptr;
    p.union_pages = wk.union_pages;
    p.row_mask = wk.row_mask;
    p.bundle_qid = wk.bundle_qid;
    p.bundle_order = wk.bundle_order;
    p.part_o = wk.part_o;
    p.part_lse = wk.part_lse;
    p.item_slot = wk.item_slot;
    p.q_pos = q_pos;
    p.q_end = q_end;
    p.page_len = page_len;
    p.O = O;
    p.lse = lse;
    p.err = ds->err;
    p.cap_union = wk.cap_union;
    p.num_logical_pages = num_logical_pages;
    p.P_phys = P_phys;
    p.T = T;
    p.kv_len = kv_len;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.g = g;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.bstride = wk.bstride;
    p.nsk = nsk;
    p.nsv = nsv;
    const int wait_ms = g_wait_limit_ms.load();
    p.wait_limit_ns = (unsigned long long)(wait_ms > 0 ? wait_ms : 2000) * 1000000ull;
    p.dbg_skip_stage = g_skip_stage.load();
    p.walk_slot = (int)(g_walk_slot.fetch_add(1u) % (unsigned)qup::kWalkSlots);
    const cudaError_t e =
        qup::launch_union_attn(es, T, tm[0], tm[1], tmq, p, ds->sms, smem, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QUP_OK : QUP_ERR_CUDA;
}

}  // namespace

extern "C" {

int qup_sparse_prefill_attn(const void* Q, int q_dtype, const void* K_cache, const void* V_cache, int kv_dtype,
                            const float* k_scale, const float* v_scale, const int32_t* page_table,
                            int num_logical_pages, int P_phys, int T, const int32_t* topk, int Ksel,
                            const qup_groups* groups, const int32_t* q_pos, int kv_len, int Hq, int Hkv, int Nq,
                            int d, float softmax_scale, void* O, float* lse, void* stream) {
    if (Nq > 0 && !q_pos) return QUP_ERR_ARG;
    return attn_impl(Q, q_dtype, K_cache, V_cache, kv_dtype, k_scale, v_scale, page_table, num_logical_pages,
                     P_phys, T, topk, Ksel, groups, nullptr, q_pos, kv_len, nullptr, nullptr, Hq, Hkv, Nq, d,
                     softmax_scale, O, lse, stream);
}

int qup_batch_prepare(const int32_t* topk, const int32_t* q_pos, int Hq, int Nq, int Ksel, int T, int R,
                      const int32_t* q_ptr, const int32_t* page_ptr, const int32_t* kv_len, int total_pages,
                      int32_t* topk_global, int32_t* q_end, int32_t* page_len, void* stream) {
    if (Hq <= 0 || Nq < 0 || Ksel < 0 || R < 0 || total_pages < 0) return QUP_ERR_ARG;
    if (!(T == 16 || T == 32 || T == 64 || T == 128)) return QUP_ERR_ARG;
    if ((int64_t)total_pages * T >= ((int64_t)1 << 31)) return QUP_ERR_ARG;
    if (Nq > 0 && (!q_pos || !q_end || !q_ptr || !page_ptr || !kv_len || R == 0 ||
                   (Ksel > 0 && (!topk || !topk_global))))
        return QUP_ERR_ARG;
    if (total_pages > 0 && (!page_len || !page_ptr || !kv_len || R == 0)) return QUP_ERR_ARG;
    DevState* ds = nullptr;
    int rc = device_state(&ds);
    if (rc) return rc;
    return qup::launch_batch_prepare(topk, q_pos, Hq, Nq, Ksel, T, R, q_ptr, page_ptr, kv_len, total_pages,
                                     topk_global, q_end, page_len, ds->err,
                                     static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QUP_OK
               : QUP_ERR_CUDA;
}

int qup_pivot_select(const void* q_idx, const void* page_key, int dtype, const int32_t* q_pos, int Nq, int Hkv,
                     int g, int d_idx, int num_logical_pages, int T, int group_size, int n_cand, int Ksel,
                     int refine, int32_t* topk, void* stream) {
    if (Nq < 0 || Hkv <= 0 || g <= 0 || g > 32 || T <= 0 || group_size <= 0) return QUP_ERR_ARG;
    if (dtype != QUP_BF16 && dtype != QUP_F32) return QUP_ERR_ARG;
    if (d_idx <= 0 || d_idx > qup::kMaxSelDim || d_idx % (dtype == QUP_BF16 ? 8 : 4) != 0) return QUP_ERR_ARG;
    if (num_logical_pages <= 0 || num_logical_pages > qup::kMaxSelPages) return QUP_ERR_ARG;
    if (n_cand <= 0 || n_cand > qup::kMaxSelCand || Ksel <= 0 || Ksel > n_cand) return QUP_ERR_ARG;
    if (refine != 0 && refine != 1) return QUP_ERR_ARG;
    if (Nq > 0 && (!q_idx || !page_key || !q_pos || !topk)) return QUP_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(q_idx) & 15) || (reinterpret_cast<uintptr_t>(page_key) & 15)) return QUP_ERR_ARG;
    DevState* ds = nullptr;
    int rc = device_state(&ds);
    if (rc) return rc;
    if (qup::pivot_select_smem(num_logical_pages, d_idx, dtype == QUP_BF16 ? 2 : 4, n_cand) > (size_t)ds->smem_optin)
        return QUP_ERR_ARG;
    return qup::launch_pivot_select(q_idx, page_key, dtype == QUP_BF16, q_pos, Nq, Hkv, g, d_idx, num_logical_pages,
                                    T, group_size, n_cand, Ksel, refine == 1, topk,
                                    static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QUP_OK
               : QUP_ERR_CUDA;
}

int qup_sparse_prefill_attn_batch(const void* Q, int q_dtype, const void* K_cache, const void* V_cache,
                                  int kv_dtype, const float* k_scale, const float* v_scale,
                                  const int32_t* page_table, int total_pages, int P_phys, int T,
                                  const int32_t* topk_global, int Ksel, const qup_groups* groups,
                                  const int32_t* q_end, const int32_t* page_len, int Hq, int Hkv, int Nq, int d,
                                  float softmax_scale, void* O, float* lse, void* stream) {
    if (Nq > 0 && (!q_end || !page_len)) return QUP_ERR_ARG;
    return attn_impl(Q, q_dtype, K_cache, V_cache, kv_dtype, k_scale, v_scale, page_table, total_pages, P_phys, T,
                     topk_global, Ksel, groups, nullptr, nullptr, 0, q_end, page_len, Hq, Hkv, Nq, d, softmax_scale, O,
                     lse, stream);
}

int qup_page_major_workspace(int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages, int T, size_t* ws_bytes,
                              int64_t* item_cap, int64_t* slot_cap, int32_t* tile_pages) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Nq < 0 || Ksel < 0 || num_logical_pages <= 0) return QUP_ERR_ARG;
    if (!(T == 16 || T == 32 || T == 64 || T == 128)) return QUP_ERR_ARG;
    const int g = Hq / Hkv;
    if (g > 32 || 128 % g != 0) return QUP_ERR_ARG;
    const int NW = (num_logical_pages + 31) / 32;
    if (qup::page_major_build_smem(g, NW) > 227u * 1024u) return QUP_ERR_ARG;
    const int Pt = 256 / T, ntiles = (num_logical_pages + Pt - 1) / Pt, MQ = 128 / g;
    // items of one KV head: sum over tiles of ceil(queries meeting the tile / MQ)
    const int64_t touch = (int64_t)Nq * std::min<int64_t>(ntiles, (int64_t)g * Ksel);
    const int64_t icap = std::max<int64_t>((touch + MQ - 1) / MQ + ntiles, 1);
    const int64_t scap = std::max<int64_t>((int64_t)Hq * Nq * std::min<int64_t>(ntiles, Ksel), 1);
    if (icap * Hkv * Pt >= ((int64_t)1 << 31) || scap >= ((int64_t)1 << 31)) return QUP_ERR_ARG;
    size_t off = 0;
    off = align256(off + sizeof(int32_t) * (size_t)Hkv * ntiles);      // tile counts
    off = align256(off + sizeof(int32_t) * (size_t)Hkv * ntiles);      // tile fill cursors
    off = align256(off + sizeof(int32_t) * (size_t)Hq * Nq);           // row tile counts
    off = align256(off + sizeof(int64_t) * (size_t)Hkv * ntiles);      // tile item bases
    off = align256(off + sizeof(int64_t) * (size_t)(2 + Hkv));         // totals
    if (ws_bytes) *ws_bytes = off;
    if (item_cap) *item_cap = icap;
    if (slot_cap) *slot_cap = scap;
    if (tile_pages) *tile_pages = Pt;
    return QUP_OK;
}

int qup_page_major_items(const int32_t* topk, int Hq, int Hkv, int Nq, int Ksel, int num_logical_pages, int T,
                         qup_page_items* out, void* ws, size_t ws_bytes, void* stream) {
    size_t need = 0;
    int64_t icap = 0, scap = 0;
    int32_t Pt = 0;
    int rc = qup_page_major_workspace(Hq, Hkv, Nq, Ksel, num_logical_pages, T, &need, &icap, &scap, &Pt);
    if (rc) return rc;
    if (!out || !out->n_items || !out->item_ptr || !out->item_pages || !out->item_mask || !out->item_qid ||
        !out->item_slot || !out->item_order || !out->row_off)
        return QUP_ERR_ARG;
    if ((Nq > 0 && Ksel > 0 && !topk) || !ws) return QUP_ERR_ARG;
    if (ws_bytes < need || out->item_cap < icap || out->slot_cap < scap) return QUP_ERR_CAPACITY;
    DevState* ds = nullptr;
    if ((rc = device_state(&ds))) return rc;
    out->tile_pages = Pt;
    if (Nq == 0) return QUP_OK;
    const int g = Hq / Hkv, NW = (num_logical_pages + 31) / 32, ntiles = (num_logical_pages + Pt - 1) / Pt;
    char* base = static_cast<char*>(ws);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char* q = base + off;
        off = align256(off + bytes);
        return q;
    };
    int32_t* tile_cnt = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)Hkv * ntiles));
    int32_t* tile_fill = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)Hkv * ntiles));
    int32_t* row_cnt = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)Hq * Nq));
    int64_t* tile_base = reinterpret_cast<int64_t*>(take(sizeof(int64_t) * (size_t)Hkv * ntiles));
    int64_t* totals = reinterpret_cast<int64_t*>(take(sizeof(int64_t) * (size_t)(2 + Hkv)));
    if (Ksel == 0) {
        if (cudaMemsetAsync(out->n_items, 0, sizeof(int32_t) * Hkv, static_cast<cudaStream_t>(stream)) != cudaSuccess ||
            cudaMemsetAsync(out->row_off, 0, sizeof(int64_t) * ((size_t)Hq * Nq + 1),
                            static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return QUP_ERR_CUDA;
        return QUP_OK;
    }
    return qup::launch_page_major_build(topk, Hq, Hkv, Nq, Ksel, num_logical_pages, NW, Pt, ntiles, 128 / g,
                                        out->item_cap, out->slot_cap, tile_cnt, tile_fill, row_cnt, tile_base,
                                        out->row_off, totals, out->n_items, out->item_ptr, out->item_pages,
                                        out->item_mask, out->item_qid, out->item_slot, out->item_order, ds->err,
                                        static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QUP_OK
               : QUP_ERR_CUDA;
}

int qup_page_major_attn(const void* Q, int q_dtype, const void* K_cache, const void* V_cache, int kv_dtype,
                        const float* k_scale, const float* v_scale, const int32_t* page_table, int num_logical_pages,
                        int P_phys, int T, const qup_page_items* items, const int32_t* q_pos, int kv_len, int Hq,
                        int Hkv, int Nq, int d, float softmax_scale, float* part_o, float* part_lse, void* O,
                        float* lse, void* stream) {
    if (!items || !items->n_items || !items->item_ptr || !items->item_pages || !items->item_mask ||
        !items->item_qid || !items->item_slot || !items->item_order || !items->row_off || items->item_cap < 1 ||
        items->tile_pages != 256 / T)
        return QUP_ERR_ARG;
    if (Nq > 0 && (!q_pos || !part_o || !part_lse || !O)) return QUP_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(part_o) & 15) return QUP_ERR_ARG;
    Work wk;
    wk.n_bundles = items->n_items;
    wk.union_ptr = items->item_ptr;
    wk.union_pages = items->item_pages;
    wk.row_mask = items->item_mask;
    wk.bundle_qid = items->item_qid;
    wk.bundle_order = items->item_order;
    wk.cap_union = items->item_cap * Hkv * items->tile_pages;
    wk.bstride = (int)items->item_cap;
    wk.part_o = part_o;
    wk.part_lse = part_lse;
    wk.item_slot = items->item_slot;
    int rc = attn_impl(Q, q_dtype, K_cache, V_cache, kv_dtype, k_scale, v_scale, page_table, num_logical_pages, P_phys,
                       T, nullptr, 0, nullptr, &wk, q_pos, kv_len, nullptr, nullptr, Hq, Hkv, Nq, d, softmax_scale, O,
                       lse, stream);
    if (rc || Nq == 0) return rc;
    return qup::launch_page_major_merge(part_o, part_lse, items->row_off, Hq, Nq, q_dtype == QUP_BF16 ? 1 : 0, O, lse,
                                        static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QUP_OK
               : QUP_ERR_CUDA;
}

int qup_get_error(int* code, void* stream) {
    if (!code) return QUP_ERR_ARG;
    DevState* ds = nullptr;
    int rc = device_state(&ds);
    if (rc) return rc;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QUP_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err_word, sizeof(v)) != cudaSuccess) return QUP_ERR_CUDA;
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero)) != cudaSuccess) return QUP_ERR_CUDA;
    *code = (int)v;
    return QUP_OK;
}

const char* qup_error_string(int code) {
    switch (code) {
        case QUP_OK: return "ok";
        case QUP_ERR_ARG: return "invalid argument";
        case QUP_ERR_CAPACITY: return "workspace or union capacity too small";
        case QUP_ERR_CUDA: return "CUDA runtime or launch failure";
        case QUP_ERR_PAGE_ID: return "page ID out of range";
        case QUP_ERR_PHYS_PAGE: return "page_table entry out of range";
        case QUP_ERR_GROUP: return "malformed group";
        case QUP_ERR_TIMEOUT: return "pipeline wait timed out";
        default: return "multiple errors (bitwise OR of codes)";
    }
}

int qup_set_debug(int wait_limit_ms, int skip_stage) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_wait_limit_ms = wait_limit_ms > 0 ? wait_limit_ms : 0;
    g_skip_stage = skip_stage >= 0 ? skip_stage : -1;
    return QUP_OK;
}

int qup_set_checked(int on) {
    g_checked = on ? 1 : 0;
    return QUP_OK;
}

int qup_num_sms(void) {
    DevState* ds = nullptr;
    return device_state(&ds) == QUP_OK ? ds->sms : 0;
}

int qup_exp2_poly(const float* x, float* y, int n, void* stream) {
    if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return QUP_ERR_ARG;
    return qup::launch_exp2_poly(x, y, n, (cudaStream_t)stream) == cudaSuccess ? QUP_OK : QUP_ERR_CUDA;
}

}  // extern "C"

namespace qup {

unsigned long long context_id() {
    typedef CUresult (*GetCurrentFn)(CUcontext*);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(f);
    });
    if (!get_current || !get_id) return 0;
    CUcontext c = nullptr;
    if (get_current(&c) != CUDA_SUCCESS) return 0;
    if (c == nullptr) {  // no context on this thread yet: cudaSetDevice makes the primary one current
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return 0;
        if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
    }
    unsigned long long id = 0;
    if (get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id + 1;  // never 0
}

cudaError_t ensure_smem_attr(const void* fn, size_t smem) {
    struct Entry {
        unsigned long long ctx;
        const void* fn;
        size_t smem;
    };
    static std::mutex mu;
    static Entry table[256];
    static int n = 0;
    const unsigned long long ctx = context_id();
    if (ctx == 0) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < n; ++i)
        if (table[i].ctx == ctx && table[i].fn == fn) {
            if (table[i].smem >= smem) return cudaSuccess;
            const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e == cudaSuccess) table[i].smem = smem;
            return e;
        }
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) {
        if (n < 256) table[n++] = Entry{ctx, fn, smem};
        else table[(size_t)(ctx + (uintptr_t)fn) % 256] = Entry{ctx, fn, smem};  // full: overwrite one
    }
    return e;
}

}  // namespace qup
