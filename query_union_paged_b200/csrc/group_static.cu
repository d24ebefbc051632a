// group_static.cu -- qup_sparse_group_static: the grouping call with its scratch
// workspace in a fixed device array of this library instead of a caller buffer.
//
// Who needs it: a caller that holds no device allocator at the point of the
// call (a plain C host program that owns only its input and output buffers),
// or one whose device memory is fixed once at start-up and that may not
// allocate per call (a serving loop that forbids allocation after warm-up).
// Such a caller cannot provide the `ws` buffer qup_sparse_group asks for;
// this entry point takes that scratch from g_group_scratch below and
// otherwise runs the same kernels, so its outputs equal qup_sparse_group's.
//
// Nothing here calls cudaMalloc, cudaFree or any routine that allocates.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "query_union_paged.h"

namespace {

// Scratch of every qup_sparse_group_static call on a device.  No byte has to
// start at zero: each grouping kernel writes its part of the workspace
// before any kernel reads it.
__device__ __align__(256) unsigned char g_group_scratch[QUP_STATIC_GROUP_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchAddr {
    unsigned long long ctx;  // context the address was looked up in (0: not yet)
    void* ptr;               // device address of g_group_scratch in that context
};
ScratchAddr g_scratch[kMaxDevices];

// Looks the symbol up once per device context, with that device current: a device reset or a
// non-primary context gets a new context ID and a fresh lookup, so a stale address is never used.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QUP_ERR_CUDA;
    const unsigned long long ctx = qup::context_id();
    if (ctx == 0) return QUP_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    ScratchAddr& a = g_scratch[dev];
    if (a.ctx != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_group_scratch) != cudaSuccess || p == nullptr) return QUP_ERR_CUDA;
        a.ptr = p;
        a.ctx = ctx;
    }
    *out = a.ptr;
    return QUP_OK;
}

}  // namespace

extern "C" int qup_sparse_group_static(const int32_t* topk, int Hq, int Hkv, int Nq, int Ksel,
                                       int num_logical_pages, int max_group, int window, qup_groups* out,
                                       void* stream) {
    size_t need = 0;
    int64_t cap = 0;
    int rc = qup_group_workspace(Hq, Hkv, Nq, Ksel, num_logical_pages, max_group, window, &need, &cap);
    if (rc) return rc;
    if (need > (size_t)QUP_STATIC_GROUP_SCRATCH_BYTES) return QUP_ERR_CAPACITY;
    void* ws = nullptr;
    if ((rc = scratch_address(&ws))) return rc;
    return qup_sparse_group(topk, Hq, Hkv, Nq, Ksel, num_logical_pages, max_group, window, out, ws,
                            (size_t)QUP_STATIC_GROUP_SCRATCH_BYTES, stream);
}
