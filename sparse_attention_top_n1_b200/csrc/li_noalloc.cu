// li_noalloc.cu -- li_indexer without a caller-provided workspace.
//
// For callers that cannot give the library device memory (an operator
// interface with no workspace mechanism, or a serving loop that keeps
// cudaMalloc off its hot path), the workspace of an indexer call lives in a
// scratch array compiled into the library.  Every GPU that loads the library
// holds LI_NOALLOC_SCRATCH_BYTES of device memory for it until the process
// exits.  This file allocates nothing: it finds the array's device address
// (once per device and context) and hands it to li_indexer as the workspace.
#include <cstdio>
#include <mutex>

#include "li_internal.cuh"

namespace li {
li_status report_error(li_status s, const char *msg);
}

namespace {

// The scratch memory.  In host code this name is only a stand-in for the
// device symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LI_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
struct ScratchAddr {
    void *ptr;
    uint64_t ctx;    // id of the context the address belongs to (0: none cached)
};
ScratchAddr g_scratch[kMaxDevices] = {};

// The current device's address of the scratch array.  It is looked up with
// cudaGetSymbolAddress on the first call in each context of the device (the
// first call, which should precede any stream capture, and again after a
// cudaDeviceReset re-created the context, since the old address died with
// the old context); later calls in the same context reuse it.
li_status scratch_for_current_device(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return li::report_error(LI_ERR_CUDA, "li_indexer_noalloc: no CUDA device");
    if (dev < 0 || dev >= kMaxDevices)
        return li::report_error(LI_ERR_CUDA, "li_indexer_noalloc: device ordinal out of range");
    const uint64_t ctx = li::current_context_id();
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (ctx == 0 || g_scratch[dev].ctx != ctx || !g_scratch[dev].ptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            char msg[160];
            snprintf(msg, sizeof msg, "li_indexer_noalloc: cannot locate the scratch array (%s)",
                     cudaGetErrorString(e));
            return li::report_error(LI_ERR_CUDA, msg);
        }
        g_scratch[dev].ptr = p;
        g_scratch[dev].ctx = li::current_context_id();   // current now, if it was not before
    }
    *out = g_scratch[dev].ptr;
    return LI_OK;
}

}  // namespace

extern "C" {

li_status li_indexer_noalloc(const li_params *p, const void *query, const void *key,
                             const void *weights, const int32_t *act_seq_q,
                             const int32_t *act_seq_k, const int32_t *block_table,
                             int32_t *sparse_indices, float *sparse_values, void *stream)
{
    size_t need = 0;
    li_status st = li_workspace_size(p, &need);       // validates the parameters too
    if (st != LI_OK) return st;
    if (need > LI_NOALLOC_SCRATCH_BYTES) {
        char msg[200];
        snprintf(msg, sizeof msg,
                 "li_indexer_noalloc: this problem needs %zu bytes of scratch, more than the "
                 "%u bytes the library holds; call li_indexer with a workspace",
                 need, (unsigned)LI_NOALLOC_SCRATCH_BYTES);
        return li::report_error(LI_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    st = scratch_for_current_device(&scratch);
    if (st != LI_OK) return st;
    return li_indexer(p, query, key, weights, act_seq_q, act_seq_k, block_table, sparse_indices,
                      sparse_values, scratch, LI_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
