// decode_noalloc.cu -- blasst_decode_noalloc: the split-KV decode with its
// split partials kept in a fixed, library-owned device array instead of
// caller or stream-ordered allocations.
//
// Who needs it: callers that must not allocate device memory while serving,
// e.g. an inference engine that reserves (nearly) all device memory for its
// own pool up front, where any extra cudaMalloc/cudaMallocAsync either fails
// or fragments that pool, or a latency-critical loop where an allocation or
// free could stall the device.  Those callers pass their inputs and outputs
// and nothing else.
//
// Cost: every GPU that loads this library holds kNoAllocScratchBytes of
// device memory for this array until the process exits.
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/blasst.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = BLASST_NOALLOC_SCRATCH_BYTES;

// The scratch array.  In host code this name is only a host-side stand-in:
// its device address must be fetched with cudaGetSymbolAddress on each device.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device; resolved once
// per device (the first call on a device loads the module there).
blasst_status scratch_for_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        char msg[160];
        std::snprintf(msg, sizeof msg, "cudaGetDevice: %s",
                      e == cudaSuccess ? "device index out of range" : cudaGetErrorString(e));
        blasst::set_last_error(msg);
        return BLASST_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || !p) {
            char msg[160];
            std::snprintf(msg, sizeof msg, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
            blasst::set_last_error(msg);
            return BLASST_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return BLASST_OK;
}

}  // namespace

extern "C" {

BLASST_API blasst_status blasst_decode_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                               int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                                               float lambda, int causal, uint32_t *skip_mask,
                                               unsigned long long *skip_count, void *stream,
                                               const blasst_opts *opts) {
    blasst_opts op;
    std::memset(&op, 0, sizeof op);
    if (opts) std::memcpy(&op, opts, opts->struct_size < sizeof op ? opts->struct_size : sizeof op);
    op.struct_size = sizeof op;
    if (op.workspace) return BLASST_ERR_INVALID;  // the scratch is the library's, not the caller's
    const int splits = op.num_splits ? op.num_splits : 16;
    if (B <= 0 || Hq <= 0 || Lq <= 0 || splits <= 0) return BLASST_ERR_INVALID;
    const size_t need = blasst_decode_workspace_bytes(B, Hq, Lq, op.dv, splits);
    if (need == 0 || need > kNoAllocScratchBytes) {
        char msg[160];
        std::snprintf(msg, sizeof msg, "decode partials need %zu bytes; the fixed scratch holds %zu", need,
                      kNoAllocScratchBytes);
        blasst::set_last_error(msg);
        return BLASST_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    blasst_status st = scratch_for_current_device(&scratch);
    if (st != BLASST_OK) return st;
    // every byte the kernels read from the scratch is written earlier in the
    // same call (each split writes all its partial rows), so nothing is cleared
    op.workspace = scratch;
    op.workspace_bytes = kNoAllocScratchBytes;
    return blasst_decode(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask, skip_count,
                         stream, &op);
}

}  // extern "C"
