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
// One resolved address per (device, context).  A context made current through the
// driver API is a different context from the runtime's primary one, and the array
// has a different address in each.
struct ScratchAddr {
    int dev;
    CUcontext ctx;
    void *addr;
};
ScratchAddr g_scratch_addr[kMaxDevices];
int g_n_scratch_addr = 0;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    }
    return fn;
}

blasst_status fail(const char *what, cudaError_t e) {
    char msg[160];
    std::snprintf(msg, sizeof msg, "%s: %s", what, cudaGetErrorString(e));
    blasst::set_last_error(msg);
    return BLASST_ERR_CUDA;
}

// Device address of the scratch array for the current device and context.  The
// first call there resolves it (cudaGetSymbolAddress, which loads this module on
// the device); later calls reuse the cached address.
blasst_status scratch_for_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail("cudaGetDevice", e);
    CUcontext ctx = nullptr;
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (get_ctx) get_ctx(&ctx);  // null before the runtime has made a context current
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_n_scratch_addr; i++) {
        if (g_scratch_addr[i].dev == dev && g_scratch_addr[i].ctx == ctx && ctx) {
            *out = g_scratch_addr[i].addr;
            return BLASST_OK;
        }
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) return fail("cudaGetSymbolAddress(scratch)", e);
    if (!ctx && get_ctx) get_ctx(&ctx);  // the lookup above made the primary context current
    if (ctx && g_n_scratch_addr < kMaxDevices) g_scratch_addr[g_n_scratch_addr++] = ScratchAddr{dev, ctx, p};
    *out = p;
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
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Lk <= 0 || d <= 0) return BLASST_ERR_INVALID;
    // the split count and value width exactly as blasst_decode will resolve them
    // (MLA defaults to 2 splits, GQA/MQA to 16, -1 to the adaptive count)
    int splits = 0;
    const long long rows = (Hkv > 0 && Hq % Hkv == 0) ? (long long)(Hq / Hkv) * Lq : 0;
    if (rows <= 0 || rows > 0x7fffffffLL) return BLASST_ERR_INVALID;
    blasst_status st = blasst::decode_split_count(d, op.num_splits, B, Hkv, (int)rows, Lk, &splits);
    if (st != BLASST_OK) return st;
    op.num_splits = splits;
    const int dv = op.dv ? op.dv : d;
    const size_t need = blasst_decode_workspace_bytes(B, Hq, Lq, dv, splits);
    if (need == 0 || need > kNoAllocScratchBytes) {
        char msg[160];
        std::snprintf(msg, sizeof msg, "decode partials need %zu bytes; the fixed scratch holds %zu", need,
                      kNoAllocScratchBytes);
        blasst::set_last_error(msg);
        return BLASST_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    st = scratch_for_current_device(&scratch);
    if (st != BLASST_OK) return st;
    // every byte the kernels read from the scratch is written earlier in the
    // same call (each split writes all its partial rows), so nothing is cleared
    op.workspace = scratch;
    op.workspace_bytes = kNoAllocScratchBytes;
    return blasst_decode(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask, skip_count,
                         stream, &op);
}

}  // extern "C"
