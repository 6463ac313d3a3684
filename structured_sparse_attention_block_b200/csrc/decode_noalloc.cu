// Decode that allocates nothing: cowa_decode with its split-KV scratch held
// in a fixed device array inside the library instead of a caller workspace.
//
// Some callers cannot allocate device memory at all: a plugin running inside
// another runtime that owns every byte of device memory and hands the plugin
// only its input and output buffers, or a latency-critical serving loop in
// which cudaMalloc (which may synchronise the whole device) is not allowed.
// They still pass q, the caches, seqlens, o and lse; the partial outputs of
// the KV splits go to the static array below.
#include <cuda.h>
#include <stdio.h>

#include <mutex>

#include "../../include/cowa.h"
#include "kernels.cuh"

namespace cowa {
int set_error_detail(int status, const char *detail);
}

namespace {

// Scratch of the split-KV partials.  Every GPU that loads the library holds
// this much device memory until the process exits.
constexpr size_t kScratchBytes = COWA_DECODE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// In host code g_decode_scratch names a host-side stand-in, not the device
// array, so the kernels get the device address that cudaGetSymbolAddress
// reports.  That address belongs to the CUDA context the library's module is
// loaded in, so it is looked up once per context, with the context current,
// and cached under the context's ID: the primary context of each device, a
// driver-API context that a host runtime makes current instead, or the new
// primary context after a device reset (context IDs are never reused within
// a process, so a stale address is never handed out).
std::mutex g_scratch_mu;
struct ScratchEntry {
    unsigned long long ctx_id;
    void *addr;
};
ScratchEntry g_scratch_addr[64];
int g_scratch_used = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// ID of the current context (0 when the driver entry points are unavailable,
// in which case the address is looked up on every call).
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *a = nullptr, *b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<CtxGetCurrentFn>(a);
            get_id = reinterpret_cast<CtxGetIdFn>(b);
        }
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

int scratch_address(void **out)
{
    unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    for (int i = 0; id && i < g_scratch_used; ++i)
        if (g_scratch_addr[i].ctx_id == id) {
            *out = g_scratch_addr[i].addr;
            return COWA_OK;
        }
    // (with no context current yet, the runtime makes the device's primary
    // context current here; its ID is read again below)
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "cudaGetSymbolAddress(decode scratch): %s", cudaGetErrorString(e));
        return cowa::set_error_detail(COWA_ERR_CUDA, msg);
    }
    if (!id) id = current_context_id();
    if (id) {
        // a full table (64 contexts seen) recycles its oldest slot
        g_scratch_addr[g_scratch_used < 64 ? g_scratch_used++ : (int)(id % 64)] = {id, ptr};
    }
    *out = ptr;
    return COWA_OK;
}

}  // namespace

extern "C" int cowa_decode_noalloc(const cowa_shape_t *shape, cowa_quad_t quad, float softmax_scale,
                                   const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *seqlens, void *o, float *lse, void *stream)
{
    // The partials need B * Hq * splits * (d + 1) floats; refuse shapes whose
    // partials do not fit the static array.  A size of 0 means the shape or
    // quadruple is invalid: cowa_decode below reports exactly why.
    const size_t need = cowa_decode_workspace_size(shape, quad);
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "cowa_decode_noalloc: this shape needs %zu bytes of split scratch, above the %zu-byte "
                 "static limit; use cowa_decode with a workspace",
                 need, kScratchBytes);
        return cowa::set_error_detail(COWA_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    if (need > 0) {
        const int r = scratch_address(&scratch);
        if (r != COWA_OK) return r;
    }
    // Same validation, kernels and launches as cowa_decode; only the scratch
    // differs.  The split kernel writes every partial it owns before the merge
    // reads it, so stale contents from an earlier call are never used.
    return cowa_decode(shape, quad, softmax_scale, q, k_cache, v_cache, seqlens, o, lse, scratch,
                       kScratchBytes, stream);
}
