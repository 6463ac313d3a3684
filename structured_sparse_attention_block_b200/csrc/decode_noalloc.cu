// Decode that allocates nothing: cowa_decode with its split-KV scratch held
// in a fixed device array inside the library instead of a caller workspace.
//
// Some callers cannot allocate device memory at all: a plugin running inside
// another runtime that owns every byte of device memory and hands the plugin
// only its input and output buffers, or a latency-critical serving loop in
// which cudaMalloc (which may synchronise the whole device) is not allowed.
// They still pass q, the caches, seqlens, o and lse; the partial outputs of
// the KV splits go to the static array below.
#include <mutex>
#include <stdio.h>

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
// reports, looked up once per device with that device current.
std::mutex g_scratch_mu;
void *g_scratch_addr[64] = {};

int scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cowa::set_error_detail(COWA_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return cowa::set_error_detail(COWA_ERR_UNSUPPORTED, "device index above 63");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
        if (e != cudaSuccess) {
            char msg[256];
            snprintf(msg, sizeof msg, "cudaGetSymbolAddress(decode scratch): %s", cudaGetErrorString(e));
            return cowa::set_error_detail(COWA_ERR_CUDA, msg);
        }
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
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
