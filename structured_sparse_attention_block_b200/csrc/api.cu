// C ABI of the CoWA library: argument checks, workspace carving and kernel
// launches.  Declarations and contracts are in include/cowa.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "../../include/cowa.h"
#include "common.cuh"
#include "kernels.cuh"

#include <atomic>
#include <mutex>
#include <vector>

namespace cowa {
__device__ int g_cowa_device_error = 0;

// The timeout self-test kernel's launcher (selftest.cu).
cudaError_t launch_wait_selftest(int *err, cudaStream_t st);

// Records a status and its detail for cowa_last_error_detail() from code
// outside this file.
int set_error_detail(int status, const char *detail);

static std::atomic<unsigned long long> g_launches{0};

// Kernel trace: while on, every launch records an event pair on its stream.
// The events are created up front by cowa_trace_start so that recording
// costs two cudaEventRecord calls per launch and no allocation.
struct TraceRec {
    const char *name;
    cudaEvent_t a, b;
};
static std::mutex g_trace_mu;
static std::atomic<int> g_trace_on{0};
static int g_trace_dev = -1;
static std::vector<TraceRec> g_trace;  // capacity entries, events created
static char g_trace_only[64] = "";     // trace only this kernel ("" = all)
static size_t g_trace_used = 0;
static size_t g_trace_dropped = 0;
static thread_local long long tl_open = -1;  // record opened by launch_begin

void launch_begin(const char *name, cudaStream_t st)
{
    g_launches.fetch_add(1, std::memory_order_relaxed);
    tl_open = -1;
    if (!g_trace_on.load(std::memory_order_acquire)) return;
    if (g_trace_only[0] && strcmp(name, g_trace_only) != 0) return;
    int dev = -1;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (!g_trace_on.load(std::memory_order_relaxed) || dev != g_trace_dev ||
        g_trace_used == g_trace.size()) {
        ++g_trace_dropped;
        return;
    }
    TraceRec &r = g_trace[g_trace_used];
    r.name = name;
    if (cudaEventRecord(r.a, st) != cudaSuccess) {
        ++g_trace_dropped;
        return;
    }
    tl_open = (long long)g_trace_used++;
}

void launch_end(cudaStream_t st)
{
    if (tl_open < 0) return;
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if ((size_t)tl_open < g_trace_used && cudaEventRecord(g_trace[tl_open].b, st) != cudaSuccess)
        g_trace[tl_open].name = nullptr;  // unusable record
    tl_open = -1;
}

void trace_clear_locked()
{
    for (TraceRec &r : g_trace) {
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    g_trace.clear();
    g_trace_used = g_trace_dropped = 0;
    g_trace_dev = -1;
}
}

namespace {

thread_local char tl_detail[256] = "";

int fail(int status, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(tl_detail, sizeof tl_detail, fmt, ap);
    va_end(ap);
    return status;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(COWA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

struct DeviceInfo {
    int checked = 0, ok = 0, sms = 148;
    int *err = nullptr;  // device address of the error word on this device
};
DeviceInfo g_dev[64];

int check_device(int *sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    DeviceInfo &di = g_dev[dev & 63];
    if (!di.checked) {
        int major = 0, minor = 0, sm = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&sm, cudaDevAttrMultiProcessorCount, dev);
        di.ok = (major == 10 && minor == 0);
        di.sms = sm > 0 ? sm : 148;
        if (di.ok) {
            e = cudaGetSymbolAddress((void **)&di.err, cowa::g_cowa_device_error);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
        }
        di.checked = 1;
    }
    if (!di.ok) return fail(COWA_ERR_UNSUPPORTED, "device %d is not sm_100 (B200)", dev);
    if (sms) *sms = di.sms;
    return COWA_OK;
}

int *device_error_word()
{
    int dev = 0;
    cudaGetDevice(&dev);
    return g_dev[dev & 63].err;
}

constexpr long long kMaxLen = 1ll << 30;

long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int check_quad(cowa_quad_t q)
{
    if (q.S < 0 || q.N < 0 || q.G < 0 || q.W < 0)
        return fail(COWA_ERR_INVALID_ARG, "window quadruple (%d,%d,%d,%d) has a negative field",
                    q.S, q.N, q.G, q.W);
    return COWA_OK;
}

int check_strides(const int64_t *st, const char *name)
{
    for (int a = 0; a < 3; ++a)
        if (st[a] < 0 || st[a] % 8)
            return fail(COWA_ERR_ALIGNMENT, "%s stride[%d] = %lld is not a non-negative multiple of 8 elements",
                        name, a, (long long)st[a]);
    return COWA_OK;
}

int check_ptr(const void *p, bool needed, const char *name)
{
    if (!needed) return COWA_OK;
    if (!p) return fail(COWA_ERR_INVALID_ARG, "%s is NULL", name);
    if ((uintptr_t)p % 16) return fail(COWA_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);
    return COWA_OK;
}

int check_shape(const cowa_shape_t *s, cowa_quad_t q, bool decode)
{
    if (!s) return fail(COWA_ERR_INVALID_ARG, "shape is NULL");
    if (s->B < 0 || s->Lq < 0 || s->Lk < 0 || s->Hq < 0 || s->Hkv < 0 || s->kv_head_offset < 0)
        return fail(COWA_ERR_INVALID_ARG, "negative size in shape");
    if (s->Lq >= kMaxLen || s->Lk >= kMaxLen || s->B > 65535 || s->Hq > 65535 || s->Hkv > 65535)
        return fail(COWA_ERR_UNSUPPORTED, "sequence length must be < 2^30, B/heads <= 65535");
    // the tiled kernels use 1-D grids of (tile, head, batch) blocks; no
    // problem that fits in device memory comes near this bound
    if (!decode && (s->B * s->Hq * cdiv(s->Lq, 32) > 0x7fffffffll ||
                    s->B * s->Hkv * cdiv(s->Lk, 32) > 0x7fffffffll))
        return fail(COWA_ERR_UNSUPPORTED, "B * heads * length / 32 exceeds 2^31 - 1");
    if (s->Hq > 0 && (s->Hkv == 0 || s->Hq % s->Hkv))
        return fail(COWA_ERR_INVALID_ARG, "Hq=%lld is not a multiple of Hkv=%lld", (long long)s->Hq,
                    (long long)s->Hkv);
    if (s->d != 64 && s->d != 128)
        return fail(COWA_ERR_UNSUPPORTED, "head dim %lld (supported: 64, 128)", (long long)s->d);
    if (s->kv_head_offset + s->Hkv > kMaxLen)
        return fail(COWA_ERR_INVALID_ARG, "kv_head_offset too large");
    int r = check_quad(q);
    if (r) return r;
    if ((r = check_strides(s->q_stride, "q")) || (r = check_strides(s->k_stride, "k")) ||
        (r = check_strides(s->v_stride, "v")) || (r = check_strides(s->o_stride, "o")))
        return r;
    if (decode) {
        if (s->Lq != 1) return fail(COWA_ERR_INVALID_ARG, "decode needs Lq == 1 (got %lld)", (long long)s->Lq);
        if (s->Hkv > 0 && s->Hq / s->Hkv > 16)
            return fail(COWA_ERR_UNSUPPORTED, "decode supports up to 16 query heads per KV head");
    }
    return COWA_OK;
}

float resolve_scale(float scale, int64_t d) { return scale > 0.f ? scale : 1.0f / sqrtf((float)d); }

template <typename P>
void fill_common(P &p, const cowa_shape_t *s, cowa_quad_t q, float scale)
{
    for (int a = 0; a < 3; ++a) {
        p.qs[a] = s->q_stride[a];
        p.ks[a] = s->k_stride[a];
        p.vs[a] = s->v_stride[a];
        p.os[a] = s->o_stride[a];
    }
    p.Hq = (int)s->Hq;
    p.Hkv = (int)s->Hkv;
    p.g = s->Hkv > 0 ? (int)(s->Hq / s->Hkv) : 1;
    p.S = q.S; p.N = q.N; p.G = q.G; p.W = q.W;
    p.kv_head_offset = (int)s->kv_head_offset;
    p.scale = resolve_scale(scale, s->d);
    p.scale_log2 = p.scale * 1.4426950408889634f;
    p.err = device_error_word();
}

size_t sched_bytes(long long heads, long long tiles) { return align256((size_t)(heads * tiles) * 8 * sizeof(int)); }


// Splits of each (batch, KV head) key range.  The split kernel is memory
// bound and its CTAs all do about the same work, so the time is set by the
// number of full waves of resident CTAs: pick the smallest split count whose
// waves-per-unit-of-work is within 3 % of the best, over 1 .. 64 splits and
// at least four key tiles per split.
int decode_splits(const cowa_shape_t *s, cowa_quad_t q, int sms)
{
    const long long pairs = s->B * s->Hkv;
    if (pairs <= 0) return 1;
    long long keys = (long long)q.S + q.N + q.W;
    if (keys > s->Lk) keys = s->Lk;
    const long long tiles = cdiv(keys, cowa::kDecBN) + 3;
    const long long resident = (long long)sms * cowa::decode_ctas_per_sm((int)s->d);
    // at most 64 splits (the merge's limit) and at least four key tiles each
    long long max_sp = tiles / 4 < 64 ? tiles / 4 : 64;
    if (max_sp < 1) max_sp = 1;
    double best = 1e30;
    for (long long sp = 1; sp <= max_sp; ++sp) {
        const double v = (double)cdiv(pairs * sp, resident) / (double)sp;
        if (v < best) best = v;
    }
    for (long long sp = 1; sp <= max_sp; ++sp)
        if ((double)cdiv(pairs * sp, resident) / (double)sp <= best * 1.03) return (int)sp;
    return (int)max_sp;
}

}  // namespace

int cowa::set_error_detail(int status, const char *detail) { return fail(status, "%s", detail); }

extern "C" {

const char *cowa_status_string(int status)
{
    switch (status) {
    case COWA_OK: return "COWA_OK";
    case COWA_ERR_INVALID_ARG: return "COWA_ERR_INVALID_ARG";
    case COWA_ERR_UNSUPPORTED: return "COWA_ERR_UNSUPPORTED";
    case COWA_ERR_ALIGNMENT: return "COWA_ERR_ALIGNMENT";
    case COWA_ERR_WORKSPACE: return "COWA_ERR_WORKSPACE";
    case COWA_ERR_CUDA: return "COWA_ERR_CUDA";
    case COWA_ERR_TIMEOUT: return "COWA_ERR_TIMEOUT";
    case COWA_ERR_DEVICE: return "COWA_ERR_DEVICE";
    default: return "COWA_ERR_UNKNOWN";
    }
}

const char *cowa_last_error_detail(void) { return tl_detail; }

int cowa_abi_version(void) { return COWA_ABI_VERSION; }

uint64_t cowa_launch_count(void) { return cowa::g_launches.load(std::memory_order_relaxed); }

int cowa_trace_start(int64_t capacity, const char *only)
{
    if (capacity < 0 || capacity > (1 << 20))
        return fail(COWA_ERR_INVALID_ARG, "trace capacity %lld outside 0 .. 2^20", (long long)capacity);
    if (only && strlen(only) >= sizeof cowa::g_trace_only)
        return fail(COWA_ERR_INVALID_ARG, "trace filter longer than %d characters",
                    (int)sizeof cowa::g_trace_only - 1);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    cowa::g_trace_on.store(0, std::memory_order_release);
    std::lock_guard<std::mutex> lk(cowa::g_trace_mu);
    cowa::trace_clear_locked();
    cowa::g_trace.reserve((size_t)capacity);
    for (int64_t i = 0; i < capacity; ++i) {
        cowa::TraceRec r{nullptr, nullptr, nullptr};
        if ((e = cudaEventCreate(&r.a)) != cudaSuccess) break;
        if ((e = cudaEventCreate(&r.b)) != cudaSuccess) {
            cudaEventDestroy(r.a);
            break;
        }
        cowa::g_trace.push_back(r);
    }
    if (e != cudaSuccess) {
        cowa::trace_clear_locked();
        return cuda_fail(e, "cudaEventCreate");
    }
    cowa::g_trace_dev = dev;
    snprintf(cowa::g_trace_only, sizeof cowa::g_trace_only, "%s", only ? only : "");
    cowa::g_trace_on.store(capacity > 0 ? 1 : 0, std::memory_order_release);
    return COWA_OK;
}

int cowa_trace_stop(void)
{
    cowa::g_trace_on.store(0, std::memory_order_release);
    return COWA_OK;
}

int64_t cowa_trace_size(void)
{
    std::lock_guard<std::mutex> lk(cowa::g_trace_mu);
    return (int64_t)cowa::g_trace_used;
}

int64_t cowa_trace_dropped(void)
{
    std::lock_guard<std::mutex> lk(cowa::g_trace_mu);
    return (int64_t)cowa::g_trace_dropped;
}

int cowa_trace_entry(int64_t i, const char **name, float *ms)
{
    std::lock_guard<std::mutex> lk(cowa::g_trace_mu);
    if (i < 0 || (size_t)i >= cowa::g_trace_used || !name || !ms)
        return fail(COWA_ERR_INVALID_ARG, "trace entry %lld of %lld (or NULL output)", (long long)i,
                    (long long)cowa::g_trace_used);
    const cowa::TraceRec &r = cowa::g_trace[(size_t)i];
    if (!r.name) return fail(COWA_ERR_CUDA, "trace entry %lld has no end event", (long long)i);
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float t = 0.f;
    e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    *name = r.name;
    *ms = t;
    return COWA_OK;
}

cowa_quad_t cowa_default_quad(int64_t Lk, int64_t Hkv, int32_t S, int32_t N)
{
    cowa_quad_t q;
    q.S = S;
    q.N = N;
    q.G = 0;
    long long rest = (long long)Lk - N;
    long long W = (Hkv > 0 && rest > 0) ? cdiv(rest, Hkv) : 0;
    q.W = (int32_t)(W > 0x7fffffff ? 0x7fffffff : W);
    return q;
}

size_t cowa_fwd_workspace_size(const cowa_shape_t *s, cowa_quad_t q)
{
    if (check_shape(s, q, false)) return 0;
    return sched_bytes(s->Hkv, cdiv(s->Lq, cowa::kFwd5BM)) + 256;
}

size_t cowa_bwd_workspace_size(const cowa_shape_t *s, cowa_quad_t q)
{
    if (check_shape(s, q, false)) return 0;
    // per-row (-LSE*log2e, -delta) pairs padded to 64 rows (also holds the
    // warp-level path's delta), then two schedules sized for the finer tiling
    return align256((size_t)(s->B * s->Hq * cowa::bwd5_lq_pad(s->Lq)) * sizeof(float2)) +
           sched_bytes(s->Hkv, cdiv(s->Lq, 64)) + sched_bytes(s->Hkv, cdiv(s->Lk, 64)) + 256;
}

size_t cowa_decode_workspace_size(const cowa_shape_t *s, cowa_quad_t q)
{
    if (check_shape(s, q, true)) return 0;
    int sms = 148;
    if (check_device(&sms)) return 0;
    const long long sp = decode_splits(s, q, sms);
    const long long rows = s->B * s->Hq * sp;
    return align256((size_t)(rows * s->d) * sizeof(float)) + align256((size_t)rows * sizeof(float)) + 256;
}

int cowa_fwd(const cowa_shape_t *s, cowa_quad_t quad, float softmax_scale, const void *q, const void *k,
             const void *v, void *o, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    int r = check_shape(s, quad, false);
    if (r) return r;
    const bool qrows = s->B * s->Lq * s->Hq > 0, krows = s->B * s->Lk * s->Hkv > 0;
    if ((r = check_ptr(q, qrows, "q")) || (r = check_ptr(k, qrows && krows, "k")) ||
        (r = check_ptr(v, qrows && krows, "v")) || (r = check_ptr(o, qrows, "o")) ||
        (r = check_ptr(lse, qrows, "lse")))
        return r;
    if (!qrows) return COWA_OK;
    if ((r = check_device(nullptr))) return r;
    const size_t need = cowa_fwd_workspace_size(s, quad);
    if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
        return fail(COWA_ERR_WORKSPACE, "fwd workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
    cudaStream_t st = (cudaStream_t)stream;
    cowa::AttnParams p{};
    fill_common(p, s, quad, softmax_scale);
    p.q = q; p.k = k; p.v = v; p.o = o; p.lse = lse;
    p.B = (int)s->B; p.Lq = (int)s->Lq; p.Lk = (int)s->Lk;
    p.lse_ld = s->Lq;
    if (s->Lk == 0) {
        // no keys at all: every row sees nothing (O = 0, LSE = -inf)
        cudaError_t e = cowa::launch_zero_rows(o, p.os, p.B, p.Lq, p.Hq, (int)s->d, st);
        if (e == cudaSuccess) e = cowa::launch_fill_f32(lse, s->B * s->Hq * s->Lq, -INFINITY, st);
        return e == cudaSuccess ? COWA_OK : cuda_fail(e, "constant output launch");
    }
    const int BN = cowa::fwd5_bn((int)s->d);
    p.nqt = (int)cdiv(s->Lq, cowa::kFwd5BM);
    p.nkt = (int)cdiv(s->Lk, BN);
    cudaError_t e = cowa::launch_fwd_sm100(p, (int)s->d, st);
    if (e == cudaErrorInvalidValue) return fail(COWA_ERR_CUDA, "TMA descriptor encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return COWA_OK;
}

int cowa_bwd(const cowa_shape_t *s, cowa_quad_t quad, float softmax_scale, const void *q, const void *k,
             const void *v, const void *o, const float *lse, const void *dout, void *dq, void *dk, void *dv,
             void *ws, size_t ws_bytes, void *stream)
{
    int r = check_shape(s, quad, false);
    if (r) return r;
    const bool qrows = s->B * s->Lq * s->Hq > 0, krows = s->B * s->Lk * s->Hkv > 0;
    if ((r = check_ptr(q, qrows, "q")) || (r = check_ptr(k, krows, "k")) || (r = check_ptr(v, krows, "v")) ||
        (r = check_ptr(o, qrows, "o")) || (r = check_ptr(lse, qrows, "lse")) ||
        (r = check_ptr(dout, qrows, "dout")) || (r = check_ptr(dq, qrows, "dq")) ||
        (r = check_ptr(dk, krows, "dk")) || (r = check_ptr(dv, krows, "dv")))
        return r;
    if (!qrows && !krows) return COWA_OK;
    if ((r = check_device(nullptr))) return r;
    const size_t need = cowa_bwd_workspace_size(s, quad);
    if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
        return fail(COWA_ERR_WORKSPACE, "bwd workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
    cudaStream_t st = (cudaStream_t)stream;
    cowa::AttnParams p{};
    fill_common(p, s, quad, softmax_scale);
    p.q = q; p.k = k; p.v = v; p.o = (void *)o; p.lse_in = lse; p.dout = dout;
    p.dq = dq; p.dk = dk; p.dv = dv;
    p.B = (int)s->B; p.Lq = (int)s->Lq; p.Lk = (int)s->Lk;
    p.lse_ld = s->Lq;
    char *rows_ws = (char *)ws;
    const int D = (int)s->d;
    cudaError_t e;
    if (s->Lq > 0 && s->Lk > 0) {
        // tensor-core path: dK/dV over key tiles of 128, dQ over query tiles of 128
        // (the tcgen05 kernels form their tile ranges themselves: no schedule)
        const int nqt = (int)cdiv(s->Lq, cowa::kBwd5QTile), nkt = (int)cdiv(s->Lk, cowa::kBwd5KeyTile);
        e = cowa::launch_bwd_sm100(p, D, (float2 *)rows_ws, (int)cowa::bwd5_lq_pad(s->Lq), nqt, nkt, st);
        if (e == cudaErrorInvalidValue) return fail(COWA_ERR_CUDA, "TMA descriptor encoding failed");
        if (e != cudaSuccess) return cuda_fail(e, "backward launch");
        return COWA_OK;
    }
    // no queries or no keys: every gradient is zero
    e = qrows ? cowa::launch_zero_rows(dq, p.qs, p.B, p.Lq, p.Hq, D, st) : cudaSuccess;
    if (e == cudaSuccess && krows) e = cowa::launch_zero_rows(dk, p.ks, p.B, p.Lk, p.Hkv, D, st);
    if (e == cudaSuccess && krows) e = cowa::launch_zero_rows(dv, p.vs, p.B, p.Lk, p.Hkv, D, st);
    if (e != cudaSuccess) return cuda_fail(e, "constant gradient launch");
    return COWA_OK;
}

static int decode_common(const cowa_shape_t *s, cowa_quad_t quad, float softmax_scale, const void *q,
                         const void *k_cache, const void *v_cache, const int32_t *seqlens, void *o, float *lse,
                         void *ws, size_t ws_bytes, void *stream, const int32_t *origin, int32_t horizon);

int cowa_decode(const cowa_shape_t *s, cowa_quad_t quad, float softmax_scale, const void *q, const void *k_cache,
                const void *v_cache, const int32_t *seqlens, void *o, float *lse, void *ws, size_t ws_bytes,
                void *stream)
{
    return decode_common(s, quad, softmax_scale, q, k_cache, v_cache, seqlens, o, lse, ws, ws_bytes, stream,
                         nullptr, 0);
}

int64_t cowa_wcache_rows(cowa_quad_t quad, int32_t horizon)
{
    if (quad.S < 0 || quad.N < 0 || quad.G < 0 || quad.W < 0 || horizon <= 0) return 0;
    const long long rows = (long long)quad.S + quad.N + quad.W + 2ll * horizon;
    return rows >= kMaxLen ? 0 : rows;
}

int cowa_decode_windowed(const cowa_shape_t *s, cowa_quad_t quad, float softmax_scale, int32_t horizon,
                         const int32_t *origin, const void *q, const void *k_win, const void *v_win,
                         const int32_t *seqlens, void *o, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    const int64_t rows = cowa_wcache_rows(quad, horizon);
    if (rows == 0) return fail(COWA_ERR_INVALID_ARG, "bad quadruple or horizon %d", horizon);
    if (s && s->Lk != rows)
        return fail(COWA_ERR_INVALID_ARG, "windowed cache has %lld rows, expected %lld", (long long)s->Lk,
                    (long long)rows);
    if (s && s->B * s->Hq > 0 && !origin) return fail(COWA_ERR_INVALID_ARG, "origin is NULL");
    return decode_common(s, quad, softmax_scale, q, k_win, v_win, seqlens, o, lse, ws, ws_bytes, stream, origin,
                         horizon);
}

static int wcache_params(const cowa_shape_t *s, cowa_quad_t quad, int32_t horizon, const int32_t *origin,
                         cowa::WCacheParams &p)
{
    if (!s) return fail(COWA_ERR_INVALID_ARG, "shape is NULL");
    int r = check_quad(quad);
    if (r) return r;
    const int64_t rows = cowa_wcache_rows(quad, horizon);
    if (rows == 0) return fail(COWA_ERR_INVALID_ARG, "bad horizon %d", horizon);
    if (s->B < 0 || s->Hkv < 0 || s->Lk < 0 || s->kv_head_offset < 0 || s->B > 65535 || s->Hkv > 65535 ||
        s->Lk >= kMaxLen)
        return fail(COWA_ERR_INVALID_ARG, "bad sizes in shape");
    if (s->d != 64 && s->d != 128)
        return fail(COWA_ERR_UNSUPPORTED, "head dim %lld (supported: 64, 128)", (long long)s->d);
    if ((r = check_strides(s->k_stride, "k")) || (r = check_strides(s->v_stride, "v"))) return r;
    if (s->B * s->Hkv > 0 && !origin) return fail(COWA_ERR_INVALID_ARG, "origin is NULL");
    p = cowa::WCacheParams{};
    for (int a = 0; a < 3; ++a) {
        p.ks[a] = s->k_stride[a];
        p.vs[a] = s->v_stride[a];
    }
    p.origin = origin;
    p.B = (int)s->B;
    p.Hkv = (int)s->Hkv;
    p.rows = (int)rows;
    p.horizon = horizon;
    p.Lsrc = (int)s->Lk;
    p.S = quad.S;
    p.N = quad.N;
    p.G = quad.G;
    p.W = quad.W;
    p.kv_head_offset = (int)s->kv_head_offset;
    p.err = device_error_word();
    return COWA_OK;
}

int cowa_wcache_build(const cowa_shape_t *s, cowa_quad_t quad, int32_t horizon, const int32_t *origin,
                      const void *k_full, const void *v_full, void *k_win, void *v_win, void *stream)
{
    cowa::WCacheParams p;
    int r = wcache_params(s, quad, horizon, origin, p);
    if (r) return r;
    const bool work = s->B * s->Hkv > 0;
    if ((r = check_ptr(k_full, work && s->Lk > 0, "k_full")) || (r = check_ptr(v_full, work && s->Lk > 0, "v_full")) ||
        (r = check_ptr(k_win, work, "k_win")) || (r = check_ptr(v_win, work, "v_win")))
        return r;
    if (!work) return COWA_OK;
    if ((r = check_device(nullptr))) return r;
    p.err = device_error_word();
    p.ksrc = k_full;
    p.vsrc = v_full;
    p.kw = k_win;
    p.vw = v_win;
    cudaError_t e = cowa::launch_wcache_build(p, (int)s->d, (cudaStream_t)stream);
    return e == cudaSuccess ? COWA_OK : cuda_fail(e, "windowed cache build launch");
}

int cowa_wcache_append(const cowa_shape_t *s, cowa_quad_t quad, int32_t horizon, const int32_t *origin,
                       const int32_t *pos, const void *k_new, const void *v_new, void *k_win, void *v_win,
                       void *stream)
{
    cowa::WCacheParams p;
    int r = wcache_params(s, quad, horizon, origin, p);
    if (r) return r;
    const bool work = s->B * s->Hkv > 0;
    if ((r = check_ptr(k_new, work, "k_new")) || (r = check_ptr(v_new, work, "v_new")) ||
        (r = check_ptr(k_win, work, "k_win")) || (r = check_ptr(v_win, work, "v_win")))
        return r;
    if (work && !pos) return fail(COWA_ERR_INVALID_ARG, "pos is NULL");
    if (!work) return COWA_OK;
    if ((r = check_device(nullptr))) return r;
    p.err = device_error_word();
    p.ksrc = k_new;
    p.vsrc = v_new;
    p.kw = k_win;
    p.vw = v_win;
    p.pos = pos;
    cudaError_t e = cowa::launch_wcache_append(p, (int)s->d, (cudaStream_t)stream);
    return e == cudaSuccess ? COWA_OK : cuda_fail(e, "windowed cache append launch");
}

static int decode_common(const cowa_shape_t *s, cowa_quad_t quad, float softmax_scale, const void *q,
                         const void *k_cache, const void *v_cache, const int32_t *seqlens, void *o, float *lse,
                         void *ws, size_t ws_bytes, void *stream, const int32_t *origin, int32_t horizon)
{
    int r = check_shape(s, quad, true);
    if (r) return r;
    const bool rows = s->B * s->Hq > 0, cache = s->B * s->Lk * s->Hkv > 0;
    if ((r = check_ptr(q, rows, "q")) || (r = check_ptr(k_cache, rows && cache, "k_cache")) ||
        (r = check_ptr(v_cache, rows && cache, "v_cache")) || (r = check_ptr(o, rows, "o")) ||
        (r = check_ptr(lse, rows, "lse")))
        return r;
    if (rows && !seqlens) return fail(COWA_ERR_INVALID_ARG, "seqlens is NULL");
    if (!rows) return COWA_OK;
    int sms = 148;
    if ((r = check_device(&sms))) return r;
    const size_t need = cowa_decode_workspace_size(s, quad);
    if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
        return fail(COWA_ERR_WORKSPACE, "decode workspace needs %zu bytes, 256-byte aligned (got %zu)", need,
                    ws_bytes);
    cowa::DecodeParams p{};
    fill_common(p, s, quad, softmax_scale);
    p.q = q; p.kc = k_cache; p.vc = v_cache; p.seqlens = seqlens; p.o = o; p.lse = lse;
    p.B = (int)s->B;
    p.Lcap = (int)s->Lk;
    p.splits = decode_splits(s, quad, sms);
    const size_t rows_p = (size_t)(s->B * s->Hq * p.splits);
    p.part_o = (float *)ws;
    p.part_lse = (float *)((char *)ws + align256(rows_p * s->d * sizeof(float)));
    p.origin = origin;
    p.horizon = horizon;
    cudaError_t e = cowa::launch_decode(p, (int)s->d, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return COWA_OK;
}

// ------------------------------------------------------- packed batches --
static int check_varlen(const cowa_varlen_shape_t *s, cowa_quad_t q)
{
    if (!s) return fail(COWA_ERR_INVALID_ARG, "shape is NULL");
    if (s->B < 0 || s->total_q < 0 || s->total_k < 0 || s->max_q < 0 || s->max_k < 0 || s->Hq < 0 ||
        s->Hkv < 0 || s->kv_head_offset < 0)
        return fail(COWA_ERR_INVALID_ARG, "negative size in shape");
    if (s->total_q >= kMaxLen || s->total_k >= kMaxLen || s->B > 65535 || s->Hq > 65535 || s->Hkv > 65535)
        return fail(COWA_ERR_UNSUPPORTED, "token counts must be < 2^30, sequences/heads <= 65535");
    if (s->max_q > s->total_q || s->max_k > s->total_k)
        return fail(COWA_ERR_INVALID_ARG, "longest sequence exceeds the token count");
    if (s->Hq > 0 && (s->Hkv == 0 || s->Hq % s->Hkv))
        return fail(COWA_ERR_INVALID_ARG, "Hq=%lld is not a multiple of Hkv=%lld", (long long)s->Hq,
                    (long long)s->Hkv);
    if (s->d != 64 && s->d != 128)
        return fail(COWA_ERR_UNSUPPORTED, "head dim %lld (supported: 64, 128)", (long long)s->d);
    if (s->kv_head_offset + s->Hkv > kMaxLen) return fail(COWA_ERR_INVALID_ARG, "kv_head_offset too large");
    if (s->B * s->Hq * cdiv(s->max_q, 32) > 0x7fffffffll || s->B * s->Hkv * cdiv(s->max_k, 32) > 0x7fffffffll)
        return fail(COWA_ERR_UNSUPPORTED, "sequences * heads * length / 32 exceeds 2^31 - 1");
    int r = check_quad(q);
    if (r) return r;
    const int64_t *st[4] = {s->q_stride, s->k_stride, s->v_stride, s->o_stride};
    const char *nm[4] = {"q", "k", "v", "o"};
    for (int t = 0; t < 4; ++t)
        for (int a = 0; a < 2; ++a)
            if (st[t][a] < 0 || st[t][a] % 8)
                return fail(COWA_ERR_ALIGNMENT, "%s stride[%d] = %lld is not a non-negative multiple of 8 elements",
                            nm[t], a, (long long)st[t][a]);
    return COWA_OK;
}

// AttnParams of a packed batch: one batch entry of total rows, per-sequence
// offsets from cu_q / cu_k, schedules per sequence
static void fill_varlen(cowa::AttnParams &p, const cowa_varlen_shape_t *s, cowa_quad_t q, float scale,
                        const int32_t *cu_q, const int32_t *cu_k)
{
    for (int a = 0; a < 2; ++a) {
        p.qs[a + 1] = s->q_stride[a];
        p.ks[a + 1] = s->k_stride[a];
        p.vs[a + 1] = s->v_stride[a];
        p.os[a + 1] = s->o_stride[a];
    }
    p.qs[0] = p.ks[0] = p.vs[0] = p.os[0] = 0;
    p.Hq = (int)s->Hq;
    p.Hkv = (int)s->Hkv;
    p.g = s->Hkv > 0 ? (int)(s->Hq / s->Hkv) : 1;
    p.S = q.S; p.N = q.N; p.G = q.G; p.W = q.W;
    p.kv_head_offset = (int)s->kv_head_offset;
    p.scale = resolve_scale(scale, s->d);
    p.scale_log2 = p.scale * 1.4426950408889634f;
    p.err = device_error_word();
    p.B = (int)s->B;
    p.Lq = (int)s->max_q;
    p.Lk = (int)s->max_k;
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.total_q = (int)s->total_q;
    p.total_k = (int)s->total_k;
    p.lse_ld = s->total_q;
}

// Work list of a packed batch for tiles of 128 rows: (sequence, tile) items,
// at most total/128 + B of them, and the scratch of the list builder
// (3 ints per possible tile count of one sequence).
struct WorkList {
    long long items, max_tiles;
    size_t list_bytes() const { return align256((size_t)items * sizeof(int2)); }
    size_t scratch_bytes() const { return align256((size_t)(3 * (max_tiles + 1)) * sizeof(int)); }
    size_t bytes() const { return list_bytes() + scratch_bytes(); }
};
static WorkList work_list(long long total, long long max_len, long long B)
{
    return WorkList{total / 128 + B + 1, cdiv(max_len, 128)};
}

// Builds the list into ws (list, then scratch); returns the pointer to the list.
static cudaError_t build_work_list(const WorkList &wl, const int32_t *cu, long long B, bool descending, char *ws,
                                   int2 **list, cudaStream_t st)
{
    *list = (int2 *)ws;
    return cowa::launch_varlen_worklist(cu, (int)B, 128, (int)wl.max_tiles, descending, *list, (int)wl.items,
                                        (int *)(ws + wl.list_bytes()), device_error_word(), st);
}

size_t cowa_fwd_varlen_workspace_size(const cowa_varlen_shape_t *s, cowa_quad_t q)
{
    if (check_varlen(s, q)) return 0;
    // the kernels form their tile ranges themselves; the work list of the
    // query tiles sizes the grid to the real tiles
    return work_list(s->total_q, s->max_q, s->B).bytes() + 256;
}

size_t cowa_bwd_varlen_workspace_size(const cowa_varlen_shape_t *s, cowa_quad_t q)
{
    if (check_varlen(s, q)) return 0;
    return align256((size_t)(s->B * s->Hq * cowa::bwd5_lq_pad(s->max_q)) * sizeof(float2)) +
           work_list(s->total_q, s->max_q, s->B).bytes() + work_list(s->total_k, s->max_k, s->B).bytes() + 256;
}

int cowa_fwd_varlen(const cowa_varlen_shape_t *s, cowa_quad_t quad, float softmax_scale, const int32_t *cu_q,
                    const int32_t *cu_k, const void *q, const void *k, const void *v, void *o, float *lse, void *ws,
                    size_t ws_bytes, void *stream)
{
    int r = check_varlen(s, quad);
    if (r) return r;
    const bool qrows = s->B * s->total_q * s->Hq > 0 && s->max_q > 0;
    if (!qrows) return COWA_OK;
    if (s->total_k == 0 || s->max_k == 0)
        return fail(COWA_ERR_UNSUPPORTED, "packed batch without keys (every output would be empty)");
    if ((r = check_ptr(q, true, "q")) || (r = check_ptr(k, true, "k")) || (r = check_ptr(v, true, "v")) ||
        (r = check_ptr(o, true, "o")) || (r = check_ptr(lse, true, "lse")))
        return r;
    if (!cu_q || !cu_k) return fail(COWA_ERR_INVALID_ARG, "cu_q / cu_k is NULL");
    if ((r = check_device(nullptr))) return r;
    const size_t need = cowa_fwd_varlen_workspace_size(s, quad);
    if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
        return fail(COWA_ERR_WORKSPACE, "fwd workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
    cudaStream_t st = (cudaStream_t)stream;
    cowa::AttnParams p{};
    fill_varlen(p, s, quad, softmax_scale, cu_q, cu_k);
    p.q = q; p.k = k; p.v = v; p.o = o; p.lse = lse;
    const int BN = cowa::fwd5_bn((int)s->d);
    p.nqt = (int)cdiv(s->max_q, cowa::kFwd5BM);
    p.nkt = (int)cdiv(s->max_k, BN);
    const WorkList wq = work_list(s->total_q, s->max_q, s->B);
    int2 *list = nullptr;
    cudaError_t e = build_work_list(wq, cu_q, s->B, true, (char *)ws, &list, st);
    if (e != cudaSuccess) return cuda_fail(e, "work list launch");
    p.work = list;
    p.work_n = (int)wq.items;
    e = cowa::launch_fwd_sm100(p, (int)s->d, st);
    if (e == cudaErrorInvalidValue) return fail(COWA_ERR_CUDA, "TMA descriptor encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return COWA_OK;
}

int cowa_bwd_varlen(const cowa_varlen_shape_t *s, cowa_quad_t quad, float softmax_scale, const int32_t *cu_q,
                    const int32_t *cu_k, const void *q, const void *k, const void *v, const void *o,
                    const float *lse, const void *dout, void *dq, void *dk, void *dv, void *ws, size_t ws_bytes,
                    void *stream)
{
    int r = check_varlen(s, quad);
    if (r) return r;
    if (s->B == 0 || s->Hq == 0 || (s->total_q == 0 && s->total_k == 0)) return COWA_OK;
    if (s->total_q == 0 || s->total_k == 0 || s->max_q == 0 || s->max_k == 0)
        return fail(COWA_ERR_UNSUPPORTED, "packed batch without queries or keys (every gradient would be zero)");
    if ((r = check_ptr(q, true, "q")) || (r = check_ptr(k, true, "k")) || (r = check_ptr(v, true, "v")) ||
        (r = check_ptr(o, true, "o")) || (r = check_ptr(lse, true, "lse")) || (r = check_ptr(dout, true, "dout")) ||
        (r = check_ptr(dq, true, "dq")) || (r = check_ptr(dk, true, "dk")) || (r = check_ptr(dv, true, "dv")))
        return r;
    if (!cu_q || !cu_k) return fail(COWA_ERR_INVALID_ARG, "cu_q / cu_k is NULL");
    if ((r = check_device(nullptr))) return r;
    const size_t need = cowa_bwd_varlen_workspace_size(s, quad);
    if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
        return fail(COWA_ERR_WORKSPACE, "bwd workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
    cudaStream_t st = (cudaStream_t)stream;
    cowa::AttnParams p{};
    fill_varlen(p, s, quad, softmax_scale, cu_q, cu_k);
    p.q = q; p.k = k; p.v = v; p.o = (void *)o; p.lse_in = lse; p.dout = dout;
    p.dq = dq; p.dk = dk; p.dv = dv;
    char *rows_ws = (char *)ws;
    const long long lq_pad = cowa::bwd5_lq_pad(s->max_q);
    const int D = (int)s->d;
    const int nqt = (int)cdiv(s->max_q, cowa::kBwd5QTile), nkt = (int)cdiv(s->max_k, cowa::kBwd5KeyTile);
    // work lists: query tiles (dQ, last tile first), key tiles (dK/dV, first
    // tile first)
    const WorkList wq = work_list(s->total_q, s->max_q, s->B), wk = work_list(s->total_k, s->max_k, s->B);
    char *lists = rows_ws + align256((size_t)(s->B * s->Hq * lq_pad) * sizeof(float2));
    int2 *list_q = nullptr, *list_k = nullptr;
    cudaError_t e = build_work_list(wq, cu_q, s->B, true, lists, &list_q, st);
    if (e == cudaSuccess) e = build_work_list(wk, cu_k, s->B, false, lists + wq.bytes(), &list_k, st);
    if (e != cudaSuccess) return cuda_fail(e, "work list launch");
    e = cowa::launch_bwd_sm100(p, D, (float2 *)rows_ws, (int)lq_pad, nqt, nkt, st, list_q, (int)wq.items, list_k,
                               (int)wk.items);
    if (e == cudaErrorInvalidValue) return fail(COWA_ERR_CUDA, "TMA descriptor encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return COWA_OK;
}

// ------------------------------------------------------------------- MALA --
// MassAlloc Attention: full causal scoring, blocks of kMalaBM query rows x
// kMalaBN keys kept when some row gives them at least tau of its softmax
// mass (the reading is in include/cowa.h and csrc/mala.cu).

static int check_mala(const cowa_shape_t *s, float tau)
{
    const cowa_quad_t full = {0, 0, 0, 0};
    int r = check_shape(s, full, false);
    if (r) return r;
    if (s->kv_head_offset != 0) return fail(COWA_ERR_INVALID_ARG, "MALA has no per-head windows: kv_head_offset must be 0");
    if (!(tau >= 0.f) || !(tau <= 1e30f)) return fail(COWA_ERR_INVALID_ARG, "tau must be a finite value >= 0");
    return COWA_OK;
}

size_t cowa_mala_keep_bytes(const cowa_shape_t *s)
{
    if (check_mala(s, 0.f)) return 0;
    return (size_t)(s->B * s->Hq * cdiv(s->Lq, cowa::kMalaBM) * cdiv(s->Lk, cowa::kMalaBN));
}

int cowa_mala_fwd(const cowa_shape_t *s, float tau, float softmax_scale, const void *q, const void *k, const void *v,
                  void *o, float *lse, uint8_t *keep, void *stream)
{
    int r = check_mala(s, tau);
    if (r) return r;
    const bool qrows = s->B * s->Lq * s->Hq > 0, krows = s->B * s->Lk * s->Hkv > 0;
    if ((r = check_ptr(q, qrows, "q")) || (r = check_ptr(k, qrows && krows, "k")) ||
        (r = check_ptr(v, qrows && krows, "v")) || (r = check_ptr(o, qrows, "o")) ||
        (r = check_ptr(lse, qrows, "lse")))
        return r;
    if (qrows && krows && !keep) return fail(COWA_ERR_INVALID_ARG, "keep is NULL");
    if (!qrows) return COWA_OK;
    if ((r = check_device(nullptr))) return r;
    cudaStream_t st = (cudaStream_t)stream;
    cowa::AttnParams p{};
    fill_common(p, s, cowa_quad_t{0, 0, 0, 0}, softmax_scale);
    p.q = q; p.k = k; p.v = v; p.o = o; p.lse = lse;
    p.B = (int)s->B; p.Lq = (int)s->Lq; p.Lk = (int)s->Lk;
    p.lse_ld = s->Lq;
    if (s->Lk == 0) {
        // no keys: every row sees nothing (O = 0, LSE = -inf); no blocks
        cudaError_t e = cowa::launch_zero_rows(o, p.os, p.B, p.Lq, p.Hq, (int)s->d, st);
        if (e == cudaSuccess) e = cowa::launch_fill_f32(lse, s->B * s->Hq * s->Lq, -INFINITY, st);
        return e == cudaSuccess ? COWA_OK : cuda_fail(e, "constant output launch");
    }
    p.nqt = (int)cdiv(s->Lq, cowa::kMalaBM);
    p.nkt = (int)cdiv(s->Lk, cowa::kMalaBN);
    cudaError_t e = cowa::launch_mala_fwd(p, (int)s->d, keep, tau, st);
    if (e == cudaErrorInvalidValue) return fail(COWA_ERR_CUDA, "TMA descriptor encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "MALA forward launch");
    return COWA_OK;
}

size_t cowa_mala_bwd_workspace_size(const cowa_shape_t *s)
{
    if (check_mala(s, 0.f)) return 0;
    return cowa_bwd_workspace_size(s, cowa_quad_t{0, (int32_t)s->Lk, 0, 0});
}

int cowa_mala_bwd(const cowa_shape_t *s, float softmax_scale, const void *q, const void *k, const void *v,
                  const void *o, const float *lse, const uint8_t *keep, const void *dout, void *dq, void *dk, void *dv,
                  void *ws, size_t ws_bytes, void *stream)
{
    int r = check_mala(s, 0.f);
    if (r) return r;
    const bool qrows = s->B * s->Lq * s->Hq > 0, krows = s->B * s->Lk * s->Hkv > 0;
    if (qrows && krows && !keep) return fail(COWA_ERR_INVALID_ARG, "keep is NULL");
    if (!qrows || !krows) {
        // no pair at all: the gradients are those of cowa_bwd (zero)
        return cowa_bwd(s, cowa_quad_t{0, (int32_t)s->Lk, 0, 0}, softmax_scale, q, k, v, o, lse, dout, dq, dk, dv, ws,
                        ws_bytes, stream);
    }
    if ((r = check_ptr(q, true, "q")) || (r = check_ptr(k, true, "k")) || (r = check_ptr(v, true, "v")) ||
        (r = check_ptr(o, true, "o")) || (r = check_ptr(lse, true, "lse")) || (r = check_ptr(dout, true, "dout")) ||
        (r = check_ptr(dq, true, "dq")) || (r = check_ptr(dk, true, "dk")) || (r = check_ptr(dv, true, "dv")))
        return r;
    if ((r = check_device(nullptr))) return r;
    // the backward of every causal pair (the scores are full), with the
    // forward's block decisions: pairs of skipped blocks keep only -P * delta
    const cowa_quad_t full = {0, (int32_t)s->Lk, 0, 0};
    const size_t need = cowa_bwd_workspace_size(s, full);
    if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
        return fail(COWA_ERR_WORKSPACE, "MALA bwd workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
    cudaStream_t st = (cudaStream_t)stream;
    cowa::AttnParams p{};
    fill_common(p, s, full, softmax_scale);
    p.q = q; p.k = k; p.v = v; p.o = (void *)o; p.lse_in = lse; p.dout = dout;
    p.dq = dq; p.dk = dk; p.dv = dv;
    p.B = (int)s->B; p.Lq = (int)s->Lq; p.Lk = (int)s->Lk;
    p.lse_ld = s->Lq;
    p.keep = keep;
    p.keep_nqt = (int)cdiv(s->Lq, cowa::kMalaBM);
    p.keep_nkt = (int)cdiv(s->Lk, cowa::kMalaBN);
    const int nqt = (int)cdiv(s->Lq, cowa::kBwd5QTile), nkt = (int)cdiv(s->Lk, cowa::kBwd5KeyTile);
    cudaError_t e = cowa::launch_bwd_sm100(p, (int)s->d, (float2 *)ws, (int)cowa::bwd5_lq_pad(s->Lq), nqt, nkt, st);
    if (e == cudaErrorInvalidValue) return fail(COWA_ERR_CUDA, "TMA descriptor encoding failed");
    if (e != cudaSuccess) return cuda_fail(e, "MALA backward launch");
    return COWA_OK;
}

size_t cowa_schedule_workspace_size(int64_t Lq, int64_t Lk, int32_t BM, int32_t BN)
{
    if (Lq < 0 || Lk < 0 || BM <= 0 || BN <= 0) return 0;
    const long long n = cdiv(Lq, BM) > cdiv(Lk, BN) ? cdiv(Lq, BM) : cdiv(Lk, BN);
    return sched_bytes(1, n) + 256;
}

int cowa_tile_classes(int64_t Lq, int64_t Lk, int64_t kv_head, cowa_quad_t quad, int32_t BM, int32_t BN,
                      int transposed, uint8_t *out, void *ws, size_t ws_bytes, void *stream)
{
    int r = check_quad(quad);
    if (r) return r;
    if (Lq < 0 || Lk < 0 || Lq >= kMaxLen || Lk >= kMaxLen || kv_head < 0 || kv_head >= kMaxLen)
        return fail(COWA_ERR_INVALID_ARG, "bad length or head");
    if ((BM != 64 && BM != 128 && BM != 32) || (BN != 64 && BN != 96 && BN != 128))
        return fail(COWA_ERR_UNSUPPORTED, "tiling %dx%d (supported: 32/64/128 x 64/96/128)", BM, BN);
    if (Lq == 0 || Lk == 0) return COWA_OK;
    if (!out) return fail(COWA_ERR_INVALID_ARG, "out is NULL");
    if ((r = check_device(nullptr))) return r;
    const size_t need = cowa_schedule_workspace_size(Lq, Lk, BM, BN);
    if (!ws || ws_bytes < need || (uintptr_t)ws % 256)
        return fail(COWA_ERR_WORKSPACE, "schedule workspace needs %zu bytes", need);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cowa::launch_schedule((int *)ws, 1, (int)kv_head, (int)Lq, (int)Lk, quad.S, quad.N, quad.G,
                                          quad.W, BM, BN, transposed ? 1 : 0, st);
    if (e == cudaSuccess)
        e = cowa::launch_tile_classes((const int *)ws, out, (int)kv_head, (int)Lq, (int)Lk, quad.S, quad.N, quad.G,
                                      quad.W, BM, BN, transposed ? 1 : 0, st);
    if (e != cudaSuccess) return cuda_fail(e, "schedule launch");
    return COWA_OK;
}

int cowa_selftest_wait_timeout(void *stream)
{
    const int rc = check_device(nullptr);
    if (rc != COWA_OK) return rc;
    const cudaError_t e = cowa::launch_wait_selftest(device_error_word(), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait self-test launch");
    return COWA_OK;
}

int cowa_get_device_error(void *stream)
{
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, cowa::g_cowa_device_error, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    e = cudaMemcpyToSymbol(cowa::g_cowa_device_error, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    if (v == COWA_ERR_TIMEOUT) return fail(COWA_ERR_TIMEOUT, "a kernel's bounded wait ran out");
    if (v) return fail(COWA_ERR_DEVICE, "a kernel's device-side check failed (code %d)", v);
    return COWA_OK;
}

}  // extern "C"
