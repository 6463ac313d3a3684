// Device-side building blocks of the CoWA library: window geometry, the
// visible-tile schedule, and thin wrappers over PTX instructions.
//
// Window rule ("CoWindow Attention: Full Causal Coverage Is a Collective
// Property", paper digest, method key points; breakpoints fixed by this
// library): for aligned query position p = i + Lk - Lq and key j,
// d = p - j; visible iff d >= 0 and (j < S or d < N or c <= d < e) with
// c = N + G + h*W, e = c + W for the global KV head h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace cowa {

constexpr int kSchedInts = 8;  // n, lo0, hi0, lo1, hi1, lo2, hi2, pad

// Per-head window geometry in 32-bit key units; [c, e) is the long window's
// distance range, clamped so that nothing overflows (a window starting past
// any reachable distance is empty).
struct Win {
    int S, N, c, e;
};

__host__ __device__ inline Win make_win(int S, int N, int G, int W, long long h)
{
    const long long big = 1ll << 30;
    long long c = (long long)N + G + h * (long long)W;
    long long e = c + W;
    Win w;
    w.S = S < big ? S : (int)big;
    w.N = N < big ? N : (int)big;
    w.c = (int)(c < big ? c : big);
    w.e = (int)(e < big ? e : big);
    return w;
}

__host__ __device__ __forceinline__ bool visible(int p, int j, const Win &w)
{
    const int d = p - j;
    return d >= 0 && (j < w.S || d < w.N || (d >= w.c && d < w.e));
}

// Bits lo..hi of a 32-bit word (clipped to 0..31; none when lo > hi).
__host__ __device__ __forceinline__ uint32_t span_bits(int lo, int hi)
{
    lo = lo > 0 ? lo : 0;
    hi = hi < 31 ? hi : 31;
    return lo > hi ? 0u : ((0xFFFFFFFFu >> (31 - (hi - lo))) << lo);
}

// The visible set of one query row (keys) or one key (query positions) as at
// most three runs [a, b], ascending, disjoint and not touching; an absent run
// has a > b.  A thread of the tcgen05 kernels owns one row or one key for the
// whole CTA, so it forms its runs once; a tile is then fully visible to it
// when one run covers the tile's span, and its edge bitmask is the union of
// the runs' bits.
struct Runs3 {
    int a0, b0, a1, b1, a2, b2;
};

// Adds run [a, b] (a not below any earlier run's start) to the runs formed
// so far, merging it with the open run when they overlap or touch.
struct RunBuilder {
    Runs3 r{1, 0, 1, 0, 1, 0};
    int n = 0, ca = 1, cb = 0;  // runs closed so far; the open run
    __host__ __device__ void close()
    {
        if (ca > cb) return;
        if (n == 0) { r.a0 = ca; r.b0 = cb; }
        else if (n == 1) { r.a1 = ca; r.b1 = cb; }
        else { r.a2 = ca; r.b2 = cb; }
        ++n;
    }
    __host__ __device__ void add(int a, int b)
    {
        if (a > b) return;
        if (ca <= cb && a <= cb + 1) {
            cb = b > cb ? b : cb;
            return;
        }
        close();
        ca = a;
        cb = b;
    }
    __host__ __device__ Runs3 done()
    {
        close();
        return r;
    }
};

// Keys seen by the query at aligned position p: sink [0, min(S-1, p)], long
// [p-e+1, p-c] and near [p-N+1, p], clipped at key 0 (in this order their
// starts do not decrease, since e >= N).
__host__ __device__ inline Runs3 row_key_runs(int p, const Win &w)
{
    RunBuilder rb;
    rb.add(0, w.S - 1 < p ? w.S - 1 : p);
    if (w.e > w.c) rb.add(p - w.e + 1 > 0 ? p - w.e + 1 : 0, p - w.c);
    if (w.N > 0) rb.add(p - w.N + 1 > 0 ? p - w.N + 1 : 0, p);
    return rb.done();
}

// Aligned query positions (at most pmax) that see key j: sink [j, pmax] for
// j < S, near [j, j+N-1] and long [j+c, j+e-1].
__host__ __device__ inline Runs3 key_pos_runs(int j, const Win &w, int pmax)
{
    RunBuilder rb;
    const int near_hi = w.N > 0 ? (j + (w.N - 1) < pmax ? j + (w.N - 1) : pmax) : j - 1;
    const int first_hi = j < w.S ? pmax : near_hi;  // the sink reaches every later position
    rb.add(j, first_hi);
    if (w.e > w.c) rb.add(j + w.c, j + (w.e - 1) < pmax ? j + (w.e - 1) : pmax);
    return rb.done();
}

// Whether one run holds all of [lo, hi].
__host__ __device__ __forceinline__ bool runs_cover(const Runs3 &r, int lo, int hi)
{
    return (r.a0 <= lo && hi <= r.b0) || (r.a1 <= lo && hi <= r.b1) || (r.a2 <= lo && hi <= r.b2);
}

// Bit k set when index j0 + k lies in a run.
__host__ __device__ __forceinline__ uint32_t runs_bits(const Runs3 &r, int j0)
{
    return span_bits(r.a0 - j0, r.b0 - j0) | span_bits(r.a1 - j0, r.b1 - j0) | span_bits(r.a2 - j0, r.b2 - j0);
}

// Key tiles visited by a query tile whose in-range rows have aligned
// positions pa..pb: the union over rows of the sink, near and long key
// intervals, each contiguous, so every listed tile holds a visible pair.
// The ranges as the tile loops read them: n, then three [lo, lo + len)
// ranges, ascending and disjoint, with the unused ones zero.
struct TileRanges {
    int n, lo0, len0, lo1, len1, lo2, len2;
};

// Sort three half-open ranges (hi <= lo: absent) and merge those that overlap
// or touch, in scalars only (a runtime-indexed array would live in local
// memory on the device).
__host__ __device__ inline TileRanges merge3(int l0, int h0, int l1, int h1, int l2, int h2)
{
    const int none = 0x7fffffff;
    if (h0 <= l0) l0 = h0 = none;
    if (h1 <= l1) l1 = h1 = none;
    if (h2 <= l2) l2 = h2 = none;
    auto cswap = [](int &la, int &ha, int &lb, int &hb) {
        if (lb < la) {
            const int tl = la, th = ha;
            la = lb;
            ha = hb;
            lb = tl;
            hb = th;
        }
    };
    cswap(l0, h0, l1, h1);
    cswap(l1, h1, l2, h2);
    cswap(l0, h0, l1, h1);
    TileRanges t{0, 0, 0, 0, 0, 0, 0};
    if (l0 == none) return t;
    int cl = l0, ch = h0;
    auto emit = [&](int lo, int hi) {
        if (t.n == 0) {
            t.lo0 = lo;
            t.len0 = hi - lo;
        } else if (t.n == 1) {
            t.lo1 = lo;
            t.len1 = hi - lo;
        } else {
            t.lo2 = lo;
            t.len2 = hi - lo;
        }
        ++t.n;
    };
    if (l1 != none) {
        if (l1 <= ch) {
            ch = h1 > ch ? h1 : ch;
        } else {
            emit(cl, ch);
            cl = l1;
            ch = h1;
        }
    }
    if (l2 != none) {
        if (l2 <= ch) {
            ch = h2 > ch ? h2 : ch;
        } else {
            emit(cl, ch);
            cl = l2;
            ch = h2;
        }
    }
    emit(cl, ch);
    return t;
}

// Key tiles (of BN) a query tile with aligned positions [pa, pb] visits:
// sink [0, S-1], near [pa-N+1, pb], long [pa-e+1, pb-c], clipped at 0.
__host__ __device__ inline TileRanges query_tile_ranges(int pa, int pb, const Win &w, int BN)
{
    int l0 = 0, h0 = 0, l1 = 0, h1 = 0, l2 = 0, h2 = 0;
    if (pb >= 0) {
        const int pa0 = pa > 0 ? pa : 0;
        if (w.S > 0) {
            l0 = 0;
            h0 = (w.S - 1 < pb ? w.S - 1 : pb) / BN + 1;
        }
        if (w.N > 0) {
            const int a = pa0 - w.N + 1 > 0 ? pa0 - w.N + 1 : 0;
            l1 = a / BN;
            h1 = pb / BN + 1;
        }
        if (w.e > w.c && pb - w.c >= 0) {
            const int a = pa0 - (w.e - 1) > 0 ? pa0 - (w.e - 1) : 0;
            l2 = a / BN;
            h2 = (pb - w.c) / BN + 1;
        }
    }
    return merge3(l0, h0, l1, h1, l2, h2);
}

// Query tiles (of BM) whose rows see some key of [c0, c1]: aligned
// positions sink [c0, Lk-1] (keys < S), near [c0, c1+N-1], long
// [c0+c, c1+e-1], within the rows' positions [max(Lk-Lq, 0), Lk-1].
__host__ __device__ inline TileRanges key_tile_ranges(int c0, int c1, int Lq, int Lk, const Win &w, int BM)
{
    const long long delta = (long long)Lk - Lq;
    const long long pmin = delta > 0 ? delta : 0, pmax = (long long)Lk - 1;
    auto rows = [&](long long a, long long b, int &l, int &h) {
        if (a < pmin) a = pmin;
        if (b > pmax) b = pmax;
        if (a <= b) {
            l = (int)((a - delta) / BM);
            h = (int)((b - delta) / BM) + 1;
        }
    };
    int l0 = 0, h0 = 0, l1 = 0, h1 = 0, l2 = 0, h2 = 0;
    if (c0 < w.S) rows(c0, pmax, l0, h0);
    if (w.N > 0) rows(c0, (long long)c1 + w.N - 1, l1, h1);
    if (w.e > w.c) rows((long long)c0 + w.c, (long long)c1 + w.e - 1, l2, h2);
    return merge3(l0, h0, l1, h1, l2, h2);
}

// True when every pair of the tile (rows pa..pb, all in range; columns
// c0..c0+BN-1) is visible, so the tile needs no element mask.  Per column
// j >= S the rows that see it form j + D with D = [0,N) u [c,e); a row
// range fits one connected part [a,b] of D iff j lies in [pb-b, pa-a].  Sink
// columns j < S need j <= pa.  The tile is full iff its columns are covered
// by the union of those (at most three) column intervals.  Scalars only.
// Labels the tiles of cowa_tile_classes; the tcgen05 kernels test coverage
// per thread instead (runs_cover on the thread's visible runs, then a warp
// vote).
__host__ __device__ inline bool tile_full(int pa, int pb, int c0, int BN, int Lk, const Win &w)
{
    const int c1 = c0 + BN - 1;
    if (c1 >= Lk || pa < 0) return false;
    const bool has_near = w.N > 0, has_long = w.e > w.c;
    const bool touch = has_near && has_long && w.c <= w.N;  // near and long windows adjoin
    // sink [0, min(S-1, pa)]
    const int lo0 = 0, hi0 = w.S > 0 ? (w.S - 1 < pa ? w.S - 1 : pa) : -1;
    // near, or near and long together when they adjoin: [pb-(end-1), pa], j >= S
    int lo1 = pb - ((touch ? w.e : w.N) - 1);
    lo1 = lo1 < w.S ? w.S : lo1;
    const int hi1 = has_near ? pa : -1;
    // long on its own: [pb-(e-1), pa-c], j >= S
    int lo2 = pb - (w.e - 1);
    lo2 = lo2 < w.S ? w.S : lo2;
    const int hi2 = (has_long && !touch) ? pa - w.c : -1;
    // greedy cover of [c0, c1]
    int x = c0;
#pragma unroll
    for (int pass = 0; pass < 3; ++pass) {
        if (lo0 <= x && x <= hi0) x = hi0 + 1;
        if (lo1 <= x && x <= hi1) x = hi1 + 1;
        if (lo2 <= x && x <= hi2) x = hi2 + 1;
    }
    return x > c1;
}

// ---------------------------------------------------------------------------
// PTX wrappers (sm_80+ forms that sm_100a keeps: cp.async, ldmatrix, mma.sync)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid)
{
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t r[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t r[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Offset (in elements) of element (r, c) of a [rows][D] bf16 tile whose
// 16-byte chunks are XOR-swizzled by the row index, so that ldmatrix of 8
// consecutive rows at one column touches 8 distinct bank groups.
template <int D>
__device__ __forceinline__ int swz(int r, int c)
{
    return r * D + ((((c >> 3) ^ (r & 7))) << 3) + (c & 7);
}

// Copy a [rows][D] bf16 tile from global memory (row pointer stride in
// elements) into a swizzled shared tile; rows >= nvalid are zero-filled.
template <int D, int ROWS, int NTHREADS>
__device__ __forceinline__ void load_tile(__nv_bfloat16 *sm, const __nv_bfloat16 *g,
                                          long long row_stride, int nvalid, int tid)
{
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    constexpr int TOTAL = ROWS * CPR;
    const uint32_t base = smem_u32(sm);
#pragma unroll
    for (int it = 0; it < (TOTAL + NTHREADS - 1) / NTHREADS; ++it) {
        const int idx = it * NTHREADS + tid;
        if (TOTAL % NTHREADS == 0 || idx < TOTAL) {
            const int r = idx / CPR, ch = idx % CPR;
            const bool ok = r < nvalid;
            const __nv_bfloat16 *src = g + (ok ? (long long)r * row_stride : 0) + ch * 8;
            cp_async16(base + 2u * (uint32_t)swz<D>(r, ch * 8), src, ok);
        }
    }
}

}  // namespace cowa
