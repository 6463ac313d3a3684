// CoWA single-token decode: split-KV over the visible keys, then an
// LSE-weighted merge.
//
// The new token sits at p = seqlens[b] - 1 of its sequence.  The keys it sees
// under KV head h are at most three intervals (sink [0, S), near (p-N, p],
// long [p-e+1, p-c]); they are merged, cut into 64-key tiles that start at
// each interval's first key, and the tiles are shared out over `splits` CTAs
// per (batch, KV head).  Invisible keys are never read, which is where the
// decode saving of the paper's operator benchmark comes from.  The g query
// heads of the KV head share every K/V tile: they form the rows of a
// 16-row MMA block (rows g..15 are zero).  Each of the 4 warps owns 16 keys of
// a tile and keeps its own online-softmax state; the warps and then the
// splits are merged with their LSEs.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.cuh"

namespace cowa {

__device__ __forceinline__ float ex2d(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------- windowed cache --
// Keys a decode cache serving query positions [o, o + R) of one KV head must
// hold: sink [0, S), near [o-N+1, o+R-1] and long [o-e+1, o+R-1-c], clipped
// at 0, merged and stored back to back in ascending key order.  Every key
// interval a query in that range sees lies inside one stored interval (the
// stored intervals are separated by keys none of the queries sees).
struct WindowStore {
    TileRanges t;  // stored key intervals, ascending; row offsets 0, len0, len0 + len1
};

__device__ inline WindowStore window_store(int o, int R, const Win &w)
{
    int l0 = 0, h0 = 0, l1 = 0, h1 = 0, l2 = 0, h2 = 0;
    const long long top = (long long)o + R - 1;  // last query position served
    if (R > 0 && top >= 0) {
        if (w.S > 0) h0 = (int)min((long long)w.S, top + 1);
        if (w.N > 0) {
            l1 = (int)max(0ll, (long long)o - w.N + 1);
            h1 = (int)(top + 1);
        }
        if (w.e > w.c && top - w.c >= 0) {
            l2 = (int)max(0ll, (long long)o - w.e + 1);
            h2 = (int)(top - w.c + 1);
        }
    }
    WindowStore ws;
    ws.t = merge3(l0, h0, l1, h1, l2, h2);
    return ws;
}

// stored row of the keys [j, j + n), or -1 unless one stored interval holds them all
__device__ inline int window_row(const WindowStore &ws, int j, int n)
{
    const TileRanges &t = ws.t;
    if (t.n > 0 && j >= t.lo0 && j + n <= t.lo0 + t.len0) return j - t.lo0;
    if (t.n > 1 && j >= t.lo1 && j + n <= t.lo1 + t.len1) return t.len0 + (j - t.lo1);
    if (t.n > 2 && j >= t.lo2 && j + n <= t.lo2 + t.len2) return t.len0 + t.len1 + (j - t.lo2);
    return -1;
}

// key of stored row i, or -1 past the stored keys
__device__ inline int window_key(const WindowStore &ws, int i)
{
    const TileRanges &t = ws.t;
    if (i < 0) return -1;
    if (i < t.len0) return t.lo0 + i;
    i -= t.len0;
    if (i < t.len1) return t.lo1 + i;
    i -= t.len1;
    if (i < t.len2) return t.lo2 + i;
    return -1;
}

// The keys the query at position p sees (at most three merged intervals, in
// key units), each with the cache row of its first key and its tile count.
struct KeySpans {
    TileRanges t;
    int row0, row1, row2;  // cache row of each interval's first key
    int tiles0, tiles1, tiles2, total_tiles;
};

__device__ inline KeySpans decode_spans(int p, const Win &w)
{
    int l0 = 0, h0 = 0, l1 = 0, h1 = 0, l2 = 0, h2 = 0;
    if (p >= 0) {
        if (w.S > 0) h0 = min(w.S, p + 1);
        if (w.N > 0) {
            l1 = max(0, p - w.N + 1);
            h1 = p + 1;
        }
        if (w.e > w.c && p - w.c >= 0) {
            l2 = max(0, p - w.e + 1);
            h2 = p - w.c + 1;
        }
    }
    KeySpans ks;
    ks.t = merge3(l0, h0, l1, h1, l2, h2);
    ks.row0 = ks.t.lo0;
    ks.row1 = ks.t.lo1;
    ks.row2 = ks.t.lo2;
    ks.tiles0 = (ks.t.len0 + kDecBN - 1) / kDecBN;
    ks.tiles1 = (ks.t.len1 + kDecBN - 1) / kDecBN;
    ks.tiles2 = (ks.t.len2 + kDecBN - 1) / kDecBN;
    ks.total_tiles = ks.tiles0 + ks.tiles1 + ks.tiles2;
    return ks;
}

template <int D>
__global__ void __launch_bounds__(128) decode_split_kernel(const DecodeParams p)
{
    constexpr int BN = kDecBN, NT = 128, KS = D / 16, ND = D / 8, STAGES = 3;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __nv_bfloat16 *sK = reinterpret_cast<__nv_bfloat16 *>(smem_raw);   // [STAGES][BN][D]
    __nv_bfloat16 *sV = sK + STAGES * BN * D;                           // [STAGES][BN][D]
    __nv_bfloat16 *sQ = sV + STAGES * BN * D;                           // [16][D]
    // after the key loop the K/V stages are reused as the warp-merge scratch
    float *sRed = reinterpret_cast<float *>(smem_raw);

    // the merge kernel may be scheduled now; it waits for this grid to
    // complete before it reads any partial
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, hl = blockIdx.y, b = blockIdx.z;
    const int g = p.g;
    int seq = p.seqlens[b];
    const int org = p.origin ? p.origin[b] : 0;
    // never read outside the cache: a full cache holds keys [0, Lcap); a
    // windowed one serves query positions [origin, origin + horizon)
    const bool bad = p.origin ? (org < 0 || seq - 1 < org || seq - 1 >= org + p.horizon)
                              : (seq < 0 || seq > p.Lcap);
    if (bad) {
        if (tid == 0 && split == 0) atomicExch(p.err, 7);
        seq = 0;
    }
    const int pq = seq - 1;
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    KeySpans ks = decode_spans(pq, w);
    if (p.origin && !bad) {
        const WindowStore wst = window_store(org, p.horizon, w);
        bool held = true;
        if (ks.t.n > 0) {
            ks.row0 = window_row(wst, ks.t.lo0, ks.t.len0);
            held &= ks.row0 >= 0 && ks.row0 + ks.t.len0 <= p.Lcap;
        }
        if (ks.t.n > 1) {
            ks.row1 = window_row(wst, ks.t.lo1, ks.t.len1);
            held &= ks.row1 >= 0 && ks.row1 + ks.t.len1 <= p.Lcap;
        }
        if (ks.t.n > 2) {
            ks.row2 = window_row(wst, ks.t.lo2, ks.t.len2);
            held &= ks.row2 >= 0 && ks.row2 + ks.t.len2 <= p.Lcap;
        }
        if (!held) {  // cannot happen for positions in the horizon; read nothing
            if (tid == 0 && split == 0) atomicExch(p.err, 7);
            ks = decode_spans(-1, w);
        }
    }
    const int t_begin = (int)((long long)ks.total_tiles * split / p.splits);
    const int t_end = (int)((long long)ks.total_tiles * (split + 1) / p.splits);
    const int ntiles = t_end - t_begin;

    // tile index -> (first key, valid keys)
    auto tile_at = [&](int t, int &k0, int &nk) {  // cache row of the tile's first key, keys in it
        if (t < ks.tiles0) {
            k0 = ks.row0 + t * BN;
            nk = min(BN, ks.t.len0 - t * BN);
            return;
        }
        t -= ks.tiles0;
        if (t < ks.tiles1) {
            k0 = ks.row1 + t * BN;
            nk = min(BN, ks.t.len1 - t * BN);
            return;
        }
        t -= ks.tiles1;
        k0 = ks.row2 + t * BN;
        nk = min(BN, ks.t.len2 - t * BN);
    };

    const __nv_bfloat16 *kg = reinterpret_cast<const __nv_bfloat16 *>(p.kc) + b * p.ks[0] + hl * p.ks[2];
    const __nv_bfloat16 *vg = reinterpret_cast<const __nv_bfloat16 *>(p.vc) + b * p.vs[0] + hl * p.vs[2];
    auto load_kv = [&](int t, int stage) {
        int k0, nk;
        tile_at(t, k0, nk);
        if (!dcheck(k0 >= 0 && nk >= 0 && k0 + nk <= p.Lcap, p.err)) nk = 0;  // rows of the cache only
        load_tile<D, BN, NT>(sK + stage * BN * D, kg + (long long)k0 * p.ks[1], p.ks[1], nk, tid);
        load_tile<D, BN, NT>(sV + stage * BN * D, vg + (long long)k0 * p.vs[1], p.vs[1], nk, tid);
    };

    // query rows of this group (rows >= g are zero)
    const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(p.q) + b * p.qs[0] + (long long)hl * g * p.qs[2];
    load_tile<D, 16, NT>(sQ, qg, p.qs[2], g, tid);
    cp_async_commit();
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        if (s < ntiles) load_kv(t_begin + s, s);
        cp_async_commit();
    }

    cp_async_wait<STAGES - 1>();  // the query group
    __syncthreads();
    uint32_t qa[KS][4];
#pragma unroll
    for (int kk = 0; kk < KS; ++kk)
        ldsm_x4(qa[kk], smem_u32(sQ + swz<D>(lane & 15, kk * 16 + (lane >> 4) * 8)));

    float acc[ND][4];
#pragma unroll
    for (int n = 0; n < ND; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    float mx[2] = {-CUDART_INF_F, -CUDART_INF_F}, l[2] = {0.f, 0.f};
    const int kw = warp * 16;  // this warp's keys within a tile

    for (int t = 0; t < ntiles; ++t) {
        const int stage = t % STAGES;
        if (t + STAGES - 1 < ntiles) load_kv(t_begin + t + STAGES - 1, (t + STAGES - 1) % STAGES);
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        __syncthreads();
        int k0, nk;
        tile_at(t_begin + t, k0, nk);
        const __nv_bfloat16 *cK = sK + stage * BN * D;
        const __nv_bfloat16 *cV = sV + stage * BN * D;

        float s[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            uint32_t bf[4];
            const int key = kw + (lane & 7) + (lane >> 4) * 8;
            const int col = kk * 16 + ((lane >> 3) & 1) * 8;
            ldsm_x4(bf, smem_u32(cK + swz<D>(key, col)));
            mma16816(s[0], qa[kk], bf[0], bf[1]);
            mma16816(s[1], qa[kk], bf[2], bf[3]);
        }
        float tm[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int key = kw + n * 8 + (lane & 3) * 2 + (c & 1);
                const float x = key < nk ? s[n][c] * p.scale_log2 : -CUDART_INF_F;
                s[n][c] = x;
                tm[c >> 1] = fmaxf(tm[c >> 1], x);
            }
        float alpha[2], msafe[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            tm[r] = fmaxf(tm[r], __shfl_xor_sync(0xffffffffu, tm[r], 1));
            tm[r] = fmaxf(tm[r], __shfl_xor_sync(0xffffffffu, tm[r], 2));
            const float mnew = fmaxf(mx[r], tm[r]);
            msafe[r] = mnew == -CUDART_INF_F ? 0.f : mnew;
            alpha[r] = ex2d(mx[r] - msafe[r]);
            mx[r] = mnew;
            l[r] *= alpha[r];
        }
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float e = ex2d(s[n][c] - msafe[c >> 1]);
                s[n][c] = e;
                l[c >> 1] += e;
            }
#pragma unroll
        for (int n = 0; n < ND; ++n) {
            acc[n][0] *= alpha[0]; acc[n][1] *= alpha[0];
            acc[n][2] *= alpha[1]; acc[n][3] *= alpha[1];
        }
        uint32_t pa_[4];
        pa_[0] = pack_bf16(s[0][0], s[0][1]);
        pa_[1] = pack_bf16(s[0][2], s[0][3]);
        pa_[2] = pack_bf16(s[1][0], s[1][1]);
        pa_[3] = pack_bf16(s[1][2], s[1][3]);
#pragma unroll
        for (int d2 = 0; d2 < D / 16; ++d2) {
            uint32_t bf[4];
            const int key = kw + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int col = d2 * 16 + (lane >> 4) * 8;
            ldsm_x4_t(bf, smem_u32(cV + swz<D>(key, col)));
            mma16816(acc[2 * d2], pa_, bf[0], bf[1]);
            mma16816(acc[2 * d2 + 1], pa_, bf[2], bf[3]);
        }
        __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();

    // merge the four warps: rows 0..7 live in (lane>>2), c = 0,1 (row r = 0)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    }
    float *wm = sRed;              // [4][16] running max per warp and row
    float *wl = wm + 64;           // [4][16] sums
    float *wo = wl + 64;           // [4][16][D] unnormalised O (only rows < g used)
    if ((lane & 3) == 0) {
        const int row = lane >> 2;
        wm[warp * 16 + row] = mx[0];
        wl[warp * 16 + row] = l[0];
        wm[warp * 16 + row + 8] = mx[1];
        wl[warp * 16 + row + 8] = l[1];
    }
#pragma unroll
    for (int n = 0; n < ND; ++n) {
        const int col = n * 8 + (lane & 3) * 2;
        const int row = lane >> 2;
        wo[(warp * 16 + row) * D + col] = acc[n][0];
        wo[(warp * 16 + row) * D + col + 1] = acc[n][1];
        wo[(warp * 16 + row + 8) * D + col] = acc[n][2];
        wo[(warp * 16 + row + 8) * D + col + 1] = acc[n][3];
    }
    __syncthreads();
    const long long pbase = (((long long)b * p.Hq + (long long)hl * g) * p.splits + split);
    for (int idx = tid; idx < g * D; idx += NT) {
        const int row = idx / D, col = idx % D;
        float m = -CUDART_INF_F;
        for (int u = 0; u < 4; ++u) m = fmaxf(m, wm[u * 16 + row]);
        const float ms = m == -CUDART_INF_F ? 0.f : m;
        float lsum = 0.f, o = 0.f;
        for (int u = 0; u < 4; ++u) {
            const float f = ex2d(wm[u * 16 + row] - ms);
            lsum += f * wl[u * 16 + row];
            o += f * wo[(u * 16 + row) * D + col];
        }
        const long long pi = pbase + (long long)row * p.splits;
        if (!dcheck(pi < (long long)p.B * p.Hq * p.splits, p.err)) break;
        p.part_o[pi * D + col] = lsum > 0.f ? o / lsum : 0.f;
        if (col == 0)  // log2-domain LSE of this split
            p.part_lse[pi] = lsum > 0.f ? m + __log2f(lsum) : -CUDART_INF_F;
    }
}

template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p)
{
    // thread s < splits holds split s: the max and the weights are block
    // reductions, then every thread merges columns with the weights from
    // shared memory (splits <= 64)
    __shared__ float red[4], wsum[4], wt[64];
    // every partial of the split grid (the launch's programmatic
    // predecessor, or any earlier work when launched plainly) is complete
    // and visible past this point
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int row = blockIdx.x;  // b * Hq + hq
    const int b = row / p.Hq, hq = row % p.Hq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float *pl = p.part_lse + (long long)row * p.splits;
    const float *po = p.part_o + (long long)row * p.splits * D;
    const float lv = tid < p.splits ? pl[tid] : -CUDART_INF_F;
    float m = lv;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float ms = m == -CUDART_INF_F ? 0.f : m;
    const float wv = tid < p.splits ? ex2d(lv - ms) : 0.f;
    if (tid < 64) wt[tid] = wv;
    float l = wv;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) wsum[warp] = l;
    __syncthreads();
    const float lsum = (wsum[0] + wsum[1]) + (wsum[2] + wsum[3]);
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.o) + b * p.os[0] + hq * p.os[2];
    for (int col = tid; col < D; col += blockDim.x) {
        float acc = 0.f;
        for (int sp = 0; sp < p.splits; ++sp) acc += wt[sp] * po[(long long)sp * D + col];
        o[col] = __float2bfloat16_rn(lsum > 0.f ? acc / lsum : 0.f);
    }
    if (tid == 0) p.lse[row] = lsum > 0.f ? (m + __log2f(lsum)) * 0.69314718055994531f : -CUDART_INF_F;
}

// One thread per 16-byte piece of a row: row i of the windowed cache of
// (b, h) takes key j of the source when the cache holds j and j <= origin
// (a key the source has); other rows are zeroed (later appends fill them).
template <int D>
__global__ void __launch_bounds__(128) wcache_build_kernel(const WCacheParams p)
{
    constexpr int PIECES = D * 2 / 16, ROWS = 128 / PIECES;
    const int h = blockIdx.y, b = blockIdx.z;
    const int i = blockIdx.x * ROWS + threadIdx.x / PIECES, c = threadIdx.x % PIECES;
    if (i >= p.rows) return;
    const int o = p.origin[b];
    int j = -1;
    if (o >= 0 && o < p.Lsrc) {
        const WindowStore ws = window_store(o, p.horizon, make_win(p.S, p.N, p.G, p.W, (long long)h + p.kv_head_offset));
        j = window_key(ws, i);
        if (j > o) j = -1;  // a future key: appended later
    } else if (i == 0 && c == 0 && h == 0) {
        atomicExch(p.err, 7);
    }
    const long long dst = (((long long)b * p.rows + i) * p.Hkv + h) * D + c * 8;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
    if (j >= 0) {
        kv = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p.ksrc) + b * p.ks[0] +
                                              (long long)j * p.ks[1] + h * p.ks[2] + c * 8);
        vv = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p.vsrc) + b * p.vs[0] +
                                              (long long)j * p.vs[1] + h * p.vs[2] + c * 8);
    }
    *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.kw) + dst) = kv;
    *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.vw) + dst) = vv;
}

// The K/V row of the token at pos[b] (source [B, Hkv, d], strides b and h)
// goes to its row of every KV head's windowed cache that holds it; a
// position outside [origin, origin + horizon) is refused on the device.
template <int D>
__global__ void __launch_bounds__(128) wcache_append_kernel(const WCacheParams p)
{
    constexpr int PIECES = D * 2 / 16, HEADS = 128 / PIECES;
    const int b = blockIdx.y;
    const int h = blockIdx.x * HEADS + threadIdx.x / PIECES, c = threadIdx.x % PIECES;
    if (h >= p.Hkv) return;
    const int o = p.origin[b], j = p.pos[b];
    if (o < 0 || j < o || j >= o + p.horizon) {
        if (h == 0 && c == 0) atomicExch(p.err, 7);
        return;
    }
    const WindowStore ws = window_store(o, p.horizon, make_win(p.S, p.N, p.G, p.W, (long long)h + p.kv_head_offset));
    const int i = window_row(ws, j, 1);
    if (i < 0 || i >= p.rows) return;  // no query of the horizon sees key j through this head
    const long long dst = (((long long)b * p.rows + i) * p.Hkv + h) * D + c * 8;
    *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.kw) + dst) = *reinterpret_cast<const uint4 *>(
        reinterpret_cast<const __nv_bfloat16 *>(p.ksrc) + b * p.ks[0] + h * p.ks[2] + c * 8);
    *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.vw) + dst) = *reinterpret_cast<const uint4 *>(
        reinterpret_cast<const __nv_bfloat16 *>(p.vsrc) + b * p.vs[0] + h * p.vs[2] + c * 8);
}

template <int D>
static cudaError_t launch_wcache_build_d(const WCacheParams &p, cudaStream_t st)
{
    constexpr int ROWS = 128 / (D * 2 / 16);
    dim3 grid((p.rows + ROWS - 1) / ROWS, p.Hkv, p.B);
    launch_begin("wcache_build", st);
    wcache_build_kernel<D><<<grid, 128, 0, st>>>(p);
    launch_end(st);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_wcache_append_d(const WCacheParams &p, cudaStream_t st)
{
    constexpr int HEADS = 128 / (D * 2 / 16);
    dim3 grid((p.Hkv + HEADS - 1) / HEADS, p.B);
    launch_begin("wcache_append", st);
    wcache_append_kernel<D><<<grid, 128, 0, st>>>(p);
    launch_end(st);
    return cudaGetLastError();
}

cudaError_t launch_wcache_build(const WCacheParams &p, int D, cudaStream_t st)
{
    if (p.B == 0 || p.Hkv == 0 || p.rows == 0) return cudaSuccess;
    return D == 128 ? launch_wcache_build_d<128>(p, st) : launch_wcache_build_d<64>(p, st);
}

cudaError_t launch_wcache_append(const WCacheParams &p, int D, cudaStream_t st)
{
    if (p.B == 0 || p.Hkv == 0 || p.rows == 0) return cudaSuccess;
    return D == 128 ? launch_wcache_append_d<128>(p, st) : launch_wcache_append_d<64>(p, st);
}

template <int D>
static cudaError_t launch_decode_d(const DecodeParams &p, cudaStream_t st)
{
    constexpr int smem = decode_smem_bytes(D);
    static_assert((128 + 64 * D) * 4 <= 6 * kDecBN * D * 2, "merge scratch must fit the K/V stages");
    static std::atomic<bool> configured[64];
    cudaError_t e = once_per_device(configured, [] {
        return cudaFuncSetAttribute(decode_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (e != cudaSuccess) return e;
    dim3 grid(p.splits, p.Hkv, p.B);
    launch_begin("decode_split", st);
    decode_split_kernel<D><<<grid, 128, smem, st>>>(p);
    launch_end(st);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the merge is launched as a programmatic dependent of the split kernel:
    // its blocks are scheduled while the splits still run (the split kernel
    // allows it at its start) and wait on the device for the split grid to
    // complete, so the second launch adds no gap of its own
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.B * p.Hq));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    launch_begin("decode_combine", st);
    e = cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, p);
    launch_end(st);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams &p, int D, cudaStream_t st)
{
    if (p.B == 0 || p.Hq == 0) return cudaSuccess;
    return D == 128 ? launch_decode_d<128>(p, st) : launch_decode_d<64>(p, st);
}

}  // namespace cowa
