// CoWA training backward, warp-level MMA version.
//
// Three kernels on the caller's stream:
//  1. delta[b, hq, i] = sum_x dO[b, i, hq, x] * O[b, i, hq, x] (fp32).
//  2. dK/dV pass, key-tile major: one CTA per (key tile of 64, KV head,
//     batch), 4 warps of 16 keys.  It walks the query tiles of the key-tile
//     major schedule for each of the g query heads of its KV head,
//     recomputes S^T = K Q^T, P^T = exp(scale*S^T - LSE), dP^T = V dO^T,
//     dS^T = P^T (dP^T - delta), and accumulates dV += P^T dO and
//     dK += dS^T Q in registers; dK is scaled by softmax_scale at the end.
//  3. dQ pass, query-tile major: one CTA per (query tile of 64, query head,
//     batch) over the same key tiles the forward visits; dQ += dS K.
// Each output element has one writer, so the result is deterministic.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.cuh"

namespace cowa {

__device__ __forceinline__ float ex2b(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------- delta ----
template <int D>
__global__ void delta_kernel(const AttnParams p)
{
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const long long total = (long long)p.B * p.Hq * p.Lq;
    if (row >= total) return;
    const int i = (int)(row % p.Lq);
    const int hq = (int)((row / p.Lq) % p.Hq);
    const int b = (int)(row / ((long long)p.Lq * p.Hq));
    const __nv_bfloat16 *o = reinterpret_cast<const __nv_bfloat16 *>(p.o) + b * p.os[0] +
                             (long long)i * p.os[1] + hq * p.os[2];
    const __nv_bfloat16 *dout = reinterpret_cast<const __nv_bfloat16 *>(p.dout) + b * p.os[0] +
                                (long long)i * p.os[1] + hq * p.os[2];
    constexpr int PER = D / 32;
    float s = 0.f;
#pragma unroll
    for (int x = 0; x < PER; x += 2) {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(o + lane * PER + x);
        const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162 *>(dout + lane * PER + x);
        s += __bfloat162float(a.x) * __bfloat162float(c.x) + __bfloat162float(a.y) * __bfloat162float(c.y);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) p.delta[((long long)b * p.Hq + hq) * p.Lq + i] = s;
}

// ----------------------------------------------------------- dK / dV ----
// QB: query rows per inner step (the key-tile-major schedule's BM).
template <int D, int QB>
__global__ void __launch_bounds__(128) dkdv_mma_kernel(const AttnParams p)
{
    constexpr int BN = kBwdBN, NT = 128, KS = D / 16, NQ = QB / 8, ND = D / 8;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __nv_bfloat16 *sK = reinterpret_cast<__nv_bfloat16 *>(smem_raw);
    __nv_bfloat16 *sV = sK + BN * D;
    __nv_bfloat16 *sQ = sV + BN * D;          // [2][QB][D]
    __nv_bfloat16 *sdO = sQ + 2 * QB * D;     // [2][QB][D]
    float *sL = reinterpret_cast<float *>(sdO + 2 * QB * D);  // [2][QB] LSE*log2e
    float *sDl = sL + 2 * QB;                                  // [2][QB] delta

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kt = blockIdx.x, hl = blockIdx.y, b = blockIdx.z;
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    const int delta_pos = p.Lk - p.Lq;
    const int c0 = kt * BN;
    const int ncols = min(BN, p.Lk - c0);

    const int4 *e4 = reinterpret_cast<const int4 *>(p.sched_t + ((size_t)hl * p.nkt + kt) * kSchedInts);
    const int4 e0 = e4[0], e1 = e4[1];
    const int nr = e0.x;
    const int lo[3] = {e0.y, e0.w, e1.y};
    const int len[3] = {e0.z - e0.y, e1.x - e0.w, e1.z - e1.y};
    int nq = 0;
    for (int r = 0; r < nr; ++r) nq += len[r];
    const int ntask = nq * p.g;
    auto task = [&](int t, int &hq, int &qt) {
        hq = hl * p.g + t / nq;
        int u = t % nq, r = 0;
        while (r < nr - 1 && u >= len[r]) { u -= len[r]; ++r; }
        qt = lo[r] + u;
    };

    const __nv_bfloat16 *kg = reinterpret_cast<const __nv_bfloat16 *>(p.k) + b * p.ks[0] +
                              (long long)c0 * p.ks[1] + hl * p.ks[2];
    const __nv_bfloat16 *vg = reinterpret_cast<const __nv_bfloat16 *>(p.v) + b * p.vs[0] +
                              (long long)c0 * p.vs[1] + hl * p.vs[2];
    load_tile<D, BN, NT>(sK, kg, p.ks[1], ncols, tid);
    load_tile<D, BN, NT>(sV, vg, p.vs[1], ncols, tid);
    cp_async_commit();

    auto load_q = [&](int t, int buf) {
        int hq, qt;
        task(t, hq, qt);
        const int i0 = qt * QB;
        const int nrows = min(QB, p.Lq - i0);
        const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(p.q) + b * p.qs[0] +
                                  (long long)i0 * p.qs[1] + hq * p.qs[2];
        const __nv_bfloat16 *dg = reinterpret_cast<const __nv_bfloat16 *>(p.dout) + b * p.os[0] +
                                  (long long)i0 * p.os[1] + hq * p.os[2];
        load_tile<D, QB, NT>(sQ + buf * QB * D, qg, p.qs[1], nrows, tid);
        load_tile<D, QB, NT>(sdO + buf * QB * D, dg, p.os[1], nrows, tid);
        const long long rb = ((long long)b * p.Hq + hq) * p.Lq + i0;
        for (int r = tid; r < QB; r += NT) {
            const bool ok = r < nrows;
            const float lv = ok ? p.lse_in[rb + r] : 0.f;
            sL[buf * QB + r] = lv == -CUDART_INF_F ? CUDART_INF_F : lv * 1.4426950408889634f;
            sDl[buf * QB + r] = ok ? p.delta[rb + r] : 0.f;
        }
    };

    float dk[ND][4], dv[ND][4];
#pragma unroll
    for (int n = 0; n < ND; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) dk[n][c] = dv[n][c] = 0.f;

    const int k0 = warp * 16;  // this warp's keys within the tile
    if (ntask > 0) {
        load_q(0, 0);
        cp_async_commit();
    }
    for (int t = 0; t < ntask; ++t) {
        const int buf = t & 1;
        int hq, qt;
        task(t, hq, qt);
        (void)hq;
        __syncthreads();  // buffer buf^1 free (previous compute done) / LSE writes visible below
        if (t + 1 < ntask) {
            load_q(t + 1, buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const __nv_bfloat16 *cQ = sQ + buf * QB * D;
        const __nv_bfloat16 *cdO = sdO + buf * QB * D;
        const float *cL = sL + buf * QB;
        const float *cDl = sDl + buf * QB;
        const int i0 = qt * QB;
        const int nrows = min(QB, p.Lq - i0);
        const bool full = tile_full(i0 + delta_pos, i0 + nrows - 1 + delta_pos, c0, BN, p.Lk, w);

        // S^T and dP^T: rows = this warp's 16 keys, cols = QB queries
        float st[NQ][4], dpt[NQ][4];
#pragma unroll
        for (int n = 0; n < NQ; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) st[n][c] = dpt[n][c] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            uint32_t ka[4], va[4];
            ldsm_x4(ka, smem_u32(sK + swz<D>(k0 + (lane & 15), kk * 16 + (lane >> 4) * 8)));
            ldsm_x4(va, smem_u32(sV + swz<D>(k0 + (lane & 15), kk * 16 + (lane >> 4) * 8)));
#pragma unroll
            for (int n2 = 0; n2 < NQ / 2; ++n2) {
                uint32_t qb[4], db[4];
                const int qr = n2 * 16 + (lane & 7) + (lane >> 4) * 8;
                const int col = kk * 16 + ((lane >> 3) & 1) * 8;
                ldsm_x4(qb, smem_u32(cQ + swz<D>(qr, col)));
                ldsm_x4(db, smem_u32(cdO + swz<D>(qr, col)));
                mma16816(st[2 * n2], ka, qb[0], qb[1]);
                mma16816(st[2 * n2 + 1], ka, qb[2], qb[3]);
                mma16816(dpt[2 * n2], va, db[0], db[1]);
                mma16816(dpt[2 * n2 + 1], va, db[2], db[3]);
            }
        }
        // P^T and dS^T
#pragma unroll
        for (int n = 0; n < NQ; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int qc = n * 8 + (lane & 3) * 2 + (c & 1);  // query within tile
                const int key = c0 + k0 + (lane >> 2) + (c >> 1) * 8;
                float pr = ex2b(st[n][c] * p.scale_log2 - cL[qc]);
                if (!full && !visible(i0 + qc + delta_pos, key, w)) pr = 0.f;
                if (qc >= nrows) pr = 0.f;
                st[n][c] = pr;
                dpt[n][c] = pr * (dpt[n][c] - cDl[qc]);
            }
        // dV += P^T dO ; dK += dS^T Q   (K-dim = queries)
#pragma unroll
        for (int k2 = 0; k2 < QB / 16; ++k2) {
            uint32_t pa_[4], sa[4];
            pa_[0] = pack_bf16(st[2 * k2][0], st[2 * k2][1]);
            pa_[1] = pack_bf16(st[2 * k2][2], st[2 * k2][3]);
            pa_[2] = pack_bf16(st[2 * k2 + 1][0], st[2 * k2 + 1][1]);
            pa_[3] = pack_bf16(st[2 * k2 + 1][2], st[2 * k2 + 1][3]);
            sa[0] = pack_bf16(dpt[2 * k2][0], dpt[2 * k2][1]);
            sa[1] = pack_bf16(dpt[2 * k2][2], dpt[2 * k2][3]);
            sa[2] = pack_bf16(dpt[2 * k2 + 1][0], dpt[2 * k2 + 1][1]);
            sa[3] = pack_bf16(dpt[2 * k2 + 1][2], dpt[2 * k2 + 1][3]);
#pragma unroll
            for (int d2 = 0; d2 < D / 16; ++d2) {
                uint32_t db[4], qb[4];
                const int qr = k2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = d2 * 16 + (lane >> 4) * 8;
                ldsm_x4_t(db, smem_u32(cdO + swz<D>(qr, col)));
                ldsm_x4_t(qb, smem_u32(cQ + swz<D>(qr, col)));
                mma16816(dv[2 * d2], pa_, db[0], db[1]);
                mma16816(dv[2 * d2 + 1], pa_, db[2], db[3]);
                mma16816(dk[2 * d2], sa, qb[0], qb[1]);
                mma16816(dk[2 * d2 + 1], sa, qb[2], qb[3]);
            }
        }
    }

    cp_async_wait<0>();  // the K/V group is still pending when no query tile sees this key tile

    // epilogue: rows = keys
    __nv_bfloat16 *dkg = reinterpret_cast<__nv_bfloat16 *>(p.dk) + b * p.ks[0] + hl * p.ks[2];
    __nv_bfloat16 *dvg = reinterpret_cast<__nv_bfloat16 *>(p.dv) + b * p.vs[0] + hl * p.vs[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int key = k0 + (lane >> 2) + r * 8;
        if (key >= ncols) continue;
        const long long j = c0 + key;
#pragma unroll
        for (int n = 0; n < ND; ++n) {
            const int col = n * 8 + (lane & 3) * 2;
            *reinterpret_cast<uint32_t *>(dkg + j * p.ks[1] + col) =
                pack_bf16(dk[n][2 * r] * p.scale, dk[n][2 * r + 1] * p.scale);
            *reinterpret_cast<uint32_t *>(dvg + j * p.vs[1] + col) =
                pack_bf16(dv[n][2 * r], dv[n][2 * r + 1]);
        }
    }
}

// ------------------------------------------------------------------ dQ ----
template <int D>
__global__ void __launch_bounds__(128) dq_mma_kernel(const AttnParams p)
{
    constexpr int BM = kBwdBM, BN = kBwdBN, NT = 128, KS = D / 16, NB = BN / 8, ND = D / 8;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __nv_bfloat16 *sQ = reinterpret_cast<__nv_bfloat16 *>(smem_raw);
    __nv_bfloat16 *sdO = sQ + BM * D;
    __nv_bfloat16 *sK = sdO + BM * D;   // [2][BN][D]
    __nv_bfloat16 *sV = sK + 2 * BN * D;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = gridDim.x - 1 - blockIdx.x;
    const int hq = blockIdx.y, b = blockIdx.z;
    const int hl = hq / p.g;
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    const int delta_pos = p.Lk - p.Lq;
    const int i0 = qt * BM;
    const int nrows = min(BM, p.Lq - i0);
    const int pa = i0 + delta_pos, pb = i0 + nrows - 1 + delta_pos;

    const int4 *e4 = reinterpret_cast<const int4 *>(p.sched + ((size_t)hl * p.nqt + qt) * kSchedInts);
    const int4 e0 = e4[0], e1 = e4[1];
    const int nr = e0.x;
    const int lo[3] = {e0.y, e0.w, e1.y};
    const int len[3] = {e0.z - e0.y, e1.x - e0.w, e1.z - e1.y};
    int ntiles = 0;
    for (int r = 0; r < nr; ++r) ntiles += len[r];
    auto tile_of = [&](int t) {
        int r = 0;
        while (r < nr - 1 && t >= len[r]) { t -= len[r]; ++r; }
        return lo[r] + t;
    };

    const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(p.q) + b * p.qs[0] +
                              (long long)i0 * p.qs[1] + hq * p.qs[2];
    const __nv_bfloat16 *dg = reinterpret_cast<const __nv_bfloat16 *>(p.dout) + b * p.os[0] +
                              (long long)i0 * p.os[1] + hq * p.os[2];
    const __nv_bfloat16 *kg = reinterpret_cast<const __nv_bfloat16 *>(p.k) + b * p.ks[0] + hl * p.ks[2];
    const __nv_bfloat16 *vg = reinterpret_cast<const __nv_bfloat16 *>(p.v) + b * p.vs[0] + hl * p.vs[2];
    auto load_kv = [&](int kt, int buf) {
        const int nvalid = min(BN, p.Lk - kt * BN);
        load_tile<D, BN, NT>(sK + buf * BN * D, kg + (long long)kt * BN * p.ks[1], p.ks[1], nvalid, tid);
        load_tile<D, BN, NT>(sV + buf * BN * D, vg + (long long)kt * BN * p.vs[1], p.vs[1], nvalid, tid);
    };
    load_tile<D, BM, NT>(sQ, qg, p.qs[1], nrows, tid);
    load_tile<D, BM, NT>(sdO, dg, p.os[1], nrows, tid);
    cp_async_commit();
    if (ntiles > 0) load_kv(tile_of(0), 0);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int r0 = warp * 16;
    uint32_t qa[KS][4], da[KS][4];
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        ldsm_x4(qa[kk], smem_u32(sQ + swz<D>(r0 + (lane & 15), kk * 16 + (lane >> 4) * 8)));
        ldsm_x4(da[kk], smem_u32(sdO + swz<D>(r0 + (lane & 15), kk * 16 + (lane >> 4) * 8)));
    }
    float lrow[2], drow[2];
    const long long rb = ((long long)b * p.Hq + hq) * p.Lq;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = r0 + (lane >> 2) + r * 8;
        const bool ok = row < nrows;
        const float lv = ok ? p.lse_in[rb + i0 + row] : -CUDART_INF_F;
        lrow[r] = lv == -CUDART_INF_F ? CUDART_INF_F : lv * 1.4426950408889634f;
        drow[r] = ok ? p.delta[rb + i0 + row] : 0.f;
    }
    const int prow0 = pa + r0 + (lane >> 2);

    float acc[ND][4];
#pragma unroll
    for (int n = 0; n < ND; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

    for (int t = 0; t < ntiles; ++t) {
        const int buf = t & 1;
        const int kt = tile_of(t);
        if (t + 1 < ntiles) {
            load_kv(tile_of(t + 1), buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const __nv_bfloat16 *cK = sK + buf * BN * D;
        const __nv_bfloat16 *cV = sV + buf * BN * D;
        float s[NB][4], dp[NB][4];
#pragma unroll
        for (int n = 0; n < NB; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[n][c] = dp[n][c] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk)
#pragma unroll
            for (int n2 = 0; n2 < NB / 2; ++n2) {
                uint32_t kb[4], vb[4];
                const int key = n2 * 16 + (lane & 7) + (lane >> 4) * 8;
                const int col = kk * 16 + ((lane >> 3) & 1) * 8;
                ldsm_x4(kb, smem_u32(cK + swz<D>(key, col)));
                ldsm_x4(vb, smem_u32(cV + swz<D>(key, col)));
                mma16816(s[2 * n2], qa[kk], kb[0], kb[1]);
                mma16816(s[2 * n2 + 1], qa[kk], kb[2], kb[3]);
                mma16816(dp[2 * n2], da[kk], vb[0], vb[1]);
                mma16816(dp[2 * n2 + 1], da[kk], vb[2], vb[3]);
            }
        const bool full = tile_full(pa, pb, kt * BN, BN, p.Lk, w);
#pragma unroll
        for (int n = 0; n < NB; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int r = c >> 1;
                float pr = ex2b(s[n][c] * p.scale_log2 - lrow[r]);
                if (!full) {
                    const int j = kt * BN + n * 8 + (lane & 3) * 2 + (c & 1);
                    if (!visible(prow0 + r * 8, j, w)) pr = 0.f;
                }
                s[n][c] = pr * (dp[n][c] - drow[r]);  // dS
            }
#pragma unroll
        for (int k2 = 0; k2 < BN / 16; ++k2) {
            uint32_t sa[4];
            sa[0] = pack_bf16(s[2 * k2][0], s[2 * k2][1]);
            sa[1] = pack_bf16(s[2 * k2][2], s[2 * k2][3]);
            sa[2] = pack_bf16(s[2 * k2 + 1][0], s[2 * k2 + 1][1]);
            sa[3] = pack_bf16(s[2 * k2 + 1][2], s[2 * k2 + 1][3]);
#pragma unroll
            for (int d2 = 0; d2 < D / 16; ++d2) {
                uint32_t kb[4];
                const int key = k2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = d2 * 16 + (lane >> 4) * 8;
                ldsm_x4_t(kb, smem_u32(cK + swz<D>(key, col)));
                mma16816(acc[2 * d2], sa, kb[0], kb[1]);
                mma16816(acc[2 * d2 + 1], sa, kb[2], kb[3]);
            }
        }
        __syncthreads();
    }

    __nv_bfloat16 *dqg = reinterpret_cast<__nv_bfloat16 *>(p.dq) + b * p.qs[0] + hq * p.qs[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = r0 + (lane >> 2) + r * 8;
        if (row >= nrows) continue;
        __nv_bfloat16 *drow_p = dqg + (long long)(i0 + row) * p.qs[1];
#pragma unroll
        for (int n = 0; n < ND; ++n) {
            const int col = n * 8 + (lane & 3) * 2;
            *reinterpret_cast<uint32_t *>(drow_p + col) =
                pack_bf16(acc[n][2 * r] * p.scale, acc[n][2 * r + 1] * p.scale);
        }
    }
}

// ------------------------------------------------------------ launcher ----
template <int D>
static cudaError_t launch_bwd_d(const AttnParams &p, cudaStream_t st)
{
    constexpr int QB = D == 128 ? 32 : 64;
    constexpr int smem_kv = (2 * kBwdBN * D + 4 * QB * D) * 2 + 4 * QB * 4;
    constexpr int smem_q = (2 * kBwdBM * D + 4 * kBwdBN * D) * 2;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(dkdv_mma_kernel<D, QB>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(dq_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
        if (e != cudaSuccess) return e;
        configured[dev & 63] = true;
    }
    const long long rows = (long long)p.B * p.Hq * p.Lq;
    if (rows > 0) {
        launch_begin("delta_mma", st);
        delta_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p);
        launch_end(st);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.nkt > 0) {
        dim3 g1(p.nkt, p.Hkv, p.B);
        launch_begin("dkdv_mma", st);
        dkdv_mma_kernel<D, QB><<<g1, 128, smem_kv, st>>>(p);
        launch_end(st);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int nqt = (p.Lq + kBwdBM - 1) / kBwdBM;
    if (nqt > 0) {
        dim3 g2(nqt, p.Hq, p.B);
        launch_begin("dq_mma", st);
        dq_mma_kernel<D><<<g2, 128, smem_q, st>>>(p);
        launch_end(st);
        e = cudaGetLastError();
    }
    return e;
}

cudaError_t launch_bwd_mma(const AttnParams &p, int D, cudaStream_t st)
{
    if (p.B == 0 || p.Hq == 0) return cudaSuccess;
    return D == 128 ? launch_bwd_d<128>(p, st) : launch_bwd_d<64>(p, st);
}

}  // namespace cowa
