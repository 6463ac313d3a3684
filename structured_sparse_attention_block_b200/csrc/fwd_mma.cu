// CoWA training / prefill forward, warp-level MMA version.
//
// One CTA per (query tile of 128 rows, query head, batch); 8 warps, 16 rows
// each.  The CTA walks only the key tiles its schedule entry lists (the
// sink, near and long bands of its KV head), double-buffering K/V tiles in
// shared memory with cp.async, and keeps an online softmax in registers
// (running max and sum per row, O rescaled when the max grows).  Tiles that
// tile_full() proves fully visible skip the element mask.  Output: O in
// bf16 and the natural-log LSE in fp32.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.cuh"

namespace cowa {

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

template <int D>
__global__ void __launch_bounds__(256, 1) fwd_mma_kernel(const AttnParams p)
{
    constexpr int BM = kFwdBM, BN = kFwdBN, NT = 256, KS = D / 16, NB = BN / 8, ND = D / 8;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __nv_bfloat16 *sQ = reinterpret_cast<__nv_bfloat16 *>(smem_raw);
    __nv_bfloat16 *sK = sQ + BM * D;
    __nv_bfloat16 *sV = sK + 2 * BN * D;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = gridDim.x - 1 - blockIdx.x;  // long rows first
    const int hq = blockIdx.y, b = blockIdx.z;
    const int hl = hq / p.g;
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    const int delta = p.Lk - p.Lq;
    const int i0 = qt * BM;
    const int nrows = min(BM, p.Lq - i0);
    const int pa = i0 + delta, pb = i0 + nrows - 1 + delta;

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
    const __nv_bfloat16 *kg = reinterpret_cast<const __nv_bfloat16 *>(p.k) + b * p.ks[0] + hl * p.ks[2];
    const __nv_bfloat16 *vg = reinterpret_cast<const __nv_bfloat16 *>(p.v) + b * p.vs[0] + hl * p.vs[2];

    auto load_kv = [&](int kt, int buf) {
        const int nvalid = min(BN, p.Lk - kt * BN);
        load_tile<D, BN, NT>(sK + buf * BN * D, kg + (long long)kt * BN * p.ks[1], p.ks[1], nvalid, tid);
        load_tile<D, BN, NT>(sV + buf * BN * D, vg + (long long)kt * BN * p.vs[1], p.vs[1], nvalid, tid);
    };

    load_tile<D, BM, NT>(sQ, qg, p.qs[1], nrows, tid);
    cp_async_commit();
    if (ntiles > 0) load_kv(tile_of(0), 0);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int r0 = warp * 16;
    uint32_t qa[KS][4];
#pragma unroll
    for (int kk = 0; kk < KS; ++kk)
        ldsm_x4(qa[kk], smem_u32(sQ + swz<D>(r0 + (lane & 15), kk * 16 + (lane >> 4) * 8)));

    float acc[ND][4];
#pragma unroll
    for (int n = 0; n < ND; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    float mx[2] = {-CUDART_INF_F, -CUDART_INF_F}, l[2] = {0.f, 0.f};
    const int prow0 = pa + r0 + (lane >> 2);  // aligned position of this thread's first row

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

        float s[NB][4];
#pragma unroll
        for (int n = 0; n < NB; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk)
#pragma unroll
            for (int n2 = 0; n2 < NB / 2; ++n2) {
                uint32_t bf[4];
                const int key = n2 * 16 + (lane & 7) + (lane >> 4) * 8;
                const int col = kk * 16 + ((lane >> 3) & 1) * 8;
                ldsm_x4(bf, smem_u32(cK + swz<D>(key, col)));
                mma16816(s[2 * n2], qa[kk], bf[0], bf[1]);
                mma16816(s[2 * n2 + 1], qa[kk], bf[2], bf[3]);
            }

        const bool full = tile_full(pa, pb, kt * BN, BN, p.Lk, w);
        float tm[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
        for (int n = 0; n < NB; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float x = s[n][c] * p.scale_log2;
                if (!full) {
                    const int prow = prow0 + (c >> 1) * 8;
                    const int j = kt * BN + n * 8 + (lane & 3) * 2 + (c & 1);
                    if (!visible(prow, j, w)) x = -CUDART_INF_F;
                }
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
            alpha[r] = ex2(mx[r] - msafe[r]);
            mx[r] = mnew;
            l[r] *= alpha[r];
        }
#pragma unroll
        for (int n = 0; n < NB; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float e = ex2(s[n][c] - msafe[c >> 1]);
                s[n][c] = e;
                l[c >> 1] += e;
            }
#pragma unroll
        for (int n = 0; n < ND; ++n) {
            acc[n][0] *= alpha[0]; acc[n][1] *= alpha[0];
            acc[n][2] *= alpha[1]; acc[n][3] *= alpha[1];
        }
#pragma unroll
        for (int k2 = 0; k2 < BN / 16; ++k2) {
            uint32_t pa_[4];
            pa_[0] = pack_bf16(s[2 * k2][0], s[2 * k2][1]);
            pa_[1] = pack_bf16(s[2 * k2][2], s[2 * k2][3]);
            pa_[2] = pack_bf16(s[2 * k2 + 1][0], s[2 * k2 + 1][1]);
            pa_[3] = pack_bf16(s[2 * k2 + 1][2], s[2 * k2 + 1][3]);
#pragma unroll
            for (int d2 = 0; d2 < D / 16; ++d2) {
                uint32_t bf[4];
                const int key = k2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = d2 * 16 + (lane >> 4) * 8;
                ldsm_x4_t(bf, smem_u32(cV + swz<D>(key, col)));
                mma16816(acc[2 * d2], pa_, bf[0], bf[1]);
                mma16816(acc[2 * d2 + 1], pa_, bf[2], bf[3]);
            }
        }
        __syncthreads();
    }

    // epilogue
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    }
    __nv_bfloat16 *og = reinterpret_cast<__nv_bfloat16 *>(p.o) + b * p.os[0] + hq * p.os[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = r0 + (lane >> 2) + r * 8;
        const int i = i0 + row;
        if (row >= nrows) continue;
        const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
        __nv_bfloat16 *orow = og + (long long)i * p.os[1];
#pragma unroll
        for (int n = 0; n < ND; ++n) {
            const int col = n * 8 + (lane & 3) * 2;
            *reinterpret_cast<uint32_t *>(orow + col) =
                pack_bf16(acc[n][2 * r] * inv, acc[n][2 * r + 1] * inv);
        }
        if ((lane & 3) == 0)
            p.lse[((long long)b * p.Hq + hq) * p.Lq + i] =
                l[r] > 0.f ? mx[r] * 0.69314718055994531f + logf(l[r]) : -CUDART_INF_F;
    }
}

template <int D>
static cudaError_t launch_fwd_d(const AttnParams &p, cudaStream_t st)
{
    constexpr int smem = (kFwdBM * D + 4 * kFwdBN * D) * 2;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(fwd_mma_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured[dev & 63] = true;
    }
    dim3 grid(p.nqt, p.Hq, p.B);
    launch_begin("fwd_mma", st);
    fwd_mma_kernel<D><<<grid, 256, smem, st>>>(p);
    launch_end(st);
    return cudaGetLastError();
}

cudaError_t launch_fwd_mma(const AttnParams &p, int D, cudaStream_t st)
{
    if (p.nqt == 0 || p.Hq == 0 || p.B == 0) return cudaSuccess;
    return D == 128 ? launch_fwd_d<128>(p, st) : launch_fwd_d<64>(p, st);
}

}  // namespace cowa
