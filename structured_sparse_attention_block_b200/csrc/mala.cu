// MassAlloc Attention (MALA) forward on the 5th-generation tensor cores, d = 64
// (d = 128 runs the kernel of mala_d128.cu: two heads per CTA, 128-key tiles).
//
// "Two new attention models slash redundancy..." (first section) and the
// abstract of "CoWindow Attention: Full Causal Coverage Is a Collective
// Property" describe MALA as keeping the full causal QK scoring and letting
// attention's own softmax statistics decide where the rest of a block's work
// is skipped.  The reading this library fixes (the pages give no rule):
//   scores on every causal pair (bottom-right alignment); the softmax
//   statistics of each row over all of its causal keys (LSE); per block of
//   kMalaBM query rows x kMalaBN keys of one head, the mass each row gives
//   the block, sum_j P_ij; the block is kept when some row gives it at least
//   tau, and only kept blocks contribute to O = sum_j P_ij v_j, with P taken
//   against the full LSE (the dropped mass is not redistributed).
//
// One CTA per (query tile of 128 rows, query head, batch), two passes over
// the causal key tiles (64 keys):
//   pass 1: S = Q K^T into tensor memory, the softmax warps fold each row's
//           max and exp-sum online -> LSE;
//   pass 2: S again; P = 2^(S*scale*log2e - LSE*log2e) in fp32, the row's
//           mass in the tile, the largest mass over the 128 rows (warp
//           shuffles, then the four warps through shared memory) decides
//           the tile; a kept tile's P (bf16) goes to tensor memory and
//           O += P V runs, a skipped tile issues no PV MMA.
// The decisions are written to keep[b][hq][query tile][key tile] (1 kept,
// 0 skipped or beyond the causal diagonal) for the backward.
// Warps: 0-7 softmax, two warpgroups on every tile, warpgroup x on key
// columns [32x, 32x + 32) of each 64-key tile (thread = query row): pass 1
// keeps a max and exp-sum per half and merges the halves once at its end;
// pass 2 adds the two halves' row masses through shared memory before the
// decision; 8 TMA producer, 9 MMA issuer.
// Tensor memory: S in two 64-column buffers (pass item i in buffer i % 2, so
// S of the next tile is computed while the current one is read), P in two
// 32-column buffers (tile t in buffer t % 2), O (d columns).  Every mbarrier
// wait is bounded and reports a timeout through the error word.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace cowa {

using namespace sm100;

struct MalaArgs {
    CUtensorMap tq, tk, tv;
    AttnParams p;
    uint8_t *keep;  // [B, Hq, nqt, nkt] decisions
    float tau;
};

template <int D>
struct MalaCfg {
    static constexpr int BM = kMalaBM, BN = kMalaBN;
    static constexpr int ST = 4;
    static constexpr int KB = D / 64;
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int T_S = 0, T_P = 2 * BN, T_O = 3 * BN;  // S x2, P x2 (BN/2 each), O
    static_assert(T_O + D <= 512, "tensor-memory plan");
    static constexpr int NBAR = 10 + 2 * ST;
    static constexpr int SMEM = 1024 + Q_BYTES + ST * STAGE_BYTES + 8 * NBAR + 16 + 64 + 2048 + 1024;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
    static constexpr uint32_t IDESC_O = idesc_bf16(128, D, 0, 1);
};

template <int D>
__global__ void __launch_bounds__(320, 1) mala_fwd_kernel(const __grid_constant__ MalaArgs a)
{
    using C = MalaCfg<D>;
    constexpr int BM = C::BM, BN = C::BN, ST = C::ST, KB = C::KB;
    const AttnParams &p = a.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const uint32_t sQ = base, sStage = base + C::Q_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::Q_BYTES + ST * C::STAGE_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *kflag = reinterpret_cast<volatile int *>(tmem_slot + 2);  // [2] decision of tile t in t % 2
    float *red = reinterpret_cast<float *>(tmem_slot + 4);                  // [2][8] per-warp largest mass
    float *half = red + 16;                                                 // [2][2][128] row mass per half
    float2 *stat = reinterpret_cast<float2 *>(half + 512);                  // [128] (max, sum) of columns 32..63
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t BAR_Q = bar0;
    auto KV_FULL = [&](int s) { return bar0 + 8u * (1 + s); };
    auto KV_EMPTY = [&](int s) { return bar0 + 8u * (1 + ST + s); };
    auto S_FULL = [&](int x) { return bar0 + 8u * (1 + 2 * ST + x); };
    auto S_FREE = [&](int x) { return bar0 + 8u * (3 + 2 * ST + x); };
    auto P_FULL = [&](int y) { return bar0 + 8u * (5 + 2 * ST + y); };
    auto P_DONE = [&](int y) { return bar0 + 8u * (7 + 2 * ST + y); };
    const uint32_t FIN = bar0 + 8u * (9 + 2 * ST);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const TilePos pos = tile_pos(p.Hq, p.B);
    const int qt = p.nqt - 1 - pos.step;  // long rows first
    const int hq = pos.slot, hl = hq / p.g, b = pos.b;
    const int i0 = qt * BM;
    const int delta = p.Lk - p.Lq;
    const int nrows = min(BM, p.Lq - i0);
    const int pa = i0 + delta, pb = i0 + nrows - 1 + delta;
    // causal key tiles of the query tile: 0 .. pb / BN, within the keys
    const int nt = pb < 0 ? 0 : min(pb / BN + 1, p.nkt);

    if (tid == 0) {
        mbar_init(BAR_Q, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(KV_FULL(s), 1);
            mbar_init(KV_EMPTY(s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(S_FULL(x), 1);
            mbar_init(S_FREE(x), 8);  // one arrival per softmax warp
            mbar_init(P_FULL(x), 8);  // one arrival per softmax warp
            mbar_init(P_DONE(x), 1);
        }
        mbar_init(FIN, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 9) {
        tmem_alloc(smem_addr(tmem_slot), 512);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&a.tq);
        prefetch_tmap(&a.tk);
        prefetch_tmap(&a.tv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nitems = 2 * nt;  // pass 1 tiles, then pass 2 tiles

    if (warp == 8) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            mbar_expect_tx(BAR_Q, C::Q_BYTES);
            for (int kb = 0; kb < KB; ++kb) tma_load_4d(sQ + kb * BM * 128, &a.tq, BAR_Q, kb * 64, i0, hq, b);
            int issued = 0;
            for (int i = 0; i < nitems; ++i) {
                const int s = i % ST;
                if (i >= ST && !mbar_wait(KV_EMPTY(s), ((i / ST) - 1) & 1, p.err, abort_flag)) break;
                const bool second = i >= nt;
                const int kt = second ? i - nt : i;
                if (!dcheck(kt * BN < p.Lk, p.err)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_expect_tx(KV_FULL(s), second ? 2 * C::KV_BYTES : C::KV_BYTES);
                const uint32_t sk = sStage + s * C::STAGE_BYTES, sv = sk + C::KV_BYTES;
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(sk + kb * BN * 128, &a.tk, KV_FULL(s), kb * 64, kt * BN, hl, b);
                    if (second) tma_load_4d(sv + kb * BN * 128, &a.tv, KV_FULL(s), kb * 64, kt * BN, hl, b);
                }
                issued = i + 1;
            }
            mbar_wait(BAR_Q, 0, p.err, abort_flag);
            for (int i = issued > ST ? issued - ST : 0; i < issued; ++i)
                mbar_wait(KV_FULL(i % ST), (i / ST) & 1, p.err, abort_flag);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA
        // the whole warp runs the loop; one elected lane issues
        const uint32_t FULL = 0xffffffffu;
        bool ok = __all_sync(FULL, mbar_wait(BAR_Q, 0, p.err, abort_flag));
        const uint64_t dq0 = sdesc(sQ, 16, 1024), dk0 = sdesc(sStage, 16, 1024);
        const uint64_t dv0 = sdesc(sStage + C::KV_BYTES, BN * 128, 1024);
        bool have_o = false;  // O holds a kept tile's product
        auto pv = [&](int t) -> bool {  // O += P(t) V_t when tile t is kept
            const int y = t & 1, i = nt + t, s = i % ST;
            if (!__all_sync(FULL, mbar_wait(P_FULL(y), (t >> 1) & 1, p.err, abort_flag))) return false;
            tc_fence_after();
            const bool keep = kflag[y] != 0;
            if (elect_one()) {
                if (keep) {
                    const uint32_t so = (uint32_t)s * C::STAGE_BYTES;
#pragma unroll
                    for (int k2 = 0; k2 < BN / 16; ++k2)
                        mma_ts(tmem + C::T_O, tmem + C::T_P + y * (BN / 2) + k2 * 8, sdesc_add(dv0, so + k2 * 2048),
                               C::IDESC_O, (have_o || k2 > 0) ? 1u : 0u);
                }
                mma_commit(P_DONE(y));
                mma_commit(KV_EMPTY(s));
            }
            __syncwarp();
            have_o = have_o || keep;
            return true;
        };
        for (int i = 0; ok && i < nitems; ++i) {
            const int s = i % ST, x = i & 1;
            if (!(ok = __all_sync(FULL, mbar_wait(KV_FULL(s), (i / ST) & 1, p.err, abort_flag)))) break;
            // S buffer x was read by the softmax warps (item i - 2)
            if (i >= 2 && !(ok = __all_sync(FULL, mbar_wait(S_FREE(x), ((i >> 1) - 1) & 1, p.err, abort_flag))))
                break;
            tc_fence_after();
            const uint32_t so = (uint32_t)s * C::STAGE_BYTES;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;
                    mma_ss(tmem + C::T_S + x * BN, sdesc_add(dq0, (kk >> 2) * BM * 128 + off),
                           sdesc_add(dk0, so + (kk >> 2) * BN * 128 + off), C::IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(S_FULL(x));
                if (i < nt) mma_commit(KV_EMPTY(s));  // pass 1 needs K only for S
            }
            __syncwarp();
            if (i >= nt + 1) ok = pv(i - nt - 1);
        }
        if (ok && nt > 0) ok = pv(nt - 1);
        if (elect_one()) mma_commit(FIN);
        __syncwarp();
        mbar_wait(FIN, 0, p.err, abort_flag);
    } else {
        // -------------------------------------------------------- softmax
        constexpr int HB = BN / 2;       // columns per warpgroup
        const int xg = warp >> 2;        // warpgroup: key columns [xg*HB, xg*HB + HB) of a tile
        const int r = (warp & 3) * 32 + lane;  // row of the query tile
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int prow = pa + r;
        const bool valid = r < nrows;  // a query row of the sequence
        const float c = p.scale_log2;
        float m = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        auto sync_wgs = [] { asm volatile("bar.sync 1, 256;" ::: "memory"); };  // the 8 softmax warps
        auto load_s = [&](int i, uint32_t (&sr)[HB]) -> bool {
            const int x = i & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(S_FULL(x), (i >> 1) & 1, p.err, abort_flag))) return false;
            tc_fence_after();
            tmem_ld32(tmem + C::T_S + x * BN + xg * HB + lane_off, sr);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S_FREE(x));
            // causal mask on the tiles that reach past the row's position or
            // past the keys (a whole tile at or before pa is visible)
            const int j0 = (i < nt ? i : i - nt) * BN + xg * HB;
            if (j0 + HB - 1 > pa || j0 + HB > p.Lk) {
#pragma unroll
                for (int e = 0; e < HB; ++e)
                    if (j0 + e > prow || j0 + e >= p.Lk) sr[e] = __float_as_uint(-CUDART_INF_F);
            }
            return true;
        };
        // pass 1: the row's max and exp-sum over this warpgroup's half of
        // every causal key tile
        for (int t = 0; ok && t < nt; ++t) {
            uint32_t sr[HB];
            if (!(ok = load_s(t, sr))) break;
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int e = 0; e < HB; e += 2) mx = max3(mx, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
            const float mn = fmaxf(m, mx * c);
            if (mn != -CUDART_INF_F) {
                float sum = 0.f;
#pragma unroll
                for (int e = 0; e < HB; ++e) sum += fast_ex2(__uint_as_float(sr[e]) * c - mn);
                l = l * fast_ex2(m - mn) + sum;
                m = mn;
            }
        }
        // the two halves' statistics merged (every warp passes this barrier:
        // a failed wait leaves ok false but the warp still arrives)
        if (xg == 1) stat[r] = make_float2(m, l);
        sync_wgs();
        if (xg == 0) {
            const float2 o2 = stat[r];
            const float mn = fmaxf(m, o2.x);
            if (mn != -CUDART_INF_F) {
                l = l * fast_ex2(m - mn) + o2.y * fast_ex2(o2.x - mn);
                m = mn;
            }
            stat[r] = make_float2(m, l);
        }
        sync_wgs();
        if (xg == 1) {
            const float2 mine = stat[r];
            m = mine.x;
            l = mine.y;
        }
        ok = __all_sync(0xffffffffu, ok && !*abort_flag);
        const float lse2 = (valid && l > 0.f) ? m + __log2f(l) : CUDART_INF_F;  // +inf: P = 0
        // pass 2: P against the full statistic, the block decision, P of kept blocks
        bool any = false;
        uint8_t *krow = a.keep + (((long long)b * p.Hq + hq) * p.nqt + qt) * p.nkt;
        for (int t = 0; t < nt; ++t) {
            uint32_t sr[HB];
            const bool got = ok && load_s(nt + t, sr);
            ok = got;
            float mass = 0.f;
#pragma unroll
            for (int e = 0; e < HB; ++e) {
                const float pe = got ? fast_ex2(__uint_as_float(sr[e]) * c - lse2) : 0.f;
                mass += pe;
                sr[e] = __float_as_uint(pe);
            }
            const int y = t & 1;
            // row mass = the two halves' sums; the largest over the 128 rows
            half[(y * 2 + xg) * 128 + r] = mass;
            sync_wgs();
            const float rowm = half[y * 256 + r] + half[y * 256 + 128 + r];
            float wmax = valid ? rowm : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, off));
            if (lane == 0) red[y * 8 + warp] = wmax;
            sync_wgs();
            float cmax = red[y * 8];
#pragma unroll
            for (int w2 = 1; w2 < 8; ++w2) cmax = fmaxf(cmax, red[y * 8 + w2]);
            const bool keep = cmax >= a.tau;
            if (!ok) continue;  // every warp keeps meeting the barriers above; nothing else is waited for
            if (t >= 2) {
                // PV of tile t-2 read this P buffer (P_DONE(y) has completed
                // phase (t >> 1) - 1 or is about to; never phase t >> 1)
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(P_DONE(y), ((t >> 1) - 1) & 1, p.err, abort_flag))))
                    continue;
                tc_fence_after();
            }
            if (keep) {
                uint32_t pk[HB / 2];
#pragma unroll
                for (int e = 0; e < HB / 2; ++e) pk[e] = pack2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]));
                tmem_st16(tmem + C::T_P + y * (BN / 2) + xg * (HB / 2) + lane_off, pk);
                tmem_wait_st();
            }
            if (r == 0 && xg == 0) {
                kflag[y] = keep ? 1 : 0;
                krow[t] = keep ? 1 : 0;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(P_FULL(y));
            any = any || keep;
        }
        // tiles past the causal diagonal are never kept
        for (int t = nt + xg * 128 + r; t < p.nkt; t += 256) krow[t] = 0;
        // epilogue: O = the kept tiles' P V (P is already normalised), LSE;
        // warpgroup x writes columns [x*D/2, x*D/2 + D/2)
        ok = __all_sync(0xffffffffu, ok && mbar_wait(FIN, 0, p.err, abort_flag));
        tc_fence_after();
        const bool have = ok && any;
        __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + b * p.os[0] + (long long)(i0 + r) * p.os[1] +
                              hq * p.os[2] + xg * (D / 2);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[16];
            if (have) {
                tmem_ld16(tmem + C::T_O + xg * (D / 2) + cc * 16 + lane_off, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = 0u;
            }
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pk[e] = pack2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1]));
            if (valid) {
                uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 16);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
        if (valid && xg == 0)
            p.lse[((long long)b * p.Hq + hq) * p.lse_ld + i0 + r] =
                l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, 512);
}

template <int D>
static cudaError_t launch_mala_fwd_d(const AttnParams &p, uint8_t *keep, float tau, cudaStream_t st)
{
    using C = MalaCfg<D>;
    static std::atomic<bool> configured[64];
    cudaError_t e = once_per_device(configured, [] {
        return cudaFuncSetAttribute(mala_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    });
    if (e != cudaSuccess) return e;
    MalaArgs a;
    memset(&a, 0, sizeof a);
    a.p = p;
    a.keep = keep;
    a.tau = tau;
    if (!make_bshd_map(&a.tq, p.q, D, p.Lq, p.Hq, p.B, p.qs, C::BM) ||
        !make_bshd_map(&a.tk, p.k, D, p.Lk, p.Hkv, p.B, p.ks, C::BN) ||
        !make_bshd_map(&a.tv, p.v, D, p.Lk, p.Hkv, p.B, p.vs, C::BN))
        return cudaErrorInvalidValue;
    const unsigned blocks = tile_grid_blocks(p.nqt, p.Hq, p.B);
    if (!blocks) return cudaErrorInvalidConfiguration;
    launch_begin("mala_fwd", st);
    mala_fwd_kernel<D><<<blocks, 320, C::SMEM, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

cudaError_t launch_mala_fwd(const AttnParams &p, int D, uint8_t *keep, float tau, cudaStream_t st)
{
    if (p.nqt == 0 || p.Hq == 0 || p.B == 0) return cudaSuccess;
    return D == 128 ? launch_mala_fwd_d128(p, keep, tau, st) : launch_mala_fwd_d<64>(p, keep, tau, st);
}

}  // namespace cowa
