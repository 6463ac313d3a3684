// CoWA training backward on the 5th-generation tensor cores.
//
// Three kernels on the caller's stream; each output element has one writer,
// so the result is deterministic.
//
// 1. bwd_prep_kernel: for every query row, (-LSE*log2(e), -delta) with
//    delta = rowsum(dO * O), rows padded to a multiple of 64 (padding and rows
//    that see no key get (-inf, 0), so their probabilities are 0).
//
// 2. dK/dV pass, key-tile major: one CTA per (128 keys, KV head, batch).
//    The keys are the rows of every accumulator (tensor-memory lanes).
//    Tasks are (query head of the group, query tile of BM rows) from the
//    key-tile-major schedule.  Per task u:
//        S^T = K Q^T,  dP^T = V dO^T                   (MMA, into tensor memory)
//        P^T = 2^(S^T*scale*log2e - LSE*log2e),  dS^T = P^T (dP^T - delta)
//                                                      (warpgroup u % 2, thread = key)
//        dV += P^T dO,  dK += dS^T Q                   (MMA, P^T and dS^T from
//                                                       tensor memory)
//    Two warpgroups take alternate tasks so one computes while the MMAs of
//    the other run.  Two MMA-issuing warps split the MMAs by role: one
//    issues S^T/dP^T (writing only the score region), the other the gradient
//    MMAs (the only writer of dK and dV), so neither waits on the other's
//    barriers.  The scores are released (S_FREE) as soon as a warpgroup
//    holds them in registers; P^T/dS^T of a warpgroup's task are written only
//    after the gradient MMAs of its previous task complete (G_DONE).  A Q/dO
//    stage is released by the gradient issuer: the score MMAs of its task
//    completed before P^T of the task existed.  dK is scaled by
//    softmax_scale in the epilogue.  Two forms:
//    dkdv_sm100_kernel (d = 128): K and V stay in tensor memory as the A
//      operands of S^T and dP^T, so every MMA reads only Q or dO from shared
//      memory (two shared-memory operands cap an MMA at 128 bytes per
//      cycle); one score region (the 512 columns hold K, V, dK, dV, the
//      scores and two P^T/dS^T regions), 32-query tasks;
//    dkdv_sm100_ss_kernel (d = 64): K and V in shared memory, two full task
//      buffers (scores of task u+2 land in buffer u % 2 while the other
//      warpgroup works), 64-query tasks.
//
// 3. dq_sm100_kernel, query-tile major like the forward: per visible key tile
//        S = Q K^T,  dP = dO V^T,  dS = P (dP - delta),  dQ += dS K.
//    For d = 64 a CTA takes two query heads of a GQA group (same mask, same
//    K/V tiles) with one warpgroup and one MMA-issuing warp each (their
//    tensor-memory columns are disjoint, so the issuers need no ordering
//    between them; a K/V stage is released once both have committed).  As in
//    the dK/dV pass, S and dP of
//    tile t+1 are issued once the warpgroup has read those of tile t
//    (S_FREE), ahead of dQ += dS(t) K_t; dS(t+1) is written after that dQ
//    MMA completes (DONE).
//
// The elementwise warpgroups never read or write tensor-memory columns that
// an MMA still uses: S/dP and P/dS live in separate regions, and a
// tcgen05.commit tracks every earlier MMA of the issuing thread.  Every
// mbarrier wait is bounded and reports a timeout through the error word.
#include <math_constants.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace cowa {

using namespace sm100;

// ------------------------------------------------------------- preprocess --
// One row per D/8 lanes (16 bytes of O and of dO each), several rows per warp.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const AttnParams p, float2 *lsd, int lq_pad)
{
    constexpr int LPR = D / 8, RPW = 32 / LPR;  // lanes per row, rows per warp
    const int lane = threadIdx.x & 31, piece = lane % LPR;
    const long long row = ((long long)blockIdx.x * 8 + (threadIdx.x >> 5)) * RPW + lane / LPR;
    const long long total = (long long)p.B * p.Hq * lq_pad;
    const bool live = row < total;
    float s = 0.f, nl = -CUDART_INF_F;
    if (live) {
        const int i = (int)(row % lq_pad);
        const long long bh = row / lq_pad;  // b * Hq + hq
        const int hq = (int)(bh % p.Hq), b = (int)(bh / p.Hq);
        const SeqGeom sg = seq_geom(p, b);
        if (i < sg.Lq) {
            const long long off = sg.tb * p.os[0] + (long long)(sg.qoff + i) * p.os[1] + hq * p.os[2] + piece * 8;
            const uint4 ov = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p.o) + off);
            const uint4 dv = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p.dout) + off);
            const uint32_t oa[4] = {ov.x, ov.y, ov.z, ov.w}, da[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&oa[e]));
                const float2 df = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&da[e]));
                s += of.x * df.x + of.y * df.y;
            }
            const float lv = p.lse_in[((long long)sg.tb * p.Hq + hq) * p.lse_ld + sg.qoff + i];
            nl = lv == -CUDART_INF_F ? -CUDART_INF_F : -lv * 1.4426950408889634f;
        }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (live && piece == 0) lsd[row] = make_float2(nl, nl == -CUDART_INF_F ? 0.f : -s);
}

// ------------------------------------------------------------------ dK/dV --
struct BwdArgs {
    CUtensorMap tq, tk, tv, tdo;
    AttnParams p;
    const float2 *lsd;
    int lq_pad;
    int npair;
};

// Grid order of the key-major dK/dV pass: the sink tile (key tile 0, seen
// by every query) of every (KV head, batch) first, then (batch, KV head)
// after (batch, KV head) with their key tiles ascending, so the CTAs resident
// together are neighbouring key tiles of one head, which read the same query
// rows (measured at 32K, d = 128: DRAM reads 9.0 -> 1.6 GB per launch, L2 hit
// rate 63 -> 91 %); the long sink CTAs start in the first wave.
// With by_head false the order is tile step slowest and (KV head, batch)
// fastest, every head's sink tile first (at d = 64 this measured faster:
// recall8k 0.334 against 0.360 ms; its query rows fit L2 either way).  A
// packed batch's grid runs over the key-major work list's items instead, in
// the matching order (below); false when the CTA has no item.
__device__ __forceinline__ bool dkdv_order(const AttnParams &p, int &kt, int &hl, int &b, bool by_head)
{
    if (p.work) {
        // the list holds rank 0 (each sequence's first key tile, the sink)
        // first: with by_head, those of every KV head go first, then each
        // head's remaining items in list order, head after head
        const unsigned H = (unsigned)p.Hkv, n = (unsigned)p.work_n, lin = blockIdx.x;
        const unsigned n0 = by_head ? min((unsigned)p.work_n0, n) : 0u;
        unsigned item;
        if (!by_head) {
            item = lin / H;
            hl = (int)(lin % H);
        } else if (lin < H * n0) {
            item = lin / H;
            hl = (int)(lin % H);
        } else {
            const unsigned r = lin - H * n0, per = n - n0;  // per > 0: lin < H * n
            hl = (int)(r / per);
            item = n0 + (r - (unsigned)hl * per);
        }
        const int2 it = p.work[item];
        b = it.x;
        kt = it.y;
        return it.x >= 0;
    }
    if (!by_head) {
        const TilePos t = tile_pos(p.Hkv, p.B);
        kt = t.step;
        hl = t.slot;
        b = t.b;
        return true;
    }
    const unsigned hb_n = (unsigned)p.Hkv * (unsigned)p.B, lin = blockIdx.x;
    if (lin < hb_n) {
        kt = 0;
        b = (int)(lin / (unsigned)p.Hkv);
        hl = (int)(lin % (unsigned)p.Hkv);
    } else {
        const unsigned per = (unsigned)(p.nkt - 1), r = lin - hb_n, hb = r / per;
        kt = 1 + (int)(r - hb * per);
        b = (int)(hb / (unsigned)p.Hkv);
        hl = (int)(hb % (unsigned)p.Hkv);
    }
    return true;
}

// dK/dV, d = 128: K and V resident in tensor memory.
// Tensor-memory plan of a dK/dV CTA (512 columns, 128 lanes = its keys):
//   [0, D)            dK accumulator (fp32)
//   [D, 2D)           dV accumulator (fp32)
//   [2D, 2D + D/2)    K of the CTA's keys, bf16 pairs: the A operand of S^T
//   [2D + D/2, 3D)    V, the A operand of dP^T
//   [3D, 3D + BM)     S^T of the current task (fp32)
//   [3D + BM, 3D+2BM) dP^T of the current task
//   3D + 2BM + x*BM   P^T (BM/2 columns of bf16 pairs), then dS^T, of the
//                     tasks of warpgroup x
// D = 128: BM = 32 ends at 512; D = 64: BM = 64 ends at 448.
template <int D>
struct KvCfg {
    static constexpr int BN = kBwd5KeyTile;  // keys per CTA
    static constexpr int BM = bwd5_kv_bm(D);  // queries per task
    static constexpr int ST = 8;              // Q/dO stages
    static constexpr int KB = D / 64;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int QT_BYTES = BM * D * 2;
    static constexpr int LSD_BYTES = BM * 8;
    static constexpr int STAGE_BYTES = (2 * QT_BYTES + LSD_BYTES + 1023) / 1024 * 1024;
    static constexpr int T_DK = 0, T_DV = D, T_K = 2 * D, T_V = 2 * D + D / 2;
    static constexpr int T_S = 3 * D, T_DP = 3 * D + BM;
    static constexpr __host__ __device__ int t_pd(int x) { return 3 * D + 2 * BM + x * BM; }
    static_assert(3 * D + 4 * BM <= 512, "tensor-memory plan exceeds 512 columns");
    static constexpr int NBAR = 13 + 2 * ST;
    static constexpr int SMEM = 1024 + 2 * KV_BYTES + ST * STAGE_BYTES + 8 * NBAR + 16;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BM, 0, 0);
    static constexpr uint32_t IDESC_G = idesc_bf16(128, D, 0, 1);
};

template <int D, bool MALA>
__global__ void __launch_bounds__(352, 1) dkdv_sm100_kernel(const __grid_constant__ BwdArgs a)
{
    using C = KvCfg<D>;
    constexpr int BN = C::BN, BM = C::BM, ST = C::ST, KB = C::KB;
    const AttnParams &p = a.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const uint32_t sK = base, sV = base + C::KV_BYTES, sStage = base + 2 * C::KV_BYTES;
    auto stage_q = [&](int s) { return sStage + s * C::STAGE_BYTES; };
    auto stage_do = [&](int s) { return sStage + s * C::STAGE_BYTES + C::QT_BYTES; };
    auto stage_lsd = [&](int s) {
        return reinterpret_cast<const float2 *>(sm + 2 * C::KV_BYTES + s * C::STAGE_BYTES + 2 * C::QT_BYTES);
    };
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 2 * C::KV_BYTES + ST * C::STAGE_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t KV_LOADED = bar0;
    auto Q_FULL = [&](int s) { return bar0 + 8u * (1 + s); };
    auto Q_EMPTY = [&](int s) { return bar0 + 8u * (1 + ST + s); };
    auto S_FULL = [&](int x) { return bar0 + 8u * (1 + 2 * ST + x); };
    auto P_FULL = [&](int x) { return bar0 + 8u * (3 + 2 * ST + x); };
    const uint32_t DONE = bar0 + 8u * (5 + 2 * ST);
    auto FIN = [&](int r) { return bar0 + 8u * (r == 0 ? 6 + 2 * ST : 11 + 2 * ST); };  // per issuer
    auto S_FREE = [&](int x) { return bar0 + 8u * (7 + 2 * ST + x); };
    auto G_DONE = [&](int x) { return bar0 + 8u * (9 + 2 * ST + x); };
    const uint32_t KV_TM = bar0 + 8u * (12 + 2 * ST);  // K and V are in tensor memory

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int kt, hl, b;
    if (!dkdv_order(p, kt, hl, b, true)) return;
    const SeqGeom sg = seq_geom(p, b);
    const int c0 = kt * BN;
    if (c0 >= sg.Lk) return;  // past the end of this sequence of a packed batch
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    const int delta_pos = sg.Lk - sg.Lq;

    // the query tiles that see this key tile, from the same closed form as
    // the schedule builder
    const TileRanges tr = key_tile_ranges(c0, min(c0 + BN, sg.Lk) - 1, sg.Lq, sg.Lk, w, BM);
    const int nr = tr.n;
    const int lo0 = tr.lo0, lo1 = tr.lo1, lo2 = tr.lo2;
    const int len0 = tr.len0, len1 = tr.len1, len2 = tr.len2;
    const int nq = (nr > 0 ? len0 : 0) + (nr > 1 ? len1 : 0) + (nr > 2 ? len2 : 0);
    const int ntask = nq * p.g;
    auto task = [&](int u, int &hq, int &qt) {
        hq = hl * p.g + u / nq;
        int t = u % nq;
        if (t < len0 || nr == 1) { qt = lo0 + t; return; }
        t -= len0;
        if (t < len1 || nr == 2) { qt = lo1 + t; return; }
        qt = lo2 + t - len1;
    };

    if (tid == 0) {
        mbar_init(KV_LOADED, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(Q_FULL(s), 1);
            mbar_init(Q_EMPTY(s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(S_FULL(x), 1);
            mbar_init(P_FULL(x), 4);  // one arrival per warp
            mbar_init(S_FREE(x), 4);  // one arrival per warp
            mbar_init(G_DONE(x), 1);
        }
        mbar_init(DONE, 1);
        mbar_init(FIN(0), 1);
        mbar_init(FIN(1), 1);
        mbar_init(KV_TM, 8);  // one arrival per elementwise warp
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
        prefetch_tmap(&a.tdo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            mbar_expect_tx(KV_LOADED, 2 * C::KV_BYTES);
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_4d(sK + kb * BN * 128, &a.tk, KV_LOADED, kb * 64, sg.koff + c0, hl, sg.tb);
                tma_load_4d(sV + kb * BN * 128, &a.tv, KV_LOADED, kb * 64, sg.koff + c0, hl, sg.tb);
            }
            int issued = 0;
            for (int u = 0; u < ntask; ++u) {
                const int s = u % ST;
                if (u >= ST && !mbar_wait(Q_EMPTY(s), ((u / ST) - 1) & 1, p.err, abort_flag)) break;
                int hq, qt;
                task(u, hq, qt);
                // a listed query tile holds rows; its row pairs lie in the workspace
                if (!dcheck(qt >= 0 && qt * BM < sg.Lq && (qt + 1) * BM <= a.lq_pad && hq >= hl * p.g &&
                                hq < (hl + 1) * p.g,
                            p.err)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_expect_tx(Q_FULL(s), 2 * C::QT_BYTES + C::LSD_BYTES);
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(stage_q(s) + kb * BM * 128, &a.tq, Q_FULL(s), kb * 64, sg.qoff + qt * BM, hq, sg.tb);
                    tma_load_4d(stage_do(s) + kb * BM * 128, &a.tdo, Q_FULL(s), kb * 64, sg.qoff + qt * BM, hq, sg.tb);
                }
                bulk_load(stage_q(s) + 2 * C::QT_BYTES,
                          a.lsd + ((long long)b * p.Hq + hq) * a.lq_pad + (long long)qt * BM, C::LSD_BYTES,
                          Q_FULL(s));
                issued = u + 1;
            }
            mbar_wait(KV_LOADED, 0, p.err, abort_flag);
            for (int u = issued > ST ? issued - ST : 0; u < issued; ++u)
                mbar_wait(Q_FULL(u % ST), (u / ST) & 1, p.err, abort_flag);
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------------------ MMA
        // the whole warp runs the loop; one elected lane issues.  Warp 9
        // issues the score MMAs, warp 10 the gradient MMAs.  Every A operand
        // comes from tensor memory (K, V, P^T, dS^T): only Q and dO are read
        // from shared memory.
        const uint32_t FULL = 0xffffffffu;
        const int role = warp - 9;
        bool ok = __all_sync(FULL, mbar_wait(KV_TM, 0, p.err, abort_flag));
        tc_fence_after();
        const uint64_t dq0 = sdesc(stage_q(0), 16, 1024), ddo0 = sdesc(stage_do(0), 16, 1024);
        const uint64_t dqm0 = sdesc(stage_q(0), BM * 128, 1024), ddom0 = sdesc(stage_do(0), BM * 128, 1024);
        auto sdp = [&](int u) -> bool {  // S^T, dP^T of task u
            const int s = u % ST;
            if (!__all_sync(FULL, mbar_wait(Q_FULL(s), (u / ST) & 1, p.err, abort_flag))) return false;
            tc_fence_after();
            const uint32_t so = (uint32_t)s * C::STAGE_BYTES;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qo = so + (kk >> 2) * BM * 128 + (kk & 3) * 32;
                    mma_ts(tmem + C::T_S, tmem + C::T_K + kk * 8, sdesc_add(dq0, qo), C::IDESC_S, kk > 0);
                    mma_ts(tmem + C::T_DP, tmem + C::T_V + kk * 8, sdesc_add(ddo0, qo), C::IDESC_S, kk > 0);
                }
                mma_commit(S_FULL(u & 1));
            }
            __syncwarp();
            return true;
        };
        auto grad = [&](int u) -> bool {  // dV += P^T dO, dK += dS^T Q
            const int s = u % ST, x = u & 1;
            if (!__all_sync(FULL, mbar_wait(P_FULL(x), (u >> 1) & 1, p.err, abort_flag))) return false;
            tc_fence_after();
            const uint32_t tb = tmem + C::t_pd(x);
            const uint32_t so = (uint32_t)s * C::STAGE_BYTES;
            if (elect_one()) {
#pragma unroll
                for (int k2 = 0; k2 < BM / 16; ++k2) {
                    const uint32_t acc = (u > 0 || k2 > 0) ? 1u : 0u;
                    mma_ts(tmem + C::T_DV, tb + k2 * 8, sdesc_add(ddom0, so + k2 * 2048), C::IDESC_G, acc);
                    mma_ts(tmem + C::T_DK, tb + BM / 2 + k2 * 8, sdesc_add(dqm0, so + k2 * 2048), C::IDESC_G, acc);
                }
                mma_commit(Q_EMPTY(s));
                mma_commit(G_DONE(x));
            }
            __syncwarp();
            return true;
        };
        if (role == 0) {
            for (int u = 0; ok && u < ntask; ++u) {
                if (u >= 1) {
                    // S^T and dP^T have one region: the warpgroup of task u-1
                    // has read those of task u-1
                    const int xp = (u - 1) & 1;
                    if (!(ok = __all_sync(FULL, mbar_wait(S_FREE(xp), ((u - 1) >> 1) & 1, p.err, abort_flag))))
                        break;
                    tc_fence_after();
                }
                ok = sdp(u);
            }
        } else {
            for (int u = 0; ok && u < ntask; ++u) ok = grad(u);
            if (elect_one()) mma_commit(DONE);  // every gradient MMA; the score MMAs completed before them
            __syncwarp();
        }
        if (elect_one()) mma_commit(FIN(role));
        __syncwarp();
        mbar_wait(FIN(role), 0, p.err, abort_flag);
    } else {
        // ---------------------------------------------- P^T and dS^T per key
        const int x = warp >> 2;
        const int jl = (warp & 3) * 32 + lane;  // key row within the tile
        const int jg = c0 + jl;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        // K (warpgroup 0) or V (warpgroup 1) of this key into tensor memory:
        // row jl of the 128-byte-swizzled tile, 16-byte chunk c of each
        // 64-element block stored at chunk c ^ (jl % 8)
        bool ok = __all_sync(0xffffffffu, mbar_wait(KV_LOADED, 0, p.err, abort_flag));
        {
            const unsigned char *src = sm + (x == 0 ? 0 : C::KV_BYTES) + jl * 128;
            const uint32_t dst = tmem + (x == 0 ? C::T_K : C::T_V) + lane_off;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                uint32_t r[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v4 = *reinterpret_cast<const uint4 *>(src + kb * BN * 128 + ((c ^ (jl & 7)) * 16));
                    r[4 * c] = v4.x;
                    r[4 * c + 1] = v4.y;
                    r[4 * c + 2] = v4.z;
                    r[4 * c + 3] = v4.w;
                }
                tmem_st32(dst + kb * 32, r);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(KV_TM);
        }
        const uint32_t tS = tmem + C::T_S + lane_off, tPD = tmem + C::t_pd(x) + lane_off;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        // the aligned positions that see key jg (sink, near, long), as runs
        // formed once: a task's columns need no mask when one run holds them
        const Runs3 kr = key_pos_runs(jg, w, sg.Lk - 1);
        // this warpgroup's tasks u = x, x+2, ...: query head gi of the group
        // and position t in the key tile's query-tile list, advanced without
        // division
        int gi = nq > 0 ? x / nq : 0, tq = nq > 0 ? x % nq : 0;
        // MALA block decisions of this key's column for the group's first
        // query head (nullptr for CoWA)
        const uint8_t *kbase = MALA ? p.keep + ((long long)b * p.Hq + hl * p.g) * p.keep_nqt * p.keep_nkt +
                                            jg / kMalaBN
                                      : nullptr;
        for (int k = 0; ok; ++k) {
            const int u = 2 * k + x;
            if (u >= ntask) break;
            // task set-up, independent of the scores: done while they land
            const int qt = tq < len0 || nr == 1 ? lo0 + tq
                           : (tq - len0 < len1 || nr == 2 ? lo1 + tq - len0 : lo2 + tq - len0 - len1);
            // MALA: a key of a skipped block has dP = 0 and no dV share
            const bool skip = MALA && !kbase[(gi * p.keep_nqt + qt * BM / kMalaBM) * p.keep_nkt];
            tq += 2;
            while (tq >= nq) {
                tq -= nq;
                ++gi;
            }
            const int q0 = qt * BM;
            const int nrows = min(BM, sg.Lq - q0);
            const int pa = q0 + delta_pos, pb = pa + nrows - 1;
            // no mask when every key of the warp sees every in-range column
            const bool full = __all_sync(0xffffffffu, runs_cover(kr, pa, pb));
            uint32_t vis[BM / 32];
            if (!full) {
#pragma unroll
                for (int c = 0; c < BM / 32; ++c)  // columns p = pa + c*32 + bit, in range up to pb
                    vis[c] = runs_bits(kr, pa + c * 32) & span_bits(0, pb - pa - c * 32);
            }
            const float2 *lsd = stage_lsd(u % ST);
            ok = __all_sync(0xffffffffu, mbar_wait(S_FULL(x), k & 1, p.err, abort_flag));
            if (!ok) break;
            tc_fence_after();
            // S^T and dP^T in 32-column chunks; once the last chunk is in
            // registers the region is released for the next task's scores
            // (d = 128: the whole task is one chunk)
#pragma unroll
            for (int c = 0; c < BM / 32; ++c) {
                uint32_t sr[32], dr[32];
                tmem_ld32(tS + c * 32, sr);
                tmem_ld32(tS + BM + c * 32, dr);
                tmem_wait_ld();
                if (c == BM / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(S_FREE(x));
                }
                if (!full) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((vis[c] >> e) & 1u)) sr[e] = __float_as_uint(-CUDART_INF_F);
                }
                if (skip) {  // MALA skipped block: dP = 0
#pragma unroll
                    for (int e = 0; e < 32; ++e) dr[e] = 0u;
                }
                // P^T and dS^T as bf16 pairs: entry e holds columns 2e, 2e+1
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float4 ld = *reinterpret_cast<const float4 *>(lsd + c * 32 + 2 * e);  // (-lse2, -delta) x2
                    const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                                 sc2, make_float2(ld.x, ld.z));
                    const float2 pr = make_float2(fast_ex2(xa.x), fast_ex2(xa.y));
                    const float2 t = __fadd2_rn(make_float2(__uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1])),
                                                make_float2(ld.y, ld.w));
                    const float2 ds = __fmul2_rn(pr, t);
                    pk[e] = pack2(pr.x, pr.y);
                    dk[e] = pack2(ds.x, ds.y);
                }
                if (c == 0 && k > 0) {
                    // the gradient MMAs of this warpgroup's previous task read
                    // its P^T/dS^T columns (G_DONE(x) has completed k-1 or k
                    // phases)
                    ok = __all_sync(0xffffffffu, mbar_wait(G_DONE(x), (k - 1) & 1, p.err, abort_flag));
                    if (!ok) break;
                    tc_fence_after();
                }
                if (skip) {  // and no share of dV
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                }
                tmem_st16(tPD + c * 16, pk);
                tmem_st16(tPD + BM / 2 + c * 16, dk);
            }
            if (!ok) break;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(P_FULL(x));
        }
        // epilogue: warpgroup 0 writes dK (scaled), warpgroup 1 writes dV
        ok = __all_sync(0xffffffffu, mbar_wait(DONE, 0, p.err, abort_flag) && ok);
        tc_fence_after();
        const bool have = ok && ntask > 0;
        const float f = x == 0 ? p.scale : 1.f;
        const uint32_t tg = tmem + (x == 0 ? C::T_DK : C::T_DV) + lane_off;
        __nv_bfloat16 *grow_ = x == 0
            ? reinterpret_cast<__nv_bfloat16 *>(p.dk) + sg.tb * p.ks[0] + (long long)(sg.koff + jg) * p.ks[1] +
                  hl * p.ks[2]
            : reinterpret_cast<__nv_bfloat16 *>(p.dv) + sg.tb * p.vs[0] + (long long)(sg.koff + jg) * p.vs[1] +
                  hl * p.vs[2];
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
            uint32_t g[16];
            if (have) {
                tmem_ld16(tg + c * 16, g);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) g[e] = 0u;
            }
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pk[e] = pack2(__uint_as_float(g[2 * e]) * f, __uint_as_float(g[2 * e + 1]) * f);
            if (jg < sg.Lk && dcheck(sg.koff + jg < (p.cu_q ? p.total_k : p.Lk), p.err)) {
                uint4 *dst = reinterpret_cast<uint4 *>(grow_ + c * 16);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------- dK/dV, d = 64 --
// At d = 64 the accumulators take 128 columns and two full task buffers
// (S^T, dP^T, P^T, dS^T of 64 queries, 192 columns each) fit beside them, but
// not K and V as well: this kernel reads K and V from shared memory (their
// score MMAs are then paced by shared-memory bandwidth) and double-buffers
// the scores instead, which measured faster at d = 64 (0.30 ms against 0.43
// ms for the resident-K/V form with one score region, recall8k).  Task
// pipeline as described at the top of this file.
template <int D>
struct KvSsCfg {
    static constexpr int BN = kBwd5KeyTile;  // keys per CTA
    static constexpr int BM = bwd5_kv_bm(D);  // queries per task
    static constexpr int ST = 8;  // Q/dO stages (8 measured 2 % faster than 6, 4 % than 4)
    static constexpr int KB = D / 64;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int QT_BYTES = BM * D * 2;
    static constexpr int LSD_BYTES = BM * 8;
    static constexpr int STAGE_BYTES = (2 * QT_BYTES + LSD_BYTES + 1023) / 1024 * 1024;
    // tensor memory: dK, dV, then two buffers of S^T, dP^T, P^T (bf16), dS^T (bf16)
    static constexpr int T_DK = 0, T_DV = D, T_BUF = 2 * D, BUF = 3 * BM;
    static constexpr int NBAR = 12 + 2 * ST;
    static constexpr int SMEM = 1024 + 2 * KV_BYTES + ST * STAGE_BYTES + 8 * NBAR + 16;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BM, 0, 0);
    static constexpr uint32_t IDESC_G = idesc_bf16(128, D, 0, 1);
};

template <int D, bool MALA>
__global__ void __launch_bounds__(352, 1) dkdv_sm100_ss_kernel(const __grid_constant__ BwdArgs a)
{
    using C = KvSsCfg<D>;
    constexpr int BN = C::BN, BM = C::BM, ST = C::ST, KB = C::KB;
    const AttnParams &p = a.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const uint32_t sK = base, sV = base + C::KV_BYTES, sStage = base + 2 * C::KV_BYTES;
    auto stage_q = [&](int s) { return sStage + s * C::STAGE_BYTES; };
    auto stage_do = [&](int s) { return sStage + s * C::STAGE_BYTES + C::QT_BYTES; };
    auto stage_lsd = [&](int s) {
        return reinterpret_cast<const float2 *>(sm + 2 * C::KV_BYTES + s * C::STAGE_BYTES + 2 * C::QT_BYTES);
    };
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 2 * C::KV_BYTES + ST * C::STAGE_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t KV_LOADED = bar0;
    auto Q_FULL = [&](int s) { return bar0 + 8u * (1 + s); };
    auto Q_EMPTY = [&](int s) { return bar0 + 8u * (1 + ST + s); };
    auto S_FULL = [&](int x) { return bar0 + 8u * (1 + 2 * ST + x); };
    auto P_FULL = [&](int x) { return bar0 + 8u * (3 + 2 * ST + x); };
    const uint32_t DONE = bar0 + 8u * (5 + 2 * ST);
    auto FIN = [&](int r) { return bar0 + 8u * (r == 0 ? 6 + 2 * ST : 11 + 2 * ST); };  // per issuer
    auto S_FREE = [&](int x) { return bar0 + 8u * (7 + 2 * ST + x); };
    auto G_DONE = [&](int x) { return bar0 + 8u * (9 + 2 * ST + x); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int kt, hl, b;
    if (!dkdv_order(p, kt, hl, b, false)) return;
    const SeqGeom sg = seq_geom(p, b);
    const int c0 = kt * BN;
    if (c0 >= sg.Lk) return;  // past the end of this sequence of a packed batch
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    const int delta_pos = sg.Lk - sg.Lq;

    // the query tiles that see this key tile, from the same closed form as
    // the schedule builder
    const TileRanges tr = key_tile_ranges(c0, min(c0 + BN, sg.Lk) - 1, sg.Lq, sg.Lk, w, BM);
    const int nr = tr.n;
    const int lo0 = tr.lo0, lo1 = tr.lo1, lo2 = tr.lo2;
    const int len0 = tr.len0, len1 = tr.len1, len2 = tr.len2;
    const int nq = (nr > 0 ? len0 : 0) + (nr > 1 ? len1 : 0) + (nr > 2 ? len2 : 0);
    const int ntask = nq * p.g;
    auto task = [&](int u, int &hq, int &qt) {
        hq = hl * p.g + u / nq;
        int t = u % nq;
        if (t < len0 || nr == 1) { qt = lo0 + t; return; }
        t -= len0;
        if (t < len1 || nr == 2) { qt = lo1 + t; return; }
        qt = lo2 + t - len1;
    };

    if (tid == 0) {
        mbar_init(KV_LOADED, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(Q_FULL(s), 1);
            mbar_init(Q_EMPTY(s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(S_FULL(x), 1);
            mbar_init(P_FULL(x), 4);  // one arrival per warp
            mbar_init(S_FREE(x), 4);  // one arrival per warp
            mbar_init(G_DONE(x), 1);
        }
        mbar_init(DONE, 1);
        mbar_init(FIN(0), 1);
        mbar_init(FIN(1), 1);
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
        prefetch_tmap(&a.tdo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            mbar_expect_tx(KV_LOADED, 2 * C::KV_BYTES);
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_4d(sK + kb * BN * 128, &a.tk, KV_LOADED, kb * 64, sg.koff + c0, hl, sg.tb);
                tma_load_4d(sV + kb * BN * 128, &a.tv, KV_LOADED, kb * 64, sg.koff + c0, hl, sg.tb);
            }
            int issued = 0;
            for (int u = 0; u < ntask; ++u) {
                const int s = u % ST;
                if (u >= ST && !mbar_wait(Q_EMPTY(s), ((u / ST) - 1) & 1, p.err, abort_flag)) break;
                int hq, qt;
                task(u, hq, qt);
                // a listed query tile holds rows; its row pairs lie in the workspace
                if (!dcheck(qt >= 0 && qt * BM < sg.Lq && (qt + 1) * BM <= a.lq_pad && hq >= hl * p.g &&
                                hq < (hl + 1) * p.g,
                            p.err)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_expect_tx(Q_FULL(s), 2 * C::QT_BYTES + C::LSD_BYTES);
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(stage_q(s) + kb * BM * 128, &a.tq, Q_FULL(s), kb * 64, sg.qoff + qt * BM, hq, sg.tb);
                    tma_load_4d(stage_do(s) + kb * BM * 128, &a.tdo, Q_FULL(s), kb * 64, sg.qoff + qt * BM, hq, sg.tb);
                }
                bulk_load(stage_q(s) + 2 * C::QT_BYTES,
                          a.lsd + ((long long)b * p.Hq + hq) * a.lq_pad + (long long)qt * BM, C::LSD_BYTES,
                          Q_FULL(s));
                issued = u + 1;
            }
            mbar_wait(KV_LOADED, 0, p.err, abort_flag);
            for (int u = issued > ST ? issued - ST : 0; u < issued; ++u)
                mbar_wait(Q_FULL(u % ST), (u / ST) & 1, p.err, abort_flag);
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------------------ MMA
        // the whole warp runs the loop; one elected lane issues.  Warp 9
        // issues the score MMAs, warp 10 the gradient MMAs.
        const uint32_t FULL = 0xffffffffu;
        const int role = warp - 9;
        bool ok = __all_sync(FULL, mbar_wait(KV_LOADED, 0, p.err, abort_flag));
        const uint64_t dk0 = sdesc(sK, 16, 1024), dv0 = sdesc(sV, 16, 1024);
        const uint64_t dq0 = sdesc(stage_q(0), 16, 1024), ddo0 = sdesc(stage_do(0), 16, 1024);
        const uint64_t dqm0 = sdesc(stage_q(0), BM * 128, 1024), ddom0 = sdesc(stage_do(0), BM * 128, 1024);
        auto sdp = [&](int u) -> bool {  // S^T, dP^T of task u into buffer u % 2
            const int s = u % ST, x = u & 1;
            if (!__all_sync(FULL, mbar_wait(Q_FULL(s), (u / ST) & 1, p.err, abort_flag))) return false;
            tc_fence_after();
            const uint32_t tb = tmem + C::T_BUF + x * C::BUF;
            const uint32_t so = (uint32_t)s * C::STAGE_BYTES;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ko = (kk >> 2) * BN * 128 + (kk & 3) * 32;
                    const uint32_t qo = so + (kk >> 2) * BM * 128 + (kk & 3) * 32;
                    mma_ss(tb, sdesc_add(dk0, ko), sdesc_add(dq0, qo), C::IDESC_S, kk > 0);
                    mma_ss(tb + BM, sdesc_add(dv0, ko), sdesc_add(ddo0, qo), C::IDESC_S, kk > 0);
                }
                mma_commit(S_FULL(x));
            }
            __syncwarp();
            return true;
        };
        auto grad = [&](int u) -> bool {  // dV += P^T dO, dK += dS^T Q
            const int s = u % ST, x = u & 1;
            if (!__all_sync(FULL, mbar_wait(P_FULL(x), (u >> 1) & 1, p.err, abort_flag))) return false;
            tc_fence_after();
            const uint32_t tb = tmem + C::T_BUF + x * C::BUF;
            const uint32_t so = (uint32_t)s * C::STAGE_BYTES;
            if (elect_one()) {
#pragma unroll
                for (int k2 = 0; k2 < BM / 16; ++k2) {
                    const uint32_t acc = (u > 0 || k2 > 0) ? 1u : 0u;
                    mma_ts(tmem + C::T_DV, tb + 2 * BM + k2 * 8, sdesc_add(ddom0, so + k2 * 2048), C::IDESC_G, acc);
                    mma_ts(tmem + C::T_DK, tb + 2 * BM + BM / 2 + k2 * 8, sdesc_add(dqm0, so + k2 * 2048), C::IDESC_G,
                           acc);
                }
                mma_commit(Q_EMPTY(s));
                mma_commit(G_DONE(x));
            }
            __syncwarp();
            return true;
        };
        if (role == 0) {
            for (int u = 0; ok && u < ntask; ++u) {
                if (u >= 2) {
                    // warpgroup u % 2 has read S^T and dP^T of task u-2
                    if (!(ok = __all_sync(FULL, mbar_wait(S_FREE(u & 1), ((u - 2) >> 1) & 1, p.err, abort_flag))))
                        break;
                    tc_fence_after();
                }
                ok = sdp(u);
            }
        } else {
            for (int u = 0; ok && u < ntask; ++u) ok = grad(u);
            if (elect_one()) mma_commit(DONE);  // every gradient MMA; the score MMAs completed before them
            __syncwarp();
        }
        if (elect_one()) mma_commit(FIN(role));
        __syncwarp();
        mbar_wait(FIN(role), 0, p.err, abort_flag);
    } else {
        // ---------------------------------------------- P^T and dS^T per key
        const int x = warp >> 2;
        const int jl = (warp & 3) * 32 + lane;  // key row within the tile
        const int jg = c0 + jl;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tb = tmem + C::T_BUF + x * C::BUF + lane_off;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        // the aligned positions that see key jg (sink, near, long), as runs
        // formed once: a task's columns need no mask when one run holds them
        const Runs3 kr = key_pos_runs(jg, w, sg.Lk - 1);
        // this warpgroup's tasks u = x, x+2, ...: query head gi of the group
        // and position t in the key tile's query-tile list, advanced without
        // division
        int gi = nq > 0 ? x / nq : 0, tq = nq > 0 ? x % nq : 0;
        bool ok = true;
        // MALA block decisions of this key's column for the group's first
        // query head (nullptr for CoWA)
        const uint8_t *kbase = MALA ? p.keep + ((long long)b * p.Hq + hl * p.g) * p.keep_nqt * p.keep_nkt +
                                            jg / kMalaBN
                                      : nullptr;
        for (int k = 0;; ++k) {
            const int u = 2 * k + x;
            if (u >= ntask) break;
            // task set-up, independent of the scores: done while they land
            const int qt = tq < len0 || nr == 1 ? lo0 + tq
                           : (tq - len0 < len1 || nr == 2 ? lo1 + tq - len0 : lo2 + tq - len0 - len1);
            // MALA: a key of a skipped block has dP = 0 and no dV share
            const bool skip = MALA && !kbase[(gi * p.keep_nqt + qt * BM / kMalaBM) * p.keep_nkt];
            tq += 2;
            while (tq >= nq) {
                tq -= nq;
                ++gi;
            }
            const int q0 = qt * BM;
            const int nrows = min(BM, sg.Lq - q0);
            const int pa = q0 + delta_pos, pb = pa + nrows - 1;
            // no mask when every key of the warp sees every in-range column
            const bool full = __all_sync(0xffffffffu, runs_cover(kr, pa, pb));
            uint32_t vis[BM / 32];
            if (!full) {
#pragma unroll
                for (int c = 0; c < BM / 32; ++c)  // columns p = pa + c*32 + bit, in range up to pb
                    vis[c] = runs_bits(kr, pa + c * 32) & span_bits(0, pb - pa - c * 32);
            }
            const float2 *lsd = stage_lsd(u % ST);
            ok = __all_sync(0xffffffffu, mbar_wait(S_FULL(x), k & 1, p.err, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < BM / 32; ++c) {
                uint32_t sr[32], dr[32];
                tmem_ld32(tb + c * 32, sr);
                tmem_ld32(tb + BM + c * 32, dr);
                tmem_wait_ld();
                if (c == BM / 32 - 1) {
                    // all of S^T and dP^T read: S^T/dP^T of task u+2 may land
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(S_FREE(x));
                }
                if (!full) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((vis[c] >> e) & 1u)) sr[e] = __float_as_uint(-CUDART_INF_F);
                }
                if (skip) {  // MALA skipped block: dP = 0
#pragma unroll
                    for (int e = 0; e < 32; ++e) dr[e] = 0u;
                }
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float4 ld = *reinterpret_cast<const float4 *>(lsd + c * 32 + 2 * e);  // (-lse2, -delta) x2
                    const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                                 sc2, make_float2(ld.x, ld.z));
                    const float2 pr = make_float2(fast_ex2(xa.x), fast_ex2(xa.y));
                    const float2 t = __fadd2_rn(make_float2(__uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1])),
                                                make_float2(ld.y, ld.w));
                    const float2 ds = __fmul2_rn(pr, t);
                    pk[e] = pack2(pr.x, pr.y);
                    dk[e] = pack2(ds.x, ds.y);
                }
                if (c == 0 && k > 0) {
                    // the gradient MMAs of task u-2 read P^T/dS^T of this buffer
                    // (G_DONE(x) has completed k-1 or k phases)
                    ok = __all_sync(0xffffffffu, mbar_wait(G_DONE(x), (k - 1) & 1, p.err, abort_flag));
                    if (!ok) break;
                    tc_fence_after();
                }
                if (skip) {  // and no share of dV
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                }
                tmem_st16(tb + 2 * BM + c * 16, pk);
                tmem_st16(tb + 2 * BM + BM / 2 + c * 16, dk);
            }
            if (!ok) break;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(P_FULL(x));
        }
        // epilogue: warpgroup 0 writes dK (scaled), warpgroup 1 writes dV
        ok = __all_sync(0xffffffffu, mbar_wait(DONE, 0, p.err, abort_flag) && ok);
        tc_fence_after();
        const bool have = ok && ntask > 0;
        const float f = x == 0 ? p.scale : 1.f;
        const uint32_t tg = tmem + (x == 0 ? C::T_DK : C::T_DV) + lane_off;
        __nv_bfloat16 *grow_ = x == 0
            ? reinterpret_cast<__nv_bfloat16 *>(p.dk) + sg.tb * p.ks[0] + (long long)(sg.koff + jg) * p.ks[1] +
                  hl * p.ks[2]
            : reinterpret_cast<__nv_bfloat16 *>(p.dv) + sg.tb * p.vs[0] + (long long)(sg.koff + jg) * p.vs[1] +
                  hl * p.vs[2];
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
            uint32_t g[16];
            if (have) {
                tmem_ld16(tg + c * 16, g);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) g[e] = 0u;
            }
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pk[e] = pack2(__uint_as_float(g[2 * e]) * f, __uint_as_float(g[2 * e + 1]) * f);
            if (jg < sg.Lk && dcheck(sg.koff + jg < (p.cu_q ? p.total_k : p.Lk), p.err)) {
                uint4 *dst = reinterpret_cast<uint4 *>(grow_ + c * 16);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, 512);
}

// --------------------------------------------------------------------- dQ --
template <int D>
struct DqCfg {
    static constexpr int BM = kBwd5QTile;     // queries per CTA
    static constexpr int BN = bwd5_dq_bn(D);  // keys per tile
    static constexpr int NSLOT = D == 128 ? 1 : 2;
    static constexpr int ST = D == 128 ? 2 : 4;
    static constexpr int KB = D / 64;
    static constexpr int QT_BYTES = BM * D * 2;  // one head's Q or dO tile
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    // tensor memory per slot: S, dP, dS (bf16), dQ
    static constexpr int SLOT = D == 128 ? 512 : 256;
    static constexpr int T_S = 0, T_DP = BN, T_DS = 2 * BN, T_DQ = D == 128 ? 384 : 192;
    static constexpr int NBAR = 12 + 2 * ST;
    static constexpr int SMEM = 1024 + 2 * NSLOT * QT_BYTES + ST * STAGE_BYTES + 8 * NBAR + 16;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
    static constexpr uint32_t IDESC_Q = idesc_bf16(128, D, 0, 1);
};

template <int D, bool MALA>
__global__ void __launch_bounds__(352, 1) dq_sm100_kernel(const __grid_constant__ BwdArgs a)
{
    using C = DqCfg<D>;
    constexpr int BM = C::BM, BN = C::BN, ST = C::ST, KB = C::KB, NSLOT = C::NSLOT;
    const AttnParams &p = a.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    auto sQ = [&](int x) { return base + x * 2 * C::QT_BYTES; };
    auto sDO = [&](int x) { return base + x * 2 * C::QT_BYTES + C::QT_BYTES; };
    const uint32_t sStage = base + 2 * NSLOT * C::QT_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 2 * NSLOT * C::QT_BYTES + ST * C::STAGE_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t BAR_Q = bar0;
    auto KV_FULL = [&](int s) { return bar0 + 8u * (1 + s); };
    auto KV_EMPTY = [&](int s) { return bar0 + 8u * (1 + ST + s); };
    auto S_FULL = [&](int x) { return bar0 + 8u * (1 + 2 * ST + x); };
    auto DS_FULL = [&](int x) { return bar0 + 8u * (3 + 2 * ST + x); };
    auto DONE = [&](int x) { return bar0 + 8u * (5 + 2 * ST + x); };
    auto FIN = [&](int x) { return bar0 + 8u * (x == 0 ? 7 + 2 * ST : 10 + 2 * ST); };
    auto S_FREE = [&](int x) { return bar0 + 8u * (8 + 2 * ST + x); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int qt, slot, b;  // long rows first
    if (!query_tile_item(p, p.Hkv * a.npair, a.npair, qt, slot, b)) return;
    const int hl = slot / a.npair, pair = slot % a.npair;
    const int hq0 = hl * p.g + NSLOT * pair;
    const int nslot = min(NSLOT, p.g - NSLOT * pair);
    const SeqGeom sg = seq_geom(p, b);
    const int i0 = qt * BM;
    if (i0 >= sg.Lq) return;  // past the end of this sequence of a packed batch
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    const int delta_pos = sg.Lk - sg.Lq;
    const int nrows = min(BM, sg.Lq - i0);
    const int pa = i0 + delta_pos, pb = i0 + nrows - 1 + delta_pos;

    // the key tiles this query tile visits, from the same closed form as the
    // schedule builder
    const TileRanges tr = query_tile_ranges(pa, pb, w, BN);
    const int nr = tr.n;
    const int lo0 = tr.lo0, lo1 = tr.lo1, lo2 = tr.lo2;
    const int len0 = tr.len0, len1 = tr.len1, len2 = tr.len2;
    const int ntiles = (nr > 0 ? len0 : 0) + (nr > 1 ? len1 : 0) + (nr > 2 ? len2 : 0);
    auto tile_of = [&](int t) {
        if (t < len0 || nr == 1) return lo0 + t;
        t -= len0;
        if (t < len1 || nr == 2) return lo1 + t;
        return lo2 + t - len1;
    };

    if (tid == 0) {
        mbar_init(BAR_Q, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(KV_FULL(s), 1);
            mbar_init(KV_EMPTY(s), nslot);  // one commit per MMA issuer
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(S_FULL(x), 1);
            mbar_init(DS_FULL(x), 4);  // one arrival per warp
            mbar_init(DONE(x), 1);
            mbar_init(S_FREE(x), 4);  // one arrival per warp
            mbar_init(FIN(x), 1);
        }
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
        prefetch_tmap(&a.tdo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            mbar_expect_tx(BAR_Q, nslot * 2 * C::QT_BYTES);
            for (int x = 0; x < nslot; ++x)
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(sQ(x) + kb * BM * 128, &a.tq, BAR_Q, kb * 64, sg.qoff + i0, hq0 + x, sg.tb);
                    tma_load_4d(sDO(x) + kb * BM * 128, &a.tdo, BAR_Q, kb * 64, sg.qoff + i0, hq0 + x, sg.tb);
                }
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % ST;
                if (t >= ST && !mbar_wait(KV_EMPTY(s), ((t / ST) - 1) & 1, p.err, abort_flag)) break;
                const int kt = tile_of(t);
                if (!dcheck(kt >= 0 && kt * BN < sg.Lk, p.err)) {  // a listed tile holds keys
                    *abort_flag = 1;
                    break;
                }
                mbar_expect_tx(KV_FULL(s), C::STAGE_BYTES);
                const uint32_t sk = sStage + s * C::STAGE_BYTES, sv = sk + C::KV_BYTES;
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(sk + kb * BN * 128, &a.tk, KV_FULL(s), kb * 64, sg.koff + kt * BN, hl, sg.tb);
                    tma_load_4d(sv + kb * BN * 128, &a.tv, KV_FULL(s), kb * 64, sg.koff + kt * BN, hl, sg.tb);
                }
                issued = t + 1;
            }
            mbar_wait(BAR_Q, 0, p.err, abort_flag);
            for (int t = issued > ST ? issued - ST : 0; t < issued; ++t)
                mbar_wait(KV_FULL(t % ST), (t / ST) & 1, p.err, abort_flag);
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------------------ MMA
        // the whole warp runs the loop; one elected lane issues
        const uint32_t FULL = 0xffffffffu;
        const int x = warp - 9;  // head slot served
        bool ok = x < nslot && __all_sync(FULL, mbar_wait(BAR_Q, 0, p.err, abort_flag));
        const uint64_t dq0 = sdesc(sQ(0), 16, 1024), ddo0 = sdesc(sDO(0), 16, 1024);
        const uint64_t dk0 = sdesc(sStage, 16, 1024), dv0 = sdesc(sStage + C::KV_BYTES, 16, 1024);
        const uint64_t dkm0 = sdesc(sStage, BN * 128, 1024);
        auto sdp = [&](int t) {  // S_x = Q_x K_t^T, dP_x = dO_x V_t^T
            const uint32_t so = (uint32_t)(t % ST) * C::STAGE_BYTES;
            const uint32_t ts = tmem + x * C::SLOT;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qo = x * 2 * C::QT_BYTES + (kk >> 2) * BM * 128 + (kk & 3) * 32;
                    const uint32_t ko = so + (kk >> 2) * BN * 128 + (kk & 3) * 32;
                    mma_ss(ts + C::T_S, sdesc_add(dq0, qo), sdesc_add(dk0, ko), C::IDESC_S, kk > 0);
                    mma_ss(ts + C::T_DP, sdesc_add(ddo0, qo), sdesc_add(dv0, ko), C::IDESC_S, kk > 0);
                }
                mma_commit(S_FULL(x));
            }
            __syncwarp();
        };
        auto dq = [&](int t) -> bool {  // dQ_x += dS_x K_t
            if (!__all_sync(FULL, mbar_wait(DS_FULL(x), t & 1, p.err, abort_flag))) return false;
            tc_fence_after();
            const uint32_t so = (uint32_t)(t % ST) * C::STAGE_BYTES;
            const uint32_t ts = tmem + x * C::SLOT;
            if (elect_one()) {
#pragma unroll
                for (int k2 = 0; k2 < BN / 16; ++k2)
                    mma_ts(ts + C::T_DQ, ts + C::T_DS + k2 * 8, sdesc_add(dkm0, so + k2 * 2048), C::IDESC_Q,
                           (t > 0 || k2 > 0) ? 1u : 0u);
                mma_commit(DONE(x));
            }
            __syncwarp();
            return true;
        };
        if (ok && ntiles > 0) {
            ok = __all_sync(FULL, mbar_wait(KV_FULL(0), 0, p.err, abort_flag));
            if (ok) {
                tc_fence_after();
                sdp(0);
            }
        }
        for (int t = 0; ok && t < ntiles; ++t) {
            if (t + 1 < ntiles) {
                if (!(ok = __all_sync(FULL, mbar_wait(KV_FULL((t + 1) % ST), ((t + 1) / ST) & 1, p.err, abort_flag))))
                    break;
                // warpgroup x holds S_x(t) and dP_x(t) in registers
                if (!(ok = __all_sync(FULL, mbar_wait(S_FREE(x), t & 1, p.err, abort_flag)))) break;
                tc_fence_after();
                sdp(t + 1);
            }
            ok = dq(t);
            if (elect_one()) mma_commit(KV_EMPTY(t % ST));  // this head is done with K_t and V_t
            __syncwarp();
        }
        if (x < nslot) {
            if (elect_one()) mma_commit(FIN(x));
            __syncwarp();
            mbar_wait(FIN(x), 0, p.err, abort_flag);
        }
    } else {
        // ------------------------------------------------- dS per query row
        const int x = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t ts = tmem + x * C::SLOT + lane_off;
        const int prow = pa + r;
        const bool active = x < nslot;
        const int hq = hq0 + x;
        float nl = -CUDART_INF_F, nd = 0.f;
        if (active && i0 + r < sg.Lq && dcheck(i0 + r < a.lq_pad, p.err)) {
            const float2 v = a.lsd[((long long)b * p.Hq + hq) * a.lq_pad + i0 + r];
            nl = v.x;
            nd = v.y;
        }
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nl2 = make_float2(nl, nl),
                     nd2 = make_float2(nd, nd);
        // the keys row prow sees, as runs formed once: a tile needs no mask
        // when one run holds it for every row of the warp
        const Runs3 rr = row_key_runs(prow, w);
        bool ok = true;
        for (int t = 0; active && t < ntiles; ++t) {
            // tile set-up, independent of the scores: done while they land
            const int j0 = tile_of(t) * BN;
            // MALA: a skipped block's pairs have dP = 0 (query tiles of this
            // pass are the blocks' rows, key tiles their keys)
            const bool skip = MALA && !p.keep[(((long long)b * p.Hq + hq) * p.keep_nqt + qt) * p.keep_nkt +
                                                j0 / kMalaBN];
            const bool full = __all_sync(0xffffffffu, runs_cover(rr, j0, j0 + BN - 1));
            uint32_t vis[BN / 32];
            if (!full) {
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) vis[c] = runs_bits(rr, j0 + c * 32);
            }
            ok = __all_sync(0xffffffffu, mbar_wait(S_FULL(x), t & 1, p.err, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t sr[32], dr[32];
                tmem_ld32(ts + C::T_S + c * 32, sr);
                tmem_ld32(ts + C::T_DP + c * 32, dr);
                tmem_wait_ld();
                if (c == BN / 32 - 1) {
                    // all of S and dP read: those of tile t+1 may land
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(S_FREE(x));
                }
                if (!full) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((vis[c] >> e) & 1u)) sr[e] = __float_as_uint(-CUDART_INF_F);
                }
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                                 sc2, nl2);
                    // d = 64: one key pair in four on the FMA pipe (the cubic of the forward);
                    // measured 2 % faster here, slower in the dK/dV pass
                    constexpr int PE = D == 64 ? 4 : 0, PM = PE > 0 ? PE : 1;
                    const float2 pr = (PE && e % PM == PM - 1) ? exp2_poly2(xa) : make_float2(fast_ex2(xa.x), fast_ex2(xa.y));
                    const float2 tt = skip ? nd2
                                           : __fadd2_rn(make_float2(__uint_as_float(dr[2 * e]),
                                                                    __uint_as_float(dr[2 * e + 1])),
                                                        nd2);
                    const float2 ds = __fmul2_rn(pr, tt);
                    pk[e] = pack2(ds.x, ds.y);
                }
                if (c == 0 && t > 0) {
                    // dQ += dS(t-1) K reads the dS columns (DONE(x) has
                    // completed t-1 or t phases)
                    ok = __all_sync(0xffffffffu, mbar_wait(DONE(x), (t - 1) & 1, p.err, abort_flag));
                    if (!ok) break;
                    tc_fence_after();
                }
                tmem_st16(ts + C::T_DS + c * 16, pk);
            }
            if (!ok) break;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(DS_FULL(x));
        }
        if (active && ok && ntiles > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(DONE(x), (ntiles - 1) & 1, p.err, abort_flag));
        tc_fence_after();
        if (active) {
            const bool have = ok && ntiles > 0;
            __nv_bfloat16 *drow = reinterpret_cast<__nv_bfloat16 *>(p.dq) + sg.tb * p.qs[0] +
                                  (long long)(sg.qoff + i0 + r) * p.qs[1] + hq * p.qs[2];
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
                uint32_t g[16];
                if (have) {
                    tmem_ld16(ts + C::T_DQ + c * 16, g);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) g[e] = 0u;
                }
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    pk[e] = pack2(__uint_as_float(g[2 * e]) * p.scale, __uint_as_float(g[2 * e + 1]) * p.scale);
                if (r < nrows && dcheck(sg.qoff + i0 + r < (p.cu_q ? p.total_q : p.Lq), p.err)) {
                    uint4 *dst = reinterpret_cast<uint4 *>(drow + c * 16);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ dQ, d = 128 --
// Query-tile major with Q and dO resident in tensor memory: S = Q K^T and
// dP = dO V^T take their A operands from there, dQ += dS K takes dS from
// there, so every MMA reads only K or V from shared memory.  One query head
// per CTA, key tiles of 64.  Both elementwise warpgroups work on every tile,
// warpgroup x on key columns [32x, 32x + 32): a row's dS needs no statistic
// of the other columns, so the split costs no exchange and halves the time
// from scores to dS.  Tensor memory (512 columns, lanes = query rows):
//   [0, 128) dQ (fp32), [128, 192) Q, [192, 256) dO (bf16 pairs),
//   [256, 320) S, [320, 384) dP, 384 + 32y dS of the tiles t with t % 2 = y.
// Order per tile t: S(t), dP(t) once both warpgroups hold S(t-1) and dP(t-1)
// in registers (S_FREE); dQ += dS(t) K_t once dS(t) is written (DS_FULL);
// dS(t+2) is written after dQ(t) completes (DONE).
struct DqTmCfg {
    static constexpr int D = 128, BM = kBwd5QTile, BN = 64;
    static constexpr int ST = 4;
    static constexpr int KB = D / 64;
    static constexpr int QT_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int T_DQ = 0, T_Q = 128, T_DO = 192, T_S = 256, T_DP = 320;
    static constexpr __host__ __device__ int t_ds(int y) { return 384 + 32 * y; }
    static constexpr int NBAR = 12 + 2 * ST;
    static constexpr int SMEM = 1024 + 2 * QT_BYTES + ST * STAGE_BYTES + 8 * NBAR + 16;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
    static constexpr uint32_t IDESC_Q = idesc_bf16(128, D, 0, 1);
};

template <bool MALA>
__global__ void __launch_bounds__(352, 1) dq_tm_kernel(const __grid_constant__ BwdArgs a)
{
    using C = DqTmCfg;
    constexpr int D = C::D, BM = C::BM, BN = C::BN, ST = C::ST, KB = C::KB;
    const AttnParams &p = a.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const uint32_t sQ = base, sDO = base + C::QT_BYTES, sStage = base + 2 * C::QT_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 2 * C::QT_BYTES + ST * C::STAGE_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t BAR_Q = bar0;
    auto KV_FULL = [&](int s) { return bar0 + 8u * (1 + s); };
    auto KV_EMPTY = [&](int s) { return bar0 + 8u * (1 + ST + s); };
    const uint32_t S_FULL = bar0 + 8u * (1 + 2 * ST);
    const uint32_t S_FREE = bar0 + 8u * (2 + 2 * ST);
    auto DS_FULL = [&](int y) { return bar0 + 8u * (3 + 2 * ST + y); };
    auto DONE = [&](int y) { return bar0 + 8u * (5 + 2 * ST + y); };
    auto FIN = [&](int r) { return bar0 + 8u * (7 + 2 * ST + r); };
    const uint32_t QD_TM = bar0 + 8u * (9 + 2 * ST);  // Q and dO are in tensor memory

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int qt, hq, b;  // long rows first
    if (!query_tile_item(p, p.Hq, p.g, qt, hq, b)) return;
    const int hl = hq / p.g;
    const SeqGeom sg = seq_geom(p, b);
    const int i0 = qt * BM;
    if (i0 >= sg.Lq) return;  // past the end of this sequence of a packed batch
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    const int delta_pos = sg.Lk - sg.Lq;
    const int nrows = min(BM, sg.Lq - i0);
    const int pa = i0 + delta_pos, pb = i0 + nrows - 1 + delta_pos;

    // the key tiles this query tile visits, from the same closed form as the
    // schedule builder
    const TileRanges tr = query_tile_ranges(pa, pb, w, BN);
    const int nr = tr.n;
    const int lo0 = tr.lo0, lo1 = tr.lo1, lo2 = tr.lo2;
    const int len0 = tr.len0, len1 = tr.len1, len2 = tr.len2;
    const int ntiles = (nr > 0 ? len0 : 0) + (nr > 1 ? len1 : 0) + (nr > 2 ? len2 : 0);
    auto tile_of = [&](int t) {
        if (t < len0 || nr == 1) return lo0 + t;
        t -= len0;
        if (t < len1 || nr == 2) return lo1 + t;
        return lo2 + t - len1;
    };

    if (tid == 0) {
        mbar_init(BAR_Q, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(KV_FULL(s), 1);
            mbar_init(KV_EMPTY(s), 1);
        }
        mbar_init(S_FULL, 1);
        mbar_init(S_FREE, 8);  // one arrival per elementwise warp
        for (int y = 0; y < 2; ++y) {
            mbar_init(DS_FULL(y), 8);  // one arrival per warp
            mbar_init(DONE(y), 1);
            mbar_init(FIN(y), 1);
        }
        mbar_init(QD_TM, 8);
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
        prefetch_tmap(&a.tdo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            mbar_expect_tx(BAR_Q, 2 * C::QT_BYTES);
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_4d(sQ + kb * BM * 128, &a.tq, BAR_Q, kb * 64, sg.qoff + i0, hq, sg.tb);
                tma_load_4d(sDO + kb * BM * 128, &a.tdo, BAR_Q, kb * 64, sg.qoff + i0, hq, sg.tb);
            }
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % ST;
                if (t >= ST && !mbar_wait(KV_EMPTY(s), ((t / ST) - 1) & 1, p.err, abort_flag)) break;
                const int kt = tile_of(t);
                if (!dcheck(kt >= 0 && kt * BN < sg.Lk, p.err)) {  // a listed tile holds keys
                    *abort_flag = 1;
                    break;
                }
                mbar_expect_tx(KV_FULL(s), C::STAGE_BYTES);
                const uint32_t sk = sStage + s * C::STAGE_BYTES, sv = sk + C::KV_BYTES;
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(sk + kb * BN * 128, &a.tk, KV_FULL(s), kb * 64, sg.koff + kt * BN, hl, sg.tb);
                    tma_load_4d(sv + kb * BN * 128, &a.tv, KV_FULL(s), kb * 64, sg.koff + kt * BN, hl, sg.tb);
                }
                issued = t + 1;
            }
            mbar_wait(BAR_Q, 0, p.err, abort_flag);
            for (int t = issued > ST ? issued - ST : 0; t < issued; ++t)
                mbar_wait(KV_FULL(t % ST), (t / ST) & 1, p.err, abort_flag);
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------------------ MMA
        // the whole warp runs the loop; one elected lane issues.  Warp 9
        // issues S and dP, warp 10 the dQ MMAs (the accumulator's only writer).
        const uint32_t FULL = 0xffffffffu;
        const int role = warp - 9;
        bool ok = __all_sync(FULL, mbar_wait(QD_TM, 0, p.err, abort_flag));
        tc_fence_after();
        const uint64_t dk0 = sdesc(sStage, 16, 1024), dv0 = sdesc(sStage + C::KV_BYTES, 16, 1024);
        const uint64_t dkm0 = sdesc(sStage, BN * 128, 1024);
        if (role == 0) {
            for (int t = 0; ok && t < ntiles; ++t) {
                const int s = t % ST;
                if (!(ok = __all_sync(FULL, mbar_wait(KV_FULL(s), (t / ST) & 1, p.err, abort_flag)))) break;
                if (t > 0 && !(ok = __all_sync(FULL, mbar_wait(S_FREE, (t - 1) & 1, p.err, abort_flag)))) break;
                tc_fence_after();
                const uint32_t so = (uint32_t)s * C::STAGE_BYTES;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t ko = so + (kk >> 2) * BN * 128 + (kk & 3) * 32;
                        mma_ts(tmem + C::T_S, tmem + C::T_Q + kk * 8, sdesc_add(dk0, ko), C::IDESC_S, kk > 0);
                        mma_ts(tmem + C::T_DP, tmem + C::T_DO + kk * 8, sdesc_add(dv0, ko), C::IDESC_S, kk > 0);
                    }
                    mma_commit(S_FULL);
                }
                __syncwarp();
            }
        } else {
            for (int t = 0; ok && t < ntiles; ++t) {
                const int y = t & 1;
                if (!(ok = __all_sync(FULL, mbar_wait(DS_FULL(y), (t >> 1) & 1, p.err, abort_flag)))) break;
                tc_fence_after();
                const uint32_t so = (uint32_t)(t % ST) * C::STAGE_BYTES;
                if (elect_one()) {
#pragma unroll
                    for (int k2 = 0; k2 < BN / 16; ++k2)
                        mma_ts(tmem + C::T_DQ, tmem + C::t_ds(y) + k2 * 8, sdesc_add(dkm0, so + k2 * 2048), C::IDESC_Q,
                               (t > 0 || k2 > 0) ? 1u : 0u);
                    mma_commit(DONE(y));
                    mma_commit(KV_EMPTY(t % ST));  // S(t), dP(t) completed before dS(t) existed
                }
                __syncwarp();
            }
        }
        if (elect_one()) mma_commit(FIN(role));
        __syncwarp();
        mbar_wait(FIN(role), 0, p.err, abort_flag);
    } else {
        // ------------------------------- dS of 32 key columns per query row
        const int x = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        // Q (warpgroup 0) or dO (warpgroup 1) of this row into tensor memory
        bool ok = __all_sync(0xffffffffu, mbar_wait(BAR_Q, 0, p.err, abort_flag));
        {
            const unsigned char *src = sm + (x == 0 ? 0 : C::QT_BYTES) + r * 128;
            const uint32_t dst = tmem + (x == 0 ? C::T_Q : C::T_DO) + lane_off;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v4 = *reinterpret_cast<const uint4 *>(src + kb * BM * 128 + ((c ^ (r & 7)) * 16));
                    v[4 * c] = v4.x;
                    v[4 * c + 1] = v4.y;
                    v[4 * c + 2] = v4.z;
                    v[4 * c + 3] = v4.w;
                }
                tmem_st32(dst + kb * 32, v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(QD_TM);
        }
        const int prow = pa + r;
        float nl = -CUDART_INF_F, nd = 0.f;
        if (i0 + r < sg.Lq && dcheck(i0 + r < a.lq_pad, p.err)) {
            const float2 v = a.lsd[((long long)b * p.Hq + hq) * a.lq_pad + i0 + r];
            nl = v.x;
            nd = v.y;
        }
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nl2 = make_float2(nl, nl),
                     nd2 = make_float2(nd, nd);
        const uint32_t tS = tmem + C::T_S + x * 32 + lane_off, tDP = tmem + C::T_DP + x * 32 + lane_off;
        // the keys row prow sees, as runs formed once: a half tile needs no
        // mask when one run holds it for every row of the warp
        const Runs3 rr = row_key_runs(prow, w);
        for (int t = 0; ok && t < ntiles; ++t) {
            // tile set-up, independent of the scores: done while they land
            const int j0 = tile_of(t) * BN + x * 32;
            // MALA: a skipped block's pairs have dP = 0
            const bool skip = MALA && !p.keep[(((long long)b * p.Hq + hq) * p.keep_nqt + qt) * p.keep_nkt +
                                                j0 / kMalaBN];
            const bool full = __all_sync(0xffffffffu, runs_cover(rr, j0, j0 + 31));
            const uint32_t vis = full ? 0xffffffffu : runs_bits(rr, j0);
            ok = __all_sync(0xffffffffu, mbar_wait(S_FULL, t & 1, p.err, abort_flag));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[32], dr[32];
            tmem_ld32(tS, sr);
            tmem_ld32(tDP, dr);
            tmem_wait_ld();
            // S and dP of tile t are in registers: those of tile t+1 may land
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S_FREE);
            if (!full) {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (!((vis >> e) & 1u)) sr[e] = __float_as_uint(-CUDART_INF_F);
            }
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                             sc2, nl2);
                const float2 pr = make_float2(fast_ex2(xa.x), fast_ex2(xa.y));
                const float2 tt = skip ? nd2
                                       : __fadd2_rn(make_float2(__uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1])),
                                                    nd2);
                const float2 ds = __fmul2_rn(pr, tt);
                pk[e] = pack2(ds.x, ds.y);
            }
            const int y = t & 1;
            if (t >= 2) {
                // dQ += dS(t-2) K reads these columns (DONE(y) has completed
                // phase (t >> 1) - 1 or is about to; never phase t >> 1)
                ok = __all_sync(0xffffffffu, mbar_wait(DONE(y), ((t >> 1) - 1) & 1, p.err, abort_flag));
                if (!ok) break;
                tc_fence_after();
            }
            tmem_st16(tmem + C::t_ds(y) + x * 16 + lane_off, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(DS_FULL(y));
        }
        // the last dQ MMA: DONE of the last tile's parity
        if (ok && ntiles > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(DONE((ntiles - 1) & 1), ((ntiles - 1) >> 1) & 1, p.err, abort_flag));
        tc_fence_after();
        const bool have = ok && ntiles > 0;
        __nv_bfloat16 *drow = reinterpret_cast<__nv_bfloat16 *>(p.dq) + sg.tb * p.qs[0] +
                              (long long)(sg.qoff + i0 + r) * p.qs[1] + hq * p.qs[2] + x * (D / 2);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {  // warpgroup x writes columns [64x, 64x + 64)
            uint32_t g[16];
            if (have) {
                tmem_ld16(tmem + C::T_DQ + x * (D / 2) + c * 16 + lane_off, g);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) g[e] = 0u;
            }
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                pk[e] = pack2(__uint_as_float(g[2 * e]) * p.scale, __uint_as_float(g[2 * e + 1]) * p.scale);
            if (r < nrows && dcheck(sg.qoff + i0 + r < (p.cu_q ? p.total_q : p.Lq), p.err)) {
                uint4 *dst = reinterpret_cast<uint4 *>(drow + c * 16);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, 512);
}

// ----------------------------------------------------------------- host ----
template <int D, bool MALA>
static cudaError_t launch_bwd5_d(const AttnParams &p, float2 *lsd, int lq_pad, int nqt_dq, int nkt_kv,
                                 const int2 *work_q, int work_q_n, const int2 *work_k, int work_k_n, cudaStream_t st)
{
    using K = typename std::conditional<D == 128, KvCfg<128>, KvSsCfg<64>>::type;
    using Q = DqCfg<D>;
    static std::atomic<bool> configured[64];
    cudaError_t e = once_per_device(configured, [] {
        if constexpr (D == 128) {
            cudaError_t r = cudaFuncSetAttribute(dkdv_sm100_kernel<128, MALA>, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
            if (r != cudaSuccess) return r;
            return cudaFuncSetAttribute(dq_tm_kernel<MALA>, cudaFuncAttributeMaxDynamicSharedMemorySize, DqTmCfg::SMEM);
        } else {
            cudaError_t r = cudaFuncSetAttribute(dkdv_sm100_ss_kernel<64, MALA>, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
            if (r != cudaSuccess) return r;
            return cudaFuncSetAttribute(dq_sm100_kernel<64, MALA>, cudaFuncAttributeMaxDynamicSharedMemorySize, Q::SMEM);
        }
    });
    if (e != cudaSuccess) return e;
    const long long rows = (long long)p.B * p.Hq * lq_pad;
    constexpr int PREP_ROWS = 8 * (32 / (D / 8));  // rows per 256-thread block
    if (rows > 0) {
        launch_begin("bwd_prep", st);
        bwd_prep_kernel<D><<<(unsigned)((rows + PREP_ROWS - 1) / PREP_ROWS), 256, 0, st>>>(p, lsd, lq_pad);
        launch_end(st);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    BwdArgs a;
    memset(&a, 0, sizeof a);
    a.p = p;
    a.lsd = lsd;
    a.lq_pad = lq_pad;
    // dK/dV: query tiles of BM rows, key tiles of 128
    // a packed batch is one batch entry of total_q / total_k rows
    const long long Lq_map = p.cu_q ? p.total_q : p.Lq, Lk_map = p.cu_q ? p.total_k : p.Lk;
    const long long B_map = p.cu_q ? 1 : p.B;
    if (!make_bshd_map(&a.tq, p.q, D, Lq_map, p.Hq, B_map, p.qs, K::BM) ||
        !make_bshd_map(&a.tdo, p.dout, D, Lq_map, p.Hq, B_map, p.os, K::BM) ||
        !make_bshd_map(&a.tk, p.k, D, Lk_map, p.Hkv, B_map, p.ks, K::BN) ||
        !make_bshd_map(&a.tv, p.v, D, Lk_map, p.Hkv, B_map, p.vs, K::BN))
        return cudaErrorInvalidValue;
    a.p.nkt = nkt_kv;
    a.p.work = work_k;  // packed batch: the key-major work list
    a.p.work_n = work_k_n;
    a.p.work_n0 = p.B;  // rank 0 comes first: at most one item per sequence
    if (nkt_kv > 0) {
        const unsigned g1 = work_k ? tile_grid_blocks(work_k_n, p.Hkv, 1) : tile_grid_blocks(nkt_kv, p.Hkv, p.B);
        if (!g1) return cudaErrorInvalidConfiguration;
        launch_begin("dkdv_sm100", st);
        if constexpr (D == 128)
            dkdv_sm100_kernel<128, MALA><<<g1, 352, K::SMEM, st>>>(a);
        else
            dkdv_sm100_ss_kernel<64, MALA><<<g1, 352, K::SMEM, st>>>(a);
        launch_end(st);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // dQ: query tiles of 128 rows, key tiles of BN
    const int dq_bn = D == 128 ? DqTmCfg::BN : Q::BN;
    if (!make_bshd_map(&a.tq, p.q, D, Lq_map, p.Hq, B_map, p.qs, Q::BM) ||
        !make_bshd_map(&a.tdo, p.dout, D, Lq_map, p.Hq, B_map, p.os, Q::BM) ||
        !make_bshd_map(&a.tk, p.k, D, Lk_map, p.Hkv, B_map, p.ks, dq_bn) ||
        !make_bshd_map(&a.tv, p.v, D, Lk_map, p.Hkv, B_map, p.vs, dq_bn))
        return cudaErrorInvalidValue;
    a.p.nqt = nqt_dq;
    a.p.work = work_q;  // packed batch: the query-major work list
    a.p.work_n = work_q_n;
    if (nqt_dq > 0) {
        if constexpr (D == 128) {
            // one query head per CTA, Q and dO resident in tensor memory
            const unsigned g2 = work_q ? tile_grid_blocks(work_q_n, p.Hq, 1) : tile_grid_blocks(nqt_dq, p.Hq, p.B);
            if (!g2) return cudaErrorInvalidConfiguration;
            launch_begin("dq_sm100", st);
            dq_tm_kernel<MALA><<<g2, 352, DqTmCfg::SMEM, st>>>(a);
            launch_end(st);
        } else {
            a.npair = (p.g + Q::NSLOT - 1) / Q::NSLOT;
            const unsigned g2 = work_q ? tile_grid_blocks(work_q_n, (long long)p.Hkv * a.npair, 1)
                                       : tile_grid_blocks(nqt_dq, (long long)p.Hkv * a.npair, p.B);
            if (!g2) return cudaErrorInvalidConfiguration;
            launch_begin("dq_sm100", st);
            dq_sm100_kernel<64, MALA><<<g2, 352, Q::SMEM, st>>>(a);
            launch_end(st);
        }
        e = cudaGetLastError();
    }
    return e;
}

cudaError_t launch_bwd_sm100(const AttnParams &p, int D, float2 *lsd, int lq_pad, int nqt_dq, int nkt_kv,
                             cudaStream_t st, const int2 *work_q, int work_q_n, const int2 *work_k, int work_k_n)
{
    if (p.B == 0 || p.Hq == 0) return cudaSuccess;
    // MALA's block decisions are a separate instantiation, so the CoWA
    // kernels carry none of their code
    if (p.keep)
        return D == 128 ? launch_bwd5_d<128, true>(p, lsd, lq_pad, nqt_dq, nkt_kv, work_q, work_q_n, work_k, work_k_n, st)
                        : launch_bwd5_d<64, true>(p, lsd, lq_pad, nqt_dq, nkt_kv, work_q, work_q_n, work_k, work_k_n, st);
    return D == 128 ? launch_bwd5_d<128, false>(p, lsd, lq_pad, nqt_dq, nkt_kv, work_q, work_q_n, work_k, work_k_n, st)
                    : launch_bwd5_d<64, false>(p, lsd, lq_pad, nqt_dq, nkt_kv, work_q, work_q_n, work_k, work_k_n, st);
}

}  // namespace cowa
