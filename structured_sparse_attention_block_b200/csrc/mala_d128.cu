// MassAlloc Attention (MALA) forward for d = 128: key tiles of 128 (two
// decision blocks of 64 keys each), two query heads of a GQA group per CTA.
//
// The reading is the one stated in mala.cu: full causal scoring, each row's
// softmax statistics over all of its causal keys, per block of 128 query
// rows x 64 keys of one head the largest row mass sum_j P_ij deciding
// whether the block's PV runs (mass >= tau), P taken against the full LSE.
//
// One CTA per (query tile of 128 rows, pair of query heads of one GQA group,
// batch): the two heads share every K and V tile and the causal tile range.
// Items i = 0 .. 2nt-1 walk the causal key tiles twice: pass 1 (i < nt)
// folds each row's max and exp-sum, pass 2 (i >= nt) takes
// P = 2^(S*scale*log2e - LSE*log2e) in fp32, the two blocks' row masses, the
// block decisions (the four warps of a head slot meet once per tile through
// shared memory), and writes P of the kept blocks (bf16) for
// O += P V, whose MMAs run only over kept blocks' keys.
// Tensor memory as in fwd_sm100.cu: one 128-column S region shared by the
// two slots (S_0(i), S_1(i), S_0(i+1), ... each issued once the other slot's
// softmax holds the previous one), P_x (64 columns), O_x (128 columns).
// K has a ring of three stages (both passes), V of two (pass 2 only).
// Warps: 0-3 softmax of slot 0, 4-7 of slot 1 (thread = query row), 8 TMA,
// 9 and 10 the MMA issuers of slots 0 and 1, 11 idle; the softmax
// warpgroups take registers from the fourth (setmaxnreg).  Every mbarrier
// wait is bounded and reports a timeout through the error word; the
// per-tile shared-memory meeting of a slot's warps is passed by every warp
// on every tile, also after a failed wait.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace cowa {

using namespace sm100;

struct MalaD128Args {
    CUtensorMap tq, tk, tv;
    AttnParams p;
    uint8_t *keep;  // [B, Hq, nqt, nkt] decisions, blocks of kMalaBM x kMalaBN
    float tau;
    int npair;      // head pairs per KV head: ceil(g / 2)
};

struct MalaD128Cfg {
    static constexpr int D = 128, BM = 128, BN = 128;
    static_assert(BM == kMalaBM && BN == 2 * kMalaBN, "two decision blocks per key tile");
    static constexpr int KST = 3, VST = 2;
    static constexpr int KB = D / 64;
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int T_S = 0;
    static constexpr __host__ __device__ int t_p(int x) { return 128 + 64 * x; }
    static constexpr __host__ __device__ int t_o(int x) { return 256 + 128 * x; }
    static constexpr int NBAR = 1 + 2 * (KST + VST) + 2 * 5;
    // after the barriers: tensor-memory address, abort flag, decisions [2][2],
    // per-warp block maxima [2 slots][2 tiles][4 warps][2 blocks]
    static constexpr int EXTRA = 16 + 16 + 128;
    static constexpr int SMEM = 1024 + 2 * Q_BYTES + (KST + VST) * KV_BYTES + 8 * NBAR + EXTRA;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
    static constexpr uint32_t IDESC_O = idesc_bf16(128, D, 0, 1);
    static constexpr int THREADS = 384;
    static constexpr int REG_LAUNCH = 168;  // three warps per sub-partition share its 16384 registers
    static constexpr int REG_SOFTMAX = 200, REG_OTHER = 96;
    static_assert(2 * 128 * REG_SOFTMAX + 128 * REG_OTHER <= THREADS * REG_LAUNCH, "register split exceeds the launch");
    static_assert(SMEM <= 232448, "shared memory");
};

// 2^x on the MUFU, or for one pair in POLY on the FMA pipe
template <int POLY>
__device__ __forceinline__ float2 exp2_pair(float2 xa, int e)
{
    if (POLY && e % (POLY > 0 ? POLY : 1) == POLY - 1) return exp2_poly2(xa);
    return make_float2(fast_ex2(xa.x), fast_ex2(xa.y));
}

template <int POLY>
__global__ void __launch_bounds__(384, 1) mala_fwd_d128_kernel(const __grid_constant__ MalaD128Args a)
{
    using C = MalaD128Cfg;
    constexpr int D = C::D, BM = C::BM, BN = C::BN, KST = C::KST, VST = C::VST, KB = C::KB;
    const AttnParams &p = a.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const uint32_t sQ = base;
    const uint32_t sK = base + 2 * C::Q_BYTES;
    const uint32_t sV = sK + KST * C::KV_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 2 * C::Q_BYTES + (KST + VST) * C::KV_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *kflag = reinterpret_cast<volatile int *>(tmem_slot + 4);  // [slot][tile % 2]: bit h = block h kept
    float *red = reinterpret_cast<float *>(tmem_slot + 8);                  // [slot][tile % 2][warp][block]
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t BAR_Q = bar0;
    auto K_FULL = [&](int s) { return bar0 + 8u * (1 + s); };
    auto K_EMPTY = [&](int s) { return bar0 + 8u * (1 + KST + s); };
    auto V_FULL = [&](int s) { return bar0 + 8u * (1 + 2 * KST + s); };
    auto V_EMPTY = [&](int s) { return bar0 + 8u * (1 + 2 * KST + VST + s); };
    constexpr int B1 = 1 + 2 * (KST + VST);
    auto S_FULL = [&](int x) { return bar0 + 8u * (B1 + x); };
    auto S_FREE = [&](int x) { return bar0 + 8u * (B1 + 2 + x); };
    auto P_FULL = [&](int x) { return bar0 + 8u * (B1 + 4 + x); };
    auto O_DONE = [&](int x) { return bar0 + 8u * (B1 + 6 + x); };
    auto FIN = [&](int x) { return bar0 + 8u * (B1 + 8 + x); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int qt, slot, b;  // long rows first
    if (!query_tile_item(p, p.Hkv * a.npair, a.npair, qt, slot, b)) return;
    const int hl = slot / a.npair, pair = slot % a.npair;
    const int hq0 = hl * p.g + 2 * pair;
    const int nslot = (2 * pair + 1 < p.g) ? 2 : 1;  // an odd group leaves the last head alone
    const int i0 = qt * BM;
    const int delta = p.Lk - p.Lq;
    const int nrows = min(BM, p.Lq - i0);
    const int pa = i0 + delta, pb = i0 + nrows - 1 + delta;
    // causal key tiles of the query tile: 0 .. pb / BN, within the keys
    const int nkt128 = (p.Lk + BN - 1) / BN;
    const int nt = pb < 0 ? 0 : min(pb / BN + 1, nkt128);
    const int nitems = 2 * nt;  // pass 1 tiles, then pass 2 tiles

    if (tid == 0) {
        mbar_init(BAR_Q, 1);
        for (int s = 0; s < KST; ++s) {
            mbar_init(K_FULL(s), 1);
            mbar_init(K_EMPTY(s), nslot);  // one commit per MMA issuer
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(V_FULL(s), 1);
            mbar_init(V_EMPTY(s), nslot);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(S_FULL(x), 1);
            mbar_init(S_FREE(x), 4);  // one arrival per softmax warp
            mbar_init(P_FULL(x), 4);
            mbar_init(O_DONE(x), 1);
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8) {
        setmaxnreg_dec<C::REG_OTHER>();
        if (warp == 8) {
            // -------------------------------------------------------- TMA
            // iteration j loads K for item j and V for pass-2 tile j - nt - 1
            if (lane == 0) {
                mbar_expect_tx(BAR_Q, nslot * C::Q_BYTES);
                for (int x = 0; x < nslot; ++x)
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_4d(sQ + x * C::Q_BYTES + kb * BM * 128, &a.tq, BAR_Q, kb * 64, i0, hq0 + x, b);
                int kiss = 0, viss = 0;
                bool good = true;
                for (int j = 0; good && j <= nitems; ++j) {
                    if (j < nitems) {
                        const int s = j % KST, kt = j < nt ? j : j - nt;
                        if (j >= KST && !(good = mbar_wait(K_EMPTY(s), ((j / KST) - 1) & 1, p.err, abort_flag)))
                            break;
                        if (!(good = dcheck(kt * BN < p.Lk, p.err))) {
                            *abort_flag = 1;
                            break;
                        }
                        mbar_expect_tx(K_FULL(s), C::KV_BYTES);
                        for (int kb = 0; kb < KB; ++kb)
                            tma_load_4d(sK + s * C::KV_BYTES + kb * BN * 128, &a.tk, K_FULL(s), kb * 64, kt * BN, hl, b);
                        kiss = j + 1;
                    }
                    const int u = j - nt - 1;  // pass-2 tile whose V goes now
                    if (u >= 0 && u < nt) {
                        const int s = u % VST;
                        if (u >= VST && !(good = mbar_wait(V_EMPTY(s), ((u / VST) - 1) & 1, p.err, abort_flag)))
                            break;
                        mbar_expect_tx(V_FULL(s), C::KV_BYTES);
                        for (int kb = 0; kb < KB; ++kb)
                            tma_load_4d(sV + s * C::KV_BYTES + kb * BN * 128, &a.tv, V_FULL(s), kb * 64, u * BN, hl, b);
                        viss = u + 1;
                    }
                }
                // every load this thread issued has landed before the CTA ends
                mbar_wait(BAR_Q, 0, p.err, abort_flag);
                for (int t = kiss > KST ? kiss - KST : 0; t < kiss; ++t)
                    mbar_wait(K_FULL(t % KST), (t / KST) & 1, p.err, abort_flag);
                for (int t = viss > VST ? viss - VST : 0; t < viss; ++t)
                    mbar_wait(V_FULL(t % VST), (t / VST) & 1, p.err, abort_flag);
            }
        } else if (warp == 9 || warp == 10) {
            // -------------------------------------------------------- MMA
            // issuer x, per item i: S_x(i) once the score region is free,
            // then (pass 2) PV_x of the previous pass-2 tile once its P is
            // written, over the keys of its kept blocks only
            const uint32_t FULL = 0xffffffffu;
            const int x = warp - 9;
            const int other = nslot == 2 ? x ^ 1 : x;
            bool ok = x < nslot && __all_sync(FULL, mbar_wait(BAR_Q, 0, p.err, abort_flag));
            const uint64_t dq0 = sdesc(sQ, 16, 1024);
            const uint64_t dk0 = sdesc(sK, 16, 1024);
            const uint64_t dv0 = sdesc(sV, BN * 128, 1024);
            bool have_o = false;  // O holds a kept block's product
            auto pv = [&](int u) -> bool {
                if (!__all_sync(FULL, mbar_wait(V_FULL(u % VST), (u / VST) & 1, p.err, abort_flag))) return false;
                if (!__all_sync(FULL, mbar_wait(P_FULL(x), u & 1, p.err, abort_flag))) return false;
                tc_fence_after();
                const int kf = kflag[x * 2 + (u & 1)];
                const uint32_t vo = (uint32_t)(u % VST) * C::KV_BYTES;
                if (elect_one()) {
                    bool acc = have_o;
#pragma unroll
                    for (int k2 = 0; k2 < BN / 16; ++k2) {
                        if (!((kf >> (k2 / 4)) & 1)) continue;  // block k2 / 4 skipped
                        mma_ts(tmem + C::t_o(x), tmem + C::t_p(x) + k2 * 8, sdesc_add(dv0, vo + k2 * 2048),
                               C::IDESC_O, acc ? 1u : 0u);
                        acc = true;
                    }
                    mma_commit(O_DONE(x));
                    mma_commit(V_EMPTY(u % VST));
                }
                __syncwarp();
                have_o = have_o || kf != 0;
                return true;
            };
            for (int i = 0; ok && i < nitems; ++i) {
                if (!(ok = __all_sync(FULL, mbar_wait(K_FULL(i % KST), (i / KST) & 1, p.err, abort_flag)))) break;
                // the score region: slot 1's S(i) follows slot 0's S(i), slot
                // 0's S(i) follows slot 1's S(i-1)
                const int ph = x == 1 && nslot == 2 ? i : i - 1;
                if (ph >= 0 && !(ok = __all_sync(FULL, mbar_wait(S_FREE(other), ph & 1, p.err, abort_flag)))) break;
                tc_fence_after();
                const uint32_t ko = (uint32_t)(i % KST) * C::KV_BYTES;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk & 3) * 32;
                        const uint64_t ad = sdesc_add(dq0, x * C::Q_BYTES + (kk >> 2) * BM * 128 + off);
                        const uint64_t bd = sdesc_add(dk0, ko + (kk >> 2) * BN * 128 + off);
                        mma_ss(tmem + C::T_S, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(S_FULL(x));
                    mma_commit(K_EMPTY(i % KST));
                }
                __syncwarp();
                if (i > nt && !(ok = pv(i - nt - 1))) break;
            }
            if (ok && nt > 0) ok = pv(nt - 1);
            if (x < nslot) {
                if (elect_one()) mma_commit(FIN(x));
                __syncwarp();
                mbar_wait(FIN(x), 0, p.err, abort_flag);
            }
        }
    } else {
        setmaxnreg_inc<C::REG_SOFTMAX>();
        // ---------------------------------------------------------- softmax
        const int x = warp >> 2;
        const int wq = warp & 3;  // warp within the slot's warpgroup
        const int r = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + C::T_S + lane_off;
        const uint32_t tP = tmem + C::t_p(x) + lane_off;
        const uint32_t tOx = tmem + C::t_o(x) + lane_off;
        const int prow = pa + r;
        const bool active = x < nslot;
        const bool valid = r < nrows;  // a query row of the sequence
        const float c = p.scale_log2;
        const int hq = hq0 + x;
        // one read of the row of S of item i, with the causal mask (and the
        // keys' end) applied on the tiles that reach past the row
        auto load_s = [&](int i, uint32_t (&sr)[BN]) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(S_FULL(x), i & 1, p.err, abort_flag))) return false;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc)
                tmem_ld32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[cc * 32]));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S_FREE(x));
            const int j0 = (i < nt ? i : i - nt) * BN;
            if (j0 + BN - 1 > pa || j0 + BN > p.Lk) {
                const int lim = min(prow, p.Lk - 1) - j0;  // last visible column of the row
#pragma unroll
                for (int e = 0; e < BN; ++e)
                    if (e > lim) sr[e] = __float_as_uint(-CUDART_INF_F);
            }
            return true;
        };
        bool ok = active;
        // pass 1: the row's max and exp-sum over every causal key tile
        float m = -CUDART_INF_F, l = 0.f;
        for (int t = 0; ok && t < nt; ++t) {
            uint32_t sr[BN];
            if (!(ok = load_s(t, sr))) break;
            float mx4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) mx4[k] = -CUDART_INF_F;
#pragma unroll
            for (int e = 0; e < BN; e += 8) {
                mx4[0] = max3(mx4[0], __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
                mx4[1] = max3(mx4[1], __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
                mx4[2] = max3(mx4[2], __uint_as_float(sr[e + 4]), __uint_as_float(sr[e + 5]));
                mx4[3] = max3(mx4[3], __uint_as_float(sr[e + 6]), __uint_as_float(sr[e + 7]));
            }
            const float mn = fmaxf(m, fmaxf(max3(mx4[0], mx4[1], mx4[2]), mx4[3]) * c);
            if (mn == -CUDART_INF_F) continue;  // nothing visible yet in this row
            const float2 c2 = make_float2(c, c), nm2 = make_float2(-mn, -mn);
            float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < BN / 2; ++e) {
                const float2 xa =
                    __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), c2, nm2);
                const float2 pr = exp2_pair<POLY>(xa, e);
                if (e & 1)
                    sb = __fadd2_rn(sb, pr);
                else
                    sa = __fadd2_rn(sa, pr);
            }
            l = l * fast_ex2(m - mn) + ((sa.x + sa.y) + (sb.x + sb.y));
            m = mn;
        }
        const float lse2 = (valid && l > 0.f) ? m + __log2f(l) : CUDART_INF_F;  // +inf: P = 0
        // pass 2: P against the full statistic, the block decisions, P of kept blocks
        bool any = false;
        uint8_t *krow = a.keep + (((long long)b * p.Hq + hq) * p.nqt + qt) * p.nkt;
        for (int t = 0; t < nt; ++t) {  // every warp meets its slot's barrier on every tile
            const int i = nt + t, y = t & 1;
            uint32_t sr[BN];
            const bool got = active && ok && load_s(i, sr);
            ok = got;
            float ms0 = 0.f, ms1 = 0.f;  // the row's mass in the two blocks
            if (got) {
                const float2 c2 = make_float2(c, c), nl2 = make_float2(-lse2, -lse2);
                float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int e = 0; e < BN / 2; ++e) {
                    const float2 xa =
                        __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), c2, nl2);
                    const float2 pr = exp2_pair<POLY>(xa, e);
                    if (e < BN / 4)
                        s0 = __fadd2_rn(s0, pr);
                    else
                        s1 = __fadd2_rn(s1, pr);
                    sr[e] = pack2(pr.x, pr.y);  // packed entry e holds keys 2e, 2e+1
                }
                ms0 = s0.x + s0.y;
                ms1 = s1.x + s1.y;
            }
            // the largest row mass of each block: the warp's, then the four warps'
            float w0 = valid ? ms0 : 0.f, w1 = valid ? ms1 : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                w0 = fmaxf(w0, __shfl_xor_sync(0xffffffffu, w0, off));
                w1 = fmaxf(w1, __shfl_xor_sync(0xffffffffu, w1, off));
            }
            float *rb = red + ((x * 2 + y) * 4) * 2;
            if (lane == 0) {
                rb[wq * 2] = w0;
                rb[wq * 2 + 1] = w1;
            }
            asm volatile("bar.sync %0, 128;" ::"r"(1 + x) : "memory");
            const float c0 = fmaxf(fmaxf(rb[0], rb[2]), fmaxf(rb[4], rb[6]));
            const float c1 = fmaxf(fmaxf(rb[1], rb[3]), fmaxf(rb[5], rb[7]));
            // a block holds a causal pair of the tile when its first key is at
            // or before the last row's position (and within the keys)
            const int kb0 = 2 * t;
            const bool keep0 = c0 >= a.tau && kb0 * kMalaBN <= pb && kb0 * kMalaBN < p.Lk;
            const bool keep1 = c1 >= a.tau && (kb0 + 1) * kMalaBN <= pb && (kb0 + 1) * kMalaBN < p.Lk;
            if (!ok) continue;  // the barrier above was still met
            if (t > 0) {
                // PV of the previous pass-2 tile read P_x
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(O_DONE(x), (t - 1) & 1, p.err, abort_flag)))) continue;
                tc_fence_after();
            }
            if (keep0)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) tmem_st16(tP + cc * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[cc * 16]));
            if (keep1)
#pragma unroll
                for (int cc = 2; cc < 4; ++cc) tmem_st16(tP + cc * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[cc * 16]));
            if (r == 0) {
                kflag[x * 2 + y] = (keep0 ? 1 : 0) | (keep1 ? 2 : 0);
                if (dcheck(kb0 < p.nkt, p.err)) krow[kb0] = keep0 ? 1 : 0;
                if (kb0 + 1 < p.nkt) krow[kb0 + 1] = keep1 ? 1 : 0;
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(P_FULL(x));
            any = any || keep0 || keep1;
        }
        if (active) {
            // blocks past the causal tiles are never kept
            for (int kb = 2 * nt + r; kb < p.nkt; kb += 128) krow[kb] = 0;
            // epilogue: O = the kept blocks' P V (P is already normalised), LSE
            ok = __all_sync(0xffffffffu, ok && mbar_wait(FIN(x), 0, p.err, abort_flag));
            tc_fence_after();
            const bool have = ok && __any_sync(0xffffffffu, any);
            __nv_bfloat16 *orow =
                reinterpret_cast<__nv_bfloat16 *>(p.o) + b * p.os[0] + (long long)(i0 + r) * p.os[1] + hq * p.os[2];
#pragma unroll
            for (int cc = 0; cc < D / 16; ++cc) {
                uint32_t o[16];
                if (have) {
                    tmem_ld16(tOx + cc * 16, o);
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
            if (valid)
                p.lse[((long long)b * p.Hq + hq) * p.lse_ld + i0 + r] =
                    l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, 512);
}

cudaError_t launch_mala_fwd_d128(const AttnParams &p, uint8_t *keep, float tau, cudaStream_t st)
{
    using C = MalaD128Cfg;
    // one exponential pair in four on the FMA pipe (both passes): measured
    // faster than one in eight and than one in two
    constexpr int POLY = 4;
    static std::atomic<bool> configured[64];
    cudaError_t e = once_per_device(configured, [] {
        cudaError_t r =
            cudaFuncSetAttribute(mala_fwd_d128_kernel<POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        // the register split assumes the launch count it was planned for
        cudaFuncAttributes fa;
        if (r == cudaSuccess) r = cudaFuncGetAttributes(&fa, mala_fwd_d128_kernel<POLY>);
        if (r == cudaSuccess && fa.numRegs < C::REG_LAUNCH) r = cudaErrorInvalidDeviceFunction;
        return r;
    });
    if (e != cudaSuccess) return e;
    MalaD128Args a;
    memset(&a, 0, sizeof a);
    a.p = p;
    a.keep = keep;
    a.tau = tau;
    a.npair = (p.g + 1) / 2;
    if (!make_bshd_map(&a.tq, p.q, C::D, p.Lq, p.Hq, p.B, p.qs, C::BM) ||
        !make_bshd_map(&a.tk, p.k, C::D, p.Lk, p.Hkv, p.B, p.ks, C::BN) ||
        !make_bshd_map(&a.tv, p.v, C::D, p.Lk, p.Hkv, p.B, p.vs, C::BN))
        return cudaErrorInvalidValue;
    const unsigned blocks = tile_grid_blocks(p.nqt, (long long)p.Hkv * a.npair, p.B);
    if (!blocks) return cudaErrorInvalidConfiguration;
    launch_begin("mala_fwd", st);
    mala_fwd_d128_kernel<POLY><<<blocks, C::THREADS, C::SMEM, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

}  // namespace cowa
