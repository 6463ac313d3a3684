// CoWA training / prefill forward on the 5th-generation tensor cores
// (d = 64 and 128): key tiles of 128, one score region shared by two heads.
//
// One CTA per (query tile of 128 rows, pair of query heads of one GQA group,
// batch).  Two query heads of a group have the same KV head, hence the same
// window mask and the same visible key tiles, so the CTA streams each K/V
// tile once for both.  At 128 keys both MMAs of a tile run at the tensor
// pipe's full rate (an MMA with both operands in shared memory is capped at
// 128 bytes of operand per cycle, which at 64 keys costs S = Q K^T half as
// much again), and every per-tile cost of the softmax (tile set-up, barrier
// round trips) is paid once per 128 keys.
//
// Tensor-memory columns:
//   [0, 128)          S, shared by the two slots: S_0(t), S_1(t), S_0(t+1), ...
//                     each issued once the other slot's softmax holds the
//                     previous one in registers (S_FREE)
//   [128 + 64x, +64)  P_x (bf16 pairs), the A operand of PV_x
//   [256 + d x, +d)   O_x (fp32)
// The score chain runs ahead of the softmax: S_x(t+1) is computed while
// softmax x works on tile t.  P_x is rewritten only after PV_x(t-1) has
// completed (O_DONE).  O is divided by the sum of the bf16 P that the PV MMA
// consumed, summed from the packed pairs on the ALU; the LSE uses the fp32
// sum.  The O row is rescaled in tensor memory only when the running max
// grows by more than 2^8 (until then the stale max is a valid reference).
//
// K and V have rings of their own: K_t is released when both slots' S(t) are
// complete, early, so its stages prefetch far ahead; V_t when both PV(t)
// are.  Shared memory (d = 128): 64 KB of Q, 96 KB of K, 64 KB of V.
//
// Warps: 0-3 softmax of slot 0, 4-7 of slot 1 (thread = query row), 8 TMA,
// 9 and 10 the MMA issuers of slots 0 and 1, 11 idle.  A softmax thread holds
// its row of S (128 registers): the block is launched at 168 registers per
// thread (three warps per sub-partition share its 16384) and the fourth
// warpgroup hands most of its registers to the softmax warpgroups.  The two
// slots' softmax warps run freely: making their exponential loops take turns
// on the MUFU (as an earlier 64-key kernel did) cost 9 % at 128K.  Every
// mbarrier wait is bounded and reports a timeout through the error word.
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace cowa {

using namespace sm100;

struct FwdArgs {
    CUtensorMap tq, tk, tv;
    AttnParams p;
    int npair;  // head pairs per KV head: ceil(g / 2)
};

template <int D_>
struct FwdCfg {
    static constexpr int D = D_, BM = 128, BN = 128;
    static constexpr int KST = D == 128 ? 3 : 4, VST = D == 128 ? 2 : 3;  // K and V stages
    static constexpr int KB = D / 64;           // 128-byte blocks along d
    static constexpr int Q_BYTES = BM * D * 2;  // one head's query tile
    static constexpr int KV_BYTES = BN * D * 2; // one K or V tile
    static constexpr int T_S = 0;
    static constexpr __host__ __device__ int t_p(int x) { return 128 + 64 * x; }
    static constexpr __host__ __device__ int t_o(int x) { return 256 + D * x; }
    static constexpr int NBAR = 1 + 2 * (KST + VST) + 2 * 5;
    static constexpr int SMEM = 1024 + 2 * Q_BYTES + (KST + VST) * KV_BYTES + 8 * NBAR + 16;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
    static constexpr uint32_t IDESC_O = idesc_bf16(128, D, 0, 1);
    static constexpr int THREADS = 384;
    // the launch's registers per thread: three warps per sub-partition share
    // its 16384 registers, 170 each, allocated in steps of 8
    static constexpr int REG_LAUNCH = 168;
    static constexpr int REG_SOFTMAX = 200, REG_OTHER = 96;
    static_assert(2 * 128 * REG_SOFTMAX + 128 * REG_OTHER <= THREADS * REG_LAUNCH, "register split exceeds the launch");
    static_assert(SMEM <= 232448, "shared memory");
};

// POLY > 0: one exponential pair in POLY on the FMA pipe (exp2_poly2), the
// rest on the MUFU
template <int D_, int POLY>
__global__ void __launch_bounds__(384, 1) fwd_sm100_kernel(const __grid_constant__ FwdArgs a)
{
    using C = FwdCfg<D_>;
    constexpr int D = C::D, BM = C::BM, BN = C::BN, KST = C::KST, VST = C::VST, KB = C::KB;
    const AttnParams &p = a.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const uint32_t sQ = base;  // slot x at sQ + x * Q_BYTES
    const uint32_t sK = base + 2 * C::Q_BYTES;
    const uint32_t sV = sK + KST * C::KV_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 2 * C::Q_BYTES + (KST + VST) * C::KV_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
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
    const SeqGeom sg = seq_geom(p, b);
    const int i0 = qt * BM;
    if (i0 >= sg.Lq) return;  // past the end of this sequence of a packed batch
    const Win w = make_win(p.S, p.N, p.G, p.W, (long long)hl + p.kv_head_offset);
    const int delta = sg.Lk - sg.Lq;
    const int nrows = min(BM, sg.Lq - i0);
    const int pa = i0 + delta, pb = i0 + nrows - 1 + delta;

    // the key tiles this query tile visits (sink, near, long; at most three
    // merged ranges), from the same closed form as the schedule builder
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
            mbar_init(P_FULL(x), 4);  // one arrival per softmax warp
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
            // K runs one tile ahead of V: iteration i loads K_i and V_{i-1}
            if (lane == 0) {
                mbar_expect_tx(BAR_Q, nslot * C::Q_BYTES);
                for (int x = 0; x < nslot; ++x)
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_4d(sQ + x * C::Q_BYTES + kb * BM * 128, &a.tq, BAR_Q, kb * 64, sg.qoff + i0,
                                    hq0 + x, sg.tb);
                int kiss = 0, viss = 0;  // K and V tiles issued
                bool good = true;
                for (int i = 0; good && i <= ntiles; ++i) {
                    if (i < ntiles) {
                        const int s = i % KST;
                        if (i >= KST && !(good = mbar_wait(K_EMPTY(s), ((i / KST) - 1) & 1, p.err, abort_flag)))
                            break;
                        const int kt = tile_of(i);
                        if (!(good = dcheck(kt >= 0 && kt * BN < sg.Lk, p.err))) {  // a listed tile holds keys
                            *abort_flag = 1;
                            break;
                        }
                        mbar_expect_tx(K_FULL(s), C::KV_BYTES);
                        for (int kb = 0; kb < KB; ++kb)
                            tma_load_4d(sK + s * C::KV_BYTES + kb * BN * 128, &a.tk, K_FULL(s), kb * 64,
                                        sg.koff + kt * BN, hl, sg.tb);
                        kiss = i + 1;
                    }
                    if (i > 0) {
                        const int u = i - 1, s = u % VST;
                        if (u >= VST && !(good = mbar_wait(V_EMPTY(s), ((u / VST) - 1) & 1, p.err, abort_flag)))
                            break;
                        mbar_expect_tx(V_FULL(s), C::KV_BYTES);
                        for (int kb = 0; kb < KB; ++kb)
                            tma_load_4d(sV + s * C::KV_BYTES + kb * BN * 128, &a.tv, V_FULL(s), kb * 64,
                                        sg.koff + tile_of(u) * BN, hl, sg.tb);
                        viss = i;
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
            // the whole warp runs the loop; one elected lane issues.  Issuer
            // x, per tile t: S_x(t) once the score region is free (the other
            // slot's softmax holds S(t-1) for slot 0, slot 0's holds S_0(t)
            // for slot 1; a lone slot waits for its own), then PV_x(t-1)
            // once P_x(t-1) is written.
            const uint32_t FULL = 0xffffffffu;
            const int x = warp - 9;  // head slot served
            const int other = nslot == 2 ? x ^ 1 : x;
            bool ok = x < nslot && __all_sync(FULL, mbar_wait(BAR_Q, 0, p.err, abort_flag));
            const uint64_t dq0 = sdesc(sQ, 16, 1024);
            const uint64_t dk0 = sdesc(sK, 16, 1024);
            const uint64_t dv0 = sdesc(sV, BN * 128, 1024);
            auto pv = [&](int u) -> bool {  // O_x += P_x(u) V_u
                if (!__all_sync(FULL, mbar_wait(V_FULL(u % VST), (u / VST) & 1, p.err, abort_flag))) return false;
                if (!__all_sync(FULL, mbar_wait(P_FULL(x), u & 1, p.err, abort_flag))) return false;
                tc_fence_after();
                const uint32_t vo = (uint32_t)(u % VST) * C::KV_BYTES;
                if (elect_one()) {
#pragma unroll
                    for (int k2 = 0; k2 < BN / 16; ++k2)
                        mma_ts(tmem + C::t_o(x), tmem + C::t_p(x) + k2 * 8, sdesc_add(dv0, vo + k2 * 2048),
                               C::IDESC_O, (u > 0 || k2 > 0) ? 1u : 0u);
                    mma_commit(O_DONE(x));
                    mma_commit(V_EMPTY(u % VST));  // this head is done with V_u
                }
                __syncwarp();
                return true;
            };
            for (int t = 0; ok && t < ntiles; ++t) {
                if (!(ok = __all_sync(FULL, mbar_wait(K_FULL(t % KST), (t / KST) & 1, p.err, abort_flag)))) break;
                // the score region: slot 1's S(t) follows slot 0's S(t), slot
                // 0's S(t) follows slot 1's S(t-1) (phase t of S_FREE(0), phase
                // t-1 of S_FREE(1))
                const int ph = x == 1 && nslot == 2 ? t : t - 1;
                if (ph >= 0 && !(ok = __all_sync(FULL, mbar_wait(S_FREE(other), ph & 1, p.err, abort_flag)))) break;
                tc_fence_after();
                const uint32_t ko = (uint32_t)(t % KST) * C::KV_BYTES;
                if (elect_one()) {  // S_x(t) = Q_x K_t^T
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk & 3) * 32;
                        const uint64_t ad = sdesc_add(dq0, x * C::Q_BYTES + (kk >> 2) * BM * 128 + off);
                        const uint64_t bd = sdesc_add(dk0, ko + (kk >> 2) * BN * 128 + off);
                        mma_ss(tmem + C::T_S, ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(S_FULL(x));
                    mma_commit(K_EMPTY(t % KST));  // this head is done with K_t
                }
                __syncwarp();
                if (t > 0 && !(ok = pv(t - 1))) break;
            }
            if (ok && ntiles > 0) ok = pv(ntiles - 1);
            if (x < nslot) {
                if (elect_one()) mma_commit(FIN(x));
                __syncwarp();
                mbar_wait(FIN(x), 0, p.err, abort_flag);
            }
        }
    } else {
        setmaxnreg_inc<C::REG_SOFTMAX>();
        // ---------------------------------------------------------- softmax
        const int x = warp >> 2;  // head slot of this warpgroup
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + C::T_S + lane_off;
        const uint32_t tP = tmem + C::t_p(x) + lane_off;
        const uint32_t tOx = tmem + C::t_o(x) + lane_off;
        const int prow = pa + r;
        const bool active = x < nslot;
        // the keys row prow sees (sink, long, near), as runs formed once: a
        // tile needs no mask when one run holds it for every row of the warp
        // (a valid row's runs end at its own position, so a tile reaching
        // past the sequence's last key is never held)
        const Runs3 rr = row_key_runs(prow, w);
        float m_run = -CUDART_INF_F, l = 0.f, lb = 0.f;  // l: fp32 sum of P; lb: sum of the bf16 P
        bool ok = true;
        for (int t = 0; active && t < ntiles; ++t) {
            const int j0 = tile_of(t) * BN;
            const bool full = __all_sync(0xffffffffu, runs_cover(rr, j0, j0 + BN - 1));
            ok = __all_sync(0xffffffffu, mbar_wait(S_FULL(x), t & 1, p.err, abort_flag));
            if (!ok) break;
            tc_fence_after();
            // one read of the row of S: the chunks are requested back to back
            // and waited for once
            uint32_t sr[BN];
            float mx4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) mx4[k] = -CUDART_INF_F;
            // two halves: the max of the first runs while the second loads
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h == 0) {
                    tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                    tmem_wait_ld();
                    tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
                    tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
                } else {
                    tmem_wait_ld();
                    // the row is in registers: the next score MMA may overwrite S
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(S_FREE(x));
                }
                if (!full) {
#pragma unroll
                    for (int c = 2 * h; c < 2 * h + 2; ++c) {
                        const uint32_t vis = runs_bits(rr, j0 + c * 32);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (!((vis >> e) & 1u)) sr[c * 32 + e] = __float_as_uint(-CUDART_INF_F);
                    }
                }
#pragma unroll
                for (int e = 64 * h; e < 64 * h + 64; e += 8) {
                    mx4[0] = max3(mx4[0], __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
                    mx4[1] = max3(mx4[1], __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
                    mx4[2] = max3(mx4[2], __uint_as_float(sr[e + 4]), __uint_as_float(sr[e + 5]));
                    mx4[3] = max3(mx4[3], __uint_as_float(sr[e + 6]), __uint_as_float(sr[e + 7]));
                }
            }
            const float smax = fmaxf(max3(mx4[0], mx4[1], mx4[2]), mx4[3]);
            const float tmax = smax * p.scale_log2;  // scale > 0 keeps the order
            // lazy rescale: keep the old reference max unless it is exceeded by 2^8
            const bool grow = tmax > m_run + 8.f;
            const float alpha = grow ? fast_ex2(m_run - tmax) : 1.f;
            const bool fix_o = grow && m_run != -CUDART_INF_F;
            if (grow) {
                l *= alpha;
                lb *= alpha;
                m_run = tmax;
            }
            const float nms = m_run == -CUDART_INF_F ? 0.f : -m_run;
            // P = 2^(s*scale - m) as bf16, two keys per packed f32x2 op;
            // packed entry e (< BN/2) takes keys 2e and 2e+1 and is written
            // over sr[e], already consumed
            const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(nms, nms);
            float2 la = make_float2(0.f, 0.f), lc = make_float2(0.f, 0.f), lba = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < BN / 2; ++e) {
                const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                             sc2, nm2);
                float p0, p1;
                if (POLY && e % (POLY > 0 ? POLY : 1) == POLY - 1) {  // FMA pipe, the rest on the MUFU
                    const float2 pp = exp2_poly2(xa);
                    p0 = pp.x;
                    p1 = pp.y;
                } else {
                    p0 = fast_ex2(xa.x);
                    p1 = fast_ex2(xa.y);
                }
                if (e & 1)
                    lc = __fadd2_rn(lc, make_float2(p0, p1));
                else
                    la = __fadd2_rn(la, make_float2(p0, p1));
                const uint32_t pk = pack2(p0, p1);
                lba = __fadd2_rn(lba, make_float2(__uint_as_float(pk << 16), __uint_as_float(pk & 0xffff0000u)));
                sr[e] = pk;
            }
            l += (la.x + la.y) + (lc.x + lc.y);
            lb += lba.x + lba.y;
            // P_x and O_x are rewritten from here on: PV_x(t-1) must be
            // complete (O_DONE(x) has completed t-1 or t phases: PV_x(t)
            // waits for the P_FULL arrival below)
            if (t > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(O_DONE(x), (t - 1) & 1, p.err, abort_flag));
                if (!ok) break;
                tc_fence_after();
            }
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_st16(tP + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[c * 16]));
            if (__any_sync(0xffffffffu, fix_o)) {
                // O holds tiles < t weighted against the old max: scale its row
                const float f = fix_o ? alpha : 1.f;
#pragma unroll
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t o[16];
                    const uint32_t ta = tOx + c * 16;
                    tmem_ld16(ta, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                    tmem_st16(ta, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(P_FULL(x));
        }
        // every MMA of this slot has completed (FIN follows the last PV)
        if (active) ok = __all_sync(0xffffffffu, ok && mbar_wait(FIN(x), 0, p.err, abort_flag));
        tc_fence_after();
        // epilogue: O / (sum of the bf16 P) in bf16, LSE (natural log) from the fp32 sum
        if (active) {
            const bool have = ok && ntiles > 0;
            const float inv = (l > 0.f && lb > 0.f) ? 1.f / lb : 0.f;
            const int hq = hq0 + x;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + sg.tb * p.os[0] +
                                  (long long)(sg.qoff + i0 + r) * p.os[1] + hq * p.os[2];
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
                uint32_t o[16];
                if (have) {
                    tmem_ld16(tOx + c * 16, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = 0u;
                }
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    pk[e] = pack2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                if (r < nrows && dcheck(sg.qoff + i0 + r < (p.cu_q ? p.total_q : p.Lq) && hq < p.Hq, p.err)) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 16);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            if (r < nrows && dcheck(sg.qoff + i0 + r < p.lse_ld, p.err))
                p.lse[((long long)sg.tb * p.Hq + hq) * p.lse_ld + sg.qoff + i0 + r] =
                    l > 0.f ? m_run * 0.69314718055994531f + logf(l) : -CUDART_INF_F;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, 512);
}

// ----------------------------------------------------------------- host ----
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

}  // namespace

// [B, L, H, d] bf16 tensor (strides in elements for b, l, h) as a 4-D map
// with 64-element x `rows` boxes and 128-byte swizzle.
bool make_bshd_map(CUtensorMap *m, const void *base, int d, long long L, long long H, long long B,
                   const long long st[3], int rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)st[1] * 2, (cuuint64_t)st[2] * 2, (cuuint64_t)st[0] * 2};
    for (int k = 0; k < 3; ++k)
        if (strides[k] == 0) strides[k] = 16;  // a dimension of extent 1 with stride 0
    cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_fwd_d(const AttnParams &p, cudaStream_t st)
{
    using C = FwdCfg<D>;
    // one exponential pair in eight on the FMA pipe: measured faster than
    // none (the two slots' softmax warps share the MUFU) and than one in four
    // (and at d = 64 than one in two, three, four or six)
    constexpr int POLY = 8;
    static std::atomic<bool> configured[64];
    cudaError_t e = once_per_device(configured, [] {
        cudaError_t r =
            cudaFuncSetAttribute(fwd_sm100_kernel<D, POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        // the register split assumes the launch count it was planned for: a
        // build with fewer registers per thread at launch is not run
        cudaFuncAttributes fa;
        if (r == cudaSuccess) r = cudaFuncGetAttributes(&fa, fwd_sm100_kernel<D, POLY>);
        if (r == cudaSuccess && fa.numRegs < C::REG_LAUNCH) r = cudaErrorInvalidDeviceFunction;
        return r;
    });
    if (e != cudaSuccess) return e;
    FwdArgs a;
    memset(&a, 0, sizeof a);
    a.p = p;
    a.npair = (p.g + 1) / 2;
    // a packed batch is one batch entry of total_q / total_k rows
    const long long Lq_map = p.cu_q ? p.total_q : p.Lq, Lk_map = p.cu_q ? p.total_k : p.Lk;
    const long long B_map = p.cu_q ? 1 : p.B;
    if (!make_bshd_map(&a.tq, p.q, C::D, Lq_map, p.Hq, B_map, p.qs, C::BM) ||
        !make_bshd_map(&a.tk, p.k, C::D, Lk_map, p.Hkv, B_map, p.ks, C::BN) ||
        !make_bshd_map(&a.tv, p.v, C::D, Lk_map, p.Hkv, B_map, p.vs, C::BN))
        return cudaErrorInvalidValue;
    const unsigned blocks = p.work ? tile_grid_blocks(p.work_n, (long long)p.Hkv * a.npair, 1)
                                   : tile_grid_blocks(p.nqt, (long long)p.Hkv * a.npair, p.B);
    if (!blocks) return cudaErrorInvalidConfiguration;
    launch_begin("fwd_sm100", st);
    fwd_sm100_kernel<D, POLY><<<blocks, C::THREADS, C::SMEM, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

cudaError_t launch_fwd_sm100(const AttnParams &p, int D, cudaStream_t st)
{
    if (p.nqt == 0 || p.Hq == 0 || p.B == 0) return cudaSuccess;
    return D == 128 ? launch_fwd_d<128>(p, st) : launch_fwd_d<64>(p, st);
}

}  // namespace cowa
