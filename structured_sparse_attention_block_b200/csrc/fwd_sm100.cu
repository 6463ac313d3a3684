// CoWA training / prefill forward on the 5th-generation tensor cores, d = 64
// (d = 128 runs the kernel of fwd_d128.cu, built on the same plan with 128-key
// tiles).
//
// One CTA per (query tile of 128 rows, pair of query heads of one GQA group,
// batch).  Two query heads of a group have the same KV head, hence the same
// window mask and the same visible key tiles, so the CTA streams each K/V
// tile once for both and neither head wastes work.  Eleven warps:
//   warp 8     TMA producer: both Q tiles once, then the K and V tiles the
//              schedule lists (sink, near and long bands only) into a ring of
//              shared-memory stages;
//   warps 9,10 MMA issuers, one thread each, warp 9 + x serving head slot x
//              (warp 9 also owns the tensor memory): S_x(t) = Q_x K_t^T into
//              S_x, and O_x += P_x(t) V_t
//              with P_x(t) read from its own tensor-memory region (a later MMA
//              writing S_x is not ordered after an earlier MMA's read of P from
//              the same columns, so P never shares columns with S).  S_x(t+1)
//              is issued as soon as softmax x has pulled S_x(t) into registers
//              (S_FREE), so the next score tile is computed while the softmax
//              of the current one runs; PV_x(t) follows when P_x(t) is written
//              (P_FULL).  Order per tile and slot: S_x(t+1) PV_x(t).  The two
//              slots touch disjoint tensor-memory columns, so their issuers
//              need no ordering between them, and neither slot's waits hold up
//              the other's MMAs; K_t and V_t are released once both issuers
//              have committed their tile-t MMAs;
//   warps 0-3  softmax of slot 0, warps 4-7 softmax of slot 1: thread r of a
//              warpgroup owns query row r.  Pass 1 reads the row of S in
//              32-column chunks and takes the max (edge tiles only apply the
//              element mask); pass 2 re-reads S, writes P = 2^(s*scale - m) as
//              bf16 to P_x and sums P in fp32 for the LSE.  The normalisation
//              of O uses the sum of the bf16 P the PV product used: each
//              stage holds a block of ones after V, so the PV MMA, 16 columns
//              wider than d, accumulates that sum next to O, and O is divided
//              by exactly the weights it accumulated.  The O row is
//              rescaled in tensor memory only when the max grows by more than
//              2^8 (until then the stale max is a valid reference point).
// Key tiles are 96 wide: a softmax thread reads its whole row of S_x with one
// tensor-memory round trip and keeps it in registers.  Tensor-memory columns
// (O_x is d + 16 wide: O, then the bf16 row sums): S_x at 96x, P_x at
// 192 + 64x, O_x at 320 + 96x.
// Softmax x rewrites P_x and rescales O_x for tile t only after O_DONE_x says
// PV_x(t-1) is complete.
// The exponential loops of the two slots alternate per lane quadrant (the two
// warps on one SM sub-partition): slot 1 runs tile t's after slot 0 has run
// its own, and slot 0 runs tile t+1's after slot 1's tile t.  Without this the
// two warps reach the exponentials together, share the MUFU and issue slots
// there, and leave them idle while both wait on tensor-memory loads; with it
// one warp's exponentials overlap the other's loads, max and stores.
// Every mbarrier wait is bounded; a wait that runs out records a timeout in
// the device error word and the CTA winds down.
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

template <int D>
struct FwdCfg {
    static_assert(D == 64, "d = 128 has its own kernel");
    static constexpr int BM = 128, BN = fwd5_bn(D);
    static constexpr int STAGES = 4;  // tiles t, t+1, t+2 are resident at once
    // tensor-memory column of S_x, P_x, O_x
    static constexpr __host__ __device__ int t_s(int x) { return 96 * x; }
    static constexpr __host__ __device__ int t_p(int x) { return 192 + 64 * x; }
    static constexpr __host__ __device__ int t_o(int x) { return 320 + 96 * x; }
    static constexpr int OW = D + 16;                 // O columns, then the bf16 row sums
    // exponentials on the FMA pipe: one pair in four, where the softmax paces
    // the kernel (measured against none, one in two and one in three)
    static constexpr int POLY_EVERY = 4;
    static constexpr int KB = D / 64;                 // 128-byte blocks along d
    static constexpr int Q_BYTES = BM * D * 2;        // one head's query tile
    static constexpr int KV_BYTES = BN * D * 2;       // one of K or V
    static constexpr int ONES_BYTES = BN * 128;       // bf16 1.0, one 128-byte row per key
    static constexpr int STAGE_BYTES = 2 * KV_BYTES + ONES_BYTES;
    static constexpr int NBAR = 20 + 2 * STAGES;
    static constexpr int SMEM = 1024 + 2 * Q_BYTES + STAGES * STAGE_BYTES + 8 * NBAR + 16;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
    static constexpr uint32_t IDESC_O = idesc_bf16(128, OW, 0, 1);
};

template <int D>
__global__ void __launch_bounds__(352, 1) fwd_sm100_kernel(const __grid_constant__ FwdArgs a)
{
    using C = FwdCfg<D>;
    constexpr int BM = C::BM, BN = C::BN, ST = C::STAGES, KB = C::KB;
    const AttnParams &p = a.p;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const uint32_t sQ = base;  // slot x at sQ + x * Q_BYTES
    const uint32_t sStage = base + 2 * C::Q_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 2 * C::Q_BYTES + ST * C::STAGE_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t bar0 = smem_addr(bars);
    const uint32_t BAR_Q = bar0;
    auto KV_FULL = [&](int s) { return bar0 + 8u * (1 + s); };
    auto KV_EMPTY = [&](int s) { return bar0 + 8u * (1 + ST + s); };
    auto S_FULL = [&](int x) { return bar0 + 8u * (1 + 2 * ST + x); };
    auto P_FULL = [&](int x) { return bar0 + 8u * (3 + 2 * ST + x); };
    auto O_DONE = [&](int x) { return bar0 + 8u * (5 + 2 * ST + x); };
    auto S_FREE = [&](int x) { return bar0 + 8u * (7 + 2 * ST + x); };
    auto FIN = [&](int x) { return bar0 + 8u * (9 + 2 * ST + x); };
    // exponential-loop turn of slot x in lane quadrant qd
    auto TURN = [&](int x, int qd) { return bar0 + 8u * (12 + 2 * ST + 4 * x + qd); };

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
        for (int s = 0; s < ST; ++s) {
            mbar_init(KV_FULL(s), 1);
            mbar_init(KV_EMPTY(s), nslot);  // one commit per MMA issuer
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(S_FULL(x), 1);
            mbar_init(P_FULL(x), 4);  // one arrival per softmax warp
            mbar_init(O_DONE(x), 1);
            mbar_init(S_FREE(x), 4);  // one arrival per softmax warp
            for (int qd = 0; qd < 4; ++qd) mbar_init(TURN(x, qd), 1);
        }
        mbar_init(FIN(0), 1);
        mbar_init(FIN(1), 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 9) {
        tmem_alloc(smem_addr(tmem_slot), 512);
        tmem_relinquish();
    }
    // the ones block of every stage (TMA never writes it); the PV MMA reads it
    // as B columns d .. d+15, any swizzle of an all-ones row reads ones
    for (int s = 0; s < ST; ++s) {
        uint32_t *ones = reinterpret_cast<uint32_t *>(sm + 2 * C::Q_BYTES + s * C::STAGE_BYTES + 2 * C::KV_BYTES);
        for (int k = tid; k < C::ONES_BYTES / 4; k += blockDim.x) ones[k] = 0x3F803F80u;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&a.tq);
        prefetch_tmap(&a.tk);
        prefetch_tmap(&a.tv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            const SeqGeom sp = seq_geom(p, b);  // row offsets in the tensors
            mbar_expect_tx(BAR_Q, nslot * C::Q_BYTES);
            for (int x = 0; x < nslot; ++x)
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_4d(sQ + x * C::Q_BYTES + kb * BM * 128, &a.tq, BAR_Q, kb * 64, sp.qoff + i0, hq0 + x,
                                sp.tb);
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % ST;
                if (t >= ST && !mbar_wait(KV_EMPTY(s), ((t / ST) - 1) & 1, p.err, abort_flag)) break;
                const int kt = tile_of(t);
                if (!dcheck(kt >= 0 && kt * BN < sp.Lk, p.err)) {  // a listed tile holds keys
                    *abort_flag = 1;
                    break;
                }
                mbar_expect_tx(KV_FULL(s), 2 * C::KV_BYTES);
                const uint32_t sk = sStage + s * C::STAGE_BYTES, sv = sk + C::KV_BYTES;
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(sk + kb * BN * 128, &a.tk, KV_FULL(s), kb * 64, sp.koff + kt * BN, hl, sp.tb);
                    tma_load_4d(sv + kb * BN * 128, &a.tv, KV_FULL(s), kb * 64, sp.koff + kt * BN, hl, sp.tb);
                }
                issued = t + 1;
            }
            // every load this thread issued has landed before the CTA ends
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
        // descriptor bases: Q of slot 0, K and V of stage 0 (the others are
        // fixed byte offsets from these)
        const uint64_t dq0 = sdesc(sQ, 16, 1024);
        const uint64_t dk0 = sdesc(sStage, 16, 1024);
        const uint64_t dv0 = sdesc(sStage + C::KV_BYTES, BN * 128, 1024);
        auto qk = [&](int t) {  // S_x(t) = Q_x K_t^T
            const uint32_t so = (uint32_t)(t % ST) * C::STAGE_BYTES;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;
                    const uint64_t ad = sdesc_add(dq0, x * C::Q_BYTES + (kk >> 2) * BM * 128 + off);
                    const uint64_t bd = sdesc_add(dk0, so + (kk >> 2) * BN * 128 + off);
                    mma_ss(tmem + C::t_s(x), ad, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(S_FULL(x));
            }
            __syncwarp();
        };
        auto pv = [&](int t) -> bool {  // O_x += P_x(t) V_t
            if (!__all_sync(FULL, mbar_wait(P_FULL(x), t & 1, p.err, abort_flag))) return false;
            tc_fence_after();
            const uint32_t so = (uint32_t)(t % ST) * C::STAGE_BYTES;
            if (elect_one()) {
#pragma unroll
                for (int k2 = 0; k2 < BN / 16; ++k2)
                    mma_ts(tmem + C::t_o(x), tmem + C::t_p(x) + k2 * 8, sdesc_add(dv0, so + k2 * 2048), C::IDESC_O,
                           (t > 0 || k2 > 0) ? 1u : 0u);
                mma_commit(O_DONE(x));
            }
            __syncwarp();
            return true;
        };
        if (ntiles > 0 && (ok = ok && __all_sync(FULL, mbar_wait(KV_FULL(0), 0, p.err, abort_flag)))) {
            tc_fence_after();
            qk(0);
        }
        for (int t = 0; ok && t < ntiles; ++t) {
            const int tn = t + 1;
            if (tn < ntiles) {
                if (!(ok = __all_sync(FULL, mbar_wait(KV_FULL(tn % ST), (tn / ST) & 1, p.err, abort_flag)))) break;
                // softmax x holds S_x(t) in registers: S_x may be rewritten
                if (!(ok = __all_sync(FULL, mbar_wait(S_FREE(x), t & 1, p.err, abort_flag)))) break;
                tc_fence_after();
                qk(tn);
            }
            ok = pv(t);
            if (elect_one()) mma_commit(KV_EMPTY(t % ST));  // this head is done with K_t and V_t
            __syncwarp();
        }
        if (x < nslot) {
            if (elect_one()) mma_commit(FIN(x));
            __syncwarp();
            mbar_wait(FIN(x), 0, p.err, abort_flag);
        }
    } else {
        // -------------------------------------------------------- softmax
        const int x = warp >> 2;  // head slot of this warpgroup
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tP = tmem + C::t_p(x) + lane_off;
        const uint32_t tOx = tmem + C::t_o(x) + lane_off;
        const int prow = pa + r;
        const bool active = x < nslot;
        const bool turns = nslot == 2;  // a lone head slot takes every turn
        const uint32_t my_turn = TURN(x, warp & 3), their_turn = TURN(x ^ 1, warp & 3);
        // the keys row prow sees (sink, long, near), as runs formed once:
        // a tile needs no mask when one run holds it for every row of the
        // warp (a valid row's runs end at its own position, so a tile
        // reaching past the sequence's last key is never held)
        const Runs3 rr = row_key_runs(prow, w);
        float m_run = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        for (int t = 0; active && t < ntiles; ++t) {
            // tile set-up, independent of the scores: done while they land.
            // Edge tiles build, per 32-key chunk, the bitmask of keys the row
            // sees.
            const int j0 = tile_of(t) * BN;
            const bool full = __all_sync(0xffffffffu, runs_cover(rr, j0, j0 + BN - 1));
            constexpr int NC = BN / 32;  // 32-column chunks of the row
            uint32_t vis[NC];
            if (!full) {
#pragma unroll
                for (int c = 0; c < NC; ++c) vis[c] = runs_bits(rr, j0 + c * 32);
            }
            ok = __all_sync(0xffffffffu, mbar_wait(S_FULL(x), t & 1, p.err, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + C::t_s(x) + lane_off;
            // one read of the row of S: all chunks are requested back to back
            // and waited for once
            uint32_t sr[BN];
#pragma unroll
            for (int c = 0; c < NC; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            tmem_wait_ld();
            // the row is in registers: S_x(t+1) may overwrite S_x
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S_FREE(x));
            if (!full) {
#pragma unroll
                for (int e = 0; e < BN; ++e)
                    if (!((vis[e >> 5] >> (e & 31)) & 1u)) sr[e] = __float_as_uint(-CUDART_INF_F);
            }
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
            const float smax = fmaxf(max3(mx4[0], mx4[1], mx4[2]), mx4[3]);
            const float tmax = smax * p.scale_log2;  // scale > 0 keeps the order
            // lazy rescale: keep the old reference max unless it is exceeded by 2^8
            const bool grow = tmax > m_run + 8.f;
            const float alpha = grow ? fast_ex2(m_run - tmax) : 1.f;
            const bool fix_o = grow && m_run != -CUDART_INF_F;
            if (grow) {
                l *= alpha;
                m_run = tmax;
            }
            const float nms = m_run == -CUDART_INF_F ? 0.f : -m_run;
            // P = 2^(s*scale - m) as bf16, two keys per packed f32x2 op; packed
            // entry e (< BN/2) takes keys 2e and 2e+1 and is written over
            // sr[e], already consumed
            const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(nms, nms);
            float2 la = make_float2(0.f, 0.f), lc = make_float2(0.f, 0.f);
            // slot 1's turn for tile t is phase t of its barrier (slot 0 done
            // with tile t); slot 0's for tile t > 0 is phase t-1 of its own
            // (slot 1 done with tile t-1).  Neither can run two phases ahead
            // of the other, so the parity is unambiguous.
            if (turns && (x == 1 || t > 0)) {
                ok = __all_sync(0xffffffffu, mbar_wait(my_turn, (x == 1 ? t : t - 1) & 1, p.err, abort_flag));
                if (!ok) break;
            }
#pragma unroll
            for (int e = 0; e < BN / 2; ++e) {
                const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                             sc2, nm2);
                float p0, p1;
                constexpr int PE = C::POLY_EVERY > 0 ? C::POLY_EVERY : 1;
                if (C::POLY_EVERY && e % PE == PE - 1) {  // FMA pipe, the rest on the MUFU
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
                sr[e] = pack2(p0, p1);
            }
            if (turns) {
                __syncwarp();
                if (lane == 0) mbar_arrive(their_turn);
            }
            l += (la.x + la.y) + (lc.x + lc.y);
            // P_x and O_x are rewritten from here on: PV_x(t-1) must be complete
            // (O_DONE(x) has completed t-1 or t phases: PV_x(t) waits for the
            // P_FULL arrival below)
            if (t > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(O_DONE(x), (t - 1) & 1, p.err, abort_flag));
                if (!ok) break;
                tc_fence_after();
            }
#pragma unroll
            for (int c = 0; c < NC; ++c) tmem_st16(tP + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[c * 16]));
            if (__any_sync(0xffffffffu, fix_o)) {
                // O holds tiles < t weighted against the old max: scale its row
                const float f = fix_o ? alpha : 1.f;
#pragma unroll
                for (int c = 0; c < C::OW / 16; ++c) {  // O and its bf16 row sums
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
        if (active && ok && ntiles > 0) {
            // PV_x(ntiles-2) was waited for at the last tile, so O_DONE(x) has
            // completed ntiles-1 or ntiles phases: the parity of the last one is
            // unambiguous (a parity wait only tells apart adjacent phases)
            ok = __all_sync(0xffffffffu, mbar_wait(O_DONE(x), (ntiles - 1) & 1, p.err, abort_flag));
        }
        tc_fence_after();
        // epilogue: O / (sum of the bf16 P) in bf16, LSE (natural log) from the fp32 sum
        if (active) {
            // the sequence's offsets again, rather than live across the tile loop
            const SeqGeom se = seq_geom(p, b);
            const bool have = ok && ntiles > 0;
            float lb = 0.f;  // sum of the bf16 P that O accumulated
            if (have) {
                uint32_t lv[16];
                tmem_ld16(tOx + D, lv);
                tmem_wait_ld();
                lb = __uint_as_float(lv[0]);
            }
            const float inv = (l > 0.f && lb > 0.f) ? 1.f / lb : 0.f;
            const int hq = hq0 + x;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + se.tb * p.os[0] +
                                  (long long)(se.qoff + i0 + r) * p.os[1] + hq * p.os[2];
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
                if (r < nrows && dcheck(se.qoff + i0 + r < (p.cu_q ? p.total_q : p.Lq) && hq < p.Hq, p.err)) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 16);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            if (r < nrows && dcheck(se.qoff + i0 + r < p.lse_ld, p.err))
                p.lse[((long long)se.tb * p.Hq + hq) * p.lse_ld + se.qoff + i0 + r] =
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
static cudaError_t launch_fwd5_d(const AttnParams &p, cudaStream_t st)
{
    using C = FwdCfg<D>;
    static std::atomic<bool> configured[64];
    cudaError_t e = once_per_device(configured, [] {
        return cudaFuncSetAttribute(fwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    });
    if (e != cudaSuccess) return e;
    FwdArgs a;
    memset(&a, 0, sizeof a);
    a.p = p;
    a.npair = (p.g + 1) / 2;
    // a packed batch is one batch entry of total_q / total_k rows
    const long long Lq_map = p.cu_q ? p.total_q : p.Lq, Lk_map = p.cu_q ? p.total_k : p.Lk;
    const long long B_map = p.cu_q ? 1 : p.B;
    if (!make_bshd_map(&a.tq, p.q, D, Lq_map, p.Hq, B_map, p.qs, C::BM) ||
        !make_bshd_map(&a.tk, p.k, D, Lk_map, p.Hkv, B_map, p.ks, C::BN) ||
        !make_bshd_map(&a.tv, p.v, D, Lk_map, p.Hkv, B_map, p.vs, C::BN))
        return cudaErrorInvalidValue;
    const unsigned blocks = p.work ? tile_grid_blocks(p.work_n, (long long)p.Hkv * a.npair, 1)
                                   : tile_grid_blocks(p.nqt, (long long)p.Hkv * a.npair, p.B);
    if (!blocks) return cudaErrorInvalidConfiguration;
    launch_begin("fwd_sm100", st);
    fwd_sm100_kernel<D><<<blocks, 352, C::SMEM, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

cudaError_t launch_fwd_sm100(const AttnParams &p, int D, cudaStream_t st)
{
    if (p.nqt == 0 || p.Hq == 0 || p.B == 0) return cudaSuccess;
    return D == 128 ? launch_fwd_d128(p, st) : launch_fwd5_d<64>(p, st);
}

}  // namespace cowa
