// Kernel parameter blocks and launcher declarations shared by api.cu and the
// kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace cowa {

// One-time set-up of a device for a group of kernels (their dynamic
// shared-memory limits): `fn` runs on the current device until it succeeds
// once there.  Host threads that make their first call at the same time may
// both run it, which is harmless: it only sets idempotent attributes.
template <class F>
cudaError_t once_per_device(std::atomic<bool> (&done)[64], F fn)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (done[dev & 63].load(std::memory_order_acquire)) return cudaSuccess;
    e = fn();
    if (e == cudaSuccess) done[dev & 63].store(true, std::memory_order_release);
    return e;
}

// Checking build (compiled with -DCOWA_DEBUG into libcowa_debug.so):
// device-side checks of tile, row and workspace indices against the extents
// they must stay within.  A failed check records COWA_ERR_DEVICE (7) in the
// device error word and the caller skips the guarded access (a tcgen05 CTA
// also raises its abort flag, so its pipeline winds down through the bounded
// waits); nothing traps.  In the release build every check is the constant
// true and compiles away.
__device__ __forceinline__ bool dcheck(bool ok, int *err)
{
#ifdef COWA_DEBUG
    if (!ok) atomicExch(err, 7);
    return ok;
#else
    (void)ok;
    (void)err;
    return true;
#endif
}

struct AttnParams {
    const void *q, *k, *v;
    void *o;
    float *lse;
    const void *dout;
    const float *lse_in;
    void *dq, *dk, *dv;
    long long qs[3], ks[3], vs[3], os[3];
    int B, Lq, Lk, Hq, Hkv, g;
    int S, N, G, W;
    int kv_head_offset;
    int nqt, nkt;           // query / key tiles of the launch
    float scale, scale_log2;
    int *err;               // device error word (status code of a failed device check)
    // Packed (variable-length) batch: sequence b owns query rows
    // [cu_q[b], cu_q[b+1]) and key rows [cu_k[b], cu_k[b+1]) of tensors with
    // total_q / total_k rows; Lq / Lk are then the longest sequence.  With
    // cu_q == nullptr the batch is uniform (B sequences of Lq / Lk rows).
    const int *cu_q, *cu_k;
    int total_q, total_k;
    long long lse_ld;                 // LSE row pitch: Lq, or total_q when packed
    // MALA backward: the forward's block decisions keep[b][hq][i / kMalaBM]
    // [j / kMalaBN] (nullptr for CoWA); a pair of a skipped block has dP = 0
    // and contributes nothing to dV (only -P * delta remains in dS)
    const uint8_t *keep;
    int keep_nqt, keep_nkt;
    // Packed batch: the (sequence, tile) items of the launch's tiling, heavy
    // tiles first (worklist.cu), work_n entries (the last ones (-1, -1));
    // the grid is work_n x head slots.  nullptr for a uniform batch.
    const int2 *work;
    int work_n;
    int work_n0;  // key-major list: its first work_n0 items are the tiles of rank 0 (at most one per sequence)
};

// The tile, head slot and batch entry of a CTA of a query-major pass
// (forward, dQ), whose head slots are numbered KV head by KV head (spk slots
// each).  A uniform batch's 1-D grid runs over groups of two KV heads
// (one for an odd count), and within a group over (head slot, batch)
// fastest and the tile step slowest, the last query tile first: the CTAs
// resident together then read the K/V windows of two KV heads only, which
// L2 holds (all KV heads' windows at 128K are about 100 MB), and each
// group's long CTAs start before its short ones.  A packed batch's grid
// has the same grouping over the work list's items (heaviest first) in
// place of the tile steps.  False when the CTA has no item.
__device__ __forceinline__ bool query_tile_item(const AttnParams &p, int nslot, int spk, int &qt, int &slot, int &b)
{
    const unsigned gs = (unsigned)spk * ((p.Hkv % 2 == 0) ? 2u : 1u);  // head slots per group
    if (p.work) {
        // the same grouping over the list's items (heaviest first)
        const unsigned per = gs * (unsigned)p.work_n, lin = blockIdx.x;
        const unsigned grp = lin / per, rg = lin - grp * per;
        const unsigned item = rg / gs;
        slot = (int)(grp * gs + (rg - item * gs));
        const int2 it = p.work[item];
        b = it.x;
        qt = it.y;
        return it.x >= 0;
    }
    const unsigned per = gs * (unsigned)p.B, lin = blockIdx.x;
    const unsigned grp_n = per * (unsigned)p.nqt;
    const unsigned grp = lin / grp_n, rg = lin - grp * grp_n;
    const int step = (int)(rg / per);
    const unsigned r = rg - (unsigned)step * per;
    b = (int)(r / gs);
    slot = (int)(grp * gs + (r - (unsigned)b * gs));
    qt = p.nqt - 1 - step;
    return true;
}

// Lengths and row offsets of sequence b, and its batch coordinate (b for a
// uniform batch, 0 for a packed one, whose rows are offsets into batch 0).
// A packed sequence whose offsets do not fit its tensors or exceed the
// longest length is reported and treated as empty.
struct SeqGeom {
    int Lq, Lk, qoff, koff, tb;
};
__device__ __forceinline__ SeqGeom seq_geom(const AttnParams &p, int b)
{
    SeqGeom g;
    if (!p.cu_q) {
        g.Lq = p.Lq;
        g.Lk = p.Lk;
        g.qoff = g.koff = 0;
        g.tb = b;
        return g;
    }
    g.qoff = p.cu_q[b];
    g.koff = p.cu_k[b];
    g.Lq = p.cu_q[b + 1] - g.qoff;
    g.Lk = p.cu_k[b + 1] - g.koff;
    g.tb = 0;
    const bool ok = g.qoff >= 0 && g.koff >= 0 && g.Lq >= 0 && g.Lk >= 0 && g.Lq <= p.Lq && g.Lk <= p.Lk &&
                    g.qoff <= p.total_q - g.Lq && g.koff <= p.total_k - g.Lk;
    if (!ok) {
        if (threadIdx.x == 0) atomicExch(p.err, 7);
        g.Lq = g.Lk = g.qoff = g.koff = 0;
    }
    return g;
}

struct DecodeParams {
    const void *q, *kc, *vc;
    const int *seqlens;
    void *o;
    float *lse;
    float *part_o, *part_lse;
    long long qs[3], ks[3], vs[3], os[3];
    int B, Lcap, Hq, Hkv, g, splits;
    int S, N, G, W;
    int kv_head_offset;
    float scale, scale_log2;
    int *err;
    // windowed cache: per-sequence origin positions (nullptr for a full cache)
    // and the horizon of query positions [origin, origin + horizon) it serves
    const int *origin;
    int horizon;
};

// Building and appending to a windowed decode cache (decode.cu).  The cache
// is [B, rows, Hkv, d] contiguous bf16; the source is strided (b, l, h).
struct WCacheParams {
    const void *ksrc, *vsrc;
    void *kw, *vw;
    const int *origin, *pos;
    long long ks[3], vs[3];
    int B, Hkv, rows, horizon, Lsrc;
    int S, N, G, W, kv_head_offset;
    int *err;
};
cudaError_t launch_wcache_build(const WCacheParams &p, int D, cudaStream_t st);
cudaError_t launch_wcache_append(const WCacheParams &p, int D, cudaStream_t st);

// api.cu: every kernel launch of the library is bracketed by these two calls:
// they count launches and, while tracing is on, record a CUDA event pair on
// the launching stream under the kernel's name.
void launch_begin(const char *name, cudaStream_t st);
void launch_end(cudaStream_t st);

// schedule.cu
cudaError_t launch_schedule(int *sched, int Hkv, int kv_head_offset, int Lq,
                            int Lk, int S, int N, int G, int W, int BM, int BN, int transposed,
                            cudaStream_t st);
cudaError_t launch_tile_classes(const int *sched, uint8_t *out, int kv_head, int Lq, int Lk,
                                int S, int N, int G, int W, int BM, int BN, int transposed,
                                cudaStream_t st);


// fwd_sm100.cu (tcgen05 forward)
cudaError_t launch_fwd_sm100(const AttnParams &p, int D, cudaStream_t st);
constexpr int kFwd5BM = 128;
// key-tile width of the tcgen05 forward (a softmax thread holds one row of
// a tile in registers)
__host__ __device__ constexpr int fwd5_bn(int) { return 128; }
// [B, L, H, d] bf16 tensor as a 4-D TMA map, 64-element x `rows` boxes, 128-byte swizzle
bool make_bshd_map(CUtensorMap *m, const void *base, int d, long long L, long long H, long long B,
                   const long long st[3], int rows);

// mala.cu (MALA forward): blocks of kMalaBM query rows x kMalaBN keys decide
// together; keep[b][hq][qt][kt] receives the decisions
constexpr int kMalaBM = 128, kMalaBN = 64;
cudaError_t launch_mala_fwd(const AttnParams &p, int D, uint8_t *keep, float tau, cudaStream_t st);
// mala_d128.cu: the d = 128 MALA forward, called by launch_mala_fwd
cudaError_t launch_mala_fwd_d128(const AttnParams &p, uint8_t *keep, float tau, cudaStream_t st);

// worklist.cu: the (sequence, tile) items of a packed batch for tiles of
// `tile` rows of the offsets cu [B + 1] (descending: the query-major order,
// last tile of each sequence first; else ascending: the key-major order),
// max_items entries (>= sum of the sequences' tile counts; the rest
// (-1, -1)); scratch: 3 * (max_tiles + 1) ints, max_tiles >= any
// sequence's tile count
cudaError_t launch_varlen_worklist(const int *cu, int B, int tile, int max_tiles, bool descending, int2 *list,
                                   int max_items, int *scratch, int *err, cudaStream_t st);

// fill.cu: constant outputs of the shapes the tcgen05 kernels do not take
// (zero rows of a strided [B, L, H, D] bf16 tensor; a constant fp32 array)
cudaError_t launch_zero_rows(void *t, const long long st[3], int B, int L, int H, int D, cudaStream_t s);
cudaError_t launch_fill_f32(float *p, long long n, float v, cudaStream_t s);


// bwd_sm100.cu (tcgen05 backward: preprocess, dK/dV pass, dQ pass)
// work_q / work_k: the query- and key-major work lists of a packed batch
// (nullptr for a uniform batch)
cudaError_t launch_bwd_sm100(const AttnParams &p, int D, float2 *lsd, int lq_pad, int nqt_dq, int nkt_kv,
                             cudaStream_t st, const int2 *work_q = nullptr, int work_q_n = 0,
                             const int2 *work_k = nullptr, int work_k_n = 0);
constexpr int kBwd5KeyTile = 128;   // keys per dK/dV CTA (tensor-memory lanes)
constexpr int kBwd5QTile = 128;     // queries per dQ CTA
__host__ __device__ constexpr int bwd5_kv_bm(int D) { return D == 128 ? 32 : 64; }    // queries per dK/dV task
__host__ __device__ constexpr int bwd5_dq_bn(int D) { return D == 128 ? 128 : 64; }   // keys per dQ tile
inline long long bwd5_lq_pad(long long Lq) { return (Lq + 63) / 64 * 64; }

// 1-D grid position of the MALA forward: (query head, batch) fastest, the
// tile step slowest (its kernel maps step 0 to the last query tile).  The
// CoWA passes use query_tile_item above and the dK/dV pass its own order
// (sink tiles first, then key tiles ascending head by head).
struct TilePos {
    int step, slot, b;
};
__device__ __forceinline__ TilePos tile_pos(int nslot, int B)
{
    const unsigned per = (unsigned)nslot * (unsigned)B;
    const unsigned lin = blockIdx.x;
    TilePos t;
    t.step = (int)(lin / per);
    const unsigned r = lin - (unsigned)t.step * per;
    t.b = (int)(r / (unsigned)nslot);
    t.slot = (int)(r - (unsigned)t.b * (unsigned)nslot);
    return t;
}
// Blocks of such a grid, or 0 when it would exceed the 2^31 - 1 limit.
inline unsigned tile_grid_blocks(long long ntile, long long nslot, long long B)
{
    const long long n = ntile * nslot * B;
    return n > 0x7fffffffll ? 0u : (unsigned)n;
}

// decode.cu
cudaError_t launch_decode(const DecodeParams &p, int D, cudaStream_t st);
constexpr int kDecBN = 64;
// shared memory of one split CTA: three K/V stages of kDecBN keys and the
// 16-row query block; CTAs of it that fit on one SM (228 KB, 128 threads)
constexpr int decode_smem_bytes(int D) { return (6 * kDecBN * D + 16 * D) * 2; }
constexpr int decode_ctas_per_sm(int D) { return (228 * 1024) / (decode_smem_bytes(D) + 1024); }

}  // namespace cowa
