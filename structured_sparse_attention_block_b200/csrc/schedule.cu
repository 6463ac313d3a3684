// Visible-tile schedule builder.
//
// "Block traversal skips invisible KV blocks directly, with no selection
// overhead" (CoWindow Attention paper digest, execution notes): because the
// pattern depends only on positions and the KV-head index, the tiles each
// query tile must visit are a closed-form function of the shape.  For every
// (KV head, query tile) this kernel writes the sink / near / long key-tile
// ranges, merged into at most three disjoint sorted ranges; the key-tile
// major form (for dK/dV) lists, for every key tile, the query tiles that see
// it.  The tcgen05 kernels evaluate the same closed form per CTA
// (query_tile_ranges / key_tile_ranges) instead of reading this table; it
// serves cowa_tile_classes, the schedule as a table that tests compare with
// brute force, with each visited tile labelled full or partial by
// tile_full().  (The kernels decide per warp instead: a warp skips the mask
// when each of its threads' visible runs covers the tile, which holds for
// every warp of a full tile and for no warp whose rows see only part of it.)
#include "common.cuh"
#include "kernels.cuh"

namespace cowa {

__global__ void schedule_kernel(int *sched, int kv_head_offset, int Lq, int Lk, int S, int N,
                                int G, int W, int BM, int BN, int transposed, int ntile)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = blockIdx.y;
    if (t >= ntile) return;
    const Win w = make_win(S, N, G, W, (long long)h + kv_head_offset);
    TileRanges tr;
    if (!transposed) {
        const int i0 = t * BM;
        const int i1 = (i0 + BM < Lq ? i0 + BM : Lq) - 1;
        const int delta = Lk - Lq;
        tr = query_tile_ranges(i0 + delta, i1 + delta, w, BN);
    } else {
        const int c0 = t * BN;
        const int c1 = (c0 + BN < Lk ? c0 + BN : Lk) - 1;
        tr = key_tile_ranges(c0, c1, Lq, Lk, w, BM);
    }
    int4 *e = reinterpret_cast<int4 *>(sched + ((size_t)h * ntile + t) * kSchedInts);
    e[0] = make_int4(tr.n, tr.lo0, tr.lo0 + tr.len0, tr.lo1);
    e[1] = make_int4(tr.lo1 + tr.len1, tr.lo2, tr.lo2 + tr.len2, 0);
}

cudaError_t launch_schedule(int *sched, int Hkv, int kv_head_offset, int Lq, int Lk, int S,
                            int N, int G, int W, int BM, int BN, int transposed, cudaStream_t st)
{
    const int ntile = transposed ? (Lk + BN - 1) / BN : (Lq + BM - 1) / BM;
    if (ntile == 0 || Hkv == 0) return cudaSuccess;
    dim3 grid((ntile + 127) / 128, Hkv);
    launch_begin("schedule", st);
    schedule_kernel<<<grid, 128, 0, st>>>(sched, kv_head_offset, Lq, Lk, S, N, G, W, BM, BN,
                                          transposed, ntile);
    launch_end(st);
    return cudaGetLastError();
}

// Class map of one head from its schedule: 0 skipped, 1 masked, 2 unmasked.
__global__ void tile_class_kernel(const int *sched, uint8_t *out, int kv_head, int Lq, int Lk,
                                  int S, int N, int G, int W, int BM, int BN, int transposed,
                                  int nqt, int nkt)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)nqt * nkt) return;
    const int qt = (int)(idx / nkt), kt = (int)(idx % nkt);
    const Win w = make_win(S, N, G, W, kv_head);
    const int *e = sched + (size_t)(transposed ? kt : qt) * kSchedInts;
    const int key = transposed ? qt : kt;
    bool visited = false;
    for (int r = 0; r < e[0]; ++r)
        visited |= key >= e[1 + 2 * r] && key < e[2 + 2 * r];
    uint8_t cls = 0;
    if (visited) {
        const int delta = Lk - Lq;
        const int i0 = qt * BM, i1 = (i0 + BM < Lq ? i0 + BM : Lq) - 1;
        cls = tile_full(i0 + delta, i1 + delta, kt * BN, BN, Lk, w) ? 2 : 1;
    }
    out[idx] = cls;
}

cudaError_t launch_tile_classes(const int *sched, uint8_t *out, int kv_head, int Lq, int Lk,
                                int S, int N, int G, int W, int BM, int BN, int transposed,
                                cudaStream_t st)
{
    const int nqt = (Lq + BM - 1) / BM, nkt = (Lk + BN - 1) / BN;
    const long long n = (long long)nqt * nkt;
    if (n == 0) return cudaSuccess;
    launch_begin("tile_classes", st);
    tile_class_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        sched, out, kv_head, Lq, Lk, S, N, G, W, BM, BN, transposed, nqt, nkt);
    launch_end(st);
    return cudaGetLastError();
}

}  // namespace cowa
