// Work lists of packed (variable-length) batches: the (sequence, tile) pairs
// the tiled kernels visit, so that their grids hold one CTA per real tile
// instead of one per (sequence, tile of the longest sequence).
//
// Sequence b has n_b = ceil(L_b / tile) tiles.  Items are listed by rank r,
// the tile's place in its sequence counted from the heavy end: rank 0 holds
// every sequence's heaviest tile, rank 1 the next, ...  For the query-major
// passes (forward, dQ) rank r is tile n_b - 1 - r (the last query tile sees
// the most keys); for the key-major dK/dV pass it is tile r (the first key
// tile holds the sink, which every query sees).  Within a rank the order is
// the order in which the sequences' threads claim slots (it only affects
// scheduling: every output element has one writer).  Entries past the last
// item are (-1, -1): their CTAs return at once.
//
// One block of 1024 threads: per-sequence tile counts, a histogram of them,
// the start of every rank's run (a scan over ranks), then each sequence
// writes its items.  Scratch (global, 3 * (max_tiles + 1) ints) is zeroed
// here first.
#include "kernels.cuh"

namespace cowa {

__device__ __forceinline__ int block_scan_excl(int v, int *sh, int &total)
{
    // exclusive prefix sum over the 1024 threads of the block
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = sh[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        sh[lane] = w;
    }
    __syncthreads();
    total = sh[31];
    const int before = warp > 0 ? sh[warp - 1] : 0;
    __syncthreads();
    return before + x - v;
}

__global__ void __launch_bounds__(1024) varlen_worklist_kernel(const int *cu, int B, int tile, int max_tiles,
                                                               int descending, int2 *list, int max_items,
                                                               int *scratch, int *err)
{
    __shared__ int sh[32];
    int *hist = scratch;                        // [max_tiles + 1]: sequences with n_b tiles
    int *start = scratch + (max_tiles + 1);     // [max_tiles + 1]: first slot of rank r
    int *ctr = scratch + 2 * (max_tiles + 1);   // [max_tiles + 1]: slots claimed in rank r
    const int tid = threadIdx.x;
    for (int i = tid; i < 3 * (max_tiles + 1); i += blockDim.x) scratch[i] = 0;
    __syncthreads();
    auto ntiles = [&](int b) {
        const int a = cu[b], e = cu[b + 1];
        const int n = e > a ? (e - a + tile - 1) / tile : 0;
        return n < max_tiles ? n : max_tiles;  // longer sequences are reported by the kernels
    };
    for (int b = tid; b < B; b += blockDim.x) atomicAdd(&hist[ntiles(b)], 1);
    __syncthreads();
    // count(r) = sequences with more than r tiles = sum of hist[m], m > r;
    // start(r) = sum of count(r'), r' < r.  Two scans over r in chunks.
    int carry = 0;
    for (int base = max_tiles; base >= 0; base -= blockDim.x) {  // suffix sums of hist, descending r
        const int r = base - tid;
        const int v = r >= 0 ? hist[r] : 0;
        int tot;
        const int ex = block_scan_excl(v, sh, tot);
        if (r >= 0) start[r] = carry + ex;  // sequences with more than r tiles
        carry += tot;
    }
    __syncthreads();
    carry = 0;
    for (int base = 0; base <= max_tiles; base += blockDim.x) {  // prefix sums of the counts, ascending r
        const int r = base + tid;
        const int v = r <= max_tiles ? start[r] : 0;
        int tot;
        const int ex = block_scan_excl(v, sh, tot);
        __syncthreads();
        if (r <= max_tiles) start[r] = carry + ex;
        carry += tot;
        __syncthreads();
    }
    const int total = carry;
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) {
        const int n = ntiles(b);
        for (int r = 0; r < n; ++r) {
            const int pos = start[r] + atomicAdd(&ctr[r], 1);
            if (pos < max_items) list[pos] = make_int2(b, descending ? n - 1 - r : r);
            else atomicExch(err, 7);
        }
    }
    for (int i = total + tid; i < max_items; i += blockDim.x) list[i] = make_int2(-1, -1);
}

cudaError_t launch_varlen_worklist(const int *cu, int B, int tile, int max_tiles, bool descending, int2 *list,
                                   int max_items, int *scratch, int *err, cudaStream_t st)
{
    launch_begin("varlen_worklist", st);
    varlen_worklist_kernel<<<1, 1024, 0, st>>>(cu, B, tile, max_tiles, descending ? 1 : 0, list, max_items, scratch,
                                               err);
    launch_end(st);
    return cudaGetLastError();
}

}  // namespace cowa
