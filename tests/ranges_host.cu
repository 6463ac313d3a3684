// Host-side driver for the tile-range functions the tcgen05 kernels evaluate
// per CTA (common.cuh): prints, for every query tile (mode q) or key tile
// (mode k) of one KV head, the merged ranges of visited tiles; for every
// query row (mode r) the runs of keys it sees, and for every key (mode c) the
// runs of aligned query positions that see it.  Test infrastructure: built
// and run by tests/test_ranges_cpu.py.
#include <cstdio>
#include <cstdlib>

#include "../structured_sparse_attention_block_b200/csrc/common.cuh"

int main(int argc, char **argv)
{
    if (argc != 11) return 2;
    const char mode = argv[1][0];
    const int Lq = atoi(argv[2]), Lk = atoi(argv[3]), S = atoi(argv[4]), N = atoi(argv[5]), G = atoi(argv[6]),
              W = atoi(argv[7]), h = atoi(argv[8]), BM = atoi(argv[9]), BN = atoi(argv[10]);
    const cowa::Win w = cowa::make_win(S, N, G, W, h);
    if (mode == 'r' || mode == 'c') {
        const int n = mode == 'r' ? Lq : Lk;
        for (int x = 0; x < n; ++x) {
            const cowa::Runs3 r = mode == 'r' ? cowa::row_key_runs(x + Lk - Lq, w) : cowa::key_pos_runs(x, w, Lk - 1);
            printf("%d %d %d %d %d %d\n", r.a0, r.b0, r.a1, r.b1, r.a2, r.b2);
        }
        return 0;
    }
    const int ntile = mode == 'q' ? (Lq + BM - 1) / BM : (Lk + BN - 1) / BN;
    for (int t = 0; t < ntile; ++t) {
        cowa::TileRanges r;
        if (mode == 'q') {
            const int i0 = t * BM, i1 = (i0 + BM < Lq ? i0 + BM : Lq) - 1;
            r = cowa::query_tile_ranges(i0 + Lk - Lq, i1 + Lk - Lq, w, BN);
        } else {
            const int c0 = t * BN, c1 = (c0 + BN < Lk ? c0 + BN : Lk) - 1;
            r = cowa::key_tile_ranges(c0, c1, Lq, Lk, w, BM);
        }
        printf("%d %d %d %d %d %d %d\n", r.n, r.lo0, r.len0, r.lo1, r.len1, r.lo2, r.len2);
    }
    return 0;
}
