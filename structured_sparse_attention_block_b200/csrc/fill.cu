// Outputs of the shapes the tcgen05 kernels do not take, where every value
// is a constant: a forward with no keys (each row sees nothing: O = 0, LSE =
// -inf) and a backward with no queries or no keys (zero gradients).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"

namespace cowa {

// zero rows of a strided [B, L, H, D] bf16 tensor, 16 bytes per thread
template <int D>
__global__ void __launch_bounds__(256) zero_rows_kernel(__nv_bfloat16 *t, long long s0, long long s1, long long s2,
                                                        int L, int H, long long rows)
{
    constexpr int PIECES = D / 8;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= rows * PIECES) return;
    const long long r = idx / PIECES;
    const int c = (int)(idx % PIECES);
    const int h = (int)(r % H);
    const long long bl = r / H;
    const int l = (int)(bl % L);
    const long long b = bl / L;
    *reinterpret_cast<uint4 *>(t + b * s0 + (long long)l * s1 + (long long)h * s2 + c * 8) = make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(256) fill_f32_kernel(float *p, long long n, float v)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) p[i] = v;
}

cudaError_t launch_zero_rows(void *t, const long long st[3], int B, int L, int H, int D, cudaStream_t s)
{
    const long long rows = (long long)B * L * H;
    if (rows == 0) return cudaSuccess;
    const long long threads = rows * (D / 8);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    launch_begin("zero_rows", s);
    if (D == 128)
        zero_rows_kernel<128><<<blocks, 256, 0, s>>>(reinterpret_cast<__nv_bfloat16 *>(t), st[0], st[1], st[2], L, H, rows);
    else
        zero_rows_kernel<64><<<blocks, 256, 0, s>>>(reinterpret_cast<__nv_bfloat16 *>(t), st[0], st[1], st[2], L, H, rows);
    launch_end(s);
    return cudaGetLastError();
}

cudaError_t launch_fill_f32(float *p, long long n, float v, cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    launch_begin("fill_f32", s);
    fill_f32_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p, n, v);
    launch_end(s);
    return cudaGetLastError();
}

}  // namespace cowa
