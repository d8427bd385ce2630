// xPos-like rotation prologue: a (cos, sin) table and a standalone rotation.
//
// Positions are encoded "in a manner similar to xPos" (RetNet research
// summary, "Summary"): adjacent pairs (2j, 2j+1) of q and k are turned by
// pos * theta_j, theta_j = 10000^(-2j/d).  Relative position then enters
// through (R_n q) . (R_m k), which depends only on n - m; the per-head
// decay takes the place of xPos's length scaling.
#include <algorithm>

#include "kernels.h"

namespace retnet {

// Grid (ceil(rows / per_thread), ceil(half / 128)): each thread owns one
// pair index j, forms theta_j once and fills per_thread rows, so the float64
// power is paid once per per_thread table entries.  Row t holds position
// pos0 + t * stride.
__global__ void __launch_bounds__(128)
rotation_table_kernel(float2 *__restrict__ table, int rows, int half, int d, long long pos0,
                      int stride, int per_thread) {
    const int j = blockIdx.y * 128 + threadIdx.x;
    if (j >= half) return;
    const double theta = pow(10000.0, -2.0 * (double)j / (double)d);
    const int t0 = blockIdx.x * per_thread;
    const int t1 = min(rows, t0 + per_thread);
    for (int t = t0; t < t1; ++t)
        table[(size_t)t * half + j] = rotation_cs(pos0 + (long long)t * stride, theta);
}

cudaError_t launch_rotation_table(float2 *table, int rows, int d, long long pos0,
                                  cudaStream_t stream, int stride) {
    const int half = d / 2;
    if (rows == 0 || half == 0) return cudaSuccess;
    // 32 rows per thread for long tables; short ones spread one row per
    // thread, so the grid still covers the SMs
    const int per_thread = std::max(1, std::min(32, rows / 256));
    dim3 grid((unsigned)((rows + per_thread - 1) / per_thread), (unsigned)((half + 127) / 128));
    {
        KernelTimer timer("rotation_table", stream);
        rotation_table_kernel<<<grid, 128, 0, stream>>>(table, rows, half, d, pos0, stride,
                                                        per_thread);
    }
    count_launch();
    return cudaGetLastError();
}

// One thread rotates 8 consecutive elements (4 pairs) of one (b, t, h) row.
template <typename T>
__global__ void xpos_rotate_kernel(const T *x, T *y,   // y may equal x
                                   long long rows_bt, int heads, int d, int seqlen,
                                   long long pos0) {
    const int per_row = d / 8;
    long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long total = rows_bt * heads * per_row;
    if (idx >= total) return;
    int part = (int)(idx % per_row);
    long long bth = idx / per_row;                 // (b * seqlen + t) * heads + h
    long long bt = bth / heads;
    int t = (int)(bt % seqlen);
    long long off = bth * d + part * 8;
    float e[8];
    load8(x + off, e);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        float2 cs = rotation_cs(pos0 + t, part * 4 + p, d);
        float a = e[2 * p], b = e[2 * p + 1];
        e[2 * p] = a * cs.x - b * cs.y;
        e[2 * p + 1] = a * cs.y + b * cs.x;
    }
    store8(y + off, e);
}

cudaError_t launch_xpos_rotate(const void *x, void *y, long long rows_bt, int heads, int d,
                               retnet_dtype dtype, int seqlen, long long pos0,
                               cudaStream_t stream) {
    long long total = rows_bt * heads * (d / 8);
    if (total == 0) return cudaSuccess;
    int threads = 256;
    long long blocks = (total + threads - 1) / threads;
    KernelTimer timer("xpos_rotate", stream);
    if (dtype == RETNET_BF16)
        xpos_rotate_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, stream>>>(
            (const __nv_bfloat16 *)x, (__nv_bfloat16 *)y, rows_bt, heads, d, seqlen, pos0);
    else
        xpos_rotate_kernel<float><<<(unsigned)blocks, threads, 0, stream>>>(
            (const float *)x, (float *)y, rows_bt, heads, d, seqlen, pos0);
    count_launch();
    return cudaGetLastError();
}

}  // namespace retnet
