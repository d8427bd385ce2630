// Output epilogue Y = swish(G) (.) GroupNorm(O), one group per head.
//
// RetNet adds a swish gate and GroupNorm on the retention output (research
// summary, "Summary"; the ablations in "Key points" show both matter).
// Each (token, head) is normalised over its dv channels with the biased
// variance, scaled by the per-channel affine, and multiplied by
// swish(g) = g * sigmoid(g).  Standalone this is a pure HBM stream
// (read O and G, write Y); the tensor-core prefill fuses the same
// arithmetic into its epilogue.
#include "kernels.h"

namespace retnet {

constexpr int kGnThreads = 256;
constexpr int kGnMaxChunks = 4;            // 8-element chunks per lane: dv <= 1024

template <typename T>
__global__ void __launch_bounds__(kGnThreads)
groupnorm_swish_kernel(const T *o, const T *__restrict__ g, const float *__restrict__ weight,
                       const float *__restrict__ bias, float eps, long long groups, int heads,
                       int dv, T *y) {
    const int lane = threadIdx.x & 31;
    const long long grp = (long long)blockIdx.x * (kGnThreads / 32) + (threadIdx.x >> 5);
    if (grp >= groups) return;
    const int h = (int)(grp % heads);
    const int nchunk = dv / 8;
    const T *og = o + grp * dv;
    const T *gg = g + grp * dv;
    T *yg = y + grp * dv;

    float x[kGnMaxChunks][8];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kGnMaxChunks; ++i) {
        int c = lane + 32 * i;
        if (c < nchunk) {
            load8(og + c * 8, x[i]);
#pragma unroll
            for (int e = 0; e < 8; ++e) sum += x[i][e];
        }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float mean = sum / (float)dv;
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < kGnMaxChunks; ++i) {
        int c = lane + 32 * i;
        if (c < nchunk) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float t = x[i][e] - mean;
                sq = fmaf(t, t, sq);
            }
        }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    const float rstd = rsqrtf(sq / (float)dv + eps);

#pragma unroll
    for (int i = 0; i < kGnMaxChunks; ++i) {
        int c = lane + 32 * i;
        if (c < nchunk) {
            float gv[8], out[8];
            load8(gg + c * 8, gv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                int ch = h * dv + c * 8 + e;
                float w = weight ? weight[ch] : 1.f;
                float b = bias ? bias[ch] : 0.f;
                float yh = fmaf((x[i][e] - mean) * rstd, w, b);
                float sw = gv[e] / (1.f + expf(-gv[e]));
                out[e] = sw * yh;
            }
            store8(yg + c * 8, out);
        }
    }
}

cudaError_t launch_groupnorm_swish(const void *o, const void *g, const float *weight,
                                   const float *bias, float eps, long long rows, int heads,
                                   int dv, retnet_dtype dtype, void *y, cudaStream_t stream) {
    long long groups = rows * heads;
    if (groups == 0) return cudaSuccess;
    const int per_block = kGnThreads / 32;
    long long blocks = (groups + per_block - 1) / per_block;
    KernelTimer timer("groupnorm_swish", stream);
    if (dtype == RETNET_BF16)
        groupnorm_swish_kernel<__nv_bfloat16><<<(unsigned)blocks, kGnThreads, 0, stream>>>(
            (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)g, weight, bias, eps, groups,
            heads, dv, (__nv_bfloat16 *)y);
    else
        groupnorm_swish_kernel<float><<<(unsigned)blocks, kGnThreads, 0, stream>>>(
            (const float *)o, (const float *)g, weight, bias, eps, groups, heads, dv,
            (float *)y);
    count_launch();
    return cudaGetLastError();
}

}  // namespace retnet
