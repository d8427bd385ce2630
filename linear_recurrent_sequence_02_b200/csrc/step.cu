// Recurrent decode step: S <- gamma S + k^T v ; o = q S.
//
// The recurrent form of retention costs O(1) per token and keeps no KV
// cache (RetNet research summary, "Summary"; "Beyond Transformers ...",
// "Efficient Inference").  Per (sequence, head) the whole float32 state
// [dk, dv] is read and written once, so the step is an HBM stream:
// 8 * dk * dv bytes per head-step against ~5 dk dv flops.
//
// Layout of the work: CTA (sequence, head, 32-column slab of S) owns every
// row of its slab, so its 32 outputs are complete inside the CTA.  Each
// thread owns a float4 of columns for dk/32 rows, issues all of its state
// loads first, updates S in place and accumulates o; the 32 row lanes are
// reduced by warp shuffles and then across the eight warps in shared memory.
#include <algorithm>
#include <cmath>

#include "kernels.h"

namespace retnet {

constexpr int kStepThreads = 256;
constexpr int kStepCols = 32;       // state columns per CTA
constexpr int kStepLanes = kStepThreads / (kStepCols / 4);   // 32 row lanes

// (cos, sin) of pos * theta_j for the pairs of this step, formed on the host
// in float64 (the position is a host scalar), j < dk / 2 <= 128.
struct StepRotation {
    float2 cs[128];
};

template <typename T>
__device__ __forceinline__ void load4(const T *p, float *o);
template <>
__device__ __forceinline__ void load4<float>(const float *p, float *o) {
    float4 f = *reinterpret_cast<const float4 *>(p);
    o[0] = f.x; o[1] = f.y; o[2] = f.z; o[3] = f.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p, float *o) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u.y));
    o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
}

template <typename T, int DK>
__global__ void __launch_bounds__(kStepThreads)
retention_step_kernel(const T *__restrict__ q, const T *__restrict__ k,
                      const T *__restrict__ v, HeadGammas gam, StepRotation rot,
                      float *__restrict__ state, T *__restrict__ out, int bh0, int heads,
                      int dv, int rotate) {
    constexpr int RPL = DK / kStepLanes;             // rows per thread: 2, 4 or 8
    const int bh = bh0 + blockIdx.y;                 // sequence * heads + head
    const int h = bh % heads;
    const int col0 = blockIdx.x * kStepCols;         // a head's slabs run side by side
    const float g = gam.g[h];
    const int cgi = threadIdx.x % (kStepCols / 4);   // float4 column group in the slab
    const int rl = threadIdx.x / (kStepCols / 4);    // row lane

    __shared__ float qs[DK], ks[DK];
    __shared__ float4 red[kStepThreads / 32][kStepCols / 4];

    grid_dependency_wait();          // the state may come from the kernel before
    // Issue this thread's state loads first: they do not depend on q, k, v.
    float *S = state + (size_t)bh * DK * dv + col0 + cgi * 4;
    float4 s[RPL];
#pragma unroll
    for (int i = 0; i < RPL; ++i) s[i] = *reinterpret_cast<const float4 *>(S + (size_t)(rl + i * kStepLanes) * dv);

    // Rotated q and k of the whole head (every row of the slab is used).
    if (threadIdx.x < DK / 2) {
        const int r = 2 * threadIdx.x;
        const T *qh = q + (size_t)bh * DK + r;
        const T *kh = k + (size_t)bh * DK + r;
        float q0 = to_f32(qh[0]), q1 = to_f32(qh[1]);
        float k0 = to_f32(kh[0]), k1 = to_f32(kh[1]);
        if (rotate) {
            const float2 cs = rot.cs[threadIdx.x];
            float a = q0;
            q0 = a * cs.x - q1 * cs.y;
            q1 = a * cs.y + q1 * cs.x;
            a = k0;
            k0 = a * cs.x - k1 * cs.y;
            k1 = a * cs.y + k1 * cs.x;
        }
        qs[r] = q0; qs[r + 1] = q1;
        ks[r] = k0; ks[r + 1] = k1;
    }
    float vv[4];
    load4<T>(v + (size_t)bh * dv + col0 + cgi * 4, vv);
    __syncthreads();

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
        const int rr = rl + i * kStepLanes;
        const float kr = ks[rr], qr = qs[rr];
        float4 t = s[i];
        t.x = fmaf(g, t.x, kr * vv[0]);
        t.y = fmaf(g, t.y, kr * vv[1]);
        t.z = fmaf(g, t.z, kr * vv[2]);
        t.w = fmaf(g, t.w, kr * vv[3]);
        *reinterpret_cast<float4 *>(S + (size_t)rr * dv) = t;
        acc.x = fmaf(qr, t.x, acc.x);
        acc.y = fmaf(qr, t.y, acc.y);
        acc.z = fmaf(qr, t.z, acc.z);
        acc.w = fmaf(qr, t.w, acc.w);
    }
    // Row lanes of one column group: four per warp (lanes cgi, cgi+8,
    // cgi+16, cgi+24) meet by shuffles, then the eight warps in shared memory.
#pragma unroll
    for (int m = 8; m < 32; m <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane < kStepCols / 4) red[warp][lane] = acc;
    __syncthreads();
    if (threadIdx.x < kStepCols / 4) {
        float4 t = red[0][threadIdx.x];
#pragma unroll
        for (int w = 1; w < kStepThreads / 32; ++w) {
            const float4 u = red[w][threadIdx.x];
            t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
        }
        T *oh = out + (size_t)bh * dv + col0 + threadIdx.x * 4;
        oh[0] = from_f32<T>(t.x);
        oh[1] = from_f32<T>(t.y);
        oh[2] = from_f32<T>(t.z);
        oh[3] = from_f32<T>(t.w);
    }
}

template <typename T>
static cudaError_t launch_step_t(const void *q, const void *k, const void *v,
                                 const HeadGammas &gam, const StepRotation &rot, float *state,
                                 void *out, int batch, int heads, int dk, int dv, int rotate,
                                 cudaStream_t stream) {
    const long long bh_total = (long long)batch * heads;
    KernelTimer timer("retention_step", stream);
    // grid.y holds (sequence, head) rows; more than 65535 of them take several launches
    for (long long bh0 = 0; bh0 < bh_total; bh0 += 65535) {
        const dim3 grid((unsigned)(dv / kStepCols), (unsigned)std::min(65535LL, bh_total - bh0));
        cudaError_t e = cudaSuccess;
        switch (dk) {
            case 64:
                e = launch_overlapped(retention_step_kernel<T, 64>, grid, dim3(kStepThreads), 0,
                                      stream, (const T *)q, (const T *)k, (const T *)v, gam, rot,
                                      state, (T *)out, (int)bh0, heads, dv, rotate);
                break;
            case 128:
                e = launch_overlapped(retention_step_kernel<T, 128>, grid, dim3(kStepThreads), 0,
                                      stream, (const T *)q, (const T *)k, (const T *)v, gam, rot,
                                      state, (T *)out, (int)bh0, heads, dv, rotate);
                break;
            case 256:
                e = launch_overlapped(retention_step_kernel<T, 256>, grid, dim3(kStepThreads), 0,
                                      stream, (const T *)q, (const T *)k, (const T *)v, gam, rot,
                                      state, (T *)out, (int)bh0, heads, dv, rotate);
                break;
            default:
                return cudaErrorInvalidValue;
        }
        count_launch();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_retention_step(const void *q, const void *k, const void *v,
                                  const HeadGammas &gam, float *state, void *out, int batch,
                                  int heads, int dk, int dv, retnet_dtype dtype, long long pos,
                                  int rotate, cudaStream_t stream) {
    if (batch == 0) return cudaSuccess;
    StepRotation rot;
    const double two_pi = 6.283185307179586476925286766559;
    for (int j = 0; j < 128; ++j) rot.cs[j] = make_float2(1.f, 0.f);
    if (rotate) {
        for (int j = 0; j < dk / 2; ++j) {
            const double theta = std::pow(10000.0, -2.0 * j / dk);
            const double a = (double)pos * theta;
            const double r = a - two_pi * std::nearbyint(a / two_pi);
            rot.cs[j] = make_float2((float)std::cos(r), (float)std::sin(r));
        }
    }
    cudaError_t err = dtype == RETNET_BF16
                          ? launch_step_t<__nv_bfloat16>(q, k, v, gam, rot, state, out, batch,
                                                         heads, dk, dv, rotate, stream)
                          : launch_step_t<float>(q, k, v, gam, rot, state, out, batch, heads,
                                                 dk, dv, rotate, stream);
    return err;
}

}  // namespace retnet
