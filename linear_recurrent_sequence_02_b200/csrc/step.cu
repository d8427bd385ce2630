// Recurrent decode step: S <- gamma S + k^T v ; o = q S.
//
// The recurrent form of retention costs O(1) per token and keeps no KV
// cache (RetNet research summary, "Summary"; "Beyond Transformers ...",
// "Efficient Inference").  Per (sequence, head) the whole float32 state
// [dk, dv] is read and written once, so the step is an HBM stream:
// 8 * dk * dv bytes per head-step against ~5 dk dv flops.
//
// Layout of the work: a thread-block cluster owns one (sequence, head).
// Each CTA of the cluster owns a slab of 32 state rows; each thread owns a
// float4 of columns and walks a few rows, so o's partial sums need no
// shuffles.  Partials are reduced across the row lanes in shared memory and
// across the cluster through distributed shared memory, by cluster rank 0.
#include <cooperative_groups.h>

#include "kernels.h"

namespace cg = cooperative_groups;

namespace retnet {

constexpr int kStepThreads = 256;
constexpr int kStepRows = 32;       // state rows per CTA

template <typename T>
__global__ void __launch_bounds__(kStepThreads)
retention_step_kernel(const T *__restrict__ q, const T *__restrict__ k,
                      const T *__restrict__ v, HeadGammas gam, float *__restrict__ state,
                      T *__restrict__ out, int heads, int dk, int dv, long long pos,
                      int rotate) {
    cg::cluster_group cluster = cg::this_cluster();
    const int bh = blockIdx.x;                       // sequence * heads + head
    const int h = bh % heads;
    const int slab = blockIdx.y;                     // == rank in the (1, dk/32) cluster
    const int row0 = slab * kStepRows;
    const float g = gam.g[h];

    __shared__ float qs[kStepRows], ks[kStepRows];
    __shared__ float4 red[kStepThreads];
    __shared__ float4 partial[64];                   // dv / 4 <= 64

    // Rotated q, k entries of this CTA's rows (row pairs are never split:
    // kStepRows is even and row0 is a multiple of it).
    const T *qh = q + (size_t)bh * dk;
    const T *kh = k + (size_t)bh * dk;
    if (threadIdx.x < kStepRows / 2) {
        int r = row0 + 2 * threadIdx.x;
        float q0 = to_f32(qh[r]), q1 = to_f32(qh[r + 1]);
        float k0 = to_f32(kh[r]), k1 = to_f32(kh[r + 1]);
        if (rotate) {
            float2 cs = rotation_cs(pos, r / 2, dk);
            float a = q0, b = q1;
            q0 = a * cs.x - b * cs.y;
            q1 = a * cs.y + b * cs.x;
            a = k0; b = k1;
            k0 = a * cs.x - b * cs.y;
            k1 = a * cs.y + b * cs.x;
        }
        qs[2 * threadIdx.x] = q0; qs[2 * threadIdx.x + 1] = q1;
        ks[2 * threadIdx.x] = k0; ks[2 * threadIdx.x + 1] = k1;
    }

    const int ncg = dv / 4;                          // float4 column groups
    const int nrl = kStepThreads / ncg;              // row lanes
    const int cgi = threadIdx.x % ncg;
    const int rl = threadIdx.x / ncg;
    float vv[4];
    {
        const T *vh = v + (size_t)bh * dv + cgi * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) vv[i] = to_f32(vh[i]);
    }
    __syncthreads();

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float *S = state + (size_t)bh * dk * dv;
    const int rows_per_lane = kStepRows / nrl;       // 2, 4 or 8
#pragma unroll 8
    for (int i = 0; i < rows_per_lane; ++i) {
        int rr = rl + i * nrl;                       // row within the slab
        float4 *p = reinterpret_cast<float4 *>(S + (size_t)(row0 + rr) * dv) + cgi;
        float4 s = *p;
        float kr = ks[rr], qr = qs[rr];
        s.x = fmaf(g, s.x, kr * vv[0]);
        s.y = fmaf(g, s.y, kr * vv[1]);
        s.z = fmaf(g, s.z, kr * vv[2]);
        s.w = fmaf(g, s.w, kr * vv[3]);
        *p = s;
        acc.x = fmaf(qr, s.x, acc.x);
        acc.y = fmaf(qr, s.y, acc.y);
        acc.z = fmaf(qr, s.z, acc.z);
        acc.w = fmaf(qr, s.w, acc.w);
    }
    red[threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.x < ncg) {
        float4 t = red[threadIdx.x];
        for (int l = 1; l < nrl; ++l) {
            float4 u = red[l * ncg + threadIdx.x];
            t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
        }
        partial[threadIdx.x] = t;
    }
    cluster.sync();
    if (cluster.block_rank() == 0 && threadIdx.x < ncg) {
        float4 t = partial[threadIdx.x];
        const unsigned nblk = cluster.num_blocks();
        for (unsigned r = 1; r < nblk; ++r) {
            const float4 *rp = cluster.map_shared_rank(partial, r);
            float4 u = rp[threadIdx.x];
            t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
        }
        T *oh = out + (size_t)bh * dv + threadIdx.x * 4;
        oh[0] = from_f32<T>(t.x);
        oh[1] = from_f32<T>(t.y);
        oh[2] = from_f32<T>(t.z);
        oh[3] = from_f32<T>(t.w);
    }
    cluster.sync();       // keep every CTA's shared memory alive until rank 0 has read it
}

cudaError_t launch_retention_step(const void *q, const void *k, const void *v,
                                  const HeadGammas &gam, float *state, void *out, int batch,
                                  int heads, int dk, int dv, retnet_dtype dtype, long long pos,
                                  int rotate, cudaStream_t stream) {
    if (batch == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(batch * heads), (unsigned)(dk / kStepRows), 1);
    cfg.blockDim = dim3(kStepThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)(dk / kStepRows);
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err;
    KernelTimer timer("retention_step", stream);
    if (dtype == RETNET_BF16)
        err = cudaLaunchKernelEx(&cfg, retention_step_kernel<__nv_bfloat16>,
                                 (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                 (const __nv_bfloat16 *)v, gam, state, (__nv_bfloat16 *)out,
                                 heads, dk, dv, pos, rotate);
    else
        err = cudaLaunchKernelEx(&cfg, retention_step_kernel<float>, (const float *)q,
                                 (const float *)k, (const float *)v, gam, state, (float *)out,
                                 heads, dk, dv, pos, rotate);
    count_launch();
    return err;
}

}  // namespace retnet
