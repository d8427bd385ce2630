// Chunkwise-recurrent retention on CUDA cores, float32 arithmetic.
//
// The chunkwise form computes in parallel inside a chunk and carries a
// recurrent state from chunk to chunk (RetNet research summary, "Summary";
// "Key points": cost O(d n (b + h)) for chunk b).  For a chunk of L tokens
// starting at c0 (local indices i, j) and head decay g:
//     O_c   = (Q_c K_c^T (.) D) V_c + (Q_c (.) xi) S_prev,
//     D_ij  = g^(i-j) for i >= j else 0,   xi_i = g^(i+1),
//     S     = g^L S_prev + K_c^T (V_c (.) zeta),   zeta_j = g^(L-1-j).
// This path serves float32 inputs (where tensor-core formats cannot hold
// the 1e-4 tolerance) and any shape the tensor-core path does not take.
//
// Two kernels:
//   state pass   one CTA per (sequence, head, 64 x 64 block of S) walks the
//                chunks in order, writing S_prev of every chunk to the
//                workspace and the final state to state_out;
//   output pass  one CTA per (sequence, head, chunk, 32-row tile) forms the
//                cross-chunk term from S_prev and the masked intra-chunk
//                contraction, all from shared-memory tiles, each thread
//                accumulating a 4-row register tile.
// Powers g^e for e = 0..chunk are tabulated per CTA with powf.
#include "kernels.h"

namespace retnet {

constexpr int kSimtThreads = 256;
constexpr int kTile = 32;

// Loads rows [t0, t0 + 32) of one head of x [B, n, H, D] into sm[32][ld],
// rotating pairs by the table when asked; rows at or beyond `valid` read 0.
template <typename T, int D>
__device__ __forceinline__ void load_rot_tile(float *sm, int ld, const T *x, int b, int h,
                                              int heads, int n, int t0, int valid,
                                              const float2 *table, int rotate) {
    constexpr int HALF = D / 2;
    for (int idx = threadIdx.x; idx < kTile * HALF; idx += kSimtThreads) {
        int jj = idx / HALF, p = idx - jj * HALF;
        float x0 = 0.f, x1 = 0.f;
        if (jj < valid) {
            int t = t0 + jj;
            const T *row = x + (((size_t)b * n + t) * heads + h) * D;
            x0 = to_f32(row[2 * p]);
            x1 = to_f32(row[2 * p + 1]);
            if (rotate) {
                float2 cs = table[(size_t)t * HALF + p];
                float a = x0;
                x0 = a * cs.x - x1 * cs.y;
                x1 = a * cs.y + x1 * cs.x;
            }
        }
        sm[jj * ld + 2 * p] = x0;
        sm[jj * ld + 2 * p + 1] = x1;
    }
}

// Columns [c0, c0 + 64) of the same rows into sm[32][64] (c0 even, so
// rotation pairs stay whole): the state pass's slice of d_k.
template <typename T, int D>
__device__ __forceinline__ void load_rot_slice(float *sm, const T *x, int b, int h, int heads,
                                               int n, int t0, int valid, const float2 *table,
                                               int rotate, int c0) {
    constexpr int HALF = D / 2;
    for (int idx = threadIdx.x; idx < kTile * 32; idx += kSimtThreads) {
        int jj = idx / 32, p = idx - jj * 32;             // pair p of the slice
        float x0 = 0.f, x1 = 0.f;
        if (jj < valid) {
            int t = t0 + jj;
            const T *row = x + (((size_t)b * n + t) * heads + h) * D + c0;
            x0 = to_f32(row[2 * p]);
            x1 = to_f32(row[2 * p + 1]);
            if (rotate) {
                float2 cs = table[(size_t)t * HALF + c0 / 2 + p];
                float a = x0;
                x0 = a * cs.x - x1 * cs.y;
                x1 = a * cs.y + x1 * cs.x;
            }
        }
        sm[jj * 64 + 2 * p] = x0;
        sm[jj * 64 + 2 * p + 1] = x1;
    }
}

// ------------------------------------------------------------- state pass
template <typename T, int DK>
__global__ void __launch_bounds__(kSimtThreads)
simt_state_kernel(const T *__restrict__ k, const T *__restrict__ v,
                  const float2 *__restrict__ table, HeadGammas gam, const float *state_in,
                  float *state_out, float *__restrict__ s_prev, int heads, int n, int dv,
                  int chunk, int nchunks, int rotate) {
    // CTA (sequence-head, 64-column slab, 64-row slice of d_k): rows of
    // U = K^T V are independent, so the slices need no reduction, and
    // DK/64 times as many CTAs stream as with whole-height slabs.
    constexpr int RPT = 4;                        // state rows per thread (64 / 16)
    const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
    const int col0 = blockIdx.y * 64;
    const int row0 = blockIdx.z * 64;
    const int rl = threadIdx.x / 16, cq = threadIdx.x % 16;
    const float g = gam.g[h];

    extern __shared__ float smem[];
    float *ksm = smem;                            // [32][64]: this slice of d_k
    float *vsm = ksm + kTile * 64;                // [32][64]
    float *gpow = vsm + kTile * 64;               // [chunk + 1]
    for (int e = threadIdx.x; e <= chunk; e += kSimtThreads) gpow[e] = powf(g, (float)e);

    float S[RPT][4];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        int a = row0 + rl + 16 * i;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        if (state_in)
            s = *reinterpret_cast<const float4 *>(state_in + ((size_t)bh * DK + a) * dv + col0 +
                                                  cq * 4);
        S[i][0] = s.x; S[i][1] = s.y; S[i][2] = s.z; S[i][3] = s.w;
    }
    __syncthreads();

    for (int c = 0; c < nchunks; ++c) {
        const int c0 = c * chunk;
        const int L = min(chunk, n - c0);
        float *sp = s_prev + ((size_t)bh * nchunks + c) * DK * dv;
        const float gL = gpow[L];
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            int a = row0 + rl + 16 * i;
            *reinterpret_cast<float4 *>(sp + (size_t)a * dv + col0 + cq * 4) =
                make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) S[i][e] *= gL;
        }
        for (int j0 = 0; j0 < L; j0 += kTile) {
            __syncthreads();
            const int valid = min(kTile, L - j0);
            load_rot_slice<T, DK>(ksm, k, b, h, heads, n, c0 + j0, valid, table, rotate, row0);
            for (int idx = threadIdx.x; idx < kTile * 64; idx += kSimtThreads) {
                int jj = idx / 64, cc = idx % 64;
                float val = 0.f;
                if (jj < valid) {
                    int j = j0 + jj;
                    val = to_f32(v[(((size_t)b * n + c0 + j) * heads + h) * dv + col0 + cc]) *
                          gpow[L - 1 - j];
                }
                vsm[jj * 64 + cc] = val;
            }
            __syncthreads();
#pragma unroll 4
            for (int jj = 0; jj < kTile; ++jj) {
                float4 vv = *reinterpret_cast<const float4 *>(vsm + jj * 64 + cq * 4);
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    float kr = ksm[jj * 64 + rl + 16 * i];
                    S[i][0] = fmaf(kr, vv.x, S[i][0]);
                    S[i][1] = fmaf(kr, vv.y, S[i][1]);
                    S[i][2] = fmaf(kr, vv.z, S[i][2]);
                    S[i][3] = fmaf(kr, vv.w, S[i][3]);
                }
            }
        }
    }
    if (state_out) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            int a = row0 + rl + 16 * i;
            *reinterpret_cast<float4 *>(state_out + ((size_t)bh * DK + a) * dv + col0 + cq * 4) =
                make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
        }
    }
}

// ------------------------------------------------------------- output pass
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads)
simt_output_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const float2 *__restrict__ table, HeadGammas gam,
                   const float *__restrict__ s_prev, T *__restrict__ out, int heads, int n,
                   int chunk, int nchunks, int rotate) {
    // Accumulators: each thread owns a 4-row x (DV/32)-column tile of the
    // output (rows 4 rg .. 4 rg + 3; columns u * 32 VW + VW cg + e), so every
    // S_prev or V value read from shared memory serves four rows and the
    // column vectors of a warp are contiguous (conflict-free).
    constexpr int RO = kTile / 8;                 // rows per thread
    constexpr int VW = DV >= 128 ? 4 : 2;         // column vector width
    constexpr int NG = DV / (32 * VW);            // column vectors per thread
    constexpr int CPT = NG * VW;                  // columns per thread
    constexpr int LDQ = DK + 1;
    const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
    const int c = blockIdx.y;
    const int c0 = c * chunk;
    const int L = min(chunk, n - c0);
    const int r0 = blockIdx.z * kTile;
    if (r0 >= L) return;
    const int rows = min(kTile, L - r0);
    const int rg = threadIdx.x / 32, cg = threadIdx.x % 32;     // accumulator tile
    const int r = threadIdx.x / 8, cq = threadIdx.x % 8;         // score layout
    const float g = gam.g[h];

    extern __shared__ float smem[];
    float *qsm = smem;                            // [32][DK+1]
    float *ksm = qsm + kTile * LDQ;               // [32][DK+1]
    float *vsm = ksm + kTile * LDQ;               // [32][DV]
    float *psm = vsm + kTile * DV;                // [32][33]
    float *gpow = psm + kTile * 33;               // [chunk + 1]
    for (int e = threadIdx.x; e <= chunk; e += kSimtThreads) gpow[e] = powf(g, (float)e);
    load_rot_tile<T, DK>(qsm, LDQ, q, b, h, heads, n, c0 + r0, rows, table, rotate);

    float acc[RO][CPT];
#pragma unroll
    for (int i = 0; i < RO; ++i)
#pragma unroll
        for (int e = 0; e < CPT; ++e) acc[i][e] = 0.f;

    // acc[i][:] += w[i] * (the thread's columns of row `row` of vsm)
    auto axpy_rows = [&](const float *w, int row) {
#pragma unroll
        for (int u = 0; u < NG; ++u) {
            float x[VW];
            const float *src = vsm + row * DV + u * 32 * VW + cg * VW;
            if constexpr (VW == 4) {
                const float4 f = *reinterpret_cast<const float4 *>(src);
                x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
            } else {
                const float2 f = *reinterpret_cast<const float2 *>(src);
                x[0] = f.x; x[1] = f.y;
            }
#pragma unroll
            for (int i = 0; i < RO; ++i)
#pragma unroll
                for (int e = 0; e < VW; ++e)
                    acc[i][u * VW + e] = fmaf(w[i], x[e], acc[i][u * VW + e]);
        }
    };

    // cross-chunk term (Q (.) xi) S_prev
    const float *sp = s_prev + ((size_t)bh * nchunks + c) * DK * DV;
    for (int a0 = 0; a0 < DK; a0 += kTile) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kTile * DV / 4; idx += kSimtThreads)
            reinterpret_cast<float4 *>(vsm)[idx] =
                reinterpret_cast<const float4 *>(sp + (size_t)a0 * DV)[idx];
        __syncthreads();
#pragma unroll 4
        for (int aa = 0; aa < kTile; ++aa) {
            float w[RO];
#pragma unroll
            for (int i = 0; i < RO; ++i) w[i] = qsm[(RO * rg + i) * LDQ + a0 + aa];
            axpy_rows(w, aa);
        }
    }
#pragma unroll
    for (int i = 0; i < RO; ++i) {
        const float xi = gpow[min(r0 + RO * rg + i + 1, chunk)];
#pragma unroll
        for (int e = 0; e < CPT; ++e) acc[i][e] *= xi;
    }

    // intra-chunk term (Q K^T (.) D) V over key tiles up to this row tile
    for (int kt = 0; kt <= (int)blockIdx.z; ++kt) {
        const int j0 = kt * kTile;
        const int kvalid = min(kTile, L - j0);
        __syncthreads();
        load_rot_tile<T, DK>(ksm, LDQ, k, b, h, heads, n, c0 + j0, kvalid, table, rotate);
        for (int idx = threadIdx.x; idx < kTile * DV; idx += kSimtThreads) {
            int jj = idx / DV, cc = idx % DV;
            vsm[idx] = jj < kvalid
                           ? to_f32(v[(((size_t)b * n + c0 + j0 + jj) * heads + h) * DV + cc])
                           : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int jj = cq + 8 * m;
            float s = 0.f;
#pragma unroll 8
            for (int a = 0; a < DK; ++a) s = fmaf(qsm[r * LDQ + a], ksm[jj * LDQ + a], s);
            const int i_loc = r0 + r, j_loc = j0 + jj;
            psm[r * 33 + jj] = (i_loc >= j_loc) ? s * gpow[i_loc - j_loc] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < kTile; ++jj) {
            float w[RO];
#pragma unroll
            for (int i = 0; i < RO; ++i) w[i] = psm[(RO * rg + i) * 33 + jj];
            axpy_rows(w, jj);
        }
    }

#pragma unroll
    for (int i = 0; i < RO; ++i) {
        const int row = RO * rg + i;
        if (row < rows) {
            T *orow = out + (((size_t)b * n + c0 + r0 + row) * heads + h) * DV;
#pragma unroll
            for (int u = 0; u < NG; ++u)
#pragma unroll
                for (int e = 0; e < VW; ++e)
                    orow[u * 32 * VW + cg * VW + e] = from_f32<T>(acc[i][u * VW + e]);
        }
    }
}

// ------------------------------------------------------------- host side
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t simt_workspace_bytes(int batch, int heads, int seqlen, int dk, int dv, int chunk) {
    size_t nchunks = ((size_t)seqlen + chunk - 1) / chunk;
    size_t table = align256((size_t)seqlen * (dk / 2) * sizeof(float2));
    size_t sprev = align256((size_t)batch * heads * nchunks * dk * dv * sizeof(float));
    return table + sprev;
}

template <typename T, int DK, int DV>
static cudaError_t launch_simt_typed(const ChunkwiseArgs &a, cudaStream_t stream) {
    const int nchunks = (a.seqlen + a.chunk - 1) / a.chunk;
    char *ws = (char *)a.workspace;
    float2 *table = (float2 *)ws;
    float *s_prev = (float *)(ws + align256((size_t)a.seqlen * (DK / 2) * sizeof(float2)));
    cudaError_t err;
    if (a.rotate && a.seqlen > 0) {
        err = launch_rotation_table(table, a.seqlen, DK, a.pos0, stream);
        if (err != cudaSuccess) return err;
    }
    const int bh = a.batch * a.heads;
    if (bh == 0) return cudaSuccess;

    size_t smem_a = (size_t)(kTile * 64 + kTile * 64 + a.chunk + 1) * sizeof(float);
    auto ka = simt_state_kernel<T, DK>;
    err = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a);
    if (err != cudaSuccess) return err;
    {
        KernelTimer timer("simt_state", stream);
        ka<<<dim3(bh, DV / 64, DK / 64), kSimtThreads, smem_a, stream>>>(
            (const T *)a.k, (const T *)a.v, table, a.gam, a.state_in, a.state_out, s_prev,
            a.heads, a.seqlen, DV, a.chunk, nchunks, a.rotate);
    }
    count_launch();
    err = cudaGetLastError();
    if (err != cudaSuccess || nchunks == 0) return err;

    size_t smem_b =
        (size_t)(2 * kTile * (DK + 1) + kTile * DV + kTile * 33 + a.chunk + 1) * sizeof(float);
    auto kb = simt_output_kernel<T, DK, DV>;
    err = cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b);
    if (err != cudaSuccess) return err;
    const int rtiles = (a.chunk + kTile - 1) / kTile;
    {
        KernelTimer timer("simt_output", stream);
        kb<<<dim3(bh, nchunks, rtiles), kSimtThreads, smem_b, stream>>>(
            (const T *)a.q, (const T *)a.k, (const T *)a.v, table, a.gam, s_prev, (T *)a.out,
            a.heads, a.seqlen, a.chunk, nchunks, a.rotate);
    }
    count_launch();
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (a.gate)
        err = launch_groupnorm_swish(a.out, a.gate->g, a.gate->weight, a.gate->bias,
                                     a.gate->eps, (long long)a.batch * a.seqlen, a.heads, DV,
                                     a.dtype, a.out, stream);
    return err;
}

template <typename T, int DK>
static cudaError_t launch_simt_dk(const ChunkwiseArgs &a, cudaStream_t s) {
    switch (a.dv) {
        case 64: return launch_simt_typed<T, DK, 64>(a, s);
        case 128: return launch_simt_typed<T, DK, 128>(a, s);
        case 256: return launch_simt_typed<T, DK, 256>(a, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t launch_simt_t(const ChunkwiseArgs &a, cudaStream_t s) {
    switch (a.dk) {
        case 64: return launch_simt_dk<T, 64>(a, s);
        case 128: return launch_simt_dk<T, 128>(a, s);
        case 256: return launch_simt_dk<T, 256>(a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_chunkwise_simt(const ChunkwiseArgs &a, cudaStream_t stream) {
    return a.dtype == RETNET_BF16 ? launch_simt_t<__nv_bfloat16>(a, stream)
                                  : launch_simt_t<float>(a, stream);
}

}  // namespace retnet
