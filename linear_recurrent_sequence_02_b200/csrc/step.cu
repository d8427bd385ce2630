// Recurrent form: S <- gamma S + k^T v ; o = q S, token by token.
//
// The recurrent form of retention costs O(1) per token and keeps no KV
// cache (RetNet research summary, "Summary"; "Beyond Transformers ...",
// "Efficient Inference").  Per (sequence, head) the whole float32 state
// [dk, dv] is read once and written once per launch, so a one-token decode
// step is an HBM stream of 8 * dk * dv bytes per head against ~4 dk dv
// flops; a launch over T tokens (multi-token decode, or continuing a
// sequence by a short chunk) moves the same state bytes for T times the
// flops.
//
// Layout of the work: CTA (sequence, head, 32-column slab of S) owns every
// row of its slab, so its 32 outputs are complete inside the CTA.  Each
// thread owns a float4 of columns for dk/32 rows and issues its state loads
// first.  The rotated q and k rows are staged in shared memory, every
// thread updates its state and accumulates its part of o, and the 32 row
// lanes are reduced by warp shuffles and then across the eight warps in
// shared memory.  Two kernels share this arithmetic exactly:
//   retention_step_kernel    one token, the state updated in place;
//   retention_tokens_kernel  up to kGroup tokens per reduction round, the
//                            state held in registers across all tokens of
//                            the launch, so the barriers and the reduction
//                            are paid once per group rather than per token.
// The (cos, sin) of every rotated position are formed on the host in
// float64, the same for both kernels, which makes a T-token launch equal to
// T single steps bit for bit.
#include <algorithm>
#include <cmath>

#include "kernels.h"

namespace retnet {

constexpr int kStepThreads = 256;
constexpr int kStepCols = 32;       // state columns per CTA
constexpr int kStepLanes = kStepThreads / (kStepCols / 4);   // 32 row lanes
constexpr int kGroup = 8;           // tokens per reduction round (multi-token kernel)
constexpr int kRotPairs = 3072;     // (cos, sin) pairs per multi-token launch: 24 KB

// (cos, sin) of pos * theta_j for the pairs of this step, formed on the host
// in float64 (the position is a host scalar), j < dk / 2 <= 128.
struct StepRotation {
    float2 cs[128];
};
// (cos, sin) for the tokens of one multi-token launch: cs[t * dk/2 + j].
struct TokenRotation {
    float2 cs[kRotPairs];
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

// The per-token arithmetic both kernels share, written with explicit
// roundings so that the compiler contracts nothing differently in the two.
__device__ __forceinline__ void rotate_pair(float &x0, float &x1, float2 cs) {
    const float a = x0;
    x0 = __fmaf_rn(a, cs.x, -__fmul_rn(x1, cs.y));
    x1 = __fmaf_rn(a, cs.y, __fmul_rn(x1, cs.x));
}
// s <- g s + kr v ; acc += qr s
__device__ __forceinline__ void update_row(float4 &s, float4 &acc, float g, float kr, float qr,
                                           const float *vv) {
    s.x = __fmaf_rn(g, s.x, __fmul_rn(kr, vv[0]));
    s.y = __fmaf_rn(g, s.y, __fmul_rn(kr, vv[1]));
    s.z = __fmaf_rn(g, s.z, __fmul_rn(kr, vv[2]));
    s.w = __fmaf_rn(g, s.w, __fmul_rn(kr, vv[3]));
    acc.x = __fmaf_rn(qr, s.x, acc.x);
    acc.y = __fmaf_rn(qr, s.y, acc.y);
    acc.z = __fmaf_rn(qr, s.z, acc.z);
    acc.w = __fmaf_rn(qr, s.w, acc.w);
}
// Row lanes of one column group: four per warp (lanes cgi, cgi+8, cgi+16,
// cgi+24) meet by shuffles.
__device__ __forceinline__ void reduce_lanes(float4 &acc) {
#pragma unroll
    for (int m = 8; m < 32; m <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
    }
}
// the eight warps' partial sums of column group c, added in warp order
template <typename T>
__device__ __forceinline__ void write_output(const float4 (*red)[kStepCols / 4], int c, T *dst) {
    float4 o = red[0][c];
#pragma unroll
    for (int w = 1; w < kStepThreads / 32; ++w) {
        const float4 u = red[w][c];
        o.x += u.x; o.y += u.y; o.z += u.z; o.w += u.w;
    }
    dst[0] = from_f32<T>(o.x);
    dst[1] = from_f32<T>(o.y);
    dst[2] = from_f32<T>(o.z);
    dst[3] = from_f32<T>(o.w);
}

// q, k [batch, heads, DK]; v, out [batch, heads, dv]; state [batch, heads, DK, dv].
template <typename T, int DK>
__global__ void __launch_bounds__(kStepThreads)
retention_step_kernel(const T *__restrict__ q, const T *__restrict__ k,
                      const T *__restrict__ v, HeadGammas gam, StepRotation rot,
                      float *__restrict__ state, T *__restrict__ out, int bh0, int heads,
                      int dv, int rotate, long long bh_total, unsigned *err) {
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
#ifdef RETNET_CHECK_BOUNDS
    // debug build: this CTA's (sequence, head) row and columns exist
    if (!__syncthreads_and(in_bounds(bh, bh_total, err, kSiteStep) &&
                           in_bounds(col0 + cgi * 4 + 3, dv, err, kSiteStep)))
        return;
#endif
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
            rotate_pair(q0, q1, rot.cs[threadIdx.x]);
            rotate_pair(k0, k1, rot.cs[threadIdx.x]);
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
        update_row(s[i], acc, g, ks[rr], qs[rr], vv);
        *reinterpret_cast<float4 *>(S + (size_t)rr * dv) = s[i];
    }
    reduce_lanes(acc);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane < kStepCols / 4) red[warp][lane] = acc;
    __syncthreads();
    if (threadIdx.x < kStepCols / 4)
        write_output<T>(red, threadIdx.x, out + (size_t)bh * dv + col0 + threadIdx.x * 4);
}

// Tokens [tok0, tok0 + ntok) of q, k [batch, tokens, heads, DK] and v, out
// [batch, tokens, heads, dv]; state [batch, heads, DK, dv] in registers
// throughout.  rot.cs[(t - tok0) * DK/2 + j] rotates token t.
template <typename T, int DK>
__global__ void __launch_bounds__(kStepThreads, 2)
retention_tokens_kernel(const T *__restrict__ q, const T *__restrict__ k,
                        const T *__restrict__ v, HeadGammas gam, TokenRotation rot,
                        float *__restrict__ state, T *__restrict__ out, int bh0, int heads,
                        int tokens, int tok0, int ntok, int dv, int rotate, long long bh_total,
                        unsigned *err) {
    constexpr int RPL = DK / kStepLanes;
    constexpr int kPairs = DK / 2;
    const int bh = bh0 + blockIdx.y;
    const int b = bh / heads, h = bh % heads;
    const int col0 = blockIdx.x * kStepCols;
    const float g = gam.g[h];
    const int cgi = threadIdx.x % (kStepCols / 4);
    const int rl = threadIdx.x / (kStepCols / 4);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    __shared__ float qs[kGroup][DK], ks[kGroup][DK];
    __shared__ float4 red[kGroup][kStepThreads / 32][kStepCols / 4];

    grid_dependency_wait();          // the state may come from the kernel before
#ifdef RETNET_CHECK_BOUNDS
    // debug build: this CTA's row, columns and tokens exist
    if (!__syncthreads_and(in_bounds(bh, bh_total, err, kSiteStep) &&
                           in_bounds(col0 + cgi * 4 + 3, dv, err, kSiteStep) &&
                           in_bounds(tok0 + ntok - 1, tokens, err, kSiteStep)))
        return;
#endif
    float *S = state + (size_t)bh * DK * dv + col0 + cgi * 4;
    float4 s[RPL];
#pragma unroll
    for (int i = 0; i < RPL; ++i) s[i] = *reinterpret_cast<const float4 *>(S + (size_t)(rl + i * kStepLanes) * dv);

    const size_t row0 = ((size_t)b * tokens + tok0) * heads + h;   // (b, tok0, h)
    const size_t qk_step = (size_t)heads * DK, v_step = (size_t)heads * dv;
    const T *qb = q + row0 * DK;
    const T *kb = k + row0 * DK;
    const T *vb = v + row0 * dv + col0 + cgi * 4;
    T *ob = out + row0 * dv + col0;

    for (int g0 = 0; g0 < ntok; g0 += kGroup) {
        const int cnt = min(kGroup, ntok - g0);
        // this thread's v columns for the group's tokens
        float vv[kGroup][4];
#pragma unroll
        for (int u = 0; u < kGroup; ++u)
            if (u < cnt) load4<T>(vb + (size_t)(g0 + u) * v_step, vv[u]);
        // rotated q and k rows of the group's tokens
        for (int p = threadIdx.x; p < cnt * kPairs; p += kStepThreads) {
            const int u = p / kPairs, j = p % kPairs;
            const size_t off = (size_t)(g0 + u) * qk_step + 2 * j;
            float q0 = to_f32(qb[off]), q1 = to_f32(qb[off + 1]);
            float k0 = to_f32(kb[off]), k1 = to_f32(kb[off + 1]);
            if (rotate) {
                const float2 cs = rot.cs[(g0 + u) * kPairs + j];
                rotate_pair(q0, q1, cs);
                rotate_pair(k0, k1, cs);
            }
            qs[u][2 * j] = q0; qs[u][2 * j + 1] = q1;
            ks[u][2 * j] = k0; ks[u][2 * j + 1] = k1;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kGroup; ++u) {
            if (u < cnt) {
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int i = 0; i < RPL; ++i) {
                    const int rr = rl + i * kStepLanes;
                    update_row(s[i], acc, g, ks[u][rr], qs[u][rr], vv[u]);
                }
                reduce_lanes(acc);
                if (lane < kStepCols / 4) red[u][warp][lane] = acc;
            }
        }
        __syncthreads();
        if (threadIdx.x < cnt * (kStepCols / 4)) {
            const int u = threadIdx.x / (kStepCols / 4), c = threadIdx.x % (kStepCols / 4);
            write_output<T>(red[u], c, ob + (size_t)(g0 + u) * v_step + 4 * c);
        }
        // The next group's staging rewrites qs and ks only after every
        // thread has passed the barrier above, and red only after the next
        // barrier, which the output threads reach after their reads.
    }
#pragma unroll
    for (int i = 0; i < RPL; ++i)
        *reinterpret_cast<float4 *>(S + (size_t)(rl + i * kStepLanes) * dv) = s[i];
}

// theta_j = 10000^(-2j/dk) for the three head sizes, formed once per process
// (every decode step needs all of them; the power is the costly part).
static const double *host_thetas(int dk) {
    struct Table {
        double t[128];
        explicit Table(int d) {
            for (int j = 0; j < 128; ++j) t[j] = j < d / 2 ? std::pow(10000.0, -2.0 * j / d) : 0.0;
        }
    };
    static const Table t64(64), t128(128), t256(256);
    return dk == 64 ? t64.t : dk == 128 ? t128.t : t256.t;
}

// (cos, sin) of pos * theta_j, theta_j = 10000^(-2j/dk), in float64 on the host
static float2 host_cs(long long pos, int j, int dk) {
    const double two_pi = 6.283185307179586476925286766559;
    const double theta = host_thetas(dk)[j];
    const double a = (double)pos * theta;
    const double r = a - two_pi * std::nearbyint(a / two_pi);
    return make_float2((float)std::cos(r), (float)std::sin(r));
}

template <typename T, int DK>
static cudaError_t launch_step_dk(const void *q, const void *k, const void *v,
                                  const HeadGammas &gam, float *state, void *out,
                                  long long bh_total, int heads, int dv, long long pos,
                                  int rotate, cudaStream_t stream) {
    StepRotation rot;
    for (int j = 0; j < 128; ++j)
        rot.cs[j] = (rotate && j < DK / 2) ? host_cs(pos, j, DK) : make_float2(1.f, 0.f);
    // grid.y holds (sequence, head) rows; more than 65535 of them take several launches
    for (long long bh0 = 0; bh0 < bh_total; bh0 += 65535) {
        const dim3 grid((unsigned)(dv / kStepCols), (unsigned)std::min(65535LL, bh_total - bh0));
        const cudaError_t e = launch_overlapped(
            retention_step_kernel<T, DK>, grid, dim3(kStepThreads), 0, stream, (const T *)q,
            (const T *)k, (const T *)v, gam, rot, state, (T *)out, (int)bh0, heads, dv, rotate,
            bh_total, device_error_word());
        count_launch();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename T, int DK>
static cudaError_t launch_tokens_dk(const void *q, const void *k, const void *v,
                                    const HeadGammas &gam, float *state, void *out,
                                    long long bh_total, int tokens, int heads, int dv,
                                    long long pos, int rotate, cudaStream_t stream) {
    constexpr int kPairs = DK / 2;
    constexpr int kPerLaunch = kRotPairs / kPairs;   // tokens whose rotation fits the parameters
    TokenRotation rot;
    for (int tok0 = 0; tok0 < tokens; tok0 += kPerLaunch) {
        const int ntok = std::min(kPerLaunch, tokens - tok0);
        for (int u = 0; u < ntok; ++u)
            for (int j = 0; j < kPairs; ++j)
                rot.cs[u * kPairs + j] =
                    rotate ? host_cs(pos + tok0 + u, j, DK) : make_float2(1.f, 0.f);
        for (long long bh0 = 0; bh0 < bh_total; bh0 += 65535) {
            const dim3 grid((unsigned)(dv / kStepCols),
                            (unsigned)std::min(65535LL, bh_total - bh0));
            const cudaError_t e = launch_overlapped(
                retention_tokens_kernel<T, DK>, grid, dim3(kStepThreads), 0, stream,
                (const T *)q, (const T *)k, (const T *)v, gam, rot, state, (T *)out, (int)bh0,
                heads, tokens, tok0, ntok, dv, rotate, bh_total, device_error_word());
            count_launch();
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

template <typename T, int DK>
static cudaError_t launch_dk(const void *q, const void *k, const void *v, const HeadGammas &gam,
                             float *state, void *out, int batch, int tokens, int heads, int dv,
                             long long pos, int rotate, cudaStream_t stream) {
    const long long bh_total = (long long)batch * heads;
    return tokens == 1 ? launch_step_dk<T, DK>(q, k, v, gam, state, out, bh_total, heads, dv,
                                                pos, rotate, stream)
                       : launch_tokens_dk<T, DK>(q, k, v, gam, state, out, bh_total, tokens,
                                                  heads, dv, pos, rotate, stream);
}

template <typename T>
static cudaError_t launch_recurrent_t(const void *q, const void *k, const void *v,
                                      const HeadGammas &gam, float *state, void *out, int batch,
                                      int tokens, int heads, int dk, int dv, long long pos,
                                      int rotate, cudaStream_t stream) {
    KernelTimer timer("retention_step", stream);
    switch (dk) {
        case 64:
            return launch_dk<T, 64>(q, k, v, gam, state, out, batch, tokens, heads, dv, pos,
                                    rotate, stream);
        case 128:
            return launch_dk<T, 128>(q, k, v, gam, state, out, batch, tokens, heads, dv, pos,
                                     rotate, stream);
        case 256:
            return launch_dk<T, 256>(q, k, v, gam, state, out, batch, tokens, heads, dv, pos,
                                     rotate, stream);
        default:
            return cudaErrorInvalidValue;
    }
}

cudaError_t launch_retention_recurrent(const void *q, const void *k, const void *v,
                                       const HeadGammas &gam, float *state, void *out,
                                       int batch, int tokens, int heads, int dk, int dv,
                                       retnet_dtype dtype, long long pos, int rotate,
                                       cudaStream_t stream) {
    if (batch == 0 || tokens == 0) return cudaSuccess;
    return dtype == RETNET_BF16
               ? launch_recurrent_t<__nv_bfloat16>(q, k, v, gam, state, out, batch, tokens,
                                                   heads, dk, dv, pos, rotate, stream)
               : launch_recurrent_t<float>(q, k, v, gam, state, out, batch, tokens, heads, dk,
                                           dv, pos, rotate, stream);
}

}  // namespace retnet
