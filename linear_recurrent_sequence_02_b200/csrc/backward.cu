// Streaming passes of the backward pass.
//
// The gradients of retention (RetNet research summary, "Summary": the
// parallel form is the one used for training) are three causal retentions:
//     dQ^ = ret(dO, V, K^),  dK^ = rev ret(rev V, rev dO, rev Q^),
//     dV  = rev ret(rev K^, rev Q^, rev dO),
// with Q^ = R q, K^ = R k the rotated inputs and rev() time reversal; then
// dq = R^T dQ^ and dk = R^T dK^.  The retentions run on the forward
// chunkwise kernels; these two kernels form their inputs and bring their
// outputs back:
//   backward_prep_kernel  reads q, k, v, dO once and writes K^ and the
//                         reversed sequences of Q^, K^, V and dO;
//   backward_post_kernel  writes dq = R^T dQ^ (in place), dk = R^T rev(dK~)
//                         and dv = rev(dV~), where dK~, dV~ are the outputs
//                         of the two reversed-time retentions.
// One CTA per token t: the token's (cos, sin) pairs are formed once in
// shared memory and serve every (sequence, head) row; each thread moves
// 8-element parts of rows, all loads of a round first.
#include "kernels.h"

namespace retnet {

constexpr int kBwdThreads = 256;
constexpr int kBwdBatch = 2;       // parts in flight per thread and tensor

// Eight elements as loaded (16 bytes of bf16, 32 of float), converted to
// float only when used, so that the loads of a round stay few registers.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { u = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ void to_float(float *e) const {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            e[2 * i] = f.x;
            e[2 * i + 1] = f.y;
        }
    }
    __device__ __forceinline__ void store(__nv_bfloat16 *p) const { *reinterpret_cast<uint4 *>(p) = u; }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = reinterpret_cast<const float4 *>(p)[0];
        b = reinterpret_cast<const float4 *>(p)[1];
    }
    __device__ __forceinline__ void to_float(float *e) const {
        e[0] = a.x; e[1] = a.y; e[2] = a.z; e[3] = a.w;
        e[4] = b.x; e[5] = b.y; e[6] = b.z; e[7] = b.w;
    }
    __device__ __forceinline__ void store(float *p) const {
        reinterpret_cast<float4 *>(p)[0] = a;
        reinterpret_cast<float4 *>(p)[1] = b;
    }
};

__device__ __forceinline__ void turn(float *e, const float2 *cs, float sign) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float c = cs[p].x, s = sign * cs[p].y;
        const float a = e[2 * p], b = e[2 * p + 1];
        e[2 * p] = a * c - b * s;
        e[2 * p + 1] = a * s + b * c;
    }
}

// Row-part task index -> element offsets of token t and of token n-1-t.
struct PartIndex {
    size_t at_t, at_rev;
    int part;
};
__device__ __forceinline__ PartIndex part_index(int task, int parts, int heads, int n, int t,
                                                int d) {
    PartIndex x;
    x.part = task % parts;
    const int bh = task / parts;
    const int b = bh / heads, h = bh % heads;
    x.at_t = (((size_t)b * n + t) * heads + h) * d + x.part * 8;
    x.at_rev = (((size_t)b * n + (n - 1 - t)) * heads + h) * d + x.part * 8;
    return x;
}

__device__ __forceinline__ void token_table(float2 *cs, int dk, long long pos, int rotate,
                                            const BackwardThetas &th) {
    if ((int)threadIdx.x < dk / 2)
        cs[threadIdx.x] = rotate ? rotation_cs(pos, th.theta[threadIdx.x]) : make_float2(1.f, 0.f);
    __syncthreads();
}

// Each round: up to kBwdBatch (q, k) parts and kBwdBatch (v, dO) parts per
// thread, all loads issued before any is used.
template <typename T>
__global__ void __launch_bounds__(kBwdThreads, sizeof(T) == 2 ? 4 : 2)
backward_prep_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const T *__restrict__ dout, T *__restrict__ kh, T *__restrict__ rkh,
                     T *__restrict__ rqh, T *__restrict__ rv, T *__restrict__ rdo,
                     BackwardThetas th, int batch, int heads, int n, int dk, int dv,
                     long long pos0, int rotate) {
    __shared__ float2 cs[128];
    const int t = blockIdx.x;
    token_table(cs, dk, pos0 + t, rotate, th);
    const int rows = batch * heads;
    const int pk = dk / 8, pv = dv / 8;
    const int tk = rows * pk, tv = rows * pv;
    for (int base = threadIdx.x; base < max(tk, tv); base += kBwdBatch * kBwdThreads) {
        Raw8<T> rq[kBwdBatch], rk[kBwdBatch], rvv[kBwdBatch], ro[kBwdBatch];
#pragma unroll
        for (int u = 0; u < kBwdBatch; ++u) {
            const int task = base + u * kBwdThreads;
            if (task < tk) {
                const PartIndex x = part_index(task, pk, heads, n, t, dk);
                rq[u].load(q + x.at_t);
                rk[u].load(k + x.at_t);
            }
            if (task < tv) {
                const PartIndex x = part_index(task, pv, heads, n, t, dv);
                rvv[u].load(v + x.at_t);
                ro[u].load(dout + x.at_t);
            }
        }
#pragma unroll
        for (int u = 0; u < kBwdBatch; ++u) {
            const int task = base + u * kBwdThreads;
            if (task < tk) {
                const PartIndex x = part_index(task, pk, heads, n, t, dk);
                float eq[8], ek[8];
                rq[u].to_float(eq);
                rk[u].to_float(ek);
                turn(eq, cs + 4 * x.part, 1.f);
                turn(ek, cs + 4 * x.part, 1.f);
                store8(kh + x.at_t, ek);
                store8(rkh + x.at_rev, ek);
                store8(rqh + x.at_rev, eq);
            }
            if (task < tv) {
                const PartIndex x = part_index(task, pv, heads, n, t, dv);
                rvv[u].store(rv + x.at_rev);
                ro[u].store(rdo + x.at_rev);
            }
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads, sizeof(T) == 2 ? 4 : 2)
backward_post_kernel(T *__restrict__ dq, const T *__restrict__ dk_rev,
                     const T *__restrict__ dv_rev, T *__restrict__ dk, T *__restrict__ dv,
                     BackwardThetas th, int batch, int heads, int n, int dkd, int dvd,
                     long long pos0, int rotate) {
    __shared__ float2 cs[128];
    const int t = blockIdx.x;
    token_table(cs, dkd, pos0 + t, rotate, th);
    const int rows = batch * heads;
    const int pk = dkd / 8, pv = dvd / 8;
    const int tk = rows * pk, tv = rows * pv;
    for (int base = threadIdx.x; base < max(tk, tv); base += kBwdBatch * kBwdThreads) {
        Raw8<T> rq[kBwdBatch], rk[kBwdBatch], rvv[kBwdBatch];
#pragma unroll
        for (int u = 0; u < kBwdBatch; ++u) {
            const int task = base + u * kBwdThreads;
            if (task < tk) {
                const PartIndex x = part_index(task, pk, heads, n, t, dkd);
                rq[u].load(dq + x.at_t);
                rk[u].load(dk_rev + x.at_rev);
            }
            if (task < tv) {
                const PartIndex x = part_index(task, pv, heads, n, t, dvd);
                rvv[u].load(dv_rev + x.at_rev);
            }
        }
#pragma unroll
        for (int u = 0; u < kBwdBatch; ++u) {
            const int task = base + u * kBwdThreads;
            if (task < tk) {
                // dq = R^T dQ^ in place; dk = R^T (dK~ at the reversed token)
                const PartIndex x = part_index(task, pk, heads, n, t, dkd);
                float eq[8], ek[8];
                rq[u].to_float(eq);
                rk[u].to_float(ek);
                turn(eq, cs + 4 * x.part, -1.f);
                turn(ek, cs + 4 * x.part, -1.f);
                store8(dq + x.at_t, eq);
                store8(dk + x.at_t, ek);
            }
            if (task < tv) {
                // dv = dV~ at the reversed token
                const PartIndex x = part_index(task, pv, heads, n, t, dvd);
                rvv[u].store(dv + x.at_t);
            }
        }
    }
}

BackwardThetas backward_thetas(int dk) {
    BackwardThetas th;
    for (int j = 0; j < 128; ++j) th.theta[j] = j < dk / 2 ? std::pow(10000.0, -2.0 * j / dk) : 0.0;
    return th;
}

// The tensor-core backward (bf16, d = 256): the same reads, but the three
// retentions' operands are written already in the form their prep pass
// would give, so that they run without it.  With e = (position mod fold) + 1
// in each retention's own time order (t forward, p = n-1-t reversed):
//   ret 1 (dQ^):  Qt = g^e dO,      Kt = g^-e V,       values R k   at t
//   ret 2 (dK~):  Qt = g^e V,       Kt = g^-e dO,      values R q   at p
//   ret 3 (dV~):  Qt = g^e (R k),   Kt = g^-e (R q),   values dO    at p
// Qt, Kt in the prefill's [b*H + h][time][256] layout, values in [B, n, H, 256].
struct BackwardFold {
    float log2g[kMaxHeads];
};

__global__ void __launch_bounds__(kBwdThreads, 2)
backward_fold_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                     const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dout,
                     __nv_bfloat16 *__restrict__ qt1, __nv_bfloat16 *__restrict__ kt1,
                     __nv_bfloat16 *__restrict__ val1, __nv_bfloat16 *__restrict__ qt2,
                     __nv_bfloat16 *__restrict__ kt2, __nv_bfloat16 *__restrict__ val2,
                     __nv_bfloat16 *__restrict__ qt3, __nv_bfloat16 *__restrict__ kt3,
                     __nv_bfloat16 *__restrict__ val3, BackwardThetas th, BackwardFold bf,
                     int batch, int heads, int n, int fold, long long pos0, int rotate) {
    constexpr int D = 256, kParts = D / 8;
    using T = __nv_bfloat16;
    __shared__ float2 cs[128];
    const int t = blockIdx.x, p = n - 1 - t;
    token_table(cs, D, pos0 + t, rotate, th);
    const float e1 = (float)(t % fold + 1), e2 = (float)(p % fold + 1);
    const int tasks = batch * heads * kParts;
    for (int base = threadIdx.x; base < tasks; base += kBwdBatch * kBwdThreads) {
        Raw8<T> rq[kBwdBatch], rk[kBwdBatch], rvv[kBwdBatch], ro[kBwdBatch];
#pragma unroll
        for (int u = 0; u < kBwdBatch; ++u) {
            const int task = base + u * kBwdThreads;
            if (task < tasks) {
                const PartIndex x = part_index(task, kParts, heads, n, t, D);
                rq[u].load(q + x.at_t);
                rk[u].load(k + x.at_t);
                rvv[u].load(v + x.at_t);
                ro[u].load(dout + x.at_t);
            }
        }
#pragma unroll
        for (int u = 0; u < kBwdBatch; ++u) {
            const int task = base + u * kBwdThreads;
            if (task >= tasks) continue;
            const PartIndex x = part_index(task, kParts, heads, n, t, D);
            const int bh = task / kParts, h = bh % heads;
            // rows of the [b*H + h][time][256] operands at t and at p
            const size_t ot = ((size_t)bh * n + t) * D + x.part * 8;
            const size_t op = ((size_t)bh * n + p) * D + x.part * 8;
            const float l2 = bf.log2g[h];
            const float s1 = exp2f(e1 * l2), s1i = exp2f(-e1 * l2);
            const float s2 = exp2f(e2 * l2), s2i = exp2f(-e2 * l2);
            float eq[8], ek[8], ev[8], eo[8], y[8];
            rq[u].to_float(eq);
            rk[u].to_float(ek);
            rvv[u].to_float(ev);
            ro[u].to_float(eo);
            turn(eq, cs + 4 * x.part, 1.f);
            turn(ek, cs + 4 * x.part, 1.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = s1 * eo[i];
            store8(qt1 + ot, y);
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = s1i * ev[i];
            store8(kt1 + ot, y);
            store8(val1 + x.at_t, ek);
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = s2 * ev[i];
            store8(qt2 + op, y);
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = s2i * eo[i];
            store8(kt2 + op, y);
            store8(val2 + x.at_rev, eq);
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = s2 * ek[i];
            store8(qt3 + op, y);
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = s2i * eq[i];
            store8(kt3 + op, y);
            ro[u].store(val3 + x.at_rev);
        }
    }
}

cudaError_t launch_backward_fold(const void *q, const void *k, const void *v, const void *dout,
                                 void *const *qt, void *const *kt, void *const *vals,
                                 const float *gammas, int batch, int heads, int n, int fold,
                                 long long pos0, int rotate, cudaStream_t stream) {
    if ((long long)batch * n == 0) return cudaSuccess;
    const BackwardThetas th = backward_thetas(256);
    BackwardFold bf;
    for (int h = 0; h < kMaxHeads; ++h)
        bf.log2g[h] = h < heads ? (float)std::log2((double)gammas[h]) : 0.f;
    using T = __nv_bfloat16;
    KernelTimer timer("backward_prep", stream);
    backward_fold_kernel<<<n, kBwdThreads, 0, stream>>>(
        (const T *)q, (const T *)k, (const T *)v, (const T *)dout, (T *)qt[0], (T *)kt[0],
        (T *)vals[0], (T *)qt[1], (T *)kt[1], (T *)vals[1], (T *)qt[2], (T *)kt[2], (T *)vals[2],
        th, bf, batch, heads, n, fold, pos0, rotate);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_backward_prep(const void *q, const void *k, const void *v, const void *dout,
                                 void *kh, void *rkh, void *rqh, void *rv, void *rdo, int batch,
                                 int heads, int n, int dk, int dv, retnet_dtype dtype,
                                 long long pos0, int rotate, cudaStream_t stream) {
    if ((long long)batch * n == 0) return cudaSuccess;
    const BackwardThetas th = backward_thetas(dk);
    KernelTimer timer("backward_prep", stream);
    if (dtype == RETNET_BF16) {
        using T = __nv_bfloat16;
        backward_prep_kernel<T><<<n, kBwdThreads, 0, stream>>>(
            (const T *)q, (const T *)k, (const T *)v, (const T *)dout, (T *)kh, (T *)rkh,
            (T *)rqh, (T *)rv, (T *)rdo, th, batch, heads, n, dk, dv, pos0, rotate);
    } else {
        backward_prep_kernel<float><<<n, kBwdThreads, 0, stream>>>(
            (const float *)q, (const float *)k, (const float *)v, (const float *)dout,
            (float *)kh, (float *)rkh, (float *)rqh, (float *)rv, (float *)rdo, th, batch, heads,
            n, dk, dv, pos0, rotate);
    }
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_backward_post(void *dq, const void *dk_rev, const void *dv_rev, void *dk,
                                 void *dv, int batch, int heads, int n, int dkd, int dvd,
                                 retnet_dtype dtype, long long pos0, int rotate,
                                 cudaStream_t stream) {
    if ((long long)batch * n == 0) return cudaSuccess;
    const BackwardThetas th = backward_thetas(dkd);
    KernelTimer timer("backward_post", stream);
    if (dtype == RETNET_BF16) {
        using T = __nv_bfloat16;
        backward_post_kernel<T><<<n, kBwdThreads, 0, stream>>>(
            (T *)dq, (const T *)dk_rev, (const T *)dv_rev, (T *)dk, (T *)dv, th, batch, heads, n,
            dkd, dvd, pos0, rotate);
    } else {
        backward_post_kernel<float><<<n, kBwdThreads, 0, stream>>>(
            (float *)dq, (const float *)dk_rev, (const float *)dv_rev, (float *)dk, (float *)dv,
            th, batch, heads, n, dkd, dvd, pos0, rotate);
    }
    count_launch();
    return cudaGetLastError();
}

}  // namespace retnet
