// Chunkwise-recurrent retention on the sm_100a tensor cores (tcgen05/TMEM/TMA).
//
// The chunkwise form computes in parallel within a chunk and carries a
// recurrent state between chunks (RetNet research summary, "Summary";
// "Key points": chunk b = 512, head dimension 256).  For a chunk of L tokens
// (local indices i, j) and head decay g:
//     O_c = (Q K^T (.) D) V + (Q (.) xi) S_prev,  D_ij = g^(i-j) (i >= j),
//     xi_i = g^(i+1),   S_c = g^L S_prev + K^T (V (.) zeta),  zeta_j = g^(L-1-j).
//
// Decay folded into the operands.  With Qt_i = g^(i+1) R q_i and
// Kt_j = g^-(j+1) R k_j (R: the xPos-like rotation), Qt_i . Kt_j =
// g^(i-j) (R q_i . R k_j), so the intra-chunk score needs only the causal
// mask; Qt S_prev is already the xi-scaled cross term; and
// K^T (V (.) zeta) = g^L Kt^T V.  The fold needs g^-L representable with
// room to spare; the host admits a head only when L * log2(1/g) <= 100.
//
// Kernels (all bf16 operands, f32 accumulation):
//   tc_prep    rotation + decay fold of q and k into Qt, Kt [B*H, n, 256]
//   tc_state   per (sequence, head, 128x128 quarter of S): walks the chunks,
//              accumulating Kt^T V onto the state in TMEM, scaling by g^L,
//              and writing S_prev of every chunk (bf16) and the final state
//   tc_output  per (sequence, head, chunk, 128-row block): S = Qt Kt^T in
//              TMEM, causal mask in registers, P (bf16) to shared memory,
//              O += P V; then O += Qt S_prev; epilogue writes O, or
//              swish(G) * GroupNorm(O) when a gate is given.
// Roles inside a CTA: warp 0 issues TMA loads, warp 1 allocates TMEM and
// issues tcgen05.mma, warps 2-5 move data between TMEM, registers and
// memory.  Every mbarrier wait is bounded (about 2 s); on timeout the CTA
// records kDevErrTimeout and unwinds.
#include <cmath>

#include "kernels.h"
#include "sm100.cuh"

namespace retnet {

using namespace sm100;

constexpr int kD = 256;            // head dimension served here (dk = dv = 256)
constexpr int kBlk = 128;          // rows per tile
constexpr int kTcThreads = 192;    // 6 warps
constexpr uint32_t kBox = 16384;   // one 128-row x 64-col bf16 box (128-B swizzle)

struct TcHeadParams {
    float log2g[kMaxHeads];        // log2(gamma_h)
    float decay_chunk[kMaxHeads];  // gamma_h^chunk
    float decay_last[kMaxHeads];   // gamma_h^(length of the last chunk)
};

// ------------------------------------------------------------------ prep
// One thread: 8 consecutive elements (4 rotation pairs) of q and of k for
// one (b, t, h).  Writes Qt, Kt in [b*H + h][t][:] layout.
__global__ void __launch_bounds__(256)
tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
               const float2 *__restrict__ table, TcHeadParams hp, __nv_bfloat16 *__restrict__ qt,
               __nv_bfloat16 *__restrict__ kt, int batch, int heads, int n, int chunk,
               int rotate) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = (long long)batch * n * heads * (kD / 8);
    if (idx >= total) return;
    const int part = (int)(idx % (kD / 8));
    const long long bth = idx / (kD / 8);
    const int h = (int)(bth % heads);
    const long long bt = bth / heads;
    const int t = (int)(bt % n);
    const int b = (int)(bt / n);
    const int i = t % chunk;
    const float e = (float)(i + 1) * hp.log2g[h];
    const float sq = exp2f(e), sk = exp2f(-e);
    float xq[8], xk[8];
    load8(q + bth * kD + part * 8, xq);
    load8(k + bth * kD + part * 8, xk);
    float oq[8], ok[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        float c = sq, s = 0.f, ck = sk, sk2 = 0.f;
        if (rotate) {
            float2 cs = table[(size_t)t * (kD / 2) + part * 4 + p];
            c = cs.x * sq; s = cs.y * sq;
            ck = cs.x * sk; sk2 = cs.y * sk;
        }
        float a = xq[2 * p], bb = xq[2 * p + 1];
        oq[2 * p] = a * c - bb * s;
        oq[2 * p + 1] = a * s + bb * c;
        a = xk[2 * p]; bb = xk[2 * p + 1];
        ok[2 * p] = a * ck - bb * sk2;
        ok[2 * p + 1] = a * sk2 + bb * ck;
    }
    const size_t dst = (((size_t)b * heads + h) * n + t) * kD + part * 8;
    store8(qt + dst, oq);
    store8(kt + dst, ok);
}

// ------------------------------------------------------------------ state pass
struct TcStateSmem {
    static constexpr int kStages = 3;
    static constexpr uint32_t kStage = 4 * kBox;       // Kt 128x128 + V 128x128
    static constexpr uint32_t kBytes = kStages * kStage + 1024;
};

__global__ void __launch_bounds__(kTcThreads, 1)
tc_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                TcHeadParams hp, const float *__restrict__ state_in, float *__restrict__ state_out,
                __nv_bfloat16 *__restrict__ s_prev, int heads, int n, int chunk, int nchunks,
                unsigned *err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int S = TcStateSmem::kStages;
    __shared__ uint64_t full[S], empty[S], acc_full, acc_ready;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.x / 4;
    const int quarter = blockIdx.x % 4;
    const int mh = quarter / 2, nh = quarter % 2;      // d_k half, d_v half
    const int b = bh / heads, h = bh % heads;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_ready, 128);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int it = 0;
            for (int c = 0; c < nchunks && !abort_flag; ++c) {
                const int c0 = c * chunk;
                const int L = min(chunk, n - c0);
                for (int st = 0; st * kBlk < L; ++st, ++it) {
                    const int s = it % S;
                    if (it >= S && !mbar_wait(&empty[s], ((it / S) - 1) & 1, &abort_flag, err))
                        break;
                    uint8_t *kb = smem + s * TcStateSmem::kStage;
                    uint8_t *vb = kb + 2 * kBox;
                    mbar_expect_tx(&full[s], TcStateSmem::kStage);
                    const int t0 = c0 + st * kBlk;
                    for (int x = 0; x < 2; ++x) {
                        tma_load_3d(kb + x * kBox, &tm_k, &full[s], 128 * mh + 64 * x, t0, bh);
                        tma_load_4d(vb + x * kBox, &tm_v, &full[s], 128 * nh + 64 * x, h, t0, b);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, 128, 1, 1);
            int it = 0;
            for (int c = 0; c < nchunks; ++c) {
                if (!mbar_wait(&acc_ready, c & 1, &abort_flag, err)) break;
                tc_fence_after();
                const int L = min(chunk, n - c * chunk);
                bool ok = true;
                for (int st = 0; st * kBlk < L; ++st, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(&full[s], (it / S) & 1, &abort_flag, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t kb = smem_u32(smem + s * TcStateSmem::kStage);
                    const uint32_t vb = kb + 2 * kBox;
#pragma unroll
                    for (int ks = 0; ks < kBlk / 16; ++ks) {
                        // A = Kt^T (M = d_k, K = tokens), B = V (N = d_v, K = tokens):
                        // both MN-major; 16 tokens = two 8-row atoms = 2048 B.
                        uint64_t ad = smem_desc_sw128(kb + ks * 2048, kBox, 1024);
                        uint64_t bd = smem_desc_sw128(vb + ks * 2048, kBox, 1024);
                        mma_bf16(tmem, ad, bd, idesc, 1u);
                    }
                    mma_commit(&empty[s]);
                }
                if (!ok) break;
                mma_commit(&acc_full);
            }
        }
    } else {
        // epilogue warpgroup: warp w owns TMEM lanes 32*(w%4) .. +31
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;                      // row of the d_k half
        const int krow = 128 * mh + row;                     // row of S
        const uint32_t taddr = tmem + ((uint32_t)(32 * q4) << 16);
        const size_t sbase = ((size_t)bh * kD + krow) * kD + 128 * nh;
        // initial state -> TMEM and S_prev[0]
        {
            __nv_bfloat16 *dst = s_prev + (((size_t)bh * nchunks + 0) * kD + krow) * kD + 128 * nh;
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t r[32];
                if (state_in) {
                    const float4 *src = reinterpret_cast<const float4 *>(state_in + sbase + 32 * cb);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4) {
                        float4 f = src[v4];
                        r[4 * v4] = __float_as_uint(f.x); r[4 * v4 + 1] = __float_as_uint(f.y);
                        r[4 * v4 + 2] = __float_as_uint(f.z); r[4 * v4 + 3] = __float_as_uint(f.w);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = 0u;
                }
                tmem_st32(taddr + 32 * cb, r);
                uint4 *o = reinterpret_cast<uint4 *>(dst + 32 * cb);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    o[v] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1])),
                                      pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                                      pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                                      pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&acc_ready);
        }
        for (int c = 0; c < nchunks; ++c) {
            if (!warp_wait(&acc_full, c & 1, &abort_flag, err)) break;
            tc_fence_after();
            const bool last = (c == nchunks - 1);
            const float decay = last ? hp.decay_last[h] : hp.decay_chunk[h];
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t r[32];
                tmem_ld32(taddr + 32 * cb, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * decay);
                if (!last) {
                    tmem_st32(taddr + 32 * cb, r);
                    __nv_bfloat16 *dst =
                        s_prev + (((size_t)bh * nchunks + c + 1) * kD + krow) * kD + 128 * nh + 32 * cb;
                    uint4 *o = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        o[v] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1])),
                                          pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                                          pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                                          pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
                } else if (state_out) {
                    float4 *o = reinterpret_cast<float4 *>(state_out + sbase + 32 * cb);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4)
                        o[v4] = make_float4(__uint_as_float(r[4 * v4]), __uint_as_float(r[4 * v4 + 1]),
                                            __uint_as_float(r[4 * v4 + 2]), __uint_as_float(r[4 * v4 + 3]));
                }
            }
            if (!last) {
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&acc_ready);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ------------------------------------------------------------------ output pass
struct TcOutSmem {
    static constexpr uint32_t kQ = 0;                  // Qt  128 x 256  (4 boxes)
    static constexpr uint32_t kK = 4 * kBox;           // Kt  128 x 256  (4 boxes)
    static constexpr uint32_t kV = 8 * kBox;           // V   128 x 256  (4 boxes)
    static constexpr uint32_t kS = 4 * kBox;           // S_prev 256 x 256 over K and V
    static constexpr uint32_t kP = 12 * kBox;          // P   128 x 128  (2 boxes)
    static constexpr uint32_t kBytes = 14 * kBox + 1024;
};

struct TcOutArgs {
    int heads, n, chunk, nchunks, rblocks, has_state_in;
    __nv_bfloat16 *out;
    const __nv_bfloat16 *gate;
    const float *gn_weight, *gn_bias;
    float eps;
    unsigned *err;
};

__global__ void __launch_bounds__(kTcThreads, 1)
tc_output_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_s,
                 TcOutArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t q_full, k_full, v_full, s_full, k_empty, v_empty, sqk_full, p_full, o_full;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    // heavy row blocks first: blockIdx.x -> (r from the last block down, bh, c)
    const int per_r = gridDim.x / a.rblocks;
    const int r = a.rblocks - 1 - (int)(blockIdx.x / per_r);
    const int rest = blockIdx.x % per_r;
    const int c = rest % a.nchunks;
    const int bh = rest / a.nchunks;
    const int b = bh / a.heads, h = bh % a.heads;
    const int c0 = c * a.chunk;
    const int L = min(a.chunk, a.n - c0);
    if (r * kBlk >= L) return;                            // past a short last chunk
    const bool has_s = (c > 0) || a.has_state_in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    unsigned *err = a.err;

    if (threadIdx.x == 0) {
        mbar_init(&q_full, 1); mbar_init(&k_full, 1); mbar_init(&v_full, 1);
        mbar_init(&s_full, 1); mbar_init(&k_empty, 1); mbar_init(&v_empty, 1);
        mbar_init(&sqk_full, 1); mbar_init(&p_full, 128); mbar_init(&o_full, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t tO = tmem;             // columns   0..255: O  (128 x 256 f32)
    const uint32_t tS = tmem + 256;       // columns 256..383: S  (128 x 128 f32)

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v); tma_prefetch_desc(&tm_s);
            const int tq = c0 + r * kBlk;
            mbar_expect_tx(&q_full, 4 * kBox);
            for (int x = 0; x < 4; ++x)
                tma_load_3d(smem + TcOutSmem::kQ + x * kBox, &tm_q, &q_full, 64 * x, tq, bh);
            for (int t = 0; t <= r; ++t) {
                const int tk = c0 + t * kBlk;
                if (t > 0 && !mbar_wait(&k_empty, (t - 1) & 1, &abort_flag, err)) break;
                mbar_expect_tx(&k_full, 4 * kBox);
                for (int x = 0; x < 4; ++x)
                    tma_load_3d(smem + TcOutSmem::kK + x * kBox, &tm_k, &k_full, 64 * x, tk, bh);
                if (t > 0 && !mbar_wait(&v_empty, (t - 1) & 1, &abort_flag, err)) break;
                mbar_expect_tx(&v_full, 4 * kBox);
                for (int x = 0; x < 4; ++x)
                    tma_load_4d(smem + TcOutSmem::kV + x * kBox, &tm_v, &v_full, 64 * x, h, tk, b);
            }
            if (has_s && !abort_flag && mbar_wait(&k_empty, r & 1, &abort_flag, err) &&
                mbar_wait(&v_empty, r & 1, &abort_flag, err)) {
                mbar_expect_tx(&s_full, 8 * kBox);
                const int srow = (bh * a.nchunks + c) * kD;
                for (int x = 0; x < 4; ++x)
                    tma_load_2d(smem + TcOutSmem::kS + x * 2 * kBox, &tm_s, &s_full, 64 * x, srow);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_pv = idesc_bf16(128, 256, 0, 1);
            const uint32_t sQ = smem_u32(smem + TcOutSmem::kQ);
            const uint32_t sK = smem_u32(smem + TcOutSmem::kK);
            const uint32_t sV = smem_u32(smem + TcOutSmem::kV);
            const uint32_t sP = smem_u32(smem + TcOutSmem::kP);
            const uint32_t sS = smem_u32(smem + TcOutSmem::kS);
            bool ok = mbar_wait(&q_full, 0, &abort_flag, err);
            for (int t = 0; ok && t <= r; ++t) {
                if (!mbar_wait(&k_full, t & 1, &abort_flag, err)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks / 4) * kBox + (ks % 4) * 32;
                    mma_bf16(tS, smem_desc_sw128(sQ + off, 16, 1024),
                             smem_desc_sw128(sK + off, 16, 1024), id_qk, ks > 0);
                }
                mma_commit(&sqk_full);
                mma_commit(&k_empty);
                if (!mbar_wait(&p_full, t & 1, &abort_flag, err)) { ok = false; break; }
                if (!mbar_wait(&v_full, t & 1, &abort_flag, err)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kBlk / 16; ++ks) {
                    const uint32_t offp = (ks / 4) * kBox + (ks % 4) * 32;
                    mma_bf16(tO, smem_desc_sw128(sP + offp, 16, 1024),
                             smem_desc_sw128(sV + ks * 2048, kBox, 1024), id_pv,
                             (t > 0 || ks > 0) ? 1u : 0u);
                }
                mma_commit(&v_empty);
            }
            if (ok && has_s) {
                if (mbar_wait(&s_full, 0, &abort_flag, err)) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t off = (ks / 4) * kBox + (ks % 4) * 32;
                        mma_bf16(tO, smem_desc_sw128(sQ + off, 16, 1024),
                                 smem_desc_sw128(sS + ks * 2048, 2 * kBox, 1024), id_pv, 1u);
                    }
                }
            }
            mma_commit(&o_full);
        }
    } else {
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;                         // row of the 128-row block
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        uint8_t *prow = smem + TcOutSmem::kP + row * 128;
        bool ok = true;
        for (int t = 0; t <= r; ++t) {
            if (!warp_wait(&sqk_full, t & 1, &abort_flag, err)) { ok = false; break; }
            if (t > 0 && !warp_wait(&v_empty, (t - 1) & 1, &abort_flag, err)) { ok = false; break; }
            tc_fence_after();
            const bool diag = (t == r);
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t v[32];
                tmem_ld32(tS + lane_off + 32 * cb, v);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {          // 16-byte chunks of 8 columns
                    uint32_t w[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const int j0 = 32 * cb + 8 * ch + 2 * e2;
                        float lo = __uint_as_float(v[8 * ch + 2 * e2]);
                        float hi = __uint_as_float(v[8 * ch + 2 * e2 + 1]);
                        if (diag) {
                            lo = (row >= j0) ? lo : 0.f;
                            hi = (row >= j0 + 1) ? hi : 0.f;
                        }
                        w[e2] = pack_bf16x2(lo, hi);
                    }
                    const int col = 32 * cb + 8 * ch;             // first column of the chunk
                    const int box = col / 64;
                    const int c16 = (col % 64) / 8;
                    uint4 *dst = reinterpret_cast<uint4 *>(prow + box * kBox +
                                                           ((c16 ^ (row & 7)) * 16));
                    *dst = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_async_shared();
            tc_fence_before();
            mbar_arrive(&p_full);
        }
        if (ok && warp_wait(&o_full, 0, &abort_flag, err)) {
            tc_fence_after();
            // Every lane runs the TMEM loads (they are warp-collective); only
            // rows inside the sequence store.
            const int t = c0 + r * kBlk + row;
            const bool valid = t < a.n;
            __nv_bfloat16 *orow = a.out + (((size_t)b * a.n + (valid ? t : 0)) * a.heads + h) * kD;
            if (!a.gate) {
#pragma unroll 1
                for (int cb = 0; cb < 8; ++cb) {
                    uint32_t v[32];
                    tmem_ld32(tO + lane_off + 32 * cb, v);
                    tmem_wait_ld();
                    if (valid) {
                        uint4 *o = reinterpret_cast<uint4 *>(orow + 32 * cb);
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8)
                            o[q8] = make_uint4(
                                pack_bf16x2(__uint_as_float(v[8 * q8]), __uint_as_float(v[8 * q8 + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * q8 + 2]), __uint_as_float(v[8 * q8 + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * q8 + 4]), __uint_as_float(v[8 * q8 + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * q8 + 6]), __uint_as_float(v[8 * q8 + 7])));
                    }
                }
            } else {
                // GroupNorm over this row's 256 channels, then the swish gate
                float sum = 0.f;
#pragma unroll 1
                for (int cb = 0; cb < 8; ++cb) {
                    uint32_t v[32];
                    tmem_ld32(tO + lane_off + 32 * cb, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) sum += __uint_as_float(v[e]);
                }
                const float mean = sum * (1.f / kD);
                float sq = 0.f;
#pragma unroll 1
                for (int cb = 0; cb < 8; ++cb) {
                    uint32_t v[32];
                    tmem_ld32(tO + lane_off + 32 * cb, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float d = __uint_as_float(v[e]) - mean;
                        sq = fmaf(d, d, sq);
                    }
                }
                const float rstd = rsqrtf(sq * (1.f / kD) + a.eps);
                const __nv_bfloat16 *grow =
                    a.gate + (((size_t)b * a.n + (valid ? t : 0)) * a.heads + h) * kD;
                const float *wv = a.gn_weight ? a.gn_weight + h * kD : nullptr;
                const float *bv = a.gn_bias ? a.gn_bias + h * kD : nullptr;
#pragma unroll 1
                for (int cb = 0; cb < 8; ++cb) {
                    uint32_t v[32];
                    tmem_ld32(tO + lane_off + 32 * cb, v);
                    tmem_wait_ld();
                    if (valid) {
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8) {
                            float gv[8], y[8];
                            load8(grow + 32 * cb + 8 * q8, gv);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int ch = 32 * cb + 8 * q8 + e;
                                float yh = (__uint_as_float(v[8 * q8 + e]) - mean) * rstd;
                                if (wv) yh *= wv[ch];
                                if (bv) yh += bv[ch];
                                y[e] = gv[e] / (1.f + __expf(-gv[e])) * yh;
                            }
                            store8(orow + 32 * cb + 8 * q8, y);
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return (EncodeTiledFn)p;
    }();
    return fn;
}

// bf16 tensor map, 128-byte swizzle, innermost dimension first.
static bool make_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                     const cuuint64_t *strides_bytes, const cuuint32_t *box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base),
                    dims, strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static size_t align1k(size_t x) { return (x + 1023) & ~(size_t)1023; }

struct TcLayout {
    size_t table, qt, kt, sprev, total;
};

static TcLayout tc_layout(int batch, int heads, int n, int chunk) {
    TcLayout l;
    const size_t bh = (size_t)batch * heads;
    const size_t nchunks = ((size_t)n + chunk - 1) / chunk;
    l.table = 0;
    l.qt = align1k((size_t)n * (kD / 2) * sizeof(float2));
    l.kt = l.qt + align1k(bh * n * kD * 2);
    l.sprev = l.kt + align1k(bh * n * kD * 2);
    l.total = l.sprev + align1k(bh * nchunks * kD * kD * 2);
    return l;
}

bool tc_shape_ok(int dk, int dv, retnet_dtype dtype, int chunk) {
    if (dk != kD || dv != kD || dtype != RETNET_BF16) return false;
    return chunk == 128 || chunk == 256 || chunk == 512 || chunk == 1024;
}

bool tc_gammas_ok(int chunk, const float *gammas, int heads) {
    for (int h = 0; h < heads; ++h) {
        const double g = gammas[h];
        if (!(g > 0.0)) return false;
        if (chunk * -std::log2(g) > 100.0) return false;
    }
    return true;
}

size_t tc_workspace_bytes(int batch, int heads, int seqlen, int chunk) {
    return tc_layout(batch, heads, seqlen, chunk).total;
}

cudaError_t launch_chunkwise_tc(const ChunkwiseArgs &a, const float *gammas, cudaStream_t stream) {
    const int n = a.seqlen, H = a.heads, B = a.batch, C = a.chunk;
    const int BH = B * H;
    if (BH == 0) return cudaSuccess;
    if (n == 0) {                                   // nothing to scan: state passes through
        if (!a.state_out) return cudaSuccess;
        size_t bytes = (size_t)BH * kD * kD * sizeof(float);
        if (a.state_in)
            return a.state_in == a.state_out
                       ? cudaSuccess
                       : cudaMemcpyAsync(a.state_out, a.state_in, bytes, cudaMemcpyDeviceToDevice,
                                         stream);
        return cudaMemsetAsync(a.state_out, 0, bytes, stream);
    }
    const int nchunks = (n + C - 1) / C;
    const int last_len = n - (nchunks - 1) * C;
    const TcLayout lay = tc_layout(B, H, n, C);
    char *ws = (char *)a.workspace;
    float2 *table = (float2 *)(ws + lay.table);
    __nv_bfloat16 *qt = (__nv_bfloat16 *)(ws + lay.qt);
    __nv_bfloat16 *kt = (__nv_bfloat16 *)(ws + lay.kt);
    __nv_bfloat16 *sp = (__nv_bfloat16 *)(ws + lay.sprev);
    unsigned *err = device_error_word();
    if (!err) return cudaErrorInvalidValue;

    TcHeadParams hp;
    for (int h = 0; h < kMaxHeads; ++h) hp.log2g[h] = hp.decay_chunk[h] = hp.decay_last[h] = 0.f;
    for (int h = 0; h < H; ++h) {
        const double g = gammas[h];
        hp.log2g[h] = (float)std::log2(g);
        hp.decay_chunk[h] = (float)std::pow(g, (double)C);
        hp.decay_last[h] = (float)std::pow(g, (double)last_len);
    }

    // tensor maps
    CUtensorMap tm_q, tm_k, tm_v, tm_s;
    {
        cuuint64_t dims[3] = {kD, (cuuint64_t)n, (cuuint64_t)BH};
        cuuint64_t str[2] = {kD * 2, (cuuint64_t)n * kD * 2};
        cuuint32_t box[3] = {64, kBlk, 1};
        if (!make_map(&tm_q, qt, 3, dims, str, box) || !make_map(&tm_k, kt, 3, dims, str, box))
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[4] = {kD, (cuuint64_t)H, (cuuint64_t)n, (cuuint64_t)B};
        cuuint64_t str[3] = {kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)n * H * kD * 2};
        cuuint32_t box[4] = {64, 1, kBlk, 1};
        if (!make_map(&tm_v, a.v, 4, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {kD, (cuuint64_t)BH * nchunks * kD};
        cuuint64_t str[1] = {kD * 2};
        cuuint32_t box[2] = {64, 256};
        if (!make_map(&tm_s, sp, 2, dims, str, box)) return cudaErrorInvalidValue;
    }

    cudaError_t e;
    if (a.rotate) {
        e = launch_rotation_table(table, n, kD, a.pos0, stream);
        if (e != cudaSuccess) return e;
    }
    {
        const long long total = (long long)B * n * H * (kD / 8);
        const unsigned blocks = (unsigned)((total + 255) / 256);
        KernelTimer timer("tc_prep", stream);
        tc_prep_kernel<<<blocks, 256, 0, stream>>>((const __nv_bfloat16 *)a.q,
                                                   (const __nv_bfloat16 *)a.k, table, hp, qt, kt,
                                                   B, H, n, C, a.rotate);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const int smem = (int)TcStateSmem::kBytes;
        e = cudaFuncSetAttribute(tc_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        KernelTimer timer("tc_state", stream);
        tc_state_kernel<<<BH * 4, kTcThreads, smem, stream>>>(tm_k, tm_v, hp, a.state_in,
                                                             a.state_out, sp, H, n, C, nchunks,
                                                             err);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        TcOutArgs oa;
        oa.heads = H; oa.n = n; oa.chunk = C; oa.nchunks = nchunks; oa.rblocks = C / kBlk;
        oa.has_state_in = a.state_in != nullptr;
        oa.out = (__nv_bfloat16 *)a.out;
        oa.gate = a.gate ? (const __nv_bfloat16 *)a.gate->g : nullptr;
        oa.gn_weight = a.gate ? a.gate->weight : nullptr;
        oa.gn_bias = a.gate ? a.gate->bias : nullptr;
        oa.eps = a.gate ? a.gate->eps : 0.f;
        oa.err = err;
        const int smem = (int)TcOutSmem::kBytes;
        e = cudaFuncSetAttribute(tc_output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem);
        if (e != cudaSuccess) return e;
        const unsigned grid = (unsigned)(BH * nchunks * oa.rblocks);
        KernelTimer timer("tc_output", stream);
        tc_output_kernel<<<grid, kTcThreads, smem, stream>>>(tm_q, tm_k, tm_v, tm_s, oa);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace retnet
