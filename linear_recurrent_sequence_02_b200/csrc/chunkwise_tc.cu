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
// One CTA per token t: its 128 (cos, sin) pairs are formed once (angle
// (pos0 + t) * theta_j in float64, reduced to [-pi, pi], then a float32
// sincos) and applied to every (sequence, head) row of q and k at that
// token, together with the decay fold.  Writes Qt, Kt in [b*H + h][t][:].
struct TcPrepParams {
    double theta[kD / 2];          // 10000^(-2j/256), formed on the host
    float log2g[kMaxHeads];        // log2(gamma_h)
};

__global__ void __launch_bounds__(256)
tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
               TcPrepParams pp, __nv_bfloat16 *__restrict__ qt, __nv_bfloat16 *__restrict__ kt,
               int batch, int heads, int n, int chunk, long long pos0, int rotate) {
    __shared__ float2 cs[kD / 2];
    const int t = blockIdx.x;
    if (threadIdx.x < kD / 2) {
        float2 v = make_float2(1.f, 0.f);
        if (rotate) {
            const double two_pi = 6.283185307179586476925286766559;
            const double inv_two_pi = 0.15915494309189533576888376337251;
            const double a = (double)(pos0 + t) * pp.theta[threadIdx.x];
            const double red = a - two_pi * rint(a * inv_two_pi);
            float sn, cn;
            sincosf((float)red, &sn, &cn);
            v = make_float2(cn, sn);
        }
        cs[threadIdx.x] = v;
    }
    __syncthreads();
    const int i = t % chunk;                        // index inside the chunk
    const int tasks = batch * heads * (kD / 8);
    for (int task = threadIdx.x; task < tasks; task += blockDim.x) {
        const int part = task % (kD / 8);
        const int bhi = task / (kD / 8);
        const int h = bhi % heads, b = bhi / heads;
        const float e = (float)(i + 1) * pp.log2g[h];
        const float sq = exp2f(e), sk = exp2f(-e);
        const size_t src = (((size_t)b * n + t) * heads + h) * kD + part * 8;
        float xq[8], xk[8], oq[8], ok[8];
        load8(q + src, xq);
        load8(k + src, xk);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 r = cs[part * 4 + p];
            const float cq = r.x * sq, sq2 = r.y * sq, ck = r.x * sk, sk2 = r.y * sk;
            float a = xq[2 * p], bb = xq[2 * p + 1];
            oq[2 * p] = a * cq - bb * sq2;
            oq[2 * p + 1] = a * sq2 + bb * cq;
            a = xk[2 * p]; bb = xk[2 * p + 1];
            ok[2 * p] = a * ck - bb * sk2;
            ok[2 * p + 1] = a * sk2 + bb * ck;
        }
        const size_t dst = (((size_t)b * heads + h) * n + t) * kD + part * 8;
        store8(qt + dst, oq);
        store8(kt + dst, ok);
    }
}

// ------------------------------------------------------------------ state pass
// One CTA per (sequence, head, 128x128 quarter of S).  Warp 0 streams Kt and
// V sub-tiles of 128 tokens through a 3-stage TMA ring; warp 1 accumulates
// U_c = Kt_c^T V_c of every chunk into one of two TMEM buffers (M = d_k
// quarter, N = d_v quarter, both operands MN-major); warps 2-5 keep the
// running state row in registers, S <- g^L (S + U_c), hand the buffer back
// as soon as it is read, and write S_prev of the next chunk (bf16) or the
// final state (f32).  The tensor core never waits for the state update.
struct TcStateSmem {
    static constexpr int kStages = 3;
    static constexpr uint32_t kStage = 4 * kBox;       // Kt 128x128 + V 128x128
    static constexpr uint32_t kBytes = kStages * kStage + 1024;
};

__device__ __forceinline__ void store_bf16_row(__nv_bfloat16 *dst, const float *v, int count) {
    for (int i = 0; i < count; i += 8)
        *reinterpret_cast<uint4 *>(dst + i) =
            make_uint4(sm100::pack_bf16x2(v[i], v[i + 1]), sm100::pack_bf16x2(v[i + 2], v[i + 3]),
                       sm100::pack_bf16x2(v[i + 4], v[i + 5]), sm100::pack_bf16x2(v[i + 6], v[i + 7]));
}

__global__ void __launch_bounds__(kTcThreads, 1)
tc_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                TcHeadParams hp, const float *__restrict__ state_in, float *__restrict__ state_out,
                __nv_bfloat16 *__restrict__ s_prev, int heads, int n, int chunk, int nchunks,
                unsigned *err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int S = TcStateSmem::kStages;
    __shared__ uint64_t full[S], empty[S], acc_full[2], acc_free[2];
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
        for (int x = 0; x < 2; ++x) {
            mbar_init(&acc_full[x], 1);
            mbar_init(&acc_free[x], 128);
        }
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 256);
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
            bool ok = true;
            for (int c = 0; ok && c < nchunks; ++c) {
                const int buf = c & 1;
                if (c >= 2 && !mbar_wait(&acc_free[buf], ((c - 2) >> 1) & 1, &abort_flag, err)) break;
                tc_fence_after();
                const int L = min(chunk, n - c * chunk);
                uint32_t accumulate = 0;
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
                        const uint64_t ad = smem_desc_sw128(kb + ks * 2048, kBox, 1024);
                        const uint64_t bd = smem_desc_sw128(vb + ks * 2048, kBox, 1024);
                        mma_bf16(tmem + 128 * buf, ad, bd, idesc, accumulate);
                        accumulate = 1;
                    }
                    mma_commit(&empty[s]);
                }
                if (ok) mma_commit(&acc_full[buf]);
            }
        }
    } else {
        // state warpgroup: warp w owns TMEM lanes 32*(w%4) .. +31 = rows of the d_k half
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;
        const int krow = 128 * mh + row;                     // row of S
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const size_t sbase = ((size_t)bh * kD + krow) * kD + 128 * nh;
        float st[128];
        if (state_in) {
            const float4 *src = reinterpret_cast<const float4 *>(state_in + sbase);
#pragma unroll
            for (int v4 = 0; v4 < 32; ++v4) {
                const float4 f = src[v4];
                st[4 * v4] = f.x; st[4 * v4 + 1] = f.y; st[4 * v4 + 2] = f.z; st[4 * v4 + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 128; ++e) st[e] = 0.f;
        }
        store_bf16_row(s_prev + ((size_t)bh * nchunks * kD + krow) * kD + 128 * nh, st, 128);
        for (int c = 0; c < nchunks; ++c) {
            const int buf = c & 1;
            if (!warp_wait(&acc_full[buf], (c >> 1) & 1, &abort_flag, err)) break;
            tc_fence_after();
            const bool last = (c == nchunks - 1);
            const float decay = last ? hp.decay_last[h] : hp.decay_chunk[h];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t v[32];
                tmem_ld32(tmem + 128 * buf + lane_off + 32 * cb, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    st[32 * cb + e] = decay * (st[32 * cb + e] + __uint_as_float(v[e]));
            }
            tc_fence_before();
            mbar_arrive(&acc_free[buf]);                     // buffer free for chunk c + 2
            if (!last) {
                store_bf16_row(s_prev + (((size_t)bh * nchunks + c + 1) * kD + krow) * kD + 128 * nh,
                               st, 128);
            } else if (state_out) {
                float4 *o = reinterpret_cast<float4 *>(state_out + sbase);
#pragma unroll
                for (int v4 = 0; v4 < 32; ++v4)
                    o[v4] = make_float4(st[4 * v4], st[4 * v4 + 1], st[4 * v4 + 2], st[4 * v4 + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ output pass
// One CTA per (sequence, head, chunk, 128-row block), heavy blocks first.
// TMEM (512 columns): O [0,256) f32; Qt [256,384) bf16 pairs (A operand);
// two S/P buffers [384,448) and [448,512): S = Qt Kt^T for a 64-key tile in
// f32; P (bf16 pairs, A operand of P V) for keys 0-31 overwrites columns
// 0-15 and for keys 32-63 columns 32-47 of the same buffer.
// Shared memory: a K ring (3 x 32 KB) carrying the Kt tiles with the four
// 64-row parts of S_prev interleaved, a V ring (2 x 32 KB), and a 64 KB
// tile buffer that holds Qt (TMA, then copied to TMEM by tcgen05.cp), then
// the gate G, then the output rows for the TMA store.
// Warps: 0 TMA, 1 MMA (+ TMEM allocation), 2-9 two warpgroups that split
// the columns of every TMEM row (S/P tiles: 32 + 32; O: 128 + 128).
// MMA order per key tile t: QK^T(t), Qt S_prev part t (t < 4), P V(t-1),
// so the mask pass of one tile overlaps the tensor core work around it.
constexpr int kKeyTile = 64;
constexpr uint32_t kBox64 = 8192;                  // one 64-row x 64-col bf16 box
constexpr int kKRing = 3, kVRing = 2;
constexpr int kOutThreads = 320;                   // 10 warps
constexpr int kEpiThreads = 256;

struct TcOutSmem {
    static constexpr uint32_t kStage = 4 * kBox64;     // 64 rows x 256 cols
    static constexpr uint32_t kK = 0;
    static constexpr uint32_t kV = kKRing * kStage;
    static constexpr uint32_t kY = kV + kVRing * kStage;   // 128 rows x 256 cols (4 boxes)
    static constexpr uint32_t kBytes = kY + 4 * kBox + 1024;
};

struct TcOutArgs {
    int heads, n, chunk, nchunks, rblocks, has_state_in, has_gate;
    const float *gn_weight, *gn_bias;
    float eps;
    unsigned *err;
};

__global__ void __launch_bounds__(kOutThreads, 1)
tc_output_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_s,
                 const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_out,
                 TcOutArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t kfull[kKRing], kempty[kKRing], vfull[kVRing], vempty[kVRing];
    __shared__ uint64_t s_full[2], p_full[2], s_free[2], q_full, q_copied, o_full, g_full;
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
    const int kend = min(kBlk * (r + 1), L);              // keys this row block sees
    const int nk = (kend + kKeyTile - 1) / kKeyTile;
    const bool has_s = (c > 0) || a.has_state_in;
    const int nsp = has_s ? 4 : 0;                        // S_prev parts in the K ring
    const int t0row = c0 + r * kBlk;                      // first token of the block
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    unsigned *err = a.err;
    uint8_t *ybuf = smem + TcOutSmem::kY;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kKRing; ++s) { mbar_init(&kfull[s], 1); mbar_init(&kempty[s], 1); }
        for (int s = 0; s < kVRing; ++s) { mbar_init(&vfull[s], 1); mbar_init(&vempty[s], 1); }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1); mbar_init(&p_full[s], kEpiThreads); mbar_init(&s_free[s], 1);
        }
        mbar_init(&q_full, 1);
        mbar_init(&q_copied, 1);
        mbar_init(&o_full, 1);
        mbar_init(&g_full, 1);
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
    const uint32_t tO = tmem, tQ = tmem + 256;
    auto tSP = [tmem](int t) -> uint32_t { return tmem + 384 + 64 * (t & 1); };

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v); tma_prefetch_desc(&tm_s);
            mbar_expect_tx(&q_full, 4 * kBox);
            for (int x = 0; x < 4; ++x)
                tma_load_3d(ybuf + x * kBox, &tm_q, &q_full, 64 * x, t0row, bh);
            const int srow = (bh * a.nchunks + c) * kD;
            int it = 0;
            bool ok = true;
            auto load_s = [&](int p) -> bool {
                const int s = it % kKRing;
                if (it >= kKRing && !mbar_wait(&kempty[s], ((it / kKRing) - 1) & 1, &abort_flag, err))
                    return false;
                uint8_t *dst = smem + TcOutSmem::kK + s * TcOutSmem::kStage;
                mbar_expect_tx(&kfull[s], TcOutSmem::kStage);
                for (int x = 0; x < 4; ++x)
                    tma_load_2d(dst + x * kBox64, &tm_s, &kfull[s], 64 * x, srow + 64 * p);
                ++it;
                return true;
            };
            for (int t = 0; ok && t < nk; ++t) {
                const int tk = c0 + t * kKeyTile;
                const int s = it % kKRing;
                if (it >= kKRing && !mbar_wait(&kempty[s], ((it / kKRing) - 1) & 1, &abort_flag, err)) { ok = false; break; }
                uint8_t *kd = smem + TcOutSmem::kK + s * TcOutSmem::kStage;
                mbar_expect_tx(&kfull[s], TcOutSmem::kStage);
                for (int x = 0; x < 4; ++x)
                    tma_load_3d(kd + x * kBox64, &tm_k, &kfull[s], 64 * x, tk, bh);
                ++it;
                if (t < nsp && !(ok = load_s(t))) break;
                const int vs = t % kVRing;
                if (t >= kVRing && !mbar_wait(&vempty[vs], ((t / kVRing) - 1) & 1, &abort_flag, err)) { ok = false; break; }
                uint8_t *vd = smem + TcOutSmem::kV + vs * TcOutSmem::kStage;
                mbar_expect_tx(&vfull[vs], TcOutSmem::kStage);
                for (int x = 0; x < 4; ++x)
                    tma_load_4d(vd + x * kBox64, &tm_v, &vfull[vs], 64 * x, h, tk, b);
            }
            for (int p = nk; ok && p < nsp; ++p) ok = load_s(p);
            // the gate tile reuses the Qt buffer once Qt sits in TMEM
            if (ok && a.has_gate && mbar_wait(&q_copied, 0, &abort_flag, err)) {
                tma_prefetch_desc(&tm_g);
                mbar_expect_tx(&g_full, 4 * kBox);
                for (int x = 0; x < 4; ++x)
                    tma_load_4d(ybuf + x * kBox, &tm_g, &g_full, 64 * x, h, t0row, b);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(128, kKeyTile, 0, 0);
            const uint32_t id_pv = idesc_bf16(128, 256, 0, 1);
            const uint32_t sK = smem_u32(smem + TcOutSmem::kK);
            const uint32_t sV = smem_u32(smem + TcOutSmem::kV);
            const uint32_t sY = smem_u32(ybuf);
            bool ok = mbar_wait(&q_full, 0, &abort_flag, err);
            if (ok) {
                tc_fence_after();
                // Qt (K-major, 128-byte swizzle) -> TMEM, 16 columns of K per copy
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks)
                    tmem_cp_128x256b(tQ + 8 * ks,
                                     smem_desc_sw128(sY + (ks / 4) * kBox + (ks % 4) * 32, 16, 1024));
                mma_commit(&q_copied);
            }
            bool o_written = false;
            int it = 0;
            auto qs_part = [&](int p) -> bool {
                const int s = it % kKRing;
                if (!mbar_wait(&kfull[s], (it / kKRing) & 1, &abort_flag, err)) return false;
                tc_fence_after();
                const uint32_t base = sK + s * TcOutSmem::kStage;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(tO, tQ + 8 * (4 * p + kk),
                                smem_desc_sw128(base + kk * 2048, kBox64, 1024), id_pv,
                                (o_written || kk > 0) ? 1u : 0u);
                o_written = true;
                mma_commit(&kempty[s]);
                ++it;
                return true;
            };
            for (int t = 0; ok && t <= nk; ++t) {
                if (t < nk) {
                    const int s = it % kKRing;
                    if (!mbar_wait(&kfull[s], (it / kKRing) & 1, &abort_flag, err)) { ok = false; break; }
                    if (t >= 2 && !mbar_wait(&s_free[t & 1], ((t - 2) >> 1) & 1, &abort_flag, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t base = sK + s * TcOutSmem::kStage;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_bf16_ts(tSP(t), tQ + 8 * ks,
                                    smem_desc_sw128(base + (ks / 4) * kBox64 + (ks % 4) * 32, 16, 1024),
                                    id_qk, ks > 0 ? 1u : 0u);
                    mma_commit(&kempty[s]);
                    mma_commit(&s_full[t & 1]);
                    ++it;
                    if (t < nsp && !(ok = qs_part(t))) break;
                }
                if (t >= 1) {
                    const int u = t - 1;
                    if (!mbar_wait(&p_full[u & 1], (u >> 1) & 1, &abort_flag, err)) { ok = false; break; }
                    if (!mbar_wait(&vfull[u % kVRing], (u / kVRing) & 1, &abort_flag, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t base = sV + (u % kVRing) * TcOutSmem::kStage;
#pragma unroll
                    for (int kk = 0; kk < kKeyTile / 16; ++kk)   // P halves at columns 0 and 32
                        mma_bf16_ts(tO, tSP(u) + 8 * kk + (kk >= 2 ? 16 : 0),
                                    smem_desc_sw128(base + kk * 2048, kBox64, 1024), id_pv,
                                    (o_written || kk > 0) ? 1u : 0u);
                    o_written = true;
                    mma_commit(&vempty[u % kVRing]);
                    mma_commit(&s_free[u & 1]);
                }
            }
            for (int p = nk; ok && p < nsp; ++p) ok = qs_part(p);
            mma_commit(&o_full);
        }
    } else {
        // two warpgroups: wg 0 owns S columns [0,32) and O columns [0,128),
        // wg 1 owns S columns [32,64) and O columns [128,256)
        const int wg = (warp - 2) / 4;
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;                         // row of the 128-row block
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const int lrow = r * kBlk + row;                        // row within the chunk
        const int t_row = t0row + row;
        bool ok = true;
        for (int t = 0; t < nk; ++t) {
            if (!warp_wait(&s_full[t & 1], (t >> 1) & 1, &abort_flag, err)) { ok = false; break; }
            tc_fence_after();
            uint32_t v[32];
            tmem_ld32(tSP(t) + lane_off + 32 * wg, v);
            tmem_wait_ld();
            const int j0 = t * kKeyTile + 32 * wg;              // first key of this half tile
            uint32_t w[16];
            if (j0 + 31 <= lrow) {                              // every key at or before the row
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float x0 = (lrow >= j0 + 2 * e) ? __uint_as_float(v[2 * e]) : 0.f;
                    const float x1 = (lrow >= j0 + 2 * e + 1) ? __uint_as_float(v[2 * e + 1]) : 0.f;
                    w[e] = pack_bf16x2(x0, x1);
                }
            }
            // P (bf16 pairs) goes to the first 16 columns of this warpgroup's own
            // 32 S columns, so it never overwrites S the other warpgroup still reads.
            tmem_st16(tSP(t) + lane_off + 32 * wg, w);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[t & 1]);
        }
        const bool go = ok && warp_wait(&o_full, 0, &abort_flag, err) &&
                        (!a.has_gate || warp_wait(&g_full, 0, &abort_flag, err));
        // The K ring is idle once O is complete: its first bytes hold the
        // two warpgroups' partial row sums.
        float (*red)[kBlk] = reinterpret_cast<float (*)[kBlk]>(smem + TcOutSmem::kK);
        float mean = 0.f, rstd = 1.f;
        if (go) tc_fence_after();
        if (a.has_gate) {
            // GroupNorm statistics over the row's 256 channels; each
            // warpgroup sums its half and the halves meet in shared memory.
            float sum = 0.f;
            if (go) {
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t v[32];
                    tmem_ld32(tO + lane_off + 128 * wg + 32 * cb, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) sum += __uint_as_float(v[e]);
                }
            }
            red[wg][row] = sum;
            named_barrier(1, kEpiThreads);
            mean = (red[0][row] + red[1][row]) * (1.f / kD);
            named_barrier(1, kEpiThreads);
            float sq = 0.f;
            if (go) {
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t v[32];
                    tmem_ld32(tO + lane_off + 128 * wg + 32 * cb, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float d = __uint_as_float(v[e]) - mean;
                        sq = fmaf(d, d, sq);
                    }
                }
            }
            red[wg][row] = sq;
            named_barrier(1, kEpiThreads);
            rstd = rsqrtf((red[0][row] + red[1][row]) * (1.f / kD) + a.eps);
        }
        if (go) {
            // This row's slot in the 128-byte-swizzled output/gate tile.
            uint8_t *yrow = ybuf + row * 128;
            const int sw = row & 7;
            const float *wv = a.gn_weight ? a.gn_weight + h * kD : nullptr;
            const float *bv = a.gn_bias ? a.gn_bias + h * kD : nullptr;
#pragma unroll 1
            for (int k4 = 0; k4 < 4; ++k4) {
                const int cb = 4 * wg + k4;                       // 32-column block
                uint32_t v[32];
                tmem_ld32(tO + lane_off + 32 * cb, v);
                tmem_wait_ld();
                uint8_t *box = yrow + (cb >> 1) * kBox;
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    uint4 *slot = reinterpret_cast<uint4 *>(box + ((((cb & 1) * 4 + q8) ^ sw) * 16));
                    float y[8];
                    if (a.has_gate) {
                        uint4 graw = *slot;
                        const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&graw);
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const float2 gg = __bfloat1622float2(g2[e2]);
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                const int e = 2 * e2 + hh;
                                const int ch = 32 * cb + 8 * q8 + e;
                                float yh = (__uint_as_float(v[8 * q8 + e]) - mean) * rstd;
                                if (wv) yh *= wv[ch];
                                if (bv) yh += bv[ch];
                                const float g = hh ? gg.y : gg.x;
                                y[e] = __fdividef(g, 1.f + __expf(-g)) * yh;
                            }
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) y[e] = __uint_as_float(v[8 * q8 + e]);
                    }
                    *slot = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                                       pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
                }
            }
            fence_async_shared();
        }
        // Both epilogue warpgroups reach this barrier on every path.
        named_barrier(1, kEpiThreads);
        if (wg == 0 && row == 0 && !abort_flag) {
            for (int x = 0; x < 4; ++x) tma_store_4d(&tm_out, ybuf + x * kBox, 64 * x, h, t0row, b);
            tma_store_commit();
            tma_store_wait_read();
        }
        (void)t_row;
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
    l.qt = 0;
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

    // tensor maps: 128-row boxes for the state pass, 64-row boxes for the output pass
    CUtensorMap tm_q128, tm_k128, tm_v128, tm_k64, tm_v64, tm_s64;
    {
        cuuint64_t dims[3] = {kD, (cuuint64_t)n, (cuuint64_t)BH};
        cuuint64_t str[2] = {kD * 2, (cuuint64_t)n * kD * 2};
        cuuint32_t box128[3] = {64, kBlk, 1};
        cuuint32_t box64[3] = {64, kKeyTile, 1};
        if (!make_map(&tm_k128, kt, 3, dims, str, box128) ||
            !make_map(&tm_k64, kt, 3, dims, str, box64) ||
            !make_map(&tm_q128, qt, 3, dims, str, box128))
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[4] = {kD, (cuuint64_t)H, (cuuint64_t)n, (cuuint64_t)B};
        cuuint64_t str[3] = {kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)n * H * kD * 2};
        cuuint32_t box128[4] = {64, 1, kBlk, 1};
        cuuint32_t box64[4] = {64, 1, kKeyTile, 1};
        if (!make_map(&tm_v128, a.v, 4, dims, str, box128) ||
            !make_map(&tm_v64, a.v, 4, dims, str, box64))
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {kD, (cuuint64_t)BH * nchunks * kD};
        cuuint64_t str[1] = {kD * 2};
        cuuint32_t box[2] = {64, 64};
        if (!make_map(&tm_s64, sp, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    // output and gate tiles: 128 tokens x 64 channels of one head
    CUtensorMap tm_out, tm_g;
    {
        cuuint64_t dims[4] = {kD, (cuuint64_t)H, (cuuint64_t)n, (cuuint64_t)B};
        cuuint64_t str[3] = {kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)n * H * kD * 2};
        cuuint32_t box[4] = {64, 1, kBlk, 1};
        if (!make_map(&tm_out, a.out, 4, dims, str, box)) return cudaErrorInvalidValue;
        if (!make_map(&tm_g, a.gate ? a.gate->g : a.out, 4, dims, str, box))
            return cudaErrorInvalidValue;
    }

    cudaError_t e;
    {
        TcPrepParams pp;
        for (int j = 0; j < kD / 2; ++j) pp.theta[j] = std::pow(10000.0, -2.0 * j / kD);
        for (int h = 0; h < kMaxHeads; ++h) pp.log2g[h] = hp.log2g[h];
        KernelTimer timer("tc_prep", stream);
        tc_prep_kernel<<<n, 256, 0, stream>>>((const __nv_bfloat16 *)a.q,
                                             (const __nv_bfloat16 *)a.k, pp, qt, kt, B, H, n, C,
                                             a.pos0, a.rotate);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const int smem = (int)TcStateSmem::kBytes;
        e = cudaFuncSetAttribute(tc_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        KernelTimer timer("tc_state", stream);
        tc_state_kernel<<<BH * 4, kTcThreads, smem, stream>>>(tm_k128, tm_v128, hp, a.state_in,
                                                             a.state_out, sp, H, n, C, nchunks,
                                                             err);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        TcOutArgs oa;
        oa.heads = H; oa.n = n; oa.chunk = C; oa.nchunks = nchunks; oa.rblocks = C / kBlk;
        oa.has_state_in = a.state_in != nullptr;
        oa.has_gate = a.gate != nullptr;
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
        tc_output_kernel<<<grid, kOutThreads, smem, stream>>>(tm_q128, tm_k64, tm_v64, tm_s64, tm_g,
                                                             tm_out, oa);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace retnet
