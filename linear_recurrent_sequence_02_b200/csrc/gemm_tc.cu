// Dense projection GEMM on the sm_100a tensor cores: Y = X W^T.
//
// Multi-scale retention replaces multi-head attention inside the RetNet
// block, with the swish gate and GroupNorm on its output (RetNet research
// summary, "Summary"); the layer around the retention operator projects the
// input X to Q, K, V and the gate G, and projects the gated output back with
// W_O.  Those projections are plain GEMMs: this kernel serves them.
//
//   X [M, K] bf16 row-major (K contiguous), W [N, K] bf16 row-major (the
//   [out_features, in_features] layout of a linear layer's weight), Y bf16
//   [M, N] with f32 accumulation.  The N columns may be split into up to
//   four outputs of `n_split` columns each (the fused Q/K/V/G projection
//   writes four dense [M, H*d] tensors).
//
// Persistent: one CTA per SM walks 128 x 256 output tiles in a grouped
// raster (16 row blocks at a time, so neighbouring CTAs share X and W tiles
// through L2).  Warp 0 streams 128 x 64 X and 256 x 64 W sub-tiles by TMA
// (128-byte swizzle) through a four-stage ring; warp 1 issues
// tcgen05.mma (M = 128, N = 256, K = 16, both operands K-major) into one of
// two TMEM accumulators (2 x 256 columns); warps 2-5 read the finished
// accumulator, round to bf16 and store, while the MMAs of the next tile run
// into the other accumulator.  Every wait is bounded (about 2 s); on
// timeout the CTA records kDevErrTimeout, lets its own loads and MMAs
// finish, frees its tensor memory and returns.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace retnet {

using namespace sm100;

namespace {

constexpr int kGemmM = 128;                 // rows of X per tile (TMEM lanes)
constexpr int kGemmN = 256;                 // columns of Y per tile (TMEM columns)
constexpr int kGemmK = 64;                  // K per stage: one 128-byte swizzle row
constexpr int kGemmStages = 4;
constexpr uint32_t kGemmABytes = kGemmM * kGemmK * 2;        // 16 KB
constexpr uint32_t kGemmBBytes = kGemmN * kGemmK * 2;        // 32 KB
constexpr uint32_t kGemmStage = kGemmABytes + kGemmBBytes;   // 48 KB
constexpr uint32_t kGemmSmem = kGemmStages * kGemmStage + 1024;
constexpr int kGemmThreads = 192;           // 6 warps
constexpr int kGemmGroup = 16;              // row blocks per raster group

struct GemmArgs {
    __nv_bfloat16 *out[4];
    long long m;                            // rows
    int n, k;                               // columns of Y, reduction length
    int n_split;                            // columns per output
    int tiles_m, tiles_n;
    unsigned *err;
    GemmFold fold;                          // outputs 0 and 1 as Qt, Kt (fold.on)
};

// Where row `grow` of a tile whose 256 columns go to output `which` at
// column c_in lands, and, for a folded output, the row's position and
// decay factor.
struct GemmRow {
    __nv_bfloat16 *dst;                     // the row's first column; null: not written
    bool fold;
    float scale;
    const float2 *cs;                       // 128 (cos, sin) pairs at the base position tb
    float delta;                            // t - tb, below kFoldTableStride
};

__device__ __forceinline__ GemmRow gemm_row(const GemmArgs &a, long long grow, int which,
                                            int c_in, bool live) {
    GemmRow r{nullptr, false, 1.f, nullptr, 0.f};
    if (!live) return r;
    // (a select chain, not a dynamic index, keeps a.out out of local memory)
    __nv_bfloat16 *base = which == 0   ? a.out[0]
                          : which == 1 ? a.out[1]
                          : which == 2 ? a.out[2]
                                       : a.out[3];
    if (a.fold.on && which < 2) {
        const long long b = grow / a.fold.n;
        const int t = (int)(grow - b * a.fold.n);
        const int h = c_in / 256;
        // debug build: the row of Qt / Kt lies inside the [B*H, n] operand
        if (!in_bounds((b * a.fold.heads + h) * (long long)a.fold.n + t, a.m * a.fold.heads, a.err,
                       kSiteGemm))
            return r;
        const float e = (float)(t % a.fold.fold + 1) * a.fold.log2g[h];
        r.scale = exp2f(which == 0 ? e : -e);
        r.cs = a.fold.table + (size_t)(t / kFoldTableStride) * 128;
        r.delta = (float)(t % kFoldTableStride);
        r.fold = true;
        r.dst = base + ((b * a.fold.heads + h) * (long long)a.fold.n + t) * 256;
    } else {
        r.dst = base + grow * a.n_split + c_in;
    }
    return r;
}

// log2 of theta_{j+1} / theta_j = 10000^(-1/128), and that ratio.
constexpr float kLog2ThetaStep = -0.10381025296523007f;
constexpr float kThetaStep = 0.930572040929699f;

// Stores columns [32 cb, 32 cb + 32) of the row (bf16), folded if asked:
// pair j = 16 cb + p turned by the angle (pos0 + t) theta_j and scaled.  The
// (cos, sin) of (pos0 + tb) theta_j come from the table (one row per 32
// positions, so the 32 rows of a warp read the same entries); those of
// (t - tb) theta_j, an angle below 32, from the fast sine and cosine, whose
// error there (a few 1e-6) is far below the bf16 rounding of the result.
__device__ __forceinline__ void gemm_store32(const GemmRow &r, int cb, const uint32_t (&v)[32]) {
    uint4 *d4 = reinterpret_cast<uint4 *>(r.dst + 32 * cb);
    if (r.fold) {
        float4 cs4[8];                      // pairs 16 cb .. 16 cb + 15, two per float4
        const float4 *src = reinterpret_cast<const float4 *>(r.cs + 16 * cb);
#pragma unroll
        for (int i = 0; i < 8; ++i) cs4[i] = src[i];
        float th = exp2f((float)(16 * cb) * kLog2ThetaStep);  // theta_{16 cb}
        uint32_t y[16];
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            float sd, cd;
            __sincosf(r.delta * th, &sd, &cd);
            th *= kThetaStep;
            const float cb0 = (p & 1) ? cs4[p / 2].z : cs4[p / 2].x;
            const float sb0 = (p & 1) ? cs4[p / 2].w : cs4[p / 2].y;
            const float c = (cb0 * cd - sb0 * sd) * r.scale;
            const float sn = (sb0 * cd + cb0 * sd) * r.scale;
            const float x0 = __uint_as_float(v[2 * p]), x1 = __uint_as_float(v[2 * p + 1]);
            y[p] = pack_bf16x2(x0 * c - x1 * sn, x0 * sn + x1 * c);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) d4[q] = make_uint4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
        return;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
        d4[q] = make_uint4(
            pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
            pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
            pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
            pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
}

__device__ __forceinline__ void gemm_tile(const GemmArgs &a, int t, int &mb, int &nb) {
    const int per_group = kGemmGroup * a.tiles_n;
    const int g = t / per_group, r = t % per_group;
    const int m0 = g * kGemmGroup;
    const int gm = min(kGemmGroup, a.tiles_m - m0);
    mb = m0 + r % gm;
    nb = r / gm;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_w, GemmArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[kGemmStages], empty[kGemmStages], acc_full[2], acc_free[2], drain;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    unsigned *err = a.err;
    const int tiles = a.tiles_m * a.tiles_n;
    const int ksteps = (a.k + kGemmK - 1) / kGemmK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&acc_full[x], 1);
            mbar_init(&acc_free[x], 128);
        }
        mbar_init(&drain, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    grid_dependency_wait();                         // X may come from the kernel before

    int pit = 0;                                    // producer: stages issued
    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
                int mb, nb;
                gemm_tile(a, t, mb, nb);
                for (int ks = 0; ks < ksteps; ++ks, ++pit) {
                    const int s = pit % kGemmStages;
                    if (pit >= kGemmStages &&
                        !mbar_wait(&empty[s], ((pit / kGemmStages) - 1) & 1, &abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t *ab = smem + s * kGemmStage;
                    mbar_expect_tx(&full[s], kGemmStage);
                    tma_load_2d(ab, &tm_x, &full[s], ks * kGemmK, mb * kGemmM);
                    tma_load_2d(ab + kGemmABytes, &tm_w, &full[s], ks * kGemmK, nb * kGemmN);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kGemmM, kGemmN, 0, 0);
            int it = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int buf = lt & 1;
                if (lt >= 2 && !mbar_wait(&acc_free[buf], ((lt - 2) >> 1) & 1, &abort_flag, err))
                    break;
                tc_fence_after();
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kGemmStages;
                    if (!mbar_wait(&full[s], (it / kGemmStages) & 1, &abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ab = smem_u32(smem + s * kGemmStage);
                    const uint32_t bb = ab + kGemmABytes;
#pragma unroll
                    for (int kk = 0; kk < kGemmK / 16; ++kk)
                        mma_bf16(tmem + kGemmN * buf, smem_desc_sw128(ab + kk * 32, 16, 1024),
                                 smem_desc_sw128(bb + kk * 32, 16, 1024), idesc,
                                 (ks > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&empty[s]);
                }
                if (ok) mma_commit(&acc_full[buf]);
            }
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 = rows of the tile
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            if (!warp_wait(&acc_full[buf], (lt >> 1) & 1, &abort_flag, err)) break;
            tc_fence_after();
            int mb, nb;
            gemm_tile(a, t, mb, nb);
            const long long grow = (long long)mb * kGemmM + row;
            const int col0 = nb * kGemmN;
            const int which = col0 / a.n_split;
            const int c_in = col0 % a.n_split;
            const bool live = grow < a.m && in_bounds(which, 4, err, kSiteGemm);
            const GemmRow r = gemm_row(a, grow, which, c_in, live);
#pragma unroll 1
            for (int cb = 0; cb < kGemmN / 32; ++cb) {
                uint32_t v[32];
                tmem_ld32(tmem + kGemmN * buf + lane_off + 32 * cb, v);
                tmem_wait_ld();
                if (cb == kGemmN / 32 - 1) {             // accumulator fully read
                    tc_fence_before();
                    mbar_arrive(&acc_free[buf]);
                }
                if (live && r.dst) gemm_store32(r, cb, v);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    // Every role has finished, so abort_flag is final.  After an abort, wait
    // (bounded) for the loads still in flight (at most the last kGemmStages
    // issued) and for the MMAs before freeing shared and tensor memory.
    if (abort_flag && warp == 0 && lane == 0)
        for (int j = max(0, pit - kGemmStages); j < pit; ++j)
            mbar_drain(&full[j % kGemmStages], (j / kGemmStages) & 1, err);
    if (warp == 1) {
        if (abort_flag && lane == 0) {
            mma_commit(&drain);
            mbar_drain(&drain, 0, err);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Paired variant: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05 cta_group::2 (M = 256).  CTA k loads rows [128k, 128k+128) of the
// tile's X block and rows [128k, 128k+128) of its W block (half of N), so a
// 64-wide K step costs each CTA 32 KB of loads instead of 48 KB; each CTA
// keeps its 128 rows x 256 columns of the product in its own TMEM (two
// accumulators).  The leader (rank 0) issues the MMAs; both CTAs' loads
// count on the leader's full barrier, and its commits arrive on both CTAs'
// empty and acc_full barriers.  On an abort the leader settles and drains
// the loads of both CTAs before the pair's last cluster barrier.
// The ring has three 64 KB stages of two K steps each: fewer, larger stages
// keep more bytes in flight per stage round trip (three 64 KB stages stream
// about 1.6x what six 32 KB stages do per CTA, measured on B200), and the
// layer step went 212.7 -> 206.5 us (200M shape), 478 -> 453 us (3B-like).
constexpr int kPairM = 256;                // rows per pair tile
constexpr int kPairStages = 3;
constexpr int kPairKSub = 2;               // 64-wide K steps per stage
constexpr uint32_t kPairHalf = kGemmM * kGemmK * 2;          // 16 KB: 128 rows x 64
constexpr uint32_t kPairStage = 2 * kPairKSub * kPairHalf;   // 64 KB per CTA: X, then W
constexpr uint32_t kPairSmem = kPairStages * kPairStage + 1024;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
gemm_bf16_tn_pair_kernel(const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_w, GemmArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[kPairStages], empty[kPairStages], acc_full[2], acc_free[2], drain;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag, issued;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    unsigned *err = a.err;
    const int tiles = a.tiles_m * a.tiles_n;        // tiles_m counts 256-row blocks here
    const int ksteps = (a.k + kGemmK - 1) / kGemmK;
    const int cluster = blockIdx.x / 2, nclusters = gridDim.x / 2;
    const uint32_t peer_abort = mapa_shared(smem_u32(&abort_flag), rank ^ 1u);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&acc_full[x], 1);
            mbar_init(&acc_free[x], 2 * 128);
        }
        mbar_init(&drain, 1);
        abort_flag = 0;
        issued = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, 512);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    grid_dependency_wait();
    auto abort_both = [&]() {
        abort_flag = 1;
        st_cluster_u32(peer_abort, 1u);
    };

    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            int it = 0;
            for (int t = cluster; ok && t < tiles; t += nclusters) {
                int mb, nb;
                gemm_tile(a, t, mb, nb);
                for (int ks = 0; ks < ksteps; ks += kPairKSub) {
                    const int s = it % kPairStages;
                    if (it >= kPairStages &&
                        !mbar_wait(&empty[s], ((it / kPairStages) - 1) & 1, &abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    uint8_t *ab = smem + s * kPairStage;
                    const uint32_t lbar = mapa_shared(smem_u32(&full[s]), 0);
                    if (leader) mbar_expect_tx(&full[s], 2 * kPairStage);
                    // a K step past the end reads zeros, which add nothing
                    for (int j = 0; j < kPairKSub; ++j) {
                        tma_load_2d_pair(ab + j * kPairHalf, &tm_x, lbar, (ks + j) * kGemmK,
                                         mb * kPairM + kGemmM * (int)rank);
                        tma_load_2d_pair(ab + (kPairKSub + j) * kPairHalf, &tm_w, lbar,
                                         (ks + j) * kGemmK, nb * kGemmN + kGemmM * (int)rank);
                    }
                    ++it;
                    *(volatile int *)&issued = it;
                }
            }
            if (!ok) abort_both();
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            const uint32_t idesc = idesc_bf16(kPairM, kGemmN, 0, 0);
            int it = 0, lt = 0;
            bool ok = true;
            for (int t = cluster; ok && t < tiles; t += nclusters, ++lt) {
                const int buf = lt & 1;
                if (lt >= 2 && !mbar_wait(&acc_free[buf], ((lt - 2) >> 1) & 1, &abort_flag, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int ks = 0; ks < ksteps; ks += kPairKSub, ++it) {
                    const int s = it % kPairStages;
                    if (!mbar_wait(&full[s], (it / kPairStages) & 1, &abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ab = smem_u32(smem + s * kPairStage);
#pragma unroll
                    for (int j = 0; j < kPairKSub; ++j) {
                        const uint32_t xa = ab + j * kPairHalf;
                        const uint32_t wb = ab + (kPairKSub + j) * kPairHalf;
#pragma unroll
                        for (int kk = 0; kk < kGemmK / 16; ++kk)
                            mma_bf16_pair(tmem + kGemmN * buf, smem_desc_sw128(xa + kk * 32, 16, 1024),
                                          smem_desc_sw128(wb + kk * 32, 16, 1024), idesc,
                                          (ks + j > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[s], 3);
                }
                if (ok) mma_commit_pair(&acc_full[buf], 3);
            }
            if (!ok) abort_both();
        }
    } else {
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        int lt = 0;
        bool ok = true;
        for (int t = cluster; t < tiles; t += nclusters, ++lt) {
            const int buf = lt & 1;
            if (!warp_wait(&acc_full[buf], (lt >> 1) & 1, &abort_flag, err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            int mb, nb;
            gemm_tile(a, t, mb, nb);
            const long long grow = (long long)mb * kPairM + kGemmM * (int)rank + row;
            const int col0 = nb * kGemmN;
            const int which = col0 / a.n_split;
            const int c_in = col0 % a.n_split;
            const bool live = grow < a.m && in_bounds(which, 4, err, kSiteGemm);
            const GemmRow r = gemm_row(a, grow, which, c_in, live);
            const uint32_t l_free = mapa_shared(smem_u32(&acc_free[buf]), 0);
#pragma unroll 1
            for (int cb = 0; cb < kGemmN / 32; ++cb) {
                uint32_t v[32];
                tmem_ld32(tmem + kGemmN * buf + lane_off + 32 * cb, v);
                tmem_wait_ld();
                if (cb == kGemmN / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive_cluster(l_free);
                }
                if (live && r.dst) gemm_store32(r, cb, v);
            }
        }
        if (!ok && lane == 0) abort_both();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    // After an abort: the leader settles the loads only one CTA issued and
    // drains the last stages of both; then the MMAs.
    if (abort_flag && leader && warp == 0 && lane == 0) {
        const int own = issued;
        const int peer = (int)ld_cluster_u32(mapa_shared(smem_u32(&issued), 1));
        const int last = max(own, peer);
        for (int j = max(0, last - kPairStages); j < last; ++j) {
            uint64_t *bar = &full[j % kPairStages];
            if (j >= own) mbar_expect_tx(bar, kPairStage);
            else if (j >= peer) mbar_complete_tx(bar, kPairStage);
            mbar_drain(bar, (j / kPairStages) & 1, err);
        }
    }
    if (abort_flag && leader && warp == 1 && lane == 0) {
        mma_commit_pair(&drain, 1);
        mbar_drain(&drain, 0, err);
    }
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

}  // namespace

bool gemm_shape_ok(long long m, int n, int k, int n_split) {
    if (m < 0 || n <= 0 || k <= 0 || k % kGemmK != 0 || n % kGemmN != 0) return false;
    if (n_split <= 0 || n_split % kGemmN != 0 || n % n_split != 0 || n / n_split > 4) return false;
    const long long tiles = (m + kGemmM - 1) / kGemmM * (long long)(n / kGemmN);
    return tiles < (1LL << 31);
}

cudaError_t launch_gemm_bf16(const void *x, const void *w, void *const *outs, long long m, int n,
                             int k, int n_split, cudaStream_t stream, const char *timer_name,
                             const GemmFold *fold) {
    if (m == 0) return cudaSuccess;
    CUtensorMap tm_x, tm_w;
    {
        cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)m};
        cuuint64_t str[1] = {(cuuint64_t)k * 2};
        cuuint32_t box[2] = {kGemmK, kGemmM};
        if (!make_tensor_map_bf16(&tm_x, x, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)n};
        cuuint64_t str[1] = {(cuuint64_t)k * 2};
        cuuint32_t box[2] = {kGemmK, kGemmN};
        if (!make_tensor_map_bf16(&tm_w, w, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    GemmArgs a;
    for (int i = 0; i < 4; ++i) a.out[i] = i < n / n_split ? (__nv_bfloat16 *)outs[i] : nullptr;
    a.m = m;
    a.n = n;
    a.k = k;
    a.n_split = n_split;
    a.tiles_n = n / kGemmN;
    if (fold) a.fold = *fold;
    else a.fold.on = 0;
    a.err = device_error_word();
    if (!a.err) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e;
    // CTA pairs (256-row tiles) unless the rows fill no more than one
    // 128-row block per tile column.  (Measured on B200 at the layer shapes,
    // 16384 x 4096 x 1024 and 16384 x 1024 x 1024: 114 and 35 us against
    // 124 and 42 us for single CTAs; no shape measured slower.)
    if (m > kGemmM) {
        a.tiles_m = (int)((m + kPairM - 1) / kPairM);
        CUtensorMap tm_wh;                          // W in halves of 128 rows
        {
            cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)n};
            cuuint64_t str[1] = {(cuuint64_t)k * 2};
            cuuint32_t box[2] = {kGemmK, kGemmM};
            if (!make_tensor_map_bf16(&tm_wh, w, 2, dims, str, box)) return cudaErrorInvalidValue;
        }
        e = cudaFuncSetAttribute(gemm_bf16_tn_pair_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t qc = {};
        qc.gridDim = dim3(2 * (unsigned)std::max(1, sms / 2));
        qc.blockDim = dim3(kGemmThreads);
        qc.dynamicSmemBytes = kPairSmem;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, gemm_bf16_tn_pair_kernel, &qc) !=
                cudaSuccess ||
            clusters < 1)
            clusters = std::max(1, sms / 2);
        const long long tiles = (long long)a.tiles_m * a.tiles_n;
        clusters = (int)std::min<long long>(tiles, clusters);
        KernelTimer timer(timer_name, stream);
        e = launch_overlapped(gemm_bf16_tn_pair_kernel, dim3(2 * clusters), dim3(kGemmThreads),
                              kPairSmem, stream, tm_x, tm_wh, a);
        count_launch();
        return e;
    }
    a.tiles_m = (int)((m + kGemmM - 1) / kGemmM);
    e = cudaFuncSetAttribute(gemm_bf16_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemmSmem);
    if (e != cudaSuccess) return e;
    const long long tiles = (long long)a.tiles_m * a.tiles_n;
    const unsigned grid = (unsigned)std::min<long long>(tiles, sms);
    KernelTimer timer(timer_name, stream);
    e = launch_overlapped(gemm_bf16_tn_kernel, dim3(grid), dim3(kGemmThreads), kGemmSmem, stream,
                          tm_x, tm_w, a);
    count_launch();
    return e;
}

}  // namespace retnet
