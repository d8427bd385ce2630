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
//   tc_state   per (sequence, head, 128 x DVC block of S, DVC = 64, 128 or
//              256): walks the chunks, accumulating each chunk's Kt^T V in
//              TMEM, carrying S <- g^L (S + Kt^T V) in registers, and writing
//              S_prev of every chunk (bf16) and the final state (f32)
//   tc_output  persistent, work items (sequence, head, chunk, 128-row
//              block): S = Qt Kt^T in TMEM, causal mask in registers, P
//              (bf16) to shared memory, O += P V; then O += Qt S_prev; the
//              epilogue writes O, or swish(G) * GroupNorm(O) when a gate is
//              given.
// Roles inside a CTA: warp 0 issues TMA loads, warp 1 allocates TMEM and
// issues tcgen05.mma, the remaining warps move data between TMEM, registers
// and memory.  Every mbarrier wait is bounded (about 2 s); on timeout the
// CTA records kDevErrTimeout and unwinds.
#include <algorithm>
#include <cmath>

#include "kernels.h"
#include "sm100.cuh"

namespace retnet {

using namespace sm100;

constexpr int kD = 256;            // head dimension served here (dk = dv = 256)
constexpr int kBlk = 128;          // rows per tile
constexpr uint32_t kBox = 16384;   // one 128-row x 64-col bf16 box (128-B swizzle)

struct TcHeadParams {
    float log2g[kMaxHeads];        // log2(gamma_h)
    float decay_chunk[kMaxHeads];  // gamma_h^chunk
    float decay_last[kMaxHeads];   // gamma_h^(length of the last chunk)
};

// ------------------------------------------------------------------ prep
// Rotation and decay fold of k (and of q when write_q) into Kt (Qt), laid
// out [b*H + h][t][256].  One warp per token t (grid-stride): every row of
// that token, all B*H (sequence, head) pairs, rotates by the same angles, so
// the lane's four (cos, sin) pairs, rotation pairs j = 4 lane .. 4 lane + 3
// of (pos0 + t) * theta_j, are formed once in registers and serve all of
// them.  A row of 256 elements is one 16-byte part per lane (coalesced);
// rows go four at a time with all their loads issued before any arithmetic,
// the first four before the angles are formed.  The fold exponent
// (t mod fold) + 1 is also per token; only the head's log2(gamma) varies by row.
struct TcPrepParams {
    double theta[kD / 2];          // 10000^(-2j/256), formed on the host
    float log2g[kMaxHeads];        // log2(gamma_h)
};

__global__ void __launch_bounds__(256)
tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
               TcPrepParams pp, __nv_bfloat16 *__restrict__ qt, __nv_bfloat16 *__restrict__ kt,
               int batch, int heads, int n, int fold, long long pos0, int rotate,
               int write_q, unsigned *err) {
    constexpr int kRound = 4;                       // rows per round
    const long long elems = (long long)batch * n * heads * kD;   // of q, k, Qt and Kt
    const int lane = threadIdx.x % 32;
    const int warp0 = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) / 32);
    const int nwarps = (int)(gridDim.x * (long long)blockDim.x / 32);
    const int rows = batch * heads;                 // row r = b * heads + h
    const long long row_in = (long long)heads * kD;            // q/k: one token of all heads
    const long long seq_in = (long long)n * row_in;            // q/k: one sequence
    const long long row_out = (long long)n * kD;               // Qt/Kt: one (sequence, head)
    double th[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) th[p] = pp.theta[4 * lane + p];
    grid_dependency_wait();                         // q, k may come from the kernel before

    uint4 rq[kRound] = {}, rk[kRound] = {};
    int rb[kRound], rh[kRound];
    for (int t = warp0; t < n; t += nwarps) {
        int b = 0, h = 0;                           // (sequence, head) of the round's first row
        auto load_round = [&](int r0) {
            int bb = b, hh = h;
#pragma unroll
            for (int x = 0; x < kRound; ++x) {
                rb[x] = bb; rh[x] = hh;
                if (r0 + x < rows) {
                    const long long src = bb * seq_in + t * row_in + hh * kD + 8 * lane;
                    if (in_bounds(src + 7, elems, err, kSitePrep)) {
                        if (write_q) rq[x] = *reinterpret_cast<const uint4 *>(q + src);
                        rk[x] = *reinterpret_cast<const uint4 *>(k + src);
                    }
                }
                if (++hh == heads) { hh = 0; ++bb; }
            }
            b = bb; h = hh;
        };
        load_round(0);
        float2 cs[4];
#pragma unroll
        for (int p = 0; p < 4; ++p)
            cs[p] = rotate ? rotation_cs(pos0 + t, th[p]) : make_float2(1.f, 0.f);
        const float ef = (float)(t % fold + 1);
        const long long dst0 = (long long)t * kD + 8 * lane;
        for (int r0 = 0; r0 < rows; r0 += kRound) {
            if (r0 > 0) load_round(r0);
#pragma unroll
            for (int x = 0; x < kRound; ++x) {
                const int r = r0 + x;
                if (r >= rows) continue;
                const float e = ef * pp.log2g[rh[x]];
                const float sq = exp2f(e), sk = exp2f(-e);
                const __nv_bfloat162 *hq = reinterpret_cast<const __nv_bfloat162 *>(&rq[x]);
                const __nv_bfloat162 *hk = reinterpret_cast<const __nv_bfloat162 *>(&rk[x]);
                float oq[8], ok[8];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float cq = cs[p].x * sq, sq2 = cs[p].y * sq;
                    const float ck = cs[p].x * sk, sk2 = cs[p].y * sk;
                    const float2 xq = __bfloat1622float2(hq[p]);
                    const float2 xk = __bfloat1622float2(hk[p]);
                    oq[2 * p] = xq.x * cq - xq.y * sq2;
                    oq[2 * p + 1] = xq.x * sq2 + xq.y * cq;
                    ok[2 * p] = xk.x * ck - xk.y * sk2;
                    ok[2 * p + 1] = xk.x * sk2 + xk.y * ck;
                }
                const long long dst = r * row_out + dst0;
                if (!in_bounds(dst + 7, elems, err, kSitePrep)) continue;
                if (write_q) store8(qt + dst, oq);
                store8(kt + dst, ok);
            }
        }
    }
}

// ------------------------------------------------------------------ state pass
// One CTA per (sequence, head, 128 x DVC block of S): the d_k half mh and
// d_v columns [DVC nv, DVC nv + DVC).  DVC is 64, 128 or 256 (eight, four
// or two CTAs per sequence-head), chosen per shape by tc_state_columns.
// Warp 0 streams Kt and V sub-tiles of kTok tokens (128; 64 at DVC = 256,
// so that four stages fit) through a TMA ring;
// warp 1 accumulates U_c = Kt_c^T V_c of every chunk into one of two TMEM
// buffers (M = d_k half, N = DVC, both operands MN-major); the state
// warpgroups (one per 128 of the DVC columns) keep the running state row in
// registers, S <- g^L (S + U_c), hand the buffer back as soon as it is
// read, and write S_prev of the next chunk (bf16) or the final state (f32).
// The tensor core never waits for the state update.
template <int DVC>
struct TcStateSmem {
    static constexpr int kTok = DVC == 256 ? 64 : 128;         // tokens per stage
    static constexpr uint32_t kTokBox = kTok * 128;            // kTok rows x 64 channels
    static constexpr int kVBoxes = DVC / 64;
    static constexpr uint32_t kStage = (2 + kVBoxes) * kTokBox; // Kt kTok x 128 + V kTok x DVC
    static constexpr int kStages = DVC == 128 ? 3 : 4;
    static constexpr uint32_t kBytes = kStages * kStage + 1024;
    static constexpr int kGroups = DVC > 128 ? DVC / 128 : 1;  // state warpgroups
    static constexpr int kCols = DVC / kGroups;                 // d_v columns per state thread
    static constexpr int kThreads = 64 + 128 * kGroups;
    static constexpr uint32_t kBufCols = DVC < 128 ? 128 : DVC; // TMEM columns per U buffer
    static constexpr uint32_t kTmemCols = 2 * kBufCols;
};

__device__ __forceinline__ void store_bf16_row(__nv_bfloat16 *dst, const float *v, int count) {
    for (int i = 0; i < count; i += 8)
        *reinterpret_cast<uint4 *>(dst + i) =
            make_uint4(sm100::pack_bf16x2(v[i], v[i + 1]), sm100::pack_bf16x2(v[i + 2], v[i + 3]),
                       sm100::pack_bf16x2(v[i + 4], v[i + 5]), sm100::pack_bf16x2(v[i + 6], v[i + 7]));
}

#ifdef RETNET_TEST_HOOKS
// Test hook (debug build only): when set, the state pass's first CTA never
// issues its first TMA load, so its MMA warp's wait runs out and the CTA
// takes the timeout path.  Set by retnet_test_set_hooks.
static __device__ int g_hook_skip_first_load = 0;
#endif

template <int DVC>
__global__ void __launch_bounds__(TcStateSmem<DVC>::kThreads, 1)
tc_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                TcHeadParams hp, const float *__restrict__ state_in, float *__restrict__ state_out,
                __nv_bfloat16 *__restrict__ s_prev, int heads, int n, int chunk, int nchunks,
                unsigned *err) {
    using Smem = TcStateSmem<DVC>;
    constexpr int S = Smem::kStages;
    constexpr int kParts = 2 * (kD / DVC);             // CTAs per sequence-head
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[S], empty[S], acc_full[2], acc_free[2], drain;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.x / kParts;
    const long long nbh = gridDim.x / kParts;               // sequence-heads of the launch
    const int part = blockIdx.x % kParts;
    const int mh = part / (kD / DVC), nv = part % (kD / DVC);   // d_k half, d_v block
    const int b = bh / heads, h = bh % heads;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&acc_full[x], 1);
            mbar_init(&acc_free[x], 128 * Smem::kGroups);
        }
        mbar_init(&drain, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, Smem::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    grid_dependency_wait();                             // Kt from the prep kernel

    int it = 0, skipped = -1;              // producer: ring items issued, one never issued
    if (warp == 0) {
        if (lane == 0) {
            for (int c = 0; c < nchunks && !abort_flag; ++c) {
                const int c0 = c * chunk;
                const int L = min(chunk, n - c0);
                for (int st = 0; st * Smem::kTok < L; ++st, ++it) {
                    const int s = it % S;
                    if (it >= S && !mbar_wait(&empty[s], ((it / S) - 1) & 1, &abort_flag, err))
                        break;
#ifdef RETNET_TEST_HOOKS
                    if (it == 0 && blockIdx.x == 0 &&
                        *(volatile int *)&g_hook_skip_first_load) {
                        skipped = 0;                       // never issued: its wait runs out
                        continue;
                    }
#endif
                    uint8_t *kb = smem + s * Smem::kStage;
                    uint8_t *vb = kb + 2 * Smem::kTokBox;
                    mbar_expect_tx(&full[s], Smem::kStage);
                    const int t0 = c0 + st * Smem::kTok;
                    for (int x = 0; x < 2; ++x)
                        tma_load_3d(kb + x * Smem::kTokBox, &tm_k, &full[s], 128 * mh + 64 * x, t0,
                                    bh);
                    for (int x = 0; x < Smem::kVBoxes; ++x)
                        tma_load_4d(vb + x * Smem::kTokBox, &tm_v, &full[s], DVC * nv + 64 * x, h,
                                    t0, b);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, DVC, 1, 1);
            int it = 0;
            bool ok = true;
            for (int c = 0; ok && c < nchunks; ++c) {
                const int buf = c & 1;
                if (c >= 2 && !mbar_wait(&acc_free[buf], ((c - 2) >> 1) & 1, &abort_flag, err)) break;
                tc_fence_after();
                const int L = min(chunk, n - c * chunk);
                uint32_t accumulate = 0;
                for (int st = 0; st * Smem::kTok < L; ++st, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(&full[s], (it / S) & 1, &abort_flag, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t kb = smem_u32(smem + s * Smem::kStage);
                    const uint32_t vb = kb + 2 * Smem::kTokBox;
#pragma unroll
                    for (int ks = 0; ks < Smem::kTok / 16; ++ks) {
                        // A = Kt^T (M = d_k, K = tokens), B = V (N = d_v, K = tokens):
                        // both MN-major, 64 channels per box (the leading
                        // byte offset); 16 tokens = two 8-row atoms = 2048 B.
                        const uint64_t ad = smem_desc_sw128(kb + ks * 2048, Smem::kTokBox, 1024);
                        const uint64_t bd = smem_desc_sw128(vb + ks * 2048, Smem::kTokBox, 1024);
                        mma_bf16(tmem + Smem::kBufCols * buf, ad, bd, idesc, accumulate);
                        accumulate = 1;
                    }
                    mma_commit(&empty[s]);
                }
                if (ok) mma_commit(&acc_full[buf]);
            }
        }
    } else {
        // state warpgroups: warp w owns TMEM lanes 32*(w%4) .. +31 = rows of
        // the d_k half; warpgroup wg owns kCols of the CTA's DVC columns
        constexpr int kCols = Smem::kCols;
        const int wg = (warp - 2) / 4;
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;
        const int krow = 128 * mh + row;                     // row of S
        const int col0 = DVC * nv + kCols * wg;              // first column of S
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const size_t sbase = ((size_t)bh * kD + krow) * kD + col0;
        const long long state_elems = nbh * kD * kD;
        const long long sprev_elems = nbh * nchunks * kD * kD;
        float st[kCols];
        if (state_in && in_bounds((long long)sbase + kCols - 1, state_elems, err, kSiteState)) {
            const float4 *src = reinterpret_cast<const float4 *>(state_in + sbase);
#pragma unroll
            for (int v4 = 0; v4 < kCols / 4; ++v4) {
                const float4 f = src[v4];
                st[4 * v4] = f.x; st[4 * v4 + 1] = f.y; st[4 * v4 + 2] = f.z; st[4 * v4 + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < kCols; ++e) st[e] = 0.f;
        }
        {
            const size_t o0 = ((size_t)bh * nchunks * kD + krow) * kD + col0;
            if (in_bounds((long long)o0 + kCols - 1, sprev_elems, err, kSiteState))
                store_bf16_row(s_prev + o0, st, kCols);
        }
        for (int c = 0; c < nchunks; ++c) {
            const int buf = c & 1;
            if (!warp_wait(&acc_full[buf], (c >> 1) & 1, &abort_flag, err)) break;
            tc_fence_after();
            const bool last = (c == nchunks - 1);
            const float decay = last ? hp.decay_last[h] : hp.decay_chunk[h];
#pragma unroll
            for (int cb = 0; cb < kCols / 32; ++cb) {
                uint32_t v[32];
                tmem_ld32(tmem + Smem::kBufCols * buf + lane_off + kCols * wg + 32 * cb, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    st[32 * cb + e] = decay * (st[32 * cb + e] + __uint_as_float(v[e]));
            }
            tc_fence_before();
            mbar_arrive(&acc_free[buf]);                     // buffer free for chunk c + 2
            if (!last) {
                const size_t o1 = (((size_t)bh * nchunks + c + 1) * kD + krow) * kD + col0;
                if (in_bounds((long long)o1 + kCols - 1, sprev_elems, err, kSiteState))
                    store_bf16_row(s_prev + o1, st, kCols);
            } else if (state_out && in_bounds((long long)sbase + kCols - 1, state_elems, err, kSiteState)) {
                float4 *o = reinterpret_cast<float4 *>(state_out + sbase);
#pragma unroll
                for (int v4 = 0; v4 < kCols / 4; ++v4)
                    o[v4] = make_float4(st[4 * v4], st[4 * v4 + 1], st[4 * v4 + 2], st[4 * v4 + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    // Every role has finished, so abort_flag is final.  After an abort, wait
    // (bounded) for what this CTA still has in flight: the TMA loads (at most
    // the last S issued) before shared memory goes away, the MMAs before
    // tensor memory is freed.
    if (abort_flag && warp == 0 && lane == 0)
        for (int j = max(0, it - S); j < it; ++j)
            if (j != skipped) mbar_drain(&full[j % S], (j / S) & 1, err);
    if (warp == 1) {
        if (abort_flag && lane == 0) {
            mma_commit(&drain);
            mbar_drain(&drain, 0, err);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, Smem::kTmemCols);
    }
}

// ------------------------------------------------------------------ output pass
// Persistent: one CTA per SM walks work items (sequence, head, chunk,
// 128-row block), so the loads and the first
// QK^T of the next item overlap the epilogue of the current one.
// TMEM (512 columns, allocated once): O [0,256) f32; Qt [256,384) bf16 pairs
// (A operand); S [384,512): S = Qt Kt^T for a 128-key tile in f32 (N = 128
// keeps tcgen05.mma at its full rate).  The mask pass reads S, releases the
// buffer at once (so QK^T of the next tile overlaps the rest of the pass and
// P V) and writes P (bf16) to a 32 KB shared-memory tile, the A operand of P V.
//
// Shared memory: a ring of three 64 KB slots carrying every tile in the
// order it is consumed; per item
//     Qt, Kt(0), then for t = 0..nk-1: Kt(t+1), S_prev half t (t < 2), V(t),
//     the remaining S_prev half, and the gate/output tile.
// Qt is moved into TMEM by tcgen05.cp; the gate/output tile receives G by
// TMA (or is merely reserved), is overwritten in place by the output rows,
// leaves by TMA store and is released by the storing thread.
// Warps: 0 TMA, 1 MMA (+ TMEM allocation), 2-9 two warpgroups: for each
// tile wg w masks and converts S columns [64w, 64w+64); in the epilogue wg w
// owns O columns [128w, 128w+128).
// MMA order per item: copy Qt, QK^T(0), then for each tile t: QK^T(t+1),
// Qt S_prev half t (t < 2), P V(t).
constexpr int kKeyTile = 128;
constexpr int kSlots = 3;
constexpr uint32_t kSlot = 4 * kBox;               // 64 KB: 128 rows x 256 cols
constexpr int kOutThreads = 320;                   // 10 warps
constexpr int kEpiThreads = 256;

struct TcOutSmem {
    static constexpr uint32_t kP = kSlots * kSlot;     // P tile; the epilogue's row sums
    static constexpr uint32_t kBytes = kP + 2 * kBox + 1024;
};

struct TcOutArgs {
    int heads, n, chunk, nchunks, rblocks, has_state_in, has_gate, items;
    const float *gn_weight, *gn_bias;
    float eps;
    unsigned *err;
    // Parallel form: the whole sequence is one "chunk" with Qt, Kt folded per
    // 128-token block, so key tile t of row block r still needs the factor
    // g^(128 (r - t)), applied in the mask pass.
    int parallel;
    float log2g[kMaxHeads];
    // Paired output pass only: fold_q = 1 loads raw q and applies the rotation
    // and the decay fold in shared memory (the prep pass then writes only Kt);
    // fold = the decay fold's block length (the chunk, or 128 in the parallel
    // form); theta_j = 10000^(-2j/256); pos0 and rotate as for the call.
    int fold_q, fold, rotate;
    long long pos0;
    double theta[kD / 2];
};

struct TcItem {
    int r, c, bh, b, h, c0, nk, nsp, t0row;
    bool valid;
};

// Work item w: group g = w / rblocks is one (sequence, head, chunk); its
// row blocks sit at consecutive w, so CTAs working side by side share that
// chunk's Kt, V and S_prev tiles through L2.  The row block is rotated by
// the group index, r = (w + g) mod rblocks, so a CTA striding by the grid
// size still meets a mix of heavy and light blocks.
// With kBalance (the parallel form, one chunk per sequence-head, whose row
// block r costs r + 1 key tiles): item k of the decreasing-cost order is row
// block R - 1 - k / BH of sequence-head k mod BH, and the CTAs take these k
// in rounds of gridDim.x, forward in even rounds and backward in odd ones,
// so every CTA's total stays close to the average.
template <bool kBalance>
__device__ __forceinline__ TcItem tc_item(const TcOutArgs &a, int w) {
    TcItem it;
    int g;
    if (kBalance) {
        const int P = gridDim.x;
        const int j = w / P, x = w - j * P;
        const int m = min(P, a.items - j * P);
        const int k = j * P + ((j & 1) ? m - 1 - x : x);
        const int nbh = a.items / a.rblocks;
        g = k % nbh;                                   // one chunk: group = sequence-head
        it.r = a.rblocks - 1 - k / nbh;
    } else {
        g = w / a.rblocks;
        it.r = (w + g) % a.rblocks;
    }
    it.c = g % a.nchunks;
    it.bh = g / a.nchunks;
    it.b = it.bh / a.heads;
    it.h = it.bh % a.heads;
    it.c0 = it.c * a.chunk;
    const int L = min(a.chunk, a.n - it.c0);
    it.valid = it.r * kBlk < L;                        // false past a short last chunk
    const int kend = min(kBlk * (it.r + 1), L);        // keys this row block sees
    it.nk = (kend + kKeyTile - 1) / kKeyTile;
    it.nsp = (it.c > 0 || a.has_state_in) ? 2 : 0;     // S_prev halves (128 d_k rows each)
    it.t0row = it.c0 + it.r * kBlk;
    return it;
}

template <bool kBalance>
__global__ void __launch_bounds__(kOutThreads, 1)
tc_output_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_s,
                 const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_out,
                 TcOutArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    // rfull[s]: one phase per operand tile loaded into slot s (the MMA
    // thread counts them per slot).  The gate/output tile has its own
    // barrier, g_full, one phase per item, waited in order by the epilogue.
    // (Were the gate tile counted on its slot's rfull, the MMA thread, which
    // never waits for it, could reach the next operand tile of that slot
    // while the gate load is still landing and mistake the slot's phase two
    // back for the one it needs: the same parity.)
    __shared__ uint64_t rfull[kSlots], rempty[kSlots], g_full;
    __shared__ uint64_t s_full, s_read, p_full[2], p_free[2], o_full, o_free, drain;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    __shared__ uint32_t op_n[kSlots], g_n;            // operand tiles per slot, gate tiles

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    unsigned *err = a.err;
    const long long nbh = a.items / (a.nchunks * a.rblocks);   // sequence-heads
    auto slot_ptr = [smem](int it) -> uint8_t * { return smem + (it % kSlots) * kSlot; };
    uint8_t *pbuf = smem + TcOutSmem::kP;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&rfull[s], 1);
            mbar_init(&rempty[s], 1);
            op_n[s] = 0;
        }
        mbar_init(&g_full, 1);
        g_n = 0;
        mbar_init(&s_full, 1);
        mbar_init(&s_read, kEpiThreads);
        for (int x = 0; x < 2; ++x) {                    // one P half per warpgroup
            mbar_init(&p_full[x], kEpiThreads / 2);
            mbar_init(&p_free[x], 1);
        }
        mbar_init(&o_full, 1);
        mbar_init(&o_free, kEpiThreads);
        mbar_init(&drain, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v); tma_prefetch_desc(&tm_s);
        if (a.has_gate) tma_prefetch_desc(&tm_g);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t tO = tmem, tQ = tmem + 256, tS = tmem + 384;
    grid_dependency_wait();                             // Qt, Kt, S_prev from the kernels before

    int pit = 0;                           // producer: ring items issued
    if (warp == 0) {
        if (lane == 0) {
            int &it = pit;
            bool ok = true;
            auto acquire = [&]() -> bool {
                if (it < kSlots) return true;
                return mbar_wait(&rempty[it % kSlots], ((it / kSlots) - 1) & 1, &abort_flag, err);
            };
            auto issue = [&](const CUtensorMap *map, int rank, int c1, int c2, int c3,
                             uint64_t *bar) {
                uint8_t *d = slot_ptr(it);
                mbar_expect_tx(bar, kSlot);
                for (int x = 0; x < 4; ++x) {
                    if (rank == 2) tma_load_2d(d + x * kBox, map, bar, 64 * x, c1);
                    else if (rank == 3) tma_load_3d(d + x * kBox, map, bar, 64 * x, c1, c2);
                    else tma_load_4d(d + x * kBox, map, bar, 64 * x, c1, c2, c3);
                }
                ++it;
            };
            for (int w = blockIdx.x; ok && w < a.items; w += gridDim.x) {
                const TcItem m = tc_item<kBalance>(a, w);
                if (!m.valid) continue;
                const int srow = (m.bh * a.nchunks + m.c) * kD;
                // debug build: the item's tile coordinates lie inside its tensors
                if (!in_bounds(m.t0row, a.n, err, kSiteOutput) || !in_bounds(m.bh, nbh, err, kSiteOutput) ||
                    !in_bounds(srow + kD - 1, nbh * a.nchunks * kD, err, kSiteOutput)) {
                    abort_flag = 1;
                    ok = false;
                    break;
                }
                // an operand tile: counted on its slot's rfull
                auto op = [&](const CUtensorMap *map, int rank, int c1, int c2, int c3) {
                    *(volatile uint32_t *)&op_n[it % kSlots] += 1;
                    issue(map, rank, c1, c2, c3, &rfull[it % kSlots]);
                };
                if (!(ok = acquire())) break;
                op(&tm_q, 3, m.t0row, m.bh, 0);
                if (!(ok = acquire())) break;
                op(&tm_k, 3, m.c0, m.bh, 0);
                for (int t = 0; ok && t < m.nk; ++t) {
                    if (t + 1 < m.nk) {
                        if (!(ok = acquire())) break;
                        op(&tm_k, 3, m.c0 + (t + 1) * kKeyTile, m.bh, 0);
                    }
                    if (t < m.nsp) {
                        if (!(ok = acquire())) break;
                        op(&tm_s, 2, srow + kBlk * t, 0, 0);
                    }
                    if (!(ok = acquire())) break;
                    op(&tm_v, 4, m.h, m.c0 + t * kKeyTile, m.b);
                }
                for (int p = m.nk; ok && p < m.nsp; ++p) {
                    if (!(ok = acquire())) break;
                    op(&tm_s, 2, srow + kBlk * p, 0, 0);
                }
                if (ok && (ok = acquire())) {                // the gate/output tile
                    *(volatile uint32_t *)&g_n += 1;
                    if (a.has_gate) {
                        issue(&tm_g, 4, m.h, m.t0row, m.b, &g_full);
                    } else {
                        mbar_arrive(&g_full);                 // reserved for the output rows
                        ++it;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(128, kKeyTile, 0, 0);
            const uint32_t id_pv = idesc_bf16(128, 256, 0, 1);
            const uint32_t sbase = smem_u32(smem);
            const uint32_t sP = sbase + TcOutSmem::kP;
            int it = 0, nqk = 0, npv = 0, li = 0;
            uint32_t opar = 0;                         // per slot: parity of its next rfull phase
            bool ok = true;
            auto take = [&]() -> bool {
                const int s = it % kSlots;
                if (!mbar_wait(&rfull[s], (opar >> s) & 1u, &abort_flag, err)) return false;
                opar ^= 1u << s;
                tc_fence_after();
                return true;
            };
            for (int w = blockIdx.x; ok && w < a.items; w += gridDim.x, ++li) {
                const TcItem m = tc_item<kBalance>(a, w);
                if (!m.valid) { --li; continue; }
                bool o_written = false;
                // O is free once the previous item's epilogue has read it
                auto claim_o = [&]() -> bool {
                    if (o_written || li == 0) return true;
                    return mbar_wait(&o_free, (li - 1) & 1, &abort_flag, err);
                };
                // Qt (K-major, 128-byte swizzle) -> TMEM, 16 columns of K per copy.
                // The PTX ISA orders tcgen05.cp before later tcgen05.mma of the
                // same thread, but not after earlier ones: the previous item's
                // MMAs, the last readers of Qt, must have completed (o_full)
                // before the copy may overwrite it.
                if (li > 0 && !(ok = mbar_wait(&o_full, (li - 1) & 1, &abort_flag, err))) break;
                tc_fence_after();
                if (!(ok = take())) break;
                {
                    const uint32_t base = sbase + (it % kSlots) * kSlot;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        tmem_cp_128x256b(tQ + 8 * ks,
                                         smem_desc_sw128(base + (ks / 4) * kBox + (ks % 4) * 32, 16, 1024));
                    mma_commit(&rempty[it % kSlots]);
                    ++it;
                }
                auto qk = [&](int t) -> bool {
                    if (nqk >= 1 && !mbar_wait(&s_read, (nqk - 1) & 1, &abort_flag, err)) return false;
                    if (!take()) return false;
                    const uint32_t base = sbase + (it % kSlots) * kSlot;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_bf16_ts(tS, tQ + 8 * ks,
                                    smem_desc_sw128(base + (ks / 4) * kBox + (ks % 4) * 32, 16, 1024),
                                    id_qk, ks > 0 ? 1u : 0u);
                    mma_commit(&rempty[it % kSlots]);
                    mma_commit(&s_full);
                    ++it;
                    ++nqk;
                    (void)t;
                    return true;
                };
                // O += Qt[:, 128p .. 128p+128) S_prev[128p .. 128p+128, :]
                auto qs_half = [&](int p) -> bool {
                    if (!take() || !claim_o()) return false;
                    const uint32_t base = sbase + (it % kSlots) * kSlot;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tO, tQ + 8 * (8 * p + kk),
                                    smem_desc_sw128(base + kk * 2048, kBox, 1024), id_pv,
                                    (o_written || kk > 0) ? 1u : 0u);
                    o_written = true;
                    mma_commit(&rempty[it % kSlots]);
                    ++it;
                    return true;
                };
                ok = qk(0);
                for (int t = 0; ok && t < m.nk; ++t) {
                    if (t + 1 < m.nk && !(ok = qk(t + 1))) break;
                    if (t < m.nsp && !(ok = qs_half(t))) break;
                    // P V in two halves of 64 keys, each issued as soon as its
                    // warpgroup has written that half of P
                    if (!(ok = take() && claim_o())) break;
                    const uint32_t base = sbase + (it % kSlots) * kSlot;
                    for (int hx = 0; ok && hx < 2; ++hx) {
                        if (!mbar_wait(&p_full[hx], npv & 1, &abort_flag, err)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int kk = 4 * hx + k4;
                            mma_bf16(tO, smem_desc_sw128(sP + hx * kBox + k4 * 32, 16, 1024),
                                     smem_desc_sw128(base + kk * 2048, kBox, 1024), id_pv,
                                     (o_written || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(&p_free[hx]);
                    }
                    if (!ok) break;
                    o_written = true;
                    mma_commit(&rempty[it % kSlots]);
                    ++it;
                    ++npv;
                }
                for (int p = m.nk; ok && p < m.nsp; ++p) ok = qs_half(p);
                if (!ok) break;
                mma_commit(&o_full);
                ++it;                                          // skip the gate/output item
            }
        }
    } else {
        // two warpgroups: for every tile wg w masks and converts S columns
        // [64w, 64w+64); in the epilogue wg w owns O columns [128w, 128w+128)
        const int wg = (warp - 2) / 4;
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;                         // row of the 128-row block
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        uint8_t *prow = pbuf + wg * kBox + row * 128;           // this row in P box wg
        int it_base = 0, ntile = 0, li = 0;
        bool ok = true;
        for (int w = blockIdx.x; ok && w < a.items; w += gridDim.x, ++li) {
            const TcItem m = tc_item<kBalance>(a, w);
            if (!m.valid) { --li; continue; }
            const int lrow = m.r * kBlk + row;                  // row within the chunk
            for (int t = 0; t < m.nk; ++t, ++ntile) {
                if (!warp_wait(&s_full, ntile & 1, &abort_flag, err)) { ok = false; break; }
                tc_fence_after();
                uint32_t v0[32], v1[32];
                const uint32_t col = tS + lane_off + 64 * wg;
                tmem_ld32(col, v0);
                tmem_ld32(col + 32, v1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&s_read);                           // S may be overwritten now
                const int j0 = t * kKeyTile + 64 * wg;          // first key of this half tile
                uint32_t wv[32];
                if (a.parallel && t < m.r) {                    // a whole earlier block
                    const float tf = exp2f((float)(kKeyTile * (m.r - t)) * a.log2g[m.h]);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        wv[e] = pack_bf16x2(tf * __uint_as_float(v0[2 * e]), tf * __uint_as_float(v0[2 * e + 1]));
                        wv[16 + e] = pack_bf16x2(tf * __uint_as_float(v1[2 * e]), tf * __uint_as_float(v1[2 * e + 1]));
                    }
                } else if (j0 + 63 <= lrow) {                   // every key at or before the row
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        wv[e] = pack_bf16x2(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1]));
                        wv[16 + e] = pack_bf16x2(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1]));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int j = j0 + 2 * e;
                        const float x0 = (lrow >= j) ? __uint_as_float(v0[2 * e]) : 0.f;
                        const float x1 = (lrow >= j + 1) ? __uint_as_float(v0[2 * e + 1]) : 0.f;
                        const float y0 = (lrow >= j + 32) ? __uint_as_float(v1[2 * e]) : 0.f;
                        const float y1 = (lrow >= j + 33) ? __uint_as_float(v1[2 * e + 1]) : 0.f;
                        wv[e] = pack_bf16x2(x0, x1);
                        wv[16 + e] = pack_bf16x2(y0, y1);
                    }
                }
                // the previous tile's P must have been consumed by its P V
                if (ntile >= 1 && !warp_wait(&p_free[wg], (ntile - 1) & 1, &abort_flag, err)) { ok = false; break; }
                // 64 keys of this row = eight 16-byte chunks of the 128-byte-swizzled box
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4 *>(prow + ((ch ^ (row & 7)) * 16)) =
                        make_uint4(wv[4 * ch], wv[4 * ch + 1], wv[4 * ch + 2], wv[4 * ch + 3]);
                fence_async_shared();
                tc_fence_before();
                mbar_arrive(&p_full[wg]);
            }
            // ring items of this work item: Qt, nk Kt tiles, nsp S_prev halves,
            // nk V tiles, then the gate/output tile
            const int ig = it_base + 1 + 2 * m.nk + m.nsp;
            it_base = ig + 1;
            uint8_t *ybuf = slot_ptr(ig);
            const bool go = ok && warp_wait(&o_full, li & 1, &abort_flag, err) &&
                            warp_wait(&g_full, li & 1, &abort_flag, err);
            // the P tile is idle between items: it holds the partial row sums
            float (*red)[kBlk] = reinterpret_cast<float (*)[kBlk]>(pbuf);   // [4][128]
            float mean = 0.f, rstd = 1.f;
            if (go) tc_fence_after();
            if (a.has_gate) {
                // GroupNorm statistics over the row's 256 channels: each
                // warpgroup sums its half (values and squares, shifted by the
                // row's first value for accuracy); the halves meet in shared memory.
                float sum = 0.f, sq = 0.f, shift = 0.f;
                if (go) {
                    uint32_t v0[32];
                    tmem_ld32(tO + lane_off, v0);           // column 0 of the row: the shift
                    tmem_wait_ld();
                    shift = __uint_as_float(v0[0]);
#pragma unroll 1
                    for (int cb = 0; cb < 4; ++cb) {
                        uint32_t v[32];
                        tmem_ld32(tO + lane_off + 128 * wg + 32 * cb, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const float d = __uint_as_float(v[e]) - shift;
                            sum += d;
                            sq = fmaf(d, d, sq);
                        }
                    }
                }
                red[2 * wg][row] = sum;
                red[2 * wg + 1][row] = sq;
                named_barrier(1, kEpiThreads);
                const float ms = (red[0][row] + red[2][row]) * (1.f / kD);  // mean of x - shift
                const float m2 = (red[1][row] + red[3][row]) * (1.f / kD);
                mean = shift + ms;
                rstd = rsqrtf(fmaxf(m2 - ms * ms, 0.f) + a.eps);
                named_barrier(1, kEpiThreads);              // red is reused as P next
            }
            if (go) {
                // This row's slot in the 128-byte-swizzled gate/output tile.
                uint8_t *yrow = ybuf + row * 128;
                const int sw = row & 7;
                const float *gw = a.gn_weight ? a.gn_weight + m.h * kD : nullptr;
                const float *gb = a.gn_bias ? a.gn_bias + m.h * kD : nullptr;
#pragma unroll 1
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int cb = 4 * wg + k4;                   // 32-column block of O
                    uint32_t v[32];
                    tmem_ld32(tO + lane_off + 32 * cb, v);
                    tmem_wait_ld();
                    if (k4 == 3) {                                // O fully read: free it
                        tc_fence_before();
                        mbar_arrive(&o_free);
                    }
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
                                    if (gw) yh *= gw[ch];
                                    if (gb) yh += gb[ch];
                                    y[e] = swish_fast(hh ? gg.y : gg.x) * yh;
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
            } else {
                mbar_arrive(&o_free);
            }
            // Both epilogue warpgroups reach this barrier on every path.
            named_barrier(1, kEpiThreads);
            if (wg == 0 && row == 0) {
                if (!abort_flag) {
                    for (int x = 0; x < 4; ++x)
                        tma_store_4d(&tm_out, ybuf + x * kBox, 64 * x, m.h, m.t0row, m.b);
                    tma_store_commit();
                    tma_store_wait_read();
                }
                mbar_arrive(&rempty[ig % kSlots]);             // the tile may be refilled
            }
            if (!go) ok = false;
        }
    }
    tc_fence_before();
    __syncthreads();
    // Every role has finished, so abort_flag is final.  After an abort, wait
    // (bounded) for what this CTA still has in flight: the TMA loads (at most
    // the last kSlots issued) before shared memory goes away, the MMAs before
    // tensor memory is freed.
    if (abort_flag && warp == 0 && lane == 0) {
        for (int j = 0; j < kSlots; ++j)
            if (op_n[j] > 0) mbar_drain(&rfull[j], (op_n[j] - 1) & 1, err);
        if (g_n > 0) mbar_drain(&g_full, (g_n - 1) & 1, err);
    }
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

// ------------------------------------------------------------------ paired output pass
// The output pass on CTA pairs: the two CTAs of a cluster work as one
// (tcgen05 cta_group::2, M = 256).  A pair-item is the row blocks (2p, 2p+1)
// of one chunk; CTA k owns row block 2p + k in its own TMEM (same layout as
// tc_output: O [0,256), Qt [256,384), S [384,512)).  The B operands are
// split by N between the CTAs: for Qt Kt^T each CTA loads 64 of the tile's
// 128 keys, for P V and Qt S_prev 128 of the 256 d_v columns, so a key tile
// costs each CTA 64 KB of loads instead of 128 KB and a ring of six 32 KB
// slots holds twice the tiles of tc_output's three 64 KB slots.  The pair
// spends one 128 x 128 tile of wasted MMA work per pair-item where the
// lower row block stops short of the upper one's last key tile.
//
// Roles as in tc_output, with the leader (rank 0) issuing every MMA:
//   warp 0 (both CTAs): TMA loads into its own slots.  Operand loads count
//     on the leader's rfull barrier of the slot (the leader arms it for both
//     CTAs' bytes); the gate/output tile (two slots), and raw q when the
//     pair folds it, count on this CTA's own lfull barriers.  Each CTA
//     completes one lfull phase for every ring item, so lfull follows the
//     ring order; rfull[s] has one phase per operand item of slot s, and
//     its users count those per slot.  A CTA can refill a gate slot as soon
//     as its own epilogue is done, possibly before the other CTA reaches it;
//     counting rfull phases per operand item keeps such a load in the phase
//     of its own item (its slot's previous operand item was consumed before
//     the slot could pass on).
//   warp 1: TMEM allocation (both CTAs, paired); the leader's lane 0
//     issues the copies and MMAs, whose commits arrive on the barrier of
//     the same offset in both CTAs (rempty, s_full, p_free, o_full).
//   warps 2-9 (both CTAs): the mask pass and the epilogue on this CTA's
//     rows; their arrivals (s_read, p_full, o_free) go to the leader.
// A timeout in either CTA raises both CTAs' abort flags; at the end the
// leader settles and drains the operand loads of both CTAs before the
// cluster's last barrier, so neither CTA exits with loads still landing in
// its shared memory.
constexpr int kPairSlots = 6;
constexpr uint32_t kPairSlot = 2 * kBox;           // 32 KB
constexpr int kPairThreads = 448;                  // 14 warps: the 10 of tc_output + 4 fold warps
// Bits naming the paired pass's waits in the error word (see mbar_wait).
enum PairWaitSite : unsigned {
    kWaitRempty = 1u << 16, kWaitRfull = 1u << 17, kWaitOFree = 1u << 18,
    kWaitOFullMma = 1u << 19, kWaitQReady = 1u << 20, kWaitSRead = 1u << 21,
    kWaitPFull = 1u << 22, kWaitLfullFold = 1u << 23, kWaitSFull = 1u << 24,
    kWaitPFree = 1u << 25, kWaitOFullEpi = 1u << 26, kWaitLfullEpi = 1u << 27,
};
constexpr int kFoldThreads = 128;

struct TcPairSmem {
    static constexpr uint32_t kP = kPairSlots * kPairSlot;   // P tile; the epilogue's row sums
    static constexpr uint32_t kBytes = kP + 2 * kBox + 1024;
};

struct TcPairItem {
    int p, c, bh, b, h, c0, nk, nsp, r, t0row;
    bool valid;                                    // some row of the pair lies in the chunk
};

// Pair-item w: group g = w / np is one (sequence, head, chunk) with np row-
// block pairs at consecutive w, rotated by the group index as in tc_item.
__device__ __forceinline__ TcPairItem tc_pair_item(const TcOutArgs &a, int w, int rank) {
    const int np = (a.rblocks + 1) / 2;
    TcPairItem it;
    const int g = w / np;
    it.p = (w + g) % np;
    it.c = g % a.nchunks;
    it.bh = g / a.nchunks;
    it.b = it.bh / a.heads;
    it.h = it.bh % a.heads;
    it.c0 = it.c * a.chunk;
    const int L = min(a.chunk, a.n - it.c0);
    it.valid = 2 * it.p * kBlk < L;
    const int kend = min(kBlk * (2 * it.p + 2), L);   // keys the pair's rows see
    it.nk = (kend + kKeyTile - 1) / kKeyTile;
    it.nsp = (it.c > 0 || a.has_state_in) ? 2 : 0;
    it.r = 2 * it.p + rank;
    it.t0row = it.c0 + it.r * kBlk;
    return it;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
tc_output_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kh,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_s,
                      const __grid_constant__ CUtensorMap tm_g,
                      const __grid_constant__ CUtensorMap tm_out,
                      const __grid_constant__ CUtensorMap tm_qraw, TcOutArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t rfull[kPairSlots], rempty[kPairSlots], lfull[kPairSlots];
    __shared__ uint64_t s_full, s_read, p_full[2], p_free[2], o_full, o_free, drain, q_ready;
    // raw q halves (fold mode): one phase per item, waited in sequence by the
    // fold warps (a slot's lfull would let them alias a phase two ahead)
    __shared__ uint64_t qfull[2];
    __shared__ uint32_t q_n[2];                    // raw-q halves this CTA issued
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    __shared__ uint32_t op_n[kPairSlots];          // operand items this CTA issued per slot
    __shared__ uint32_t lf_n[kPairSlots];          // lfull phases this CTA armed per slot

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    unsigned *err = a.err;
    const int np = (a.rblocks + 1) / 2;
    const long long nbh = a.items / (a.nchunks * np);
    const int cluster = blockIdx.x / 2, nclusters = gridDim.x / 2;
    auto slot_ptr = [smem](int it) -> uint8_t * { return smem + (it % kPairSlots) * kPairSlot; };
    uint8_t *pbuf = smem + TcPairSmem::kP;
    // the leader's copy of a barrier, as a shared::cluster address
    auto at_leader = [](uint64_t *bar) -> uint32_t { return mapa_shared(smem_u32(bar), 0); };
    const uint32_t peer_abort = mapa_shared(smem_u32(&abort_flag), rank ^ 1u);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairSlots; ++s) {
            mbar_init(&rfull[s], 1);
            mbar_init(&rempty[s], 1);
            mbar_init(&lfull[s], 1);
        }
        mbar_init(&s_full, 1);
        // cross-CTA signals arrive once per warp (lane 0, after __syncwarp)
        mbar_init(&s_read, 2 * kEpiThreads / 32);
        for (int x = 0; x < 2; ++x) {                    // one P half per warpgroup, both CTAs
            mbar_init(&p_full[x], 2 * (kEpiThreads / 2) / 32);
            mbar_init(&p_free[x], 1);
        }
        mbar_init(&o_full, 1);
        mbar_init(&o_free, 2 * kEpiThreads / 32);
        mbar_init(&drain, 1);
        mbar_init(&q_ready, 2 * kFoldThreads / 32);
        mbar_init(&qfull[0], 1);
        mbar_init(&qfull[1], 1);
        q_n[0] = q_n[1] = 0;
        abort_flag = 0;
        for (int s = 0; s < kPairSlots; ++s) op_n[s] = lf_n[s] = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, 512);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_kh);
        tma_prefetch_desc(&tm_v); tma_prefetch_desc(&tm_s);
        if (a.has_gate) tma_prefetch_desc(&tm_g);
        if (a.fold_q) tma_prefetch_desc(&tm_qraw);
    }
    tc_fence_before();
    cluster_sync();                                   // both CTAs' barriers and TMEM exist
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t tO = tmem, tQ = tmem + 256, tS = tmem + 384;
    grid_dependency_wait();                           // Qt, Kt, S_prev from the kernels before

    // Raises this CTA's and the peer's abort flags (after a failed wait).
    auto abort_both = [&]() {
        abort_flag = 1;
        st_cluster_u32(peer_abort, 1u);
    };

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            auto acquire = [&]() -> bool {
                if (it < kPairSlots) return true;
                return mbar_wait(&rempty[it % kPairSlots], ((it / kPairSlots) - 1) & 1,
                                 &abort_flag, err, kWaitRempty);
            };
            // one operand item: `boxes` boxes of 16 KB (or 8 KB for Kt halves) into
            // this CTA's slot, counted on the leader's rfull (armed for both CTAs)
            auto issue_op = [&](int kind, int c1, int c2, int c3) {
                uint8_t *d = slot_ptr(it);
                uint64_t *bar = &rfull[it % kPairSlots];
                const uint32_t lbar = at_leader(bar);
                *(volatile uint32_t *)&op_n[it % kPairSlots] += 1;
                *(volatile uint32_t *)&lf_n[it % kPairSlots] += 1;
                mbar_arrive(&lfull[it % kPairSlots]);          // keeps lfull in ring order
                if (leader) mbar_expect_tx(bar, 2 * kPairSlot);
                if (kind == 0) {                               // Qt: two 64-col boxes
                    for (int x = 0; x < 2; ++x)
                        tma_load_3d_pair(d + x * kBox, &tm_q, lbar, 64 * (c3 + x), c1, c2);
                } else if (kind == 1) {                        // Kt half: 64 keys x 256
                    for (int x = 0; x < 4; ++x)
                        tma_load_3d_pair(d + x * (kBox / 2), &tm_kh, lbar, 64 * x, c1, c2);
                } else if (kind == 2) {                        // S_prev half: 128 d_v cols
                    for (int x = 0; x < 2; ++x)
                        tma_load_2d_pair(d + x * kBox, &tm_s, lbar, 128 * (int)rank + 64 * x, c1);
                } else {                                       // V: 128 d_v cols x 128 keys
                    for (int x = 0; x < 2; ++x)
                        tma_load_4d_pair(d + x * kBox, &tm_v, lbar, 128 * (int)rank + 64 * x, c2,
                                         c1, c3);
                }
                ++it;
            };
            for (int w = cluster; ok && w < a.items; w += nclusters) {
                const TcPairItem m = tc_pair_item(a, w, rank);
                if (!m.valid) continue;
                const int srow = (m.bh * a.nchunks + m.c) * kD;
                if (!in_bounds(m.bh, nbh, err, kSiteOutputPair) ||
                    !in_bounds(srow + kD - 1, nbh * a.nchunks * kD, err, kSiteOutputPair)) {
                    ok = false;
                    abort_both();
                    break;
                }
                for (int half = 0; ok && half < 2; ++half) {
                    if (!(ok = acquire())) break;
                    if (a.fold_q) {
                        // raw q rows of this CTA, folded in place by the fold
                        // warps (counted on lfull; rfull only kept in order)
                        uint8_t *d = slot_ptr(it);
                        *(volatile uint32_t *)&lf_n[it % kPairSlots] += 1;
                        mbar_arrive(&lfull[it % kPairSlots]);      // keeps lfull in ring order
                        uint64_t *qb = &qfull[half];
                        *(volatile uint32_t *)&q_n[half] += 1;
                        mbar_expect_tx(qb, kPairSlot);
                        for (int x = 0; x < 2; ++x)
                            tma_load_4d(d + x * kBox, &tm_qraw, qb, 128 * half + 64 * x, m.h,
                                        m.t0row, m.b);
                        ++it;
                    } else {
                        issue_op(0, m.t0row, m.bh, 2 * half);
                    }
                }
                if (!ok || !(ok = acquire())) break;
                issue_op(1, m.c0 + 64 * (int)rank, m.bh, 0);
                for (int t = 0; ok && t < m.nk; ++t) {
                    if (t + 1 < m.nk) {
                        if (!(ok = acquire())) break;
                        issue_op(1, m.c0 + (t + 1) * kKeyTile + 64 * (int)rank, m.bh, 0);
                    }
                    if (t < m.nsp) {
                        if (!(ok = acquire())) break;
                        issue_op(2, srow + kBlk * t, 0, 0);
                    }
                    if (!(ok = acquire())) break;
                    issue_op(3, m.c0 + t * kKeyTile, m.h, m.b);
                }
                for (int p = m.nk; ok && p < m.nsp; ++p) {
                    if (!(ok = acquire())) break;
                    issue_op(2, srow + kBlk * p, 0, 0);
                }
                // the gate/output tile: two slots of this CTA, each counted on
                // its own lfull (or only reserved for the output rows)
                for (int half = 0; ok && half < 2; ++half) {
                    if (!(ok = acquire())) break;
                    uint8_t *gs = slot_ptr(it);
                    uint64_t *lb = &lfull[it % kPairSlots];
                    *(volatile uint32_t *)&lf_n[it % kPairSlots] += 1;
                    if (a.has_gate) {
                        mbar_expect_tx(lb, 2 * kBox);
                        for (int x = 0; x < 2; ++x)
                            tma_load_4d(gs + x * kBox, &tm_g, lb, 128 * half + 64 * x, m.h,
                                        m.t0row, m.b);
                    } else {
                        mbar_arrive(lb);
                    }
                    ++it;
                }
            }
            if (!ok) abort_both();
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            const uint32_t id_qk = idesc_bf16(256, kKeyTile, 0, 0);
            const uint32_t id_pv = idesc_bf16(256, 256, 0, 1);
            const uint32_t sP = smem_u32(pbuf);
            int it = 0, nqk = 0, npv = 0, li = 0;
            uint32_t opar = 0;                         // per slot: parity of its next rfull phase
            bool ok = true;
            auto take = [&]() -> bool {
                const int s = it % kPairSlots;
                if (!mbar_wait(&rfull[s], (opar >> s) & 1u, &abort_flag, err, kWaitRfull)) return false;
                opar ^= 1u << s;
                tc_fence_after();
                return true;
            };
            auto slot_addr = [&](int i) -> uint32_t { return smem_u32(slot_ptr(i)); };
            for (int w = cluster; ok && w < a.items; w += nclusters, ++li) {
                const TcPairItem m = tc_pair_item(a, w, 0);
                if (!m.valid) { --li; continue; }
                bool o_written = false;
                auto claim_o = [&]() -> bool {
                    if (o_written || li == 0) return true;
                    return mbar_wait(&o_free, (li - 1) & 1, &abort_flag, err, kWaitOFree);
                };
                // the previous item's MMAs read Qt from TMEM: they must be
                // complete before the copy below overwrites it (cp is ordered
                // before later MMAs of this thread, not after earlier ones)
                if (li > 0 && !(ok = mbar_wait(&o_full, (li - 1) & 1, &abort_flag, err, kWaitOFullMma))) break;
                tc_fence_after();
                // Qt of both CTAs -> their TMEM, 16 columns of K per copy: as
                // loaded, or once the fold warps of both CTAs have folded it
                if (a.fold_q) {
                    if (!(ok = mbar_wait(&q_ready, li & 1, &abort_flag, err, kWaitQReady))) break;
                    tc_fence_after();
                } else if (!(ok = take())) {
                    break;
                }
                const uint32_t qa = slot_addr(it);
                const int sa = it % kPairSlots;
                ++it;
                if (!a.fold_q && !(ok = take())) break;
                const uint32_t qb = slot_addr(it);
                const int sb = it % kPairSlots;
                ++it;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t base = (ks < 8 ? qa : qb) + ((ks / 4) % 2) * kBox + (ks % 4) * 32;
                    tmem_cp_128x256b_pair(tQ + 8 * ks, smem_desc_sw128(base, 16, 1024));
                }
                mma_commit_pair(&rempty[sa], 3);
                mma_commit_pair(&rempty[sb], 3);
                // S = Qt Kt^T for key tile t: each CTA holds 64 of its keys
                auto qk = [&]() -> bool {
                    if (nqk >= 1 && !mbar_wait(&s_read, (nqk - 1) & 1, &abort_flag, err, kWaitSRead)) return false;
                    if (!take()) return false;
                    const uint32_t base = slot_addr(it);
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_bf16_ts_pair(tS, tQ + 8 * ks,
                                         smem_desc_sw128(base + (ks / 4) * (kBox / 2) + (ks % 4) * 32,
                                                         16, 1024),
                                         id_qk, ks > 0 ? 1u : 0u);
                    mma_commit_pair(&rempty[it % kPairSlots], 3);
                    mma_commit_pair(&s_full, 3);
                    ++it;
                    ++nqk;
                    return true;
                };
                // O += Qt[:, 128p .. 128p+128) S_prev[128p .. 128p+128, :]
                auto qs_half = [&](int p) -> bool {
                    if (!take() || !claim_o()) return false;
                    const uint32_t base = slot_addr(it);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts_pair(tO, tQ + 8 * (8 * p + kk),
                                         smem_desc_sw128(base + kk * 2048, kBox, 1024), id_pv,
                                         (o_written || kk > 0) ? 1u : 0u);
                    o_written = true;
                    mma_commit_pair(&rempty[it % kPairSlots], 3);
                    ++it;
                    return true;
                };
                ok = qk();
                for (int t = 0; ok && t < m.nk; ++t) {
                    if (t + 1 < m.nk && !(ok = qk())) break;
                    if (t < m.nsp && !(ok = qs_half(t))) break;
                    if (!(ok = take() && claim_o())) break;
                    const uint32_t base = slot_addr(it);
                    for (int hx = 0; ok && hx < 2; ++hx) {
                        if (!mbar_wait(&p_full[hx], npv & 1, &abort_flag, err, kWaitPFull)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int kk = 4 * hx + k4;
                            mma_bf16_pair(tO, smem_desc_sw128(sP + hx * kBox + k4 * 32, 16, 1024),
                                          smem_desc_sw128(base + kk * 2048, kBox, 1024), id_pv,
                                          (o_written || kk > 0) ? 1u : 0u);
                        }
                        mma_commit_pair(&p_free[hx], 3);
                    }
                    if (!ok) break;
                    o_written = true;
                    mma_commit_pair(&rempty[it % kPairSlots], 3);
                    ++it;
                    ++npv;
                }
                for (int p = m.nk; ok && p < m.nsp; ++p) ok = qs_half(p);
                if (!ok) break;
                mma_commit_pair(&o_full, 3);
                it += 2;                                       // skip the gate/output slots
            }
            if (!ok) abort_both();
        }
    } else if (warp >= 10) {
        // Fold warps: rotate and decay-scale this CTA's raw q rows in place,
        // Qt_i = g^(lf+1) R q_i (lf: the row's index in its fold block).
        // Thread j owns the pair (2j, 2j+1) and walks the 128 rows in eight
        // interleaved runs of 16; each run starts from an exact (cos, sin)
        // and steps the complex factor g e^{i theta_j} per row.
        if (a.fold_q) {
            const int j = threadIdx.x - 10 * 32;               // pair column 0..127
            const uint32_t l_q_ready = at_leader(&q_ready);
            const double theta = a.theta[j];
            float st_c = 1.f, st_s = 0.f;                      // e^{i theta_j}
            if (a.rotate) {
                const float2 r = rotation_cs(1, theta);
                st_c = r.x;
                st_s = r.y;
            }
            const int bx = j / 32;                             // 64-column box
            const uint32_t in_row = (uint32_t)((j % 4) * 4);
            const int ch = (j % 32) / 4;                       // 16-byte chunk in the row
            int it_base = 0, fi = 0;
            bool ok = true;
            for (int w = cluster; ok && w < a.items; w += nclusters, ++fi) {
                const TcPairItem m = tc_pair_item(a, w, rank);
                if (!m.valid) { --fi; continue; }
                const int qi = it_base;
                it_base += 2 + 2 * m.nk + m.nsp + 2;
                const int qs = qi + bx / 2;                    // this column's slot (warp-uniform)
                if (!warp_wait(&qfull[bx / 2], fi & 1, &abort_flag, err, kWaitLfullFold)) {
                    ok = false;
                    break;
                }
                uint8_t *box = slot_ptr(qs) + (bx % 2) * kBox;
                const float lg = a.log2g[m.h];
                const float gc = exp2f(lg) * st_c, gs = exp2f(lg) * st_s;   // g e^{i theta}
                const int lf0 = a.fold == kBlk ? 0 : m.r * kBlk;            // fold index of row 0
                float zc[8], zs[8];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const float2 r = a.rotate ? rotation_cs(a.pos0 + m.t0row + 16 * g, theta)
                                              : make_float2(1.f, 0.f);
                    const float sc = exp2f((float)(lf0 + 16 * g + 1) * lg);
                    zc[g] = r.x * sc;
                    zs[g] = r.y * sc;
                }
#pragma unroll 2
                for (int i = 0; i < 16; ++i) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const int row = 16 * g + i;
                        uint32_t *pw = reinterpret_cast<uint32_t *>(
                            box + row * 128 + ((ch ^ (row & 7)) * 16) + in_row);
                        const uint32_t raw = *pw;
                        const float2 x =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw));
                        const float c = zc[g], sn = zs[g];
                        *pw = pack_bf16x2(x.x * c - x.y * sn, x.x * sn + x.y * c);
                        zc[g] = c * gc - sn * gs;
                        zs[g] = c * gs + sn * gc;
                    }
                }
                fence_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(l_q_ready);
            }
            if (!ok && lane == 0) abort_both();
        }
    } else {
        const int wg = (warp - 2) / 4;
        const int q4 = warp % 4;
        const int row = 32 * q4 + lane;
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const uint32_t l_s_read = at_leader(&s_read), l_o_free = at_leader(&o_free);
        const uint32_t l_p_full = at_leader(&p_full[wg]);
        uint8_t *prow = pbuf + wg * kBox + row * 128;
        int it_base = 0, ntile = 0, li = 0;
        bool ok = true;
        for (int w = cluster; ok && w < a.items; w += nclusters, ++li) {
            const TcPairItem m = tc_pair_item(a, w, rank);
            if (!m.valid) { --li; continue; }
            const int lrow = m.r * kBlk + row;                  // row within the chunk
            for (int t = 0; t < m.nk; ++t, ++ntile) {
                if (!warp_wait(&s_full, ntile & 1, &abort_flag, err, kWaitSFull)) { ok = false; break; }
                tc_fence_after();
                uint32_t v0[32], v1[32];
                const uint32_t col = tS + lane_off + 64 * wg;
                tmem_ld32(col, v0);
                tmem_ld32(col + 32, v1);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(l_s_read);   // S may be overwritten now
                const int j0 = t * kKeyTile + 64 * wg;
                uint32_t wv[32];
                if (a.parallel && t < m.r) {
                    const float tf = exp2f((float)(kKeyTile * (m.r - t)) * a.log2g[m.h]);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        wv[e] = pack_bf16x2(tf * __uint_as_float(v0[2 * e]), tf * __uint_as_float(v0[2 * e + 1]));
                        wv[16 + e] = pack_bf16x2(tf * __uint_as_float(v1[2 * e]), tf * __uint_as_float(v1[2 * e + 1]));
                    }
                } else if (j0 + 63 <= lrow) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        wv[e] = pack_bf16x2(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1]));
                        wv[16 + e] = pack_bf16x2(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1]));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int j = j0 + 2 * e;
                        const float x0 = (lrow >= j) ? __uint_as_float(v0[2 * e]) : 0.f;
                        const float x1 = (lrow >= j + 1) ? __uint_as_float(v0[2 * e + 1]) : 0.f;
                        const float y0 = (lrow >= j + 32) ? __uint_as_float(v1[2 * e]) : 0.f;
                        const float y1 = (lrow >= j + 33) ? __uint_as_float(v1[2 * e + 1]) : 0.f;
                        wv[e] = pack_bf16x2(x0, x1);
                        wv[16 + e] = pack_bf16x2(y0, y1);
                    }
                }
                if (ntile >= 1 && !warp_wait(&p_free[wg], (ntile - 1) & 1, &abort_flag, err, kWaitPFree)) { ok = false; break; }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4 *>(prow + ((ch ^ (row & 7)) * 16)) =
                        make_uint4(wv[4 * ch], wv[4 * ch + 1], wv[4 * ch + 2], wv[4 * ch + 3]);
                fence_async_shared();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(l_p_full);
            }
            // ring items of this pair-item: Qt (2), nk Kt halves, nsp S_prev
            // halves, nk V halves, then the gate/output tile (2 slots)
            const int ig = it_base + 2 + 2 * m.nk + m.nsp;
            it_base = ig + 2;
            uint8_t *ya = slot_ptr(ig), *yb = slot_ptr(ig + 1);
            const bool go =
                ok && warp_wait(&o_full, li & 1, &abort_flag, err, kWaitOFullEpi) &&
                warp_wait(&lfull[ig % kPairSlots], (ig / kPairSlots) & 1, &abort_flag, err, kWaitLfullEpi) &&
                warp_wait(&lfull[(ig + 1) % kPairSlots], ((ig + 1) / kPairSlots) & 1, &abort_flag,
                          err, kWaitLfullEpi);
            float (*red)[kBlk] = reinterpret_cast<float (*)[kBlk]>(pbuf);   // [4][128]
            float mean = 0.f, rstd = 1.f;
            if (go) tc_fence_after();
            if (a.has_gate) {
                float sum = 0.f, sq = 0.f, shift = 0.f;
                if (go) {
                    uint32_t v0[32];
                    tmem_ld32(tO + lane_off, v0);
                    tmem_wait_ld();
                    shift = __uint_as_float(v0[0]);
#pragma unroll 1
                    for (int cb = 0; cb < 4; ++cb) {
                        uint32_t v[32];
                        tmem_ld32(tO + lane_off + 128 * wg + 32 * cb, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const float d = __uint_as_float(v[e]) - shift;
                            sum += d;
                            sq = fmaf(d, d, sq);
                        }
                    }
                }
                red[2 * wg][row] = sum;
                red[2 * wg + 1][row] = sq;
                named_barrier(1, kEpiThreads);
                const float ms = (red[0][row] + red[2][row]) * (1.f / kD);
                const float m2 = (red[1][row] + red[3][row]) * (1.f / kD);
                mean = shift + ms;
                rstd = rsqrtf(fmaxf(m2 - ms * ms, 0.f) + a.eps);
                named_barrier(1, kEpiThreads);
            }
            if (go) {
                const int sw = row & 7;
                const float *gw = a.gn_weight ? a.gn_weight + m.h * kD : nullptr;
                const float *gb = a.gn_bias ? a.gn_bias + m.h * kD : nullptr;
#pragma unroll 1
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int cb = 4 * wg + k4;
                    uint32_t v[32];
                    tmem_ld32(tO + lane_off + 32 * cb, v);
                    tmem_wait_ld();
                    if (k4 == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(l_o_free);
                    }
                    const int bx = cb >> 1;                       // 64-column box
                    uint8_t *box = (bx < 2 ? ya : yb) + (bx % 2) * kBox + row * 128;
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
                                    if (gw) yh *= gw[ch];
                                    if (gb) yh += gb[ch];
                                    y[e] = swish_fast(hh ? gg.y : gg.x) * yh;
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
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(l_o_free);
            }
            named_barrier(1, kEpiThreads);
            if (wg == 0 && row == 0) {
                if (!abort_flag && m.t0row < a.n) {           // rows past the sequence: nothing
                    for (int x = 0; x < 4; ++x)
                        tma_store_4d(&tm_out, (x < 2 ? ya : yb) + (x % 2) * kBox, 64 * x, m.h,
                                     m.t0row, m.b);
                    tma_store_commit();
                    tma_store_wait_read();
                }
                mbar_arrive(&rempty[ig % kPairSlots]);        // both slots may be refilled
                mbar_arrive(&rempty[(ig + 1) % kPairSlots]);
            }
            if (!go) ok = false;
        }
        if (!ok && lane == 0) abort_both();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                   // both CTAs' roles are done
    // After an abort in either CTA, wait (bounded) for everything still in
    // flight: the leader settles and drains the operand loads of both CTAs
    // (they count on its barriers) and its MMAs; each CTA its own gate loads.
    const bool aborted = abort_flag != 0;
    if (aborted && warp == 0 && lane == 0) {
        // each CTA: the latest armed lfull phase of every slot (gate tiles), and
        // the raw q halves
        for (int j = 0; j < kPairSlots; ++j)
            if (lf_n[j] > 0) mbar_drain(&lfull[j], (lf_n[j] - 1) & 1, err);
        for (int h2 = 0; h2 < 2; ++h2)
            if (q_n[h2] > 0) mbar_drain(&qfull[h2], (q_n[h2] - 1) & 1, err);
        if (leader) {
            // Each producer runs at most kPairSlots ring items past the MMAs,
            // so every slot has at most one operand phase still open, and the
            // two CTAs' operand counts of a slot differ by at most one.
            for (int j = 0; j < kPairSlots; ++j) {
                const uint32_t own = op_n[j];
                const uint32_t peer = ld_cluster_u32(mapa_shared(smem_u32(&op_n[j]), 1));
                if (own == 0 && peer == 0) continue;
                if (peer > own) mbar_expect_tx(&rfull[j], kPairSlot);       // only the peer loaded
                else if (own > peer) mbar_complete_tx(&rfull[j], kPairSlot); // only the leader
                mbar_drain(&rfull[j], ((own > peer ? own : peer) - 1) & 1, err);
            }
        }
    }
    if (aborted && warp == 1 && leader && lane == 0) {
        mma_commit_pair(&drain, 1);
        mbar_drain(&drain, 0, err);
    }
    tc_fence_before();
    cluster_sync();                                   // the pair's loads and MMAs have landed
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
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
bool make_tensor_map_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
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

// Chunk length the kernels compute with.  The chunkwise form's outputs and
// final state do not depend on the chunk length (every length gives the
// recurrence's result), so a chunk shorter than one 128-row tile is computed
// with 128-token chunks; longer chunks run as given.
static int effective_chunk(int chunk) { return chunk < kBlk ? kBlk : chunk; }

bool tc_shape_ok(int dk, int dv, retnet_dtype dtype, int chunk) {
    if (dk != kD || dv != kD || dtype != RETNET_BF16) return false;
    return (chunk >= 1 && chunk < kBlk) || chunk == 128 || chunk == 256 || chunk == 512 ||
           chunk == 1024;
}

bool tc_gammas_ok(int chunk, const float *gammas, int heads) {
    chunk = effective_chunk(chunk);
    for (int h = 0; h < heads; ++h) {
        const double g = gammas[h];
        if (!(g > 0.0)) return false;
        if (chunk * -std::log2(g) > 100.0) return false;
    }
    return true;
}

size_t tc_workspace_bytes(int batch, int heads, int seqlen, int chunk) {
    return tc_layout(batch, heads, seqlen, effective_chunk(chunk)).total;
}

void tc_operand_layout(int batch, int heads, int seqlen, int chunk, size_t *qt, size_t *kt,
                       int *fold) {
    const TcLayout l = tc_layout(batch, heads, seqlen, effective_chunk(chunk));
    *qt = l.qt;
    *kt = l.kt;
    *fold = effective_chunk(chunk);
}

// The parallel form runs the output pass over the whole sequence as one
// block of whole 128-row tiles.
static int parallel_span(int n) { return (n + kBlk - 1) / kBlk * kBlk; }

// d_v columns per state CTA (64, 128 or 256).  A state CTA streams its d_k
// half of Kt and its columns of V over the whole sequence, 2 (128 + DVC)
// bytes per token, one ring stage after another, so the pass takes about
// waves x (t0 + bytes per CTA / rate per CTA).  Measured on B200 over
// n = 128 .. 8192 (the pass alone, CUDA events): t0 about 10 us and
// 64-80 GB/s per CTA at every width.  So 16 sequence-heads take 64 columns
// (128 CTAs), 32 take 128 (128 CTAs), and 40 take 256 (80 CTAs, one wave:
// 36 us at n = 2048 against 43 us for two waves of 160 CTAs at 128).  The
// smallest estimate wins, the narrower width on a tie.
static int tc_state_columns(int seq_heads, int n, int sms) {
    int best = 64;
    double best_us = 0.0;
    for (int dvc = 64; dvc <= kD; dvc *= 2) {
        const long long ctas = (long long)seq_heads * 2 * (kD / dvc);
        const long long waves = (ctas + sms - 1) / sms;
        const double us = (double)waves * (10.0 + (double)n * 2.0 * (128 + dvc) / 70e3);
        if (dvc == 64 || us < best_us) {
            best = dvc;
            best_us = us;
        }
    }
    return best;
}

size_t tc_parallel_workspace_bytes(int batch, int heads, int seqlen) {
    return seqlen > 0 ? tc_layout(batch, heads, seqlen, parallel_span(seqlen)).total : 0;
}

cudaError_t launch_chunkwise_tc(const ChunkwiseArgs &a, const float *gammas, cudaStream_t stream,
                                bool parallel) {
    const int n = a.seqlen, H = a.heads, B = a.batch;
    // parallel form: one chunk spanning the sequence, decay folded per 128-row block
    const int C = parallel ? parallel_span(n) : effective_chunk(a.chunk);
    const int fold = parallel ? kBlk : C;
    const int BH = B * H;
    if (BH == 0 || (parallel && n == 0)) return cudaSuccess;
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

    // tensor maps: every tile is 128 rows (tokens, or d_k rows of S_prev) by
    // 64 channels, 128-byte swizzled
    CUtensorMap tm_q, tm_k, tm_v, tm_s;
    {
        cuuint64_t dims[3] = {kD, (cuuint64_t)n, (cuuint64_t)BH};
        cuuint64_t str[2] = {kD * 2, (cuuint64_t)n * kD * 2};
        cuuint32_t box[3] = {64, kBlk, 1};
        if (!make_tensor_map_bf16(&tm_k, kt, 3, dims, str, box) || !make_tensor_map_bf16(&tm_q, qt, 3, dims, str, box))
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[4] = {kD, (cuuint64_t)H, (cuuint64_t)n, (cuuint64_t)B};
        cuuint64_t str[3] = {kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)n * H * kD * 2};
        cuuint32_t box[4] = {64, 1, kBlk, 1};
        if (!make_tensor_map_bf16(&tm_v, a.v, 4, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {kD, (cuuint64_t)BH * nchunks * kD};
        cuuint64_t str[1] = {kD * 2};
        cuuint32_t box[2] = {64, kBlk};
        if (!make_tensor_map_bf16(&tm_s, sp, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    // output and gate tiles: 128 tokens x 64 channels of one head
    CUtensorMap tm_out, tm_g;
    {
        cuuint64_t dims[4] = {kD, (cuuint64_t)H, (cuuint64_t)n, (cuuint64_t)B};
        cuuint64_t str[3] = {kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)n * H * kD * 2};
        cuuint32_t box[4] = {64, 1, kBlk, 1};
        if (!make_tensor_map_bf16(&tm_out, a.out, 4, dims, str, box)) return cudaErrorInvalidValue;
        if (!make_tensor_map_bf16(&tm_g, a.gate ? a.gate->g : a.out, 4, dims, str, box))
            return cudaErrorInvalidValue;
    }

    cudaError_t e;
    // The output pass runs on CTA pairs for two or more row blocks per chunk
    // (a 128-token chunk would leave half of every pair idle); in mode 1 it
    // also folds q itself, and the prep pass writes only Kt.
    const int pair_mode = output_pairing_mode();
    const bool pairs = pair_mode != 0 && C / kBlk >= 2;
    const bool fold_q = pairs && pair_mode == 1 && !a.prefolded;
    double pp_theta[kD / 2];
    for (int j = 0; j < kD / 2; ++j) pp_theta[j] = std::pow(10000.0, -2.0 * j / kD);
    if (!a.prefolded) {
        TcPrepParams pp;
        for (int j = 0; j < kD / 2; ++j) pp.theta[j] = pp_theta[j];
        for (int h = 0; h < kMaxHeads; ++h) pp.log2g[h] = hp.log2g[h];
        // one warp per token, eight per CTA, at most eight CTAs per SM
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int blocks = std::max(1, std::min((n + 7) / 8, 8 * sms));
        KernelTimer timer("tc_prep", stream);
        const int wq = fold_q ? 0 : 1;
        e = launch_overlapped(tc_prep_kernel, dim3(blocks), dim3(256), 0, stream,
                              (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.k, pp, qt, kt,
                              B, H, n, fold, a.pos0, a.rotate, wq, err);
        count_launch();
        if (e != cudaSuccess) return e;
    }
    if (!parallel) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int dvc = tc_state_columns(BH, n, sms);
        // Kt and V as the state pass reads them: sub-tiles of 64 tokens at
        // 256 columns, else the 128-token tiles of the output pass
        CUtensorMap sk = tm_k, sv = tm_v;
        if (dvc == 256) {
            const cuuint32_t rows = (cuuint32_t)TcStateSmem<256>::kTok;
            cuuint64_t kdims[3] = {kD, (cuuint64_t)n, (cuuint64_t)BH};
            cuuint64_t kstr[2] = {kD * 2, (cuuint64_t)n * kD * 2};
            cuuint32_t kbox[3] = {64, rows, 1};
            cuuint64_t vdims[4] = {kD, (cuuint64_t)H, (cuuint64_t)n, (cuuint64_t)B};
            cuuint64_t vstr[3] = {kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)n * H * kD * 2};
            cuuint32_t vbox[4] = {64, 1, rows, 1};
            if (!make_tensor_map_bf16(&sk, kt, 3, kdims, kstr, kbox) ||
                !make_tensor_map_bf16(&sv, a.v, 4, vdims, vstr, vbox))
                return cudaErrorInvalidValue;
        }
        KernelTimer timer("tc_state", stream);
        auto launch = [&](auto kernel, int smem, int threads) -> cudaError_t {
            cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem);
            if (r != cudaSuccess) return r;
            return launch_overlapped(kernel, dim3(BH * 2 * (kD / dvc)), dim3(threads), smem, stream,
                                     sk, sv, hp, a.state_in, a.state_out, sp, H, n, C, nchunks, err);
        };
        if (dvc == 64)
            e = launch(tc_state_kernel<64>, (int)TcStateSmem<64>::kBytes, TcStateSmem<64>::kThreads);
        else if (dvc == 128)
            e = launch(tc_state_kernel<128>, (int)TcStateSmem<128>::kBytes,
                       TcStateSmem<128>::kThreads);
        else
            e = launch(tc_state_kernel<256>, (int)TcStateSmem<256>::kBytes,
                       TcStateSmem<256>::kThreads);
        count_launch();
        if (e != cudaSuccess) return e;
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
        oa.parallel = parallel ? 1 : 0;

        for (int h = 0; h < kMaxHeads; ++h) oa.log2g[h] = hp.log2g[h];
        oa.fold_q = fold_q ? 1 : 0;
        oa.fold = fold;
        oa.rotate = a.rotate;
        oa.pos0 = a.pos0;
        for (int j = 0; j < kD / 2; ++j) oa.theta[j] = pp_theta[j];
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        // CTA pairs serve chunks of two or more row blocks; a chunk of one
        // (128) would leave half of every pair idle.
        if (pairs) {
            oa.items = BH * nchunks * ((oa.rblocks + 1) / 2);
            CUtensorMap tm_qraw;                  // raw q, folded inside the output pass
            {
                cuuint64_t dims[4] = {kD, (cuuint64_t)H, (cuuint64_t)n, (cuuint64_t)B};
                cuuint64_t str[3] = {kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)n * H * kD * 2};
                cuuint32_t box[4] = {64, 1, kBlk, 1};
                if (!make_tensor_map_bf16(&tm_qraw, a.q, 4, dims, str, box))
                    return cudaErrorInvalidValue;
            }
            CUtensorMap tm_kh;                    // Kt in halves of 64 keys
            {
                cuuint64_t dims[3] = {kD, (cuuint64_t)n, (cuuint64_t)BH};
                cuuint64_t str[2] = {kD * 2, (cuuint64_t)n * kD * 2};
                cuuint32_t box[3] = {64, kKeyTile / 2, 1};
                if (!make_tensor_map_bf16(&tm_kh, kt, 3, dims, str, box))
                    return cudaErrorInvalidValue;
            }
            const int smem = (int)TcPairSmem::kBytes;
            e = cudaFuncSetAttribute(tc_output_pair_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            // as many pairs as fit on the GPU at once (whole clusters per GPC)
            cudaLaunchConfig_t qc = {};
            qc.gridDim = dim3(2 * (unsigned)std::max(1, sms / 2));
            qc.blockDim = dim3(kPairThreads);
            qc.dynamicSmemBytes = smem;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, tc_output_pair_kernel, &qc) !=
                    cudaSuccess ||
                clusters < 1)
                clusters = std::max(1, sms / 2);
            clusters = std::min(clusters, oa.items);
            KernelTimer timer("tc_output", stream);
            e = launch_overlapped(tc_output_pair_kernel, dim3(2 * clusters), dim3(kPairThreads),
                                  smem, stream, tm_q, tm_kh, tm_v, tm_s, tm_g, tm_out, tm_qraw,
                                  oa);
            count_launch();
            if (e != cudaSuccess) return e;
        } else {
            oa.items = BH * nchunks * oa.rblocks;
            const int smem = (int)TcOutSmem::kBytes;
            // The parallel form deals its items in decreasing key-tile count
            // (tc_item): its row blocks cost 1 .. n/128 tiles, and the plain
            // stride left the busiest CTA 1.3-1.7x the average.  Measured on
            // B200: 142 -> 104 us at B=8, H=4, n=2048; 538 -> 460 us at B=1,
            // H=16, n=8192.
            auto kernel = parallel ? tc_output_kernel<true> : tc_output_kernel<false>;
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            const unsigned grid = (unsigned)std::min(oa.items, sms);
            KernelTimer timer("tc_output", stream);
            e = launch_overlapped(kernel, dim3(grid), dim3(kOutThreads), smem, stream,
                                  tm_q, tm_k, tm_v, tm_s, tm_g, tm_out, oa);
            count_launch();
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace retnet

#ifdef RETNET_TEST_HOOKS
// Debug build only: lowers the wall-time limit of the pipeline waits in this
// file's kernels, and makes the state pass's first CTA skip its first load.
extern "C" RETNET_API retnet_status retnet_test_set_hooks(unsigned long long wait_limit_ns,
                                                          int skip_first_state_load) {
    if (wait_limit_ns == 0 || (skip_first_state_load != 0 && skip_first_state_load != 1))
        return RETNET_ERR_INVALID_ARG;
    if (cudaMemcpyToSymbol(retnet::sm100::g_hook_wait_limit_ns, &wait_limit_ns,
                           sizeof(wait_limit_ns)) != cudaSuccess ||
        cudaMemcpyToSymbol(retnet::g_hook_skip_first_load, &skip_first_state_load,
                           sizeof(int)) != cudaSuccess)
        return RETNET_ERR_CUDA;
    return RETNET_OK;
}
#endif
