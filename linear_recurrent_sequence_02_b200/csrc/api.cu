// C ABI entry points: host-side validation, then dispatch to the kernels.
//
// Every check runs before anything is enqueued, so a rejected call leaves
// all buffers untouched and launches nothing.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "kernels.h"

namespace retnet {

static std::atomic<unsigned long long> g_launches{0};
void count_launch(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

static std::atomic<bool> g_overlap{true};
bool launch_overlap_enabled() { return g_overlap.load(std::memory_order_relaxed); }

static std::atomic<int> g_pairs{0};
int output_pairing_mode() { return g_pairs.load(std::memory_order_relaxed); }

__device__ unsigned g_device_error = 0u;

void *current_context() {
    typedef int (*CtxGetCurrentFn)(void **);
    static CtxGetCurrentFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (CtxGetCurrentFn) nullptr;
        return (CtxGetCurrentFn)p;
    }();
    void *ctx = nullptr;
    if (!fn || fn(&ctx) != 0) return nullptr;
    return ctx;
}

static SymbolAddressCache g_error_word_cache;

unsigned *device_error_word() {
    void *p = nullptr;
    if (g_error_word_cache.get(g_device_error, &p) != cudaSuccess) return nullptr;
    return (unsigned *)p;
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
// Block length of the parallel form's decay fold (one 128-row tile).
constexpr int kParallelFoldBlock = 128;
static bool head_dim_ok(int d) { return d == 64 || d == 128 || d == 256; }
static bool dtype_ok(retnet_dtype t) { return t == RETNET_F32 || t == RETNET_BF16; }
static size_t elem_size(retnet_dtype t) { return t == RETNET_BF16 ? 2 : 4; }

static retnet_status load_gammas(const float *gammas, int heads, HeadGammas *out) {
    if (!gammas || heads < 1 || heads > kMaxHeads) return RETNET_ERR_INVALID_ARG;
    for (int h = 0; h < kMaxHeads; ++h) out->g[h] = 0.f;
    for (int h = 0; h < heads; ++h) {
        float g = gammas[h];
        if (!(g >= 0.f && g <= 1.f)) return RETNET_ERR_INVALID_ARG;   // also rejects NaN
        out->g[h] = g;
    }
    return RETNET_OK;
}

static retnet_status check_shape(const retnet_shape *s, int chunk) {
    if (!s) return RETNET_ERR_INVALID_ARG;
    if (s->batch < 0 || s->seqlen < 0 || s->heads < 1 || s->heads > kMaxHeads)
        return RETNET_ERR_INVALID_ARG;
    if (!dtype_ok(s->dtype)) return RETNET_ERR_INVALID_ARG;
    if (chunk < 1 || chunk > 1024) return RETNET_ERR_INVALID_ARG;
    if (s->dk <= 0 || s->dv <= 0) return RETNET_ERR_INVALID_ARG;
    if (!head_dim_ok(s->dk) || !head_dim_ok(s->dv)) return RETNET_ERR_UNSUPPORTED;
    return RETNET_OK;
}

// Kernel family for a call; gammas == nullptr answers for any admissible decay.
static retnet_algo resolve_algo(const retnet_shape *s, int chunk, retnet_algo algo,
                                const float *gammas) {
    const bool shape_ok = tc_shape_ok(s->dk, s->dv, s->dtype, chunk);
    const bool gam_ok = !gammas || tc_gammas_ok(chunk, gammas, s->heads);
    if (algo == RETNET_ALGO_AUTO) return shape_ok && gam_ok ? RETNET_ALGO_TENSOR : RETNET_ALGO_SIMT;
    return algo;
}

static size_t workspace_for(const retnet_shape *s, int chunk, retnet_algo resolved) {
    if (resolved == RETNET_ALGO_TENSOR) return tc_workspace_bytes(s->batch, s->heads, s->seqlen, chunk);
    return simt_workspace_bytes(s->batch, s->heads, s->seqlen, s->dk, s->dv, chunk);
}

// Backward pass layout of the caller's workspace: five [B, n, H, d] buffers
// (rotated k; reversed v, dO, rotated q, rotated k), then the workspace of
// the forward calls it makes.
struct BackwardLayout {
    size_t kh, rv, rdo, rqh, rkh, fwd, fwd_bytes, total;
};
static size_t align1k(size_t x) { return (x + 1023) & ~(size_t)1023; }
// the forward call shapes: (q, k in dv, values in dk) and (q, k in dk, values in dv)
static retnet_shape backward_shape_a(const retnet_shape *s) {
    retnet_shape t = *s;
    t.dk = s->dv;
    t.dv = s->dk;
    return t;
}
// Forward workspace for either call shape; gammas == nullptr takes the
// larger of the two kernel families where AUTO could pick either.
static size_t backward_fwd_bytes(const retnet_shape *s, int chunk, retnet_algo algo,
                                 const float *gammas) {
    size_t n = 0;
    const retnet_shape shapes[2] = {backward_shape_a(s), *s};
    for (const retnet_shape &t : shapes) {
        size_t m;
        if (gammas) {
            m = workspace_for(&t, chunk, resolve_algo(&t, chunk, algo, gammas));
        } else {
            m = workspace_for(&t, chunk, RETNET_ALGO_SIMT);
            if (resolve_algo(&t, chunk, algo, nullptr) == RETNET_ALGO_TENSOR) {
                const size_t tc = workspace_for(&t, chunk, RETNET_ALGO_TENSOR);
                m = algo == RETNET_ALGO_TENSOR ? tc : (tc > m ? tc : m);
            }
        }
        n = m > n ? m : n;
    }
    return n;
}
static BackwardLayout backward_layout(const retnet_shape *s, int chunk, retnet_algo algo,
                                      const float *gammas) {
    const size_t es = elem_size(s->dtype);
    const size_t rows = (size_t)s->batch * s->seqlen * s->heads;
    const size_t bk = align1k(rows * s->dk * es), bv = align1k(rows * s->dv * es);
    BackwardLayout l;
    l.kh = 0;
    l.rv = l.kh + bk;
    l.rdo = l.rv + bv;
    l.rqh = l.rdo + bv;
    l.rkh = l.rqh + bk;
    l.fwd = l.rkh + bk;
    l.fwd_bytes = backward_fwd_bytes(s, chunk, algo, gammas);
    l.total = l.fwd + l.fwd_bytes;
    return l;
}

// The tensor-core backward whose retentions run without their prep pass
// (bf16, d_k = d_v = 256): the three retentions' values and the outputs of
// the two reversed-time ones, then one prefill workspace per retention,
// whose Qt and Kt the fold kernel fills.
struct FusedBackwardLayout {
    size_t val[3], out2, out3, fwd[3], fwd_bytes, total;
};
static bool backward_fusable(const retnet_shape *s, int chunk, retnet_algo algo) {
    return algo != RETNET_ALGO_SIMT && s->dtype == RETNET_BF16 && s->dk == 256 && s->dv == 256 &&
           tc_shape_ok(s->dk, s->dv, s->dtype, chunk);
}
static FusedBackwardLayout fused_backward_layout(const retnet_shape *s, int chunk) {
    const size_t b = align1k((size_t)s->batch * s->seqlen * s->heads * 256 * 2);
    FusedBackwardLayout l;
    size_t at = 0;
    for (int i = 0; i < 3; ++i, at += b) l.val[i] = at;
    l.out2 = at;
    l.out3 = at + b;
    at += 2 * b;
    l.fwd_bytes = align1k(tc_workspace_bytes(s->batch, s->heads, s->seqlen, chunk));
    for (int i = 0; i < 3; ++i, at += l.fwd_bytes) l.fwd[i] = at;
    l.total = at;
    return l;
}

}  // namespace retnet

using namespace retnet;

extern "C" {

const char *retnet_status_string(retnet_status status) {
    switch (status) {
        case RETNET_OK: return "ok";
        case RETNET_ERR_INVALID_ARG: return "invalid argument";
        case RETNET_ERR_UNSUPPORTED: return "unsupported shape or option";
        case RETNET_ERR_CUDA: return "CUDA error";
        case RETNET_ERR_TIMEOUT: return "device-side wait timed out";
        case RETNET_ERR_WORKSPACE: return "workspace missing or too small";
        case RETNET_ERR_BOUNDS: return "device-side index check failed (debug build)";
    }
    return "unknown status";
}

unsigned long long retnet_kernel_launch_count(void) {
    return g_launches.load(std::memory_order_relaxed);
}

retnet_status retnet_set_launch_overlap(int enable) {
    if (enable != 0 && enable != 1) return RETNET_ERR_INVALID_ARG;
    g_overlap.store(enable == 1, std::memory_order_relaxed);
    return RETNET_OK;
}

retnet_status retnet_set_output_pairing(int mode) {
    if (mode < 0 || mode > 2) return RETNET_ERR_INVALID_ARG;
    g_pairs.store(mode, std::memory_order_relaxed);
    return RETNET_OK;
}

retnet_status retnet_default_gammas(int heads, float *gammas) {
    if (!gammas || heads < 1 || heads > kMaxHeads) return RETNET_ERR_INVALID_ARG;
    for (int h = 0; h < heads; ++h) gammas[h] = (float)(1.0 - std::ldexp(1.0, -5 - h));
    return RETNET_OK;
}

retnet_status retnet_xpos_rotate(const void *x, void *y, int batch, int seqlen, int heads, int d,
                                 retnet_dtype dtype, long long pos0, retnet_stream_t stream) {
    if (batch < 0 || seqlen < 0 || heads < 1 || pos0 < 0 || !dtype_ok(dtype))
        return RETNET_ERR_INVALID_ARG;
    if (d <= 0 || d % 8 != 0 || d > 1024) return RETNET_ERR_INVALID_ARG;
    if ((long long)batch * seqlen == 0) return RETNET_OK;
    if (!x || !y || !aligned16(x) || !aligned16(y)) return RETNET_ERR_INVALID_ARG;
    RETNET_CUDA_TRY(launch_xpos_rotate(x, y, (long long)batch * seqlen, heads, d, dtype, seqlen,
                                       pos0, (cudaStream_t)stream));
    return RETNET_OK;
}

retnet_status retnet_chunkwise_workspace_size(const retnet_shape *shape, int chunk,
                                              retnet_algo algo, size_t *bytes) {
    if (!bytes) return RETNET_ERR_INVALID_ARG;
    retnet_status st = check_shape(shape, chunk);
    if (st != RETNET_OK) return st;
    if (algo != RETNET_ALGO_AUTO && algo != RETNET_ALGO_SIMT && algo != RETNET_ALGO_TENSOR)
        return RETNET_ERR_INVALID_ARG;
    if (algo == RETNET_ALGO_TENSOR && !tc_shape_ok(shape->dk, shape->dv, shape->dtype, chunk))
        return RETNET_ERR_UNSUPPORTED;
    size_t n = workspace_for(shape, chunk, RETNET_ALGO_SIMT);
    if (resolve_algo(shape, chunk, algo, nullptr) == RETNET_ALGO_TENSOR) {
        // AUTO may still pick SIMT at call time (decays outside the fold's range)
        size_t t = workspace_for(shape, chunk, RETNET_ALGO_TENSOR);
        n = algo == RETNET_ALGO_TENSOR ? t : (t > n ? t : n);
    }
    *bytes = n;
    return RETNET_OK;
}

retnet_status retnet_retention_chunkwise(const void *q, const void *k, const void *v,
                                         const float *gammas, int chunk, void *out,
                                         const retnet_shape *shape, long long pos0, int rotate,
                                         const float *state_in, float *state_out,
                                         const retnet_gate *gate, retnet_algo algo,
                                         void *workspace, size_t workspace_bytes,
                                         retnet_stream_t stream) {
    retnet_status st = check_shape(shape, chunk);
    if (st != RETNET_OK) return st;
    if (pos0 < 0 || (rotate != 0 && rotate != 1)) return RETNET_ERR_INVALID_ARG;
    if (algo != RETNET_ALGO_AUTO && algo != RETNET_ALGO_SIMT && algo != RETNET_ALGO_TENSOR)
        return RETNET_ERR_INVALID_ARG;
    ChunkwiseArgs a;
    st = load_gammas(gammas, shape->heads, &a.gam);
    if (st != RETNET_OK) return st;
    const long long tokens = (long long)shape->batch * shape->seqlen;
    if (tokens > 0) {
        if (!q || !k || !v || !out) return RETNET_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
            return RETNET_ERR_INVALID_ARG;
    }
    if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
        return RETNET_ERR_INVALID_ARG;
    if (gate) {
        if (tokens > 0 && (!gate->g || !aligned16(gate->g))) return RETNET_ERR_INVALID_ARG;
        if (!(gate->eps >= 0.f)) return RETNET_ERR_INVALID_ARG;
    }
    retnet_algo resolved = resolve_algo(shape, chunk, algo, gammas);
    if (resolved == RETNET_ALGO_TENSOR &&
        (!tc_shape_ok(shape->dk, shape->dv, shape->dtype, chunk) ||
         !tc_gammas_ok(chunk, gammas, shape->heads)))
        return RETNET_ERR_UNSUPPORTED;
    size_t need = workspace_for(shape, chunk, resolved);
    if (need > 0 && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)))
        return RETNET_ERR_WORKSPACE;
    if (shape->batch == 0) return RETNET_OK;

    a.q = q; a.k = k; a.v = v; a.out = out;
    a.state_in = state_in; a.state_out = state_out; a.gate = gate;
    a.batch = shape->batch; a.heads = shape->heads; a.seqlen = shape->seqlen;
    a.dk = shape->dk; a.dv = shape->dv; a.chunk = chunk; a.dtype = shape->dtype;
    a.pos0 = pos0; a.rotate = rotate; a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    if (resolved == RETNET_ALGO_TENSOR) {
        if ((uintptr_t)workspace & 1023u) return RETNET_ERR_WORKSPACE;
        RETNET_CUDA_TRY(launch_chunkwise_tc(a, gammas, (cudaStream_t)stream));
    } else {
        RETNET_CUDA_TRY(launch_chunkwise_simt(a, (cudaStream_t)stream));
    }
    return RETNET_OK;
}

retnet_status retnet_parallel_workspace_size(const retnet_shape *shape, size_t *bytes) {
    if (!bytes) return RETNET_ERR_INVALID_ARG;
    retnet_status st = check_shape(shape, kParallelFoldBlock);
    if (st != RETNET_OK) return st;
    if (!tc_shape_ok(shape->dk, shape->dv, shape->dtype, kParallelFoldBlock))
        return RETNET_ERR_UNSUPPORTED;
    *bytes = tc_parallel_workspace_bytes(shape->batch, shape->heads, shape->seqlen);
    return RETNET_OK;
}

retnet_status retnet_retention_parallel(const void *q, const void *k, const void *v,
                                        const float *gammas, void *out,
                                        const retnet_shape *shape, long long pos0, int rotate,
                                        const retnet_gate *gate, void *workspace,
                                        size_t workspace_bytes, retnet_stream_t stream) {
    retnet_status st = check_shape(shape, kParallelFoldBlock);
    if (st != RETNET_OK) return st;
    if (pos0 < 0 || (rotate != 0 && rotate != 1)) return RETNET_ERR_INVALID_ARG;
    ChunkwiseArgs a;
    st = load_gammas(gammas, shape->heads, &a.gam);
    if (st != RETNET_OK) return st;
    const long long tokens = (long long)shape->batch * shape->seqlen;
    if (tokens > 0) {
        if (!q || !k || !v || !out) return RETNET_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
            return RETNET_ERR_INVALID_ARG;
    }
    if (gate) {
        if (tokens > 0 && (!gate->g || !aligned16(gate->g))) return RETNET_ERR_INVALID_ARG;
        if (!(gate->eps >= 0.f)) return RETNET_ERR_INVALID_ARG;
    }
    if (!tc_shape_ok(shape->dk, shape->dv, shape->dtype, kParallelFoldBlock) ||
        !tc_gammas_ok(kParallelFoldBlock, gammas, shape->heads))
        return RETNET_ERR_UNSUPPORTED;
    const size_t need = tc_parallel_workspace_bytes(shape->batch, shape->heads, shape->seqlen);
    if (need > 0 && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 1023u)))
        return RETNET_ERR_WORKSPACE;
    if (tokens == 0) return RETNET_OK;
    a.q = q; a.k = k; a.v = v; a.out = out;
    a.state_in = nullptr; a.state_out = nullptr; a.gate = gate;
    a.batch = shape->batch; a.heads = shape->heads; a.seqlen = shape->seqlen;
    a.dk = shape->dk; a.dv = shape->dv; a.chunk = kParallelFoldBlock; a.dtype = shape->dtype;
    a.pos0 = pos0; a.rotate = rotate; a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    RETNET_CUDA_TRY(launch_chunkwise_tc(a, gammas, (cudaStream_t)stream, true));
    return RETNET_OK;
}

retnet_status retnet_backward_workspace_size(const retnet_shape *shape, int chunk,
                                             retnet_algo algo, size_t *bytes) {
    if (!bytes) return RETNET_ERR_INVALID_ARG;
    retnet_status st = check_shape(shape, chunk);
    if (st != RETNET_OK) return st;
    if (algo != RETNET_ALGO_AUTO && algo != RETNET_ALGO_SIMT && algo != RETNET_ALGO_TENSOR)
        return RETNET_ERR_INVALID_ARG;
    if (algo == RETNET_ALGO_TENSOR && !tc_shape_ok(shape->dk, shape->dv, shape->dtype, chunk))
        return RETNET_ERR_UNSUPPORTED;
    size_t need = 0;
    if ((long long)shape->batch * shape->seqlen > 0) {
        need = backward_layout(shape, chunk, algo, nullptr).total;
        if (backward_fusable(shape, chunk, algo))      // whichever the decays select
            need = std::max(need, fused_backward_layout(shape, chunk).total);
    }
    *bytes = need;
    return RETNET_OK;
}

retnet_status retnet_retention_backward(const void *q, const void *k, const void *v,
                                        const void *d_out, const float *gammas, int chunk,
                                        void *dq, void *dk, void *dv, const retnet_shape *shape,
                                        long long pos0, int rotate, retnet_algo algo,
                                        void *workspace, size_t workspace_bytes,
                                        retnet_stream_t stream) {
    retnet_status st = check_shape(shape, chunk);
    if (st != RETNET_OK) return st;
    if (pos0 < 0 || (rotate != 0 && rotate != 1)) return RETNET_ERR_INVALID_ARG;
    if (algo != RETNET_ALGO_AUTO && algo != RETNET_ALGO_SIMT && algo != RETNET_ALGO_TENSOR)
        return RETNET_ERR_INVALID_ARG;
    ChunkwiseArgs base;
    st = load_gammas(gammas, shape->heads, &base.gam);
    if (st != RETNET_OK) return st;
    const long long tokens = (long long)shape->batch * shape->seqlen;
    if (tokens > 0) {
        const void *ptrs[7] = {q, k, v, d_out, dq, dk, dv};
        for (const void *p : ptrs)
            if (!p || !aligned16(p)) return RETNET_ERR_INVALID_ARG;
    }
    const retnet_shape sa = backward_shape_a(shape);
    const retnet_algo ra = resolve_algo(&sa, chunk, algo, gammas);
    const retnet_algo rb = resolve_algo(shape, chunk, algo, gammas);
    for (int x = 0; x < 2; ++x) {
        const retnet_shape &t = x ? *shape : sa;
        if ((x ? rb : ra) == RETNET_ALGO_TENSOR &&
            (!tc_shape_ok(t.dk, t.dv, t.dtype, chunk) || !tc_gammas_ok(chunk, gammas, t.heads)))
            return RETNET_ERR_UNSUPPORTED;
    }
    if (tokens == 0) return RETNET_OK;
    const bool fused = ra == RETNET_ALGO_TENSOR && rb == RETNET_ALGO_TENSOR &&
                       backward_fusable(shape, chunk, algo);
    const BackwardLayout lay = backward_layout(shape, chunk, algo, gammas);
    const size_t need = fused ? fused_backward_layout(shape, chunk).total : lay.total;
    if (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 1023u))
        return RETNET_ERR_WORKSPACE;

    const cudaStream_t s = (cudaStream_t)stream;
    if (fused) {
        // the fold kernel writes every retention's operands; the retentions
        // then run from their Qt, Kt without a prep pass
        const FusedBackwardLayout fl = fused_backward_layout(shape, chunk);
        char *ws = (char *)workspace;
        size_t qt_off = 0, kt_off = 0;
        int fold = 0;
        tc_operand_layout(shape->batch, shape->heads, shape->seqlen, chunk, &qt_off, &kt_off,
                          &fold);
        void *qt[3], *kt[3], *vals[3];
        for (int i = 0; i < 3; ++i) {
            qt[i] = ws + fl.fwd[i] + qt_off;
            kt[i] = ws + fl.fwd[i] + kt_off;
            vals[i] = ws + fl.val[i];
        }
        RETNET_CUDA_TRY(launch_backward_fold(q, k, v, d_out, qt, kt, vals, gammas,
                                             shape->batch, shape->heads, shape->seqlen, fold,
                                             pos0, rotate, s));
        void *outs[3] = {dq, ws + fl.out2, ws + fl.out3};
        for (int i = 0; i < 3; ++i) {
            ChunkwiseArgs a = base;
            a.q = nullptr; a.k = nullptr; a.v = vals[i]; a.out = outs[i];
            a.state_in = nullptr; a.state_out = nullptr; a.gate = nullptr;
            a.batch = shape->batch; a.heads = shape->heads; a.seqlen = shape->seqlen;
            a.dk = 256; a.dv = 256; a.chunk = chunk; a.dtype = shape->dtype;
            a.pos0 = 0; a.rotate = 0;
            a.workspace = ws + fl.fwd[i];
            a.workspace_bytes = fl.fwd_bytes;
            a.prefolded = true;
            RETNET_CUDA_TRY(launch_chunkwise_tc(a, gammas, s));
        }
        RETNET_CUDA_TRY(launch_backward_post(dq, ws + fl.out2, ws + fl.out3, dk, dv, shape->batch,
                                             shape->heads, shape->seqlen, 256, 256,
                                             shape->dtype, pos0, rotate, s));
        return RETNET_OK;
    }
    const int B = shape->batch, n = shape->seqlen, H = shape->heads;
    const int DK = shape->dk, DV = shape->dv;
    const retnet_dtype dt = shape->dtype;
    char *ws = (char *)workspace;
    void *kh = ws + lay.kh, *rv = ws + lay.rv, *rdo = ws + lay.rdo, *rqh = ws + lay.rqh,
         *rkh = ws + lay.rkh;
    // rotated k; the reversed sequences of v, dO, rotated q and rotated k
    RETNET_CUDA_TRY(launch_backward_prep(q, k, v, d_out, kh, rkh, rqh, rv, rdo, B, H, n, DK, DV,
                                         dt, pos0, rotate, s));

    // three forward retentions without rotation, state or epilogue
    base.state_in = nullptr;
    base.state_out = nullptr;
    base.gate = nullptr;
    base.batch = B; base.heads = H; base.seqlen = n; base.chunk = chunk; base.dtype = dt;
    base.pos0 = 0; base.rotate = 0;
    base.workspace = ws + lay.fwd;
    base.workspace_bytes = lay.fwd_bytes;
    auto forward = [&](const retnet_shape &t, retnet_algo r, const void *fq, const void *fk,
                       const void *fv, void *fo) -> cudaError_t {
        ChunkwiseArgs a = base;
        a.q = fq; a.k = fk; a.v = fv; a.out = fo;
        a.dk = t.dk; a.dv = t.dv;
        return r == RETNET_ALGO_TENSOR ? launch_chunkwise_tc(a, gammas, s)
                                       : launch_chunkwise_simt(a, s);
    };
    // dQ^ = causal retention of (dO, V, K^)            -> dq (rotated frame)
    RETNET_CUDA_TRY(forward(sa, ra, d_out, v, kh, dq));
    // rev(dK^) = causal retention of rev(V, dO, Q^)     -> the k^ buffer
    RETNET_CUDA_TRY(forward(sa, ra, rv, rdo, rqh, kh));
    // rev(dV) = causal retention of rev(K^, Q^, dO)     -> the rev(v) buffer
    RETNET_CUDA_TRY(forward(*shape, rb, rkh, rqh, rdo, rv));
    // back to the caller's frame and time order
    RETNET_CUDA_TRY(launch_backward_post(dq, kh, rv, dk, dv, B, H, n, DK, DV, dt, pos0, rotate,
                                         s));
    return RETNET_OK;
}

retnet_status retnet_retention_step(const void *q, const void *k, const void *v,
                                    const float *gammas, float *state, void *out, int batch,
                                    int heads, int dk, int dv, retnet_dtype dtype, long long pos,
                                    int rotate, retnet_stream_t stream) {
    if (batch < 0 || heads < 1 || heads > kMaxHeads || !dtype_ok(dtype) || pos < 0 ||
        (rotate != 0 && rotate != 1))
        return RETNET_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0) return RETNET_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return RETNET_ERR_UNSUPPORTED;
    HeadGammas gam;
    retnet_status st = load_gammas(gammas, heads, &gam);
    if (st != RETNET_OK) return st;
    if (batch == 0) return RETNET_OK;
    if (!q || !k || !v || !state || !out) return RETNET_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out))
        return RETNET_ERR_INVALID_ARG;
    RETNET_CUDA_TRY(launch_retention_recurrent(q, k, v, gam, state, out, batch, 1, heads, dk, dv,
                                               dtype, pos, rotate, (cudaStream_t)stream));
    return RETNET_OK;
}

retnet_status retnet_retention_recurrent(const void *q, const void *k, const void *v,
                                         const float *gammas, float *state, void *out,
                                         const retnet_shape *shape, long long pos0, int rotate,
                                         retnet_stream_t stream) {
    if (!shape || shape->batch < 0 || shape->seqlen < 0 || shape->heads < 1 ||
        shape->heads > kMaxHeads || !dtype_ok(shape->dtype) || pos0 < 0 ||
        (rotate != 0 && rotate != 1))
        return RETNET_ERR_INVALID_ARG;
    if (shape->dk <= 0 || shape->dv <= 0) return RETNET_ERR_INVALID_ARG;
    if (!head_dim_ok(shape->dk) || !head_dim_ok(shape->dv)) return RETNET_ERR_UNSUPPORTED;
    HeadGammas gam;
    retnet_status st = load_gammas(gammas, shape->heads, &gam);
    if (st != RETNET_OK) return st;
    if ((long long)shape->batch * shape->seqlen == 0) return RETNET_OK;
    if (!q || !k || !v || !state || !out) return RETNET_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out))
        return RETNET_ERR_INVALID_ARG;
    RETNET_CUDA_TRY(launch_retention_recurrent(q, k, v, gam, state, out, shape->batch,
                                               shape->seqlen, shape->heads, shape->dk, shape->dv,
                                               shape->dtype, pos0, rotate,
                                               (cudaStream_t)stream));
    return RETNET_OK;
}

retnet_status retnet_groupnorm_swish(const void *o, const void *g, const float *weight,
                                     const float *bias, float eps, long long rows, int heads,
                                     int dv, retnet_dtype dtype, void *y,
                                     retnet_stream_t stream) {
    if (rows < 0 || heads < 1 || !dtype_ok(dtype) || !(eps >= 0.f)) return RETNET_ERR_INVALID_ARG;
    if (dv <= 0 || dv % 8 != 0 || dv > 1024) return RETNET_ERR_INVALID_ARG;
    if (rows == 0) return RETNET_OK;
    if (!o || !g || !y || !aligned16(o) || !aligned16(g) || !aligned16(y))
        return RETNET_ERR_INVALID_ARG;
    RETNET_CUDA_TRY(launch_groupnorm_swish(o, g, weight, bias, eps, rows, heads, dv, dtype, y,
                                           (cudaStream_t)stream));
    return RETNET_OK;
}

#ifdef RETNET_TEST_HOOKS
// Debug build only: synchronises `stream`, returns the raw device error word
// (timeout and bounds bits, with the kSite* bits of the kernels whose index
// checks failed) in *word and clears it.
RETNET_API retnet_status retnet_test_error_word(retnet_stream_t stream, unsigned *word) {
    if (!word) return RETNET_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RETNET_ERR_CUDA;
    unsigned zero = 0;
    if (cudaMemcpyFromSymbol(word, g_device_error, sizeof(*word)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return RETNET_ERR_CUDA;
    return RETNET_OK;
}
#endif

retnet_status retnet_check_device_errors(retnet_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RETNET_ERR_CUDA;
    unsigned word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess)
        return RETNET_ERR_CUDA;
    if (word == 0) return RETNET_OK;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return RETNET_ERR_CUDA;
    if (word & kDevErrTimeout) return RETNET_ERR_TIMEOUT;
    return (word & kDevErrBounds) ? RETNET_ERR_BOUNDS : RETNET_ERR_CUDA;
}

}  // extern "C"
