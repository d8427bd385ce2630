// The multi-scale retention (MSR) layer around the retention operator, and
// the plain projection it is built from.
//
// Retention replaces multi-head attention, with a swish gate and GroupNorm
// added on its output (RetNet research summary, "Summary"; "Key points":
// the 200M model's hidden size 1024, head dimension 256).  For an input X
// [B*n, hidden]:
//     Q, K, V, G = X W_Q^T, X W_K^T, X W_V^T, X W_G^T      (one fused GEMM)
//     Y = swish(G) (.) GroupNorm_h(retention(R Q, R K, V))  (chunkwise prefill)
//     out = Y W_O^T                                         (second GEMM)
// with the rotation R, the per-head decays and the GroupNorm of
// retnet_retention_chunkwise.  Weights use the [out_features, in_features]
// layout of a linear layer.
//
// When the retention runs on the tensor cores, the projection GEMM's
// epilogue also applies R and the decay fold to Q and K and writes them as
// the prefill's Qt, Kt operands, so the prefill starts at its state pass:
// Q and K never go through HBM unfolded.
#include <cmath>

#include "kernels.h"

namespace retnet {
namespace {

size_t align1k(size_t x) { return (x + 1023) & ~(size_t)1023; }

// Workspace of the layer: Q, K, V, G and the retention output Y, each
// [B*n, H*d] bf16, the prefill's own workspace, then the rotation table
// [n, 128] (cos, sin) pairs that the projection's epilogue reads.
struct MsrLayout {
    size_t q, k, v, g, y, fwd, fwd_bytes, table, total;
};

retnet_status msr_layout(const retnet_shape *s, int hidden, int chunk, MsrLayout *l) {
    if (!s || s->batch < 0 || s->seqlen < 0 || s->heads < 1 || s->heads > kMaxHeads)
        return RETNET_ERR_INVALID_ARG;
    if (s->dtype != RETNET_BF16 || s->dk != s->dv) return RETNET_ERR_UNSUPPORTED;
    const long long rows = (long long)s->batch * s->seqlen;
    const int hd = s->heads * s->dk;
    if (hidden <= 0 || !gemm_shape_ok(rows, 4 * hd, hidden, hd) ||
        !gemm_shape_ok(rows, hidden, hd, hidden))
        return RETNET_ERR_UNSUPPORTED;
    size_t fwd = 0;
    retnet_status st = retnet_chunkwise_workspace_size(s, chunk, RETNET_ALGO_AUTO, &fwd);
    if (st != RETNET_OK) return st;
    const size_t part = align1k((size_t)rows * hd * 2);
    l->q = 0;
    l->k = l->q + part;
    l->v = l->k + part;
    l->g = l->v + part;
    l->y = l->g + part;
    l->fwd = l->y + part;
    l->fwd_bytes = fwd;
    l->table = l->fwd + align1k(fwd);
    l->total = l->table + align1k((size_t)s->seqlen * 128 * sizeof(float2));
    return RETNET_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace retnet

using namespace retnet;

extern "C" {

retnet_status retnet_linear(const void *x, const void *w, void *y, long long rows,
                            int in_features, int out_features, retnet_stream_t stream) {
    if (rows < 0 || in_features <= 0 || out_features <= 0) return RETNET_ERR_INVALID_ARG;
    if (!gemm_shape_ok(rows, out_features, in_features, out_features))
        return RETNET_ERR_UNSUPPORTED;
    if (rows == 0) return RETNET_OK;
    if (!x || !w || !y || !aligned16(x) || !aligned16(w) || !aligned16(y))
        return RETNET_ERR_INVALID_ARG;
    void *outs[1] = {y};
    RETNET_CUDA_TRY(launch_gemm_bf16(x, w, outs, rows, out_features, in_features, out_features,
                                     (cudaStream_t)stream));
    return RETNET_OK;
}

retnet_status retnet_msr_workspace_size(const retnet_shape *shape, int hidden, int chunk,
                                        size_t *bytes) {
    if (!bytes) return RETNET_ERR_INVALID_ARG;
    MsrLayout l;
    retnet_status st = msr_layout(shape, hidden, chunk, &l);
    if (st != RETNET_OK) return st;
    *bytes = l.total;
    return RETNET_OK;
}

retnet_status retnet_msr_layer(const void *x, const void *w_qkvg, const void *w_o,
                               const float *gammas, int chunk, void *y,
                               const retnet_shape *shape, int hidden, long long pos0,
                               const float *gn_weight, const float *gn_bias, float eps,
                               const float *state_in, float *state_out, void *workspace,
                               size_t workspace_bytes, retnet_stream_t stream) {
    MsrLayout l;
    retnet_status st = msr_layout(shape, hidden, chunk, &l);
    if (st != RETNET_OK) return st;
    if (!gammas || pos0 < 0 || !(eps >= 0.f)) return RETNET_ERR_INVALID_ARG;
    for (int h = 0; h < shape->heads; ++h)
        if (!(gammas[h] >= 0.f && gammas[h] <= 1.f)) return RETNET_ERR_INVALID_ARG;
    const long long rows = (long long)shape->batch * shape->seqlen;
    if (rows > 0) {
        if (!x || !w_qkvg || !w_o || !y || !aligned16(x) || !aligned16(w_qkvg) ||
            !aligned16(w_o) || !aligned16(y))
            return RETNET_ERR_INVALID_ARG;
    }
    if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
        return RETNET_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < l.total || ((uintptr_t)workspace & 1023u))
        return RETNET_ERR_WORKSPACE;
    const cudaStream_t s = (cudaStream_t)stream;
    char *ws = (char *)workspace;
    const int hd = shape->heads * shape->dk;
    void *q = ws + l.q, *k = ws + l.k, *v = ws + l.v, *g = ws + l.g, *o = ws + l.y;
    retnet_gate gate;
    gate.g = g;
    gate.weight = gn_weight;
    gate.bias = gn_bias;
    gate.eps = eps;
    // the tensor-core prefill, as retnet_retention_chunkwise would choose it
    const bool fused = rows > 0 && tc_shape_ok(shape->dk, shape->dv, shape->dtype, chunk) &&
                       tc_gammas_ok(chunk, gammas, shape->heads);
    if (!fused) {
        if (rows > 0) {
            void *outs[4] = {q, k, v, g};
            RETNET_CUDA_TRY(launch_gemm_bf16(x, w_qkvg, outs, rows, 4 * hd, hidden, hd, s,
                                             "gemm_qkvg"));
        }
        st = retnet_retention_chunkwise(q, k, v, gammas, chunk, o, shape, pos0, 1, state_in,
                                        state_out, &gate, RETNET_ALGO_AUTO, ws + l.fwd,
                                        l.fwd_bytes, stream);
        if (st != RETNET_OK) return st;
    } else {
        size_t qt_off = 0, kt_off = 0;
        GemmFold fold;
        fold.on = 1;
        fold.n = shape->seqlen;
        fold.heads = shape->heads;
        tc_operand_layout(shape->batch, shape->heads, shape->seqlen, chunk, &qt_off, &kt_off,
                          &fold.fold);
        for (int h = 0; h < kMaxHeads; ++h)
            fold.log2g[h] = h < shape->heads ? (float)std::log2((double)gammas[h]) : 0.f;
        float2 *table = reinterpret_cast<float2 *>(ws + l.table);
        RETNET_CUDA_TRY(launch_rotation_table(
            table, (shape->seqlen + kFoldTableStride - 1) / kFoldTableStride, 256, pos0, s,
            kFoldTableStride));
        fold.table = table;
        char *fwd = ws + l.fwd;
        void *outs[4] = {fwd + qt_off, fwd + kt_off, v, g};
        RETNET_CUDA_TRY(launch_gemm_bf16(x, w_qkvg, outs, rows, 4 * hd, hidden, hd, s,
                                         "gemm_qkvg", &fold));
        ChunkwiseArgs a;
        a.q = nullptr; a.k = nullptr; a.v = v; a.out = o;
        a.state_in = state_in; a.state_out = state_out; a.gate = &gate;
        a.batch = shape->batch; a.heads = shape->heads; a.seqlen = shape->seqlen;
        a.dk = shape->dk; a.dv = shape->dv; a.chunk = chunk; a.dtype = shape->dtype;
        a.pos0 = pos0; a.rotate = 1; a.workspace = fwd; a.workspace_bytes = l.fwd_bytes;
        for (int h = 0; h < kMaxHeads; ++h) a.gam.g[h] = h < shape->heads ? gammas[h] : 0.f;
        a.prefolded = true;
        RETNET_CUDA_TRY(launch_chunkwise_tc(a, gammas, s));
    }
    if (rows > 0) {
        void *outs[1] = {y};
        RETNET_CUDA_TRY(launch_gemm_bf16(o, w_o, outs, rows, hidden, hd, hidden, s, "gemm_out"));
    }
    return RETNET_OK;
}

}  // extern "C"
