// Internal launcher declarations shared between api.cu and the kernel files.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace retnet {

// rotate.cu ---------------------------------------------------------------
// table[t * (d/2) + j] = (cos, sin) of (pos0 + t * stride) * theta_j, t < rows.
cudaError_t launch_rotation_table(float2 *table, int rows, int d, long long pos0,
                                  cudaStream_t stream, int stride = 1);
cudaError_t launch_xpos_rotate(const void *x, void *y, long long rows_bt, int heads, int d,
                               retnet_dtype dtype, int seqlen, long long pos0,
                               cudaStream_t stream);

// backward.cu --------------------------------------------------------------
// theta_j = 10000^(-2j/dk) for j < dk/2 <= 128, formed on the host.
struct BackwardThetas {
    double theta[128];
};
// K^ = R k; rev(R k), rev(R q), rev(v), rev(dO) (rev: token t -> n-1-t).
cudaError_t launch_backward_prep(const void *q, const void *k, const void *v, const void *dout,
                                 void *kh, void *rkh, void *rqh, void *rv, void *rdo, int batch,
                                 int heads, int n, int dk, int dv, retnet_dtype dtype,
                                 long long pos0, int rotate, cudaStream_t stream);
// bf16, d = 256, the tensor-core backward: from q, k, v, dO, the three
// retentions' Qt, Kt (qt[i], kt[i], each in the prefill's [B*H, n, 256]
// layout with the decay folded over `fold`) and values (vals[i], [B, n, H,
// 256]): ret 1 = (dO, V; R k), ret 2 = rev(V, dO; R q), ret 3 = rev(R k, R q; dO).
cudaError_t launch_backward_fold(const void *q, const void *k, const void *v, const void *dout,
                                 void *const *qt, void *const *kt, void *const *vals,
                                 const float *gammas, int batch, int heads, int n, int fold,
                                 long long pos0, int rotate, cudaStream_t stream);
// dq <- R^T dq (in place); dk = R^T rev(dk_rev); dv = rev(dv_rev).
cudaError_t launch_backward_post(void *dq, const void *dk_rev, const void *dv_rev, void *dk,
                                 void *dv, int batch, int heads, int n, int dkd, int dvd,
                                 retnet_dtype dtype, long long pos0, int rotate,
                                 cudaStream_t stream);

// step.cu ----------------------------------------------------------------
// q, k [batch, tokens, heads, dk]; v, out [batch, tokens, heads, dv] (with
// tokens = 1 this is the [batch, heads, d] layout of a single step).
cudaError_t launch_retention_recurrent(const void *q, const void *k, const void *v,
                                       const HeadGammas &gam, float *state, void *out,
                                       int batch, int tokens, int heads, int dk, int dv,
                                       retnet_dtype dtype, long long pos, int rotate,
                                       cudaStream_t stream);

// groupnorm.cu -------------------------------------------------------------
cudaError_t launch_groupnorm_swish(const void *o, const void *g, const float *weight,
                                   const float *bias, float eps, long long rows, int heads,
                                   int dv, retnet_dtype dtype, void *y, cudaStream_t stream);

// chunkwise_simt.cu --------------------------------------------------------
struct ChunkwiseArgs {
    const void *q, *k, *v;
    void *out;
    const float *state_in;
    float *state_out;
    const retnet_gate *gate;     // may be null
    int batch, heads, seqlen, dk, dv, chunk;
    retnet_dtype dtype;
    long long pos0;
    int rotate;
    HeadGammas gam;
    void *workspace;
    size_t workspace_bytes;
    // Tensor-core path only: Qt and Kt are already in the workspace (the MSR
    // layer's projection GEMM folded them), so the prep pass is skipped and
    // q, k are not read.
    bool prefolded = false;
};
size_t simt_workspace_bytes(int batch, int heads, int seqlen, int dk, int dv, int chunk);
cudaError_t launch_chunkwise_simt(const ChunkwiseArgs &a, cudaStream_t stream);

// chunkwise_tc.cu ----------------------------------------------------------
// Shape/dtype/chunk admitted by the tensor-core path.
bool tc_shape_ok(int dk, int dv, retnet_dtype dtype, int chunk);
// Every head's decay admits the decay fold: gamma > 0 and chunk*log2(1/gamma) <= 100.
bool tc_gammas_ok(int chunk, const float *gammas, int heads);
size_t tc_workspace_bytes(int batch, int heads, int seqlen, int chunk);
// Byte offsets of Qt and Kt ([B*H, n, 256] bf16 each) in the workspace, and
// the block length their decay is folded over (the chunk, or 128 for chunks
// below 128).
void tc_operand_layout(int batch, int heads, int seqlen, int chunk, size_t *qt, size_t *kt,
                       int *fold);
// parallel: the parallel form over the whole sequence (a.chunk, state_in and
// state_out unused; decays must pass tc_gammas_ok at chunk 128).
cudaError_t launch_chunkwise_tc(const ChunkwiseArgs &a, const float *gammas, cudaStream_t stream,
                                bool parallel = false);
size_t tc_parallel_workspace_bytes(int batch, int heads, int seqlen);
// Tensor map of a bf16 tensor for TMA (128-byte swizzle), innermost
// dimension first; false if the driver rejects it.
bool make_tensor_map_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                          const cuuint64_t *strides_bytes, const cuuint32_t *box);

// gemm_tc.cu ---------------------------------------------------------------
// Rotation and decay fold applied by the GEMM's epilogue to outputs 0 and 1
// (the MSR layer's Q and K, 256 columns per head): with row r = b n + t,
// column 2j, 2j+1 of head h is turned by the angle (pos0 + t) theta_j,
// theta_j = 10000^(-j/128), and scaled by gamma_h^(+(t mod fold + 1))
// (output 0) or gamma_h^(-(t mod fold + 1)) (output 1), and written as Qt,
// Kt in the prefill's [b*H + h][t][256] layout instead of [m, n_split].
// The angle is split as (pos0 + tb) theta_j + (t - tb) theta_j with
// tb = t rounded down to a multiple of kFoldTableStride: the first part's
// (cos, sin) is table[(t / kFoldTableStride) * 128 + j] (launch_rotation_table
// with that stride), the second (below 32 theta_j) is formed in registers.
constexpr int kFoldTableStride = 32;
struct GemmFold {
    int on;
    int n, heads, fold;
    const float2 *table;           // [ceil(n / kFoldTableStride), 128] device
    float log2g[kMaxHeads];
};
// Y = X W^T on the tensor cores: X [m, k], W [n, k], bf16, f32 accumulation.
// Columns [j n_split, (j+1) n_split) of Y go to outs[j] ([m, n_split], dense).
// timer_name: the kernel timer's name for this launch (a string literal).
// fold (optional): outputs 0 and 1 folded as GemmFold describes.
bool gemm_shape_ok(long long m, int n, int k, int n_split);
cudaError_t launch_gemm_bf16(const void *x, const void *w, void *const *outs, long long m, int n,
                             int k, int n_split, cudaStream_t stream,
                             const char *timer_name = "gemm", const GemmFold *fold = nullptr);

}  // namespace retnet
