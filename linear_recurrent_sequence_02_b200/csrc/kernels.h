// Internal launcher declarations shared between api.cu and the kernel files.
#pragma once

#include "common.cuh"

namespace retnet {

// rotate.cu ---------------------------------------------------------------
// table[t * (d/2) + j] = (cos, sin) of (pos0 + t) * theta_j, t < n.
cudaError_t launch_rotation_table(float2 *table, int n, int d, long long pos0,
                                  cudaStream_t stream);
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
};
size_t simt_workspace_bytes(int batch, int heads, int seqlen, int dk, int dv, int chunk);
cudaError_t launch_chunkwise_simt(const ChunkwiseArgs &a, cudaStream_t stream);

// chunkwise_tc.cu ----------------------------------------------------------
// Shape/dtype/chunk admitted by the tensor-core path.
bool tc_shape_ok(int dk, int dv, retnet_dtype dtype, int chunk);
// Every head's decay admits the decay fold: gamma > 0 and chunk*log2(1/gamma) <= 100.
bool tc_gammas_ok(int chunk, const float *gammas, int heads);
size_t tc_workspace_bytes(int batch, int heads, int seqlen, int chunk);
// parallel: the parallel form over the whole sequence (a.chunk, state_in and
// state_out unused; decays must pass tc_gammas_ok at chunk 128).
cudaError_t launch_chunkwise_tc(const ChunkwiseArgs &a, const float *gammas, cudaStream_t stream,
                                bool parallel = false);
size_t tc_parallel_workspace_bytes(int batch, int heads, int seqlen);

}  // namespace retnet
