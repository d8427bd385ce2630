// Chunkwise prefill for callers that cannot allocate device memory.
//
// retnet_retention_chunkwise takes its scratch space from a workspace the
// caller allocates.  Some callers cannot do that at run time: a plugin
// inside a serving process that reserves all device memory at start-up and
// gives its plugins no allocator, or a latency-critical path where
// cudaMalloc's implicit device-wide synchronisation is not acceptable.  For
// them, retnet_retention_chunkwise_noalloc runs the same kernels on a fixed
// scratch array compiled into this library (RETNET_NOALLOC_SCRATCH_BYTES per
// device, held by every GPU that loads the library until the process exits)
// and allocates nothing itself.
#include "kernels.h"

// The scratch array: the stated maximum plus room to round its start up to
// the 1024-byte boundary the tensor-core path's TMA buffers need.  In host
// code this name is only a stand-in for the symbol, not a device address:
// its address comes from cudaGetSymbolAddress, taken once per CUDA context
// (per device, and again after a cudaDeviceReset) with that context current.
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[RETNET_NOALLOC_SCRATCH_BYTES + 1024];

namespace retnet {
namespace {

SymbolAddressCache g_scratch_cache;

// Device address of the scratch array in the current context.
cudaError_t scratch_on_current_device(void **out) {
    return g_scratch_cache.get(g_noalloc_scratch, out);
}

}  // namespace
}  // namespace retnet

using namespace retnet;

extern "C" retnet_status retnet_retention_chunkwise_noalloc(
    const void *q, const void *k, const void *v, const float *gammas, int chunk, void *out,
    const retnet_shape *shape, long long pos0, int rotate, const float *state_in,
    float *state_out, const retnet_gate *gate, retnet_algo algo, retnet_stream_t stream) {
    if (!shape || !gammas || shape->heads < 1 || shape->heads > kMaxHeads)
        return RETNET_ERR_INVALID_ARG;
    // Size the scratch for the kernel family this call will run.
    retnet_algo resolved = algo;
    if (algo == RETNET_ALGO_AUTO)
        resolved = tc_shape_ok(shape->dk, shape->dv, shape->dtype, chunk) &&
                           tc_gammas_ok(chunk, gammas, shape->heads)
                       ? RETNET_ALGO_TENSOR
                       : RETNET_ALGO_SIMT;
    size_t need = 0;
    retnet_status st = retnet_chunkwise_workspace_size(shape, chunk, resolved, &need);
    if (st != RETNET_OK) return st;
    if (need > (size_t)RETNET_NOALLOC_SCRATCH_BYTES) return RETNET_ERR_WORKSPACE;
    void *base = nullptr;
    if (scratch_on_current_device(&base) != cudaSuccess) return RETNET_ERR_CUDA;
    void *scratch = (void *)(((uintptr_t)base + 1023) & ~(uintptr_t)1023);
    // The kernels write every scratch byte they read within the call, so the
    // previous call's contents need no clearing.
    return retnet_retention_chunkwise(q, k, v, gammas, chunk, out, shape, pos0, rotate, state_in,
                                      state_out, gate, resolved, scratch,
                                      (size_t)RETNET_NOALLOC_SCRATCH_BYTES, stream);
}
