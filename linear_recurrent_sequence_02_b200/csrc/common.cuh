// Shared device helpers for the retention kernels (internal header).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/retnet.h"

namespace retnet {

constexpr int kMaxHeads = 256;

// Per-head decay constants travel by value in the kernel parameter block.
struct HeadGammas {
    float g[kMaxHeads];
};

// Device-side error word (bit flags), read by retnet_check_device_errors.
enum DeviceError : unsigned {
    kDevErrTimeout = 1u,
    kDevErrBounds = 2u,          // an index check of a RETNET_CHECK_BOUNDS build failed
};
unsigned *device_error_word();   // device address of the current context's error word

// The current CUDA context (a CUcontext), or null if none is current.
void *current_context();

// Device address of a __device__ variable in the current context, looked up
// once per context (cudaGetSymbolAddress, with that context current) and
// cached.  Keyed by context, not device ordinal, so an address never outlives
// the context it belongs to (after cudaDeviceReset the primary context is a
// new one).  Use it in the translation unit that defines the variable.
class SymbolAddressCache {
  public:
    template <typename T>
    cudaError_t get(const T &symbol, void **out) {
        void *ctx = current_context();
        if (!ctx) {                        // no context yet: the runtime creates it
            cudaError_t e = cudaFree(nullptr);
            if (e != cudaSuccess) return e;
            ctx = current_context();
            if (!ctx) return cudaErrorDeviceUninitialized;
        }
        Lock lk(this);
        for (int i = 0; i < n_; ++i)
            if (ctx_[i] == ctx) {
                *out = ptr_[i];
                return cudaSuccess;
            }
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, symbol);
        if (e != cudaSuccess) return e;
        const int slot = n_ < kEntries ? n_++ : (next_++ % kEntries);
        ctx_[slot] = ctx;
        ptr_[slot] = p;
        *out = p;
        return cudaSuccess;
    }

  private:
    static constexpr int kEntries = 64;
    struct Lock {
        explicit Lock(SymbolAddressCache *c) : c_(c) { c_->lock(); }
        ~Lock() { c_->unlock(); }
        SymbolAddressCache *c_;
    };
    void lock() { while (busy_.test_and_set(std::memory_order_acquire)) {} }
    void unlock() { busy_.clear(std::memory_order_release); }
    std::atomic_flag busy_ = ATOMIC_FLAG_INIT;
    void *ctx_[kEntries] = {};
    void *ptr_[kEntries] = {};
    int n_ = 0, next_ = 0;
};

// Index checks of the debug build.  With RETNET_CHECK_BOUNDS defined,
// in_bounds(i, n, err) tests 0 <= i < n; a failed test records kDevErrBounds
// in the error word and the caller skips the access.  Without it the test
// is the constant true and compiles away.
// `site` (one of the kSite* bits) also goes into the word, so a debug run
// can tell which kernel's check failed (retnet_test_error_word).
enum BoundsSite : unsigned {
    kSitePrep = 1u << 8, kSiteState = 1u << 9, kSiteOutput = 1u << 10,
    kSiteOutputPair = 1u << 11, kSiteStep = 1u << 12, kSiteGemm = 1u << 13,
};
#ifdef RETNET_CHECK_BOUNDS
__device__ __forceinline__ bool in_bounds(long long i, long long n, unsigned *err,
                                          unsigned site = 0) {
    if (i >= 0 && i < n) return true;
    if (err) atomicOr(err, (unsigned)kDevErrBounds | site);
    return false;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(long long, long long, unsigned *,
                                                    unsigned = 0) {
    return true;
}
#endif

// Counts host-side kernel launches (see retnet_kernel_launch_count).
void count_launch(unsigned n = 1);

// Records CUDA events around one launch on `stream` while the profiler is
// enabled (retnet_profiler_enable); a no-op otherwise.  `name` must be a
// string literal.
class KernelTimer {
  public:
    KernelTimer(const char *name, cudaStream_t stream);
    ~KernelTimer();
    KernelTimer(const KernelTimer &) = delete;
    KernelTimer &operator=(const KernelTimer &) = delete;

  private:
    cudaStream_t stream_;
    const char *name_ = nullptr;
    void *start_ = nullptr;
    void *stop_ = nullptr;
    bool captured_ = false;
};

// ------------------------------------------------------ programmatic launch
// The kernels of one call, and of consecutive calls, follow each other on a
// stream.  Launched with programmatic stream serialisation, a kernel is
// launched as its predecessor's CTAs exit rather than after the whole grid
// has drained, so the launch gap and its set-up (barriers, TMEM allocation,
// descriptor prefetch) overlap the predecessor's tail.  Each such kernel
// calls grid_dependency_wait() before its first global-memory access: it
// returns once the predecessor grid has completed and its writes are
// visible (at once when the kernel was launched normally).  No kernel
// triggers its successor early (griddepcontrol.launch_dependents): waiting
// CTAs of the successor then sit on SMs that the rest of this grid needs,
// which measured slower.  Since every CTA passes its wait before it exits,
// a kernel never starts before its predecessors' predecessors completed.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Host: whether launches carry the programmatic-serialisation attribute
// (retnet_set_launch_overlap; on by default).
bool launch_overlap_enabled();
// Host: how the tensor-core output pass runs (retnet_set_output_pairing):
// 0 single CTAs (default), 1 CTA pairs folding q themselves, 2 CTA pairs
// reading the prep pass's folded q.
int output_pairing_mode();

template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = launch_overlap_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------------ rotation
// (cos, sin) of the angle pos * theta in float32.  The angle is reduced in
// float64 to a fraction of pi in [-1, 1], and sincospif, whose own argument
// reduction is exact, turns it into the pair.  The prefill prologue, the
// standalone rotation and the rotation table use this; the decode kernels
// take pairs formed on the host in float64 instead.
__device__ __forceinline__ float2 rotation_cs(long long pos, double theta) {
    const double inv_pi = 0.31830988618379067153776752674503;
    const double x = (double)pos * theta * inv_pi;           // angle / pi
    const double xr = x - 2.0 * rint(0.5 * x);               // in [-1, 1]
    float sn, cn;
    sincospif((float)xr, &sn, &cn);
    return make_float2(cn, sn);
}

// ---------------------------------------------------------------- element IO
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Loads 8 consecutive elements as float (16-byte aligned for bf16, 32 for f32).
__device__ __forceinline__ void load8(const float *p, float *out) {
    float4 a = reinterpret_cast<const float4 *>(p)[0];
    float4 b = reinterpret_cast<const float4 *>(p)[1];
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *out) {
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        out[2 * i] = f.x;
        out[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void store8(float *p, const float *v) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float *v) {
    uint4 u;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4 *>(p) = u;
}

// ---------------------------------------------------------------- rotation
// (cos, sin) of pos * theta_j with theta_j = 10000^(-2j/d) formed here in
// float64; accurate to a few 1e-7 for any position.
__device__ __forceinline__ float2 rotation_cs(long long pos, int j, int d) {
    return rotation_cs(pos, pow(10000.0, -2.0 * (double)j / (double)d));
}

// ---------------------------------------------------------------- launches
#define RETNET_CUDA_TRY(expr)                                  \
    do {                                                       \
        cudaError_t err__ = (expr);                            \
        if (err__ != cudaSuccess) return RETNET_ERR_CUDA;      \
    } while (0)

}  // namespace retnet
