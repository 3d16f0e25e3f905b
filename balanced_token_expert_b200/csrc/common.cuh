// common.cuh -- helpers shared by the libbase kernels (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/base.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libbase is written for sm_100a (B200) only"
#endif

namespace base {

constexpr int kWarp = 32;

// Sticky device-side error word: the first kernel that gives up a bounded
// wait (or detects an impossible state) records its code here.  Read and
// cleared by base_device_error().  libbase is built as one translation unit
// (libbase.cu), so this is the only definition.
__device__ int64_t g_device_error = 0;

__device__ __forceinline__ void record_error(int64_t code) {
    atomicCAS(reinterpret_cast<unsigned long long*>(&g_device_error), 0ull,
              static_cast<unsigned long long>(code));
}

__device__ __forceinline__ bool device_error_set() {
    return *reinterpret_cast<volatile int64_t*>(&g_device_error) != 0;
}

// Test hooks, set by base_test_inject (host side, process-wide; the
// launchers copy them into the kernels' parameters).  With every field at its
// default nothing changes.  They exist so that a test can watch a bounded wait
// give up: a shorter wait limit, and an arrival that never comes (one auction
// CTA that leaves before its first grid barrier, or one single-CTA GEMM CTA
// that never issues its first TMA load).  No hook makes a kernel fault.
struct TestHooks {
    long long wait_ns;          // > 0: limit of every bounded wait, in ns
    int auction_absent_cta;     // >= 0: this auction CTA returns at once
    int gemm_drop_first_load;   // 1: CTA 0 of a one-CTA GEMM skips its first load
};
static TestHooks g_test_hooks = {0, -1, 0};

// Iteration limit for every spin-wait in the library (try_wait already
// suspends the thread for a while per attempt, so this is well above any
// legitimate wait and far below a hung GPU).
constexpr long long kSpinLimit = 1ll << 26;

// SM count of the current device (host side, cached per device ordinal)
static inline int num_sms() {
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
    int* slot = dev < 64 ? &cache[dev] : nullptr;
    if (slot && *slot > 0) return *slot;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (slot) *slot = n;
    return n;
}

// Programmatic dependent launch: a kernel launched with launch_pdl may start
// while the previous kernel on the stream finishes; it calls pdl_wait() before
// reading anything earlier kernels wrote, and pdl_trigger() to let the next
// kernel start early in turn (the next grid launches once every CTA of this
// one has triggered or exited).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <class... KArgs, class... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__host__ __device__ __forceinline__ size_t align_up(size_t x, size_t a) {
    return (x + a - 1) / a * a;
}

// q = rint(s * 2^16), half to even, saturated to +-(2^31 - 1).
__device__ __forceinline__ int32_t quantize_score(float s) {
    const float x = s * BASE_QSCALE;       // exact: scaling by a power of two
    int32_t r = __float2int_rn(x);         // round to nearest even, saturating
    return r < -2147483647 ? -2147483647 : r;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

}  // namespace base

#define BASE_RETURN_IF_LAUNCH_FAILED()                       \
    do {                                                     \
        cudaError_t e_ = cudaGetLastError();                 \
        if (e_ != cudaSuccess) return BASE_ERR_CUDA;         \
    } while (0)

#define BASE_RETURN_IF(cond, code) \
    do {                           \
        if (cond) return (code);   \
    } while (0)
