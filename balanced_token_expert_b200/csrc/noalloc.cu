// noalloc.cu -- base_permute without a caller workspace, for callers that
// cannot allocate device memory.
//
// Some callers of this library only ever hold the input and output buffers
// and a stream: a plugin running inside another runtime that owns all device
// memory, or a serving loop that must not call cudaMalloc while it runs.
// They cannot pass base_permute the workspace it needs for its per-slice
// expert counts.  base_permute_noalloc keeps that scratch in the file-scope
// array below instead, a fixed 4 MiB reserved in every GPU that loads the
// library, until the process exits.
//
// The scratch holds the expert counts of at most ceil(T / 256) token slices
// (ceil(T / 256) * E int32), so a call needs
// ceil(T / 256) * E <= kNoallocScratchInts (for example T = 131072 tokens
// with E up to 2048 experts); larger shapes are rejected with
// BASE_ERR_WORKSPACE before anything is launched.  Every count the kernels
// read is written earlier in the same call, so nothing has to be cleared
// between calls.  All calls share the one array: calls that overlap on the
// GPU (different streams, or other threads) race on it and must be ordered
// by the caller.
#include <mutex>

#include "common.cuh"

namespace base {

int launch_sort_by_expert(const int32_t* assign, int T, int E, int32_t* perm, int32_t* inv,
                          int32_t* offsets, const float* s, float* gate, void* ws,
                          cudaStream_t stream);
int launch_move_rows(const void* src, const int32_t* idx, int T, int D, void* dst, bool scatter,
                     cudaStream_t stream);

namespace noalloc {

constexpr size_t kNoallocScratchInts = (size_t)1 << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_permute_scratch[kNoallocScratchInts];

// device address of g_permute_scratch, looked up once per device ordinal and
// kept for the life of the process (stale after cudaDeviceReset or in another
// driver context on the same device: such callers use base_permute)
static void* g_scratch_addr[kMaxDevices];
static std::mutex g_scratch_mutex;

static int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BASE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BASE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_permute_scratch) != cudaSuccess || ptr == nullptr)
            return BASE_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return BASE_OK;
}

}  // namespace noalloc
}  // namespace base

extern "C" int base_permute_noalloc(const void* h, const int32_t* assign, int T, int D, int E,
                                    int32_t* perm, int32_t* inv, int32_t* offsets, void* x_perm,
                                    const float* s, float* gate, cudaStream_t stream) {
    using namespace base;
    if (!assign || !perm || !inv || !offsets || T < 1 || E < 2 || E > 1024)
        return BASE_ERR_INVALID_ARG;
    if ((h == nullptr) != (x_perm == nullptr)) return BASE_ERR_INVALID_ARG;
    if ((s == nullptr) != (gate == nullptr)) return BASE_ERR_INVALID_ARG;
    if (h && (D < 8 || D % 8 != 0 || reinterpret_cast<uintptr_t>(h) % 16 != 0 ||
              reinterpret_cast<uintptr_t>(x_perm) % 16 != 0))
        return BASE_ERR_INVALID_ARG;
    const size_t need = (size_t)((T + 255) / 256) * (size_t)E;
    if (need > noalloc::kNoallocScratchInts) return BASE_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int st0 = noalloc::scratch_address(&scratch);
    if (st0 != BASE_OK) return st0;
    int st = launch_sort_by_expert(assign, T, E, perm, inv, offsets, s, gate, scratch, stream);
    if (st != BASE_OK || !h) return st;
    return launch_move_rows(h, perm, T, D, x_perm, false, stream);
}
