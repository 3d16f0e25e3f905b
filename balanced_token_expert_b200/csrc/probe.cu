// probe.cu -- measured latency floors of the synchronisation steps the
// auction is built from, so that its time can be set against a latency
// roofline (rounds x the floor of each kind of round) instead of only the HBM
// one, which does not bind it.  One cooperative grid of the auction's shape
// (one 512-thread CTA per SM) times, in nanoseconds of the global timer:
//   [0] a grid barrier (the auction's flag barrier, all CTAs),
//   [1] a block barrier of 512 threads,
//   [2] a dependent load that hits L2 (a pointer chase over 1 MB),
//   [3] a dependent shared-memory load.
#include "common.cuh"

namespace base {
namespace probe {

constexpr int kProbeThreads = 512;
constexpr int kIters = 256;
constexpr int kChase = 1 << 18;  // 1 MB of int32 links: L2-resident

struct ProbeParams {
    auction::Ctrl* ctrl;
    unsigned* bar_flags;
    unsigned long long wait_ns;
    int32_t* chase;  // [kChase] a permutation cycle
    double* out;     // [4] device
};

__global__ void __launch_bounds__(kProbeThreads, 1) latency_probe_kernel(
    const __grid_constant__ ProbeParams p) {
    __shared__ int s_flag[16];
    __shared__ int32_t s_chain[1024];
    unsigned gen = 0;
    // the chase: link i -> (i * 4099 + 1) mod kChase (a single cycle: 4099 odd)
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < kChase; i += gridDim.x * blockDim.x)
        p.chase[i] = (int32_t)(((long long)i * 4099 + 1) % kChase);
    for (int i = threadIdx.x; i < 1024; i += blockDim.x) s_chain[i] = (i * 37 + 11) & 1023;
    if (!auction::grid_sync(p, gen, s_flag)) return;
    // [0] grid barriers
    uint64_t t0 = auction::globaltimer();
    for (int i = 0; i < kIters; ++i)
        if (!auction::grid_sync(p, gen, s_flag)) return;
    const uint64_t t_grid = auction::globaltimer() - t0;
    if (blockIdx.x != 0) return;
    // [1] block barriers
    t0 = auction::globaltimer();
    for (int i = 0; i < kIters * 4; ++i) __syncthreads();
    const uint64_t t_cta = auction::globaltimer() - t0;
    if (threadIdx.x != 0) return;
    // [2] dependent L2 loads (warm the line set first)
    int j = 0;
    for (int i = 0; i < kIters; ++i) j = __ldcg(p.chase + j);
    t0 = auction::globaltimer();
    for (int i = 0; i < kIters * 4; ++i) j = __ldcg(p.chase + j);
    const uint64_t t_l2 = auction::globaltimer() - t0;
    // [3] dependent shared-memory loads
    int k = j & 1023;
    t0 = auction::globaltimer();
    for (int i = 0; i < kIters * 16; ++i) k = *reinterpret_cast<volatile int32_t*>(s_chain + k);
    const uint64_t t_smem = auction::globaltimer() - t0;
    p.out[0] = (double)t_grid / kIters;
    p.out[1] = (double)t_cta / (kIters * 4);
    p.out[2] = (double)t_l2 / (kIters * 4) + 0.0 * (double)k;
    p.out[3] = (double)t_smem / (kIters * 16);
}

}  // namespace probe

size_t probe_workspace_bytes() {
    return align_up(sizeof(auction::Ctrl), 256) + align_up(sizeof(unsigned) * auction::kMaxGrid, 256) +
           align_up(sizeof(int32_t) * probe::kChase, 256);
}

int launch_latency_probe(double* out, void* ws, cudaStream_t stream) {
    using namespace probe;
    unsigned char* w = static_cast<unsigned char*>(ws);
    ProbeParams prm{};
    prm.ctrl = reinterpret_cast<auction::Ctrl*>(w);
    prm.bar_flags = reinterpret_cast<unsigned*>(w + align_up(sizeof(auction::Ctrl), 256));
    prm.chase = reinterpret_cast<int32_t*>(w + align_up(sizeof(auction::Ctrl), 256) +
                                           align_up(sizeof(unsigned) * auction::kMaxGrid, 256));
    prm.wait_ns = g_test_hooks.wait_ns > 0 ? (unsigned long long)g_test_hooks.wait_ns
                                           : auction::kWaitNs;
    prm.out = out;
    if (cudaMemsetAsync(w, 0, (size_t)(reinterpret_cast<unsigned char*>(prm.chase) - w), stream) !=
        cudaSuccess)
        return BASE_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, latency_probe_kernel, kProbeThreads,
                                                      0) != cudaSuccess ||
        per_sm < 1)
        return BASE_ERR_UNSUPPORTED;
    const int grid = std::min(num_sms(), auction::kMaxGrid);
    void* args[] = {&prm};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(latency_probe_kernel), dim3(grid),
                                    dim3(kProbeThreads), args, 0, stream) != cudaSuccess)
        return BASE_ERR_CUDA;
    return BASE_OK;
}

}  // namespace base
