// ep.cu -- the data movement of expert parallelism ("BASE Layers: Simplifying
// Training of Large, Sparse Models", wikillm.com summary, Method: Sharding;
// fig. 2's forward pass) as two kernels that each fuse a permutation with
// its all-to-all over peer memory.
//
// G workers each hold T tokens and E/G experts (El = E/G); the balanced
// assignment gives every expert exactly C = T/E of each worker's tokens, so a
// worker's expert-major slot s (from the sort by expert: perm[s] = token)
// belongs to expert e = s / C, i.e. to worker r = e / El, local expert
// j = e % El, position c = s % C.  Worker r receives its experts' rows
// expert-major, the G sources of one expert together:
//     recv_r[(j G + g) C + c] = h_g[perm_g[(r El + j) C + c]]
// (sort_by_expert, the route all-to-all and the receive-side regrouping in
// one pass: ep_dispatch), and after its experts ran, sends every output row
// straight to the token it belongs to:
//     out_g[perm_g[(r El + j) C + c]] = y_r[(j G + g) C + c]
// (the return all-to-all and inverse_sort in one pass: ep_combine).
//
// Every access is a plain 16-byte load or store, so the pointers of other
// workers may be peer mappings over NVLink (no TMA, no multicast).  One
// launch serves any subset of the workers: the sources [g0, g0 + ns) of a
// dispatch and the receivers [r0, r0 + nr) of a combine.  A worker's own
// launch takes its own rank; one launch over every worker's buffers on one
// GPU emulates the whole exchange.
#include "common.cuh"

namespace base {
namespace ep {

constexpr int kMaxWorkers = 8;  // one NVSwitch node

// one row of vec 16-byte pieces by a warp, four loads in flight per lane
// before their stores (without that, the compiler keeps every load behind
// the previous store: the row's reads would wait one after another)
__device__ __forceinline__ void copy_row(const uint4* __restrict__ s, uint4* __restrict__ d,
                                         int vec, int lane) {
    int v = lane;
    for (; v + 3 * kWarp < vec; v += 4 * kWarp) {
        const uint4 a0 = __ldg(s + v), a1 = __ldg(s + v + kWarp);
        const uint4 a2 = __ldg(s + v + 2 * kWarp), a3 = __ldg(s + v + 3 * kWarp);
        d[v] = a0;
        d[v + kWarp] = a1;
        d[v + 2 * kWarp] = a2;
        d[v + 3 * kWarp] = a3;
    }
    for (; v < vec; v += kWarp) d[v] = __ldg(s + v);
}

struct Ptrs {
    const uint4* src[kMaxWorkers];  // dispatch: h_g;  combine: y_r
    uint4* dst[kMaxWorkers];        // dispatch: recv_r;  combine: out_g
    const int32_t* perm[kMaxWorkers];
    const float* gate[kMaxWorkers];  // dispatch: gate_g (slot order), nullable
    float* gate_out[kMaxWorkers];    // dispatch: recv_gate_r, nullable
};

// One warp per row; the row's 16-byte vectors over the lanes.  Items are
// (source g, slot s) pairs, g in [g0, g0 + ns).
__global__ void __launch_bounds__(256) ep_dispatch_kernel(const __grid_constant__ Ptrs p, int g0,
                                                          int ns, int G, int T, int El, int C,
                                                          int vec) {
    const int lane = lane_id();
    const long long items = (long long)ns * T;
    const long long nwarps = (long long)gridDim.x * (blockDim.x / kWarp);
    pdl_wait();
    pdl_trigger();
    for (long long it = blockIdx.x * (long long)(blockDim.x / kWarp) + warp_id(); it < items;
         it += nwarps) {
        const int gi = (int)(it / T);
        const int s = (int)(it - (long long)gi * T);
        const int g = g0 + gi;
        const int e = s / C, c = s - e * C;
        const int r = e / El, j = e - r * El;
        const long long row = ((long long)j * G + g) * C + c;
        const int t = __ldg(p.perm[g] + s);
        if ((unsigned)t >= (unsigned)T) {  // not a token: recorded, the row skipped
            if (lane == 0) record_error(2101);
            continue;
        }
        copy_row(p.src[g] + (long long)t * vec, p.dst[r] + row * vec, vec, lane);
        if (lane == 0 && p.gate[g] && p.gate_out[r]) p.gate_out[r][row] = __ldg(p.gate[g] + s);
    }
}

// Items are (receiver r, row i), r in [r0, r0 + nr).
__global__ void __launch_bounds__(256) ep_combine_kernel(const __grid_constant__ Ptrs p, int r0,
                                                         int nr, int G, int T, int El, int C,
                                                         int vec) {
    const int lane = lane_id();
    const long long items = (long long)nr * T;
    const long long nwarps = (long long)gridDim.x * (blockDim.x / kWarp);
    pdl_wait();
    pdl_trigger();
    for (long long it = blockIdx.x * (long long)(blockDim.x / kWarp) + warp_id(); it < items;
         it += nwarps) {
        const int ri = (int)(it / T);
        const int i = (int)(it - (long long)ri * T);
        const int r = r0 + ri;
        const int c = i % C;
        const int jg = i / C;  // j G + g
        const int j = jg / G, g = jg - j * G;
        const int s = (r * El + j) * C + c;
        const int t = __ldg(p.perm[g] + s);
        if ((unsigned)t >= (unsigned)T) {
            if (lane == 0) record_error(2102);
            continue;
        }
        copy_row(p.src[r] + (long long)i * vec, p.dst[g] + (long long)t * vec, vec, lane);
    }
}

}  // namespace ep

static int ep_grid(long long items) {
    long long blocks = (items + 7) / 8;  // eight rows per block, one per warp
    const long long cap = (long long)num_sms() * 64;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

int launch_ep_dispatch(const void* const* h, const int32_t* const* perm, const float* const* gate,
                       void* const* recv, float* const* recv_gate, int g0, int ns, int G, int T,
                       int D, int E, cudaStream_t stream) {
    ep::Ptrs p{};
    for (int g = 0; g < G; ++g) {
        p.dst[g] = static_cast<uint4*>(recv[g]);
        p.gate_out[g] = recv_gate ? recv_gate[g] : nullptr;
    }
    for (int g = g0; g < g0 + ns; ++g) {
        p.src[g] = static_cast<const uint4*>(h[g - g0]);
        p.perm[g] = perm[g - g0];
        p.gate[g] = gate ? gate[g - g0] : nullptr;
    }
    const int El = E / G, C = T / E;
    const long long items = (long long)ns * T;
    if (launch_pdl(ep::ep_dispatch_kernel, dim3(ep_grid(items)), dim3(256), 0, stream, p, g0, ns,
                   G, T, El, C, D * 2 / 16) != cudaSuccess)
        return BASE_ERR_CUDA;
    return BASE_OK;
}

int launch_ep_combine(const void* const* y, const int32_t* const* perm, void* const* out, int r0,
                      int nr, int G, int T, int D, int E, cudaStream_t stream) {
    ep::Ptrs p{};
    for (int g = 0; g < G; ++g) {
        p.dst[g] = static_cast<uint4*>(out[g]);
        p.perm[g] = perm[g];
    }
    for (int r = r0; r < r0 + nr; ++r) p.src[r] = static_cast<const uint4*>(y[r - r0]);
    const int El = E / G, C = T / E;
    const long long items = (long long)nr * T;
    if (launch_pdl(ep::ep_combine_kernel, dim3(ep_grid(items)), dim3(256), 0, stream, p, r0, nr, G,
                   T, El, C, D * 2 / 16) != cudaSuccess)
        return BASE_ERR_CUDA;
    return BASE_OK;
}

}  // namespace base
