// routing.cu -- the bandwidth-bound steps of the BASE layer:
//   * fp32 affinity scores s = h w^T with their quantisation (fig. 2
//     "affinities"; SIMT fp32 FMA: the tensor cores have no fp32-input mode
//     accurate to 1e-5),
//   * greedy test-time routing (argmax over experts, "Test time"),
//   * the expert-major permutation (fig. 2 sort_by_expert) as a stable
//     counting sort, and the 16-byte-vector row gather / scatter used by the
//     permute, the combine (inverse_sort) and the backward.
#include <algorithm>

#include "common.cuh"

namespace base {
namespace routing {

// ---------------------------------------------------------------------------
// fp32 scores: one warp per (token, 32 experts); lanes split D.
// ---------------------------------------------------------------------------
__global__ void scores_f32_kernel(const float* __restrict__ h, const float* __restrict__ w,
                                  int T, int D, int E, float* __restrict__ s,
                                  int32_t* __restrict__ q) {
    const int lane = lane_id();
    const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / kWarp;
    const long long nw = (gridDim.x * (long long)blockDim.x) / kWarp;
    for (long long item = gw; item < (long long)T * E; item += nw) {
        const int t = (int)(item / E), e = (int)(item % E);
        const float* hr = h + (size_t)t * D;
        const float* wr = w + (size_t)e * D;
        float acc = 0.f;
        for (int d = lane; d < D; d += kWarp) acc = fmaf(__ldg(hr + d), __ldg(wr + d), acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            if (s) s[item] = acc;
            if (q) q[item] = quantize_score(acc);
        }
    }
}

// ---------------------------------------------------------------------------
// greedy routing: a group of lanes per token row, argmax with lowest index on
// ties, per-block expert histogram folded into the global counts.
// ---------------------------------------------------------------------------
__global__ void greedy_kernel(const int32_t* __restrict__ q, int T, int E,
                              int32_t* __restrict__ assign, int32_t* __restrict__ counts) {
    extern __shared__ int32_t s_hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    __syncthreads();
    // lanes per token: one per 16-byte piece of the row when E % 4 == 0
    // (int4 loads), else one per entry
    const bool vec = (E & 3) == 0;
    const int words = vec ? E / 4 : E;
    int G = 1;
    while (G < words && G < kWarp) G <<= 1;
    const int lane = lane_id(), sub = lane / G, gl = lane % G;
    const int per_warp = kWarp / G;
    const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / kWarp;
    const long long nw = (gridDim.x * (long long)blockDim.x) / kWarp;
    for (long long base = gw * per_warp; base < T; base += nw * per_warp) {
        const long long t = base + sub;
        const bool valid = t < T;
        int best_v = INT32_MIN, best_e = INT32_MAX;
        if (valid) {
            const int32_t* row = q + (size_t)t * E;
            if (vec) {
                const int4* r4 = reinterpret_cast<const int4*>(row);
                for (int j = gl; j < E / 4; j += G) {
                    const int4 v = __ldg(r4 + j);
                    const int e0 = 4 * j;
                    // conditional moves, not branches (the first of equal values stays)
                    bool g = v.x > best_v;
                    best_e = g ? e0 : best_e;
                    best_v = g ? v.x : best_v;
                    g = v.y > best_v;
                    best_e = g ? e0 + 1 : best_e;
                    best_v = g ? v.y : best_v;
                    g = v.z > best_v;
                    best_e = g ? e0 + 2 : best_e;
                    best_v = g ? v.z : best_v;
                    g = v.w > best_v;
                    best_e = g ? e0 + 3 : best_e;
                    best_v = g ? v.w : best_v;
                }
            } else {
                for (int e = gl; e < E; e += G) {
                    const int v = __ldg(row + e);
                    const bool g = v > best_v;
                    best_e = g ? e : best_e;
                    best_v = g ? v : best_v;
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            if (off >= G) continue;
            const int ov = __shfl_xor_sync(0xffffffffu, best_v, off);
            const int oe = __shfl_xor_sync(0xffffffffu, best_e, off);
            const bool tk = (ov > best_v) | ((ov == best_v) & (oe < best_e));
            best_v = tk ? ov : best_v;
            best_e = tk ? oe : best_e;
        }
        if (valid && gl == 0) {
            assign[t] = best_e;
            if (counts) atomicAdd(&s_hist[best_e], 1);
        }
    }
    if (counts) {
        __syncthreads();
        for (int e = threadIdx.x; e < E; e += blockDim.x)
            if (s_hist[e]) atomicAdd(&counts[e], s_hist[e]);
    }
}

// ---------------------------------------------------------------------------
// stable counting sort of tokens by expert (expert-major slots, ascending
// token inside an expert): perm, inv, offsets and the permuted gate scores
// ---------------------------------------------------------------------------
// The sort runs over P slices of consecutive tokens, one CTA
// per slice, in two launches:
//   slice_hist_kernel   the expert counts of every slice (shared atomics);
//   slice_rank_kernel   each CTA sums the counts of the slices before its own
//                       (its starting slot per expert) and of all slices (the
//                       expert offsets, an exclusive scan over experts), then
//                       ranks its tokens in order: warp w takes a contiguous
//                       part of the slice, counts it per expert, the counts
//                       become per-warp starting slots, and each 32-token group
//                       is ranked with match_any (ties in token order).
constexpr int kSliceMax = 8192;  // tokens per slice: 32 warps x 8 groups of 32

__global__ void __launch_bounds__(1024) slice_hist_kernel(const int32_t* __restrict__ assign,
                                                          int T, int E, int slice,
                                                          int32_t* __restrict__ cnt) {
    extern __shared__ int32_t sh[];  // [E]
    for (int e = threadIdx.x; e < E; e += blockDim.x) sh[e] = 0;
    pdl_wait();
    pdl_trigger();
    __syncthreads();
    const int t0 = blockIdx.x * slice, t1 = min(T, t0 + slice);
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const int e = assign[t];
        if (e >= 0 && e < E) atomicAdd(&sh[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[(size_t)blockIdx.x * E + e] = sh[e];
}

__global__ void __launch_bounds__(1024) slice_rank_kernel(const int32_t* __restrict__ assign,
                                                          int T, int E, int slice,
                                                          const int32_t* __restrict__ cnt,
                                                          int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ inv,
                                                          int32_t* __restrict__ offsets,
                                                          const float* __restrict__ s,
                                                          float* __restrict__ gate) {
    extern __shared__ int32_t sm[];
    int32_t* wc = sm;                  // [32][E]: per-warp counts, then running slots
    int32_t* s_warp = sm + 32 * E;     // [32] block-scan partials
    const int w = warp_id(), lane = lane_id();
    pdl_wait();
    pdl_trigger();
    const unsigned lt = (1u << lane) - 1;
    const int b = blockIdx.x;
    const int s0 = b * slice, s1 = min(T, s0 + slice);
    const int per = ((s1 - s0 + 31) / 32 + 31) / 32 * 32;  // tokens per warp (multiple of 32)
    const int t0 = min(s1, s0 + w * per), t1 = min(s1, t0 + per);
    const int ni = (t1 - t0 + kWarp - 1) / kWarp;         // <= kSliceMax / 1024 groups
    for (int e = lane; e < E; e += kWarp) wc[w * E + e] = 0;
    int ev[kSliceMax / 1024];
#pragma unroll
    for (int i = 0; i < kSliceMax / 1024; ++i) {
        const int t = t0 + i * kWarp + lane;
        ev[i] = (i < ni && t < t1) ? assign[t] : -1;
        if (i < ni && t < t1 && (ev[i] < 0 || ev[i] >= E)) {  // not an expert: recorded, skipped
            record_error(2001);
            ev[i] = -1;
        }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < kSliceMax / 1024; ++i) {
        if (i < ni) {
            const int e = ev[i];
            const unsigned peers = __match_any_sync(0xffffffffu, e >= 0 ? e : -1 - lane);
            if (e >= 0 && (peers & lt) == 0) wc[w * E + e] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    // thread e: the slices before this one and all slices, then this slice's
    // warps; an exclusive scan of the totals over the experts
    const int e_me = threadIdx.x;  // E <= 1024 = blockDim
    int before = 0, total = 0, run = 0;
    if (e_me < E) {
        for (int bb = 0; bb < (int)gridDim.x; ++bb) {
            const int c = cnt[(size_t)bb * E + e_me];
            before += bb < b ? c : 0;
            total += c;
        }
        for (int v = 0; v < 32; ++v) {
            const int c = wc[v * E + e_me];
            wc[v * E + e_me] = run;
            run += c;
        }
    }
    int incl = e_me < E ? total : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[w] = incl;
    __syncthreads();
    if (w == 0) {
        const int v = s_warp[lane];
        int vi = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, vi, off);
            if (lane >= off) vi += o;
        }
        s_warp[lane] = vi - v;
    }
    __syncthreads();
    if (e_me < E) {
        const int off_e = incl - total + s_warp[w];  // expert e's first slot
        if (b == 0) {
            offsets[e_me] = off_e;
            if (e_me == E - 1) offsets[E] = off_e + total;
        }
        const int base = off_e + before;
        for (int v = 0; v < 32; ++v) wc[v * E + e_me] += base;
    }
    __syncthreads();
    float gv[kSliceMax / 1024];
#pragma unroll
    for (int i = 0; i < kSliceMax / 1024; ++i) {
        const int t = t0 + i * kWarp + lane;
        gv[i] = (gate && i < ni && ev[i] >= 0) ? s[(size_t)t * E + ev[i]] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kSliceMax / 1024; ++i) {
        if (i < ni) {
            const int t = t0 + i * kWarp + lane;
            const int e = ev[i];
            const unsigned peers = __match_any_sync(0xffffffffu, e >= 0 ? e : -1 - lane);
            int slot = 0;
            if (e >= 0) slot = wc[w * E + e] + __popc(peers & lt);
            __syncwarp();
            if (e >= 0 && (peers & lt) == 0) wc[w * E + e] += __popc(peers);
            __syncwarp();
            if (e >= 0) {
                perm[slot] = t;
                inv[t] = slot;
                if (gate) gate[slot] = gv[i];
            }
        }
    }
}

// ---------------------------------------------------------------------------
// row gather / scatter of bf16 rows with 16-byte vectors:
//   gather:  dst[r] = src[idx[r]]        scatter: dst[idx[r]] = src[r]
// ---------------------------------------------------------------------------
template <bool kScatter>
__global__ void __launch_bounds__(256) move_rows_kernel(const uint4* __restrict__ src,
                                                        const int32_t* __restrict__ idx, int T,
                                                        int vec_per_row, uint4* __restrict__ dst) {
    // one warp per row: the index is read once, the row's 16-byte vectors are
    // spread over the lanes (coalesced), several loads in flight per lane
    constexpr int kUnroll = 4;
    const int lane = lane_id();
    const long long nwarps = (long long)gridDim.x * (blockDim.x / kWarp);
    pdl_wait();
    pdl_trigger();
    for (long long r = blockIdx.x * (long long)(blockDim.x / kWarp) + warp_id(); r < T; r += nwarps) {
        const int m = __ldg(idx + r);
        if ((unsigned)m >= (unsigned)T) {  // not a row: recorded, the row skipped
            if (lane == 0) record_error(2002);
            continue;
        }
        const uint4* s_row = src + (kScatter ? r : (long long)m) * vec_per_row;
        uint4* d_row = dst + (kScatter ? (long long)m : r) * vec_per_row;
        int c = lane;
        for (; c + (kUnroll - 1) * kWarp < vec_per_row; c += kUnroll * kWarp) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) v[u] = __ldcs(s_row + c + u * kWarp);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) __stcs(d_row + c + u * kWarp, v[u]);
        }
        for (; c < vec_per_row; c += kWarp) __stcs(d_row + c, __ldcs(s_row + c));
    }
}

}  // namespace routing

int launch_scores_f32(const float* h, const float* w, int T, int D, int E, float* s, int32_t* q,
                      cudaStream_t stream) {
    const long long items = (long long)T * E;
    const int threads = 256;
    long long blocks = (items * kWarp + threads - 1) / threads;
    if (blocks > num_sms() * 16) blocks = num_sms() * 16;
    routing::scores_f32_kernel<<<(int)blocks, threads, 0, stream>>>(h, w, T, D, E, s, q);
    BASE_RETURN_IF_LAUNCH_FAILED();
    return BASE_OK;
}

int launch_greedy(const int32_t* q, int T, int E, int32_t* assign, int32_t* counts,
                  cudaStream_t stream) {
    if (counts && cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream) != cudaSuccess)
        return BASE_ERR_CUDA;
    const int threads = 256;
    const int words = (E & 3) == 0 ? E / 4 : E;  // the kernel's lanes per token
    int G = 1;
    while (G < words && G < kWarp) G <<= 1;
    const long long warps_needed = ((long long)T * G + kWarp - 1) / kWarp;
    long long blocks = (warps_needed * kWarp + threads - 1) / threads;
    if (blocks > num_sms() * 8) blocks = num_sms() * 8;
    if (blocks < 1) blocks = 1;
    routing::greedy_kernel<<<(int)blocks, threads, sizeof(int32_t) * E, stream>>>(q, T, E, assign,
                                                                                   counts);
    BASE_RETURN_IF_LAUNCH_FAILED();
    return BASE_OK;
}

// the slices' expert counts: at most ceil(T / 256) slices (slices hold >= 512 tokens)
size_t permute_workspace_bytes(int T, int E) {
    const size_t nslices = (size_t)(T + 255) / 256;
    return align_up(sizeof(int32_t) * nslices * E, 256) + 256;
}

// perm / inv / offsets (+ gate) from an assignment.  An expert index out of
// range is recorded in the device error word and its token is skipped.
int launch_sort_by_expert(const int32_t* assign, int T, int E, int32_t* perm, int32_t* inv,
                          int32_t* offsets, const float* s, float* gate, void* ws,
                          cudaStream_t stream) {
    using namespace routing;
    // slices of at least 512 tokens, at most 128 of them up to 1M tokens (every
    // CTA reads the counts of all slices)
    const int slice = std::min(kSliceMax, std::max(512, (T + 127) / 128));
    const int P = (T + slice - 1) / slice;
    int32_t* cnt = static_cast<int32_t*>(ws);  // [P][E]
    if (launch_pdl(slice_hist_kernel, dim3(P), dim3(1024), sizeof(int32_t) * E, stream, assign, T,
                   E, slice, cnt) != cudaSuccess)
        return BASE_ERR_CUDA;
    const size_t sm = sizeof(int32_t) * (32 * (size_t)E + 32);
    if (cudaFuncSetAttribute(slice_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm) != cudaSuccess)
        return BASE_ERR_CUDA;
    if (launch_pdl(slice_rank_kernel, dim3(P), dim3(1024), sm, stream, assign, T, E, slice,
                   (const int32_t*)cnt, perm, inv, offsets, s, gate) != cudaSuccess)
        return BASE_ERR_CUDA;
    return BASE_OK;
}

int launch_move_rows(const void* src, const int32_t* idx, int T, int D, void* dst, bool scatter,
                     cudaStream_t stream) {
    const int vec = D * 2 / 16;
    const int threads = 256;  // eight rows in flight per block, one per warp
    long long blocks = ((long long)T + threads / kWarp - 1) / (threads / kWarp);
    if (blocks > num_sms() * 64) blocks = num_sms() * 64;
    if (blocks < 1) blocks = 1;
    const cudaError_t err =
        scatter ? launch_pdl(routing::move_rows_kernel<true>, dim3((int)blocks), dim3(threads), 0,
                             stream, static_cast<const uint4*>(src), idx, T, vec,
                             static_cast<uint4*>(dst))
                : launch_pdl(routing::move_rows_kernel<false>, dim3((int)blocks), dim3(threads), 0,
                             stream, static_cast<const uint4*>(src), idx, T, vec,
                             static_cast<uint4*>(dst));
    if (err != cudaSuccess) return BASE_ERR_CUDA;
    return BASE_OK;
}

}  // namespace base

// ---------------------------------------------------------------------------
// Non-finite scores ("Paper vs code", Non-finite scores: the released code
// replaces NaN and infinite affinities with the minimum finite score before
// solving).  Pass 1: per-block minimum of the finite scores and count of the
// others; pass 2: every block reduces the partials and, when something is not
// finite, rewrites those entries of s and q (q = rint(min 2^16), the
// quantisation of the minimum).  With no finite score at all the minimum is
// taken as 0.
// ---------------------------------------------------------------------------
namespace base {
namespace routing {

constexpr int kSanThreads = 256;
constexpr int kSanMaxBlocks = 1024;

__device__ __forceinline__ void block_min_count(float& m, int& c, float* s_m, int* s_c) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        m = fminf(m, __shfl_xor_sync(0xffffffffu, m, off));
        c += __shfl_xor_sync(0xffffffffu, c, off);
    }
    if (lane_id() == 0) {
        s_m[warp_id()] = m;
        s_c[warp_id()] = c;
    }
    __syncthreads();
    if (warp_id() == 0) {
        const int nw = blockDim.x / kWarp;
        m = lane_id() < nw ? s_m[lane_id()] : INFINITY;
        c = lane_id() < nw ? s_c[lane_id()] : 0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            m = fminf(m, __shfl_xor_sync(0xffffffffu, m, off));
            c += __shfl_xor_sync(0xffffffffu, c, off);
        }
        if (lane_id() == 0) {
            s_m[0] = m;
            s_c[0] = c;
        }
    }
    __syncthreads();
    m = s_m[0];
    c = s_c[0];
}

__global__ void __launch_bounds__(kSanThreads) sanitize_reduce_kernel(const float* __restrict__ s,
                                                                      long long n,
                                                                      float* __restrict__ pmin,
                                                                      int* __restrict__ pcnt) {
    __shared__ float s_m[32];
    __shared__ int s_c[32];
    float m = INFINITY;
    int c = 0;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const float v = __ldg(s + i);
        if (isfinite(v)) m = fminf(m, v);
        else ++c;
    }
    block_min_count(m, c, s_m, s_c);
    if (threadIdx.x == 0) {
        pmin[blockIdx.x] = m;
        pcnt[blockIdx.x] = c;
    }
}

__global__ void __launch_bounds__(kSanThreads) sanitize_fix_kernel(float* __restrict__ s,
                                                                   int32_t* __restrict__ q,
                                                                   long long n, int nparts,
                                                                   const float* __restrict__ pmin,
                                                                   const int* __restrict__ pcnt) {
    __shared__ float s_m[32];
    __shared__ int s_c[32];
    float m = INFINITY;
    int c = 0;
    for (int i = threadIdx.x; i < nparts; i += blockDim.x) {
        m = fminf(m, pmin[i]);
        c += pcnt[i];
    }
    block_min_count(m, c, s_m, s_c);
    if (c == 0) return;
    if (!isfinite(m)) m = 0.f;  // nothing finite
    const int32_t qm = quantize_score(m);
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        if (!isfinite(s[i])) {
            s[i] = m;
            if (q) q[i] = qm;
        }
    }
}

}  // namespace routing

size_t sanitize_workspace_bytes() {
    return align_up(2 * sizeof(float) * routing::kSanMaxBlocks, 256);
}

int launch_sanitize_scores(float* s, int32_t* q, int T, int E, void* ws, cudaStream_t stream) {
    using namespace routing;
    const long long n = (long long)T * E;
    long long blocks = (n + kSanThreads * 4 - 1) / (kSanThreads * 4);
    if (blocks > num_sms() * 4) blocks = num_sms() * 4;
    if (blocks > kSanMaxBlocks) blocks = kSanMaxBlocks;
    if (blocks < 1) blocks = 1;
    float* pmin = static_cast<float*>(ws);
    int* pcnt = reinterpret_cast<int*>(pmin + kSanMaxBlocks);
    sanitize_reduce_kernel<<<(int)blocks, kSanThreads, 0, stream>>>(s, n, pmin, pcnt);
    BASE_RETURN_IF_LAUNCH_FAILED();
    sanitize_fix_kernel<<<(int)blocks, kSanThreads, 0, stream>>>(s, q, n, (int)blocks, pmin, pcnt);
    BASE_RETURN_IF_LAUNCH_FAILED();
    return BASE_OK;
}

}  // namespace base
