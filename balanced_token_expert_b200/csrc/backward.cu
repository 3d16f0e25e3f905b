// backward.cu -- gradient of the BASE layer with the assignment held fixed.
//
// The released code computes the routing affinities without gradient and the
// centroids receive gradient only through the sigmoid gate ("Paper vs code",
// gradient into routing), so for L = <out, dout>:
//   dy = dout[perm];  dgate = <dy, f>;  ds = dgate sigma (1 - sigma)
//   dF = sigma dy;    dH1 = dF W2_e;    dA1 = dH1 * act'(A1)
//   dW2_e = dF_e^T H1_e;  dW1_e = dA1_e^T x_e
//   dx = dA1 W1_e + dy + ds w_e;  dh[perm[r]] = dx[r]
//   dw_e = sum over the expert's slots of ds_r x_r
// The four contractions run on the tcgen05 GEMM: dH1 and dx read the
// weights as MN-major operands (no transposed copy), dW1 / dW2 read the
// activations as MN-major operands and reduce over each expert's slot range.
#include <algorithm>

#include "common.cuh"

namespace base {

int launch_move_rows(const void* src, const int32_t* idx, int T, int D, void* dst, bool scatter,
                     cudaStream_t stream);
int launch_bwd_gemms(const void* dF, const void* dA1_in, void* dA1, const void* a1, const void* h1,
                     const void* x_perm, const void* dy, const float* ds, const void* w,
                     const int32_t* perm, const int32_t* offsets, int32_t* tile_start,
                     const void* W1, const void* W2, int act, int T, int D, int E, int F,
                     void* dh, float* dW1, float* dW2, cudaStream_t stream);

namespace bwd {

// dF = sigma(gate) dy (bf16) and ds = <dy, f> sigma (1 - sigma), one warp per slot
__global__ void gate_grad_kernel(const __nv_bfloat16* __restrict__ dy,
                                 const __nv_bfloat16* __restrict__ f,
                                 const float* __restrict__ gate, int T, int D,
                                 __nv_bfloat16* __restrict__ dF, float* __restrict__ ds,
                                 const int32_t* __restrict__ offsets, int E, int C) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int e = 0; e <= E; ++e)
            if (offsets[e] != e * C) {
                record_error(4001);  // the backward needs the balanced slot layout
                break;
            }
    }
    const int lane = lane_id();
    const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / kWarp;
    const long long nw = (gridDim.x * (long long)blockDim.x) / kWarp;
    const int vec = D / 8;
    for (long long r = gw; r < T; r += nw) {
        const float g = gate[r];
        const float sg = 1.f / (1.f + expf(-g));
        const uint4* dyr = reinterpret_cast<const uint4*>(dy + (size_t)r * D);
        const uint4* fr = reinterpret_cast<const uint4*>(f + (size_t)r * D);
        uint4* dFr = reinterpret_cast<uint4*>(dF + (size_t)r * D);
        float dot = 0.f;
        for (int j = lane; j < vec; j += kWarp) {
            const uint4 a = __ldg(dyr + j), b = __ldg(fr + j);
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a0 = __uint_as_float(av[i] << 16), a1 = __uint_as_float(av[i] & 0xFFFF0000u);
                const float b0 = __uint_as_float(bv[i] << 16), b1 = __uint_as_float(bv[i] & 0xFFFF0000u);
                dot = fmaf(a0, b0, dot);
                dot = fmaf(a1, b1, dot);
                const __nv_bfloat162 p = __floats2bfloat162_rn(sg * a0, sg * a1);
                o[i] = *reinterpret_cast<const uint32_t*>(&p);
            }
            dFr[j] = make_uint4(o[0], o[1], o[2], o[3]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (lane == 0) ds[r] = dot * sg * (1.f - sg);
    }
}

// dw[e][d] = sum_{r in segment e} ds[r] x_perm[r][d], in two deterministic
// steps.  Partials: a block per (2048 columns, expert, row split), every
// thread 8 consecutive columns read as one 16-byte vector per row; the
// partial sums go to part[z][e][d].  Then every (e, d) adds its splits in
// order.  HBM-bound: the T x D bf16 rows are read once.
__global__ void __launch_bounds__(256) centroid_grad_partial_kernel(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ ds,
    const int32_t* __restrict__ offsets, int D, int E, int splits, float* __restrict__ part) {
    const int e = blockIdx.y, z = blockIdx.z;
    const int d0 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    const int r0 = __ldg(offsets + e), r1 = __ldg(offsets + e + 1);
    const int per = (r1 - r0 + splits - 1) / splits;
    const int a = r0 + z * per, b = min(r1, a + per);
    if (d0 >= D) return;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int r = a; r < b; ++r) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)r * D + d0));
        const float sv = __ldg(ds + r);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] = fmaf(sv, __uint_as_float(w[i] << 16), acc[2 * i]);
            acc[2 * i + 1] = fmaf(sv, __uint_as_float(w[i] & 0xFFFF0000u), acc[2 * i + 1]);
        }
    }
    float4* o = reinterpret_cast<float4*>(part + ((size_t)z * E + e) * D + d0);
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

__global__ void centroid_grad_reduce_kernel(const float* __restrict__ part, int splits, long long n,
                                            float* __restrict__ dw) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int z = 0; z < splits; ++z) acc += __ldg(part + (size_t)z * n + i);
        dw[i] = acc;
    }
}

static int centroid_splits(int E, int D, int C) {
    const int bxy = ((D / 8 + 255) / 256) * E;
    int splits = (8 * num_sms() + bxy - 1) / bxy;
    splits = std::min(splits, std::max(1, C / 16));
    return std::max(1, std::min(splits, 64));
}

}  // namespace bwd

size_t backward_workspace_bytes(int T, int E, int D, int F) {
    size_t b = 0;
    b += align_up((size_t)T * D * 2, 256);  // dy
    b += align_up((size_t)T * D * 2, 256);  // dF
    b += align_up((size_t)T * 4, 256);      // ds
    b += align_up((size_t)T * F * 2, 256);  // dA1
    b += align_up((size_t)(E + 1) * 4, 256);
    b += align_up(sizeof(float) * 64 * (size_t)E * D, 256);  // centroid-gradient partials
    return b;
}

int launch_layer_bwd(const void* h, const void* w, const void* W1, const void* W2, int act, int T,
                     int D, int E, int F, const base_layer_saved* sv, const void* dout, void* dh,
                     float* dw, float* dW1, float* dW2, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
    (void)h;
    if (T % E != 0 || (T / E) % 64 != 0 || D % 64 != 0 || F % 64 != 0) return BASE_ERR_UNSUPPORTED;
    const int C = T / E;
    unsigned char* p = static_cast<unsigned char*>(ws);
    size_t o = 0;
    __nv_bfloat16* dy = reinterpret_cast<__nv_bfloat16*>(p + o); o += align_up((size_t)T * D * 2, 256);
    __nv_bfloat16* dF = reinterpret_cast<__nv_bfloat16*>(p + o); o += align_up((size_t)T * D * 2, 256);
    float* ds = reinterpret_cast<float*>(p + o); o += align_up((size_t)T * 4, 256);
    __nv_bfloat16* dA1 = reinterpret_cast<__nv_bfloat16*>(p + o); o += align_up((size_t)T * F * 2, 256);
    int32_t* tile_start = reinterpret_cast<int32_t*>(p + o); o += align_up((size_t)(E + 1) * 4, 256);
    float* dw_part = reinterpret_cast<float*>(p + o); o += align_up(sizeof(float) * 64 * (size_t)E * D, 256);
    if (o > ws_bytes) return BASE_ERR_WORKSPACE;

    int st = launch_move_rows(dout, sv->perm, T, D, dy, false, stream);
    if (st != BASE_OK) return st;
    {
        const int threads = 256;
        long long blocks = ((long long)T * kWarp + threads - 1) / threads;
        if (blocks > num_sms() * 16) blocks = num_sms() * 16;
        bwd::gate_grad_kernel<<<(int)blocks, threads, 0, stream>>>(
            dy, static_cast<const __nv_bfloat16*>(sv->f), sv->gate, T, D, dF, ds, sv->offsets, E, C);
        BASE_RETURN_IF_LAUNCH_FAILED();
    }
    {
        const int splits = bwd::centroid_splits(E, D, C);
        dim3 grid((D / 8 + 255) / 256, E, splits);
        bwd::centroid_grad_partial_kernel<<<grid, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(sv->x_perm), ds, sv->offsets, D, E, splits, dw_part);
        BASE_RETURN_IF_LAUNCH_FAILED();
        const long long n = (long long)E * D;
        long long blocks = (n + 255) / 256;
        if (blocks > num_sms() * 8) blocks = num_sms() * 8;
        bwd::centroid_grad_reduce_kernel<<<(int)blocks, 256, 0, stream>>>(dw_part, splits, n, dw);
        BASE_RETURN_IF_LAUNCH_FAILED();
    }
    return launch_bwd_gemms(dF, nullptr, dA1, sv->a1, sv->h1, sv->x_perm, dy, ds, w, sv->perm,
                            sv->offsets, tile_start, W1, W2, act, T, D, E, F, dh, dW1, dW2, stream);
}

}  // namespace base
