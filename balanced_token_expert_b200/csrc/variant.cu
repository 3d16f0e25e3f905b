// variant.cu -- the layer norm of the released code's expert sublayers
// ("BASE Layers: Simplifying Training of Large, Sparse Models", wikillm.com
// summary, "Placement and shape": each expert sublayer is layer norm,
// projection up, ReLU, projection back and a residual connection).  It runs
// on the slot-ordered tokens with the gain and bias of each row's expert; the
// projections and the residual / blend run in the tensor-core GEMM.
#include "common.cuh"

namespace base {
namespace variant {

constexpr int kLnThreads = 256;  // 8 warps; one warp per row
constexpr float kLnEps = 1e-5f;  // the pages name no epsilon: the common default

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// y[r] = (x[r] - mean) / sqrt(var + eps) * gamma[e] + beta[e] for the row's
// expert e (offsets[e] <= r < offsets[e + 1]); biased variance; statistics
// in fp32 from two passes over the row (the second from L1).
__global__ void __launch_bounds__(kLnThreads) layer_norm_rows_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ offsets, int T, int D, int E,
    const float* __restrict__ gamma, const float* __restrict__ beta, int stride,
    __nv_bfloat16* __restrict__ y) {
    extern __shared__ int32_t s_off[];  // E + 1
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = __ldg(offsets + i);
    __syncthreads();
    const int lane = lane_id();
    const int nv = D / 8;
    const int wpb = blockDim.x / kWarp;
    for (long long r = (long long)blockIdx.x * wpb + warp_id(); r < T;
         r += (long long)gridDim.x * wpb) {
        int lo = 0, hi = E;  // the last e with offsets[e] <= r
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_off[mid] <= r) lo = mid;
            else hi = mid;
        }
        const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)r * D);
        float sum = 0.f;
        for (int v = lane; v < nv; v += kWarp) {
            float f[8];
            bf16x8_to_f32(__ldg(xr + v), f);
#pragma unroll
            for (int i = 0; i < 8; ++i) sum += f[i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float mean = sum / (float)D;
        float sq = 0.f;
        for (int v = lane; v < nv; v += kWarp) {
            float f[8];
            bf16x8_to_f32(__ldg(xr + v), f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float d = f[i] - mean;
                sq = fmaf(d, d, sq);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
        const float rstd = rsqrtf(sq / (float)D + kLnEps);
        const float4* g4 = reinterpret_cast<const float4*>(gamma + (size_t)lo * stride);
        const float4* b4 = reinterpret_cast<const float4*>(beta + (size_t)lo * stride);
        uint4* yr = reinterpret_cast<uint4*>(y + (size_t)r * D);
        for (int v = lane; v < nv; v += kWarp) {
            float f[8];
            bf16x8_to_f32(__ldg(xr + v), f);
            const float4 ga = __ldg(g4 + 2 * v), gb = __ldg(g4 + 2 * v + 1);
            const float4 ba = __ldg(b4 + 2 * v), bb = __ldg(b4 + 2 * v + 1);
            const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            const float b[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = fmaf((f[i] - mean) * rstd, g[i], b[i]);
            uint4 w;
            w.x = __bfloat16_as_ushort(__float2bfloat16_rn(o[0])) |
                  ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o[1])) << 16);
            w.y = __bfloat16_as_ushort(__float2bfloat16_rn(o[2])) |
                  ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o[3])) << 16);
            w.z = __bfloat16_as_ushort(__float2bfloat16_rn(o[4])) |
                  ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o[5])) << 16);
            w.w = __bfloat16_as_ushort(__float2bfloat16_rn(o[6])) |
                  ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o[7])) << 16);
            yr[v] = w;
        }
    }
}

}  // namespace variant

// gamma, beta: the parameters of expert 0 for this sublayer; expert e's at
// e * stride floats further (16-byte aligned rows: D % 8 == 0, stride % 4 == 0)
int launch_layer_norm_rows(const void* x, const int32_t* offsets, int T, int D, int E,
                           const float* gamma, const float* beta, int stride, void* y,
                           cudaStream_t stream) {
    using namespace variant;
    const int wpb = kLnThreads / kWarp;
    long long blocks = ((long long)T + wpb - 1) / wpb;
    if (blocks > num_sms() * 8) blocks = num_sms() * 8;
    if (blocks < 1) blocks = 1;
    layer_norm_rows_kernel<<<(int)blocks, kLnThreads, sizeof(int32_t) * (E + 1), stream>>>(
        static_cast<const __nv_bfloat16*>(x), offsets, T, D, E, gamma, beta, stride,
        static_cast<__nv_bfloat16*>(y));
    BASE_RETURN_IF_LAUNCH_FAILED();
    return BASE_OK;
}

}  // namespace base
