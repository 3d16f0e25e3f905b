// gemm.cu -- persistent, warp-specialised tcgen05 GEMM for sm_100a with the
// BASE layer's epilogues fused in.
//
//   D[m, n] = sum_k A[m, k] B[n, k]     A, B bf16 in global memory, fp32 in TMEM
//
// Rows of A may be split into groups (the experts' slot segments,
// offsets[g] .. offsets[g+1]); group g multiplies with its own block of B
// rows (the expert's weight matrix).  Tiles are 128 x BN x 64:
//   warp 0      one lane issues TMA loads of the A and B tiles into a ring of
//               STAGES shared-memory stages (128-byte swizzle),
//   warp 1      allocates TMEM (two BN-column fp32 accumulators) and one lane
//               issues tcgen05.mma (M=128, N=BN, K=16) per 16-wide K slice,
//   warps 4..11 the epilogue: tcgen05.ld of the accumulator (warp w reads
//               TMEM lanes 32 (w%4) .., two warps per lane quadrant split the
//               columns), the fused element-wise work and 16-byte stores; the
//               two accumulators let the epilogue of one tile overlap the MMAs
//               of the next.
// Operands may also be MN-major (A stored K x M, B stored K x N, M/N
// contiguous), read as 64 x 64 TMA boxes and described to the tensor core as
// MN-major 128-byte-swizzled tiles; the backward uses this to multiply by
// transposed activations and weights without transposing them in memory.
// In K-grouped mode (the weight gradients) group g reduces over its own slot
// range offsets[g] .. offsets[g+1] along K and writes its own M x N block.
// Every mbarrier wait is bounded; a wait that gives up records an error code
// in the device error word and the kernel winds down (waiting, bounded, for
// its own TMA copies and MMAs in flight, then freeing TMEM).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "tc.cuh"

namespace base {
namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;
// warp 0: TMA, warp 1: MMA, warps 2-3: idle, warps 4..: epilogue, two per
// TMEM lane quadrant (warp w reads lanes 32 (w % 4) ..), each half the columns
constexpr int kEpiWarps = 8;
constexpr int kTsSmem = 384;  // groups + 1 whose tile prefix a grouped GEMM computes itself
constexpr int kThreads = 128 + 32 * kEpiWarps;

enum Epi : int {
    EPI_SCORES = 0,  // s (fp32) and q = rint(s 2^16) (int32)
    EPI_ACT = 1,     // h1 = act(acc) bf16, a1 = acc bf16 (optional)
    EPI_GATE = 2,    // y = sigmoid(gate[row]) acc + x[row] bf16, f = acc bf16 (optional);
                     // mix 1: y = acc + x[row]; mix 2: y = x0 + a (acc + x[row] - x0),
                     // a = sigmoid(gate[row]), x0 = side2[row]
    EPI_DACT = 3,    // dA1 = acc * act'(a1[row]) bf16
    EPI_DX = 4,      // dh[idx[row]] = acc + dy[row] + ds[row] w_g  bf16
    EPI_F32 = 5,     // out_f32[g][row][col] = acc (K-grouped weight gradients)
};

struct Args {
    int M;                       // rows of A
    int N;                       // columns of D per group (rows of B per group)
    int K;
    int groups;                  // 1 when offsets == nullptr
    const int32_t* offsets;      // [groups+1] row segments of A (nullable)
    const int32_t* tile_start;   // [groups+1] prefix sums of the groups' 128-row tiles
    int b_rows_per_group;        // row offset of group g's B block = g * b_rows_per_group
    int n_tiles;                 // ceil(N / BN)
    int ld;                      // row stride (elements) of outputs and side inputs
    int act;                     // base_act
    float* out_f32;
    int32_t* out_q;
    __nv_bfloat16* out0;
    __nv_bfloat16* out1;
    const float* gate;
    const __nv_bfloat16* side;
    const __nv_bfloat16* side2;  // centroids w (EPI_DX)
    const int32_t* idx;          // destination rows (EPI_DX)
    int kgroup;                  // 1: groups split K (weight gradients), M and N fixed
    int m_tiles;                 // K-grouped mode: tiles along M per group
    int mix;                     // EPI_GATE: 0 eq. 1, 1 residual only, 2 residual then blend
    int32_t* out_assign;         // EPI_SCORES, one N tile: greedy argmax of q per row (nullable)
    int32_t* out_counts;         // with out_assign: tokens per expert, added to (zeroed by the host)
    int staged;                  // set by the launcher: output tensor maps are valid
    unsigned long long wait_ns;  // set by the launcher: limit of every bounded wait
    int drop_first_load;         // set by the launcher: test hook (one-CTA kernels only)
};

struct TileInfo {
    int group, a_row, b_row, n0, m_local0, group_rows;
    int k0, kblocks;  // first K index and number of 64-wide K blocks
};

// bm: rows of A per tile (128, or 256 for a CTA pair)
// ts: the groups' tile prefix (shared memory when the kernel computed it,
// else a.tile_start); read with plain loads
__device__ __forceinline__ TileInfo decode_tile(const Args& a, int tile, int bn, int bm,
                                                const int32_t* ts_) {
    TileInfo ti;
    ti.k0 = 0;
    ti.kblocks = (a.K + BK - 1) / BK;
    if (a.kgroup) {
        const int per = a.m_tiles * a.n_tiles;
        const int g = tile / per, local = tile % per;
        const int nt = local / a.m_tiles, m = local % a.m_tiles;
        const int k0 = __ldg(a.offsets + g);
        ti.group = g;
        ti.a_row = m * bm;
        ti.m_local0 = m * bm;
        ti.group_rows = a.M;
        ti.n0 = nt * bn;
        ti.b_row = nt * bn;
        ti.k0 = k0;
        ti.kblocks = (__ldg(a.offsets + g + 1) - k0) / BK;
        return ti;
    }
    if (a.offsets == nullptr) {
        const int mt = (a.M + bm - 1) / bm;
        const int nt = tile / mt, m = tile % mt;
        ti.group = 0;
        ti.a_row = m * bm;
        ti.m_local0 = m * bm;
        ti.group_rows = a.M;
        ti.n0 = nt * bn;
        ti.b_row = nt * bn;
        return ti;
    }
    // group g holds tiles [tile_start[g] * n_tiles, tile_start[g+1] * n_tiles)
    int lo = 0, hi = a.groups;  // find the last g with tile_start[g] * n_tiles <= tile
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ts_[mid] * a.n_tiles <= tile) lo = mid; else hi = mid;
    }
    const int g = lo;
    const int ts = ts_[g];
    const int mtg = ts_[g + 1] - ts;
    const int local = tile - ts * a.n_tiles;
    const int nt = local / mtg, m = local % mtg;
    const int r0 = __ldg(a.offsets + g);
    ti.group = g;
    ti.a_row = r0 + m * bm;
    ti.m_local0 = m * bm;
    ti.group_rows = __ldg(a.offsets + g + 1) - r0;
    ti.n0 = nt * bn;
    ti.b_row = g * a.b_rows_per_group + nt * bn;
    return ti;
}

__device__ __forceinline__ float act_fwd(float x, int act) {
    if (act == BASE_RELU) return fmaxf(x, 0.f);
    return 0.5f * x * (1.f + erff(x * 0.70710678118654752f));
}

__device__ __forceinline__ float act_grad(float x, int act) {
    if (act == BASE_RELU) return x > 0.f ? 1.f : 0.f;
    return 0.5f * (1.f + erff(x * 0.70710678118654752f)) +
           x * expf(-0.5f * x * x) * 0.39894228040143268f;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void store_bf16x16(__nv_bfloat16* dst, const float (&f)[16]) {
    uint4 a, b;
    a.x = pack_bf16x2(f[0], f[1]);
    a.y = pack_bf16x2(f[2], f[3]);
    a.z = pack_bf16x2(f[4], f[5]);
    a.w = pack_bf16x2(f[6], f[7]);
    b.x = pack_bf16x2(f[8], f[9]);
    b.y = pack_bf16x2(f[10], f[11]);
    b.z = pack_bf16x2(f[12], f[13]);
    b.w = pack_bf16x2(f[14], f[15]);
    uint4* d = reinterpret_cast<uint4*>(dst);
    d[0] = a;
    d[1] = b;
}

__device__ __forceinline__ void load_bf16x16(const __nv_bfloat16* src, float (&f)[16]) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
    const uint4 a = __ldg(s), b = __ldg(s + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// 16 accumulator columns [col, col+16) of one row.
template <int EPI>
__device__ __forceinline__ void epilogue16(const Args& a, const TileInfo& ti, int row, int col,
                                           const uint32_t (&v)[16]) {
    float f[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]);
    const size_t base = (size_t)row * a.ld + col;
    if constexpr (EPI == EPI_SCORES) {
        if (col + 16 <= a.N && (a.ld & 3) == 0) {
            if (a.out_f32) {
                float4* d = reinterpret_cast<float4*>(a.out_f32 + base);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    d[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
            }
            if (a.out_q) {
                int4* d = reinterpret_cast<int4*>(a.out_q + base);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    d[i] = make_int4(quantize_score(f[4 * i]), quantize_score(f[4 * i + 1]),
                                     quantize_score(f[4 * i + 2]), quantize_score(f[4 * i + 3]));
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (col + i < a.N) {
                    if (a.out_f32) a.out_f32[base + i] = f[i];
                    if (a.out_q) a.out_q[base + i] = quantize_score(f[i]);
                }
            }
        }
    } else if constexpr (EPI == EPI_ACT) {
        float h[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) h[i] = act_fwd(f[i], a.act);
        if (col + 16 <= a.N) {
            if (a.out1) store_bf16x16(a.out1 + base, f);
            store_bf16x16(a.out0 + base, h);
        } else {
            for (int i = 0; i < a.N - col; ++i) {
                if (a.out1) a.out1[base + i] = __float2bfloat16_rn(f[i]);
                a.out0[base + i] = __float2bfloat16_rn(h[i]);
            }
        }
    } else if constexpr (EPI == EPI_GATE) {
        const float sg = a.mix == 1 ? 1.f : 1.f / (1.f + expf(-__ldg(a.gate + row)));
        if (col + 16 <= a.N) {
            if (a.out1) store_bf16x16(a.out1 + base, f);
            float x[16];
            load_bf16x16(a.side + base, x);
            if (a.mix == 2) {
                float x0[16];
                load_bf16x16(a.side2 + base, x0);
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = fmaf(sg, (f[i] + x[i]) - x0[i], x0[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = fmaf(sg, f[i], x[i]);
            }
            store_bf16x16(a.out0 + base, x);
        } else {
            for (int i = 0; i < a.N - col; ++i) {
                if (a.out1) a.out1[base + i] = __float2bfloat16_rn(f[i]);
                const float x = __bfloat162float(a.side[base + i]);
                float y;
                if (a.mix == 2) {
                    const float x0 = __bfloat162float(a.side2[base + i]);
                    y = fmaf(sg, (f[i] + x) - x0, x0);
                } else {
                    y = fmaf(sg, f[i], x);
                }
                a.out0[base + i] = __float2bfloat16_rn(y);
            }
        }
    } else if constexpr (EPI == EPI_DACT) {
        const int nv = min(16, a.N - col);
        if (nv == 16) {
            float x[16];
            load_bf16x16(a.side + base, x);
#pragma unroll
            for (int i = 0; i < 16; ++i) f[i] *= act_grad(x[i], a.act);
            store_bf16x16(a.out0 + base, f);
        } else {
            for (int i = 0; i < nv; ++i)
                a.out0[base + i] = __float2bfloat16_rn(
                    f[i] * act_grad(__bfloat162float(a.side[base + i]), a.act));
        }
    } else if constexpr (EPI == EPI_DX) {
        const float ds = __ldg(a.gate + row);
        const __nv_bfloat16* wg = a.side2 + (size_t)ti.group * a.N + col;
        const size_t dst = (size_t)__ldg(a.idx + row) * a.ld + col;
        const int nv = min(16, a.N - col);
        if (nv == 16) {
            float dy[16], wv[16];
            load_bf16x16(a.side + base, dy);
            load_bf16x16(wg, wv);
#pragma unroll
            for (int i = 0; i < 16; ++i) f[i] = f[i] + dy[i] + ds * wv[i];
            store_bf16x16(a.out0 + dst, f);
        } else {
            for (int i = 0; i < nv; ++i)
                a.out0[dst + i] = __float2bfloat16_rn(f[i] + __bfloat162float(a.side[base + i]) +
                                                      ds * __bfloat162float(wg[i]));
        }
    } else if constexpr (EPI == EPI_F32) {
        float* o = a.out_f32 + (size_t)ti.group * a.M * a.N + (size_t)row * a.N + col;
        const int nv = min(16, a.N - col);
        if (nv == 16 && (a.N & 3) == 0) {
            float4* d = reinterpret_cast<float4*>(o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                d[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
        } else {
            for (int i = 0; i < nv; ++i) o[i] = f[i];
        }
    }
}

// The epilogues whose output rows are contiguous (h1 / a1, y / f, dA1, dW)
// stage each warp's 32 rows x 128 bytes of output in shared memory and write
// them with one TMA store: 128-byte line writes instead of 16-byte pieces of
// 32 different rows per instruction.
template <int EPI>
constexpr bool kStagedEpi = EPI == EPI_ACT || EPI == EPI_GATE || EPI == EPI_DACT || EPI == EPI_F32;
constexpr uint32_t kStageBuf = 32 * 128;  // one warp's 32 rows x 128 bytes
constexpr int kStageSlots = 2;            // per epilogue warp

// the 16 output values of pass 0 (out0 / out_f32) or pass 1 (out1: the raw
// accumulator) for columns [col, col + 16) of one row
template <int EPI>
__device__ __forceinline__ void epi_values16(const Args& a, int row, int col, int pass,
                                             const uint32_t (&v)[16], float (&o)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = __uint_as_float(v[i]);
    if (pass == 1) return;
    const size_t base = (size_t)row * a.ld + col;
    if constexpr (EPI == EPI_ACT) {
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = act_fwd(o[i], a.act);
    } else if constexpr (EPI == EPI_GATE) {
        const float sg = a.mix == 1 ? 1.f : 1.f / (1.f + expf(-__ldg(a.gate + row)));
        float x[16];
        load_bf16x16(a.side + base, x);
        if (a.mix == 2) {
            float x0[16];
            load_bf16x16(a.side2 + base, x0);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = fmaf(sg, (o[i] + x[i]) - x0[i], x0[i]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = fmaf(sg, o[i], x[i]);
        }
    } else if constexpr (EPI == EPI_DACT) {
        float x[16];
        load_bf16x16(a.side + base, x);
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] *= act_grad(x[i], a.act);
    }
}

// row `lane` of a 32 x 128-byte staging buffer in the TMA 128-byte swizzle
// (16-byte unit u of row r sits at unit u ^ (r % 8)); c = first column
template <bool F32OUT>
__device__ __forceinline__ void stage16(uint8_t* buf, int lane, int c, const float (&o)[16]) {
    uint4* rowp = reinterpret_cast<uint4*>(buf + lane * 128);
    const int sw = lane & 7;
    if constexpr (F32OUT) {
        const int u0 = c >> 2;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            rowp[(u0 + i) ^ sw] = make_uint4(__float_as_uint(o[4 * i]), __float_as_uint(o[4 * i + 1]),
                                             __float_as_uint(o[4 * i + 2]),
                                             __float_as_uint(o[4 * i + 3]));
    } else {
        const int u0 = c >> 3;
        rowp[u0 ^ sw] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                   pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
        rowp[(u0 + 1) ^ sw] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]),
                                         pack_bf16x2(o[12], o[13]), pack_bf16x2(o[14], o[15]));
    }
}

// CG = 2: a CTA pair of a cluster computes a (2 x 128) x BN tile with
// tcgen05.mma.cta_group::2: each CTA loads its own 128 rows of A and BN/2 rows
// of B (the TMA completions of both land on the leader's barrier), the leader
// issues the MMAs, each CTA's TMEM holds its 128 rows x BN accumulator and its
// epilogue writes them.
// SLOTS: staging buffers of 32 x 128 bytes per epilogue warp (one frees shared
// memory for a sixth pipeline stage)
template <int BN, int STAGES, int EPI, bool A_MN, bool B_MN, int CG = 1, int SLOTS = kStageSlots>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                const Args args) {
    static_assert(CG == 1 || CG == 2, "one CTA or a CTA pair");
    static_assert(BN % 16 == 0 && kEpiWarps == 8, "16-column chunks over two column halves");
    constexpr int BNC = BN / CG;  // rows of B loaded by one CTA
    constexpr int BMP = BM * CG;  // rows of A per tile
    constexpr uint32_t A_BYTES = BM * BK * 2;
    constexpr uint32_t B_BYTES = BNC * BK * 2;
    constexpr uint32_t TMEM_COLS = (2 * BN < 32) ? 32 : 2 * BN;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    constexpr bool kStaged = kStagedEpi<EPI>;
    constexpr uint32_t STAGE_AREA = kStaged ? kEpiWarps * SLOTS * kStageBuf : 0;
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_BYTES;
    uint8_t* sOut = smem + STAGES * (A_BYTES + B_BYTES);  // 1024-byte aligned
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + STAGE_AREA);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* done = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    // EPI_SCORES with greedy routing: the CTA's tokens per expert (after the 256
    // bytes of barriers)
    int32_t* s_ghist = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(full) + 256);
    constexpr bool kGreedy = EPI == EPI_SCORES;
    const bool greedy = kGreedy && args.out_assign != nullptr;

    const int warp = warp_id(), lane = lane_id();
    if (greedy)
        for (int e = threadIdx.x; e < args.N; e += blockDim.x) s_ghist[e] = 0;
    const uint32_t rank = (CG == 2) ? tc::cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit = (CG == 2) ? (int)(blockIdx.x / 2) : (int)blockIdx.x;
    const int nunits = (CG == 2) ? (int)(gridDim.x / 2) : (int)gridDim.x;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&tfull[i], 1);
            tc::mbar_init(&tempty[i], kEpiWarps * CG);
        }
        tc::mbar_init(done, 1);
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        if constexpr (CG == 2) {
            tc::tmem_alloc_cg2(tmem_slot, TMEM_COLS);
            tc::tmem_relinquish_cg2();
        } else {
            tc::tmem_alloc(tmem_slot, TMEM_COLS);
            tc::tmem_relinquish();
        }
    }
    if (warp == 0 && lane == 0) {
        tc::tma_prefetch_desc(&tmA);
        tc::tma_prefetch_desc(&tmB);
    }
    // launched behind another kernel (programmatic dependent launch): the set-up
    // above overlapped its tail; nothing it writes is read before this point
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // grouped tiles: the groups' tile prefix (a group of r rows has ceil(r / BMP)
    // row tiles) computed here by the idle warp 3 when the launcher passed none
    int32_t* s_ts = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(full) + 256);
    const bool ts_smem = args.offsets != nullptr && !args.kgroup && args.tile_start == nullptr;
    if (ts_smem && warp == 3) {
        int run = 0;
        for (int base = 0; base <= args.groups; base += 32) {
            const int g = base + lane;
            const int v = g < args.groups
                              ? (__ldg(args.offsets + g + 1) - __ldg(args.offsets + g) + BMP - 1) / BMP
                              : 0;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            if (g <= args.groups) s_ts[g] = run + incl - v;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    // every CTA of this grid is resident (one per SM, persistent): the next
    // kernel may start its own set-up on SMs as they free up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int32_t* tsp = ts_smem ? s_ts : args.tile_start;
    if constexpr (CG == 2) tc::cluster_sync_all();  // both CTAs' barriers and TMEM are ready
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int mtiles = args.kgroup ? args.m_tiles * args.groups
                       : args.offsets ? tsp[args.groups]
                                      : (args.M + BMP - 1) / BMP;
    const int total = mtiles * args.n_tiles;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer (both CTAs of a pair) ----------------
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        uint32_t issued_parity[STAGES];
        bool issued[STAGES];
        for (int s = 0; s < STAGES; ++s) issued[s] = false;
        for (int tile = unit; tile < total && ok; tile += nunits) {
            const TileInfo ti = decode_tile(args, tile, BN, BMP, tsp);
            const int a_row = ti.a_row + BM * (int)rank;
            for (int kb = 0; kb < ti.kblocks; ++kb) {
                if (!tc::mbar_wait(&empty[stage], phase ^ 1, 3001, args.wait_ns)) {
                    ok = false;
                    break;
                }
                if constexpr (CG == 1) {
                    // test hook: CTA 0's first load is never issued, so the MMA
                    // warp's wait for it runs out (the other copies still land)
                    if (args.drop_first_load && blockIdx.x == 0 && tile == unit && kb == 0) {
                        issued[stage] = false;
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                        continue;
                    }
                }
                uint32_t fbar;
                if constexpr (CG == 2) {
                    if (leader) tc::mbar_arrive_expect_tx(&full[stage], CG * (A_BYTES + B_BYTES));
                    fbar = tc::map_to_rank(&full[stage], 0);
                } else {
                    tc::mbar_arrive_expect_tx(&full[stage], A_BYTES + B_BYTES);
                    fbar = smem_u32(&full[stage]);
                }
                auto load = [&](void* dst, const CUtensorMap* tm, int c0, int c1) {
                    if constexpr (CG == 2) tc::tma_load_2d_cg2(dst, tm, fbar, c0, c1);
                    else tc::tma_load_2d(dst, tm, &full[stage], c0, c1);
                };
                const int kg = ti.k0 + kb * BK;
                if constexpr (A_MN) {
                    // A stored K x M: two 64(M) x 64(K) boxes
#pragma unroll
                    for (int j = 0; j < BM / 64; ++j)
                        load(sA + stage * A_BYTES + j * 8192, &tmA, a_row + 64 * j, kg);
                } else {
                    load(sA + stage * A_BYTES, &tmA, kg, a_row);
                }
                if constexpr (B_MN) {
                    // B stored K x N: BNC / 64 boxes; the group's K rows start at krow
                    const int krow = args.kgroup ? kg : ti.group * args.b_rows_per_group + kb * BK;
#pragma unroll
                    for (int j = 0; j < BNC / 64; ++j)
                        load(sB + stage * B_BYTES + j * 8192, &tmB,
                             ti.n0 + BNC * (int)rank + 64 * j, krow);
                } else {
                    load(sB + stage * B_BYTES, &tmB, kg, ti.b_row + BNC * (int)rank);
                }
                issued[stage] = true;
                issued_parity[stage] = phase;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (!ok) {
            // wind down: let the copies already issued land before the CTA exits
            // (a pair's copies complete on the leader's barrier: the peer waits
            // a fixed time instead)
            const uint64_t t0 = tc::globaltimer();
            if (CG == 1 || leader) {
                for (int s = 0; s < STAGES; ++s) {
                    if (!issued[s]) continue;
                    const uint32_t a = smem_u32(&full[s]);
                    while (!tc::mbar_try_wait(a, issued_parity[s]) &&
                           tc::globaltimer() - t0 < 100000000ull) {
                    }
                }
            } else {
                while (tc::globaltimer() - t0 < 10000000ull) {
                }
            }
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // ---------------- MMA issuer (the leader of a pair) ----------------
        constexpr uint32_t idesc = tc::idesc_bf16(BMP, BN, A_MN ? 1 : 0, B_MN ? 1 : 0);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = unit; tile < total && ok; tile += nunits) {
            if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, 3002, args.wait_ns)) break;
            tc::tc_fence_after();
            const uint32_t d_tmem = tmem_base + acc * BN;
            // only K-grouped tiles differ in depth (and need the tile's group)
            const int kblocks = args.kgroup ? decode_tile(args, tile, BN, BMP, tsp).kblocks
                                            : (args.K + BK - 1) / BK;
            for (int kb = 0; kb < kblocks; ++kb) {
                if (!tc::mbar_wait(&full[stage], phase, 3003, args.wait_ns)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
                const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    // K-major: the 16-wide K slice is 32 bytes into each 128-byte row;
                    // MN-major: it is 16 rows (2048 bytes) further down the tile
                    const uint64_t ad = A_MN ? tc::smem_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                             : tc::smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                    const uint64_t bd = B_MN ? tc::smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                             : tc::smem_desc_sw128(b_addr + kk * 32, 16, 1024);
                    if constexpr (CG == 2)
                        tc::umma_bf16_cg2(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                    else
                        tc::umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                }
                if constexpr (CG == 2) tc::umma_commit_cg2_mc(&empty[stage], 0x3);
                else tc::umma_commit(&empty[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok) break;
            if constexpr (CG == 2) tc::umma_commit_cg2_mc(&tfull[acc], 0x3);
            else tc::umma_commit(&tfull[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
        // every MMA issued by this thread has finished once `done` flips
        if constexpr (CG == 2) tc::umma_commit_cg2_mc(done, 0x1);
        else tc::umma_commit(done);
        tc::mbar_wait(done, 0, 3004, args.wait_ns);
    } else if (warp >= 4) {
        // ---------------- epilogue ----------------
        const int ew = (warp - 4) & 3;                   // lane quadrant
        const int half = (warp - 4) >> 2;                // column half
        constexpr int kChunks = BN / 16;                 // 16-column chunks per row
        constexpr int kPerHalf = (kChunks + 1) / 2;      // the second half may be empty
        const int c_begin = 16 * min(kChunks, half * kPerHalf);
        const int c_end = 16 * min(kChunks, (half + 1) * kPerHalf);
        int acc = 0;
        uint32_t acc_phase = 0;
        int slot = 0;
        const uint32_t tempty_leader0 = (CG == 2) ? tc::map_to_rank(&tempty[0], 0) : 0u;
        const uint32_t tempty_leader1 = (CG == 2) ? tc::map_to_rank(&tempty[1], 0) : 0u;
        for (int tile = unit; tile < total; tile += nunits) {
            const TileInfo ti = decode_tile(args, tile, BN, BMP, tsp);
            const bool ok = tc::mbar_wait(&tfull[acc], acc_phase, 3005, 2 * args.wait_ns);
            if (!__all_sync(0xffffffffu, ok)) break;  // the whole warp leaves together
            tc::tc_fence_after();
            const int r = BM * (int)rank + ew * 32 + lane;
            const bool valid = ti.m_local0 + r < ti.group_rows;
            const int row = ti.a_row + r;
            const uint32_t tbase = tmem_base + ((uint32_t)(ew * 32) << 16) + acc * BN;
            // staged when the warp's 32 rows all belong to the tile's group
            if (kStaged && args.staged && __all_sync(0xffffffffu, valid)) {
                constexpr int GC = (EPI == EPI_F32) ? 32 : 64;  // columns per 128-byte row piece
                // the warp's first row in the output tensor (dW: group blocks stacked)
                const int orow = (EPI == EPI_F32 ? ti.group * args.M : 0) + ti.a_row +
                                 BM * (int)rank + ew * 32;
                const int npass = (EPI != EPI_F32 && EPI != EPI_DACT && args.out1) ? 2 : 1;
#pragma unroll 1
                for (int gc = c_begin; gc < c_end && ti.n0 + gc < args.N; gc += GC) {
#pragma unroll 1
                    for (int pass = 0; pass < npass; ++pass) {
                        uint8_t* buf = sOut + ((warp - 4) * SLOTS + slot) * kStageBuf;
                        // the store issued from this slot two pieces ago has read it
                        if (lane == 0) tc::bulk_wait_read<SLOTS - 1>();
                        __syncwarp();
#pragma unroll 1
                        for (int c = 0; c < GC; c += 16) {
                            uint32_t v[16];
                            tc::tmem_ld16(tbase + gc + c, v);
                            tc::tmem_wait_ld();
                            if (ti.kblocks == 0) {
#pragma unroll
                                for (int i = 0; i < 16; ++i) v[i] = 0u;
                            }
                            float o[16];
                            epi_values16<EPI>(args, row, ti.n0 + gc + c, pass, v, o);
                            stage16<EPI == EPI_F32>(buf, lane, c, o);
                        }
                        tc::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tc::tma_store_2d(pass ? &tmO1 : &tmO0, buf, ti.n0 + gc, orow);
                            tc::bulk_commit();
                        }
                        slot = (slot + 1) % SLOTS;
                    }
                }
            } else {
                int gbest = INT32_MIN, garg = -1;  // greedy: this half's best q, lowest column
#pragma unroll 1
                for (int c0 = c_begin; c0 < c_end; c0 += 16) {
                    uint32_t v[16];
                    tc::tmem_ld16(tbase + c0, v);
                    tc::tmem_wait_ld();
                    if (ti.kblocks == 0) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = 0u;
                    }
                    if (valid && ti.n0 + c0 < args.N) epilogue16<EPI>(args, ti, row, ti.n0 + c0, v);
                    if constexpr (kGreedy) {
                        if (greedy && half == 0) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int col = ti.n0 + c0 + i;
                                const int32_t qv = quantize_score(__uint_as_float(v[i]));
                                if (col < args.N && qv > gbest) {
                                    gbest = qv;
                                    garg = col;
                                }
                            }
                        }
                    }
                }
                if constexpr (kGreedy) {
                    if (greedy && half == 0) {
                        // the first half also scans the other half's columns (the
                        // same TMEM lanes; nobody frees this accumulator before every
                        // epilogue warp has arrived), lowest column first on ties
#pragma unroll 1
                        for (int c0 = c_end; c0 < 16 * kChunks; c0 += 16) {
                            uint32_t v[16];
                            tc::tmem_ld16(tbase + c0, v);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int col = ti.n0 + c0 + i;
                                const int32_t qv = quantize_score(
                                    ti.kblocks == 0 ? 0.f : __uint_as_float(v[i]));
                                if (col < args.N && qv > gbest) {
                                    gbest = qv;
                                    garg = col;
                                }
                            }
                        }
                        if (valid && garg >= 0) {
                            args.out_assign[row] = garg;
                            atomicAdd(&s_ghist[garg], 1);
                        }
                    }
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (CG == 2) tc::mbar_arrive_remote(acc ? tempty_leader1 : tempty_leader0);
                else tc::mbar_arrive(&tempty[acc]);
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
        // the staged stores have landed before the CTA (and its shared memory) goes
        if (kStaged && lane == 0) tc::bulk_wait_all();
        if constexpr (kGreedy) {
            if (greedy) {  // the CTA's tokens per expert, one atomic per expert
                asm volatile("bar.sync 12, %0;" ::"r"(32 * kEpiWarps) : "memory");
                for (int e = threadIdx.x - 128; e < args.N && args.out_counts; e += 32 * kEpiWarps)
                    if (s_ghist[e]) atomicAdd(args.out_counts + e, s_ghist[e]);
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if constexpr (CG == 2) tc::cluster_sync_all();  // the pair is done with TMEM
    if (warp == 1) {
        tc::tc_fence_after();
        if constexpr (CG == 2) tc::tmem_dealloc_cg2(tmem_base, TMEM_COLS);
        else tc::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

__global__ void tile_prefix_kernel(const int32_t* __restrict__ offsets, int G, int bm,
                                   int32_t* __restrict__ tile_start) {
    __shared__ int32_t s_warp[32];
    const int g = threadIdx.x;
    const int lane = lane_id(), w = warp_id();
    int v = 0;
    if (g < G) v = (__ldg(offsets + g + 1) - __ldg(offsets + g) + bm - 1) / bm;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[w] = incl;
    __syncthreads();
    if (w == 0) {
        const int x = s_warp[lane];
        int xi = x;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, xi, off);
            if (lane >= off) xi += o;
        }
        s_warp[lane] = xi - x;
    }
    __syncthreads();
    const int excl = incl - v + s_warp[w];
    if (g < G) tile_start[g] = excl;
    if (g == G - 1) tile_start[G] = excl + v;
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// row-major bf16 matrix [rows][cols], box = box_rows x 64 columns, 128 B swizzle
static bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// output tensor [rows][cols] with row stride ld elements (bf16 or fp32), box =
// 32 rows x 128 bytes, 128 B swizzle: one epilogue warp's staged piece
static bool make_tmap_out(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                          uint64_t ld, bool f32) {
    auto fn = encode_fn();
    if (!fn) return false;
    const uint64_t es = f32 ? 4 : 2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * es};
    cuuint32_t box[2] = {(cuuint32_t)(128 / es), 32};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// A: a_rows x a_cols row-major (K-major: a_cols = K; MN-major: a_rows = K)
// B: b_rows x b_cols row-major (likewise).  CG = 2 launches clusters of two
// CTAs (pair tiles of 256 rows).
template <int BN, int STAGES, int EPI, bool A_MN = false, bool B_MN = false, int CG = 1,
          int SLOTS = kStageSlots>
static int launch(const void* A, uint64_t a_rows, uint64_t a_cols, const void* B, uint64_t b_rows,
                  uint64_t b_cols, const Args& args, int max_tiles, cudaStream_t stream) {
    CUtensorMap ta, tb, to0, to1;
    if (!make_tmap(&ta, A, a_rows, a_cols, A_MN ? 64 : BM)) return BASE_ERR_CUDA;
    if (!make_tmap(&tb, B, b_rows, b_cols, B_MN ? 64 : BN / CG)) return BASE_ERR_CUDA;
    memset(&to0, 0, sizeof(to0));
    memset(&to1, 0, sizeof(to1));
    Args a = args;
    a.staged = 0;
    a.wait_ns = g_test_hooks.wait_ns > 0 ? (unsigned long long)g_test_hooks.wait_ns
                                         : (unsigned long long)tc::kWaitNs;
    a.drop_first_load = (CG == 1) ? g_test_hooks.gemm_drop_first_load : 0;
    // whole 128-byte row pieces and 16-byte aligned rows
    const bool stageable = EPI == EPI_F32 ? (args.N % 32 == 0) : (args.N % 64 == 0 && args.ld % 8 == 0);
    if (kStagedEpi<EPI> && stageable) {
        a.staged = 1;
        // dW: the groups' M x N blocks stacked; otherwise M x N with row stride ld
        if (EPI == EPI_F32) {
            if (!make_tmap_out(&to0, args.out_f32, (uint64_t)args.groups * args.M, args.N, args.N,
                               true))
                return BASE_ERR_CUDA;
        } else {
            if (!make_tmap_out(&to0, args.out0, args.M, args.N, args.ld, false)) return BASE_ERR_CUDA;
            if (args.out1 && !make_tmap_out(&to1, args.out1, args.M, args.N, args.ld, false))
                return BASE_ERR_CUDA;
        }
    }
    constexpr size_t smem = STAGES * (size_t)(BM * BK * 2 + (BN / CG) * BK * 2) +
                            (kStagedEpi<EPI> ? kEpiWarps * SLOTS * kStageBuf : 0) + 1024 + 256 +
                            (EPI == EPI_SCORES ? 4 * 256 : 4 * kTsSmem);
    static_assert(smem <= 227 * 1024, "shared memory");
    static_assert(!B_MN || (BN / CG) % 64 == 0, "MN-major B needs 64-wide blocks");
    auto kern = gemm_kernel<BN, STAGES, EPI, A_MN, B_MN, CG, SLOTS>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return BASE_ERR_CUDA;
    // programmatic dependent launch: the set-up (barriers, TMEM, descriptors)
    // overlaps the previous kernel's tail; the kernel waits for it before reading
    const int grid = (CG == 1) ? std::min(num_sms(), std::max(1, max_tiles))
                               : 2 * std::min(num_sms() / 2, std::max(1, max_tiles));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int nattr = 0;
    attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[nattr].val.programmaticStreamSerializationAllowed = 1;
    ++nattr;
    if constexpr (CG == 2) {
        attr[nattr].id = cudaLaunchAttributeClusterDimension;
        attr[nattr].val.clusterDim.x = 2;
        attr[nattr].val.clusterDim.y = 1;
        attr[nattr].val.clusterDim.z = 1;
        ++nattr;
    }
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, to0, to1, a) != cudaSuccess) return BASE_ERR_CUDA;
    return BASE_OK;
}

}  // namespace gemm

// s = h w^T (+ q) for bf16 h (T x D) and w (E x D) on the tensor cores
int launch_scores_bf16(const void* h, const void* w, int T, int D, int E, float* s, int32_t* q,
                       cudaStream_t stream, int32_t* assign, int32_t* counts) {
    using namespace gemm;
    Args a{};
    if (assign && E <= 256) {  // greedy routing in the epilogue: every row in one N tile
        a.out_assign = assign;
        a.out_counts = counts;
    }
    a.M = T;
    a.N = E;
    a.K = D;
    a.groups = 1;
    a.ld = E;
    a.out_f32 = s;
    a.out_q = q;
    const int mt = (T + BM - 1) / BM;
    if (E <= 16) {
        a.n_tiles = 1;
        return launch<16, 8, EPI_SCORES>(h, T, D, w, E, D, a, mt, stream);
    } else if (E <= 32) {
        a.n_tiles = 1;
        return launch<32, 8, EPI_SCORES>(h, T, D, w, E, D, a, mt, stream);
    } else if (E <= 64) {
        a.n_tiles = 1;
        return launch<64, 8, EPI_SCORES>(h, T, D, w, E, D, a, mt, stream);
    } else if (E <= 128) {
        a.n_tiles = 1;
        return launch<128, 6, EPI_SCORES>(h, T, D, w, E, D, a, mt, stream);
    }
    a.n_tiles = (E + 255) / 256;
    return launch<256, 4, EPI_SCORES>(h, T, D, w, E, D, a, mt * a.n_tiles, stream);
}

size_t ffn_workspace_bytes(int E) { return align_up(sizeof(int32_t) * (E + 1), 256); }

// a6 + a7: h1 = act(x W1_e^T), y = sigmoid(gate) (h1 W2_e^T) + x per expert segment
int launch_expert_ffn(const void* x_perm, const int32_t* offsets, int T, int D, int F, int E,
                      const void* W1, const void* W2, int act, const float* gate, void* y_perm,
                      void* h1, void* a1, void* f, void* ws, cudaStream_t stream) {
    using namespace gemm;
    constexpr int BMP = 2 * BM;  // CTA-pair tiles
    int32_t* tile_start = static_cast<int32_t*>(ws);
    // the grouped GEMMs compute the tile prefix themselves when it fits their shared memory
    if (E + 1 > kTsSmem) {
        tile_prefix_kernel<<<1, 1024, 0, stream>>>(offsets, E, BMP, tile_start);
        BASE_RETURN_IF_LAUNCH_FAILED();
    } else {
        tile_start = nullptr;
    }
    const int max_mt = (T + BMP - 1) / BMP + E;
    Args g1{};
    g1.M = T;
    g1.N = F;
    g1.K = D;
    g1.groups = E;
    g1.offsets = offsets;
    g1.tile_start = tile_start;
    g1.b_rows_per_group = F;
    g1.n_tiles = (F + 255) / 256;
    g1.ld = F;
    g1.act = act;
    g1.out0 = static_cast<__nv_bfloat16*>(h1);
    g1.out1 = static_cast<__nv_bfloat16*>(a1);
    // few tiles per SM pair (T <= 16384): a sixth pipeline stage, one staging
    // slot per epilogue warp (measured faster there, slower on larger problems)
    const bool six = T <= 16384;
    int st = six ? launch<256, 6, EPI_ACT, false, false, 2, 1>(x_perm, T, D, W1, (uint64_t)E * F, D,
                                                               g1, max_mt * g1.n_tiles, stream)
                 : launch<256, 5, EPI_ACT, false, false, 2>(x_perm, T, D, W1, (uint64_t)E * F, D,
                                                            g1, max_mt * g1.n_tiles, stream);
    if (st != BASE_OK) return st;
    Args g2{};
    g2.M = T;
    g2.N = D;
    g2.K = F;
    g2.groups = E;
    g2.offsets = offsets;
    g2.tile_start = tile_start;
    g2.b_rows_per_group = D;
    g2.n_tiles = (D + 255) / 256;
    g2.ld = D;
    g2.out0 = static_cast<__nv_bfloat16*>(y_perm);
    g2.out1 = static_cast<__nv_bfloat16*>(f);
    g2.gate = gate;
    g2.side = static_cast<const __nv_bfloat16*>(x_perm);
    return six ? launch<256, 6, EPI_GATE, false, false, 2, 1>(h1, T, F, W2, (uint64_t)E * D, F, g2,
                                                              max_mt * g2.n_tiles, stream)
               : launch<256, 5, EPI_GATE, false, false, 2>(h1, T, F, W2, (uint64_t)E * D, F, g2,
                                                           max_mt * g2.n_tiles, stream);
}

int launch_layer_norm_rows(const void* x, const int32_t* offsets, int T, int D, int E,
                           const float* gamma, const float* beta, int stride, void* y,
                           cudaStream_t stream);

// The released code's expert: S sublayers x <- x + W2_i act(W1_i LN_i(x)) on
// every expert segment, then the blend y = x0 + a (x_S - x0), a =
// sigmoid(gate), x0 = x_perm, in the last GEMM's epilogue.  W1 (E, S, F, D),
// W2 (E, S, D, F), gamma / beta (E, S, D) fp32.  Scratch: the tile prefix,
// then ln and one more T x D bf16 buffer (sublayer outputs alternate between
// it and y_perm, the last one in y_perm).
size_t stack_workspace_bytes(int T, int E, int D) {
    return ffn_workspace_bytes(E) + 2 * align_up((size_t)T * D * 2, 256);
}

int launch_expert_stack(const void* x_perm, const int32_t* offsets, int T, int D, int F, int E,
                        int S, const void* W1, const void* W2, const float* gamma,
                        const float* beta, int act, const float* gate, void* y_perm, void* h1,
                        void* ws, cudaStream_t stream) {
    using namespace gemm;
    constexpr int BMP = 2 * BM;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    int32_t* tile_start = reinterpret_cast<int32_t*>(w8);
    void* ln = w8 + ffn_workspace_bytes(E);
    void* xb = w8 + ffn_workspace_bytes(E) + align_up((size_t)T * D * 2, 256);
    // the grouped GEMMs compute the tile prefix themselves when it fits their shared memory
    if (E + 1 > kTsSmem) {
        tile_prefix_kernel<<<1, 1024, 0, stream>>>(offsets, E, BMP, tile_start);
        BASE_RETURN_IF_LAUNCH_FAILED();
    } else {
        tile_start = nullptr;
    }
    const int max_mt = (T + BMP - 1) / BMP + E;
    const __nv_bfloat16* W1b = static_cast<const __nv_bfloat16*>(W1);
    const __nv_bfloat16* W2b = static_cast<const __nv_bfloat16*>(W2);
    const void* cur = x_perm;
    for (int i = 0; i < S; ++i) {
        int st = launch_layer_norm_rows(cur, offsets, T, D, E, gamma + (size_t)i * D,
                                        beta + (size_t)i * D, S * D, ln, stream);
        if (st != BASE_OK) return st;
        Args g1{};
        g1.M = T;
        g1.N = F;
        g1.K = D;
        g1.groups = E;
        g1.offsets = offsets;
        g1.tile_start = tile_start;
        g1.b_rows_per_group = S * F;  // expert e's sublayer i: rows (e S + i) F of W1
        g1.n_tiles = (F + 255) / 256;
        g1.ld = F;
        g1.act = act;
        g1.out0 = static_cast<__nv_bfloat16*>(h1);
        st = launch<256, 5, EPI_ACT, false, false, 2>(ln, T, D, W1b + (size_t)i * F * D,
                                                      (uint64_t)(E * S - i) * F, D, g1,
                                                      max_mt * g1.n_tiles, stream);
        if (st != BASE_OK) return st;
        const bool last = i == S - 1;
        // outputs alternate so that the last one lands in y_perm
        void* out = ((S - 1 - i) % 2 == 0) ? y_perm : xb;
        Args g2{};
        g2.M = T;
        g2.N = D;
        g2.K = F;
        g2.groups = E;
        g2.offsets = offsets;
        g2.tile_start = tile_start;
        g2.b_rows_per_group = S * D;
        g2.n_tiles = (D + 255) / 256;
        g2.ld = D;
        g2.out0 = static_cast<__nv_bfloat16*>(out);
        g2.gate = gate;
        g2.mix = last ? 2 : 1;
        g2.side = static_cast<const __nv_bfloat16*>(cur);
        g2.side2 = static_cast<const __nv_bfloat16*>(x_perm);
        st = launch<256, 5, EPI_GATE, false, false, 2>(h1, T, F, W2b + (size_t)i * D * F,
                                                       (uint64_t)(E * S - i) * D, F, g2,
                                                       max_mt * g2.n_tiles, stream);
        if (st != BASE_OK) return st;
        cur = out;
    }
    return BASE_OK;
}

}  // namespace base

namespace base {

// the four contractions of the backward (see backward.cu), on CTA pairs
int launch_bwd_gemms(const void* dF, const void* /*unused*/, void* dA1, const void* a1,
                     const void* h1, const void* x_perm, const void* dy, const float* ds,
                     const void* w, const int32_t* perm, const int32_t* offsets,
                     int32_t* tile_start, const void* W1, const void* W2, int act, int T, int D,
                     int E, int F, void* dh, float* dW1, float* dW2, cudaStream_t stream) {
    using namespace gemm;
    constexpr int BMP = 2 * BM;
    // the grouped GEMMs compute the tile prefix themselves when it fits their shared memory
    if (E + 1 > kTsSmem) {
        tile_prefix_kernel<<<1, 1024, 0, stream>>>(offsets, E, BMP, tile_start);
        BASE_RETURN_IF_LAUNCH_FAILED();
    } else {
        tile_start = nullptr;
    }
    const int max_mt = (T + BMP - 1) / BMP + E;
    // dH1 = dF W2_e (B = W2_e stored D x F: MN-major), dA1 = dH1 * act'(A1)
    Args g{};
    g.M = T;
    g.N = F;
    g.K = D;
    g.groups = E;
    g.offsets = offsets;
    g.tile_start = tile_start;
    g.b_rows_per_group = D;
    g.n_tiles = (F + 255) / 256;
    g.ld = F;
    g.act = act;
    g.side = static_cast<const __nv_bfloat16*>(a1);
    g.out0 = static_cast<__nv_bfloat16*>(dA1);
    int st = launch<256, 5, EPI_DACT, false, true, 2>(dF, T, D, W2, (uint64_t)E * D, F, g,
                                                      max_mt * g.n_tiles, stream);
    if (st != BASE_OK) return st;
    // dx = dA1 W1_e + dy + ds w_e (B = W1_e stored F x D: MN-major) -> dh[perm[r]]
    Args x{};
    x.M = T;
    x.N = D;
    x.K = F;
    x.groups = E;
    x.offsets = offsets;
    x.tile_start = tile_start;
    x.b_rows_per_group = F;
    x.n_tiles = (D + 255) / 256;
    x.ld = D;
    x.side = static_cast<const __nv_bfloat16*>(dy);
    x.gate = ds;
    x.side2 = static_cast<const __nv_bfloat16*>(w);
    x.idx = perm;
    x.out0 = static_cast<__nv_bfloat16*>(dh);
    st = launch<256, 6, EPI_DX, false, true, 2>(dA1, T, F, W1, (uint64_t)E * F, D, x,
                                                max_mt * x.n_tiles, stream);
    if (st != BASE_OK) return st;
    // dW2_e = dF_e^T H1_e: A = dF (T x D, MN-major, M = D), B = H1 (T x F, MN-major, N = F)
    Args w2{};
    w2.M = D;
    w2.N = F;
    w2.K = T;
    w2.groups = E;
    w2.offsets = offsets;
    w2.kgroup = 1;
    w2.m_tiles = (D + BMP - 1) / BMP;
    w2.n_tiles = (F + 255) / 256;
    w2.ld = F;
    w2.out_f32 = dW2;
    st = launch<256, 5, EPI_F32, true, true, 2>(dF, T, D, h1, T, F, w2,
                                                E * w2.m_tiles * w2.n_tiles, stream);
    if (st != BASE_OK) return st;
    // dW1_e = dA1_e^T x_e: A = dA1 (T x F, MN-major, M = F), B = x (T x D, MN-major, N = D)
    Args w1{};
    w1.M = F;
    w1.N = D;
    w1.K = T;
    w1.groups = E;
    w1.offsets = offsets;
    w1.kgroup = 1;
    w1.m_tiles = (F + BMP - 1) / BMP;
    w1.n_tiles = (D + 255) / 256;
    w1.ld = D;
    w1.out_f32 = dW1;
    return launch<256, 5, EPI_F32, true, true, 2>(dA1, T, F, x_perm, T, D, w1,
                                                  E * w1.m_tiles * w1.n_tiles, stream);
}

}  // namespace base
