// auction.cu -- balanced token-to-expert assignment (eq. 2 of "BASE Layers:
// Simplifying Training of Large, Sparse Models", Method / "Training
// assignment") by a Jacobi token-bidding auction with epsilon scaling.
//
// The whole auction runs on ONE thread-block cluster (1..16 CTAs of 1024
// threads).  Expert e is owned by CTA e % CL; the owner keeps the expert's
// held bids (at most C = T/E (bid, token) pairs) in its shared memory, so a
// round never leaves the chip except to read the bidders' score rows.  Most
// rounds have only a handful of bidders (the tail of every phase), so the
// cost of a round is its latency: two hardware cluster barriers per round
// instead of grid-wide barriers through global memory.
//
// One round (prices of the round start, identical to the CPU oracle's):
//   bid:     every unassigned token t (a group of lanes per token) scans
//            v_e = q[t][e] (T+1) - price[e], takes the best e* (lowest index
//            on ties) and the second best v2, and bids
//            b = q[t][e*] (T+1) - v2 + eps.  The bid goes to e*'s owner:
//            a DSMEM atomic reserves a place in e*'s bucket (the first 16 in
//            the owner's shared memory, the rest in a global overflow).
//   cluster barrier
//   resolve: one warp per owned expert with new bids keeps the C best of
//            held + new (larger bid, then smaller token), found as the k-th
//            worst key (k = held + new - C) by repeated warp minima for small
//            k or a warp radix select over (bid - min bid, T-1-token) keys;
//            rejected tokens go to the next round's list; a full expert sets
//            its price to its smallest held bid and writes it to every CTA.
//   cluster barrier
// The phase ends when nobody is unassigned; eps is divided by 8 until 1.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace base {
namespace auction {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / kWarp;
constexpr int kSB = 16;          // bids per expert kept in the owner's shared memory
constexpr int kSmallK = 8;       // rejections up to this count use repeated minima
constexpr int kHist = 256;       // radix-select bins per warp
constexpr int kEpsDivisor = 50;  // eps0 = (max q - min q)(T+1) / 50
constexpr int kEpsFactor = 8;    // eps <- eps / 8 per phase
constexpr size_t kMaxSmem = 200 * 1024;

struct Params {
    const int32_t* q;
    int T, E, C;
    int CL, EL;            // cluster size, experts per CTA
    int held_in_smem;
    long long max_rounds;
    int32_t* assign;
    int64_t* price_out;
    base_auction_stats* stats;
    const int32_t* minmax;  // [min q, max q]
    int32_t* ulist0;
    int32_t* ulist1;        // [T] each
    int64_t* gb_bid;
    int32_t* gb_tok;        // [E][T] bucket overflow
    int64_t* gh_bid;
    int32_t* gh_tok;        // [E][C] held sets when they do not fit on chip
    int32_t* gfree;         // [E][C] free-slot scratch
};

struct SmemLayout {
    size_t price, held_bid, held_tok, hcnt, cnt, sb_bid, sb_tok, hist, ctrl, total;
};

__host__ __device__ inline SmemLayout smem_layout(int E, int EL, int C, int held_in_smem) {
    SmemLayout L;
    size_t o = 0;
    L.price = o;    o += align_up(sizeof(int64_t) * E, 16);
    L.held_bid = o; o += held_in_smem ? align_up(sizeof(int64_t) * (size_t)EL * C, 16) : 0;
    L.held_tok = o; o += held_in_smem ? align_up(sizeof(int32_t) * (size_t)EL * C, 16) : 0;
    L.hcnt = o;     o += align_up(sizeof(int32_t) * EL, 16);
    L.cnt = o;      o += align_up(sizeof(int32_t) * EL, 16);
    L.sb_bid = o;   o += align_up(sizeof(int64_t) * (size_t)EL * kSB, 16);
    L.sb_tok = o;   o += align_up(sizeof(int32_t) * (size_t)EL * kSB, 16);
    L.hist = o;     o += sizeof(int32_t) * kWarps * kHist;
    L.ctrl = o;     o += 64;
    L.total = o;
    return L;
}

struct Key {
    int64_t bid;
    int32_t tok;
};

// "worse" order: smaller bid first, then larger token index first.  The C
// best keys of an expert are the ones it keeps.
__device__ __forceinline__ bool worse(const Key& a, const Key& b) {
    return a.bid < b.bid || (a.bid == b.bid && a.tok > b.tok);
}

__device__ __forceinline__ Key shfl_key(const Key& k, int src_lane_xor) {
    Key o;
    o.bid = __shfl_xor_sync(0xffffffffu, k.bid, src_lane_xor);
    o.tok = __shfl_xor_sync(0xffffffffu, k.tok, src_lane_xor);
    return o;
}

__device__ __forceinline__ Key warp_min_key(Key k) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        Key o = shfl_key(k, off);
        if (worse(o, k)) k = o;
    }
    return k;
}

__device__ __forceinline__ Key warp_max_key(Key k) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        Key o = shfl_key(k, off);
        if (worse(k, o)) k = o;
    }
    return k;
}

__device__ __forceinline__ int64_t warp_min_i64(int64_t v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

__device__ __forceinline__ int64_t warp_max_i64(int64_t v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n"
                 "barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

__device__ __forceinline__ int bit_length_u64(uint64_t x) { return x ? 64 - __clzll(x) : 0; }

// Candidates of one expert during a resolve: held slots [0, h) then the new
// bids [0, n) (the first kSB in the owner's shared memory, the rest in the
// global overflow bucket).
struct Cands {
    const int64_t* hb;
    const int32_t* ht;
    const int64_t* sbb;
    const int32_t* sbt;
    const int64_t* gbb;
    const int32_t* gbt;
    int h, n;
    __device__ __forceinline__ Key get(int c) const {
        Key k;
        if (c < h) {
            k.bid = hb[c];
            k.tok = ht[c];
        } else {
            const int j = c - h;
            if (j < kSB) {
                k.bid = sbb[j];
                k.tok = sbt[j];
            } else {
                k.bid = gbb[j - kSB];
                k.tok = gbt[j - kSB];
            }
        }
        return k;
    }
};

// The k-th worst key among the candidates (keys are unique: tokens differ).
__device__ Key kth_worst(const Cands& cd, int k, int T, int32_t* hist) {
    const int lane = lane_id();
    const int m = cd.h + cd.n;
    if (k <= kSmallK) {
        Key last = {INT64_MIN, INT32_MAX};
        for (int it = 0; it < k; ++it) {
            Key best = {INT64_MAX, -1};
            for (int c = lane; c < m; c += kWarp) {
                Key x = cd.get(c);
                if (worse(last, x) && worse(x, best)) best = x;
            }
            last = warp_min_key(best);
        }
        return last;
    }
    // radix select on the virtual key ((bid - minb) << tb) | (T - 1 - tok)
    int64_t lo = INT64_MAX, hi = INT64_MIN;
    for (int c = lane; c < m; c += kWarp) {
        const Key x = cd.get(c);
        lo = min(lo, x.bid);
        hi = max(hi, x.bid);
    }
    lo = warp_min_i64(lo);
    hi = warp_max_i64(hi);
    const int tb = bit_length_u64((uint64_t)(T - 1)) > 0 ? bit_length_u64((uint64_t)(T - 1)) : 1;
    const int NB = bit_length_u64((uint64_t)(hi - lo)) + tb;
    using u128 = unsigned __int128;
    auto vkey = [&](const Key& x) -> u128 {
        return ((u128)(uint64_t)(x.bid - lo) << tb) | (u128)(uint32_t)((T - 1) - x.tok);
    };
    int need = k, pbits = 0;
    u128 prefix = 0;
    for (int guard = 0; guard < 16; ++guard) {
        const int width = min(8, NB - pbits);
        const int shift = NB - pbits - width;
        for (int b = lane; b < kHist; b += kWarp) hist[b] = 0;
        __syncwarp();
        for (int c = lane; c < m; c += kWarp) {
            const u128 K = vkey(cd.get(c));
            if ((K >> (NB - pbits)) == prefix)
                atomicAdd(&hist[(int)((K >> shift) & (u128)((1u << width) - 1))], 1);
        }
        __syncwarp();
        int cnt8[8];
        int sum = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            cnt8[b] = hist[lane * 8 + b];
            sum += cnt8[b];
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        int run = incl - sum;
        int found_d = -1, found_before = 0, found_cnt = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            if (found_d < 0 && run < need && run + cnt8[b] >= need) {
                found_d = lane * 8 + b;
                found_before = run;
                found_cnt = cnt8[b];
            }
            run += cnt8[b];
        }
        const unsigned fm = __ballot_sync(0xffffffffu, found_d >= 0);
        const int src = __ffs(fm) - 1;
        const int d = __shfl_sync(0xffffffffu, found_d, src);
        const int before = __shfl_sync(0xffffffffu, found_before, src);
        const int cnt = __shfl_sync(0xffffffffu, found_cnt, src);
        __syncwarp();
        prefix = (prefix << width) | (u128)d;
        pbits += width;
        need -= before;
        if (need == cnt || pbits >= NB) break;
    }
    // the k-th worst is the best key whose top pbits are <= prefix
    Key best = {INT64_MIN, INT32_MAX};
    for (int c = lane; c < m; c += kWarp) {
        const Key x = cd.get(c);
        if ((vkey(x) >> (NB - pbits)) <= prefix && worse(best, x)) best = x;
    }
    return warp_max_key(best);
}

__device__ __forceinline__ int32_t* remote_i32(int32_t* p, int rank) {
    return cg::this_cluster().map_shared_rank(p, (unsigned)rank);
}
__device__ __forceinline__ int64_t* remote_i64(int64_t* p, int rank) {
    return cg::this_cluster().map_shared_rank(p, (unsigned)rank);
}

// Appends the tokens of the lanes with `rej` set to the next round's list
// (one DSMEM atomic per warp on CTA 0's counter).
__device__ __forceinline__ void push_rejected(bool rej, int32_t tok, int32_t* unext,
                                              int32_t* ucount_remote) {
    const unsigned m = __ballot_sync(0xffffffffu, rej);
    if (!m) return;
    const int lane = lane_id();
    int base = 0;
    if (lane == 0) base = atomicAdd(ucount_remote, __popc(m));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (rej) unext[base + __popc(m & ((1u << lane) - 1))] = tok;
}

__global__ void __launch_bounds__(kThreads, 1) auction_kernel(const __grid_constant__ Params p) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    extern __shared__ __align__(16) unsigned char smem[];
    const SmemLayout L = smem_layout(p.E, p.EL, p.C, p.held_in_smem);
    int64_t* s_price = reinterpret_cast<int64_t*>(smem + L.price);
    int64_t* s_hb = reinterpret_cast<int64_t*>(smem + L.held_bid);
    int32_t* s_ht = reinterpret_cast<int32_t*>(smem + L.held_tok);
    int32_t* s_hcnt = reinterpret_cast<int32_t*>(smem + L.hcnt);
    int32_t* s_cnt = reinterpret_cast<int32_t*>(smem + L.cnt);
    int64_t* s_sbb = reinterpret_cast<int64_t*>(smem + L.sb_bid);
    int32_t* s_sbt = reinterpret_cast<int32_t*>(smem + L.sb_tok);
    int32_t* s_hist = reinterpret_cast<int32_t*>(smem + L.hist);
    int32_t* s_ucount = reinterpret_cast<int32_t*>(smem + L.ctrl);                  // [4]
    unsigned long long* s_obj = reinterpret_cast<unsigned long long*>(smem + L.ctrl + 16);

    const int T = p.T, E = p.E, C = p.C, CL = p.CL, EL = p.EL;
    const int64_t scale = (int64_t)T + 1;
    const int lane = lane_id(), warp = warp_id();

    for (int e = threadIdx.x; e < E; e += kThreads) s_price[e] = 0;
    for (int i = threadIdx.x; i < EL; i += kThreads) {
        s_hcnt[i] = 0;
        s_cnt[i] = 0;
    }
    if (threadIdx.x < 4) s_ucount[threadIdx.x] = 0;
    if (threadIdx.x == 0) *s_obj = 0ull;

    const int64_t qmin = p.minmax[0], qmax = p.minmax[1];
    const int64_t range = qmax - qmin;
    int status = BASE_OK;
    if (range > 0 && range > ((int64_t)1 << 58) / scale) status = BASE_ERR_INVALID_ARG;
    int64_t eps = range * scale / kEpsDivisor;
    if (eps < 1) eps = 1;

    // lanes per bidding token: the smallest power of two >= E, at most 32
    int G = 1;
    while (G < E && G < kWarp) G <<= 1;
    const int tok_per_warp = kWarp / G;
    const int sub = lane / G, gl = lane % G;

    int32_t* ucount0 = remote_i32(s_ucount, 0);
    cluster_barrier();

    long long rounds = 0, phases = 0, bids = 0;
    int cur = 0;
    bool stop = (status != BASE_OK);
    while (!stop) {
        ++phases;
        for (int i = threadIdx.x; i < EL; i += kThreads) s_hcnt[i] = 0;
        int U = T;
        bool phase_start = true;
        while (U > 0) {
            if (rounds >= p.max_rounds) {
                status = BASE_ERR_NOT_CONVERGED;
                break;
            }
            ++rounds;
            bids += U;
            const int32_t* ulist = cur ? p.ulist1 : p.ulist0;
            int32_t* unext = cur ? p.ulist0 : p.ulist1;
            int32_t* ucount_w = ucount0 + (int)(rounds % 3);

            // ---------------- bid ----------------
            {
                const int stride = CL * kWarps * tok_per_warp;
                for (int base = (rank * kWarps + warp) * tok_per_warp; base < U; base += stride) {
                    const int i = base + sub;
                    const bool valid = i < U;
                    int t = 0;
                    if (valid) t = phase_start ? i : ulist[i];
                    int64_t v1 = INT64_MIN, v2 = INT64_MIN;
                    int e1 = INT32_MAX;
                    if (valid) {
                        const int32_t* row = p.q + (size_t)t * E;
                        for (int e = gl; e < E; e += G) {
                            const int64_t v = (int64_t)__ldg(row + e) * scale - s_price[e];
                            if (v > v1) {
                                v2 = v1;
                                v1 = v;
                                e1 = e;
                            } else if (v > v2) {
                                v2 = v;
                            }
                        }
                    }
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {
                        if (off >= G) continue;
                        const int64_t ov1 = __shfl_xor_sync(0xffffffffu, v1, off);
                        const int64_t ov2 = __shfl_xor_sync(0xffffffffu, v2, off);
                        const int oe1 = __shfl_xor_sync(0xffffffffu, e1, off);
                        if (ov1 > v1 || (ov1 == v1 && oe1 < e1)) {
                            v2 = max(v1, ov2);
                            v1 = ov1;
                            e1 = oe1;
                        } else {
                            v2 = max(v2, ov1);
                        }
                    }
                    if (valid && gl == 0) {
                        const int64_t bid = v1 + s_price[e1] - v2 + eps;
                        const int owner = e1 % CL, el = e1 / CL;
                        const int pos = atomicAdd(remote_i32(s_cnt, owner) + el, 1);
                        if (pos < kSB) {
                            remote_i64(s_sbb, owner)[el * kSB + pos] = bid;
                            remote_i32(s_sbt, owner)[el * kSB + pos] = t;
                        } else {
                            p.gb_bid[(size_t)e1 * T + (pos - kSB)] = bid;
                            p.gb_tok[(size_t)e1 * T + (pos - kSB)] = t;
                        }
                    }
                }
            }
            cluster_barrier();

            // ---------------- resolve ----------------
            for (int el = warp; el < EL; el += kWarps) {
                const int e = el * CL + rank;
                if (e >= E) continue;
                const int n = s_cnt[el];
                if (n == 0) continue;
                __syncwarp();
                if (lane == 0) s_cnt[el] = 0;
                const int h = s_hcnt[el];
                int64_t* hb = p.held_in_smem ? s_hb + (size_t)el * C : p.gh_bid + (size_t)e * C;
                int32_t* ht = p.held_in_smem ? s_ht + (size_t)el * C : p.gh_tok + (size_t)e * C;
                Cands cd;
                cd.hb = hb;
                cd.ht = ht;
                cd.sbb = s_sbb + el * kSB;
                cd.sbt = s_sbt + el * kSB;
                cd.gbb = p.gb_bid + (size_t)e * T;
                cd.gbt = p.gb_tok + (size_t)e * T;
                cd.h = h;
                cd.n = n;
                bool full = false;
                if (h + n <= C) {
                    for (int j = lane; j < n; j += kWarp) {
                        const Key x = cd.get(h + j);
                        hb[h + j] = x.bid;
                        ht[h + j] = x.tok;
                    }
                    __syncwarp();
                    if (lane == 0) s_hcnt[el] = h + n;
                    full = (h + n == C);
                } else {
                    const int k = h + n - C;
                    int32_t* hist = s_hist + warp * kHist;
                    const Key kth = kth_worst(cd, k, T, hist);
                    // free slots: rejected held slots and the empty tail, in order
                    int32_t* gfree = p.gfree + (size_t)e * C;
                    int nfree = 0;
                    for (int b0 = 0; b0 < C; b0 += kWarp) {
                        const int i = b0 + lane;
                        bool isfree = false, rej = false;
                        int32_t tok = 0;
                        if (i < C) {
                            if (i < h) {
                                const Key x = cd.get(i);
                                if (!worse(kth, x)) {
                                    isfree = true;
                                    rej = true;
                                    tok = x.tok;
                                }
                            } else {
                                isfree = true;
                            }
                        }
                        push_rejected(rej, tok, unext, ucount_w);
                        const unsigned fm = __ballot_sync(0xffffffffu, isfree);
                        if (isfree) {
                            const int r = nfree + __popc(fm & ((1u << lane) - 1));
                            if (r < kHist) hist[r] = i; else gfree[r] = i;
                        }
                        nfree += __popc(fm);
                    }
                    __syncwarp();
                    // hist was consumed by the selection; it now holds free slots
                    int nacc = 0;
                    for (int b0 = 0; b0 < n; b0 += kWarp) {
                        const int j = b0 + lane;
                        bool acc = false, rej = false;
                        Key x = {0, 0};
                        if (j < n) {
                            x = cd.get(h + j);
                            if (worse(kth, x)) acc = true; else rej = true;
                        }
                        push_rejected(rej, x.tok, unext, ucount_w);
                        const unsigned am = __ballot_sync(0xffffffffu, acc);
                        if (acc) {
                            const int r = nacc + __popc(am & ((1u << lane) - 1));
                            const int slot = (r < kHist) ? hist[r] : gfree[r];
                            hb[slot] = x.bid;
                            ht[slot] = x.tok;
                        }
                        nacc += __popc(am);
                    }
                    __syncwarp();
                    if (lane == 0) s_hcnt[el] = C;
                    full = true;
                    if (nacc != nfree && lane == 0) record_error(1000 + e);
                }
                if (full) {
                    int64_t mn = INT64_MAX;
                    for (int i = lane; i < C; i += kWarp) mn = min(mn, hb[i]);
                    mn = warp_min_i64(mn);
                    if (lane < CL) remote_i64(s_price, lane)[e] = mn;
                }
                __syncwarp();
            }
            cluster_barrier();
            U = *reinterpret_cast<volatile int32_t*>(ucount_w);
            if (rank == 0 && threadIdx.x == 0) s_ucount[(int)((rounds + 1) % 3)] = 0;
            cur ^= 1;
            phase_start = false;
        }
        if (status != BASE_OK) break;
        if (eps == 1) break;
        eps /= kEpsFactor;
        if (eps < 1) eps = 1;
    }

    // results: every owner writes its experts' tokens and prices
    unsigned long long part = 0;
    for (int el = warp; el < EL; el += kWarps) {
        const int e = el * CL + rank;
        if (e >= E) continue;
        const int h = s_hcnt[el];
        const int32_t* ht = p.held_in_smem ? s_ht + (size_t)el * C : p.gh_tok + (size_t)e * C;
        for (int j = lane; j < h; j += kWarp) {
            const int t = ht[j];
            p.assign[t] = e;
            part += (unsigned long long)(int64_t)p.q[(size_t)t * E + e];
        }
        if (lane == 0) p.price_out[e] = s_price[e];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (lane == 0 && part) atomicAdd(cluster.map_shared_rank(s_obj, 0u), part);
    cluster_barrier();
    if (rank == 0 && threadIdx.x == 0 && p.stats) {
        p.stats->status = status;
        p.stats->phases = phases;
        p.stats->rounds = rounds;
        p.stats->final_eps = eps;
        p.stats->objective = (status == BASE_OK) ? (int64_t)*s_obj : 0;
        p.stats->bids = bids;
    }
}

__global__ void minmax_init(int32_t* mm) {
    mm[0] = INT32_MAX;
    mm[1] = INT32_MIN;
}

__global__ void minmax_kernel(const int32_t* __restrict__ q, size_t n, int32_t* mm) {
    int lo = INT32_MAX, hi = INT32_MIN;
    const size_t n4 = n / 4;
    const int4* q4 = reinterpret_cast<const int4*>(q);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
         i += (size_t)gridDim.x * blockDim.x) {
        const int4 v = __ldg(q4 + i);
        lo = min(min(lo, v.x), min(v.y, min(v.z, v.w)));
        hi = max(max(hi, v.x), max(v.y, max(v.z, v.w)));
    }
    for (size_t i = n4 * 4 + blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        lo = min(lo, q[i]);
        hi = max(hi, q[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    __shared__ int slo[32], shi[32];
    if (lane_id() == 0) {
        slo[warp_id()] = lo;
        shi[warp_id()] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x / 32); ++w) {
            lo = min(lo, slo[w]);
            hi = max(hi, shi[w]);
        }
        atomicMin(&mm[0], lo);
        atomicMax(&mm[1], hi);
    }
}

struct Plan {
    int CL, EL, held_in_smem;
    size_t smem;
};

static Plan make_plan(int T, int E) {
    const int C = T / E;
    Plan pl{};
    for (int CL = 1; CL <= 16; CL <<= 1) {
        if (CL > E) break;
        const int EL = (E + CL - 1) / CL;
        const size_t b = smem_layout(E, EL, C, 1).total;
        if (b <= kMaxSmem) {
            pl.CL = CL;
            pl.EL = EL;
            pl.held_in_smem = 1;
            pl.smem = b;
            return pl;
        }
    }
    int CL = 1;
    while (CL * 2 <= 16 && CL * 2 <= E) CL <<= 1;
    pl.CL = CL;
    pl.EL = (E + CL - 1) / CL;
    pl.held_in_smem = 0;
    pl.smem = smem_layout(E, pl.EL, C, 0).total;
    return pl;
}

}  // namespace auction

// Workspace carve-up shared with the API layer.
size_t auction_workspace_bytes(int T, int E) {
    const int C = T / E;
    size_t b = 256;                                   // minmax
    b += 2 * align_up(sizeof(int32_t) * (size_t)T, 256);  // lists
    b += align_up(sizeof(int64_t) * (size_t)E * T, 256);  // overflow bids
    b += align_up(sizeof(int32_t) * (size_t)E * T, 256);  // overflow tokens
    b += align_up(sizeof(int64_t) * (size_t)E * C, 256);  // held (global fallback)
    b += align_up(sizeof(int32_t) * (size_t)E * C, 256);
    b += align_up(sizeof(int32_t) * (size_t)E * C, 256);  // free slots
    return b;
}

int launch_auction(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                   base_auction_stats* stats, void* ws, size_t ws_bytes, long long max_rounds,
                   cudaStream_t stream) {
    using namespace auction;
    if (ws_bytes < auction_workspace_bytes(T, E)) return BASE_ERR_WORKSPACE;
    const int C = T / E;
    Plan pl = make_plan(T, E);

    unsigned char* w = static_cast<unsigned char*>(ws);
    Params prm{};
    prm.q = q;
    prm.T = T;
    prm.E = E;
    prm.C = C;
    prm.max_rounds = max_rounds;
    prm.assign = assign;
    prm.price_out = price;
    prm.stats = stats;
    size_t o = 0;
    int32_t* mm = reinterpret_cast<int32_t*>(w + o); o += 256;
    prm.minmax = mm;
    prm.ulist0 = reinterpret_cast<int32_t*>(w + o); o += align_up(sizeof(int32_t) * (size_t)T, 256);
    prm.ulist1 = reinterpret_cast<int32_t*>(w + o); o += align_up(sizeof(int32_t) * (size_t)T, 256);
    prm.gb_bid = reinterpret_cast<int64_t*>(w + o); o += align_up(sizeof(int64_t) * (size_t)E * T, 256);
    prm.gb_tok = reinterpret_cast<int32_t*>(w + o); o += align_up(sizeof(int32_t) * (size_t)E * T, 256);
    prm.gh_bid = reinterpret_cast<int64_t*>(w + o); o += align_up(sizeof(int64_t) * (size_t)E * C, 256);
    prm.gh_tok = reinterpret_cast<int32_t*>(w + o); o += align_up(sizeof(int32_t) * (size_t)E * C, 256);
    prm.gfree = reinterpret_cast<int32_t*>(w + o); o += align_up(sizeof(int32_t) * (size_t)E * C, 256);

    minmax_init<<<1, 1, 0, stream>>>(mm);
    BASE_RETURN_IF_LAUNCH_FAILED();
    const size_t n = (size_t)T * E;
    int blocks = (int)std::min<size_t>((n / 4 + 255) / 256 + 1, 148 * 8);
    minmax_kernel<<<blocks, 256, 0, stream>>>(q, n, mm);
    BASE_RETURN_IF_LAUNCH_FAILED();

    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = {};
    for (int attempt = 0; attempt < 2; ++attempt) {
        prm.CL = pl.CL;
        prm.EL = pl.EL;
        prm.held_in_smem = pl.held_in_smem;
        if (cudaFuncSetAttribute(auction_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)pl.smem) != cudaSuccess)
            return BASE_ERR_CUDA;
        if (pl.CL > 8 && cudaFuncSetAttribute(auction_kernel,
                                              cudaFuncAttributeNonPortableClusterSizeAllowed,
                                              1) != cudaSuccess)
            return BASE_ERR_CUDA;
        cfg.gridDim = dim3(pl.CL, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = pl.smem;
        cfg.stream = stream;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = pl.CL;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        cudaError_t oe = cudaOccupancyMaxActiveClusters(&nclusters, auction_kernel, &cfg);
        if (oe == cudaSuccess && nclusters > 0) break;
        cudaGetLastError();
        if (attempt == 1 || pl.CL <= 8) return BASE_ERR_UNSUPPORTED;
        // 16-CTA clusters unavailable: 8 CTAs with the held sets in global memory
        pl.CL = 8;
        pl.EL = (E + 7) / 8;
        pl.held_in_smem = 0;
        pl.smem = smem_layout(E, pl.EL, C, 0).total;
    }
    if (cudaLaunchKernelEx(&cfg, auction_kernel, prm) != cudaSuccess) return BASE_ERR_CUDA;
    return BASE_OK;
}

}  // namespace base
