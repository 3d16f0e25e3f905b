// auction.cu -- balanced token-to-expert assignment (eq. 2 of "BASE Layers:
// Simplifying Training of Large, Sparse Models", Method / "Training
// assignment") by a Jacobi token-bidding auction with epsilon scaling.
//
// One round (prices of the round start; identical to the CPU oracle's):
//   bid:     every unassigned token t (a group of lanes per token) scans
//            v_e = q[t][e] (T+1) - price[e], takes the best e* (lowest index
//            on ties) and the second best v2, and bids
//            b = q[t][e*] (T+1) - v2 + eps to e*.
//   resolve: every expert keeps the C best of held + new bids (larger bid,
//            then smaller token); the others become unassigned; a full
//            expert's price is its smallest held bid.
// A phase runs rounds until nobody is unassigned; eps is divided by 8 down
// to 1 (exact optimum for integer scores).
//
// The kernel is one persistent cooperative grid (one CTA of 512 threads per
// SM) with two modes:
//   * wide rounds (the start of every phase, where all T tokens bid, and the
//     next rounds while many tokens are unassigned) use the whole GPU: bids
//     go to per-expert global buckets, a grid barrier, then one CTA per
//     expert keeps its C best with a CTA-wide radix select, a grid barrier;
//   * narrow rounds (the long tail of every phase, mostly a handful of
//     bidders) run on CTA 0 alone while the other CTAs wait for the phase to
//     end: prices live in shared memory, and for every full expert CTA 0 keeps
//     a "fringe" -- its FK worst held bids, sorted -- so a round resolves with
//     a warp-wide bitonic merge of fringe and new bids instead of a scan of
//     the expert's C held bids.  Rejected tokens' score rows are copied into
//     shared memory (cp.async) for their next bid.
// Held sets live in global memory (they are touched only when a fringe is
// rebuilt).  Every wait is bounded; a wait that gives up records an error
// and all CTAs leave.
#include <algorithm>

#include "common.cuh"

namespace base {
namespace auction {

constexpr int kThreads = 512;  // 16 warps: 128 registers per thread, no spills
constexpr int kWarps = kThreads / kWarp;
static_assert(kWarps <= 16, "the team reductions keep 16 warp minima and 16 maxima");
constexpr int kHist = 256;
constexpr int kEpsDivisor = 50;  // eps0 = (max q - min q)(T+1) / 50
constexpr int kEpsFactor = 8;    // eps <- eps / 8 per phase
// Rounds with at most this many bidders run on CTA 0: with few experts a
// narrow round stays cheaper than a grid-wide one up to a few hundred
// bidders; with 32 or more experts its resolves (several bids per expert,
// fringe rebuilds) outgrow a wide round beyond about 32 bidders.
__host__ __device__ constexpr int narrow_max_for(int E) { return E <= 16 ? 256 : 32; }
constexpr uint64_t kWaitNs = 20000000000ull;  // grid-barrier wait limit (20 s)

// ---------------------------------------------------------------- keys
// 16-byte aligned (one 128-bit load or store); every Key array in shared or
// global memory starts on a 16-byte boundary
struct __align__(16) Key {
    int64_t bid;
    int32_t tok;
    int32_t slot;  // >= 0: held slot; -1: a new bid; -2: padding
};
static_assert(sizeof(Key) == 16, "Key is 16 bytes");

// "worse" order: smaller bid first, then larger token first; an expert keeps
// the C best keys.  Written without short-circuit operators, and the key
// selects below with conditional moves per field: a short-circuit compare
// becomes divergent branches, which cost a single warp ~5x more per compare
// (measured: a 32-key warp sort 2.9 k -> 0.9 k cycles).
__device__ __forceinline__ bool worse(const Key& a, const Key& b) {
    return (a.bid < b.bid) | ((a.bid == b.bid) & (a.tok > b.tok));
}

// c ? a : b, field by field
__device__ __forceinline__ Key sel_key(bool c, const Key& a, const Key& b) {
    Key r;
    r.bid = c ? a.bid : b.bid;
    r.tok = c ? a.tok : b.tok;
    r.slot = c ? a.slot : b.slot;
    return r;
}

__device__ __forceinline__ Key pad_key() { return Key{INT64_MAX, -1, -2}; }

__device__ __forceinline__ Key shfl_key(const Key& k, int src) {
    Key o;
    o.bid = __shfl_sync(0xffffffffu, k.bid, src);
    o.tok = __shfl_sync(0xffffffffu, k.tok, src);
    o.slot = __shfl_sync(0xffffffffu, k.slot, src);
    return o;
}

__device__ __forceinline__ Key shfl_xor_key(const Key& k, int m) {
    Key o;
    o.bid = __shfl_xor_sync(0xffffffffu, k.bid, m);
    o.tok = __shfl_xor_sync(0xffffffffu, k.tok, m);
    o.slot = __shfl_xor_sync(0xffffffffu, k.slot, m);
    return o;
}

__device__ __forceinline__ Key warp_min_key(Key k) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const Key o = shfl_xor_key(k, off);
        k = sel_key(worse(o, k), o, k);
    }
    return k;
}

__device__ __forceinline__ Key warp_max_key(Key k) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const Key o = shfl_xor_key(k, off);
        k = sel_key(worse(k, o), o, k);
    }
    return k;
}

// ascending bitonic sort of one key per lane
__device__ __forceinline__ Key warp_sort(Key x) {
    const int lane = lane_id();
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const Key o = shfl_xor_key(x, j);
            const bool up = (lane & k) == 0;
            const bool lower = (lane & j) == 0;
            x = sel_key(lower == up ? worse(o, x) : worse(x, o), o, x);
        }
    }
    return x;
}

// sorts a bitonic sequence held one key per lane into ascending order
__device__ __forceinline__ Key warp_bitonic_merge(Key x) {
    const int lane = lane_id();
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const Key o = shfl_xor_key(x, j);
        const bool lower = (lane & j) == 0;
        x = sel_key(lower ? worse(o, x) : worse(x, o), o, x);
    }
    return x;
}

// a, b sorted ascending (one per lane) -> lo, hi: the 64 keys sorted ascending
// (element i of the result is lo in lane i for i < 32, hi in lane i-32 after)
__device__ __forceinline__ void warp_merge64(Key a, Key b, Key& lo, Key& hi) {
    const Key br = shfl_key(b, 31 - lane_id());
    const bool sw = worse(br, a);
    lo = sel_key(sw, br, a);
    hi = sel_key(sw, a, br);
    lo = warp_bitonic_merge(lo);
    hi = warp_bitonic_merge(hi);
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

template <typename X>
__device__ __forceinline__ X vload(const X* p) {
    return *reinterpret_cast<const volatile X*>(p);
}

__device__ __forceinline__ int bit_length_u64(uint64_t x) { return x ? 64 - __clzll(x) : 0; }
__device__ __forceinline__ uint64_t shr64(uint64_t x, int n) { return n >= 64 ? 0ull : (x >> n); }

// ---------------------------------------------------------------- teams
// A team is either one warp (TEAM = 32) or the whole CTA (TEAM = kThreads,
// at least 256).  Its scratch: kHist ints of histogram, 32 int64, 64 ints.
template <int TEAM>
struct Team {
    int32_t* hist;     // [kHist]
    int64_t* red;      // [32] (CTA team only)
    int32_t* cnt;      // [64] (CTA team only): warp counts, totals, results
    __device__ __forceinline__ int tid() const { return TEAM == 32 ? lane_id() : (int)threadIdx.x; }
    __device__ __forceinline__ void sync() const {
        if (TEAM == 32) __syncwarp(); else __syncthreads();
    }
    __device__ int64_t min_i64(int64_t v) const {
        v = warp_min_i64(v);
        if (TEAM == 32) return v;
        if (lane_id() == 0) red[warp_id()] = v;
        __syncthreads();
        if (warp_id() == 0) {
            int64_t x = lane_id() < TEAM / 32 ? red[lane_id()] : INT64_MAX;
            x = warp_min_i64(x);
            if (lane_id() == 0) red[0] = x;
        }
        __syncthreads();
        const int64_t r = red[0];
        __syncthreads();
        return r;
    }
    __device__ int64_t max_i64(int64_t v) const {
        v = warp_max_i64(v);
        if (TEAM == 32) return v;
        if (lane_id() == 0) red[warp_id()] = v;
        __syncthreads();
        if (warp_id() == 0) {
            int64_t x = lane_id() < TEAM / 32 ? red[lane_id()] : INT64_MIN;
            x = warp_max_i64(x);
            if (lane_id() == 0) red[0] = x;
        }
        __syncthreads();
        const int64_t r = red[0];
        __syncthreads();
        return r;
    }
    // (min, max) of v over the team in one reduction
    __device__ void minmax_i64(int64_t& lo, int64_t& hi) const {
        lo = warp_min_i64(lo);
        hi = warp_max_i64(hi);
        if (TEAM == 32) return;
        if (lane_id() == 0) {
            red[warp_id()] = lo;
            red[16 + warp_id()] = hi;
        }
        __syncthreads();
        if (warp_id() == 0) {
            int64_t x = lane_id() < TEAM / 32 ? red[lane_id()] : INT64_MAX;
            int64_t y = lane_id() < TEAM / 32 ? red[16 + lane_id()] : INT64_MIN;
            x = warp_min_i64(x);
            y = warp_max_i64(y);
            __syncwarp();
            if (lane_id() == 0) {
                red[0] = x;
                red[16] = y;
            }
        }
        __syncthreads();
        lo = red[0];
        hi = red[16];
        __syncthreads();
    }
    __device__ Key max_key(Key k) const {
        k = warp_max_key(k);
        if (TEAM == 32) return k;
        Key* sk = reinterpret_cast<Key*>(hist);  // 32 keys fit in the histogram area
        if (lane_id() == 0) sk[warp_id()] = k;
        __syncthreads();
        if (warp_id() == 0) {
            Key x = warp_max_key(lane_id() < TEAM / 32 ? sk[lane_id()] : Key{INT64_MIN, INT32_MAX, -2});
            if (lane_id() == 0) sk[0] = x;
        }
        __syncthreads();
        const Key r = sk[0];
        __syncthreads();
        return r;
    }
    // Finds the bin d of the histogram (nbins <= kHist) where the running
    // count reaches `need`: before = count of bins < d, cnt = count of bin d.
    __device__ void find_digit(int nbins, int need, int& d, int& before, int& count) const {
        if (TEAM == 32) {
            const int lane = lane_id();
            int c8[8];
            int sum = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const int bin = lane * 8 + b;
                c8[b] = bin < nbins ? hist[bin] : 0;
                sum += c8[b];
            }
            int incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            int run = incl - sum, fd = -1, fb = 0, fc = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const bool hit = (fd < 0) & (run < need) & (run + c8[b] >= need);
                fd = hit ? lane * 8 + b : fd;
                fb = hit ? run : fb;
                fc = hit ? c8[b] : fc;
                run += c8[b];
            }
            const unsigned m = __ballot_sync(0xffffffffu, fd >= 0);
            const int src = __ffs(m) - 1;
            d = __shfl_sync(0xffffffffu, fd, src);
            before = __shfl_sync(0xffffffffu, fb, src);
            count = __shfl_sync(0xffffffffu, fc, src);
            __syncwarp();
            return;
        }
        // CTA: threads 0..255 own one bin each; block scan over 8 warps
        const int t = threadIdx.x;
        const int c = (t < nbins) ? hist[t] : 0;
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane_id() >= off) incl += o;
        }
        if (t < kHist && lane_id() == 31) cnt[34 + warp_id()] = incl;  // 8 warp totals
        __syncthreads();
        int wbase = 0;
        if (t < kHist)
            for (int w = 0; w < warp_id(); ++w) wbase += cnt[34 + w];
        const int excl = wbase + incl - c;
        if ((t < nbins) & (excl < need) & (excl + c >= need)) {
            cnt[42] = t;
            cnt[43] = excl;
            cnt[44] = c;
        }
        __syncthreads();
        d = cnt[42];
        before = cnt[43];
        count = cnt[44];
        __syncthreads();
    }
    // rank of this thread among the threads with `flag`, in thread order; total
    __device__ int rank(bool flag, int& total) const {
        const unsigned m = __ballot_sync(0xffffffffu, flag);
        const int in_warp = __popc(m & ((1u << lane_id()) - 1));
        if (TEAM == 32) {
            total = __popc(m);
            return in_warp;
        }
        if (lane_id() == 0) cnt[warp_id()] = __popc(m);
        __syncthreads();
        if (warp_id() == 0) {
            const int v = lane_id() < TEAM / 32 ? cnt[lane_id()] : 0;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane_id() >= off) incl += o;
            }
            cnt[lane_id()] = incl - v;
            if (lane_id() == 31) cnt[32] = incl;
        }
        __syncthreads();
        const int r = cnt[warp_id()] + in_warp;
        total = cnt[32];
        __syncthreads();
        return r;
    }
};

// Candidates of one expert: held slots [0, h) then new bids [0, n).
struct Cands {
    const int64_t* hb;
    const int32_t* ht;
    const int64_t* nb;
    const int32_t* nt;
    int h, n;
    __device__ __forceinline__ Key get(int c) const {
        Key k;
        if (c < h) {
            k.bid = hb[c];
            k.tok = ht[c];
            k.slot = c;
        } else {
            k.bid = nb[c - h];
            k.tok = nt[c - h];
            k.slot = -1;
        }
        return k;
    }
};

// The k-th worst key among a team's candidates (1 <= k <= m; keys are
// unique).  `visit(f)` calls f(key) for each candidate this thread owns.
// Radix select on the bid (relative to the smallest bid, 8-bit digits from
// the top), then, among equal bids, on the token.
// Digit pass helper of the CTA select: warp 0 scans the 256-bin histogram
// (eight bins per lane), finds the bin where the running count reaches
// `need`, publishes (bin, count before it, its count) in out[0..2] and zeroes
// the histogram for the next pass.  The caller's barrier publishes both.
__device__ __forceinline__ void cta_find_digit(int32_t* hist, int nbins, int need, int32_t* out) {
    const int lane = lane_id();
    int c8[8];
    const int4* h4 = reinterpret_cast<const int4*>(hist + lane * 8);
    const int4 a = h4[0], b = h4[1];
    c8[0] = a.x; c8[1] = a.y; c8[2] = a.z; c8[3] = a.w;
    c8[4] = b.x; c8[5] = b.y; c8[6] = b.z; c8[7] = b.w;
    int sum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        if (lane * 8 + q >= nbins) c8[q] = 0;
        sum += c8[q];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    int run = incl - sum;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        if ((run < need) & (run + c8[q] >= need)) {
            out[0] = lane * 8 + q;
            out[1] = run;
            out[2] = c8[q];
        }
        run += c8[q];
    }
    int4* w4 = reinterpret_cast<int4*>(hist + lane * 8);
    w4[0] = make_int4(0, 0, 0, 0);
    w4[1] = make_int4(0, 0, 0, 0);
}

// The k-th worst key among a CTA's candidates (1 <= k <= m; keys unique):
// radix select on the bid (relative to the smallest, 8-bit digits from the
// top), then among equal bids on the token; two barriers per digit.
// `visit(f)` calls f(key) for each candidate this thread owns.
template <class Visit>
__device__ Key kth_worst_cta(const Team<kThreads>& tm, Visit visit, int k, int tmax) {
    const int lane = lane_id(), warp = warp_id();
    int32_t* hist = tm.hist;     // 256 bins, zero between passes
    int32_t* res = tm.cnt + 50;  // [3] a pass's result
    __syncthreads();  // the caller may still be reading the histogram area
    if (warp == 0) {
        int4* w4 = reinterpret_cast<int4*>(hist + lane * 8);
        w4[0] = make_int4(0, 0, 0, 0);
        w4[1] = make_int4(0, 0, 0, 0);
    }
    int64_t lo = INT64_MAX, hi = INT64_MIN;
    visit([&](const Key& x) {
        lo = min(lo, x.bid);
        hi = max(hi, x.bid);
    });
    lo = warp_min_i64(lo);
    hi = warp_max_i64(hi);
    if (lane == 0) {
        tm.red[warp] = lo;
        tm.red[16 + warp] = hi;
    }
    __syncthreads();
    {
        int64_t x = lane < kWarps ? tm.red[lane] : INT64_MAX;
        int64_t y = lane < kWarps ? tm.red[16 + lane] : INT64_MIN;
        lo = warp_min_i64(x);  // every warp reduces the 16 partials itself
        hi = warp_max_i64(y);
    }
    const int nbits = bit_length_u64((uint64_t)(hi - lo));
    int need = k, pbits = 0;
    uint64_t prefix = 0;
    bool whole_bucket = false;
    while (pbits < nbits) {
        const int width = min(8, nbits - pbits);
        const int shift = nbits - pbits - width;
        visit([&](const Key& x) {
            const uint64_t v = (uint64_t)(x.bid - lo);
            if (shr64(v, shift + width) == prefix)
                atomicAdd(&hist[(int)((v >> shift) & ((1u << width) - 1))], 1);
        });
        __syncthreads();
        if (warp == 0) cta_find_digit(hist, 1 << width, need, res);
        __syncthreads();
        const int d = res[0], before = res[1], cnt = res[2];
        prefix = (prefix << width) | (uint64_t)d;
        pbits += width;
        need -= before;
        if (need == cnt) {
            whole_bucket = true;
            break;
        }
    }
    Key best = Key{INT64_MIN, INT32_MAX, -2};
    if (whole_bucket) {
        // the k-th worst is the best of the candidates whose bid's top pbits
        // are <= prefix
        const int sh = nbits - pbits;
        visit([&](const Key& x) {
            best = sel_key((shr64((uint64_t)(x.bid - lo), sh) <= prefix) & worse(best, x), x, best);
        });
    } else {
        // every bid digit fixed: B* = lo + prefix; `need` of the candidates
        // with bid == B* are rejected, those with the largest tokens
        const int64_t bstar = lo + (int64_t)prefix;
        const uint32_t tm_max = (uint32_t)tmax;
        const int tbits = bit_length_u64((uint64_t)tm_max) > 0 ? bit_length_u64((uint64_t)tm_max) : 1;
        int tneed = need, tp = 0;
        uint32_t tprefix = 0;
        while (tp < tbits) {
            const int width = min(8, tbits - tp);
            const int shift = tbits - tp - width;
            visit([&](const Key& x) {
                if (x.bid != bstar) return;
                const uint32_t v = tm_max - (uint32_t)x.tok;
                if ((uint32_t)shr64(v, shift + width) == tprefix)
                    atomicAdd(&hist[(int)((v >> shift) & ((1u << width) - 1))], 1);
            });
            __syncthreads();
            if (warp == 0) cta_find_digit(hist, 1 << width, tneed, res);
            __syncthreads();
            const int d = res[0], before = res[1], cnt = res[2];
            tprefix = (tprefix << width) | (uint32_t)d;
            tp += width;
            tneed -= before;
            if (tneed == cnt) break;
        }
        const int sh = tbits - tp;
        visit([&](const Key& x) {
            bool rej = x.bid < bstar;
            if (x.bid == bstar) rej = (uint32_t)shr64(tm_max - (uint32_t)x.tok, sh) <= tprefix;
            best = sel_key(rej & worse(best, x), x, best);
        });
    }
    // the best over the CTA: warp maxima, then every warp reduces them
    best = warp_max_key(best);
    Key* wk = reinterpret_cast<Key*>(tm.hist + kHist);  // past the histogram: 16 keys
    if (lane == 0) wk[warp] = best;
    __syncthreads();
    const Key r = warp_max_key(lane < kWarps ? wk[lane] : Key{INT64_MIN, INT32_MAX, -2});
    __syncthreads();  // wk and red are free again once every warp has read them
    return r;
}

template <int TEAM, class Visit>
__device__ Key kth_worst_v(const Team<TEAM>& tm, Visit visit, int k, int tmax) {
    if constexpr (TEAM > 32) return kth_worst_cta(tm, visit, k, tmax);
    int64_t lo = INT64_MAX, hi = INT64_MIN;
    visit([&](const Key& x) {
        lo = min(lo, x.bid);
        hi = max(hi, x.bid);
    });
    tm.minmax_i64(lo, hi);
    const int nbits = bit_length_u64((uint64_t)(hi - lo));
    const int tid = tm.tid();
    // --- bid digits
    int need = k, pbits = 0;
    uint64_t prefix = 0;
    bool whole_bucket = false;
    int32_t* hist = tm.hist;
    auto clear_hist = [&]() {
        for (int b = tid; b < kHist; b += TEAM) tm.hist[b] = 0;
        tm.sync();
    };
    auto sum_hist = [&]() { tm.sync(); };
    while (pbits < nbits) {
        const int width = min(8, nbits - pbits);
        const int shift = nbits - pbits - width;
        clear_hist();
        visit([&](const Key& x) {
            const uint64_t v = (uint64_t)(x.bid - lo);
            if (shr64(v, shift + width) == prefix)
                atomicAdd(&hist[(int)((v >> shift) & ((1u << width) - 1))], 1);
        });
        sum_hist();
        int d = 0, before = 0, cnt = 0;
        tm.find_digit(1 << width, need, d, before, cnt);
        prefix = (prefix << width) | (uint64_t)d;
        pbits += width;
        need -= before;
        if (need == cnt) {
            whole_bucket = true;
            break;
        }
    }
    if (whole_bucket) {
        // reject every candidate whose bid's top pbits are <= prefix; the k-th
        // worst is the best of them
        Key best = Key{INT64_MIN, INT32_MAX, -2};
        const int sh = nbits - pbits;
        visit([&](const Key& x) {
            best = sel_key((shr64((uint64_t)(x.bid - lo), sh) <= prefix) & worse(best, x), x, best);
        });
        return tm.max_key(best);
    }
    // every bid digit fixed: B* = lo + prefix; `need` of the candidates with
    // bid == B* are rejected, the ones with the largest tokens
    const int64_t bstar = lo + (int64_t)prefix;
    const uint32_t tm_max = (uint32_t)tmax;
    const int tbits = bit_length_u64((uint64_t)tm_max) > 0 ? bit_length_u64((uint64_t)tm_max) : 1;
    int tneed = need, tp = 0;
    uint32_t tprefix = 0;
    // rank by (tmax - tok) ascending: larger tokens first
    while (tp < tbits) {
        const int width = min(8, tbits - tp);
        const int shift = tbits - tp - width;
        clear_hist();
        visit([&](const Key& x) {
            if (x.bid != bstar) return;
            const uint32_t v = tm_max - (uint32_t)x.tok;
            if ((uint32_t)shr64(v, shift + width) == tprefix)
                atomicAdd(&hist[(int)((v >> shift) & ((1u << width) - 1))], 1);
        });
        sum_hist();
        int d = 0, before = 0, cnt = 0;
        tm.find_digit(1 << width, tneed, d, before, cnt);
        tprefix = (tprefix << width) | (uint32_t)d;
        tp += width;
        tneed -= before;
        if (tneed == cnt) break;
    }
    Key best = Key{INT64_MIN, INT32_MAX, -2};
    const int sh = tbits - tp;
    visit([&](const Key& x) {
        bool rej = x.bid < bstar;
        if (x.bid == bstar) rej = (uint32_t)shr64(tm_max - (uint32_t)x.tok, sh) <= tprefix;
        best = sel_key(rej & worse(best, x), x, best);
    });
    return tm.max_key(best);
}

// Candidates read from memory on every pass; a warp with few rejections
// uses repeated minima instead of the radix select.
template <int TEAM>
__device__ Key kth_worst(const Team<TEAM>& tm, const Cands& cd, int k, int tmax) {
    const int m = cd.h + cd.n;
    const int tid = tm.tid();
    if (TEAM == 32 && k <= 8) {
        Key last = Key{INT64_MIN, INT32_MAX, -2};
        for (int it = 0; it < k; ++it) {
            Key best = pad_key();
            for (int c = tid; c < m; c += TEAM) {
                const Key x = cd.get(c);
                best = sel_key(worse(last, x) & worse(x, best), x, best);
            }
            last = warp_min_key(best);
        }
        return last;
    }
    if (TEAM > 32 && m <= 2 * TEAM) {
        // the whole candidate set fits in registers: two keys per thread
        const Key k0 = tid < m ? cd.get(tid) : pad_key();
        const Key k1 = tid + TEAM < m ? cd.get(tid + TEAM) : pad_key();
        auto visit = [&](auto f) {
            if (tid < m) f(k0);
            if (tid + TEAM < m) f(k1);
        };
        return kth_worst_v<TEAM>(tm, visit, k, tmax);
    }
    auto visit = [&](auto f) {
        for (int c = tid; c < m; c += TEAM) f(cd.get(c));
    };
    return kth_worst_v<TEAM>(tm, visit, k, tmax);
}

// ---------------------------------------------------------------- state
struct Ctrl {
    int abort;
    int ucount[3];
    int pad[2];
};

struct Params {
    const int32_t* q;
    int T, E, C, FK, NB, RC;
    int HS;  // 1: CTA 0 keeps the held sets in shared memory during narrow rounds
    long long max_rounds;
    int narrow_max;
    int32_t* assign;
    int64_t* price_out;
    base_auction_stats* stats;
    unsigned* mmenc;  // [2] max over q of enc(q) and of ~enc(q) (enc keeps the signed order)
    Ctrl* ctrl;
    unsigned* bar_flags;  // [gridDim.x] grid-barrier counts
    int64_t* gprice;   // [E]
    int32_t* hcnt;     // [E]
    int64_t* hb;       // [E][C]
    int32_t* ht;
    int32_t* bcnt;     // [E]
    int64_t* bb;       // [E][T]
    int32_t* bt;
    int32_t* ulist0;   // [T]
    int32_t* ulist1;
    int32_t* gfree;    // [E][C]
    Key* gfr;          // [E][FK] fringes built by the wide rounds
    int32_t* gfs;      // [E] their sizes (-1: none)
    unsigned long long* obj;  // [1]
    int32_t* u_trace;  // nullable: bidders of round r
    int64_t* t_trace;  // nullable: globaltimer (ns) at the start of round r
    long long trace_cap;
    int SW;        // 1: wide rounds keep the owned experts' held sets sorted in shared memory
    int own_max;   // experts a CTA owns at most: ceil(E / grid)
    int nsc;       // keys of the sorted-resolve scratch (a power of two >= C)
    unsigned long long wait_ns;  // limit of every grid-barrier wait
    int absent_cta;              // test hook: this CTA returns at once (-1: none)
};

__device__ __forceinline__ uint64_t globaltimer();

__device__ __forceinline__ void trace_round(const Params& p, long long r, int U) {
    if (r < p.trace_cap) {
        if (p.u_trace) p.u_trace[r] = U;
        if (p.t_trace) p.t_trace[r] = (int64_t)globaltimer();
    }
}

// shared memory of every CTA (narrow-mode arrays are used by CTA 0 only)
struct SmemLayout {
    size_t price, fr, fsize, hcnt, ncnt, act0, act1, nbk_b, nbk_t, list0, list1, rows, wb, wt, we,
        wp, hist, red, cnt, misc, swm, hb, ht, scratch, total;
};

constexpr int kWideChunk = 1024;  // bids a CTA stages before reserving bucket space
constexpr int kMaxOwn = 16;       // experts per CTA with sorted held sets

// Sorted held sets in the scratch area: for owned expert j and buffer s,
// bids at sw_bids(j, s) and tokens at sw_toks(j, s); the sort scratch after.
__host__ __device__ inline size_t sw_set_bytes(int C) { return align_up(12 * (size_t)C, 16); }
__host__ __device__ inline size_t sw_bytes(int own, int C) { return 2 * (size_t)own * sw_set_bytes(C); }
constexpr int kMaxGrid = 1024;    // CTAs of the cooperative grid (one per SM)

// NB: new bids per expert kept in shared memory (the rest in the global
// bucket); RC: bidders' score rows staged in shared memory per round parity.
// HS: the held sets (E x C = T keys) in shared memory too.
__host__ __device__ inline SmemLayout smem_layout(int E, int FK, int NM, int NB, int RC, int T = 0,
                                                  int HS = 0) {
    SmemLayout L;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t r = o; o += align_up(bytes, 16); return r; };
    // used by every CTA in wide rounds
    L.price = take(8 * (size_t)E);
    L.ncnt = take(4 * (size_t)E);
    L.act0 = take(4 * (size_t)E);
    L.wb = take(8 * (size_t)kWideChunk);
    L.wt = take(4 * (size_t)kWideChunk);
    L.we = take(4 * (size_t)kWideChunk);
    L.wp = take(4 * (size_t)kWideChunk);
    L.hist = take(4 * (size_t)kWarps * kHist);
    L.red = take(8 * 32);
    L.cnt = take(4 * 64);
    L.misc = take(64);
    L.swm = take(4 * 2 * kMaxOwn);  // sorted held sets: count and buffer per owned expert
    // narrow rounds (CTA 0) only; in wide rounds the scratch of the resolve
    // (or, with sorted held sets, those sets and the sort scratch)
    L.scratch = o;
    L.fr = take(sizeof(Key) * (size_t)E * FK);
    L.fsize = take(4 * (size_t)E);
    L.hcnt = take(4 * (size_t)E);
    L.act1 = take(4 * (size_t)E);
    L.nbk_b = take(8 * (size_t)E * NB);
    L.nbk_t = take(4 * (size_t)E * NB);
    L.list0 = take(4 * (size_t)NM);
    L.list1 = take(4 * (size_t)NM);
    L.rows = take(2 * 4 * (size_t)RC * E);
    L.hb = take(HS ? 8 * (size_t)T : 0);
    L.ht = take(HS ? 4 * (size_t)T : 0);
    L.total = o;
    return L;
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Grid barrier (all CTAs are co-resident: cooperative launch).  Every CTA
// publishes its barrier count in its own flag (no serialised atomics) and
// warp 0 polls all flags.  Every CTA calls it the same number of times, so
// the counts agree.  Returns false when the wait gave up or another CTA gave
// up.
template <class P>
__device__ bool grid_sync(const P& p, unsigned& gen, int* s_flag) {
    // A counter barrier: every CTA adds one to an arrival count that only
    // grows (it reaches gen * grid at barrier gen) with a release reduction
    // (no reply to wait for) and polls the count with acquire loads until it
    // gets there.  Against a count that the last arriver answers with a
    // release word, this takes one L2 trip off the barrier's critical path.
    // The count sits in bar_flags[0] (zeroed per launch).
    __syncthreads();
    ++gen;
    if (threadIdx.x == 0) {
        unsigned* count = p.bar_flags;
        const unsigned target = gen * gridDim.x;
        int ok = 1;
        // the release orders this CTA's writes before its arrival
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(count) : "memory");
        const uint64_t t0 = globaltimer();
        for (long long it = 1;; ++it) {
            unsigned c;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(count) : "memory");
            if ((int)(c - target) >= 0) break;
            // short naps while the barrier is young, longer ones in a long
            // wait (the narrow rounds of CTA 0) to spare the L2
            __nanosleep(it < 256 ? 20 : 200);
            if ((it & 63) == 0) {
                if (*reinterpret_cast<volatile int*>(&p.ctrl->abort)) {
                    ok = 0;
                    break;
                }
                if (globaltimer() - t0 > p.wait_ns || it > (1ll << 30)) {
                    atomicExch(&p.ctrl->abort, 1);
                    record_error(5001);
                    ok = 0;
                    break;
                }
            }
        }
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

// best / second-best scan of one token's row by a group of G lanes (the row
// may be in global memory or staged in shared memory: generic loads)
__device__ __forceinline__ void group_bid(const int32_t* row, const int64_t* price, int E, int G,
                                          int gl, int64_t scale, int64_t& v1, int64_t& v2,
                                          int& e1) {
    v1 = INT64_MIN;
    v2 = INT64_MIN;
    e1 = INT32_MAX;
    for (int e = gl; e < E; e += G) {
        const int64_t v = (int64_t)row[e] * scale - price[e];
        const bool g1 = v > v1, g2 = v > v2;
        v2 = g1 ? v1 : (g2 ? v : v2);
        v1 = g1 ? v : v1;
        e1 = g1 ? e : e1;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        if (off >= G) continue;
        const int64_t ov1 = __shfl_xor_sync(0xffffffffu, v1, off);
        const int64_t ov2 = __shfl_xor_sync(0xffffffffu, v2, off);
        const int oe1 = __shfl_xor_sync(0xffffffffu, e1, off);
        const bool tk = (ov1 > v1) | ((ov1 == v1) & (oe1 < e1));
        v2 = tk ? max(v1, ov2) : max(v2, ov1);
        v1 = tk ? ov1 : v1;
        e1 = tk ? oe1 : e1;
    }
}

// The same for NT tokens at once (their loads in flight together).
template <int NT>
__device__ __forceinline__ void group_bid_multi(const int32_t* __restrict__ q, const int (&t)[NT],
                                                const bool (&valid)[NT], const int64_t* price,
                                                int E, int G, int gl, int64_t scale,
                                                int64_t (&v1)[NT], int64_t (&v2)[NT],
                                                int (&e1)[NT]) {
#pragma unroll
    for (int u = 0; u < NT; ++u) {
        v1[u] = INT64_MIN;
        v2[u] = INT64_MIN;
        e1[u] = INT32_MAX;
    }
#pragma unroll 4
    for (int e = gl; e < E; e += G) {
        int32_t qv[NT];
#pragma unroll
        for (int u = 0; u < NT; ++u) qv[u] = valid[u] ? __ldg(q + (size_t)t[u] * E + e) : 0;
        const int64_t pe = price[e];
#pragma unroll
        for (int u = 0; u < NT; ++u) {
            if (!valid[u]) continue;
            const int64_t v = (int64_t)qv[u] * scale - pe;
            const bool g1 = v > v1[u], g2 = v > v2[u];
            v2[u] = g1 ? v1[u] : (g2 ? v : v2[u]);
            v1[u] = g1 ? v : v1[u];
            e1[u] = g1 ? e : e1[u];
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        if (off >= G) continue;
#pragma unroll
        for (int u = 0; u < NT; ++u) {
            const int64_t ov1 = __shfl_xor_sync(0xffffffffu, v1[u], off);
            const int64_t ov2 = __shfl_xor_sync(0xffffffffu, v2[u], off);
            const int oe1 = __shfl_xor_sync(0xffffffffu, e1[u], off);
            const bool tk = (ov1 > v1[u]) | ((ov1 == v1[u]) & (oe1 < e1[u]));
            v2[u] = tk ? max(v1[u], ov2) : max(v2[u], ov1);
            v1[u] = tk ? ov1 : v1[u];
            e1[u] = tk ? oe1 : e1[u];
        }
    }
}

// Two tokens' scans interleaved (their loads in flight together); the rows
// may be in global or shared memory (generic loads).
__device__ __forceinline__ void group_bid2(const int32_t* r0, const int32_t* r1, bool ok0, bool ok1,
                                           const int64_t* price, int E, int G, int gl,
                                           int64_t scale, int64_t (&v1)[2], int64_t (&v2)[2],
                                           int (&e1)[2]) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        v1[u] = INT64_MIN;
        v2[u] = INT64_MIN;
        e1[u] = INT32_MAX;
    }
    for (int e = gl; e < E; e += G) {
        const int32_t a0 = ok0 ? r0[e] : 0;
        const int32_t a1 = ok1 ? r1[e] : 0;
        const int64_t pe = price[e];
        const int32_t qa[2] = {a0, a1};
        const bool ok[2] = {ok0, ok1};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (!ok[u]) continue;
            const int64_t v = (int64_t)qa[u] * scale - pe;
            const bool g1 = v > v1[u], g2 = v > v2[u];
            v2[u] = g1 ? v1[u] : (g2 ? v : v2[u]);
            v1[u] = g1 ? v : v1[u];
            e1[u] = g1 ? e : e1[u];
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        if (off >= G) continue;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t ov1 = __shfl_xor_sync(0xffffffffu, v1[u], off);
            const int64_t ov2 = __shfl_xor_sync(0xffffffffu, v2[u], off);
            const int oe1 = __shfl_xor_sync(0xffffffffu, e1[u], off);
            const bool tk = (ov1 > v1[u]) | ((ov1 == v1[u]) & (oe1 < e1[u]));
            v2[u] = tk ? max(v1[u], ov2) : max(v2[u], ov1);
            v1[u] = tk ? ov1 : v1[u];
            e1[u] = tk ? oe1 : e1[u];
        }
    }
}

// Where the score rows of the next round's bidders go: list position pos <
// cap is copied into rows[pos] (E int32, 16-byte chunks, cp.async by the
// pushing lane); rows == nullptr: no staging (wide rounds).
struct RowStage {
    int32_t* rows;
    int cap;
    __device__ __forceinline__ void stage(const int32_t* q, int E, int tok, int pos) const {
        if (rows == nullptr || pos >= cap) return;
        const char* src = reinterpret_cast<const char*>(q + (size_t)tok * E);
        const uint32_t dst = smem_u32(rows + (size_t)pos * E);
        for (int off = 0; off < E * 4; off += 16)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + off), "l"(src + off)
                         : "memory");
    }
    // the same copy spread over the 32 lanes of a warp (all lanes call it)
    __device__ __forceinline__ void stage_warp(const int32_t* q, int E, int tok, int pos) const {
        if (rows == nullptr || pos >= cap) return;
        const char* src = reinterpret_cast<const char*>(q + (size_t)tok * E);
        const uint32_t dst = smem_u32(rows + (size_t)pos * E);
        for (int off = lane_id() * 16; off < E * 4; off += 32 * 16)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + off), "l"(src + off)
                         : "memory");
    }
};

// Keeps the C best of held + new for expert e (held in global memory), with
// a team of TEAM threads.  Rejected tokens are appended to `unext` through
// the counter `ucnt`.  Returns the expert's new held count; `price` is set
// when the expert is full.
template <int TEAM>
__device__ int resolve_general(const Team<TEAM>& tm, const Params& p, int e, const Cands& cd,
                               int64_t* hb, int32_t* ht, int32_t* unext, int32_t* ucnt,
                               int64_t& price, const RowStage& rs) {
    const int C = p.C, h = cd.h, n = cd.n;
    const int tid = tm.tid();
    if (h + n <= C) {
        for (int j = tid; j < n; j += TEAM) {
            const Key x = cd.get(h + j);
            hb[h + j] = x.bid;
            ht[h + j] = x.tok;
        }
        tm.sync();
        if (h + n == C) {
            int64_t mn = INT64_MAX;
            for (int i = tid; i < C; i += TEAM) mn = min(mn, hb[i]);
            price = tm.min_i64(mn);
        }
        return h + n;
    }
    const int k = h + n - C;
    const Key kth = kth_worst<TEAM>(tm, cd, k, p.T - 1);
    int32_t* gfree = p.gfree + (size_t)e * C;
    // pass 1: free slots (rejected held, then the empty tail) in slot order
    int nfree = 0;
    for (int b0 = 0; b0 < C; b0 += TEAM) {
        const int i = b0 + tid;
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
        int nrej = 0;
        const int rr = tm.rank(rej, nrej);
        int base = 0;
        if (nrej) {
            if (TEAM == 32) {
                if (lane_id() == 0) base = atomicAdd(ucnt, nrej);
                base = __shfl_sync(0xffffffffu, base, 0);
            } else {
                if (tid == 0) tm.cnt[33] = atomicAdd(ucnt, nrej);
                __syncthreads();
                base = tm.cnt[33];
                __syncthreads();
            }
        }
        if (rej) {
            unext[base + rr] = tok;
            rs.stage(p.q, p.E, tok, base + rr);
        }
        int tot = 0;
        const int r = tm.rank(isfree, tot);
        if (isfree) gfree[nfree + r] = i;
        nfree += tot;
    }
    tm.sync();
    __threadfence_block();
    // pass 2: new bids; accepted ones take the free slots in order
    int nacc = 0;
    for (int b0 = 0; b0 < n; b0 += TEAM) {
        const int j = b0 + tid;
        bool acc = false, rej = false;
        Key x = pad_key();
        if (j < n) {
            x = cd.get(h + j);
            acc = worse(kth, x);
            rej = !acc;
        }
        int nrej = 0;
        const int rr = tm.rank(rej, nrej);
        int base = 0;
        if (nrej) {
            if (TEAM == 32) {
                if (lane_id() == 0) base = atomicAdd(ucnt, nrej);
                base = __shfl_sync(0xffffffffu, base, 0);
            } else {
                if (tid == 0) tm.cnt[33] = atomicAdd(ucnt, nrej);
                __syncthreads();
                base = tm.cnt[33];
                __syncthreads();
            }
        }
        if (rej) {
            unext[base + rr] = x.tok;
            rs.stage(p.q, p.E, x.tok, base + rr);
        }
        int tot = 0;
        const int r = tm.rank(acc, tot);
        if (acc) {
            const int slot = gfree[nacc + r];
            hb[slot] = x.bid;
            ht[slot] = x.tok;
        }
        nacc += tot;
    }
    tm.sync();
    __threadfence_block();
    if (nacc != nfree && tid == 0) record_error(1000 + e);
    int64_t mn = INT64_MAX;
    for (int i = tid; i < C; i += TEAM) mn = min(mn, hb[i]);
    price = tm.min_i64(mn);
    return C;
}

// Builds the fringe of an expert holding C keys: its min(FK, C) worst held
// keys, sorted ascending, found as the FK-th worst key by a radix select,
// collected with a team-wide ranking and sorted by warp 0.  Returns the
// fringe size.
// Ascending sort (in "worse" order) of P keys in shared memory, P a power of
// two <= 2 kThreads; the whole CTA takes part (bitonic network; one warp
// in registers when P <= 64).
__device__ void cta_sort_keys(Key* a, int P) {
    if (P <= 64) {
        if (warp_id() == 0) {
            const int lane = lane_id();
            Key x0 = lane < P ? a[lane] : pad_key();
            Key x1 = lane + 32 < P ? a[lane + 32] : pad_key();
            Key lo, hi;
            warp_merge64(warp_sort(x0), warp_sort(x1), lo, hi);
            if (lane < P) a[lane] = lo;
            if (lane + 32 < P) a[lane + 32] = hi;
        }
        __syncthreads();
        return;
    }
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = threadIdx.x; t < P / 2; t += kThreads) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const Key x = a[lo], y = a[hi];
                if (up ? worse(y, x) : worse(x, y)) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            __syncthreads();
        }
    }
}

constexpr int kSortMax = kWarps * kHist * 4 / (int)sizeof(Key);  // keys the histogram area holds

// The end of a CTA-wide resolve: the k rejected keys rejs[0, k) (any order)
// and the f new fringe keys frs[0, f) (sorted), each with its candidate
// index in .slot; Xk = the k-th worst (k > 0).  Rejected tokens go to the
// next round's list, accepted bids take the freed slots (rejected held
// keys' slots, then the empty ones), the fringe gets the final slots.
__device__ void finish_cta_resolve(const Team<kThreads>& tm, const Params& p, const Cands& cd,
                                   Key* sk, int64_t* hb, int32_t* ht, int32_t* unext,
                                   int32_t* ucnt, Key* gfr, const Key* rejs, int k,
                                   const Key* frs, int f, const Key& Xk, int& h_out, int& fs_out,
                                   int64_t& price) {
    const int C = p.C, h = cd.h, n = cd.n, m = h + n;
    const int tid = threadIdx.x;
    int32_t* fslot = reinterpret_cast<int32_t*>(sk + m);  // freed slots
    if (tid == 0) {
        tm.cnt[46] = k > 0 ? atomicAdd(ucnt, k) : 0;
        tm.cnt[47] = 0;
    }
    __syncthreads();
    const int base = tm.cnt[46];
    for (int i = tid; i < k; i += kThreads) {
        const Key x = rejs[i];
        unext[base + i] = x.tok;
        if (x.slot < h) fslot[atomicAdd(&tm.cnt[47], 1)] = x.slot;
    }
    __syncthreads();
    const int kh = tm.cnt[47];
    for (int j = tid; j < C - h; j += kThreads) fslot[kh + j] = h + j;
    if (tid == 0) tm.cnt[45] = 0;
    __syncthreads();
    // accepted new bids (above the k-th worst) take the freed slots
    for (int c = h + tid; c < m; c += kThreads) {
        const Key x = sk[c];
        if ((k == 0) | worse(Xk, x)) {
            const int slot = fslot[atomicAdd(&tm.cnt[45], 1)];
            hb[slot] = x.bid;
            ht[slot] = x.tok;
            sk[c].slot = slot;
        }
    }
    __syncthreads();
    if (tm.cnt[45] != n - k + kh && tid == 0) record_error(1100);
    // the new fringe with the final slots
    for (int i = tid; i < f; i += kThreads) {
        const Key x = frs[i];
        gfr[i] = Key{x.bid, x.tok, sk[x.slot].slot};
    }
    const int nh = m - k;
    if (nh == C) price = frs[0].bid;
    h_out = nh;
    fs_out = f;
    __syncthreads();
}

// CTA-wide resolve of one expert in a wide round with every candidate (held
// keys, then new bids) copied into shared memory once.  With k rejections
// and f keys in the new fringe, the (k + f)-th worst key is found by a radix
// select over the copy and the k + f keys up to it are collected; a second
// select over those splits off the k rejected (or, for at most 64 keys, a
// sort orders them); the f others, sorted, are the new fringe (exact), and
// the price is the smallest kept bid.  Returns false, having done nothing,
// when the candidates do not fit the scratch or k + f keys do not fit the
// collection area.
__device__ bool resolve_cta_cached(const Team<kThreads>& tm, const Params& p, const Cands& cd,
                                   Key* sk, int cap, int64_t* hb, int32_t* ht, int32_t* unext,
                                   int32_t* ucnt, Key* gfr, int& h_out, int& fs_out,
                                   int64_t& price) {
    const int C = p.C, h = cd.h, n = cd.n, m = h + n;
    const int tid = threadIdx.x;
    const int k = max(0, m - C);
    const int nh = m - k;          // held after the round: min(m, C)
    const int f = min(p.FK, nh);   // the new fringe (complete when nh <= FK)
    const int S = k + f;
    // the copy (m keys) and the freed-slot list (C ints) share the scratch
    if (m == 0 || m + (C + 3) / 4 > cap || S > kSortMax || S > 2 * kThreads) return false;
    for (int c = tid; c < m; c += kThreads) sk[c] = cd.get(c);  // slot: c (held) or -1 (new)
    __syncthreads();
    auto visit = [&](auto fn) {
        for (int c = tid; c < m; c += kThreads) fn(sk[c]);
    };
    const Key Y = kth_worst_v<kThreads>(tm, visit, S, p.T - 1);
    // the S keys up to Y, with their candidate index in .slot
    Key* srt = reinterpret_cast<Key*>(tm.hist);
    if (tid == 0) tm.cnt[45] = 0;
    __syncthreads();
    for (int c = tid; c < m; c += kThreads) {
        const Key x = sk[c];
        if (!worse(Y, x)) srt[atomicAdd(&tm.cnt[45], 1)] = Key{x.bid, x.tok, c};
    }
    __syncthreads();
    if (S <= 64) {
        // one warp sorts them (padded): rejected srt[0, k), fringe srt[k, S)
        for (int i = S + tid; i < 64; i += kThreads) srt[i] = pad_key();
        __syncthreads();
        cta_sort_keys(srt, 64);
        const Key Xk = k > 0 ? srt[k - 1] : pad_key();
        finish_cta_resolve(tm, p, cd, sk, hb, ht, unext, ucnt, gfr, srt, k, srt + k, f, Xk, h_out,
                           fs_out, price);
        return true;
    }
    // k > 0 here (S > 64 > f): the k worst of the S collected keys by a
    // second select over them (two per thread, in registers); then the f
    // others are moved to the front and sorted, the rejected ones follow
    const Key k0 = tid < S ? srt[tid] : pad_key();
    const Key k1 = tid + kThreads < S ? srt[tid + kThreads] : pad_key();
    auto visit2 = [&](auto fn) {
        if (tid < S) fn(k0);
        if (tid + kThreads < S) fn(k1);
    };
    const Key Xk = kth_worst_v<kThreads>(tm, visit2, k, p.T - 1);
    if (tid == 0) {
        tm.cnt[45] = 0;  // fringe keys placed
        tm.cnt[48] = 0;  // rejected keys placed
    }
    __syncthreads();
    if (tid < S) {
        const bool rj = !worse(Xk, k0);
        srt[rj ? f + atomicAdd(&tm.cnt[48], 1) : atomicAdd(&tm.cnt[45], 1)] = k0;
    }
    if (tid + kThreads < S) {
        const bool rj = !worse(Xk, k1);
        srt[rj ? f + atomicAdd(&tm.cnt[48], 1) : atomicAdd(&tm.cnt[45], 1)] = k1;
    }
    __syncthreads();
    if (warp_id() == 0) {  // f <= 32: one key per lane
        const int lane = lane_id();
        Key x = lane < f ? srt[lane] : pad_key();
        x = warp_sort(x);
        __syncwarp();
        if (lane < f) srt[lane] = x;
    }
    __syncthreads();
    finish_cta_resolve(tm, p, cd, sk, hb, ht, unext, ucnt, gfr, srt + f, k, srt, f, Xk, h_out,
                       fs_out, price);
    return true;
}

// ---------------------------------------------------------------- sorted held sets
// Wide rounds can keep held sets sorted.  The CTA that owns expert e (e %
// grid) holds e's held keys in shared memory in "worse" order (worst first),
// in two buffers that alternate by round.  A resolve then needs no select:
// the new bids are sorted, a key's place in the merged order is its index
// plus its rank in the other list (a binary search; keys are unique), the
// first k places are rejected and the rest is the new held set.  It goes to
// the other buffer and through to the global held arrays and the fringe
// (its first FK keys, slot = index), which the narrow rounds and the final
// assignment read.
struct SortedSet {
    int64_t* b;
    int32_t* t;
};

// number of keys of the sorted list (b, t)[0, n) that are worse than x
__device__ __forceinline__ int rank_sorted(const int64_t* b, const int32_t* t, int n,
                                           const Key& x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const bool w = worse(Key{b[mid], t[mid], 0}, x);
        lo = w ? mid + 1 : lo;
        hi = w ? hi : mid;
    }
    return lo;
}

// number of keys of the sorted keys a[0, n) that are worse than x
__device__ __forceinline__ int rank_keys(const Key* a, int n, const Key& x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const bool w = worse(a[mid], x);
        lo = w ? mid + 1 : lo;
        hi = w ? hi : mid;
    }
    return lo;
}

constexpr int kSortedSmall = 2048;  // new bids sorted whole up to this many

// Ascending ("worse" order) sort of n keys in shared memory by the whole CTA:
// every warp sorts runs of 32 keys in registers, then merge levels double
// the run length; at each level a key's new place is its offset in its run
// plus its rank in the partner run (a binary search; keys are unique).
// a and tmp hold n keys each; returns the buffer that holds the result.
__device__ Key* cta_sort_keys_fast(Key* a, Key* tmp, int n) {
    const int lane = lane_id(), warp = warp_id();
    for (int r0 = warp * 32; r0 < n; r0 += kWarps * 32) {
        Key x = r0 + lane < n ? a[r0 + lane] : pad_key();
        x = warp_sort(x);
        if (r0 + lane < n) a[r0 + lane] = x;
    }
    __syncthreads();
    Key* src = a;
    Key* dst = tmp;
    for (int R = 32; R < n; R <<= 1) {
        for (int i0 = threadIdx.x; i0 < n; i0 += 2 * kThreads) {
            // two keys per thread per pass, their searches interleaved
            Key x[2];
            int pos[2], lo[2], hi[2];
            bool ok[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = i0 + u * kThreads;
                ok[u] = i < n;
                pos[u] = 0;
                lo[u] = hi[u] = 0;
                if (ok[u]) {
                    x[u] = src[i];
                    const int run = i / R;
                    const int pair0 = (run & ~1) * R;
                    const int ps = (run ^ 1) * R;  // the partner run
                    lo[u] = min(ps, n);
                    hi[u] = min(ps + R, n);
                    pos[u] = pair0 + (i - run * R) - lo[u];
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                int l = lo[u], h = hi[u];
                while (l < h) {
                    const int mid = (l + h) >> 1;
                    const bool w = worse(src[mid], x[u]);
                    l = w ? mid + 1 : l;
                    h = w ? h : mid;
                }
                if (ok[u]) dst[pos[u] + l] = x[u];  // pos + l in [0, n)
            }
        }
        __syncthreads();
        Key* t = src;
        src = dst;
        dst = t;
    }
    return src;
}

// The same for distinct 64-bit keys in ascending order (a packed key's order
// is the "worse" order: see resolve_sorted): half the shared-memory traffic
// of a 16-byte key per search step and one compare.
__device__ __forceinline__ uint64_t warp_sort_u64(uint64_t x) {
    const int lane = lane_id();
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const uint64_t o = __shfl_xor_sync(0xffffffffu, x, j);
            const bool up = (lane & k) == 0;
            const bool lower = (lane & j) == 0;
            x = ((lower == up) ? (o < x) : (x < o)) ? o : x;
        }
    }
    return x;
}

__device__ uint64_t* cta_sort_u64(uint64_t* a, uint64_t* tmp, int n) {
    const int lane = lane_id(), warp = warp_id();
    for (int r0 = warp * 32; r0 < n; r0 += kWarps * 32) {
        uint64_t x = r0 + lane < n ? a[r0 + lane] : ~0ull;
        x = warp_sort_u64(x);
        if (r0 + lane < n) a[r0 + lane] = x;
    }
    __syncthreads();
    uint64_t* src = a;
    uint64_t* dst = tmp;
    for (int R = 32; R < n; R <<= 1) {
        for (int i0 = threadIdx.x; i0 < n; i0 += 2 * kThreads) {
            uint64_t x[2];
            int pos[2], lo[2], hi[2];
            bool ok[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = i0 + u * kThreads;
                ok[u] = i < n;
                pos[u] = 0;
                lo[u] = hi[u] = 0;
                x[u] = 0;
                if (ok[u]) {
                    x[u] = src[i];
                    const int run = i / R;
                    const int pair0 = (run & ~1) * R;
                    const int ps = (run ^ 1) * R;  // the partner run
                    lo[u] = min(ps, n);
                    hi[u] = min(ps + R, n);
                    pos[u] = pair0 + (i - run * R) - lo[u];
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                int l = lo[u], h = hi[u];
                while (l < h) {
                    const int mid = (l + h) >> 1;
                    const bool w = src[mid] < x[u];
                    l = w ? mid + 1 : l;
                    h = w ? h : mid;
                }
                if (ok[u]) dst[pos[u] + l] = x[u];  // pos + l in [0, n)
            }
        }
        __syncthreads();
        uint64_t* t = src;
        src = dst;
        dst = t;
    }
    return src;
}

// Keeps the C best of the sorted held set cur[0, h) and the n new bids
// (nb, nt) of one expert.  The new held set (sorted) goes to nxt and to the
// global hb / ht / fringe gfr; rejected tokens go to unext through ucnt.
// sk, sk2: scratch of nsc keys each (nsc a power of two >= C).  Returns the new held count;
// sets price (the smallest held bid) when the expert is full.  Bids beyond
// kSortedSmall go through a radix select first (then only the accepted ones,
// at most C, are sorted).
__device__ int resolve_sorted(const Team<kThreads>& tm, const Params& p, SortedSet cur, int h,
                              SortedSet nxt, const int64_t* nb, const int32_t* nt, int n,
                              Key* sk, Key* sk2, int nsc, int64_t* hb, int32_t* ht, Key* gfr,
                              int32_t* unext, int32_t* ucnt, int64_t& price) {
    const int C = p.C, FK = p.FK, tid = threadIdx.x;
    const int m = h + n, k = max(0, m - C), nh = m - k;
    if (tid == 0) {
        tm.cnt[56] = k > 0 ? atomicAdd(ucnt, k) : 0;
        tm.cnt[57] = 0;  // new keys accepted (large case)
        tm.cnt[58] = 0;  // new keys rejected (large case)
    }
    __syncthreads();
    const int base = tm.cnt[56];
    auto keep = [&](int r, const Key& x) {
        if (r < 0 || r >= C) return;  // (only an inconsistent select could get here)
        nxt.b[r] = x.bid;
        nxt.t[r] = x.tok;
        hb[r] = x.bid;
        ht[r] = x.tok;
        if (r < FK) gfr[r] = Key{x.bid, x.tok, r};
    };
    if (n <= kSortedSmall && n <= nsc && h == 0) {
        // an expert's first bids (every phase start): when the bid range
        // leaves room for the token, each bid becomes one 64-bit key
        // ((bid - lo) << tb | (T - 1 - tok)) whose ascending order is the
        // "worse" order, and the sorted keys are the held set in order
        int64_t lo = INT64_MAX, hi = INT64_MIN;
        for (int i = tid; i < n; i += kThreads) {
            lo = min(lo, nb[i]);
            hi = max(hi, nb[i]);
        }
        tm.minmax_i64(lo, hi);
        const int tb = max(1, bit_length_u64((uint64_t)(p.T - 1)));
        if (bit_length_u64((uint64_t)(hi - lo)) + tb <= 64) {
            uint64_t* pk = reinterpret_cast<uint64_t*>(sk);
            const uint64_t tmax = (uint64_t)(p.T - 1);
            const uint64_t tmask = (1ull << tb) - 1;  // tb <= 31
            for (int i = tid; i < n; i += kThreads)
                pk[i] = ((uint64_t)(nb[i] - lo) << tb) | (tmax - (uint64_t)(uint32_t)nt[i]);
            __syncthreads();
            const uint64_t* sp = cta_sort_u64(pk, reinterpret_cast<uint64_t*>(sk2), n);
            for (int j = tid; j < n; j += kThreads) {
                const uint64_t v = sp[j];
                const Key x{lo + (int64_t)(v >> tb), (int32_t)(tmax - (v & tmask)), 0};
                if (j < k) unext[base + j] = x.tok;
                else keep(j - k, x);
            }
            __syncthreads();
            if (nh == C) price = nxt.b[0];
            return nh;
        }
    }
    if (n <= kSortedSmall && n <= nsc) {
        for (int i = tid; i < n; i += kThreads) sk[i] = Key{nb[i], nt[i], -1};
        __syncthreads();
        const Key* srt = cta_sort_keys_fast(sk, sk2, n);
        for (int i = tid; i < h; i += kThreads) {
            const Key x{cur.b[i], cur.t[i], 0};
            const int pos = i + rank_keys(srt, n, x);
            if (pos < k) unext[base + pos] = x.tok;
            else keep(pos - k, x);
        }
        for (int j = tid; j < n; j += kThreads) {
            const Key x = srt[j];
            const int pos = j + rank_sorted(cur.b, cur.t, h, x);
            if (pos < k) unext[base + pos] = x.tok;
            else keep(pos - k, x);
        }
    } else {
        // k >= 1 here: n > min(kSortedSmall, nsc) >= C.  X = the k-th worst
        // of held + new; held keys up to X are a prefix cur[0, a0)
        auto visit = [&](auto fn) {
            for (int i = tid; i < h; i += kThreads) fn(Key{cur.b[i], cur.t[i], 0});
            for (int j = tid; j < n; j += kThreads) fn(Key{nb[j], nt[j], -1});
        };
        const Key X = kth_worst_v<kThreads>(tm, visit, k, p.T - 1);
        const int r = rank_sorted(cur.b, cur.t, h, X);
        const int a0 = r + ((r < h && cur.b[r] == X.bid && cur.t[r] == X.tok) ? 1 : 0);
        for (int i = tid; i < min(a0, k); i += kThreads) unext[base + i] = cur.t[i];
        for (int j = tid; j < n; j += kThreads) {
            const Key x{nb[j], nt[j], -1};
            if (!worse(X, x)) {
                const int at = a0 + atomicAdd(&tm.cnt[58], 1);
                if (at < k) unext[base + at] = x.tok;
            } else {
                const int at = atomicAdd(&tm.cnt[57], 1);
                if (at < nsc) sk[at] = x;
            }
        }
        __syncthreads();
        const int nacc = min(tm.cnt[57], nsc);
        if (tid == 0 && (tm.cnt[57] + (h - a0) != nh || a0 + tm.cnt[58] != k)) record_error(1200);
        const Key* srt = cta_sort_keys_fast(sk, sk2, nacc);
        for (int i = a0 + tid; i < h; i += kThreads) {
            const Key x{cur.b[i], cur.t[i], 0};
            keep(i - a0 + rank_keys(srt, nacc, x), x);
        }
        for (int j = tid; j < nacc; j += kThreads) {
            const Key x = srt[j];
            keep(j + rank_sorted(cur.b + a0, cur.t + a0, h - a0, x), x);
        }
    }
    __syncthreads();
    if (nh == C) price = nxt.b[0];
    return nh;
}

template <int TEAM>
__device__ int build_fringe_radix(const Team<TEAM>& tm, const int64_t* hb, const int32_t* ht,
                                  int C, int FK, int tmax, Key* fr) {
    const int k = min(FK, C);
    if (k == 0) return 0;
    const Cands cd{hb, ht, nullptr, nullptr, C, 0};
    const Key kth = kth_worst<TEAM>(tm, cd, k, tmax);
    Key* stage = reinterpret_cast<Key*>(tm.hist);  // 64 keys fit in the histogram area
    int got = 0;
    for (int b0 = 0; b0 < C; b0 += TEAM) {
        const int i = b0 + tm.tid();
        Key x = pad_key();
        bool in = false;
        if (i < C) {
            x = Key{hb[i], ht[i], i};
            in = !worse(kth, x);
        }
        int tot = 0;
        const int r = tm.rank(in, tot);
        if (in) stage[got + r] = x;
        got += tot;
    }
    tm.sync();
    if (TEAM == 32 || warp_id() == 0) {
        Key x = lane_id() < k ? stage[lane_id()] : pad_key();
        x = warp_sort(x);
        if (lane_id() < k) fr[lane_id()] = x;
    }
    tm.sync();
    return k;
}

// Warp version: a sampled threshold first.  Each lane keeps the two worst
// keys of its stripe (the candidates); sorted, the 32 worst candidates are
// lo and the 32nd of them, theta, has at least 32 held keys at or below it.
// Those are lo plus the held keys at or below theta that are not
// candidates (usually none): collected (at most 32, else the radix build
// runs), sorted and merged into lo.  Both passes over the held keys issue
// kLoads loads before they use one (the collect's shared-memory stores would
// otherwise keep the next loads from starting: the held keys may be in shared
// memory too).
constexpr int kLoads = 8;

__device__ int build_fringe_warp(const Team<32>& tm, const int64_t* hb, const int32_t* ht, int C,
                                 int FK, int tmax, Key* fr) {
    const int k = min(FK, C);
    if (k == 0) return 0;
    const int lane = lane_id();
    Key lo, hi;
    if (C <= 64) {
        Key a = lane < C ? Key{hb[lane], ht[lane], lane} : pad_key();
        Key b = lane + 32 < C ? Key{hb[lane + 32], ht[lane + 32], lane + 32} : pad_key();
        warp_merge64(warp_sort(a), warp_sort(b), lo, hi);
    } else {
        Key a = pad_key(), b = pad_key();
        for (int i0 = 0; i0 < C; i0 += 32 * kLoads) {
            Key x[kLoads];
#pragma unroll
            for (int u = 0; u < kLoads; ++u) {
                const int i = i0 + 32 * u + lane;
                x[u] = i < C ? Key{hb[i], ht[i], i} : pad_key();
            }
#pragma unroll
            for (int u = 0; u < kLoads; ++u) {
                const bool wa = worse(x[u], a), wb = worse(x[u], b);
                b = sel_key(wa, a, sel_key(wb, x[u], b));
                a = sel_key(wa, x[u], a);
            }
        }
        warp_merge64(warp_sort(a), warp_sort(b), lo, hi);
        const Key theta = shfl_key(lo, 31);
        Key* stage = reinterpret_cast<Key*>(tm.hist);  // 32 keys
        const unsigned lt = (1u << lane) - 1;
        int got = 0;
        for (int i0 = 0; i0 < C; i0 += 32 * kLoads) {
            Key x[kLoads];
#pragma unroll
            for (int u = 0; u < kLoads; ++u) {
                const int i = i0 + 32 * u + lane;
                x[u] = i < C ? Key{hb[i], ht[i], i} : pad_key();
            }
            unsigned m[kLoads];
#pragma unroll
            for (int u = 0; u < kLoads; ++u) {
                const int i = i0 + 32 * u + lane;
                m[u] = __ballot_sync(0xffffffffu, (i < C) & !worse(theta, x[u]) & (i != a.slot) &
                                                      (i != b.slot));
            }
#pragma unroll
            for (int u = 0; u < kLoads; ++u) {
                const int pos = got + __popc(m[u] & lt);
                if (((m[u] >> lane) & 1u) & (pos < 32)) stage[pos] = x[u];
                got += __popc(m[u]);
            }
        }
        __syncwarp();
        if (got > 32) return build_fringe_radix<32>(tm, hb, ht, C, FK, tmax, fr);
        if (got > 0) {
            const Key x = lane < got ? stage[lane] : pad_key();
            __syncwarp();
            warp_merge64(lo, warp_sort(x), lo, hi);
        }
    }
    if (lane < k) fr[lane] = lo;
    __syncwarp();
    return k;
}

template <int TEAM>
__device__ int build_fringe(const Team<TEAM>& tm, const int64_t* hb, const int32_t* ht, int C,
                            int FK, int tmax, Key* fr) {
    if constexpr (TEAM == 32) return build_fringe_warp(tm, hb, ht, C, FK, tmax, fr);
    else return build_fringe_radix<TEAM>(tm, hb, ht, C, FK, tmax, fr);
}

// position of the r-th (from 0) set bit of m, 0 when m has at most r set
// bits; five branch-free halving steps (a per-lane loop of r steps diverges)
__device__ __forceinline__ int nth_set_lane(unsigned m, int r) {
    const bool found = __popc(m) > r;
    int pos = 0;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const int c = __popc(m & ((1u << w) - 1));
        const bool up = r >= c;  // the bit is in the upper half
        r = up ? r - c : r;
        m = up ? m >> w : m;
        pos = up ? pos + w : pos;
    }
    return found ? pos : 0;
}

// One bid to a full expert whose fringe holds at least two keys (the usual
// case in the last rounds of a phase): the bid is above the price, the
// fringe minimum f0, so f0 is rejected and the bid takes its slot; the new
// fringe is f1.. with the bid inserted where it belongs (when not above the
// fringe maximum of an incomplete fringe).  Every load is issued up front.
// Returns the rejected token; sets fs and the new price (the new minimum).
__device__ __forceinline__ int fringe_take_one(Key* fr, int& fs, int h, int64_t bid, int tok,
                                               int64_t* hb, int32_t* ht, int64_t& price) {
    const int lane = lane_id();
    const Key f0 = fr[0];
    const Key f1 = fr[1];
    const Key fl = fr[fs - 1];
    const Key fi = lane < fs ? fr[lane] : pad_key();
    const Key fn = lane + 1 < fs ? fr[lane + 1] : pad_key();
    const Key b = Key{bid, tok, f0.slot};
    const bool ins = (fs == h) | !worse(fl, b);
    const int pos = __popc(__ballot_sync(0xffffffffu, (lane + 1 < fs) & worse(fn, b)));
    Key out = lane < pos ? fn : (lane == pos ? b : fi);
    if (!ins) out = fn;
    const int nfs = ins ? fs : fs - 1;
    price = (ins && pos == 0) ? bid : f1.bid;
    __syncwarp();
    if (lane < nfs) fr[lane] = out;
    if (lane == 0) {
        hb[b.slot] = bid;
        ht[b.slot] = tok;
    }
    __syncwarp();
    fs = nfs;
    return f0.tok;
}

// One step of a sequential resolve: key b enters a full expert and the worst
// key leaves.  When b is worse than the fringe minimum f0, b itself leaves;
// otherwise f0 leaves and b takes its slot (inserted into the fringe as in
// fringe_take_one).  Needs fs >= 2.  Returns the token that left.
__device__ __forceinline__ int fringe_push_pop(Key* fr, int& fs, int h, int64_t bid, int tok,
                                               int64_t* hb, int32_t* ht) {
    const Key f0 = fr[0];
    if (worse(Key{bid, tok, -1}, f0)) return tok;
    int64_t price;
    return fringe_take_one(fr, fs, h, bid, tok, hb, ht, price);
}

// Warp-level resolve of one expert from its fringe and n < 32 new bids.
// The fringe holds the expert's fs worst held keys, sorted ascending; it is
// "complete" when it holds all h of them.  The k = max(0, h + n - C) worst of
// held + new are among fringe + new whenever the fringe is complete or k < fs,
// so the sorted merge of the two lists decides the round: its first k keys
// are rejected, accepted new keys take the slots of rejected fringe keys and
// then the empty slots h, h+1, ..; the survivors not above the old fringe
// maximum (all survivors when complete) form the new fringe.  Returns false
// (nothing changed) when the fringe cannot decide; sets price when the expert
// is full and its new fringe is not empty (fs == 0 afterwards: rebuild).
__device__ bool resolve_warp(const Params& p, Key* fr, int& fs, int& h, const int64_t* nb,
                             const int32_t* nt, int n, int64_t* hb, int32_t* ht,
                             int32_t* next_list, int* next_cnt, int64_t& price,
                             const RowStage& rs) {
    const int C = p.C, FK = p.FK;
    const int lane = lane_id();
    const unsigned lt = (1u << lane) - 1;
    const bool complete = (fs == h);
    const int k = max(0, h + n - C);
    if (!complete && k >= fs) return false;
    if (h == C && n >= 2 && n <= 8 && fs >= 2 && (complete || fs >= n + 1)) {
        // a few bids to a full expert: "one in, the worst out" n times keeps
        // the C best of held + new, the same set as the merge below, and
        // rejects the n worst; each step is one pass over the fringe
        int rej = -1;
        for (int i = 0; i < n; ++i) {
            const int t = fringe_push_pop(fr, fs, h, nb[i], nt[i], hb, ht);
            if (lane == i) rej = t;
        }
        int base = 0;
        if (lane == 0) base = atomicAdd(next_cnt, n);
        base = __shfl_sync(0xffffffffu, base, 0);
        if (lane < n) {
            next_list[base + lane] = rej;
            rs.stage(p.q, p.E, rej, base + lane);
        }
        __syncwarp();
        price = fr[0].bid;
        return true;
    }
    if (n == 1 && h == C && fs >= 2) {
        // one bid b to a full expert: b beats the price (the fringe minimum
        // f0), so f0 is rejected and b takes its slot; the new fringe is
        // f1.. with b inserted where it belongs (when not above the maximum)
        const Key b0 = Key{nb[0], nt[0], -1};
        const Key fi = lane < fs ? fr[lane] : pad_key();
        const Key fn = lane + 1 < fs ? fr[lane + 1] : pad_key();
        const Key f0 = shfl_key(fi, 0);
        const Key b = Key{b0.bid, b0.tok, f0.slot};
        const bool ins = complete | !worse(shfl_key(fi, fs - 1), b);
        const int pos = __popc(__ballot_sync(0xffffffffu, (lane + 1 < fs) & worse(fn, b)));
        Key out = lane < pos ? fn : (lane == pos ? b : fi);
        if (!ins) out = fn;
        const int nfs = ins ? fs : fs - 1;
        int at = 0;
        if (lane == 0) {
            hb[b.slot] = b.bid;
            ht[b.slot] = b.tok;
            at = atomicAdd(next_cnt, 1);
            next_list[at] = f0.tok;
        }
        at = __shfl_sync(0xffffffffu, at, 0);
        rs.stage_warp(p.q, p.E, f0.tok, at);
        __syncwarp();
        if (lane < nfs) fr[lane] = out;
        __syncwarp();
        fs = nfs;
        price = shfl_key(out, 0).bid;
        return true;
    }
    const Key f = lane < fs ? fr[lane] : pad_key();
    const Key thr = complete ? pad_key() : shfl_key(f, max(fs, 1) - 1);
    Key lo, hi;
    if (n == 1) {
        // one new key: insert it into the sorted fringe
        const Key b = Key{nb[0], nt[0], -1};
        const int pos = __popc(__ballot_sync(0xffffffffu, (lane < fs) & worse(f, b)));
        const Key prev = shfl_key(f, (lane + 31) & 31);
        const Key top = shfl_key(f, 31);
        lo = lane < pos ? f : (lane == pos ? b : prev);
        hi = pad_key();
        if (lane == 0 && fs == 32) hi = (pos == 32) ? b : top;
    } else {
        Key x = lane < n ? Key{nb[lane], nt[lane], -1} : pad_key();
        x = warp_sort(x);
        warp_merge64(f, x, lo, hi);
    }
    const bool rej = lane < k;  // the first k elements (k <= n < 32: all in lo)
    const unsigned freed = __ballot_sync(0xffffffffu, rej & (lo.slot >= 0));
    const int nfreed = __popc(freed);
    const unsigned acc_lo = __ballot_sync(0xffffffffu, !rej & (lo.slot == -1));
    const unsigned acc_hi = __ballot_sync(0xffffffffu, hi.slot == -1);
    // the r-th accepted new key takes the r-th freed slot, then h + (r - nfreed)
    const int r_lo = __popc(acc_lo & lt);
    const int r_hi = __popc(acc_lo) + __popc(acc_hi & lt);
    const int s_lo = __shfl_sync(0xffffffffu, lo.slot, nth_set_lane(freed, min(r_lo, 31)));
    const int s_hi = __shfl_sync(0xffffffffu, lo.slot, nth_set_lane(freed, min(r_hi, 31)));
    if ((acc_lo >> lane) & 1u) {
        lo.slot = r_lo < nfreed ? s_lo : h + (r_lo - nfreed);
        hb[lo.slot] = lo.bid;
        ht[lo.slot] = lo.tok;
    }
    if ((acc_hi >> lane) & 1u) {
        hi.slot = r_hi < nfreed ? s_hi : h + (r_hi - nfreed);
        hb[hi.slot] = hi.bid;
        ht[hi.slot] = hi.tok;
    }
    if (k > 0) {  // rejected tokens bid next round
        const unsigned rm = __ballot_sync(0xffffffffu, rej);
        int base = 0;
        if (lane == 0) base = atomicAdd(next_cnt, k);
        base = __shfl_sync(0xffffffffu, base, 0);
        if (rej) {
            next_list[base + __popc(rm & lt)] = lo.tok;
            rs.stage(p.q, p.E, lo.tok, base + __popc(rm & lt));
        }
    }
    // the new fringe: survivors not above the threshold, in order, at most FK
    const bool keep_lo = !rej & (lo.slot != -2) & !worse(thr, lo);
    const bool keep_hi = (hi.slot != -2) & !worse(thr, hi);
    const unsigned kl = __ballot_sync(0xffffffffu, keep_lo);
    const unsigned kh = __ballot_sync(0xffffffffu, keep_hi);
    const int nl = __popc(kl);
    __syncwarp();
    if (keep_lo) {
        const int pos = __popc(kl & lt);
        if (pos < FK) fr[pos] = lo;
    }
    if (keep_hi) {
        const int pos = nl + __popc(kh & lt);
        if (pos < FK) fr[pos] = hi;
    }
    __syncwarp();
    fs = min(FK, nl + __popc(kh));
    h = min(C, h + n);
    if (h == C && fs > 0) price = fr[0].bid;
    return true;
}

// The end of a phase.  Once a round has a single bidder, so has every
// following round: its one bid either goes to an expert with room (the phase
// ends) or to a full expert, which then rejects exactly its worst held key
// (every bid is above the expert's price, the smallest held bid).  One warp
// runs these rounds back to back with no block barrier: lanes take experts
// (lane + 32 j, j < NJ) for the bid, the expert's fringe decides the round,
// and the rejected token's score row is loaded into registers while the
// resolve is written back.  The rounds are the same as in the other modes.
struct ChainScratch {
    int64_t* one_b;   // [1] the bid, for resolve_warp
    int32_t* one_t;   // [1]
    int32_t* next;    // [1] a rejected token
    int32_t* cnt;     // [1]
};

template <int NJ>
__device__ __forceinline__ void chain_rounds(const Params& p, int t, int64_t eps, int64_t scale,
                                          int64_t* s_price, Key* s_fr, int32_t* s_fsize,
                                          int32_t* s_hcnt, int64_t* hbase, int32_t* htbase,
                                          const ChainScratch cs,
                                          const Team<32>& wt, long long& rounds,
                                          long long& bids, int& status) {
    const int E = p.E, C = p.C, FK = p.FK, T = p.T;
    const int lane = lane_id();
    int32_t rv[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        rv[j] = e < E ? __ldg(p.q + (size_t)t * E + e) : 0;
    }
    while (true) {
        if (rounds >= p.max_rounds) {
            status = BASE_ERR_NOT_CONVERGED;
            return;
        }
        if (lane == 0) trace_round(p, rounds, 1);
        ++rounds;
        ++bids;
        // ---- bid: best and second-best value over the experts, lowest e on ties
        int64_t v1 = INT64_MIN, v2 = INT64_MIN;
        int e1 = INT32_MAX;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int e = lane + 32 * j;
            if (e < E) {
                const int64_t v = (int64_t)rv[j] * scale - s_price[e];
                const bool g1 = v > v1, g2 = v > v2;
                v2 = g1 ? v1 : (g2 ? v : v2);
                v1 = g1 ? v : v1;
                e1 = g1 ? e : e1;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const int64_t ov1 = __shfl_xor_sync(0xffffffffu, v1, off);
            const int64_t ov2 = __shfl_xor_sync(0xffffffffu, v2, off);
            const int oe1 = __shfl_xor_sync(0xffffffffu, e1, off);
            const bool tk = (ov1 > v1) | ((ov1 == v1) & (oe1 < e1));
            v2 = tk ? max(v1, ov2) : max(v2, ov1);
            v1 = tk ? ov1 : v1;
            e1 = tk ? oe1 : e1;
        }
        const int e = e1;
        // bid = q[t][e] (T+1) - v2 + eps = price[e] + (v1 - v2) + eps
        const int64_t bid = v1 + s_price[e] - v2 + eps;
        const int h = s_hcnt[e];
        const int fs = s_fsize[e];
        Key* fr = s_fr + (size_t)e * FK;
        int64_t* hb = hbase + (size_t)e * C;
        int32_t* ht = htbase + (size_t)e * C;
        int tn = -1;
        if (h == C && fs >= 2) {
            // the fringe minimum f0 is rejected (its row loaded right away)
            tn = fr[0].tok;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int ee = lane + 32 * j;
                rv[j] = ee < E ? __ldg(p.q + (size_t)tn * E + ee) : 0;
            }
            int nfs = fs;
            int64_t price;
            fringe_take_one(fr, nfs, h, bid, t, hb, ht, price);
            if (lane == 0) {
                s_fsize[e] = nfs;
                s_price[e] = price;
            }
            __syncwarp();
        } else {
            // the general merge (a fringe that must be rebuilt first, an
            // expert with room, a fringe of one key)
            if (lane == 0) {
                cs.one_b[0] = bid;
                cs.one_t[0] = t;
                cs.cnt[0] = 0;
            }
            __syncwarp();
            int fs2 = fs, hh = h;
            int64_t price = s_price[e];
            if (fs2 != hh && max(0, hh + 1 - C) >= fs2)
                fs2 = build_fringe<32>(wt, hb, ht, hh, FK, T - 1, fr);
            resolve_warp(p, fr, fs2, hh, cs.one_b, cs.one_t, 1, hb, ht, cs.next, cs.cnt, price,
                         RowStage{nullptr, 0});
            if (hh == C && fs2 == 0) {
                fs2 = build_fringe<32>(wt, hb, ht, hh, FK, T - 1, fr);
                price = fr[0].bid;
            }
            __syncwarp();
            if (lane == 0) {
                s_fsize[e] = fs2;
                s_hcnt[e] = hh;
                if (hh == C) s_price[e] = price;
            }
            const int n = cs.cnt[0];
            if (n > 0) {
                tn = cs.next[0];
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const int ee = lane + 32 * j;
                    rv[j] = ee < E ? __ldg(p.q + (size_t)tn * E + ee) : 0;
                }
            }
            __syncwarp();
        }
        if (tn < 0) return;  // the bid found room: the phase is over
        t = tn;
    }
}

__global__ void __launch_bounds__(kThreads, 1) auction_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const SmemLayout L = smem_layout(p.E, p.FK, p.narrow_max, p.NB, p.RC, p.T, p.HS);
    int64_t* s_price = reinterpret_cast<int64_t*>(smem + L.price);
    Key* s_fr = reinterpret_cast<Key*>(smem + L.fr);
    int32_t* s_fsize = reinterpret_cast<int32_t*>(smem + L.fsize);
    int32_t* s_hcnt = reinterpret_cast<int32_t*>(smem + L.hcnt);
    int32_t* s_ncnt = reinterpret_cast<int32_t*>(smem + L.ncnt);
    int32_t* s_act0 = reinterpret_cast<int32_t*>(smem + L.act0);
    int32_t* s_act1 = reinterpret_cast<int32_t*>(smem + L.act1);
    int64_t* s_nbk_b = reinterpret_cast<int64_t*>(smem + L.nbk_b);
    int32_t* s_nbk_t = reinterpret_cast<int32_t*>(smem + L.nbk_t);
    int32_t* s_list0 = reinterpret_cast<int32_t*>(smem + L.list0);
    int32_t* s_list1 = reinterpret_cast<int32_t*>(smem + L.list1);
    int32_t* s_rows = reinterpret_cast<int32_t*>(smem + L.rows);
    int64_t* s_wb = reinterpret_cast<int64_t*>(smem + L.wb);
    int32_t* s_wt = reinterpret_cast<int32_t*>(smem + L.wt);
    int32_t* s_we = reinterpret_cast<int32_t*>(smem + L.we);
    int32_t* s_wp = reinterpret_cast<int32_t*>(smem + L.wp);
    int32_t* s_hist = reinterpret_cast<int32_t*>(smem + L.hist);
    int64_t* s_red = reinterpret_cast<int64_t*>(smem + L.red);
    int32_t* s_cnt = reinterpret_cast<int32_t*>(smem + L.cnt);
    int32_t* s_misc = reinterpret_cast<int32_t*>(smem + L.misc);
    Key* s_scratch = reinterpret_cast<Key*>(smem + L.scratch);  // wide rounds only
    const int scratch_cap = (int)((L.total - L.scratch) / sizeof(Key));
    // sorted held sets (p.SW): counts [0, kMaxOwn) and buffer selectors
    // [kMaxOwn, 2 kMaxOwn) of the owned experts; the sets and the sort
    // scratch (two buffers of nsc keys) in the scratch area
    int32_t* s_swm = reinterpret_cast<int32_t*>(smem + L.swm);
    unsigned char* s_sw = smem + L.scratch;
    Key* s_swk = reinterpret_cast<Key*>(s_sw + sw_bytes(p.own_max, p.C));
    auto sw_set = [&](int j, int sel) {
        unsigned char* b = s_sw + (size_t)(2 * j + (sel & 1)) * sw_set_bytes(p.C);
        return SortedSet{reinterpret_cast<int64_t*>(b), reinterpret_cast<int32_t*>(b + 8 * (size_t)p.C)};
    };

    const int T = p.T, E = p.E, C = p.C, FK = p.FK;
    const int64_t scale = (int64_t)T + 1;
    const int lane = lane_id(), warp = warp_id();
    const int cta = blockIdx.x, ncta = gridDim.x;
    if (cta == p.absent_cta) return;  // test hook: the others' first grid barrier gives up

    Team<kThreads> cta_team{s_hist, s_red, s_cnt};
    Team<32> warp_team{s_hist + warp * kHist, nullptr, nullptr};

    int status = BASE_OK;
    unsigned bar_gen = 0;  // grid barriers passed (the same in every CTA)
    int64_t eps = 1;
    {
        // the score range for eps0: every CTA reduces a slice of q; the first
        // phase's grid barrier publishes the result.  enc(x) = x ^ 2^31 as
        // unsigned keeps the signed order, so two atomicMax on zeroed words
        // give the max and (through ~enc) the min
        unsigned mx = 0u, mn = 0u;
        const size_t n = (size_t)T * E;
        const bool vec = (reinterpret_cast<uintptr_t>(p.q) & 15) == 0;
        const size_t n4 = vec ? n / 4 : 0;
        const int4* q4 = reinterpret_cast<const int4*>(p.q);
        for (size_t i = (size_t)cta * kThreads + threadIdx.x; i < n4; i += (size_t)ncta * kThreads) {
            const int4 v = __ldg(q4 + i);
            const unsigned a = (unsigned)v.x ^ 0x80000000u, b = (unsigned)v.y ^ 0x80000000u;
            const unsigned c = (unsigned)v.z ^ 0x80000000u, d = (unsigned)v.w ^ 0x80000000u;
            mx = max(mx, max(max(a, b), max(c, d)));
            mn = max(mn, max(max(~a, ~b), max(~c, ~d)));
        }
        for (size_t i = n4 * 4 + (size_t)cta * kThreads + threadIdx.x; i < n;
             i += (size_t)ncta * kThreads) {
            const unsigned a = (unsigned)__ldg(p.q + i) ^ 0x80000000u;
            mx = max(mx, a);
            mn = max(mn, ~a);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            mn = max(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        }
        // one pair of atomics per CTA (thousands on two words serialise)
        unsigned* s_mm = reinterpret_cast<unsigned*>(s_hist);
        if (lane == 0) {
            s_mm[warp] = mx;
            s_mm[kWarps + warp] = mn;
        }
        __syncthreads();
        if (warp == 0) {
            mx = lane < kWarps ? s_mm[lane] : 0u;
            mn = lane < kWarps ? s_mm[kWarps + lane] : 0u;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                mn = max(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            }
            if (lane == 0) {
                atomicMax(&p.mmenc[0], mx);
                atomicMax(&p.mmenc[1], mn);
            }
        }
        __syncthreads();
    }
    bool first_phase = true;

    // lanes per bidding token: the smallest power of two >= E, at most 32
    int G = 1;
    while (G < E && G < kWarp) G <<= 1;
    const int tpw = kWarp / G;
    const int sub = lane / G, gl = lane % G;

    long long rounds = 0, phases = 0, bids = 0;
    bool ok = true;
    bool reset_done = false;
    int cur = 0;  // which global list holds the bidders

    while (status == BASE_OK && ok) {
        // ---- phase start: nothing held, prices kept (in p.gprice); after a
        // narrow phase CTA 0 has done this already, before the grid barrier
        if (!reset_done) {
            for (int e = cta * kThreads + threadIdx.x; e < E; e += ncta * kThreads) {
                p.hcnt[e] = 0;
                p.bcnt[e] = 0;
                p.gfs[e] = 0;  // empty held set: an empty, complete fringe
            }
            if (cta == 0 && threadIdx.x < 3) p.ctrl->ucount[threadIdx.x] = 0;
            if (!(ok = grid_sync(p, bar_gen, s_misc))) break;
        }
        if (first_phase) {
            // eps0 = (max q - min q)(T+1) / 50, from the range every CTA has reduced
            first_phase = false;
            const int64_t qmax = (int32_t)(vload(&p.mmenc[0]) ^ 0x80000000u);
            const int64_t qmin = (int32_t)((~vload(&p.mmenc[1])) ^ 0x80000000u);
            const int64_t range = qmax - qmin;
            if (range > 0 && range > ((int64_t)1 << 58) / scale) {
                status = BASE_ERR_INVALID_ARG;
                break;
            }
            eps = range * scale / kEpsDivisor;
            if (eps < 1) eps = 1;
        }
        ++phases;
        reset_done = false;
        // owned sorted held sets start empty in buffer 0 (read after the wide
        // round's first barrier)
        if (p.SW && threadIdx.x < 2 * kMaxOwn) s_swm[threadIdx.x] = 0;
        int U = T;
        bool first = true;
        bool narrow = false;
        while (U > 0 && !narrow) {
            // ================= wide round =================
            if (rounds >= p.max_rounds) {
                status = BASE_ERR_NOT_CONVERGED;
                break;
            }
            if (cta == 0 && threadIdx.x == 0) trace_round(p, rounds, U);
            ++rounds;
            bids += U;
            const int32_t* ulist = cur ? p.ulist1 : p.ulist0;
            int32_t* unext = cur ? p.ulist0 : p.ulist1;
            int32_t* ucnt = &p.ctrl->ucount[(int)(rounds % 3)];
            for (int e = threadIdx.x; e < E; e += kThreads) s_price[e] = vload(p.gprice + e);
            __syncthreads();
            {
                // The CTA takes chunks of up to kWideChunk bidders; each bid is
                // staged in shared memory with its rank among the chunk's bids
                // to the same expert, then one global atomic per (chunk,
                // expert) reserves bucket space and the bids are written out.
                constexpr int NT = 4;
                const int per_cta = (U + ncta - 1) / ncta;
                const int CH = min(kWideChunk, max(32, per_cta));
                const int groups = kWarps * tpw;  // lane groups in the CTA
                for (long long c0 = (long long)cta * CH; c0 < U; c0 += (long long)ncta * CH) {
                    const int cn = (int)min((long long)CH, (long long)U - c0);
                    for (int e = threadIdx.x; e < E; e += kThreads) s_ncnt[e] = 0;
                    __syncthreads();
                    // warp-uniform trip count: the lane groups of a warp shuffle
                    // together, so the loop runs on the warp's first group index
                    for (int jw = warp * tpw; jw < cn; jw += groups * NT) {
                        const int j0 = jw + sub;
                        int t[NT];
                        bool valid[NT];
#pragma unroll
                        for (int u = 0; u < NT; ++u) {
                            const int j = j0 + u * groups;
                            valid[u] = j < cn;
                            const long long i = c0 + j;
                            t[u] = valid[u] ? (first ? (int)i : vload(ulist + i)) : 0;
                        }
                        int64_t v1[NT], v2[NT];
                        int e1[NT];
                        group_bid_multi<NT>(p.q, t, valid, s_price, E, G, gl, scale, v1, v2, e1);
                        if (gl == 0) {
#pragma unroll
                            for (int u = 0; u < NT; ++u) {
                                if (!valid[u]) continue;
                                const int j = j0 + u * groups;
                                s_wb[j] = v1[u] + s_price[e1[u]] - v2[u] + eps;
                                s_wt[j] = t[u];
                                s_we[j] = e1[u];
                                s_wp[j] = atomicAdd(&s_ncnt[e1[u]], 1);
                            }
                        }
                    }
                    __syncthreads();
                    for (int e = threadIdx.x; e < E; e += kThreads) {
                        const int c = s_ncnt[e];
                        if (c) s_act0[e] = atomicAdd(&p.bcnt[e], c);
                    }
                    __syncthreads();
                    for (int j = threadIdx.x; j < cn; j += kThreads) {
                        const int e = s_we[j];
                        const size_t at = (size_t)e * T + s_act0[e] + s_wp[j];
                        p.bb[at] = s_wb[j];
                        p.bt[at] = s_wt[j];
                    }
                    __syncthreads();
                }
            }
            if (!(ok = grid_sync(p, bar_gen, s_misc))) break;
            if (p.SW) {
                // every owned expert with new bids: a merge with its sorted held set
                int j = 0;
                for (int e = cta; e < E; e += ncta, ++j) {
                    const int n = vload(p.bcnt + e);
                    if (n == 0) continue;
                    __syncthreads();
                    const int sel = s_swm[kMaxOwn + j];
                    const int h0 = s_swm[j];
                    int64_t price = INT64_MIN;
                    const int nh = resolve_sorted(
                        cta_team, p, sw_set(j, sel), h0, sw_set(j, sel ^ 1), p.bb + (size_t)e * T,
                        p.bt + (size_t)e * T, n, s_swk, s_swk + p.nsc, p.nsc, p.hb + (size_t)e * C,
                        p.ht + (size_t)e * C, p.gfr + (size_t)e * FK, unext, ucnt, price);
                    if (threadIdx.x == 0) {
                        s_swm[j] = nh;
                        s_swm[kMaxOwn + j] = sel ^ 1;
                        p.hcnt[e] = nh;
                        p.bcnt[e] = 0;
                        p.gfs[e] = min(FK, nh);
                        if (nh == C) p.gprice[e] = price;
                    }
                    __syncthreads();
                }
            }
            for (int e = cta; e < E && !p.SW; e += ncta) {
                const int n = vload(p.bcnt + e);
                if (n == 0) continue;
                __syncthreads();
                const int h0 = vload(p.hcnt + e);
                int64_t* hb = p.hb + (size_t)e * C;
                int32_t* ht = p.ht + (size_t)e * C;
                Key* gfr = p.gfr + (size_t)e * FK;
                const int fs0 = vload(p.gfs + e);
                const bool warp_ok = n < 32 && (fs0 == h0 || max(0, h0 + n - C) < fs0);
                if (warp_ok) {
                    // a few bids: merge them with the expert's fringe (warp 0)
                    if (warp == 0) {
                        int fs = fs0, h = h0;
                        int64_t price = INT64_MIN;
                        resolve_warp(p, gfr, fs, h, p.bb + (size_t)e * T, p.bt + (size_t)e * T, n,
                                     hb, ht, unext, ucnt, price, RowStage{nullptr, 0});
                        if (h == C && fs == 0) {
                            fs = build_fringe<32>(warp_team, hb, ht, C, FK, T - 1, gfr);
                            price = gfr[0].bid;
                        }
                        if (lane == 0) {
                            p.gfs[e] = fs;
                            p.hcnt[e] = h;
                            p.bcnt[e] = 0;
                            if (h == C) p.gprice[e] = price;
                        }
                    }
                    __syncthreads();
                    continue;
                }
                Cands cd{hb, ht, p.bb + (size_t)e * T, p.bt + (size_t)e * T, h0, n};
                {
                    int nh = 0, fs = 0;
                    int64_t price = INT64_MIN;
                    if (resolve_cta_cached(cta_team, p, cd, s_scratch, scratch_cap, hb, ht, unext,
                                           ucnt, gfr, nh, fs, price)) {
                        if (threadIdx.x == 0) {
                            p.hcnt[e] = nh;
                            p.bcnt[e] = 0;
                            p.gfs[e] = fs;
                            if (nh == C) p.gprice[e] = price;
                        }
                        __syncthreads();
                        continue;
                    }
                }
                int64_t price = INT64_MIN;
                const int nh = resolve_general<kThreads>(cta_team, p, e, cd, hb, ht, unext, ucnt,
                                                     price, RowStage{nullptr, 0});
                const int fs = build_fringe<kThreads>(cta_team, hb, ht, nh, FK, T - 1, gfr);
                if (threadIdx.x == 0) {
                    p.hcnt[e] = nh;
                    p.bcnt[e] = 0;
                    p.gfs[e] = fs;
                    if (nh == C) p.gprice[e] = price;
                }
                __syncthreads();
            }
            // the counter the next round writes: last read two rounds ago
            if (cta == 0 && threadIdx.x == 0) p.ctrl->ucount[(int)((rounds + 1) % 3)] = 0;
            if (!(ok = grid_sync(p, bar_gen, s_misc))) break;
            U = *reinterpret_cast<volatile int*>(ucnt);
            cur ^= 1;
            first = false;
            if (U > 0 && U <= p.narrow_max) narrow = true;
        }
        if (!ok || status != BASE_OK) break;
        if (narrow) {
            // ================= narrow rounds on CTA 0 =================
            // Two block barriers per round.  A bid goes straight into its
            // expert's shared-memory bucket (the first NB; the rest to the
            // global bucket); after the barrier each warp resolves active
            // experts.  A rejected token's score row is copied into shared
            // memory (cp.async) for its bid in the next round.  Counters used
            // across a barrier are double / triple buffered by round parity.
            if (cta == 0) {
                const int32_t* ulist = cur ? p.ulist1 : p.ulist0;
                int32_t* s_nact = s_misc + 4;  // [2]
                int32_t* s_next = s_misc + 8;  // [3]
                const int NB = p.NB, RC = p.RC;
                const bool stage_rows = RC > 0 && (E % 4) == 0;
                int lc = 0;
                int r3_prev = (int)(rounds % 3);  // the counter of the round before
                bool staged = false;  // the current list's first RC rows are in s_rows[lc]
                for (int i = threadIdx.x; i < U; i += kThreads) s_list0[i] = vload(ulist + i);
                for (int e = threadIdx.x; e < E; e += kThreads) {
                    s_price[e] = vload(p.gprice + e);
                    s_hcnt[e] = vload(p.hcnt + e);
                    s_fsize[e] = vload(p.gfs + e);
                    s_ncnt[e] = 0;
                }
                for (int i = threadIdx.x; i < E * FK; i += kThreads) {
                    const Key* g = p.gfr + i;
                    s_fr[i] = Key{vload(&g->bid), vload(&g->tok), vload(&g->slot)};
                }
                // the held sets: in shared memory when they fit (written by
                // the wide rounds of other CTAs: read past L1)
                int64_t* hbase = p.hb;
                int32_t* htbase = p.ht;
                if (p.HS) {
                    hbase = reinterpret_cast<int64_t*>(smem + L.hb);
                    htbase = reinterpret_cast<int32_t*>(smem + L.ht);
                    // 16-byte pieces (all bases 16-byte aligned), then the tails
                    const int4* gb = reinterpret_cast<const int4*>(p.hb);
                    const int4* gt = reinterpret_cast<const int4*>(p.ht);
                    int4* sb = reinterpret_cast<int4*>(hbase);
                    int4* st = reinterpret_cast<int4*>(htbase);
#pragma unroll 4
                    for (int i = threadIdx.x; i < T / 2; i += kThreads) sb[i] = __ldcg(gb + i);
#pragma unroll 4
                    for (int i = threadIdx.x; i < T / 4; i += kThreads) st[i] = __ldcg(gt + i);
                    for (int i = (T / 2) * 2 + threadIdx.x; i < T; i += kThreads)
                        hbase[i] = __ldcg(p.hb + i);
                    for (int i = (T / 4) * 4 + threadIdx.x; i < T; i += kThreads)
                        htbase[i] = __ldcg(p.ht + i);
                }
                if (threadIdx.x < 5) s_misc[4 + (threadIdx.x < 2 ? threadIdx.x : threadIdx.x + 2)] = 0;
                __syncthreads();
                while (U > 0) {
                    if (U == 1 && E <= 128) {
                        // one bidder: warp 0 ends the phase alone
                        long long* s_ll = reinterpret_cast<long long*>(s_misc + 12);
                        if (warp == 0) {
                            if (U == 1 && status == BASE_OK) {
                                const int t0 = (lc ? s_list1 : s_list0)[0];
                                // scratch: the bid buckets are free between rounds
                                const ChainScratch cs{s_nbk_b, s_nbk_t, s_nbk_t + 1, s_misc + 2};
                                if (E <= 32)
                                    chain_rounds<1>(p, t0, eps, scale, s_price, s_fr, s_fsize,
                                                    s_hcnt, hbase, htbase, cs, warp_team, rounds,
                                                    bids, status);
                                else if (E <= 64)
                                    chain_rounds<2>(p, t0, eps, scale, s_price, s_fr, s_fsize,
                                                    s_hcnt, hbase, htbase, cs, warp_team, rounds,
                                                    bids, status);
                                else
                                    chain_rounds<4>(p, t0, eps, scale, s_price, s_fr, s_fsize,
                                                    s_hcnt, hbase, htbase, cs, warp_team, rounds,
                                                    bids, status);
                            }
                            if (lane == 0) {
                                s_ll[0] = rounds;
                                s_ll[1] = bids;
                                s_misc[1] = status;
                            }
                        }
                        __syncthreads();
                        rounds = s_ll[0];
                        bids = s_ll[1];
                        status = s_misc[1];
                        U = 0;
                        break;
                    }
                    if (rounds >= p.max_rounds) {
                        status = BASE_ERR_NOT_CONVERGED;
                        break;
                    }
                    if (threadIdx.x == 0) trace_round(p, rounds, U);
                    ++rounds;
                    bids += U;
                    const int ra = (int)(rounds & 1);
                    int32_t* list = lc ? s_list1 : s_list0;
                    int32_t* next = lc ? s_list0 : s_list1;
                    int32_t* act = ra ? s_act1 : s_act0;
                    // round r uses counter r % 3; r3 = rounds % 3 after the increment
                    const int r3 = r3_prev == 2 ? 0 : r3_prev + 1;
                    r3_prev = r3;
                    const int32_t* rows_cur = s_rows + (size_t)lc * RC * E;
                    int32_t* rows_next = s_rows + (size_t)(lc ^ 1) * RC * E;
                    // the counter the next round's resolve writes was last read
                    // two barriers ago
                    if (threadIdx.x == 0) s_next[r3 == 2 ? 0 : r3 + 1] = 0;
                    // ---- bid (two tokens per lane group and pass when there are as many)
                    auto place = [&](int t, int e, int64_t v1, int64_t v2) {
                        const int64_t b = v1 + s_price[e] - v2 + eps;
                        const int pos = atomicAdd(&s_ncnt[e], 1);
                        if (pos == 0) act[atomicAdd(&s_nact[ra], 1)] = e;
                        if (pos < NB) {
                            s_nbk_b[(size_t)e * NB + pos] = b;
                            s_nbk_t[(size_t)e * NB + pos] = t;
                        } else {
                            p.bb[(size_t)e * T + pos] = b;
                            p.bt[(size_t)e * T + pos] = t;
                        }
                    };
                    if (U > kWarps * tpw) {
                        for (int base = warp * tpw; base < U; base += kWarps * tpw * 2) {
                            const int i0 = base + sub, i1 = base + kWarps * tpw + sub;
                            const bool ok0 = i0 < U, ok1 = i1 < U;
                            const int t0 = ok0 ? list[i0] : 0, t1 = ok1 ? list[i1] : 0;
                            const int32_t* r0 = (staged & (i0 < RC)) ? rows_cur + (size_t)i0 * E
                                                                    : p.q + (size_t)t0 * E;
                            const int32_t* r1 = (staged & (i1 < RC)) ? rows_cur + (size_t)i1 * E
                                                                    : p.q + (size_t)t1 * E;
                            int64_t v1[2], v2[2];
                            int e1[2];
                            group_bid2(r0, r1, ok0, ok1, s_price, E, G, gl, scale, v1, v2, e1);
                            if (gl == 0) {
                                if (ok0) place(t0, e1[0], v1[0], v2[0]);
                                if (ok1) place(t1, e1[1], v1[1], v2[1]);
                            }
                        }
                    } else {
                        const int i = warp * tpw + sub;  // at most one token per lane group
                        if (warp * tpw < U) {
                            const bool valid = i < U;
                            const int t = valid ? list[i] : 0;
                            const int32_t* row = (staged & (i < RC)) ? rows_cur + (size_t)i * E
                                                                    : p.q + (size_t)t * E;
                            int64_t v1, v2;
                            int e1;
                            group_bid(row, s_price, valid ? E : 0, G, gl, scale, v1, v2, e1);
                            if (valid && gl == 0) place(t, e1, v1, v2);
                        }
                    }
                    __syncthreads();
                    // ---- resolve: a warp per active expert
                    const int nact = s_nact[ra];
                    int32_t* ncnt_next = &s_next[r3];
                    RowStage rs{stage_rows ? rows_next : nullptr, RC};
                    for (int a = warp; a < nact; a += kWarps) {
                        const int e = act[a];
                        const int n = s_ncnt[e];
                        const int h = s_hcnt[e];
                        int64_t* hb = hbase + (size_t)e * C;
                        int32_t* ht = htbase + (size_t)e * C;
                        Key* fr = s_fr + (size_t)e * FK;
                        const int64_t* nb = s_nbk_b + (size_t)e * NB;
                        const int32_t* nt = s_nbk_t + (size_t)e * NB;
                        if (n > NB) {
                            // spilled: move the shared part next to the rest
                            int64_t* gb = p.bb + (size_t)e * T;
                            int32_t* gt = p.bt + (size_t)e * T;
                            for (int j = lane; j < NB; j += 32) {
                                gb[j] = nb[j];
                                gt[j] = nt[j];
                            }
                            __syncwarp();
                            nb = gb;
                            nt = gt;
                        }
                        int64_t price = s_price[e];
                        bool done = false;
                        if (n == 1 && h == C && s_fsize[e] >= 2) {
                            int fs = s_fsize[e];
                            const int rej = fringe_take_one(fr, fs, h, nb[0], nt[0], hb, ht, price);
                            int at = 0;
                            if (lane == 0) {
                                at = atomicAdd(ncnt_next, 1);
                                next[at] = rej;
                                s_fsize[e] = fs;
                            }
                            at = __shfl_sync(0xffffffffu, at, 0);
                            rs.stage_warp(p.q, E, rej, at);
                            done = true;
                        }
                        if (!done && n < 32) {
                            int fs = s_fsize[e], hh = h;
                            if (fs != hh && max(0, hh + n - C) >= fs)  // depleted: rebuild
                                fs = build_fringe<32>(warp_team, hb, ht, hh, FK, T - 1, fr);
                            done = resolve_warp(p, fr, fs, hh, nb, nt, n, hb, ht, next, ncnt_next,
                                                price, rs);
                            if (done) {
                                if (hh == C && fs == 0) {
                                    fs = build_fringe<32>(warp_team, hb, ht, hh, FK, T - 1, fr);
                                    price = fr[0].bid;
                                }
                                if (lane == 0) {
                                    s_fsize[e] = fs;
                                    s_hcnt[e] = hh;
                                }
                            }
                        }
                        if (!done) {
                            Cands cd{hb, ht, nb, nt, h, n};
                            const int nh = resolve_general<32>(warp_team, p, e, cd, hb, ht, next,
                                                               ncnt_next, price, rs);
                            const int fs = build_fringe<32>(warp_team, hb, ht, nh, FK, T - 1, fr);
                            if (lane == 0) {
                                s_hcnt[e] = nh;
                                s_fsize[e] = fs;
                            }
                        }
                        __syncwarp();
                        if (lane == 0) {
                            if (s_hcnt[e] == C) s_price[e] = price;
                            s_ncnt[e] = 0;
                        }
                    }
                    // the row copies this warp issued land before the barrier
                    asm volatile("cp.async.wait_all;" ::: "memory");
                    // the other parity's active count: read in the previous round
                    if (threadIdx.x == 0) s_nact[ra ^ 1] = 0;
                    __syncthreads();
                    U = s_next[r3];
                    lc ^= 1;
                    staged = stage_rows;
                }
                // hand the prices back to the grid; when another phase follows,
                // reset its state now (the phase start then needs no barrier)
                const bool again = status == BASE_OK && eps != 1;
                if (p.HS && !again) {  // the last phase: the assignment is read from p.ht
                    const int4* st = reinterpret_cast<const int4*>(htbase);
                    int4* gt = reinterpret_cast<int4*>(p.ht);
                    for (int i = threadIdx.x; i < T / 4; i += kThreads) gt[i] = st[i];
                    for (int i = (T / 4) * 4 + threadIdx.x; i < T; i += kThreads) p.ht[i] = htbase[i];
                }
                for (int e = threadIdx.x; e < E; e += kThreads) {
                    p.gprice[e] = s_price[e];
                    p.hcnt[e] = again ? 0 : s_hcnt[e];
                    if (again) {
                        p.bcnt[e] = 0;
                        p.gfs[e] = 0;
                    }
                }
                if (again && threadIdx.x < 3) p.ctrl->ucount[threadIdx.x] = 0;
                if (threadIdx.x == 0) {
                    reinterpret_cast<volatile long long*>(p.obj)[1] = rounds;
                    reinterpret_cast<volatile long long*>(p.obj)[2] = bids;
                    reinterpret_cast<volatile int*>(p.obj)[6] = status;
                }
            }
            if (!(ok = grid_sync(p, bar_gen, s_misc))) break;
            // every CTA takes over CTA 0's counters (rewritten no earlier than
            // the next narrow phase, several grid barriers later)
            rounds = reinterpret_cast<volatile long long*>(p.obj)[1];
            bids = reinterpret_cast<volatile long long*>(p.obj)[2];
            status = reinterpret_cast<volatile int*>(p.obj)[6];
            reset_done = status == BASE_OK && eps != 1;
        }
        if (status != BASE_OK) break;
        if (eps == 1) break;
        eps /= kEpsFactor;
        if (eps < 1) eps = 1;
    }
    if (!ok) {
        if (cta == 0 && threadIdx.x == 0 && p.stats) p.stats->status = BASE_ERR_TIMEOUT;
        return;
    }

    // results: every CTA writes its experts' tokens
    unsigned long long part = 0;
    for (long long i = (long long)cta * kThreads + threadIdx.x; i < (long long)T;
         i += (long long)ncta * kThreads) {
        const int e = (int)(i / C);
        const int t = p.ht[i];
        if (status == BASE_OK) {
            p.assign[t] = e;
            part += (unsigned long long)(int64_t)p.q[(size_t)t * E + e];
        }
    }
    for (int e = cta * kThreads + threadIdx.x; e < E; e += ncta * kThreads)
        p.price_out[e] = p.gprice[e];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (lane == 0 && part) atomicAdd(p.obj, part);
    if (!grid_sync(p, bar_gen, s_misc)) {
        if (cta == 0 && threadIdx.x == 0 && p.stats) p.stats->status = BASE_ERR_TIMEOUT;
        return;
    }
    if (cta == 0 && threadIdx.x == 0 && p.stats) {
        p.stats->status = status;
        p.stats->phases = phases;
        p.stats->rounds = rounds;
        p.stats->final_eps = eps;
        p.stats->objective = (status == BASE_OK) ? (int64_t)*p.obj : 0;
        p.stats->bids = bids;
    }
}

// Shared-memory plan: the fringe capacity FK (<= 32), the per-expert bid
// bucket NB (<= 32) and the staged rows RC (<= 32) as large as 200 KB allows,
// the fringe first.
struct SmemPlan {
    int FK, NB, RC, HS;
    size_t bytes;
};

// ---------------------------------------------------------------- fig. 9
// The page's fig. 9 listing ("Solver"): experts bid for tokens and prices are
// per token, with the released code's rules where "Paper vs code" says the
// code differs (eps = range / 50, a won token kept in its holder's list at
// the largest score -- here that score plus one, strictly above every other
// value -- and after the iteration cap the listing's update without the
// holders' minimal bids, looping until every token has a bid).  Integer
// version on the quantised scores, the same steps as the CPU oracle's
// orc_fig9.  One cooperative grid; a round is
//   A: the CTA of expert e (e mod grid) finds e's (C+1)-th best adjusted
//      value X by a radix select over its T tokens (values in shared memory
//      when they fit) and bids raise = v - X + eps on its top C tokens (eps
//      for tokens it won last round while under the cap) with an atomic
//      max per token;
//   B: each token's largest bid is matched to the smallest expert that made
//      it (atomic min);
//   C: every token: won when its largest bid is > 0, price += that bid;
// with a grid barrier after each step.
struct Fig9Params {
    const int32_t* q;
    int32_t* qT;  // [E][T]: q by expert, written at the start (an expert's values coalesced)
    int T, E, C;
    long long max_iterations, max_rounds;
    int keys_in_smem;  // 1: an expert's T keys fit in shared memory
    int32_t* assign;
    int64_t* price_out;  // [T] final token prices
    int64_t* stats;      // [4] status, rounds, eps, objective (device)
    unsigned* mmenc;     // [2] score range (enc keeps the signed order)
    Ctrl* ctrl;          // abort flag; not-won counts by round mod 3
    unsigned* bar_flags;
    unsigned long long* bmax;  // [T] largest bid of the round
    int32_t* barg;             // [T] smallest expert with it
    int32_t* holder;           // [T] -1: not won
    int64_t* price;            // [T]
    int32_t* cnt;              // [E] tokens per expert at the end
    unsigned long long* obj;   // [1]
    unsigned long long wait_ns;
};

__global__ void __launch_bounds__(kThreads, 1) fig9_kernel(const __grid_constant__ Fig9Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    int32_t* s_hist = reinterpret_cast<int32_t*>(smem);               // kWarps * kHist
    int64_t* s_red = reinterpret_cast<int64_t*>(s_hist + kWarps * kHist);  // 32
    int32_t* s_cnt = reinterpret_cast<int32_t*>(s_red + 32);              // 64
    int32_t* s_misc = s_cnt + 64;                                         // 16
    int64_t* s_xb = reinterpret_cast<int64_t*>(s_misc + 16);              // 8: X of the owned experts
    int32_t* s_xt = reinterpret_cast<int32_t*>(s_xb + 8);                 // 8
    Key* s_keys = reinterpret_cast<Key*>(s_xt + 8);                       // T (keys_in_smem)
    const Team<kThreads> tm{s_hist, s_red, s_cnt};
    const int T = p.T, E = p.E, C = p.C;
    const int cta = blockIdx.x, ncta = gridDim.x, tid = threadIdx.x;
    unsigned bar_gen = 0;
    bool ok = true;
    // the score range, and the per-token state
    {
        unsigned mx = 0u, mn = 0u;
        for (long long i = (long long)cta * kThreads + tid; i < (long long)T * E;
             i += (long long)ncta * kThreads) {
            const unsigned a = (unsigned)__ldg(p.q + i) ^ 0x80000000u;
            mx = max(mx, a);
            mn = max(mn, ~a);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            mn = max(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        }
        if (lane_id() == 0) {
            atomicMax(&p.mmenc[0], mx);
            atomicMax(&p.mmenc[1], mn);
        }
        for (int t = cta * kThreads + tid; t < T; t += ncta * kThreads) {
            p.holder[t] = -1;
            p.price[t] = 0;
            p.bmax[t] = 0ull;
            p.barg[t] = INT32_MAX;
        }
        // q by expert: each warp transposes 32 x 32 tiles in registers (lane l
        // loads expert e0 + l of 32 tokens, then writes them as one 128-byte run)
        const long long tt = ((long long)T + 31) / 32;
        const int et = (E + 31) / 32;
        const int lane = lane_id();
        for (long long k = (long long)cta * kWarps + warp_id(); k < tt * et;
             k += (long long)ncta * kWarps) {
            const long long t0 = (k / et) * 32;
            const int e = (int)(k % et) * 32 + lane;
            int32_t v[32];
#pragma unroll
            for (int r = 0; r < 32; ++r)
                v[r] = (e < E && t0 + r < T) ? __ldg(p.q + (size_t)(t0 + r) * E + e) : 0;
            if (e < E) {
                int32_t* dst = p.qT + (size_t)e * T + t0;
                if (t0 + 32 <= T && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
                    for (int r = 0; r < 32; r += 4)
                        *reinterpret_cast<int4*>(dst + r) = make_int4(v[r], v[r + 1], v[r + 2], v[r + 3]);
                } else {
                    for (int r = 0; r < 32 && t0 + r < T; ++r) dst[r] = v[r];
                }
            }
        }
    }
    if (!(ok = grid_sync(p, bar_gen, s_misc))) return;
    const int64_t qmax = (int32_t)(vload(&p.mmenc[0]) ^ 0x80000000u);
    const int64_t qmin = (int32_t)((~vload(&p.mmenc[1])) ^ 0x80000000u);
    int64_t eps = (qmax - qmin) / 50;
    if (eps < 1) eps = 1;
    const int64_t RETAIN = qmax + 1;
    int status = BASE_OK;
    long long r = 0;
    int notwon = T;
    for (;; ++r) {
        if (r > 0 && notwon == 0) break;
        if (r >= p.max_rounds) {
            status = BASE_ERR_NOT_CONVERGED;
            break;
        }
        const bool retain_bids = r > 0 && r < p.max_iterations;  // holders bid eps
        const bool retain_top = r > 0 && r - 1 < p.max_iterations;  // won tokens at RETAIN
        // the counter round r + 1 fills: last read after round r - 2
        if (cta == 0 && tid == 0) p.ctrl->ucount[(int)((r + 1) % 3)] = 0;
        // ---- A: the experts' lists and bids
        for (int e = cta; e < E; e += ncta) {
            auto key_of = [&](int t) {  // holder / price come from other CTAs: read past L1
                const int h = __ldcg(p.holder + t);
                const int64_t qv = __ldcg(p.qT + (size_t)e * T + t);
                int64_t v;
                if (h == e && retain_top) v = RETAIN;
                else if (h == e) v = qv;
                else v = qv - (int64_t)__ldcg(reinterpret_cast<const long long*>(p.price) + t);
                return Key{v, t, 0};
            };
            if (p.keys_in_smem) {
                for (int t = tid; t < T; t += kThreads) s_keys[t] = key_of(t);
                __syncthreads();
            }
            auto visit = [&](auto fn) {
                if (p.keys_in_smem)
                    for (int t = tid; t < T; t += kThreads) fn(s_keys[t]);
                else
                    for (int t = tid; t < T; t += kThreads) fn(key_of(t));
            };
            // X: the (C+1)-th best = the (T-C)-th worst
            const Key X = kth_worst_cta(tm, visit, T - C, T - 1);
            for (int t = tid; t < T; t += kThreads) {
                const Key x = p.keys_in_smem ? s_keys[t] : key_of(t);
                if (!worse(X, x)) continue;  // not in the top C
                const int64_t bid =
                    (retain_bids && __ldcg(p.holder + t) == e) ? eps : x.bid - X.bid + eps;
                atomicMax(p.bmax + t, (unsigned long long)bid);
            }
            // keep X for step B (at most 8 owned experts: E <= 1024 < 8 grid)
            if (tid == 0) {
                s_xb[(e / ncta) & 7] = X.bid;
                s_xt[(e / ncta) & 7] = X.tok;
            }
            __syncthreads();
        }
        if (!(ok = grid_sync(p, bar_gen, s_misc))) break;
        // ---- B: the smallest expert with each token's largest bid
        for (int e = cta; e < E; e += ncta) {
            const Key X{s_xb[(e / ncta) & 7], s_xt[(e / ncta) & 7], 0};
            auto key_of = [&](int t) {  // holder / price come from other CTAs: read past L1
                const int h = __ldcg(p.holder + t);
                const int64_t qv = __ldcg(p.qT + (size_t)e * T + t);
                int64_t v;
                if (h == e && retain_top) v = RETAIN;
                else if (h == e) v = qv;
                else v = qv - (int64_t)__ldcg(reinterpret_cast<const long long*>(p.price) + t);
                return Key{v, t, 0};
            };
            for (int t = tid; t < T; t += kThreads) {
                const Key x = key_of(t);
                if (!worse(X, x)) continue;
                const int64_t bid =
                    (retain_bids && __ldcg(p.holder + t) == e) ? eps : x.bid - X.bid + eps;
                if ((unsigned long long)bid == __ldcg(p.bmax + t)) atomicMin(p.barg + t, e);
            }
        }
        if (!(ok = grid_sync(p, bar_gen, s_misc))) break;
        // ---- C: every token
        int nw = 0;
        for (int t = cta * kThreads + tid; t < T; t += ncta * kThreads) {
            const unsigned long long b = __ldcg(p.bmax + t);  // atomics of other CTAs
            if (b > 0ull) {
                p.holder[t] = __ldcg(p.barg + t);
            } else {
                p.holder[t] = -1;
                ++nw;
            }
            p.price[t] += (int64_t)b;
            p.bmax[t] = 0ull;
            p.barg[t] = INT32_MAX;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) nw += __shfl_xor_sync(0xffffffffu, nw, off);
        if (lane_id() == 0 && nw) atomicAdd(&p.ctrl->ucount[(int)(r % 3)], nw);
        if (!(ok = grid_sync(p, bar_gen, s_misc))) break;
        notwon = vload(&p.ctrl->ucount[(int)(r % 3)]);
    }
    if (!ok) {
        if (cta == 0 && tid == 0 && p.stats) p.stats[0] = BASE_ERR_TIMEOUT;
        return;
    }
    // the result: every token to its holder; balance checked
    unsigned long long part = 0;
    for (int t = cta * kThreads + tid; t < T; t += ncta * kThreads) {
        const int h = p.holder[t];
        p.price_out[t] = p.price[t];
        if (status == BASE_OK && h >= 0 && h < E) {
            p.assign[t] = h;
            atomicAdd(p.cnt + h, 1);
            part += (unsigned long long)(int64_t)__ldg(p.q + (size_t)t * E + h);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (lane_id() == 0 && part) atomicAdd(p.obj, part);
    if (!grid_sync(p, bar_gen, s_misc)) {
        if (cta == 0 && tid == 0 && p.stats) p.stats[0] = BASE_ERR_TIMEOUT;
        return;
    }
    if (cta == 0 && tid == 0) {
        if (status == BASE_OK)
            for (int e = 0; e < E; ++e)
                if (__ldcg(p.cnt + e) != C) status = BASE_ERR_NOT_CONVERGED;  // not a partition
        if (p.stats) {
            p.stats[0] = status;
            p.stats[1] = r;
            p.stats[2] = eps;
            p.stats[3] = status == BASE_OK ? (int64_t)__ldcg(p.obj) : 0;
        }
    }
}

constexpr size_t kSmemMax = 227 * 1024;  // dynamic shared memory of one CTA

static SmemPlan smem_plan(int E, int NM, int T) {
    constexpr size_t kBudget = 200 * 1024;
    SmemPlan pl{0, 0, 0, 0, 0};
    for (int fk = 32; fk >= 2; fk >>= 1) {
        if (smem_layout(E, fk, NM, 1, 0).total > kBudget) continue;
        int nb = 32;
        while (nb > 1 && smem_layout(E, fk, NM, nb, 0).total > kBudget) nb >>= 1;
        int rc = 32;
        while (rc > 0 && smem_layout(E, fk, NM, nb, rc).total > kBudget) rc >>= 1;
        pl = SmemPlan{fk, nb, rc, 0, smem_layout(E, fk, NM, nb, rc).total};
        // the held sets too, when they fit (small T)
        const size_t with_held = smem_layout(E, fk, NM, nb, rc, T, 1).total;
        if (with_held <= kBudget) {
            pl.HS = 1;
            pl.bytes = with_held;
        }
        return pl;
    }
    return pl;
}

}  // namespace auction

size_t fig9_workspace_bytes(int T, int E) {
    size_t b = align_up(2 * sizeof(unsigned), 256);
    b += align_up(sizeof(int32_t) * (size_t)T * E, 256);         // q by expert
    b += align_up(sizeof(auction::Ctrl), 256);
    b += align_up(sizeof(unsigned) * auction::kMaxGrid, 256);
    b += align_up(sizeof(unsigned long long) * (size_t)T, 256);  // bmax
    b += align_up(sizeof(int32_t) * (size_t)T, 256);             // barg
    b += align_up(sizeof(int32_t) * (size_t)T, 256);             // holder
    b += align_up(sizeof(int64_t) * (size_t)T, 256);             // price
    b += align_up(sizeof(int32_t) * (size_t)E, 256);             // counts
    b += align_up(64, 256);                                      // objective
    return b;
}

int launch_fig9(const int32_t* q, int T, int E, int32_t* assign, int64_t* price, int64_t* stats,
                long long max_iterations, long long max_rounds, void* ws, size_t ws_bytes,
                cudaStream_t stream) {
    using namespace auction;
    if (ws_bytes < fig9_workspace_bytes(T, E)) return BASE_ERR_WORKSPACE;
    unsigned char* w = static_cast<unsigned char*>(ws);
    size_t o = 0;
    auto take = [&](size_t bytes) { unsigned char* r = w + o; o += align_up(bytes, 256); return r; };
    Fig9Params prm{};
    prm.q = q;
    prm.T = T;
    prm.E = E;
    prm.C = T / E;
    prm.max_iterations = max_iterations;
    prm.max_rounds = max_rounds;
    prm.assign = assign;
    prm.price_out = price;
    prm.stats = stats;
    prm.wait_ns = g_test_hooks.wait_ns > 0 ? (unsigned long long)g_test_hooks.wait_ns : kWaitNs;
    unsigned char* zero0 = w;
    prm.mmenc = reinterpret_cast<unsigned*>(take(2 * sizeof(unsigned)));
    prm.ctrl = reinterpret_cast<Ctrl*>(take(sizeof(Ctrl)));
    prm.bar_flags = reinterpret_cast<unsigned*>(take(sizeof(unsigned) * kMaxGrid));
    const size_t zero_a = o;
    prm.bmax = reinterpret_cast<unsigned long long*>(take(sizeof(unsigned long long) * (size_t)T));
    prm.barg = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)T));
    prm.holder = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)T));
    prm.price = reinterpret_cast<int64_t*>(take(sizeof(int64_t) * (size_t)T));
    prm.qT = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)T * E));
    unsigned char* zero1 = w + o;
    prm.cnt = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)E));
    prm.obj = reinterpret_cast<unsigned long long*>(take(64));
    if (cudaMemsetAsync(zero0, 0, zero_a, stream) != cudaSuccess) return BASE_ERR_CUDA;
    if (cudaMemsetAsync(zero1, 0, (size_t)((w + o) - zero1), stream) != cudaSuccess)
        return BASE_ERR_CUDA;
    const size_t base_smem = sizeof(int32_t) * kWarps * kHist + 8 * 32 + 4 * 64 + 4 * 16 + 8 * 8 + 4 * 8;
    const size_t keys = sizeof(Key) * (size_t)T;
    prm.keys_in_smem = base_smem + keys <= kSmemMax ? 1 : 0;
    const size_t smem = base_smem + (prm.keys_in_smem ? keys : 0);
    if (cudaFuncSetAttribute(fig9_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return BASE_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fig9_kernel, kThreads, smem) !=
            cudaSuccess ||
        per_sm < 1)
        return BASE_ERR_UNSUPPORTED;
    const int grid = std::min(num_sms(), kMaxGrid);
    void* args[] = {&prm};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(fig9_kernel), dim3(grid),
                                    dim3(kThreads), args, smem, stream) != cudaSuccess)
        return BASE_ERR_CUDA;
    return BASE_OK;
}

size_t auction_workspace_bytes(int T, int E) {
    const int C = T / E;
    size_t b = align_up(2 * sizeof(unsigned), 256);         // score range
    b += align_up(sizeof(auction::Ctrl), 256);
    b += align_up(sizeof(unsigned) * auction::kMaxGrid, 256);  // grid-barrier flags
    b += align_up(64, 256);                                 // objective + counters
    b += align_up(sizeof(int64_t) * (size_t)E, 256);        // prices
    b += align_up(sizeof(int32_t) * (size_t)E, 256);        // held counts
    b += align_up(sizeof(int32_t) * (size_t)E, 256);        // bucket counts
    b += align_up(sizeof(int64_t) * (size_t)E * C, 256);    // held bids
    b += align_up(sizeof(int32_t) * (size_t)E * C, 256);    // held tokens
    b += align_up(sizeof(int64_t) * (size_t)E * T, 256);    // bucket bids
    b += align_up(sizeof(int32_t) * (size_t)E * T, 256);    // bucket tokens
    b += 2 * align_up(sizeof(int32_t) * (size_t)T, 256);    // lists
    b += align_up(sizeof(int32_t) * (size_t)E * C, 256);    // free slots
    b += align_up(sizeof(auction::Key) * (size_t)E * 32, 256);  // fringes
    b += align_up(sizeof(int32_t) * (size_t)E, 256);        // fringe sizes
    return b;
}

int launch_auction(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                   base_auction_stats* stats, void* ws, size_t ws_bytes, long long max_rounds,
                   int32_t* u_trace, int64_t* t_trace, long long trace_cap, cudaStream_t stream) {
    using namespace auction;
    if (ws_bytes < auction_workspace_bytes(T, E)) return BASE_ERR_WORKSPACE;
    const int C = T / E;
    const int NM = narrow_max_for(E);
    const SmemPlan sp = smem_plan(E, NM, T);
    if (sp.FK == 0) return BASE_ERR_UNSUPPORTED;
    const int FK = sp.FK;
    size_t smem = sp.bytes;

    unsigned char* w = static_cast<unsigned char*>(ws);
    size_t o = 0;
    auto take = [&](size_t bytes) { unsigned char* r = w + o; o += align_up(bytes, 256); return r; };
    Params prm{};
    prm.q = q;
    prm.T = T;
    prm.E = E;
    prm.C = C;
    prm.FK = FK;
    prm.NB = sp.NB;
    prm.RC = sp.RC;
    prm.HS = sp.HS;
    prm.max_rounds = max_rounds;
    prm.narrow_max = NM;
    prm.assign = assign;
    prm.price_out = price;
    prm.stats = stats;
    prm.u_trace = u_trace;
    prm.t_trace = t_trace;
    prm.trace_cap = (u_trace || t_trace) ? trace_cap : 0;
    prm.wait_ns = g_test_hooks.wait_ns > 0 ? (unsigned long long)g_test_hooks.wait_ns : kWaitNs;
    prm.absent_cta = g_test_hooks.auction_absent_cta;
    unsigned char* zero_begin = w + o;
    prm.mmenc = reinterpret_cast<unsigned*>(take(2 * sizeof(unsigned)));
    prm.ctrl = reinterpret_cast<Ctrl*>(take(sizeof(Ctrl)));
    prm.bar_flags = reinterpret_cast<unsigned*>(take(sizeof(unsigned) * kMaxGrid));
    prm.obj = reinterpret_cast<unsigned long long*>(take(64));
    prm.gprice = reinterpret_cast<int64_t*>(take(sizeof(int64_t) * (size_t)E));
    prm.hcnt = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)E));
    prm.bcnt = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)E));
    const size_t zero_bytes = (size_t)((w + o) - zero_begin);
    prm.hb = reinterpret_cast<int64_t*>(take(sizeof(int64_t) * (size_t)E * C));
    prm.ht = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)E * C));
    prm.bb = reinterpret_cast<int64_t*>(take(sizeof(int64_t) * (size_t)E * T));
    prm.bt = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)E * T));
    prm.ulist0 = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)T));
    prm.ulist1 = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)T));
    prm.gfree = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)E * C));
    prm.gfr = reinterpret_cast<Key*>(take(sizeof(Key) * (size_t)E * 32));
    prm.gfs = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)E));

    // control block, objective, prices (start at 0), counts
    if (cudaMemsetAsync(zero_begin, 0, zero_bytes, stream) != cudaSuccess) return BASE_ERR_CUDA;


    int dev = 0, nsm = 0, per_sm = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return BASE_ERR_CUDA;
    // The grid: one CTA per SM at most, and no more than the larger of E (an
    // owner for every expert) and the CTAs a phase start needs to bid all T
    // tokens in one pass (4 per lane group, 16 warps): fewer CTAs make every
    // grid barrier cheaper and leave fewer pollers during the narrow rounds.
    {
        int G = 1;
        while (G < E && G < 32) G <<= 1;
        const int per_pass = kWarps * (32 / G) * 4;
        const long long want = std::max<long long>(E, ((long long)T + per_pass - 1) / per_pass);
        if (want < nsm) nsm = (int)want;
    }
    // sorted held sets in the wide rounds when the owned experts' sets (two
    // buffers each) and the sort scratch (a power of two >= C keys, 2048 at
    // least when it fits) fit next to the narrow plan
    {
        const int own = (E + nsm - 1) / nsm;
        const size_t scratch_off = smem_layout(E, FK, NM, sp.NB, sp.RC, T, sp.HS).scratch;
        int nmin = 64;
        while (nmin < C) nmin <<= 1;
        prm.SW = 0;
        for (int nsc = std::max(nmin, kSortedSmall); nsc >= nmin && own <= kMaxOwn; nsc >>= 1) {
            const size_t need = scratch_off + sw_bytes(own, C) + 2 * sizeof(Key) * (size_t)nsc;
            if (need <= kSmemMax) {
                prm.SW = 1;
                prm.own_max = own;
                prm.nsc = nsc;
                smem = std::max(smem, need);
                break;
            }
        }
    }
    if (cudaFuncSetAttribute(auction_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return BASE_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, auction_kernel, kThreads, smem) !=
            cudaSuccess ||
        per_sm < 1)
        return BASE_ERR_UNSUPPORTED;
    const int grid = nsm;  // at most one CTA per SM (sized above), all co-resident
    if (grid > kMaxGrid) return BASE_ERR_UNSUPPORTED;
    void* args[] = {&prm};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(auction_kernel), dim3(grid),
                                    dim3(kThreads), args, smem, stream) != cudaSuccess)
        return BASE_ERR_CUDA;
    return BASE_OK;
}

}  // namespace base
