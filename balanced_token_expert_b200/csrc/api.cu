// api.cu -- the C ABI of libbase (declared in include/base.h): host-side
// argument checks, workspace carving and the order of the launches.
#include <cstdint>
#include <cstring>

#include "common.cuh"

namespace base {

int launch_scores_f32(const float* h, const float* w, int T, int D, int E, float* s, int32_t* q,
                      cudaStream_t stream);
int launch_scores_bf16(const void* h, const void* w, int T, int D, int E, float* s, int32_t* q,
                       cudaStream_t stream, int32_t* assign = nullptr, int32_t* counts = nullptr);
int launch_greedy(const int32_t* q, int T, int E, int32_t* assign, int32_t* counts,
                  cudaStream_t stream);
size_t auction_workspace_bytes(int T, int E);
int launch_auction(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                   base_auction_stats* stats, void* ws, size_t ws_bytes, long long max_rounds,
                   int32_t* u_trace, int64_t* t_trace, long long trace_cap, cudaStream_t stream);
size_t probe_workspace_bytes();
int launch_latency_probe(double* out, void* ws, cudaStream_t stream);
size_t fig9_workspace_bytes(int T, int E);
int launch_fig9(const int32_t* q, int T, int E, int32_t* assign, int64_t* price, int64_t* stats,
                long long max_iterations, long long max_rounds, void* ws, size_t ws_bytes,
                cudaStream_t stream);
size_t permute_workspace_bytes(int T, int E);
int launch_ep_dispatch(const void* const* h, const int32_t* const* perm, const float* const* gate,
                       void* const* recv, float* const* recv_gate, int g0, int ns, int G, int T,
                       int D, int E, cudaStream_t stream);
int launch_ep_combine(const void* const* y, const int32_t* const* perm, void* const* out, int r0,
                      int nr, int G, int T, int D, int E, cudaStream_t stream);
int launch_sort_by_expert(const int32_t* assign, int T, int E, int32_t* perm, int32_t* inv,
                          int32_t* offsets, const float* s, float* gate, void* ws,
                          cudaStream_t stream);
int launch_move_rows(const void* src, const int32_t* idx, int T, int D, void* dst, bool scatter,
                     cudaStream_t stream);
size_t ffn_workspace_bytes(int E);
int launch_expert_ffn(const void* x_perm, const int32_t* offsets, int T, int D, int F, int E,
                      const void* W1, const void* W2, int act, const float* gate, void* y_perm,
                      void* h1, void* a1, void* f, void* ws, cudaStream_t stream);
size_t backward_workspace_bytes(int T, int E, int D, int F);
size_t stack_workspace_bytes(int T, int E, int D);
size_t sanitize_workspace_bytes();
int launch_sanitize_scores(float* s, int32_t* q, int T, int E, void* ws, cudaStream_t stream);
int launch_expert_stack(const void* x_perm, const int32_t* offsets, int T, int D, int F, int E,
                        int S, const void* W1, const void* W2, const float* gamma,
                        const float* beta, int act, const float* gate, void* y_perm, void* h1,
                        void* ws, cudaStream_t stream);
int launch_layer_bwd(const void* h, const void* w, const void* W1, const void* W2, int act, int T,
                     int D, int E, int F, const base_layer_saved* sv, const void* dout, void* dh,
                     float* dw, float* dW1, float* dW2, void* ws, size_t ws_bytes,
                     cudaStream_t stream);

static bool aligned(const void* p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

static bool shapes_ok(int T, int E) { return T >= 1 && E >= 2 && E <= 1024; }

}  // namespace base

using namespace base;

extern "C" {

const char* base_status_string(int status) {
    switch (status) {
        case BASE_OK: return "ok";
        case BASE_ERR_INVALID_ARG: return "invalid argument";
        case BASE_ERR_CUDA: return "CUDA error";
        case BASE_ERR_NOT_CONVERGED: return "auction did not converge within the round cap";
        case BASE_ERR_TIMEOUT: return "a bounded device-side wait gave up";
        case BASE_ERR_WORKSPACE: return "workspace too small";
        case BASE_ERR_UNSUPPORTED: return "shape not supported by the kernels";
        default: return "unknown status";
    }
}

const char* base_version(void) { return "libbase 0.1 (sm_100a)"; }

size_t base_workspace_size(int T, int E, int D, int F) {
    if (!shapes_ok(T, E) || D < 0 || F < 0) return 0;
    size_t w = auction_workspace_bytes(T, E);
    if (sanitize_workspace_bytes() > w) w = sanitize_workspace_bytes();
    const size_t p = permute_workspace_bytes(T, E);
    if (p > w) w = p;
    const size_t f = ffn_workspace_bytes(E);
    if (f > w) w = f;
    if (F > 0 && D > 0) {
        const size_t b = backward_workspace_bytes(T, E, D, F);
        if (b > w) w = b;
    }
    return w;
}

/* Reads (and optionally clears) the sticky device error word.  Synchronous. */
int base_device_error(int64_t* code, int clear) {
    int64_t v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return BASE_ERR_CUDA;
    if (code) *code = v;
    if (clear) {
        const int64_t z = 0;
        if (cudaMemcpyToSymbol(g_device_error, &z, sizeof(z)) != cudaSuccess) return BASE_ERR_CUDA;
    }
    return BASE_OK;
}

int base_test_inject(int hook, long long value) {
    switch (hook) {
        case BASE_TEST_WAIT_LIMIT_NS:
            if (value < 0) return BASE_ERR_INVALID_ARG;
            g_test_hooks.wait_ns = value;
            return BASE_OK;
        case BASE_TEST_AUCTION_ABSENT_CTA:
            if (value < -1 || value > 1 << 20) return BASE_ERR_INVALID_ARG;
            g_test_hooks.auction_absent_cta = (int)value;
            return BASE_OK;
        case BASE_TEST_GEMM_DROP_FIRST_LOAD:
            if (value != 0 && value != 1) return BASE_ERR_INVALID_ARG;
            g_test_hooks.gemm_drop_first_load = (int)value;
            return BASE_OK;
        default:
            return BASE_ERR_INVALID_ARG;
    }
}

int base_scores(const void* h, const void* w, int dtype, int T, int D, int E, float* s,
                int32_t* q, cudaStream_t stream) {
    if (!h || !w || (!s && !q) || !shapes_ok(T, E) || D < 1) return BASE_ERR_INVALID_ARG;
    if ((s && !aligned(s, 16)) || (q && !aligned(q, 16))) return BASE_ERR_INVALID_ARG;
    if (dtype == BASE_F32) {
        if (!aligned(h, 4) || !aligned(w, 4)) return BASE_ERR_INVALID_ARG;
        return launch_scores_f32(static_cast<const float*>(h), static_cast<const float*>(w), T, D,
                                 E, s, q, stream);
    }
    if (dtype != BASE_BF16) return BASE_ERR_INVALID_ARG;
    if (D % 8 != 0 || !aligned(h, 16) || !aligned(w, 16)) return BASE_ERR_INVALID_ARG;
    return launch_scores_bf16(h, w, T, D, E, s, q, stream);
}

int base_scores_greedy(const void* h, const void* w, int dtype, int T, int D, int E, float* s,
                       int32_t* q, int32_t* assign, int32_t* counts, cudaStream_t stream) {
    if (!h || !w || !q || !assign || !shapes_ok(T, E) || D < 1) return BASE_ERR_INVALID_ARG;
    if ((s && !aligned(s, 16)) || !aligned(q, 16) || !aligned(assign, 4) ||
        (counts && !aligned(counts, 4)))
        return BASE_ERR_INVALID_ARG;
    if (dtype == BASE_BF16 && E <= 256) {
        if (D % 8 != 0 || !aligned(h, 16) || !aligned(w, 16)) return BASE_ERR_INVALID_ARG;
        if (counts && cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)E, stream) != cudaSuccess)
            return BASE_ERR_CUDA;
        return launch_scores_bf16(h, w, T, D, E, s, q, stream, assign, counts);
    }
    const int st = base_scores(h, w, dtype, T, D, E, s, q, stream);
    if (st != BASE_OK) return st;
    return base_assign_greedy(q, T, E, assign, counts, stream);
}

int base_sanitize_scores(float* s, int32_t* q, int T, int E, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
    if (!s || !ws || !shapes_ok(T, E)) return BASE_ERR_INVALID_ARG;
    if (!aligned(s, 4) || (q && !aligned(q, 4)) || !aligned(ws, 256)) return BASE_ERR_INVALID_ARG;
    if (ws_bytes < sanitize_workspace_bytes()) return BASE_ERR_WORKSPACE;
    return launch_sanitize_scores(s, q, T, E, ws, stream);
}

int base_assign_greedy(const int32_t* q, int T, int E, int32_t* assign, int32_t* counts,
                       cudaStream_t stream) {
    if (!q || !assign || !shapes_ok(T, E)) return BASE_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(assign, 4) || (counts && !aligned(counts, 4)))
        return BASE_ERR_INVALID_ARG;
    return launch_greedy(q, T, E, assign, counts, stream);
}

int base_assign_balanced(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                         base_auction_stats* stats, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
    if (!q || !assign || !price || !ws || !shapes_ok(T, E) || T % E != 0)
        return BASE_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(assign, 4) || !aligned(price, 8) || !aligned(ws, 256) ||
        (stats && !aligned(stats, 8)))
        return BASE_ERR_INVALID_ARG;
    if (ws_bytes < auction_workspace_bytes(T, E)) return BASE_ERR_WORKSPACE;
    return launch_auction(q, T, E, assign, price, stats, ws, ws_bytes, BASE_AUCTION_MAX_ROUNDS,
                          nullptr, nullptr, 0, stream);
}

int base_assign_balanced_ex(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                            base_auction_stats* stats, long long max_rounds, int32_t* u_trace,
                            int64_t* t_trace, long long trace_cap, void* ws, size_t ws_bytes,
                            cudaStream_t stream) {
    if (max_rounds < 1 || max_rounds > BASE_AUCTION_MAX_ROUNDS || trace_cap < 0)
        return BASE_ERR_INVALID_ARG;
    if ((u_trace || t_trace) && trace_cap == 0) return BASE_ERR_INVALID_ARG;
    if (!q || !assign || !price || !ws || !shapes_ok(T, E) || T % E != 0)
        return BASE_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(assign, 4) || !aligned(price, 8) || !aligned(ws, 256) ||
        (stats && !aligned(stats, 8)) || (u_trace && !aligned(u_trace, 4)) ||
        (t_trace && !aligned(t_trace, 8)))
        return BASE_ERR_INVALID_ARG;
    if (ws_bytes < auction_workspace_bytes(T, E)) return BASE_ERR_WORKSPACE;
    return launch_auction(q, T, E, assign, price, stats, ws, ws_bytes, max_rounds, u_trace, t_trace,
                          trace_cap, stream);
}

size_t base_probe_workspace_size(void) { return probe_workspace_bytes(); }

int base_measure_latency(double* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!out || !ws || !aligned(out, 8) || !aligned(ws, 256)) return BASE_ERR_INVALID_ARG;
    if (ws_bytes < probe_workspace_bytes()) return BASE_ERR_WORKSPACE;
    return launch_latency_probe(out, ws, stream);
}

size_t base_workspace_size_fig9(int T, int E) {
    if (!shapes_ok(T, E)) return 0;
    return fig9_workspace_bytes(T, E);
}

int base_assign_fig9(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                     int64_t* stats, long long max_iterations, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
    if (!q || !assign || !price || !ws || !shapes_ok(T, E) || T % E != 0 || max_iterations < 0)
        return BASE_ERR_INVALID_ARG;
    if (!aligned(q, 4) || !aligned(assign, 4) || !aligned(price, 8) || !aligned(ws, 256) ||
        (stats && !aligned(stats, 8)))
        return BASE_ERR_INVALID_ARG;
    if (ws_bytes < fig9_workspace_bytes(T, E)) return BASE_ERR_WORKSPACE;
    return launch_fig9(q, T, E, assign, price, stats, max_iterations, BASE_AUCTION_MAX_ROUNDS, ws,
                       ws_bytes, stream);
}

int base_permute(const void* h, const int32_t* assign, int T, int D, int E, int32_t* perm,
                 int32_t* inv, int32_t* offsets, void* x_perm, const float* s, float* gate,
                 void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!assign || !perm || !inv || !offsets || !ws || !shapes_ok(T, E)) return BASE_ERR_INVALID_ARG;
    if ((h == nullptr) != (x_perm == nullptr)) return BASE_ERR_INVALID_ARG;
    if ((s == nullptr) != (gate == nullptr)) return BASE_ERR_INVALID_ARG;
    if (h && (D < 8 || D % 8 != 0 || !aligned(h, 16) || !aligned(x_perm, 16)))
        return BASE_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return BASE_ERR_INVALID_ARG;
    if (ws_bytes < permute_workspace_bytes(T, E)) return BASE_ERR_WORKSPACE;
    int st = launch_sort_by_expert(assign, T, E, perm, inv, offsets, s, gate, ws, stream);
    if (st != BASE_OK || !h) return st;
    return launch_move_rows(h, perm, T, D, x_perm, false, stream);
}

int base_expert_ffn(const void* x_perm, const int32_t* offsets, int T, int D, int F, int E,
                    const void* W1, const void* W2, int act, const float* gate, void* y_perm,
                    void* h1, void* a1, void* f, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!x_perm || !offsets || !W1 || !W2 || !gate || !y_perm || !h1 || !ws || !shapes_ok(T, E))
        return BASE_ERR_INVALID_ARG;
    if (D < 8 || D % 8 != 0 || F < 8 || F % 8 != 0) return BASE_ERR_INVALID_ARG;
    if (act != BASE_RELU && act != BASE_GELU) return BASE_ERR_INVALID_ARG;
    const void* p16[] = {x_perm, W1, W2, y_perm, h1};
    for (const void* p : p16)
        if (!aligned(p, 16)) return BASE_ERR_INVALID_ARG;
    if ((a1 && !aligned(a1, 16)) || (f && !aligned(f, 16)) || !aligned(ws, 256))
        return BASE_ERR_INVALID_ARG;
    if (ws_bytes < ffn_workspace_bytes(E)) return BASE_ERR_WORKSPACE;
    return launch_expert_ffn(x_perm, offsets, T, D, F, E, W1, W2, act, gate, y_perm, h1, a1, f, ws,
                             stream);
}

int base_combine(const void* y_perm, const int32_t* perm, int T, int D, void* out,
                 cudaStream_t stream) {
    if (!y_perm || !perm || !out || T < 1 || D < 8 || D % 8 != 0) return BASE_ERR_INVALID_ARG;
    if (!aligned(y_perm, 16) || !aligned(out, 16)) return BASE_ERR_INVALID_ARG;
    return launch_move_rows(y_perm, perm, T, D, out, true, stream);
}

// shapes of an expert-parallel exchange: G workers (at most 8), E/G experts
// each, C = T/E tokens per expert per worker, rows of D bf16 (16-byte pieces)
static bool ep_shapes_ok(int G, int T, int D, int E) {
    return G >= 1 && G <= 8 && shapes_ok(T, E) && E % G == 0 && T % E == 0 && D >= 8 &&
           D % 8 == 0;
}

int base_ep_dispatch(const void* const* h, const int32_t* const* perm, const float* const* gate,
                     void* const* recv, float* const* recv_gate, int g0, int ns, int G, int T,
                     int D, int E, cudaStream_t stream) {
    if (!h || !perm || !recv || !ep_shapes_ok(G, T, D, E) || g0 < 0 || ns < 1 || g0 + ns > G)
        return BASE_ERR_INVALID_ARG;
    if ((gate == nullptr) != (recv_gate == nullptr)) return BASE_ERR_INVALID_ARG;
    for (int i = 0; i < ns; ++i)
        if (!h[i] || !aligned(h[i], 16) || !perm[i] || !aligned(perm[i], 4) ||
            (gate && (!gate[i] || !aligned(gate[i], 4))))
            return BASE_ERR_INVALID_ARG;
    for (int r = 0; r < G; ++r)
        if (!recv[r] || !aligned(recv[r], 16) || (recv_gate && (!recv_gate[r] || !aligned(recv_gate[r], 4))))
            return BASE_ERR_INVALID_ARG;
    return launch_ep_dispatch(h, perm, gate, recv, recv_gate, g0, ns, G, T, D, E, stream);
}

int base_ep_combine(const void* const* y, const int32_t* const* perm, void* const* out, int r0,
                    int nr, int G, int T, int D, int E, cudaStream_t stream) {
    if (!y || !perm || !out || !ep_shapes_ok(G, T, D, E) || r0 < 0 || nr < 1 || r0 + nr > G)
        return BASE_ERR_INVALID_ARG;
    for (int i = 0; i < nr; ++i)
        if (!y[i] || !aligned(y[i], 16)) return BASE_ERR_INVALID_ARG;
    for (int g = 0; g < G; ++g)
        if (!perm[g] || !aligned(perm[g], 4) || !out[g] || !aligned(out[g], 16))
            return BASE_ERR_INVALID_ARG;
    return launch_ep_combine(y, perm, out, r0, nr, G, T, D, E, stream);
}

int base_layer_fwd(const void* h, const void* w, const void* W1, const void* W2, int act,
                   int routing, int T, int D, int E, int F, void* out, const base_layer_saved* sv,
                   void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!h || !w || !W1 || !W2 || !out || !sv || !ws || !shapes_ok(T, E))
        return BASE_ERR_INVALID_ARG;
    if (!sv->s || !sv->q || !sv->assign || !sv->perm || !sv->inv || !sv->offsets || !sv->gate ||
        !sv->x_perm || !sv->h1 || !sv->y_perm)
        return BASE_ERR_INVALID_ARG;
    const bool sanitize = (routing & BASE_ROUTE_SANITIZE) != 0;
    routing &= ~BASE_ROUTE_SANITIZE;
    if (routing == BASE_ROUTE_BALANCED) {
        if (!sv->price || T % E != 0) return BASE_ERR_INVALID_ARG;
    } else if (routing != BASE_ROUTE_GREEDY) {
        return BASE_ERR_INVALID_ARG;
    }
    if (ws_bytes < base_workspace_size(T, E, D, 0)) return BASE_ERR_WORKSPACE;
    int st;
    if (routing == BASE_ROUTE_GREEDY && !sanitize) {
        // test-time routing: the argmax comes out of the score GEMM's epilogue
        st = base_scores_greedy(h, w, BASE_BF16, T, D, E, sv->s, sv->q, sv->assign, nullptr,
                                stream);
        if (st != BASE_OK) return st;
    } else {
        st = base_scores(h, w, BASE_BF16, T, D, E, sv->s, sv->q, stream);
        if (st != BASE_OK) return st;
        if (sanitize) {
            st = base_sanitize_scores(sv->s, sv->q, T, E, ws, ws_bytes, stream);
            if (st != BASE_OK) return st;
        }
        if (routing == BASE_ROUTE_BALANCED)
            st = base_assign_balanced(sv->q, T, E, sv->assign, sv->price, sv->stats, ws, ws_bytes,
                                      stream);
        else
            st = base_assign_greedy(sv->q, T, E, sv->assign, nullptr, stream);
        if (st != BASE_OK) return st;
    }
    st = base_permute(h, sv->assign, T, D, E, sv->perm, sv->inv, sv->offsets, sv->x_perm, sv->s,
                      sv->gate, ws, ws_bytes, stream);
    if (st != BASE_OK) return st;
    st = base_expert_ffn(sv->x_perm, sv->offsets, T, D, F, E, W1, W2, act, sv->gate, sv->y_perm,
                         sv->h1, sv->a1, sv->f, ws, ws_bytes, stream);
    if (st != BASE_OK) return st;
    return base_combine(sv->y_perm, sv->perm, T, D, out, stream);
}

size_t base_workspace_size_blend(int T, int E, int D, int F) {
    if (!shapes_ok(T, E) || D < 8 || F < 8) return 0;
    const size_t w = base_workspace_size(T, E, D, 0);
    const size_t st = stack_workspace_bytes(T, E, D);
    return w > st ? w : st;
}

int base_expert_stack(const void* x_perm, const int32_t* offsets, int T, int D, int F, int E,
                      int S, const void* W1, const void* W2, const float* gamma, const float* beta,
                      int act, const float* gate, void* y_perm, void* h1, void* ws,
                      size_t ws_bytes, cudaStream_t stream) {
    if (!x_perm || !offsets || !W1 || !W2 || !gamma || !beta || !gate || !y_perm || !h1 || !ws ||
        !shapes_ok(T, E))
        return BASE_ERR_INVALID_ARG;
    if (S < 1 || D < 8 || D % 8 != 0 || F < 8 || F % 8 != 0) return BASE_ERR_INVALID_ARG;
    if (act != BASE_RELU && act != BASE_GELU) return BASE_ERR_INVALID_ARG;
    const void* p16[] = {x_perm, W1, W2, gamma, beta, y_perm, h1};
    for (const void* p : p16)
        if (!aligned(p, 16)) return BASE_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return BASE_ERR_INVALID_ARG;
    if (ws_bytes < stack_workspace_bytes(T, E, D)) return BASE_ERR_WORKSPACE;
    return launch_expert_stack(x_perm, offsets, T, D, F, E, S, W1, W2, gamma, beta, act, gate,
                               y_perm, h1, ws, stream);
}

int base_layer_fwd_blend(const void* h, const void* w, const void* W1, const void* W2,
                         const float* gamma, const float* beta, int S, int act, int routing,
                         int T, int D, int E, int F, void* out, const base_layer_saved* sv,
                         void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!h || !w || !W1 || !W2 || !gamma || !beta || !out || !sv || !ws || !shapes_ok(T, E))
        return BASE_ERR_INVALID_ARG;
    if (S < 1 || D < 8 || D % 8 != 0 || F < 8 || F % 8 != 0) return BASE_ERR_INVALID_ARG;
    if (act != BASE_RELU && act != BASE_GELU) return BASE_ERR_INVALID_ARG;
    if (!sv->s || !sv->q || !sv->assign || !sv->perm || !sv->inv || !sv->offsets || !sv->gate ||
        !sv->x_perm || !sv->h1 || !sv->y_perm)
        return BASE_ERR_INVALID_ARG;
    const bool sanitize = (routing & BASE_ROUTE_SANITIZE) != 0;
    routing &= ~BASE_ROUTE_SANITIZE;
    if (routing == BASE_ROUTE_BALANCED) {
        if (!sv->price || T % E != 0) return BASE_ERR_INVALID_ARG;
    } else if (routing != BASE_ROUTE_GREEDY) {
        return BASE_ERR_INVALID_ARG;
    }
    const void* p16[] = {h, w, W1, W2, gamma, beta, out, sv->x_perm, sv->h1, sv->y_perm};
    for (const void* p : p16)
        if (!aligned(p, 16)) return BASE_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return BASE_ERR_INVALID_ARG;
    if (ws_bytes < base_workspace_size_blend(T, E, D, F)) return BASE_ERR_WORKSPACE;
    int st;
    if (routing == BASE_ROUTE_GREEDY && !sanitize) {
        // test-time routing: the argmax comes out of the score GEMM's epilogue
        st = base_scores_greedy(h, w, BASE_BF16, T, D, E, sv->s, sv->q, sv->assign, nullptr,
                                stream);
        if (st != BASE_OK) return st;
    } else {
        st = base_scores(h, w, BASE_BF16, T, D, E, sv->s, sv->q, stream);
        if (st != BASE_OK) return st;
        if (sanitize) {
            st = base_sanitize_scores(sv->s, sv->q, T, E, ws, ws_bytes, stream);
            if (st != BASE_OK) return st;
        }
        if (routing == BASE_ROUTE_BALANCED)
            st = base_assign_balanced(sv->q, T, E, sv->assign, sv->price, sv->stats, ws, ws_bytes,
                                      stream);
        else
            st = base_assign_greedy(sv->q, T, E, sv->assign, nullptr, stream);
        if (st != BASE_OK) return st;
    }
    st = base_permute(h, sv->assign, T, D, E, sv->perm, sv->inv, sv->offsets, sv->x_perm, sv->s,
                      sv->gate, ws, ws_bytes, stream);
    if (st != BASE_OK) return st;
    st = base_expert_stack(sv->x_perm, sv->offsets, T, D, F, E, S, W1, W2, gamma, beta, act,
                           sv->gate, sv->y_perm, sv->h1, ws, ws_bytes, stream);
    if (st != BASE_OK) return st;
    return base_combine(sv->y_perm, sv->perm, T, D, out, stream);
}

int base_layer_bwd(const void* h, const void* w, const void* W1, const void* W2, int act, int T,
                   int D, int E, int F, const base_layer_saved* sv, const void* dout, void* dh,
                   float* dw, float* dW1, float* dW2, void* ws, size_t ws_bytes,
                   cudaStream_t stream) {
    if (!h || !w || !W1 || !W2 || !sv || !dout || !dh || !dw || !dW1 || !dW2 || !ws ||
        !shapes_ok(T, E))
        return BASE_ERR_INVALID_ARG;
    if (D < 8 || D % 8 != 0 || F < 8 || F % 8 != 0) return BASE_ERR_INVALID_ARG;
    if (act != BASE_RELU && act != BASE_GELU) return BASE_ERR_INVALID_ARG;
    if (!sv->perm || !sv->inv || !sv->offsets || !sv->gate || !sv->x_perm || !sv->a1 || !sv->h1 ||
        !sv->f || !sv->assign)
        return BASE_ERR_INVALID_ARG;
    const void* p16[] = {h, w, W1, W2, dout, dh, dw, dW1, dW2, sv->x_perm, sv->a1, sv->h1, sv->f};
    for (const void* p : p16)
        if (!aligned(p, 16)) return BASE_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return BASE_ERR_INVALID_ARG;
    if (ws_bytes < backward_workspace_bytes(T, E, D, F)) return BASE_ERR_WORKSPACE;
    return launch_layer_bwd(h, w, W1, W2, act, T, D, E, F, sv, dout, dh, dw, dW1, dW2, ws, ws_bytes,
                            stream);
}

}  // extern "C"
