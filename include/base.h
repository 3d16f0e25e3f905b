/*
 * base.h -- C ABI of libbase, the sm_100a (B200) hot path of a BASE layer.
 *
 * A BASE layer ("BASE Layers: Simplifying Training of Large, Sparse Models",
 * Lewis et al.; the wikillm.com summary's Method section) sends every token
 * h_t (width D) to exactly one of E experts.  In training the routing is a
 * balanced linear assignment (eq. 2: maximise sum_t h_t . w_{a_t} with every
 * expert receiving exactly T/E tokens); at test time each token goes to its
 * highest-affinity expert ("Test time").  The token leaves the layer as
 * sigma(h_t . w_{a_t}) f_{a_t}(h_t) + h_t (eq. 1), where f_e is the expert's
 * position-wise FFN ("Placement and shape").  The fig. 2 listing gives the
 * order of the steps: affinities -> balanced_assignment -> sort_by_expert ->
 * gated expert + residual -> inverse_sort.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument except `stats`' host copy is DEVICE memory owned
 *     by the caller.  The library never allocates device memory, never
 *     synchronises the host and enqueues all work on `stream` (may be 0).
 *   - Tensors are dense row-major.  Base pointers are 16-byte aligned.
 *     D % 8 == 0 and F % 8 == 0 (16-byte rows); 2 <= E <= 1024; 1 <= T < 2^31.
 *     Balanced assignment needs T % E == 0 (the page's Pitfalls note that the
 *     released code silently uses integer division instead).
 *   - Inputs are const and must not alias outputs.
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns BASE_ERR_INVALID_ARG and launches nothing.  A failed
 *     launch returns BASE_ERR_CUDA.  Failures found while the kernels run
 *     are written to device memory and read back by the caller after
 *     synchronising: the auction's round cap goes to `stats->status`; a
 *     bounded wait that gave up, or unusable device data, goes to the
 *     library's sticky device error word (base_device_error).
 *   - bf16 means IEEE bfloat16 (1-8-7), fp32 IEEE binary32.
 *   - The library holds no per-call state; calls on different streams with
 *     disjoint buffers may run concurrently.
 */
#ifndef BASE_H
#define BASE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BASE_OK = 0,
    BASE_ERR_INVALID_ARG = 1,   /* bad shape, null or misaligned pointer, small workspace */
    BASE_ERR_CUDA = 2,          /* a CUDA runtime call or launch failed */
    BASE_ERR_NOT_CONVERGED = 3, /* auction hit BASE_AUCTION_MAX_ROUNDS (device status) */
    BASE_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up (device status) */
    BASE_ERR_WORKSPACE = 5,     /* workspace smaller than base_workspace_size() */
    BASE_ERR_UNSUPPORTED = 6    /* shape outside what the kernels implement */
} base_status;

typedef enum { BASE_F32 = 0, BASE_BF16 = 1 } base_dtype;
typedef enum { BASE_RELU = 0, BASE_GELU = 1 } base_act;
/* Routing of the layer forward; BASE_ROUTE_SANITIZE may be OR'ed in to
 * replace non-finite scores first (see base_sanitize_scores). */
typedef enum {
    BASE_ROUTE_BALANCED = 0,
    BASE_ROUTE_GREEDY = 1,
    BASE_ROUTE_SANITIZE = 0x100
} base_routing;

/* Quantisation scale of the affinity scores: q = rint(s * 2^16). */
#define BASE_QSCALE 65536.0f
/* Hang guard of the auction: total rounds over all phases. */
#define BASE_AUCTION_MAX_ROUNDS 1000000

/*
 * Auction statistics, written by base_assign_balanced into DEVICE memory
 * (48 bytes, 8-byte aligned).  status is a base_status; phases and rounds
 * count epsilon-scaling phases and Jacobi rounds; final_eps is the last
 * epsilon (1 on success); objective = sum_t q[t][assign[t]]; bids = total
 * number of bids over all rounds (sum of the unassigned counts).
 */
typedef struct {
    int64_t status;
    int64_t phases;
    int64_t rounds;
    int64_t final_eps;
    int64_t objective;
    int64_t bids;
} base_auction_stats;

/*
 * Device buffers of one layer forward, kept for the backward.  All owned by
 * the caller; sizes in elements.  Pointers marked "fwd-only nullable" may be
 * NULL when no backward follows.
 */
typedef struct {
    float*   s;        /* T*E   fp32 scores s = h w^T                             */
    int32_t* q;        /* T*E   int32 quantised scores                            */
    int32_t* assign;   /* T     expert of every token                             */
    int64_t* price;    /* E     final auction prices (balanced routing)           */
    base_auction_stats* stats; /* 1 (device); balanced routing only               */
    int32_t* perm;     /* T     perm[slot] = token                                */
    int32_t* inv;      /* T     inv[token] = slot                                 */
    int32_t* offsets;  /* E+1   first slot of every expert                        */
    float*   gate;     /* T     s[perm[slot], assign[perm[slot]]], slot order      */
    void*    x_perm;   /* T*D   bf16 tokens in slot order                          */
    void*    a1;       /* T*F   bf16 pre-activation (fwd-only nullable)            */
    void*    h1;       /* T*F   bf16 activation                                    */
    void*    f;        /* T*D   bf16 expert output f (fwd-only nullable)           */
    void*    y_perm;   /* T*D   bf16 layer output in slot order                    */
} base_layer_saved;

/* Human-readable name of a status code (static string). */
const char* base_status_string(int status);

/*
 * Reads the library's sticky device error word into *code (0: none) and
 * clears it when `clear` is non-zero.  A kernel writes it when one of its
 * bounded waits gives up (codes 3001-3005: tensor-core GEMM pipeline) or when
 * it meets data it cannot use (1000+e: auction bookkeeping of expert e;
 * 2001: an assignment entry outside [0, E); 2002: a permutation entry
 * outside [0, T), its row skipped; 4001: the backward was given a
 * slot layout that is not the balanced one).  Synchronises the device.
 */
int base_device_error(int64_t* code, int clear);

/*
 * Test hooks (no counterpart in the paper).  Every device-side wait in the
 * library is bounded: the auction's grid barrier gives up after 20 s (device
 * error 5001, stats->status = BASE_ERR_TIMEOUT), the tensor-core GEMM
 * pipeline's waits after 4 s (codes 3001-3005); the kernel then lets its
 * copies in flight land, frees what it holds and returns, so the context
 * stays usable.  These hooks let a test watch that happen without any fault:
 *   BASE_TEST_WAIT_LIMIT_NS        value > 0: every bounded wait gives up
 *                                  after `value` ns; 0: the defaults above.
 *   BASE_TEST_AUCTION_ABSENT_CTA   value >= 0: that CTA of the auction's grid
 *                                  returns at once, so the other CTAs' first
 *                                  grid barrier runs out; -1: off.
 *   BASE_TEST_GEMM_DROP_FIRST_LOAD 1: CTA 0 of a one-CTA tensor-core GEMM
 *                                  (the bf16 score GEMM) never issues its
 *                                  first TMA load, so its MMA warp's wait for
 *                                  that stage runs out (3003); 0: off.
 * The settings are process-wide host state read when a kernel is launched;
 * they are for tests only and are not safe to change while other threads
 * launch.  Returns BASE_ERR_INVALID_ARG for an unknown hook or value.
 */
typedef enum {
    BASE_TEST_WAIT_LIMIT_NS = 0,
    BASE_TEST_AUCTION_ABSENT_CTA = 1,
    BASE_TEST_GEMM_DROP_FIRST_LOAD = 2
} base_test_hook;
int base_test_inject(int hook, long long value);

/*
 * Latency floors for the auction's latency roofline (no counterpart in the
 * paper: a measurement aid).  One cooperative grid of the auction's shape
 * writes to out (4 doubles of DEVICE memory) the nanoseconds of
 *   [0] one grid barrier of the auction's kind over all SMs,
 *   [1] one block barrier of 512 threads,
 *   [2] one dependent load that hits L2,
 *   [3] one dependent shared-memory load.
 * ws: at least base_probe_workspace_size() bytes.  Read out after
 * synchronising the stream.
 */
size_t base_probe_workspace_size(void);
int base_measure_latency(double* out, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Library version string (static). */
const char* base_version(void);

/*
 * Workspace bytes that every call below needs at most for these sizes
 * (F may be 0 when no FFN runs).  Host only; makes no CUDA call.
 */
size_t base_workspace_size(int T, int E, int D, int F);

/*
 * a1+a2: affinity scores and their quantisation (fig. 2: affinities =
 * features @ centroids^T; the quantisation scale 2^16 is this library's).
 *   h: T*D, w: E*D, both of `dtype` (BASE_F32 or BASE_BF16).
 *   s (nullable): T*E fp32, s[t][e] = sum_d h[t][d] w[e][d], fp32 accumulation.
 *   q (nullable): T*E int32, q = rint(s * 65536) (round half to even),
 *     saturated to +-(2^31 - 1).
 *   bf16 inputs run on the tensor cores (tcgen05); fp32 inputs use fp32 FMA.
 */
int base_scores(const void* h, const void* w, int dtype, int T, int D, int E,
                float* s, int32_t* q, cudaStream_t stream);

/*
 * a1 + a2 + a3 in one pass: the scores and their quantisation as base_scores,
 * and the greedy test-time routing of base_assign_greedy on that q (argmax,
 * lowest e on ties), computed in the score GEMM's epilogue when the inputs
 * are bf16 and E <= 256 (every row's experts in one tile); otherwise
 * base_scores then base_assign_greedy.  q, assign: required; s, counts:
 * nullable (counts: E int32, tokens per expert).  base_layer_fwd's greedy
 * routing goes through this call.
 */
int base_scores_greedy(const void* h, const void* w, int dtype, int T, int D, int E, float* s,
                       int32_t* q, int32_t* assign, int32_t* counts, cudaStream_t stream);

/*
 * Non-finite scores (the wikillm.com summary's "Paper vs code", Non-finite
 * scores: the released code replaces NaN and infinite affinities with the
 * minimum finite score before solving).  Every entry of s (T*E fp32) that is
 * NaN or +-Inf becomes the smallest finite entry m (0 when none is finite),
 * and the same entries of q (nullable) become rint(m * 65536), the
 * quantisation of m.  Finite entries are not touched.  ws: at least
 * base_workspace_size(T, E, 0, 0) bytes.  Two launches, no host sync.
 */
int base_sanitize_scores(float* s, int32_t* q, int T, int E, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/*
 * a3: greedy test-time routing (Method, "Test time": each token to its
 * highest-scoring expert).  assign[t] = argmax_e q[t][e], lowest e on ties;
 * counts (nullable) E int32: number of tokens per expert.
 */
int base_assign_greedy(const int32_t* q, int T, int E, int32_t* assign, int32_t* counts,
                       cudaStream_t stream);

/*
 * a4: balanced assignment (eq. 2) by a Jacobi token-bidding auction with
 * epsilon scaling, exact for integer scores.  Values A[t][e] = q[t][e] (T+1);
 * eps starts at max(1, (max q - min q)(T+1)/50) (the released solver's
 * range/50 rule, "Paper vs code") and is divided by 8 per phase down to 1.
 * In every round each unassigned token bids best - second + eps above the
 * price of its best expert; each expert keeps its C = T/E best bids (larger
 * bid, then smaller token index) and, once full, sets its price to the
 * lowest bid it holds.  The result is an exact optimum of eq. 2.
 *   q: T*E int32 (|q| < 2^31; the scaled range (max-min)(T+1) must be < 2^58).
 *   assign: T int32 output.  price: E int64 output (final prices).
 *   stats (nullable): device base_auction_stats.
 *   ws: workspace of at least base_workspace_size(T, E, 0, 0) bytes.
 * Runs as one cooperative grid of one 512-thread CTA per SM (the score range
 * for eps is reduced inside it): rounds with many bidders use every SM, the
 * tail of each phase runs on one CTA with the prices and each expert's worst
 * held bids in shared memory, and once a single bidder is left one warp
 * finishes the phase.
 */
int base_assign_balanced(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                         base_auction_stats* stats, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/*
 * base_assign_balanced with two extras for tests and profiling:
 *   max_rounds (1 .. BASE_AUCTION_MAX_ROUNDS) lowers the round cap; when the
 *     cap is reached stats->status becomes BASE_ERR_NOT_CONVERGED and
 *     assign / price are not meaningful;
 *   u_trace (nullable, device int32[trace_cap]) receives the number of
 *     bidders of round r, and t_trace (nullable, device int64[trace_cap]) the
 *     GPU global timer (ns) at the start of round r, for r < trace_cap.
 */
int base_assign_balanced_ex(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                            base_auction_stats* stats, long long max_rounds, int32_t* u_trace,
                            int64_t* t_trace, long long trace_cap, void* ws, size_t ws_bytes,
                            cudaStream_t stream);

/*
 * The page's fig. 9 solver (the wikillm.com summary's "Solver": experts bid
 * for tokens and prices are per token), with the released code's rules that
 * "Paper vs code" describes: eps = max(1, (max q - min q) / 50) on the
 * quantised scores; a token won in a round stays in its holder's list at the
 * largest score plus one (the listing's "infinity", kept finite and strictly
 * above every other value); while the round number is below max_iterations
 * (the listing's cap, 100) the holder bids eps on it; after the cap the
 * listing's other update runs and rounds go on until every token has a bid.
 * Every round, each expert bids raise = v_j - v_{C+1} + eps on the tokens of
 * its C best adjusted values (ties: smaller token first); a token goes to its
 * largest bid (smaller expert on ties), is won when that bid is > 0, and its
 * price grows by it.  The result is balanced; it is not the exact optimum of
 * eq. 2 (the eps of one phase bounds the loss), and base_assign_balanced
 * remains the training solver.
 *   q: T*E int32; assign: T int32; price: T int64 token prices;
 *   stats (nullable): 4 int64 of device memory -- status, rounds, eps,
 *   objective (sum_t q[t][assign[t]]); status BASE_ERR_NOT_CONVERGED when
 *   BASE_AUCTION_MAX_ROUNDS pass.
 *   ws: at least base_workspace_size_fig9(T, E) bytes.  One cooperative grid.
 */
size_t base_workspace_size_fig9(int T, int E);
int base_assign_fig9(const int32_t* q, int T, int E, int32_t* assign, int64_t* price,
                     int64_t* stats, long long max_iterations, void* ws, size_t ws_bytes,
                     cudaStream_t stream);

/*
 * a5: permutation into expert-contiguous slots (fig. 2 sort_by_expert).
 * Slot order is expert-major and ascending token index inside an expert.
 *   h: T*D bf16; assign: T int32 in [0, E).
 *   perm: T (perm[slot] = t); inv: T (inv[t] = slot); offsets: E+1 int32.
 *   x_perm: T*D bf16, x_perm[slot] = h[perm[slot]].
 *   s (nullable) T*E fp32 with gate (nullable) T fp32:
 *     gate[slot] = s[perm[slot]][assign[perm[slot]]].
 */
int base_permute(const void* h, const int32_t* assign, int T, int D, int E,
                 int32_t* perm, int32_t* inv, int32_t* offsets, void* x_perm,
                 const float* s, float* gate, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * base_permute for callers that cannot allocate device memory.  The paper has
 * no counterpart: this is a deployment variant.  A caller that only holds its
 * inputs, outputs and a stream -- a plugin inside another runtime that owns
 * all device memory, or a serving loop that must not call cudaMalloc -- has
 * no workspace to give base_permute.  This entry point takes the same
 * arguments minus the workspace and keeps the scratch (the expert counts of
 * up to ceil(T/256) token slices, int32) in a 4 MiB array that the library reserves
 * in every GPU that loads it, for the life of the process.
 *   Limit: ceil(T/256) * E <= 1048576, else BASE_ERR_WORKSPACE and nothing
 *   is launched.  Allocates nothing.
 *   The first call on a device looks up the array's device address (a CUDA
 *   runtime query); make that first call before any stream capture.  The
 *   address is kept per device ordinal for the life of the process: after
 *   cudaDeviceReset, or from a driver context other than the one current at
 *   that first call, it is stale, so callers that reset the device or switch
 *   contexts must use base_permute instead.
 *   All calls share the one array, whose contents the next call overwrites
 *   before reading; calls that overlap on the GPU race on it, so the caller
 *   must order them (one stream, or events).
 */
int base_permute_noalloc(const void* h, const int32_t* assign, int T, int D, int E,
                         int32_t* perm, int32_t* inv, int32_t* offsets, void* x_perm,
                         const float* s, float* gate, cudaStream_t stream);

/*
 * a6+a7: the experts' FFNs on their slot segments with the eq. 1 combine in
 * the epilogue.  For every expert e and slot r in [offsets[e], offsets[e+1]):
 *   a1[r] = x_perm[r] W1[e]^T          (W1: E*F*D bf16)
 *   h1[r] = act(a1[r])                 (ReLU, or GELU 0.5x(1+erf(x/sqrt2)))
 *   f[r]  = h1[r] W2[e]^T              (W2: E*D*F bf16)
 *   y_perm[r] = sigmoid(gate[r]) f[r] + x_perm[r]
 * fp32 accumulation on the tensor cores; h1, a1, f, y_perm stored as bf16.
 *   h1: T*F bf16 (required: GEMM2 reads it).  a1, f: nullable.
 */
int base_expert_ffn(const void* x_perm, const int32_t* offsets, int T, int D, int F, int E,
                    const void* W1, const void* W2, int act, const float* gate,
                    void* y_perm, void* h1, void* a1, void* f, void* ws, size_t ws_bytes,
                    cudaStream_t stream);

/*
 * a8: combine (fig. 2 inverse_sort): out[perm[slot]] = y_perm[slot], T*D bf16.
 */
int base_combine(const void* y_perm, const int32_t* perm, int T, int D, void* out,
                 cudaStream_t stream);

/*
 * Expert parallelism (wikillm.com summary, Method: Sharding; fig. 2's forward
 * pass): G workers (1 <= G <= 8, one node) each hold T tokens and E/G experts
 * (El = E/G; worker r holds experts r El .. r El + El - 1), and every expert
 * gets exactly C = T/E of each worker's tokens (balanced routing: E | T, G | E).
 * These two calls are each a permutation fused with its all-to-all, as plain
 * 16-byte loads and stores through pointers to every worker's buffers: the
 * pointers of other workers may be peer mappings (NVLink); on one GPU, one
 * call over all workers' buffers runs the whole exchange.
 *
 * base_ep_dispatch -- sort_by_expert + the route all-to-all + the receive
 * side's grouping: for each source worker g in [g0, g0 + ns) and slot s of
 * its expert-major order (perm_g from base_permute, balanced: expert e =
 * s / C, c = s % C, worker r = e / El, local expert j = e % El):
 *     recv_r[(j G + g) C + c] = h_g[perm_g[s]]   (rows of D bf16)
 *     recv_gate_r[(j G + g) C + c] = gate_g[s]   (when the gate pointers are given)
 * so every worker receives its experts' rows expert-major (local expert j's
 * G C rows together: the offsets of base_expert_ffn are j G C).
 *   h, perm, gate: host arrays of ns device pointers (sources g0..g0+ns-1:
 *   T*D bf16 tokens, T int32 slot -> token, T fp32 gate scores in slot
 *   order); gate nullable (then recv_gate must be null too).
 *   recv, recv_gate: host arrays of G device pointers (T*D bf16, T fp32).
 *   A worker's own call passes g0 = its rank, ns = 1.  The receivers may read
 *   only after every source has written (a barrier across the workers).
 *   A slot whose token is out of range is recorded in the device error word
 *   (2101) and skipped.
 */
int base_ep_dispatch(const void* const* h, const int32_t* const* perm, const float* const* gate,
                     void* const* recv, float* const* recv_gate, int g0, int ns, int G, int T,
                     int D, int E, cudaStream_t stream);

/*
 * base_ep_combine -- the return all-to-all + inverse_sort: for each receiver
 * r in [r0, r0 + nr) and row i = (j G + g) C + c of its expert outputs,
 *     out_g[perm_g[(r El + j) C + c]] = y_r[i]   (rows of D bf16)
 * so every output row lands on its token in the source worker's order.
 *   y: host array of nr device pointers (receivers r0..r0+nr-1, T*D bf16);
 *   perm, out: host arrays of G device pointers (T int32, T*D bf16).
 *   Errors as base_ep_dispatch (2102).
 */
int base_ep_combine(const void* const* y, const int32_t* const* perm, void* const* out, int r0,
                    int nr, int G, int T, int D, int E, cudaStream_t stream);

/*
 * The whole layer forward on one stream without host synchronisation:
 * scores -> (balanced auction | greedy) -> permute -> expert FFN + eq. 1 ->
 * combine.  h: T*D bf16, w: E*D bf16, W1: E*F*D, W2: E*D*F bf16; out: T*D bf16.
 * sv: host struct of caller-owned device buffers (see base_layer_saved).
 * Greedy routing fills price/stats untouched and accepts any counts.
 */
int base_layer_fwd(const void* h, const void* w, const void* W1, const void* W2, int act,
                   int routing, int T, int D, int E, int F, void* out,
                   const base_layer_saved* sv, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * The released code's layer variant (the wikillm.com summary's "Paper vs
 * code", Mixing equation, and "Placement and shape"): the same routing and
 * permutation, but every expert is a stack of S sublayers
 *   x <- x + W2[e][i] act(W1[e][i] LN_i(x)),   i = 0 .. S-1,
 * with LN_i the layer norm of the row (biased variance, eps 1e-5) scaled by
 * gamma[e][i] and shifted by beta[e][i], and the token leaves the layer as
 * the convex blend  alpha_t x_S + (1 - alpha_t) h_t,  alpha_t =
 * sigmoid(h_t . w_{a_t})  (instead of eq. 1's sigmoid(.) f + h).
 *   W1: E*S*F*D bf16, W2: E*S*D*F bf16 (expert-major, then sublayer);
 *   gamma, beta: E*S*D fp32; S >= 1; the other arguments as base_layer_fwd.
 *   sv: s, q, assign, price, stats, perm, inv, offsets, gate, x_perm, h1 and
 *   y_perm are written (a1 and f are not used); ws: at least
 *   base_workspace_size_blend(T, E, D, F) bytes.  Forward only.
 */
size_t base_workspace_size_blend(int T, int E, int D, int F);
/*
 * The variant's expert step alone (its counterpart of base_expert_ffn): for
 * every expert e and slot r in [offsets[e], offsets[e+1]), starting from
 * x = x_perm[r], the S sublayers above, then
 *   y_perm[r] = x_perm[r] + sigmoid(gate[r]) (x_S - x_perm[r]).
 *   h1: T*F bf16 scratch of the sublayers; ws: base_workspace_size_blend bytes.
 */
int base_expert_stack(const void* x_perm, const int32_t* offsets, int T, int D, int F, int E,
                      int S, const void* W1, const void* W2, const float* gamma, const float* beta,
                      int act, const float* gate, void* y_perm, void* h1, void* ws,
                      size_t ws_bytes, cudaStream_t stream);
int base_layer_fwd_blend(const void* h, const void* w, const void* W1, const void* W2,
                         const float* gamma, const float* beta, int S, int act, int routing,
                         int T, int D, int E, int F, void* out, const base_layer_saved* sv,
                         void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * a9: the layer backward with the assignment held fixed (the released code
 * computes the routing affinities without gradient; the centroids receive
 * gradient only through the gate, "Paper vs code").  Given dout (T*D bf16):
 *   dy = dout[perm]; dgate = <dy, f>; ds = dgate sigma (1 - sigma);
 *   dF = sigma dy; dH1 = dF W2_e; dW2_e = dF^T H1; dA1 = dH1 * act'(A1);
 *   dW1_e = dA1^T x; dx = dA1 W1_e + dy + ds w_e; dw_e = sum_{t in e} ds h_t;
 *   dh[t] = dx[inv[t]].
 * Outputs: dh T*D bf16; dw E*D fp32; dW1 E*F*D fp32; dW2 E*D*F fp32.
 * sv must hold the forward's a1, h1, f (non-null).  The backward exists for
 * training, i.e. balanced routing: it needs T % E == 0 with (T/E) % 64 == 0,
 * D % 64 == 0 and F % 64 == 0 (BASE_ERR_UNSUPPORTED otherwise), and
 * sv->offsets must be the balanced layout e * T/E (checked on the device,
 * error word 4001).
 */
int base_layer_bwd(const void* h, const void* w, const void* W1, const void* W2, int act,
                   int T, int D, int E, int F, const base_layer_saved* sv, const void* dout,
                   void* dh, float* dw, float* dW1, float* dW2, void* ws, size_t ws_bytes,
                   cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BASE_H */
