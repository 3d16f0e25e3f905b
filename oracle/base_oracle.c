/*
 * base_oracle.c -- plain CPU oracle for the integer parts of the BASE-layer
 * hot path: the balanced assignment (a token-bidding Jacobi auction with
 * epsilon scaling), an independent Hungarian solver and a brute-force
 * enumerator that pin it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header or constant table with the CUDA library; the spec constants below
 * are restated here on purpose.
 *
 * What is computed (page "BASE Layers: Simplifying Training of Large, Sparse
 * Models", wikillm.com summary):
 *   - Method / "Training assignment", eq. 2: choose a_t for every token so as
 *     to maximise sum_t h_t . w_{a_t} subject to every expert receiving
 *     exactly T/E tokens.  Here the affinities are the integer quantised
 *     scores q[t][e].
 *   - The same section says the paper solves eq. 2 with an auction rather
 *     than the Hungarian method.  The auction below is the token-bids-for-
 *     expert Jacobi variant with per-expert prices (the page's fig. 9 listing,
 *     where experts bid for tokens, is prior art and is not followed).
 *   - The epsilon start value follows the released solver's range/50 rule
 *     described under "Paper vs code" (Epsilon bullet).  The cap on rounds
 *     is a hang guard only; the "greedy after 100 iterations" rule of the
 *     fig. 9 caption is not used (same section, "After the cap").
 *
 * The auction, step by step (all arithmetic in int64):
 *   A[t][e] = q[t][e] * (T+1).
 *   eps = max(1, floor((max q - min q) * (T+1) / 50)); price[e] = 0.
 *   phase: every token unassigned, every expert holds nothing; prices kept.
 *   round: every unassigned token t, with the prices of the round start,
 *     v_e = A[t][e] - price[e]; e* = argmax v_e (lowest e on ties);
 *     v2 = max_{e != e*} v_e; bid b_t = A[t][e*] - v2 + eps.
 *     Every expert keeps the C best of (what it held) + (new bids to it),
 *     best = larger bid, then smaller token index; the others become
 *     unassigned.  An expert that holds exactly C sets its price to the
 *     smallest bid it holds; otherwise its price is unchanged.
 *   the phase ends when no token is unassigned; stop if eps == 1, else
 *     eps = max(1, floor(eps / 8)) and start a new phase.
 * With eps == 1 in the last phase and every value a multiple of T+1 the
 * result is an exact optimum of eq. 2 (epsilon complementary slackness).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <limits.h>

#define ORC_EPS_DIVISOR 50
#define ORC_EPS_FACTOR 8

/* status codes, same meaning as the library's */
#define ORC_OK 0
#define ORC_ERR_INVALID_ARG 1
#define ORC_ERR_NOT_CONVERGED 3

typedef struct {
    int64_t bid;
    int32_t tok;
} orc_key;

/* order: larger bid first, then smaller token index first */
static int orc_key_cmp(const void* pa, const void* pb) {
    const orc_key* a = (const orc_key*)pa;
    const orc_key* b = (const orc_key*)pb;
    if (a->bid != b->bid) return (a->bid > b->bid) ? -1 : 1;
    if (a->tok != b->tok) return (a->tok < b->tok) ? -1 : 1;
    return 0;
}

/*
 * stats_out (nullable), int64[6]: status, phases, rounds, final_eps,
 *   objective (sum_t q[t][assign[t]], unscaled), bids (sum over rounds of
 *   the number of bidders).
 * u_trace (nullable): u_trace[r] = number of bidders in round r, for
 *   r < min(rounds, trace_cap).
 * Returns the status.
 */
int orc_auction(const int32_t* q, int T, int E, int64_t max_rounds,
                int32_t* assign, int64_t* price, int64_t* stats_out,
                int32_t* u_trace, int64_t trace_cap) {
    if (!q || !assign || !price || T <= 0 || E < 2 || T % E != 0 || max_rounds <= 0)
        return ORC_ERR_INVALID_ARG;
    const int C = T / E;
    const int64_t scale = (int64_t)T + 1;

    int64_t qmin = INT64_MAX, qmax = INT64_MIN;
    for (int64_t i = 0; i < (int64_t)T * E; ++i) {
        if (q[i] < qmin) qmin = q[i];
        if (q[i] > qmax) qmax = q[i];
    }
    const int64_t range = qmax - qmin;
    /* the scaled range must leave room for the price growth of every phase */
    if (range > 0 && range > ((int64_t)1 << 58) / scale) return ORC_ERR_INVALID_ARG;
    int64_t eps = range * scale / ORC_EPS_DIVISOR;
    if (eps < 1) eps = 1;

    for (int e = 0; e < E; ++e) price[e] = 0;

    int32_t* held_tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);  /* [E][C] */
    int64_t* held_bid = (int64_t*)malloc(sizeof(int64_t) * (size_t)T);  /* [E][C] */
    int32_t* held_cnt = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* unassigned = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);
    int32_t* next_unassigned = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);
    int32_t* bid_exp = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);   /* per bidder slot */
    int64_t* bid_val = (int64_t*)malloc(sizeof(int64_t) * (size_t)T);
    int32_t* nbid = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t* bucket_start = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t* bucket = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);    /* bidder slots by expert */
    int32_t* rejected = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);
    int32_t* rej_cnt = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* rej_start = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    orc_key* cand = (orc_key*)malloc(sizeof(orc_key) * (size_t)(2 * T));
    if (!held_tok || !held_bid || !held_cnt || !unassigned || !next_unassigned || !bid_exp ||
        !bid_val || !nbid || !bucket_start || !bucket || !rejected || !rej_cnt || !rej_start || !cand) {
        free(held_tok); free(held_bid); free(held_cnt); free(unassigned); free(next_unassigned);
        free(bid_exp); free(bid_val); free(nbid); free(bucket_start); free(bucket);
        free(rejected); free(rej_cnt); free(rej_start); free(cand);
        return ORC_ERR_INVALID_ARG;
    }

    int status = ORC_OK;
    int64_t phases = 0, rounds = 0, bids = 0;

    for (;;) {
        /* a new phase: nothing held, everyone unassigned, prices kept */
        ++phases;
        for (int e = 0; e < E; ++e) held_cnt[e] = 0;
        int nu = T;
        for (int t = 0; t < T; ++t) unassigned[t] = t;

        while (nu > 0) {
            if (rounds >= max_rounds) { status = ORC_ERR_NOT_CONVERGED; break; }
            if (u_trace && rounds < trace_cap) u_trace[rounds] = nu;
            bids += nu;
            ++rounds;

            /* bidding: every unassigned token, prices of the round start */
            #pragma omp parallel for schedule(static)
            for (int i = 0; i < nu; ++i) {
                const int t = unassigned[i];
                const int32_t* row = q + (int64_t)t * E;
                int best = 0;
                int64_t v1 = (int64_t)row[0] * scale - price[0];
                for (int e = 1; e < E; ++e) {
                    int64_t v = (int64_t)row[e] * scale - price[e];
                    if (v > v1) { v1 = v; best = e; }
                }
                int64_t v2 = INT64_MIN;
                for (int e = 0; e < E; ++e) {
                    if (e == best) continue;
                    int64_t v = (int64_t)row[e] * scale - price[e];
                    if (v > v2) v2 = v;
                }
                bid_exp[i] = best;
                bid_val[i] = (int64_t)row[best] * scale - v2 + eps;
            }

            /* group the bids by expert (a counting sort over bidder slots) */
            for (int e = 0; e <= E; ++e) nbid[e] = 0;
            for (int i = 0; i < nu; ++i) nbid[bid_exp[i]]++;
            bucket_start[0] = 0;
            for (int e = 0; e < E; ++e) bucket_start[e + 1] = bucket_start[e] + nbid[e];
            for (int e = 0; e < E; ++e) nbid[e] = bucket_start[e];
            for (int i = 0; i < nu; ++i) bucket[nbid[bid_exp[i]]++] = i;

            /* resolution: each expert keeps the C best of held + new; the
               candidates of expert e go to cand[rej_start[e] ...] */
            int cand_base = 0;
            for (int e = 0; e < E; ++e) {
                const int nb = bucket_start[e + 1] - bucket_start[e];
                rej_start[e] = cand_base;
                if (nb == 0) continue;
                cand_base += held_cnt[e] + nb;
            }
            rej_start[E] = cand_base;
            #pragma omp parallel for schedule(dynamic, 1)
            for (int e = 0; e < E; ++e) {
                const int nb = bucket_start[e + 1] - bucket_start[e];
                rej_cnt[e] = 0;
                if (nb == 0) continue;
                orc_key* c = cand + rej_start[e];
                int m = 0;
                for (int j = 0; j < held_cnt[e]; ++j) {
                    c[m].bid = held_bid[(int64_t)e * C + j];
                    c[m].tok = held_tok[(int64_t)e * C + j];
                    ++m;
                }
                for (int j = bucket_start[e]; j < bucket_start[e + 1]; ++j) {
                    const int slot = bucket[j];
                    c[m].bid = bid_val[slot];
                    c[m].tok = unassigned[slot];
                    ++m;
                }
                qsort(c, (size_t)m, sizeof(orc_key), orc_key_cmp);
                const int keep = m < C ? m : C;
                for (int j = 0; j < keep; ++j) {
                    held_bid[(int64_t)e * C + j] = c[j].bid;
                    held_tok[(int64_t)e * C + j] = c[j].tok;
                }
                held_cnt[e] = keep;
                rej_cnt[e] = m - keep;
                if (keep == C) price[e] = c[C - 1].bid;
            }

            /* the rejected tokens, in ascending token order, bid next round */
            int nn = 0;
            for (int e = 0; e < E; ++e) {
                if (rej_cnt[e] == 0) continue;
                const orc_key* c = cand + rej_start[e];
                const int keep = held_cnt[e];
                for (int j = 0; j < rej_cnt[e]; ++j) next_unassigned[nn++] = c[keep + j].tok;
            }
            /* a mark-and-sweep over token indices keeps the list ordered */
            if (nn > 0) {
                memset(rejected, 0, sizeof(int32_t) * (size_t)T);
                for (int j = 0; j < nn; ++j) rejected[next_unassigned[j]] = 1;
                int k = 0;
                for (int t = 0; t < T; ++t) if (rejected[t]) unassigned[k++] = t;
            }
            nu = nn;
        }
        if (status != ORC_OK) break;
        if (eps == 1) break;
        eps /= ORC_EPS_FACTOR;
        if (eps < 1) eps = 1;
    }

    int64_t objective = 0;
    if (status == ORC_OK) {
        for (int e = 0; e < E; ++e)
            for (int j = 0; j < held_cnt[e]; ++j) assign[held_tok[(int64_t)e * C + j]] = e;
        for (int t = 0; t < T; ++t) objective += q[(int64_t)t * E + assign[t]];
    }
    if (stats_out) {
        stats_out[0] = status;
        stats_out[1] = phases;
        stats_out[2] = rounds;
        stats_out[3] = eps;
        stats_out[4] = objective;
        stats_out[5] = bids;
    }
    free(held_tok); free(held_bid); free(held_cnt); free(unassigned); free(next_unassigned);
    free(bid_exp); free(bid_val); free(nbid); free(bucket_start); free(bucket);
    free(rejected); free(rej_cnt); free(rej_start); free(cand);
    return status;
}

/*
 * Hungarian method (Kuhn-Munkres with row potentials, O(n^3)), the solver the
 * page names as the alternative to the auction (Method / "Training
 * assignment").  Used only to pin the auction: eq. 2 becomes an ordinary
 * n x n assignment by giving every expert C identical slots, slot j belonging
 * to expert j / C.  Maximises sum_t q[t][slot_expert(t)].
 * Returns the optimum objective; writes assign[t] (nullable).  T <= 4096.
 */
int64_t orc_hungarian(const int32_t* q, int T, int E, int32_t* assign) {
    if (!q || T <= 0 || E < 1 || T % E != 0 || T > 4096) return INT64_MIN;
    const int n = T, C = T / E;
    /* cost[i][j] = -q[i][j / C], minimised; 1-based arrays as in the textbook */
    int64_t* u = (int64_t*)calloc((size_t)n + 1, sizeof(int64_t));
    int64_t* v = (int64_t*)calloc((size_t)n + 1, sizeof(int64_t));
    int* p = (int*)calloc((size_t)n + 1, sizeof(int));    /* p[j] = row matched to column j */
    int* way = (int*)calloc((size_t)n + 1, sizeof(int));
    int64_t* minv = (int64_t*)malloc(sizeof(int64_t) * ((size_t)n + 1));
    char* used = (char*)malloc((size_t)n + 1);
    const int64_t INF = INT64_MAX / 4;
    for (int i = 1; i <= n; ++i) {
        p[0] = i;
        int j0 = 0;
        for (int j = 0; j <= n; ++j) { minv[j] = INF; used[j] = 0; }
        do {
            used[j0] = 1;
            const int i0 = p[j0];
            int64_t delta = INF;
            int j1 = 0;
            for (int j = 1; j <= n; ++j) {
                if (used[j]) continue;
                const int64_t cost = -(int64_t)q[(int64_t)(i0 - 1) * E + (j - 1) / C];
                const int64_t cur = cost - u[i0] - v[j];
                if (cur < minv[j]) { minv[j] = cur; way[j] = j0; }
                if (minv[j] < delta) { delta = minv[j]; j1 = j; }
            }
            for (int j = 0; j <= n; ++j) {
                if (used[j]) { u[p[j]] += delta; v[j] -= delta; }
                else minv[j] -= delta;
            }
            j0 = j1;
        } while (p[j0] != 0);
        do {
            const int j1 = way[j0];
            p[j0] = p[j1];
            j0 = j1;
        } while (j0);
    }
    int64_t objective = 0;
    for (int j = 1; j <= n; ++j) {
        const int row = p[j] - 1, e = (j - 1) / C;
        objective += q[(int64_t)row * E + e];
        if (assign) assign[row] = e;
    }
    free(u); free(v); free(p); free(way); free(minv); free(used);
    return objective;
}

/*
 * Brute force over every balanced assignment (each expert exactly T/E
 * tokens), the definition of eq. 2 enumerated directly.  For tiny inputs
 * only (T <= 16).  Returns the optimum; *n_assign counts the balanced
 * assignments visited and *n_opt the optimal ones.
 */
typedef struct {
    const int32_t* q;
    int T, E;
    int cap[64];
    int cur[16];
    int64_t best;
    int64_t n_assign, n_opt;
    int32_t* best_assign;
} orc_bf_state;

static void orc_bf_rec(orc_bf_state* st, int t, int64_t acc) {
    if (t == st->T) {
        st->n_assign++;
        if (acc > st->best) {
            st->best = acc;
            st->n_opt = 1;
            if (st->best_assign)
                for (int i = 0; i < st->T; ++i) st->best_assign[i] = st->cur[i];
        } else if (acc == st->best) {
            st->n_opt++;
        }
        return;
    }
    for (int e = 0; e < st->E; ++e) {
        if (st->cap[e] == 0) continue;
        st->cap[e]--;
        st->cur[t] = e;
        orc_bf_rec(st, t + 1, acc + st->q[(int64_t)t * st->E + e]);
        st->cap[e]++;
    }
}

int64_t orc_bruteforce(const int32_t* q, int T, int E, int32_t* best_assign,
                       int64_t* n_assign, int64_t* n_opt) {
    if (!q || T <= 0 || T > 16 || E < 1 || E > 64 || T % E != 0) return INT64_MIN;
    orc_bf_state st;
    memset(&st, 0, sizeof(st));
    st.q = q; st.T = T; st.E = E;
    for (int e = 0; e < E; ++e) st.cap[e] = T / E;
    st.best = INT64_MIN;
    st.best_assign = best_assign;
    orc_bf_rec(&st, 0, 0);
    if (n_assign) *n_assign = st.n_assign;
    if (n_opt) *n_opt = st.n_opt;
    return st.best;
}

/*
 * The page's fig. 9 listing ("Solver"): an auction in which EXPERTS bid for
 * TOKENS and prices live per token, with the released code's rules where the
 * page says the code differs ("Paper vs code": eps = range / 50, winners kept
 * in their holder's list at the largest score rather than infinity, and after
 * the iteration cap the update rule changes while the loop goes on until
 * every token has a bid -- no greedy fallback).  Integer version on the
 * quantised scores S[e][t] = q[t][e] (int64):
 *   eps = max(1, floor((max q - min q) / 50));  RETAIN = max q + 1;
 *   price[t] = 0; adjusted = S; nobody has won.
 *   round r (while some token has not won):
 *     every expert takes its C + 1 largest adjusted values (ties: smaller
 *     token first) and bids raise = v_j - v_C + eps on its top C tokens;
 *     if 0 < r < max_iterations, every token won in the last round gets the
 *     bid eps from its holder instead (overwriting that holder's own bid);
 *     each token goes to its largest bid (smaller expert on ties); it is won
 *     when that bid is > 0; price[t] += that bid;
 *     adjusted[e][t] = S[e][t] - price[t], and for every won token, in its
 *     holder's row: RETAIN if r < max_iterations, else S[holder][t].
 *   The result is the last round's top-C lists (a partition of the tokens
 *   once every token has won).
 * RETAIN is the largest score plus one: with the largest score itself a kept
 * token ties with an untouched token of that score, and the tie rule could
 * push it out of its holder's list.
 * stats_out (nullable) int64[4]: status, rounds, eps, objective.
 * price_out (nullable): T int64 final token prices.
 */
typedef struct {
    int64_t v;
    int32_t t;
} orc_vt;

/* larger value first, then smaller token */
static int orc_vt_cmp(const void* pa, const void* pb) {
    const orc_vt* a = (const orc_vt*)pa;
    const orc_vt* b = (const orc_vt*)pb;
    if (a->v != b->v) return (a->v > b->v) ? -1 : 1;
    return (a->t < b->t) ? -1 : (a->t > b->t);
}

int orc_fig9(const int32_t* q, int T, int E, int64_t max_iterations, int64_t max_rounds,
             int32_t* assign, int64_t* price_out, int64_t* stats_out) {
    if (!q || !assign || T <= 0 || E < 2 || T % E != 0 || max_rounds <= 0 || max_iterations < 0)
        return ORC_ERR_INVALID_ARG;
    const int C = T / E;
    if (C + 1 > T) return ORC_ERR_INVALID_ARG;
    int64_t qmin = INT64_MAX, qmax = INT64_MIN;
    for (int64_t i = 0; i < (int64_t)T * E; ++i) {
        if (q[i] < qmin) qmin = q[i];
        if (q[i] > qmax) qmax = q[i];
    }
    int64_t eps = (qmax - qmin) / 50;
    if (eps < 1) eps = 1;
    const int64_t RETAIN = qmax + 1;
    int64_t* adj = (int64_t*)malloc(sizeof(int64_t) * (size_t)E * T);
    int64_t* bids = (int64_t*)malloc(sizeof(int64_t) * (size_t)E * T);
    int64_t* price = (int64_t*)calloc((size_t)T, sizeof(int64_t));
    char* won = (char*)calloc((size_t)T, 1);
    int32_t* holder = (int32_t*)malloc(sizeof(int32_t) * (size_t)T);
    int32_t* best_ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)E * (C + 1));
    int64_t* best_vals = (int64_t*)malloc(sizeof(int64_t) * (size_t)E * (C + 1));
    orc_vt* work = (orc_vt*)malloc(sizeof(orc_vt) * (size_t)E * T);
    if (!adj || !bids || !price || !won || !holder || !best_ids || !best_vals || !work) {
        free(adj); free(bids); free(price); free(won); free(holder); free(best_ids);
        free(best_vals); free(work);
        return ORC_ERR_INVALID_ARG;
    }
    for (int e = 0; e < E; ++e)
        for (int t = 0; t < T; ++t) adj[(int64_t)e * T + t] = q[(int64_t)t * E + e];
    for (int t = 0; t < T; ++t) holder[t] = -1;
    int status = ORC_OK;
    int64_t round = 0;
    for (;;) {
        int all = 1;
        for (int t = 0; t < T; ++t) all &= won[t];
        if (all && round > 0) break;
        if (round >= max_rounds) { status = ORC_ERR_NOT_CONVERGED; break; }
        /* each expert's C + 1 largest adjusted values */
        #pragma omp parallel for schedule(static)
        for (int e = 0; e < E; ++e) {
            orc_vt* w = work + (int64_t)e * T;
            for (int t = 0; t < T; ++t) { w[t].v = adj[(int64_t)e * T + t]; w[t].t = t; }
            qsort(w, (size_t)T, sizeof(orc_vt), orc_vt_cmp);
            for (int j = 0; j <= C; ++j) {
                best_ids[(int64_t)e * (C + 1) + j] = w[j].t;
                best_vals[(int64_t)e * (C + 1) + j] = w[j].v;
            }
        }
        memset(bids, 0, sizeof(int64_t) * (size_t)E * T);
        for (int e = 0; e < E; ++e) {
            const int64_t vc = best_vals[(int64_t)e * (C + 1) + C];
            for (int j = 0; j < C; ++j) {
                const int t = best_ids[(int64_t)e * (C + 1) + j];
                bids[(int64_t)e * T + t] = best_vals[(int64_t)e * (C + 1) + j] - vc + eps;
            }
        }
        if (round > 0 && round < max_iterations)
            for (int t = 0; t < T; ++t)
                if (won[t]) bids[(int64_t)holder[t] * T + t] = eps;
        for (int t = 0; t < T; ++t) {
            int64_t best = bids[t];
            int arg = 0;
            for (int e = 1; e < E; ++e)
                if (bids[(int64_t)e * T + t] > best) { best = bids[(int64_t)e * T + t]; arg = e; }
            won[t] = best > 0;
            holder[t] = won[t] ? arg : -1;
            price[t] += best;
        }
        for (int e = 0; e < E; ++e)
            for (int t = 0; t < T; ++t) adj[(int64_t)e * T + t] = (int64_t)q[(int64_t)t * E + e] - price[t];
        for (int t = 0; t < T; ++t)
            if (won[t])
                adj[(int64_t)holder[t] * T + t] =
                    (round < max_iterations) ? RETAIN : (int64_t)q[(int64_t)t * E + holder[t]];
        ++round;
    }
    int64_t objective = 0;
    if (status == ORC_OK) {
        for (int t = 0; t < T; ++t) assign[t] = -1;
        for (int e = 0; e < E && status == ORC_OK; ++e)
            for (int j = 0; j < C; ++j) {
                const int t = best_ids[(int64_t)e * (C + 1) + j];
                if (assign[t] != -1) { status = ORC_ERR_NOT_CONVERGED; break; }
                assign[t] = e;
            }
        if (status == ORC_OK)
            for (int t = 0; t < T; ++t) objective += q[(int64_t)t * E + assign[t]];
    }
    if (price_out) for (int t = 0; t < T; ++t) price_out[t] = price[t];
    if (stats_out) {
        stats_out[0] = status;
        stats_out[1] = round;
        stats_out[2] = eps;
        stats_out[3] = objective;
    }
    free(adj); free(bids); free(price); free(won); free(holder); free(best_ids);
    free(best_vals); free(work);
    return status;
}
