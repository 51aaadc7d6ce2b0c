/*
 * CPU oracle for the decode-time MoE layer with batch-aware expert
 * re-routing.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check in
 * __graft_entry__.py and the CPU-baseline / reference leg of bench.py may
 * load this library.  The product library (libmoe_decode.so) never calls
 * it, shares no source with it and has no fallback to it.
 *
 * Everything here is a plain, slow restatement of what the layer computes,
 * in the order the definitions below state.  Build flags:
 *   -O2 -ffp-contract=off -fno-fast-math  (no silent FMA contraction; every
 *   fused multiply-add below is an explicit fmaf()).
 *
 * Sources (web pages; cited by title and section):
 *  [R]   "Router Caching and Optimization", section "Analyzing Router
 *        Inference Cost", steps 1-3: linear projection h = x W_g, softmax,
 *        top-k selection.
 *  [OEA] "Opportunistic Expert Activation: Batch-Aware Expert Routing for
 *        Faster Decode Without Retraining", abstract and lay summary: each
 *        token keeps its most important experts, then piggybacks on experts
 *        already loaded for other tokens of the batch.
 *  [XS]  "XShare: Collaborative in-Batch Expert Sharing for Faster MoE
 *        Inference", AI summary and abstract: batch expert selection as a
 *        modular optimisation (maximise the total gating score of the
 *        selected experts), solved greedily.
 *  [LX]  "Lynx: Enabling Efficient MoE Inference through Dynamic Batch-Aware
 *        Expert Selection", section 1 (latency follows the number of distinct
 *        experts the batch activates) and section 2.2 (every token keeps
 *        k expert slots).
 *  [CS]  "Channel Selection for Mixture-of-Experts Decoding Needs No
 *        Calibration Data", methodology: a channel selector is a score plus
 *        a keep rule; top-k keeps each token's highest-scoring channels;
 *        reads are counted in 32-byte sectors.
 *
 * Readings where the pages are silent (each one is also listed in the
 * design notes):
 *  - router in fp32 with a fixed summation order (canon_dot / canon_sum);
 *  - exp is our own Cody-Waite range reduction plus a degree-7 Taylor
 *    polynomial (exp_spec), so the probabilities are reproducible bit for bit;
 *  - ranking is by logit, descending, ties to the lower expert index;
 *  - OEA fills from the union of kept sets fixed before any fill, up to k
 *    slots, short sets padded with (-1, 0);
 *  - XShare scores sum each token's top-k gate probabilities, the budget is
 *    min(M, |union of top-k sets|), ties to the lower index;
 *  - Lynx affinity binning: a token's confidence is the gap between the
 *    probabilities of its two top-ranked experts; bins of width k/E,
 *    min(32, ceil(E/k)) of them; expert scores sum 2^bin over the tokens
 *    whose top-k holds the expert; the critical set is the shortest prefix
 *    of the score order (at least k long) that holds every token's rank-0
 *    expert; each token takes its first k experts inside it;
 *  - XShare's hierarchical selection for speculative batches: a request is
 *    a run of `group` consecutive tokens (its drafts); each request first
 *    picks the k experts with the largest request score (its tokens' top-k
 *    gate probabilities summed), then the batch keeps the min(budget,
 *    |picked|) picked experts with the largest batch score (the request
 *    scores of the requests that picked the expert, summed);
 *  - gate weights are renormalised over the chosen set (all modes);
 *  - the expert FFN is SwiGLU: down( silu(gate x) * (up x) ), in fp64.
 *
 * Pins: every function here is checked by tests that do not re-run it
 * (see tests/test_oracle_*.py): exp_spec against libm within 2 ulp,
 * canon_dot against an fp64 dot within the forward error bound, the routing
 * against fp64 logits + a stable sort, OEA and XShare against their defining
 * invariants and brute force over subsets, hierarchical XShare against its
 * two closed forms (one token per request, one request per batch) and brute
 * force over the subsets of both levels, affinity binning against its
 * invariants, closed forms and hand-worked cases, the FFN against a dense
 * fp64 torch restatement, the channel top-k FFN against a torch restatement
 * over the gathered channels, the dense FFN and complementarity, and its
 * sector byte count against closed forms and brute force over addresses.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_MODE_NONE 0
#define ORACLE_MODE_OEA 1
#define ORACLE_MODE_XSHARE 2
#define ORACLE_MODE_AFFINITY 3
#define ORACLE_MODE_XSHARE_HIER 4

/* ---------------------------------------------------------------- exp ---
 * exp_spec(x) for x in [-87, 0] (softmax arguments are l - max(l) <= 0).
 * Cody-Waite: x = n ln2 + r with n = rint(x log2 e) and r computed in two
 * fmaf steps from a split ln2 = LN2_HI + LN2_LO (LN2_HI holds the leading
 * 15 significant bits of ln 2, LN2_LO the float nearest the remainder);
 * exp(r) by the Taylor series to degree 7 in Horner form with fmaf;
 * scaling by 2^n by adding n to the exponent field.  Returns +0 below -87.
 */
static const float LOG2E_F = 1.44269504088896341f;
static const float LN2_HI = 0.693145751953125f;
static const float LN2_LO = 1.42860682030941723212e-6f;

static float f_from_bits(int32_t b) { float f; memcpy(&f, &b, 4); return f; }
static int32_t bits_from_f(float f) { int32_t b; memcpy(&b, &f, 4); return b; }

float oracle_exp_spec(float x)
{
    if (!(x >= -87.0f)) return 0.0f;
    float n = rintf(x * LOG2E_F);
    float r = fmaf(-n, LN2_HI, x);
    r = fmaf(-n, LN2_LO, r);
    /* Taylor coefficients 1/j!, each the float nearest the exact value */
    float p = 1.0f / 5040.0f;
    p = fmaf(p, r, 1.0f / 720.0f);
    p = fmaf(p, r, 1.0f / 120.0f);
    p = fmaf(p, r, 1.0f / 24.0f);
    p = fmaf(p, r, 1.0f / 6.0f);
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    return f_from_bits(bits_from_f(p) + ((int32_t)n << 23));
}

void oracle_exp_spec_n(const float *x, float *y, int n)
{
    for (int i = 0; i < n; ++i) y[i] = oracle_exp_spec(x[i]);
}

/* ------------------------------------------------- canonical reductions ---
 * The fp32 order both sides use.  32 partial sums ("lanes"); then a
 * butterfly: for o = 16, 8, 4, 2, 1 every lane l adds lane l^o.  All lanes
 * end equal (fp32 addition is commutative); lane 0 is the result. */
static float butterfly32(float lane[32])
{
    for (int o = 16; o >= 1; o >>= 1) {
        float nxt[32];
        for (int l = 0; l < 32; ++l) nxt[l] = lane[l] + lane[l ^ o];
        memcpy(lane, nxt, sizeof nxt);
    }
    return lane[0];
}

/* dot(a, b) over d (d % 8 == 0): lane l owns j = 256 c + 8 l + t for
 * c = 0, 1, ... and t = 0..7, accumulated with fmaf from +0 in (c, t)
 * ascending order; groups with j >= d are skipped. */
float oracle_canon_dot(const float *a, const float *b, int d)
{
    float lane[32];
    for (int l = 0; l < 32; ++l) {
        float acc = 0.0f;
        for (int c = 0; 256 * c < d; ++c) {
            int j0 = 256 * c + 8 * l;
            if (j0 >= d) continue;
            for (int t = 0; t < 8; ++t) acc = fmaf(a[j0 + t], b[j0 + t], acc);
        }
        lane[l] = acc;
    }
    return butterfly32(lane);
}

/* sum of q[0..n): lane l adds q[l + 32 i] for i ascending, from +0. */
float oracle_canon_sum(const float *q, int n)
{
    float lane[32];
    for (int l = 0; l < 32; ++l) {
        float acc = 0.0f;
        for (int e = l; e < n; e += 32) acc = acc + q[e];
        lane[l] = acc;
    }
    return butterfly32(lane);
}

/* ------------------------------------------------------------- ranking ---
 * Expert a ranks before expert b for a token iff its logit is larger, or
 * the logits are equal and a has the lower index. */
static int ranks_before(const float *l, int a, int b)
{
    return l[a] > l[b] || (l[a] == l[b] && a < b);
}

/* order[0..E) = the token's experts in rank order (insertion sort). */
static void token_order(const float *l, int E, int *order)
{
    for (int e = 0; e < E; ++e) {
        int pos = e;
        while (pos > 0 && ranks_before(l, e, order[pos - 1])) {
            order[pos] = order[pos - 1];
            --pos;
        }
        order[pos] = e;
    }
}

/* Renormalise gate weights over a chosen set: w_s = p[e_s] / sum, the sum
 * taken in fp32 over the slots in slot order from +0.  Slots with e < 0
 * get w = 0. */
static void renormalise(const float *p, const int *sel, int k, float *w)
{
    float s = 0.0f;
    for (int j = 0; j < k; ++j)
        if (sel[j] >= 0) s = s + p[sel[j]];
    for (int j = 0; j < k; ++j) w[j] = sel[j] >= 0 ? p[sel[j]] / s : 0.0f;
}

/* ------------------------------------------------------------- router ---
 * [R] steps 1-3.  logits[b][e] = canon_dot(x[b], Wg[e]) (+ bias[e]);
 * probs[b] = softmax(logits[b]) with m = max, q = exp_spec(l - m),
 * Z = canon_sum(q), p = q / Z; topk_idx[b] = the first k experts of the
 * token's rank order; topk_w[b] = their probabilities renormalised over the
 * k chosen (the same weights the NONE rule yields). */
void oracle_route(const float *x, const float *Wg, const float *bias,
                  int B, int d, int E, int k,
                  float *logits, float *probs, int *topk_idx, float *topk_w)
{
    int *order = (int *)malloc(sizeof(int) * (size_t)E);
    float *q = (float *)malloc(sizeof(float) * (size_t)E);
    for (int b = 0; b < B; ++b) {
        float *l = logits + (size_t)b * E;
        for (int e = 0; e < E; ++e) {
            float v = oracle_canon_dot(x + (size_t)b * d, Wg + (size_t)e * d, d);
            l[e] = bias ? v + bias[e] : v;
        }
        float m = l[0];
        for (int e = 1; e < E; ++e) m = l[e] > m ? l[e] : m;
        for (int e = 0; e < E; ++e) q[e] = oracle_exp_spec(l[e] - m);
        float Z = oracle_canon_sum(q, E);
        float *p = probs + (size_t)b * E;
        for (int e = 0; e < E; ++e) p[e] = q[e] / Z;
        token_order(l, E, order);
        for (int j = 0; j < k; ++j) topk_idx[(size_t)b * k + j] = order[j];
        renormalise(p, topk_idx + (size_t)b * k, k, topk_w + (size_t)b * k);
    }
    free(order);
    free(q);
}

/* ----------------------------------------------------------- reselect ---
 * sel_idx[b][0..k) and sel_w[b][0..k) for one of five rules.
 *   NONE   : the token's top-k (standard routing, [LX] section 1).
 *   OEA    : [OEA].  K_b = first k0 of the order; U_kept = union of all
 *            K_b, fixed before any fill; F_b = the first k - k0 experts of
 *            the order that lie in U_kept and not in K_b; sel = K_b ++ F_b,
 *            padded with -1 when U_kept \ K_b is short.
 *   XSHARE : [XS].  T_b = top-k; U_base = union of T_b;
 *            s_e = sum over b ascending of [e in T_b] p[b][e] (fp32, from
 *            +0); M' = min(budget, |U_base|); S = the M' experts of U_base
 *            with the largest s (ties to the lower index) -- the exact
 *            maximiser of the modular objective sum_{e in S} s_e;
 *            sel_b = the first k experts of the order that lie in S.
 *   AFFINITY : [LX] section 2.2 (confidence analyzer, adaptive expert
 *            scorer, expert remapper) and section 2.1 (rank-0 dominates).
 *            c_b = p[b][r0] - p[b][r1] (fp32), r0, r1 the token's first two
 *            experts; nb = min(32, ceil(E/k)) bins of width k/E: bin_b =
 *            the largest j < nb with j*k <= c_b*E (fp32 product);
 *            s_e = sum over b with e in T_b of 2^bin_b (exact integers);
 *            U_base ordered by s descending, ties to the lower index;
 *            M = max(k, 1 + the largest position of any r0(b) in that
 *            order); S = its first M experts; sel_b = the first k experts
 *            of the token's order that lie in S (always k of them).
 *   XSHARE_HIER : [XS] abstract (speculative decoding: hierarchical,
 *            correlation-aware selection).  Requests R_0, R_1, ... are runs
 *            of `group` consecutive tokens (the last may be shorter).
 *            Request level: s_r[e] = sum over b in R_r ascending of
 *            [e in T_b] p[b][e] (fp32, from +0); P_r = the k experts with
 *            the largest s_r > 0 (ties to the lower index).  Batch level:
 *            C = union of the P_r; s[e] = sum over r ascending with e in
 *            P_r of s_r[e] (fp32, from +0); M' = min(budget, |C|); S = the
 *            M' experts of C with the largest s (ties to the lower index);
 *            sel_b = the first k experts of the order that lie in S.
 *            group = 1 is XSHARE; one request for the whole batch is
 *            XSHARE with budget k.
 * Weights are renormalised over the chosen set in every mode. */
void oracle_reselect(const float *logits, const float *probs,
                     int B, int E, int k, int mode, int k0, int budget, int group,
                     int *sel_idx, float *sel_w)
{
    int *order = (int *)malloc(sizeof(int) * (size_t)B * E);
    for (int b = 0; b < B; ++b) token_order(logits + (size_t)b * E, E, order + (size_t)b * E);
    unsigned char *inset = (unsigned char *)calloc((size_t)E, 1);

    if (mode == ORACLE_MODE_OEA) {
        for (int b = 0; b < B; ++b)
            for (int j = 0; j < k0; ++j) inset[order[(size_t)b * E + j]] = 1;   /* U_kept */
        for (int b = 0; b < B; ++b) {
            const int *ord = order + (size_t)b * E;
            int *sel = sel_idx + (size_t)b * k;
            int n = 0;
            for (int j = 0; j < k0; ++j) sel[n++] = ord[j];
            for (int j = k0; j < E && n < k; ++j)
                if (inset[ord[j]]) sel[n++] = ord[j];
            while (n < k) sel[n++] = -1;
        }
    } else if (mode == ORACLE_MODE_XSHARE) {
        float *s = (float *)calloc((size_t)E, sizeof(float));
        unsigned char *ubase = (unsigned char *)calloc((size_t)E, 1);
        for (int b = 0; b < B; ++b)
            for (int j = 0; j < k; ++j) ubase[order[(size_t)b * E + j]] = 1;
        for (int e = 0; e < E; ++e) {
            float acc = 0.0f;
            for (int b = 0; b < B; ++b) {
                int in_tb = 0;
                for (int j = 0; j < k; ++j) in_tb |= order[(size_t)b * E + j] == e;
                if (in_tb) acc = acc + probs[(size_t)b * E + e];
            }
            s[e] = acc;
        }
        int nbase = 0;
        for (int e = 0; e < E; ++e) nbase += ubase[e];
        int Mp = budget < nbase ? budget : nbase;
        /* greedy: take the best remaining expert of U_base, M' times */
        for (int t = 0; t < Mp; ++t) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (!ubase[e] || inset[e]) continue;
                if (best < 0 || s[e] > s[best]) best = e;   /* equal s keeps the lower index */
            }
            inset[best] = 1;
        }
        for (int b = 0; b < B; ++b) {
            const int *ord = order + (size_t)b * E;
            int *sel = sel_idx + (size_t)b * k;
            int n = 0;
            for (int j = 0; j < E && n < k; ++j)
                if (inset[ord[j]]) sel[n++] = ord[j];
            while (n < k) sel[n++] = -1;
        }
        free(s);
        free(ubase);
    } else if (mode == ORACLE_MODE_XSHARE_HIER) {
        float *sr = (float *)malloc(sizeof(float) * (size_t)E);    /* request score */
        float *s = (float *)calloc((size_t)E, sizeof(float));      /* batch score */
        unsigned char *picked = (unsigned char *)malloc((size_t)E);
        unsigned char *cand = (unsigned char *)calloc((size_t)E, 1);
        int nreq = (B + group - 1) / group;
        for (int r = 0; r < nreq; ++r) {
            int b0 = r * group, b1 = b0 + group < B ? b0 + group : B;
            for (int e = 0; e < E; ++e) {
                float acc = 0.0f;
                for (int b = b0; b < b1; ++b) {
                    int in_tb = 0;
                    for (int j = 0; j < k; ++j) in_tb |= order[(size_t)b * E + j] == e;
                    if (in_tb) acc = acc + probs[(size_t)b * E + e];
                }
                sr[e] = acc;
                picked[e] = 0;
            }
            /* the request's k best experts: take the best remaining one k times */
            for (int t = 0; t < k; ++t) {
                int best = -1;
                for (int e = 0; e < E; ++e) {
                    if (picked[e] || !(sr[e] > 0.0f)) continue;
                    if (best < 0 || sr[e] > sr[best]) best = e;   /* equal scores keep the lower index */
                }
                if (best < 0) break;
                picked[best] = 1;
            }
            for (int e = 0; e < E; ++e)
                if (picked[e]) {
                    s[e] = s[e] + sr[e];
                    cand[e] = 1;
                }
        }
        int ncand = 0;
        for (int e = 0; e < E; ++e) ncand += cand[e];
        int Mp = budget < ncand ? budget : ncand;
        for (int t = 0; t < Mp; ++t) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (!cand[e] || inset[e]) continue;
                if (best < 0 || s[e] > s[best]) best = e;
            }
            inset[best] = 1;
        }
        for (int b = 0; b < B; ++b) {
            const int *ord = order + (size_t)b * E;
            int *sel = sel_idx + (size_t)b * k;
            int n = 0;
            for (int j = 0; j < E && n < k; ++j)
                if (inset[ord[j]]) sel[n++] = ord[j];
            while (n < k) sel[n++] = -1;
        }
        free(sr);
        free(s);
        free(picked);
        free(cand);
    } else if (mode == ORACLE_MODE_AFFINITY) {
        int nb = (E + k - 1) / k;
        if (nb > 32) nb = 32;
        long long *s = (long long *)calloc((size_t)E, sizeof(long long));
        unsigned char *ubase = (unsigned char *)calloc((size_t)E, 1);
        int *pos = (int *)malloc(sizeof(int) * (size_t)E);
        for (int b = 0; b < B; ++b) {
            const int *ord = order + (size_t)b * E;
            const float *p = probs + (size_t)b * E;
            float c = E > 1 ? p[ord[0]] - p[ord[1]] : p[ord[0]];
            float cE = c * (float)E;
            int bin = 0;
            for (int j = nb - 1; j > 0; --j)
                if ((float)(j * k) <= cE) { bin = j; break; }
            for (int j = 0; j < k; ++j) {
                s[ord[j]] += 1LL << bin;
                ubase[ord[j]] = 1;
            }
        }
        /* position of each expert of U_base in the score order */
        for (int e = 0; e < E; ++e) {
            pos[e] = 0;
            if (!ubase[e]) continue;
            for (int e2 = 0; e2 < E; ++e2)
                if (ubase[e2] && (s[e2] > s[e] || (s[e2] == s[e] && e2 < e))) ++pos[e];
        }
        int M = k;
        for (int b = 0; b < B; ++b) {
            int r0 = order[(size_t)b * E];
            if (pos[r0] + 1 > M) M = pos[r0] + 1;
        }
        for (int e = 0; e < E; ++e) inset[e] = ubase[e] && pos[e] < M;
        for (int b = 0; b < B; ++b) {
            const int *ord = order + (size_t)b * E;
            int *sel = sel_idx + (size_t)b * k;
            int n = 0;
            for (int j = 0; j < E && n < k; ++j)
                if (inset[ord[j]]) sel[n++] = ord[j];
            while (n < k) sel[n++] = -1;
        }
        free(s);
        free(ubase);
        free(pos);
    } else {
        for (int b = 0; b < B; ++b)
            for (int j = 0; j < k; ++j) sel_idx[(size_t)b * k + j] = order[(size_t)b * E + j];
    }
    for (int b = 0; b < B; ++b)
        renormalise(probs + (size_t)b * E, sel_idx + (size_t)b * k, k, sel_w + (size_t)b * k);
    free(inset);
    free(order);
}

/* -------------------------------------------------------------- lists ---
 * Per-expert token lists.  active = experts with at least one assignment,
 * ascending; offsets[i] = start of active[i]'s entries (offsets[n_active]
 * = total pairs); entries of one expert in ascending token order.  Unused
 * tail entries: active = -1, offsets = total, tok = -1, w = 0.
 * Returns n_active. */
int oracle_lists(const int *sel_idx, const float *sel_w, int B, int E, int k,
                 int *active, int *offsets, int *tok, float *w)
{
    int n_active = 0, pos = 0;
    for (int e = 0; e < E; ++e) {
        int start = pos;
        for (int b = 0; b < B; ++b)
            for (int j = 0; j < k; ++j)
                if (sel_idx[(size_t)b * k + j] == e) {
                    tok[pos] = b;
                    w[pos] = sel_w[(size_t)b * k + j];
                    ++pos;
                }
        if (pos > start) {
            active[n_active] = e;
            offsets[n_active] = start;
            ++n_active;
        }
    }
    for (int i = n_active; i < E; ++i) active[i] = -1;
    for (int i = n_active; i <= E; ++i) offsets[i] = pos;
    for (int i = pos; i < B * k; ++i) { tok[i] = -1; w[i] = 0.0f; }
    return n_active;
}

/* ---------------------------------------------------------------- FFN ---
 * SwiGLU expert e on token x (fp64):  g_j = sum_i x_i Wgate[e][j][i],
 * u_j = sum_i x_i Wup[e][j][i], h_j = silu(g_j) u_j with
 * silu(z) = z / (1 + exp(-z)), o_i = sum_j Wdown[e][i][j] h_j.
 * y[r] = sum over the token's slots (slot order) of w * o, for each token r
 * listed in rows[0..n_rows) (all tokens when rows == NULL).  The bf16
 * weights decode exactly to fp64.  Tokens are independent, so they may run
 * on `threads` OpenMP threads without changing any result. */
static double bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

void oracle_ffn(const float *x, const uint16_t *Wgate, const uint16_t *Wup,
                const uint16_t *Wdown, int B, int d, int E, int k, int F,
                const int *sel_idx, const float *sel_w,
                const int *rows, int n_rows, int threads, double *y)
{
    (void)E;
    int nr = rows ? n_rows : B;
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : 1)
    for (int ri = 0; ri < nr; ++ri) {
        int b = rows ? rows[ri] : ri;
        double *yo = y + (size_t)ri * d;
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        for (int i = 0; i < d; ++i) yo[i] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = sel_idx[(size_t)b * k + j];
            if (e < 0) continue;
            double wt = (double)sel_w[(size_t)b * k + j];
            const float *xb = x + (size_t)b * d;
            for (int f = 0; f < F; ++f) {
                const uint16_t *gr = Wgate + ((size_t)e * F + f) * d;
                const uint16_t *ur = Wup + ((size_t)e * F + f) * d;
                double g = 0.0, u = 0.0;
                for (int i = 0; i < d; ++i) {
                    g += (double)xb[i] * bf16_to_double(gr[i]);
                    u += (double)xb[i] * bf16_to_double(ur[i]);
                }
                h[f] = g / (1.0 + exp(-g)) * u;
            }
            for (int i = 0; i < d; ++i) {
                const uint16_t *dr = Wdown + ((size_t)e * d + i) * F;
                double o = 0.0;
                for (int f = 0; f < F; ++f) o += bf16_to_double(dr[f]) * h[f];
                yo[i] += wt * o;
            }
        }
        free(h);
    }
}

/* ------------------------------------------------- channel top-k FFN ---
 * [CS] "Channel Selection for Mixture-of-Experts Decoding Needs No
 * Calibration Data", methodology: a channel selector is a score plus a
 * keep rule, and the top-k keep rule takes each token's c highest-scoring
 * channels.  Channel f of expert e is gate row f, up row f and down column
 * f.  Only the keep rule and the sparse FFN are restated here: the scores
 * come from the caller (any selector; the page's weight-derived reader is
 * not part of this oracle).
 * For each token r listed in rows[0..n_rows) (all tokens when rows ==
 * NULL) and each slot s with e = sel_idx[b][s] >= 0:
 *   K = the c channels with the largest score[b][s][f], equal scores to
 *       the lower channel index (channel f is kept iff fewer than c
 *       channels rank before it);
 *   h_f = silu(g_f) u_f for f in K and 0 otherwise (g, u as in oracle_ffn);
 *   o_i = sum over f ascending of Wdown[e][i][f] h_f;
 *   y[r] = sum over the slots (slot order) of w o   (fp64).
 * keep[b][s][f] (B x k x F bytes, may be NULL) receives 1 for the kept
 * channels of every slot of every token (not only the listed rows), 0
 * elsewhere and for empty slots. */
void oracle_ffn_channels(const float *x, const uint16_t *Wgate, const uint16_t *Wup,
                         const uint16_t *Wdown, int B, int d, int E, int k, int F,
                         const int *sel_idx, const float *sel_w, const float *score, int c,
                         const int *rows, int n_rows, int threads, double *y,
                         unsigned char *keep)
{
    (void)E;
    unsigned char *kp = (unsigned char *)calloc((size_t)B * k * F, 1);
    for (int b = 0; b < B; ++b)
        for (int s = 0; s < k; ++s) {
            if (sel_idx[(size_t)b * k + s] < 0) continue;
            const float *sc = score + ((size_t)b * k + s) * F;
            unsigned char *m = kp + ((size_t)b * k + s) * F;
            for (int f = 0; f < F; ++f) {
                int before = 0;
                for (int f2 = 0; f2 < F; ++f2)
                    if (sc[f2] > sc[f] || (sc[f2] == sc[f] && f2 < f)) ++before;
                m[f] = before < c;
            }
        }
    if (keep) memcpy(keep, kp, (size_t)B * k * F);
    int nr = rows ? n_rows : B;
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : 1)
    for (int ri = 0; ri < nr; ++ri) {
        int b = rows ? rows[ri] : ri;
        double *yo = y + (size_t)ri * d;
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        for (int i = 0; i < d; ++i) yo[i] = 0.0;
        for (int s = 0; s < k; ++s) {
            int e = sel_idx[(size_t)b * k + s];
            if (e < 0) continue;
            double wt = (double)sel_w[(size_t)b * k + s];
            const float *xb = x + (size_t)b * d;
            const unsigned char *m = kp + ((size_t)b * k + s) * F;
            for (int f = 0; f < F; ++f) {
                h[f] = 0.0;
                if (!m[f]) continue;
                const uint16_t *gr = Wgate + ((size_t)e * F + f) * d;
                const uint16_t *ur = Wup + ((size_t)e * F + f) * d;
                double g = 0.0, u = 0.0;
                for (int i = 0; i < d; ++i) {
                    g += (double)xb[i] * bf16_to_double(gr[i]);
                    u += (double)xb[i] * bf16_to_double(ur[i]);
                }
                h[f] = g / (1.0 + exp(-g)) * u;
            }
            for (int i = 0; i < d; ++i) {
                const uint16_t *dr = Wdown + ((size_t)e * d + i) * F;
                double o = 0.0;
                for (int f = 0; f < F; ++f) o += bf16_to_double(dr[f]) * h[f];
                yo[i] += wt * o;
            }
        }
        free(h);
    }
    free(kp);
}

/* Bytes of expert weights one call reads when every activated expert reads
 * only the union of its (token, slot) pairs' kept channels, every touched
 * 32-byte sector charged in full ([CS], methodology: reads are counted in
 * 32-byte sectors).  Addresses are byte offsets from each weight array's
 * start, which is assumed 32-byte aligned.  Wgate and Wup are [E][F][d]
 * (channel f's row: 2d contiguous bytes).  Wdown is [E][d][F] (channel f's
 * column: one bf16 in each of d rows) unless down_channel_major, which
 * charges it as [E][F][d] (the column contiguous).  Returns the bytes. */
long long oracle_channel_sector_bytes(const unsigned char *keep, const int *sel_idx,
                                      int B, int E, int k, int d, int F,
                                      int down_channel_major)
{
    unsigned char *u = (unsigned char *)malloc((size_t)F);
    long long sectors = 0;
    for (int e = 0; e < E; ++e) {
        memset(u, 0, (size_t)F);
        int any = 0;
        for (int b = 0; b < B; ++b)
            for (int s = 0; s < k; ++s)
                if (sel_idx[(size_t)b * k + s] == e) {
                    const unsigned char *m = keep + ((size_t)b * k + s) * F;
                    for (int f = 0; f < F; ++f) u[f] |= m[f];
                    any = 1;
                }
        if (!any) continue;
        for (int f = 0; f < F; ++f) {
            if (!u[f]) continue;
            /* gate and up rows (and the down column when channel-major) */
            long long first = (((long long)e * F + f) * d * 2) / 32;
            long long last = ((((long long)e * F + f) * d + d) * 2 - 1) / 32;
            sectors += (down_channel_major ? 3 : 2) * (last - first + 1);
        }
        if (!down_channel_major) {
            for (int i = 0; i < d; ++i) {
                long long prev = -1;
                for (int f = 0; f < F; ++f) {
                    if (!u[f]) continue;
                    long long sec = ((((long long)e * d + i) * F + f) * 2) / 32;
                    if (sec != prev) ++sectors;   /* f ascending: sectors ascend */
                    prev = sec;
                }
            }
        }
    }
    free(u);
    return sectors * 32;
}
