/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle for the MoE
 * routing hot path (router, dispatch, gather, combine).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (libmr.so and its Python binding) never calls, links or imports it, and it
 * shares no code, header, table or helper with the CUDA sources.
 *
 * Arithmetic is IEEE binary64 throughout.  Every top-k is a full sort with an
 * explicit (value desc, index asc) comparator; nothing is blocked, fused or
 * reordered beyond the definition.  Tokens are independent, so the per-token
 * loop may run on several host threads (OpenMP); each token's arithmetic is
 * identical whatever the thread count.
 *
 * Sources (the pages this restates):
 *  [K2-norm]  Kimi K2 "Normalize weights" page: normalisation formula and the
 *             HF MoEGate.forward excerpt (modeling_deepseek.py 423-474).
 *  [K2-add]   Kimi K2 "Add shared output" page: DeepseekV3MoE.forward and
 *             moe_infer excerpts (modeling_deepseek.py 523-533, 536-609).
 *  [V32-norm] DeepSeek-V3.2-Exp "Normalize weights" page: Gate.forward
 *             excerpt (inference/model.py 687-709).
 *  [V3-note]  DeepSeek-V3 "MoE Router" study note: affinity equation,
 *             unbiased top-K_r and renormalisation, bias, grouped routing,
 *             route_scale, official config.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define MO_OK 0
#define MO_ERR_ARG -1
#define MO_ERR_RANGE -2

/* ------------------------------------------------------------------ */
/* (value, index) pairs ordered by value descending, then index ascending:
 * the ordering every top-k below uses (lowest index wins a tie). */
typedef struct {
    double v;
    int i;
} mo_pair;

static int mo_cmp_desc(const void *pa, const void *pb)
{
    const mo_pair *a = (const mo_pair *)pa, *b = (const mo_pair *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

static int mo_cmp_double_desc(const void *pa, const void *pb)
{
    double a = *(const double *)pa, b = *(const double *)pb;
    return (a < b) - (a > b);
}

/* ------------------------------------------------------------------ */
/* Router, one token.
 *
 * logits  L_i = u_t . e_i in fp64 over the fp32 operands, no Linear bias
 *         ([K2-norm] F.linear on float32 operands; [V32-norm] linear;
 *         [V3-note] affinity equation, "no Linear bias").
 * scores  s_i = sigmoid(L_i) ([K2-norm] scores = logits.sigmoid();
 *         [V3-note] s_{i,t} = Sigmoid(u_t^T e_i)).
 * choice  c_i = s_i + b_i, used for selection only ([K2-norm]
 *         scores_for_choice; [V32-norm] original_scores kept; [V3-note]
 *         load-balance bias leaves s untouched).
 * groups  when n_group > 1: group score = sum of the two largest c in the
 *         group, keep the topk_group best groups, masked c := -inf
 *         (mask_mode 0, [V32-norm] masked_fill_ -inf, [V3-note]) or 0.0
 *         (mask_mode 1, [K2-norm] masked_fill 0.0).  With one group the step
 *         is skipped ([V32-norm] "if self.n_groups > 1"); it is a no-op then.
 * top-k   the k largest masked c ([K2-norm], [V32-norm] topk), canonical
 *         order value-desc / index-asc.
 * weights w_j = route_scale * s_{idx_j} / (sum_j s_{idx_j} + 1e-20)
 *         (unbiased s gathered: [K2-norm] scores.gather; normalise and scale:
 *         [K2-norm] formula G_i, "denominator ... + 1e-20",
 *         routed_scaling_factor; [V3-note] renormalisation, route_scale).
 *
 * margins[0] = m_(k) - m_(k+1) over the masked vector (+inf if the (k+1)-th
 *              is -inf or absent): the selection margin.
 * margins[1] = gs_(Gk) - gs_(Gk+1) (+inf when every group is kept).
 * margins[2] = smallest gap between consecutive selected masked scores
 *              (+inf for k = 1): decides the order of the k slots.
 */
/* Scoring variants of the DeepSeek-V3.2-Exp "Normalize weights" page
 * (Gate.forward): softmax scores over all N_r experts, which are then used as
 * weights without renormalisation; the group score as the group's largest
 * biased score (the page's choice when there is no bias); renormalisation
 * without the 1e-20 of the Kimi K2 code. */
typedef struct {
    int softmax;    /* 0: s = sigmoid(L); 1: s = softmax(L), weights not renormalised */
    int group_max;  /* 0: group score = sum of the two largest; 1: the largest */
    int eps;        /* 1: renormalise by sum + 1e-20 (Kimi K2); 0: by the sum */
} mo_variant;

static void mo_router_token(const float *xt, const float *W, const float *bias,
                            int d, int N_r, int n_group, int topk_group, int k,
                            double route_scale, int mask_mode, mo_variant var,
                            int32_t *idx, double *w, double *logits, double *margins,
                            double *L, double *s, double *m, mo_pair *ord,
                            double *tmp, mo_pair *gord, double *gs)
{
    const int S = N_r / n_group;
    for (int i = 0; i < N_r; ++i) {
        const float *wi = W + (size_t)i * d;
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += (double)xt[j] * (double)wi[j];
        L[i] = acc;
        if (!var.softmax)
            s[i] = 1.0 / (1.0 + exp(-acc));
        if (logits) logits[i] = acc;
    }
    if (var.softmax) {
        /* softmax over all experts, shifted by the largest logit */
        double mx = L[0], sum = 0.0;
        for (int i = 1; i < N_r; ++i)
            if (L[i] > mx) mx = L[i];
        for (int i = 0; i < N_r; ++i)
            sum += exp(L[i] - mx);
        for (int i = 0; i < N_r; ++i)
            s[i] = exp(L[i] - mx) / sum;
    }
    for (int i = 0; i < N_r; ++i)
        m[i] = s[i] + (bias ? (double)bias[i] : 0.0);

    double m_grp = INFINITY;
    if (n_group > 1) {
        for (int g = 0; g < n_group; ++g) {
            memcpy(tmp, m + (size_t)g * S, sizeof(double) * S);
            qsort(tmp, S, sizeof(double), mo_cmp_double_desc);
            if (var.group_max)
                gs[g] = tmp[0];
            else
                gs[g] = tmp[0] + tmp[1];
            gord[g].v = gs[g];
            gord[g].i = g;
        }
        qsort(gord, n_group, sizeof(mo_pair), mo_cmp_desc);
        if (topk_group < n_group)
            m_grp = gord[topk_group - 1].v - gord[topk_group].v;
        for (int r = topk_group; r < n_group; ++r) {
            const int g = gord[r].i;
            for (int i = g * S; i < (g + 1) * S; ++i)
                m[i] = (mask_mode == 0) ? -INFINITY : 0.0;
        }
    }

    for (int i = 0; i < N_r; ++i) {
        ord[i].v = m[i];
        ord[i].i = i;
    }
    qsort(ord, N_r, sizeof(mo_pair), mo_cmp_desc);

    double den = 0.0;
    for (int j = 0; j < k; ++j) {
        idx[j] = ord[j].i;
        den += s[ord[j].i];
    }
    if (var.eps)
        den += 1e-20;
    for (int j = 0; j < k; ++j) {
        if (var.softmax)
            w[j] = route_scale * s[ord[j].i];  /* softmax: not renormalised */
        else
            w[j] = route_scale * (s[ord[j].i] / den);
    }

    if (margins) {
        double m_tok = INFINITY;
        if (k < N_r && ord[k].v != -INFINITY)
            m_tok = ord[k - 1].v - ord[k].v;
        double m_ord = INFINITY;
        for (int j = 0; j + 1 < k; ++j) {
            double gap = ord[j].v - ord[j + 1].v;
            if (gap < m_ord) m_ord = gap;
        }
        margins[0] = m_tok;
        margins[1] = m_grp;
        margins[2] = m_ord;
    }
}

int mo_router2(const float *x, const float *W, const float *bias, int T, int d,
               int N_r, int n_group, int topk_group, int k, double route_scale,
               int mask_mode, int softmax, int group_max, int eps, int32_t *idx,
               double *w, double *logits, double *margins, int nthreads)
{
    const mo_variant var = {softmax != 0, group_max != 0, eps != 0};
    if (T < 0 || d <= 0 || N_r <= 0 || n_group <= 0 || N_r % n_group != 0 ||
        topk_group <= 0 || topk_group > n_group || k <= 0 || k > N_r ||
        (n_group > 1 && N_r / n_group < 2) || (mask_mode != 0 && mask_mode != 1) ||
        (mask_mode == 0 && n_group > 1 && k > topk_group * (N_r / n_group)))
        return MO_ERR_ARG;
    if (T == 0) return MO_OK;
    if (!x || !W || !idx || !w) return MO_ERR_ARG;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads) reduction(| : bad)
#endif
    {
        const int S = N_r / n_group;
        double *L = malloc(sizeof(double) * N_r);
        double *s = malloc(sizeof(double) * N_r);
        double *m = malloc(sizeof(double) * N_r);
        double *tmp = malloc(sizeof(double) * (S > 2 ? S : 2));
        double *gs = malloc(sizeof(double) * n_group);
        mo_pair *ord = malloc(sizeof(mo_pair) * N_r);
        mo_pair *gord = malloc(sizeof(mo_pair) * n_group);
        if (!L || !s || !m || !tmp || !gs || !ord || !gord) {
            bad = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
            for (int t = 0; t < T; ++t)
                mo_router_token(x + (size_t)t * d, W, bias, d, N_r, n_group,
                                topk_group, k, route_scale, mask_mode, var,
                                idx + (size_t)t * k, w + (size_t)t * k,
                                logits ? logits + (size_t)t * N_r : NULL,
                                margins ? margins + (size_t)t * 3 : NULL, L, s,
                                m, ord, tmp, gord, gs);
        }
        free(L); free(s); free(m); free(tmp); free(gs); free(ord); free(gord);
    }
    (void)nthreads;
    return bad ? MO_ERR_ARG : MO_OK;
}

/* The Kimi K2 / DeepSeek-V3 gate: sigmoid scores, top-2 group sums,
 * renormalisation with + 1e-20. */
int mo_router(const float *x, const float *W, const float *bias, int T, int d,
              int N_r, int n_group, int topk_group, int k, double route_scale,
              int mask_mode, int32_t *idx, double *w, double *logits,
              double *margins, int nthreads)
{
    return mo_router2(x, W, bias, T, d, N_r, n_group, topk_group, k, route_scale,
                      mask_mode, 0, 0, 1, idx, w, logits, margins, nthreads);
}

/* ------------------------------------------------------------------ */
/* Dispatch ([K2-add] moe_infer): tokens_per_expert from a one-hot count,
 * idxs = argsort(topk_ids.view(-1)) read as a STABLE argsort (equal expert
 * ids keep ascending flat slot order), and the inverse permutation that the
 * scatter-back new_x[idxs] = outs implies.  offsets[e] is the running
 * start_idx of expert e's slice; offsets[N_r] = T*k. */
typedef struct {
    int32_t key;  /* expert id */
    int32_t slot; /* flat slot id t*k + j */
} mo_slot;

static int mo_cmp_slot(const void *pa, const void *pb)
{
    const mo_slot *a = (const mo_slot *)pa, *b = (const mo_slot *)pb;
    if (a->key != b->key) return (a->key > b->key) - (a->key < b->key);
    return (a->slot > b->slot) - (a->slot < b->slot);
}

int mo_dispatch(const int32_t *idx, int T, int k, int N_r, int32_t *counts,
                int32_t *offsets, int32_t *perm, int32_t *inv)
{
    if (T < 0 || k <= 0 || N_r <= 0 || !counts || !offsets) return MO_ERR_ARG;
    const long n = (long)T * k;
    for (int e = 0; e < N_r; ++e) counts[e] = 0;
    for (long i = 0; i < n; ++i) {
        if (idx[i] < 0 || idx[i] >= N_r) return MO_ERR_RANGE;
        counts[idx[i]] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < N_r; ++e) offsets[e + 1] = offsets[e] + counts[e];
    if (n == 0) return MO_OK;
    if (!perm) return MO_ERR_ARG;
    mo_slot *sl = malloc(sizeof(mo_slot) * (size_t)n);
    if (!sl) return MO_ERR_ARG;
    for (long i = 0; i < n; ++i) {
        sl[i].key = idx[i];
        sl[i].slot = (int32_t)i;
    }
    qsort(sl, (size_t)n, sizeof(mo_slot), mo_cmp_slot);
    for (long i = 0; i < n; ++i) perm[i] = sl[i].slot;
    free(sl);
    if (inv)
        for (long i = 0; i < n; ++i) inv[perm[i]] = (int32_t)i;
    return MO_OK;
}

/* ------------------------------------------------------------------ */
/* Gather ([K2-add] sorted_tokens = x[idxs // k]): output row r is the token
 * row perm[rows[r]] / k of x, copied byte for byte (rows == NULL: r itself). */
int mo_gather(const void *x, long row_bytes, int T, int k, const int32_t *perm,
              const int32_t *rows, long n_rows, void *out)
{
    if (row_bytes <= 0 || k <= 0 || T < 0) return MO_ERR_ARG;
    for (long r = 0; r < n_rows; ++r) {
        long slot = rows ? rows[r] : r;
        if (slot < 0 || slot >= (long)T * k) return MO_ERR_RANGE;
        long tok = perm[slot] / k;
        if (perm[slot] < 0 || tok >= T) return MO_ERR_RANGE;
        memcpy((char *)out + r * row_bytes, (const char *)x + tok * row_bytes,
               (size_t)row_bytes);
    }
    return MO_OK;
}

/* ------------------------------------------------------------------ */
/* bf16 round-to-nearest-even of a binary64 value, written from the format's
 * definition: 8 significant bits, exponent range of binary32, subnormal
 * spacing 2^-133, overflow to infinity.  Returns the rounded value (exactly
 * representable in binary32 and binary64). */
double mo_round_bf16(double v)
{
    if (v == 0.0 || isnan(v) || isinf(v)) return v;
    int e;
    double f = frexp(fabs(v), &e);      /* |v| = f * 2^e, f in [0.5, 1) */
    int q = e - 8;                      /* spacing of 8-bit significands */
    if (q < -133) q = -133;             /* subnormal range */
    double r = nearbyint(ldexp(fabs(v), -q)); /* default mode: ties to even */
    double out = ldexp(r, q);
    const double max_bf16 = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
    if (out > max_bf16) out = INFINITY;
    (void)f;
    return v < 0 ? -out : out;
}

void mo_round_bf16_array(const double *in, long n, double *out)
{
    for (long i = 0; i < n; ++i) out[i] = mo_round_bf16(in[i]);
}

static double mo_load(const void *base, int dtype, long i)
{
    if (dtype == 0) return (double)((const float *)base)[i];
    uint32_t u = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Combine ([K2-add] scatter back new_x[idxs] = outs, then
 * view(T,k,d) * topk_weight summed over k and cast back to the row dtype;
 * DeepseekV3MoE.forward: y = y + shared_experts(identity); "Add shared
 * output" formula Delta_ffn = y_routed + y_shared).
 *
 * For token tokens[r] (r itself when tokens == NULL):
 *   acc      = sum_j w[t,j] * E[inv[t*k+j]]            (binary64)
 *   routed   = round_to_row_dtype(acc)
 *   y        = round_to_row_dtype(routed + shared[t])   (shared may be NULL)
 * Row dtype 0 = fp32 (no rounding: the oracle keeps the exact value),
 * 1 = bf16 (round to nearest even, as the two casts to the row dtype do). */
int mo_combine(const void *E, int dtype, const float *w, const int32_t *inv,
               const void *shared, int T, int d, int k, const int32_t *tokens,
               long n_tok, double *y_out, double *routed_out, int nthreads)
{
    if (d <= 0 || k <= 0 || T < 0 || (dtype != 0 && dtype != 1)) return MO_ERR_ARG;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 4) reduction(| : bad)
#endif
    for (long r = 0; r < n_tok; ++r) {
        long t = tokens ? tokens[r] : r;
        if (t < 0 || t >= T) { bad = 1; continue; }
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                long row = inv[t * k + j];
                acc += (double)w[t * k + j] * mo_load(E, dtype, row * d + c);
            }
            double routed = dtype == 1 ? mo_round_bf16(acc) : acc;
            double y = routed;
            if (shared) {
                y = routed + mo_load(shared, dtype, t * d + c);
                if (dtype == 1) y = mo_round_bf16(y);
            }
            y_out[r * d + c] = y;
            if (routed_out) routed_out[r * d + c] = routed;
        }
    }
    (void)nthreads;
    return bad ? MO_ERR_RANGE : MO_OK;
}

/* ------------------------------------------------------------------ */
/* Expert-parallel exchange ([K2-add] moe_infer, the ep_size > 1 branch).
 * ep ranks; rank r owns the experts [r*E_loc, (r+1)*E_loc), E_loc = N_r/ep
 * (tokens_per_expert.view(ep_size, -1)).
 *
 * mo_ep_splits: the bookkeeping of rank r, given every rank's
 * tokens_per_expert (counts_all [ep][N_r]):
 *   send_splits[s]    rows rank r sends to rank s (tokens_per_ep_rank:
 *                     the sum of its counts over s's experts);
 *   recv_counts[s][e] what all_to_all_single(tokens_per_expert) delivers to
 *                     rank r: source s's count for r's local expert e
 *                     (tokens_per_expert_group, viewed [ep][E_loc]);
 *   recv_splits[s]    rows rank r receives from s (output_splits: the row
 *                     sums of recv_counts). */
int mo_ep_splits(const int32_t *counts_all, int ep, int N_r, int r, int32_t *send_splits,
                 int32_t *recv_counts, int32_t *recv_splits)
{
    if (ep <= 0 || N_r <= 0 || N_r % ep != 0 || r < 0 || r >= ep) return MO_ERR_ARG;
    const int E_loc = N_r / ep;
    for (int s = 0; s < ep; ++s) {
        long send = 0, recv = 0;
        for (int e = 0; e < E_loc; ++e) {
            send += counts_all[(long)r * N_r + (long)s * E_loc + e];
            const int32_t c = counts_all[(long)s * N_r + (long)r * E_loc + e];
            recv_counts[(long)s * E_loc + e] = c;
            recv += c;
        }
        send_splits[s] = (int32_t)send;
        recv_splits[s] = (int32_t)recv;
    }
    return MO_OK;
}

/* mo_ep_recv_order: the received rows arrive source by source, and within a
 * source in its expert-sorted order; the page labels every received row
 * with its local expert (gatherd_idxs[s..s+k] = i % experts_per_rank over
 * the (source, expert) segments of tokens_per_expert_group, in that order)
 * and argsorts the labels.  The argsort is taken stable (equal labels keep
 * arrival order: by source, then the source's order), the reading used for
 * every argsort of the path.  order[j] = the received row that goes j-th
 * (sorted_tokens = gathered_tokens[order]); local_counts[e] =
 * tokens_per_expert_post_gather (the column sums of recv_counts). */
int mo_ep_recv_order(const int32_t *recv_counts, int ep, int E_loc, int32_t *order,
                     int32_t *local_counts)
{
    if (ep <= 0 || E_loc <= 0) return MO_ERR_ARG;
    long R = 0;
    for (long i = 0; i < (long)ep * E_loc; ++i) {
        if (recv_counts[i] < 0) return MO_ERR_RANGE;
        R += recv_counts[i];
    }
    for (int e = 0; e < E_loc; ++e) local_counts[e] = 0;
    mo_slot *sl = R > 0 ? malloc(sizeof(mo_slot) * (size_t)R) : NULL;
    if (R > 0 && !sl) return MO_ERR_ARG;
    long pos = 0;
    for (long seg = 0; seg < (long)ep * E_loc; ++seg) {
        const int label = (int)(seg % E_loc);
        for (int32_t c = 0; c < recv_counts[seg]; ++c, ++pos) {
            sl[pos].key = label;
            sl[pos].slot = (int32_t)pos;
        }
        local_counts[label] += recv_counts[seg];
    }
    if (R > 0) qsort(sl, (size_t)R, sizeof(mo_slot), mo_cmp_slot);
    for (long j = 0; j < R; ++j) order[j] = sl[j].slot;
    free(sl);
    return MO_OK;
}

/* ------------------------------------------------------------------ */
/* One expert layer on the expert-sorted rows ([K2-add] moe_infer: for each
 * expert i, expert_out = expert(sorted_tokens[start_idx:end_idx])), the
 * expert being one linear map with synthetic weights: the sorted row j
 * (token perm[j] / k, expert e with offsets[e] <= j < offsets[e+1]) gives
 * out[j][n] = sum_c x[token][c] * W[e][n][c], in binary64 from the bf16
 * values of x [T][d] and W [N_r][n_out][d] (bf16 bit patterns).  rows
 * selects a subset of sorted rows (NULL: all offsets[N_r]); out is
 * [n_rows][n_out].  The dot products are plain sequential loops. */
int mo_expert_gemm(const uint16_t *x, int T, int d, int k, const int32_t *perm,
                   const int32_t *offsets, int N_r, const uint16_t *W, int n_out,
                   const int32_t *rows, long n_rows, double *out, int nthreads)
{
    if (T < 0 || d <= 0 || k <= 0 || N_r <= 0 || n_out <= 0) return MO_ERR_ARG;
    const long total = offsets[N_r];
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
#endif
    for (long r = 0; r < n_rows; ++r) {
        const long j = rows ? rows[r] : r;
        if (j < 0 || j >= total || perm[j] < 0 || perm[j] / k >= T) {
            bad = 1;
            continue;
        }
        int e = 0;
        while (offsets[e + 1] <= j) ++e;  /* the expert whose segment holds j */
        const long tok = perm[j] / k;
        for (int n = 0; n < n_out; ++n) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += mo_load(x, 1, tok * d + c) * mo_load(W, 1, ((long)e * n_out + n) * d + c);
            out[r * n_out + n] = acc;
        }
    }
    (void)nthreads;
    return bad ? MO_ERR_RANGE : MO_OK;
}

int mo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
