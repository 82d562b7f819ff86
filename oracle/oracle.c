/*
 * oracle.c -- plain, slow, fp64 CPU reference of one draft-tree verification step
 * (EAGLE / EAGLE-2 speculative sampling).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code with the
 * CUDA path: its own input decoding, its own Philox, its own walk.
 *
 * What it computes, and where the pages define it ("EAGLE: Speculative Sampling
 * Requires Rethinking Feature Uncertainty", paperlayer.ai summary, abbreviated
 * "EAGLE summary" below):
 *
 *   O1 tree attention   (EAGLE summary, section 3 "Drafting and verification" and
 *                        "Training and verification": the target verifies the tree
 *                        in one pass with tree attention): every node i attends to
 *                        the prefix plus its own ancestors and itself, nothing else.
 *   O2 LM-head logits   (EAGLE summary, section 3 "Draft model": the LM head turns
 *                        features into token distributions): logits = hidden W^T.
 *   O3 accept/resample  (EAGLE summary, section 2 "Preliminaries": accept a drafted
 *                        token with probability min(1, p(t)/p_hat(t)); after a
 *                        rejection the rest of that draft is discarded and a token
 *                        is resampled; appendix A.2 "Multi-Round Speculative
 *                        Sampling": the rule is applied recursively over the k
 *                        candidates of a tree node, and sampling falls back to an
 *                        adjusted distribution; appendix B: Algorithm 1 takes the
 *                        target distribution, the candidates and their own
 *                        distributions and returns one sample of the target).
 *   O4 commit           (EAGLE summary, section 3 "Drafting and verification": the
 *                        accepted draft tokens extend the target's context, and
 *                        the features of the accepted tokens feed the next
 *                        drafting round): the root and the accepted nodes, in
 *                        root-to-leaf order, are appended to the prefix K/V cache
 *                        and their hidden rows gathered, as sequential decoding of
 *                        those tokens would have left the cache.
 *   O5 rerank           (EAGLE-2 blog, section 1: a draft token's confidence score
 *                        approximates the probability that the target accepts it;
 *                        section 4: after expansion, reranking keeps the tokens with
 *                        the highest acceptance probability as the target's input):
 *                        a node is reached only if its whole path is accepted, so its
 *                        value is the product of the confidences along the path; the
 *                        m highest-valued candidates form the verified tree.
 *   O6 draft children   (EAGLE summary, appendix A.1 "Tree Structure": in greedy decoding
 *                        a node's children are the top k tokens, otherwise k tokens are
 *                        sampled): the top k logits at T == 0, k independent races over
 *                        softmax(logits / T) at T > 0, each child's probability as its
 *                        confidence.
 *   O7 without replacement (the same passage, siblings kept distinct): the k smallest
 *                        clocks of one race, in order (successive draws), and the row
 *                        each sibling was drawn from (the parent's row without the
 *                        earlier siblings, renormalised).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - the adjusted distribution is norm(max(0, p - p_hat)) (standard speculative
 *     sampling residual); if its mass is 0 the previous p is kept;
 *   - candidates are tried in ascending node index; p is updated after each
 *     rejection and the next candidate is tested against the updated p;
 *   - p_hat(t) == 0 accepts (the ratio is +inf);
 *   - temperature T: p = softmax(logits / T); T == 0 is greedy argmax matching
 *     (EAGLE summary, section 4: "temperature=0"; EAGLE-2 blog, section 1: T = 0
 *     always takes the most probable token), ties to the lowest token index;
 *   - when the walk ends it emits one more token: the argmax (T == 0), or a sample
 *     of the current p -- the residual after the last rejection, else the
 *     unadjusted p at the final node;
 *   - sampling is the exponential race: argmin over v with p_v > 0 of E_v / p_v,
 *     E_v = -ln U_v, lowest v on ties;
 *   - uniforms are Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
 *     numbers: as easy as 1, 2, 3", SC'11) with key = seed and counter
 *     (v >> 2, b << 16 | purpose << 8 | node, offset_lo, offset_hi); word v & 3;
 *     U = (2 * (x >> 9) + 1) * 2^-24.  The accept test of candidate c uses
 *     (node c, v 0, purpose 0); the race at node n uses (node n, v, purpose 1); draft
 *     node f's race j (O6) uses (node f, v, purpose 2 + j), and O7's one race purpose 2.
 *
 * Parity pins live in the not-gpu tests: brute-force path attention and torch's
 * causal SDPA in float64 (O1), numpy float64 matmul (O2), brute-force argmax path
 * matching at T = 0 and chi-square tests of the emitted-token distribution, the
 * closed-form single-candidate acceptance probability and the race sampler (O3);
 * SDPA over the committed cache (O4); closed forms, value dominance and transitive
 * closure (O5); numpy argsort and scipy softmax, chi-square and independence (O6); the
 * law of successive draws, numpy renormalisation and the chi-square study of the
 * residual rule with and without each sibling's own row (O7).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_F32 0
#define ORC_BF16 1

#define ORC_OK 0
#define ORC_BAD_TREE 1
#define ORC_BAD_ARG 2

/* ------------------------------------------------------------------ input decoding */

static inline double orc_ld(const void *base, size_t i, int elem_type)
{
    if (elem_type == ORC_BF16) {
        uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float *)base)[i];
}

/* ------------------------------------------------------------------ Philox4x32-10 */

/* One Philox round: two 32x32->64 products, the high halves mixed with the other
 * two counter words and the key (Salmon et al. SC'11, section 3.2). */
static void orc_philox_round(uint32_t c[4], const uint32_t k[2])
{
    const uint64_t prod0 = (uint64_t)0xD2511F53u * c[0];
    const uint64_t prod1 = (uint64_t)0xCD9E8D57u * c[2];
    const uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
    const uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
    const uint32_t n0 = hi1 ^ c[1] ^ k[0];
    const uint32_t n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
}

void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int r = 0; r < 10; ++r) {
        if (r > 0) { /* Weyl key schedule between rounds */
            k[0] += 0x9E3779B9u;
            k[1] += 0xBB67AE85u;
        }
        orc_philox_round(c, k);
    }
    memcpy(out, c, sizeof c);
}

double orc_uniform(uint64_t seed, uint64_t offset, int32_t b, int32_t node, int32_t v,
                   int32_t purpose)
{
    const uint32_t ctr[4] = {(uint32_t)v >> 2,
                             ((uint32_t)b << 16) | ((uint32_t)purpose << 8) | (uint32_t)node,
                             (uint32_t)offset, (uint32_t)(offset >> 32)};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    orc_philox4x32_10(ctr, key, w);
    const uint32_t x = w[v & 3];
    return (2.0 * (double)(x >> 9) + 1.0) * ldexp(1.0, -24);
}

/* ------------------------------------------------------------------ tree */

/* A valid tree is topologically ordered: parent[0] = -1, 0 <= parent[i] < i. */
int orc_check_tree(int32_t N, const int32_t *parents)
{
    if (N < 1 || N > 64 || parents[0] != -1) return ORC_BAD_TREE;
    for (int i = 1; i < N; ++i)
        if (parents[i] < 0 || parents[i] >= i) return ORC_BAD_TREE;
    return ORC_OK;
}

/* ------------------------------------------------------------------ O1 attention */

/* out[b,i,h] = sum_j softmax_j(scale * q[b,i,h] . k_j) v_j, with j over the prefix
 * positions 0..L_b-1 of kv head h / (Hq/Hkv), then the tree nodes on the path from
 * node i up to the root (node i itself included). */
static void orc_attention_row(int b, int i, int h, int N, int Hq, int Hkv, int D, int Lmax,
                              int et, const void *q, const void *kp, const void *vp,
                              const int32_t *prefix_lens, const void *kt, const void *vt,
                              const int32_t *parents, double scale, double *out_row,
                              double *scores)
{
    const int G = Hq / Hkv;
    const int g = h / G;
    const int L = prefix_lens[b];
    const size_t qoff = (((size_t)b * N + i) * Hq + h) * (size_t)D;
    int path[64];
    int np = 0;
    for (int a = i; a >= 0; a = parents[(size_t)b * N + a]) path[np++] = a;

    const int nk = L + np;
    double mx = -INFINITY;
    for (int j = 0; j < nk; ++j) {
        size_t koff;
        const void *ksrc;
        if (j < L) {
            koff = (((size_t)b * Hkv + g) * Lmax + j) * (size_t)D;
            ksrc = kp;
        } else {
            koff = (((size_t)b * N + path[j - L]) * Hkv + g) * (size_t)D;
            ksrc = kt;
        }
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += orc_ld(q, qoff + d, et) * orc_ld(ksrc, koff + d, et);
        s *= scale;
        scores[j] = s;
        if (s > mx) mx = s;
    }
    double den = 0.0;
    for (int j = 0; j < nk; ++j) {
        scores[j] = exp(scores[j] - mx);
        den += scores[j];
    }
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    for (int j = 0; j < nk; ++j) {
        size_t voff;
        const void *vsrc;
        if (j < L) {
            voff = (((size_t)b * Hkv + g) * Lmax + j) * (size_t)D;
            vsrc = vp;
        } else {
            voff = (((size_t)b * N + path[j - L]) * Hkv + g) * (size_t)D;
            vsrc = vt;
        }
        const double wgt = scores[j] / den;
        for (int d = 0; d < D; ++d) out_row[d] += wgt * orc_ld(vsrc, voff + d, et);
    }
}

/* rows: n_rows triples (b, i, h); NULL means every row in [B, N, Hq] order.
 * out: [n_rows, D] (or [B*N*Hq, D]).  Returns ORC_BAD_TREE if any sequence's
 * parents are not a valid tree, ORC_BAD_ARG for bad shapes. */
int orc_tree_attention(int B, int N, int Hq, int Hkv, int D, int Lmax, int elem_type,
                       const void *q, const void *k_prefix, const void *v_prefix,
                       const int32_t *prefix_lens, const void *k_tree, const void *v_tree,
                       const int32_t *parents, double scale, int n_rows, const int32_t *rows,
                       double *out)
{
    if (B < 1 || N < 1 || N > 64 || Hq < 1 || Hkv < 1 || Hq % Hkv || D < 1 || Lmax < 0)
        return ORC_BAD_ARG;
    for (int b = 0; b < B; ++b) {
        if (orc_check_tree(N, parents + (size_t)b * N) != ORC_OK) return ORC_BAD_TREE;
        if (prefix_lens[b] < 0 || prefix_lens[b] > Lmax) return ORC_BAD_ARG;
    }
    const long total = rows ? n_rows : (long)B * N * Hq;
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)(Lmax + 64));
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < total; ++r) {
            int b, i, h;
            if (rows) {
                b = rows[3 * r];
                i = rows[3 * r + 1];
                h = rows[3 * r + 2];
            } else {
                b = (int)(r / ((long)N * Hq));
                i = (int)((r / Hq) % N);
                h = (int)(r % Hq);
            }
            orc_attention_row(b, i, h, N, Hq, Hkv, D, Lmax, elem_type, q, k_prefix, v_prefix,
                              prefix_lens, k_tree, v_tree, parents, scale,
                              out + (size_t)r * D, scores);
        }
        free(scores);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ O2 LM head */

static void orc_logits_row(int H, int V, int et, const void *hidden, const void *w, int row,
                           double *out)
{
#pragma omp parallel for schedule(static) if (!omp_in_parallel() && (long)V * H > (1L << 20))
    for (int v = 0; v < V; ++v) {
        double s = 0.0;
        const size_t ho = (size_t)row * H, wo = (size_t)v * H;
        for (int k = 0; k < H; ++k) s += orc_ld(hidden, ho + k, et) * orc_ld(w, wo + k, et);
        out[v] = s;
    }
}

/* logits[r, v] = sum_k hidden[row_r, k] * W[v, k]; rows NULL = all M rows. */
void orc_lm_head(int M, int H, int V, int elem_type, const void *hidden, const void *w,
                 int n_rows, const int32_t *rows, double *logits)
{
    const int nr = rows ? n_rows : M;
    if ((long)nr * V >= 4096 && nr > 1) {
#pragma omp parallel for collapse(2) schedule(static)
        for (int r = 0; r < nr; ++r)
            for (int v = 0; v < V; ++v) {
                const int row = rows ? rows[r] : r;
                double s = 0.0;
                const size_t ho = (size_t)row * H, wo = (size_t)v * H;
                for (int k = 0; k < H; ++k)
                    s += orc_ld(hidden, ho + k, elem_type) * orc_ld(w, wo + k, elem_type);
                logits[(size_t)r * V + v] = s;
            }
    } else {
        for (int r = 0; r < nr; ++r)
            orc_logits_row(H, V, elem_type, hidden, w, rows ? rows[r] : r,
                           logits + (size_t)r * V);
    }
}

/* ------------------------------------------------------------------ O3 accept / resample */

/* Exponential race: argmin over v with weight_v > 0 of (-ln U(b, node, v, purpose)) / weight_v,
 * lowest v on ties.  *rel_gap receives (second - best) / best, or +inf if only one
 * candidate. */
int32_t orc_race_purpose(int V, const double *weight, uint64_t seed, uint64_t offset, int32_t b,
                         int32_t node, int32_t purpose, double *rel_gap)
{
    double best = INFINITY, second = INFINITY;
    int32_t arg = -1;
    for (int v = 0; v < V; ++v) {
        if (!(weight[v] > 0.0)) continue;
        const double e = -log(orc_uniform(seed, offset, b, node, v, purpose));
        const double key = e / weight[v];
        if (key < best) {
            second = best;
            best = key;
            arg = v;
        } else if (key < second) {
            second = key;
        }
    }
    if (rel_gap) *rel_gap = (arg >= 0 && isfinite(second)) ? (second - best) / best : INFINITY;
    return arg;
}

/* The walk's sample (purpose 1). */
int32_t orc_race(int V, const double *weight, uint64_t seed, uint64_t offset, int32_t b,
                 int32_t node, double *rel_gap)
{
    return orc_race_purpose(V, weight, seed, offset, b, node, 1, rel_gap);
}

typedef struct {
    int mode; /* 0: float logits array, 1: double logits array, 2: hidden x W on demand */
    const void *logits;
    int N, V, H, elem_type;
    const void *hidden, *w;
} orc_rows_t;

static void orc_get_row(const orc_rows_t *src, int b, int node, double *row)
{
    const size_t base = ((size_t)b * src->N + node) * (size_t)src->V;
    if (src->mode == 0) {
        for (int v = 0; v < src->V; ++v) row[v] = ((const float *)src->logits)[base + v];
    } else if (src->mode == 1) {
        memcpy(row, (const double *)src->logits + base, sizeof(double) * (size_t)src->V);
    } else {
        orc_logits_row(src->H, src->V, src->elem_type, src->hidden, src->w, b * src->N + node,
                       row);
    }
}

typedef struct {
    int32_t near;       /* decisions within the margin */
    int32_t decisions;
    int32_t first_near; /* index of the first near decision, -1 if none */
    int32_t exact_len;  /* accepted nodes fixed before the first near decision */
    int32_t near_child; /* the child tested at the first near decision; -1 when that decision
                           is the final race or when there is none, -2 when it is a greedy
                           argmax (which decides both the match and the final token) */
} orc_diag_t;

/* Records one decision of the walk: `n_acc` nodes accepted so far, `child` the candidate
 * under test (-1 for the argmax or race that ends the walk). */
static void orc_note(orc_diag_t *dg, int is_near, int n_acc, int child)
{
    if (is_near) {
        if (dg->near == 0) {
            dg->first_near = dg->decisions;
            dg->exact_len = n_acc;
            dg->near_child = child;
        }
        dg->near++;
    }
    dg->decisions++;
}

/* One sequence of the multi-round speculative sampling walk.  Returns the number of
 * accepted drafted nodes (written to acc[]), or -1 for an invalid tree. */
static int orc_walk(const orc_rows_t *src, int b, int N, int V, const float *draft_b,
                    const int32_t *tokens_b, const int32_t *parents_b, double T, uint64_t seed,
                    uint64_t offset, double margin, int32_t *acc, int32_t *next_token,
                    orc_diag_t *dg, double *logit_row, double *p, double *r)
{
    if (orc_check_tree(N, parents_b) != ORC_OK) return -1;
    for (int i = 1; i < N; ++i)
        if (tokens_b[i] < 0 || tokens_b[i] >= V) return -1;

    int n_acc = 0;
    int cur = 0; /* the committed root */
    for (;;) {
        orc_get_row(src, b, cur, logit_row);
        if (T == 0.0) {
            /* greedy: the target's choice is argmax(logits), lowest index on ties */
            int m = 0;
            for (int v = 1; v < V; ++v)
                if (logit_row[v] > logit_row[m]) m = v;
            double second = -INFINITY;
            for (int v = 0; v < V; ++v)
                if (v != m && logit_row[v] > second) second = logit_row[v];
            orc_note(dg, V > 1 && logit_row[m] - second <= margin, n_acc, -2);
            int matched = -1;
            for (int c = cur + 1; c < N; ++c)
                if (parents_b[c] == cur && tokens_b[c] == m) {
                    matched = c;
                    break;
                }
            if (matched >= 0) {
                acc[n_acc++] = matched;
                cur = matched;
                continue;
            }
            *next_token = m;
            return n_acc;
        }

        /* p = softmax(logits / T) */
        double mx = -INFINITY;
        for (int v = 0; v < V; ++v)
            if (logit_row[v] / T > mx) mx = logit_row[v] / T;
        double z = 0.0;
        for (int v = 0; v < V; ++v) {
            p[v] = exp(logit_row[v] / T - mx);
            z += p[v];
        }
        for (int v = 0; v < V; ++v) p[v] /= z;

        int accepted = -1;
        for (int c = cur + 1; c < N && accepted < 0; ++c) {
            if (parents_b[c] != cur) continue;
            const int t_hat = tokens_b[c];
            const float *p_hat = draft_b + (size_t)c * V;
            const double u = orc_uniform(seed, offset, b, c, 0, 0);
            if (p_hat[t_hat] == 0.0f) {
                orc_note(dg, 0, n_acc, c);
                accepted = c;
                break;
            }
            const double ratio = p[t_hat] / (double)p_hat[t_hat];
            orc_note(dg, fabs(u - ratio) <= margin * (ratio > 1.0 ? ratio : 1.0), n_acc, c);
            if (u < ratio) {
                accepted = c;
                break;
            }
            /* rejected: p <- norm(max(0, p - p_hat)) */
            double mass = 0.0;
            for (int v = 0; v < V; ++v) {
                const double d = p[v] - (double)p_hat[v];
                r[v] = d > 0.0 ? d : 0.0;
                mass += r[v];
            }
            if (mass > 0.0)
                for (int v = 0; v < V; ++v) p[v] = r[v] / mass;
        }
        if (accepted >= 0) {
            acc[n_acc++] = accepted;
            cur = accepted;
            continue;
        }
        double gap;
        *next_token = orc_race(V, p, seed, offset, b, cur, &gap);
        orc_note(dg, gap <= margin, n_acc, -1);
        return n_acc;
    }
}

/* logits_mode 0: `logits` is float [B,N,V]; 1: double [B,N,V]; 2: rows are computed on
 * demand from hidden [B*N,H] and w [V,H] (elem_type).  Outputs: accepted_nodes [B,N]
 * (-1 padded), accept_len [B] and next_token [B] (-1 and -1 for an invalid tree);
 * diagnostics (may be NULL), per sequence: near_count, n_decisions, first_near, and for
 * the first near decision exact_len (accepted nodes fixed before it) and near_child (the
 * candidate it tested; -1 for the final race or none, -2 for a greedy argmax). */
int orc_tree_accept(int B, int N, int V, int logits_mode, const void *logits, int H,
                    int elem_type, const void *hidden, const void *w, const float *draft_probs,
                    const int32_t *tokens, const int32_t *parents, double temperature,
                    uint64_t seed, uint64_t offset, double margin, int32_t *accepted_nodes,
                    int32_t *accept_len, int32_t *next_token, int32_t *near_count,
                    int32_t *n_decisions, int32_t *first_near, int32_t *exact_len,
                    int32_t *near_child)
{
    if (B < 1 || B > 65535 || N < 1 || N > 64 || V < 1 || !(temperature >= 0.0))
        return ORC_BAD_ARG;
    const orc_rows_t src = {logits_mode, logits, N, V, H, elem_type, hidden, w};
#pragma omp parallel if (B > 16 && logits_mode != 2)
    {
        double *row = (double *)malloc(sizeof(double) * (size_t)V);
        double *p = (double *)malloc(sizeof(double) * (size_t)V);
        double *r = (double *)malloc(sizeof(double) * (size_t)V);
#pragma omp for schedule(dynamic, 64)
        for (int b = 0; b < B; ++b) {
            int32_t *acc = accepted_nodes + (size_t)b * N;
            for (int i = 0; i < N; ++i) acc[i] = -1;
            orc_diag_t dg = {0, 0, -1, 0, -1};
            int32_t nt = -1;
            const int n = orc_walk(&src, b, N, V, draft_probs + (size_t)b * N * V,
                                   tokens + (size_t)b * N, parents + (size_t)b * N,
                                   temperature, seed, offset, margin, acc, &nt, &dg, row, p, r);
            accept_len[b] = n;
            next_token[b] = n < 0 ? -1 : nt;
            if (near_count) near_count[b] = dg.near;
            if (n_decisions) n_decisions[b] = dg.decisions;
            if (first_near) first_near[b] = dg.first_near;
            if (exact_len) exact_len[b] = dg.near > 0 ? dg.exact_len : (n < 0 ? 0 : n);
            if (near_child) near_child[b] = dg.near_child;
        }
        free(row);
        free(p);
        free(r);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ O4 commit */

/* Post-accept commit of one step.  For sequence b with a = accept_len[b] >= 0 the
 * committed path is node 0 (the root: the token committed by the previous step, whose K/V
 * this step computed as a tree row) followed by accepted_nodes[b][0 .. a-1]; n = a + 1.
 * Row t of the path goes to position L_b + t of every kv head of the prefix cache
 * (k_prefix/v_prefix [B, Hkv, Lmax, D], elements of `esize` bytes, copied bit for bit)
 * and to row t of feat [B, N, H] (from hidden [B*N, H]); new_lens[b] = L_b + n.  Nothing
 * is written for the sequence and new_lens[b] is
 *   L_b  when a == -1 (the walk found the tree invalid);
 *   -1   when a is out of [-1, N-1], L_b out of [0, Lmax], L_b + n > Lmax, or the path is
 *        not a root-to-leaf chain of the tree (node t+1 a child of node t).
 * feat rows n .. N-1 and cache positions outside [L_b, L_b + n) are left as they are. */
void orc_commit(int B, int N, int Hkv, int D, int Lmax, int H, int esize,
                void *k_prefix, void *v_prefix, const int32_t *prefix_lens,
                const void *k_tree, const void *v_tree, const void *hidden,
                const int32_t *parents, const int32_t *accepted_nodes, const int32_t *accept_len,
                int32_t *new_lens, void *feat)
{
    const size_t row = (size_t)D * esize, hrow = (size_t)H * esize;
    for (int b = 0; b < B; ++b) {
        const int32_t L = prefix_lens[b], a = accept_len[b];
        const int32_t *acc = accepted_nodes + (size_t)b * N;
        const int32_t *par = parents + (size_t)b * N;
        if (a == -1) {
            new_lens[b] = L;
            continue;
        }
        int ok = a >= 0 && a <= N - 1 && L >= 0 && L <= Lmax && L + a + 1 <= Lmax;
        int path[64];
        path[0] = 0;
        for (int t = 1; ok && t <= a; ++t) {
            const int32_t c = acc[t - 1];
            ok = c >= 1 && c < N && par[c] == path[t - 1];
            path[t] = c;
        }
        if (!ok) {
            new_lens[b] = -1;
            continue;
        }
        const int n = a + 1;
        for (int t = 0; t < n; ++t) {
            const size_t node = (size_t)b * N + path[t];
            for (int g = 0; g < Hkv; ++g) {
                const size_t src = (node * Hkv + g) * row;
                const size_t dst = (((size_t)b * Hkv + g) * Lmax + L + t) * row;
                memcpy((char *)k_prefix + dst, (const char *)k_tree + src, row);
                memcpy((char *)v_prefix + dst, (const char *)v_tree + src, row);
            }
            memcpy((char *)feat + ((size_t)b * N + t) * hrow, (const char *)hidden + node * hrow, hrow);
        }
        new_lens[b] = L + n;
    }
}

/* ------------------------------------------------------------------ O5 rerank */

typedef struct {
    float value;
    int32_t index;
} orc_ranked;

/* higher value first, then lower index */
static int orc_rank_cmp(const void *a, const void *b)
{
    const orc_ranked *x = (const orc_ranked *)a, *y = (const orc_ranked *)b;
    if (x->value > y->value) return -1;
    if (x->value < y->value) return 1;
    return (x->index > y->index) - (x->index < y->index);
}

static int orc_index_cmp(const void *a, const void *b)
{
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Reranking of an expanded candidate tree (M candidates, topological: parent[0] = -1,
 * 0 <= parent[i] < i) down to the m-node tree the target verifies.
 *   confidence c_i is clamped to [0, 1] (NaN and negatives count as 0; the root's is not used);
 *   path value v_0 = 1, v_i = v_parent(i) * c_i in float32, root first (the decision is an
 *     integer one, so both sides take it in the same precision: float32);
 *   the k = min(m, M) candidates with the highest value are kept, ties to the lower index --
 *     with c <= 1 a node's value never exceeds its parent's, so the kept set contains every
 *     kept node's ancestors;
 *   they are renumbered in increasing candidate index (a topological order, root = 0):
 *     sel[t] = candidate index, parents_out[t] = new index of its parent, tokens_out[t],
 *     masks_out[t] = bit j set for every kept ancestor-or-self j (k <= 64);
 *   num_selected[b] = k, or -1 for a candidate tree that is not topological (nothing else
 *     written for that sequence).
 * Outputs are [B, m]; entries t >= k are -1 (masks 0). */
void orc_tree_rerank(int B, int M, int m, const int32_t *parents, const int32_t *tokens,
                     const float *confidence, int32_t *sel, int32_t *parents_out, int32_t *tokens_out,
                     uint64_t *masks_out, int32_t *num_selected)
{
    orc_ranked *r = malloc(sizeof(orc_ranked) * (size_t)M);
    float *v = malloc(sizeof(float) * (size_t)M);
    int32_t *keep = malloc(sizeof(int32_t) * (size_t)M);
    int32_t *newidx = malloc(sizeof(int32_t) * (size_t)M);
    for (int b = 0; b < B; ++b) {
        const int32_t *par = parents + (size_t)b * M;
        const int32_t *tok = tokens + (size_t)b * M;
        const float *c = confidence + (size_t)b * M;
        int32_t *o_sel = sel + (size_t)b * m, *o_par = parents_out + (size_t)b * m;
        int32_t *o_tok = tokens_out + (size_t)b * m;
        uint64_t *o_mask = masks_out + (size_t)b * m;
        for (int t = 0; t < m; ++t) {
            o_sel[t] = o_par[t] = o_tok[t] = -1;
            o_mask[t] = 0;
        }
        int topo = M >= 1 && par[0] == -1;
        for (int i = 1; topo && i < M; ++i) topo = par[i] >= 0 && par[i] < i;
        if (!topo) {  /* candidate trees may exceed the 64 rows of a verified tree */
            num_selected[b] = -1;
            continue;
        }
        v[0] = 1.0f;
        for (int i = 1; i < M; ++i) {
            const float ci = c[i] > 0.0f ? (c[i] < 1.0f ? c[i] : 1.0f) : 0.0f;
            v[i] = v[par[i]] * ci;
        }
        for (int i = 0; i < M; ++i) {
            r[i].value = v[i];
            r[i].index = i;
        }
        qsort(r, (size_t)M, sizeof(orc_ranked), orc_rank_cmp);
        const int k = m < M ? m : M;
        for (int t = 0; t < k; ++t) keep[t] = r[t].index;
        qsort(keep, (size_t)k, sizeof(int32_t), orc_index_cmp);
        for (int i = 0; i < M; ++i) newidx[i] = -1;
        for (int t = 0; t < k; ++t) newidx[keep[t]] = t;
        for (int t = 0; t < k; ++t) {
            const int32_t i = keep[t];
            o_sel[t] = i;
            o_par[t] = i == 0 ? -1 : newidx[par[i]];
            o_tok[t] = tok[i];
            uint64_t mask = 0;
            for (int32_t a = i; a >= 0; a = par[a]) mask |= 1ull << newidx[a];
            o_mask[t] = mask;
        }
        num_selected[b] = k;
    }
    free(r);
    free(v);
    free(keep);
    free(newidx);
}

/* ------------------------------------------------------------------ O6 draft children */

/* Children of the draft nodes (EAGLE summary, appendix A.1 "Tree Structure": in greedy
 * decoding a node's children are the top k tokens by probability, in non-greedy decoding k
 * tokens are sampled; section 3: the draft samples its next token through the LM head).
 * Row (b, f) of logits [B, F, V] (float32) is draft node f of sequence b:
 *   y = logit / T' with T' = T (T > 0) or 1 (T == 0); p = softmax(y) in float64;
 *   T == 0: tokens = the k largest logits in decreasing order, ties to the lower index;
 *   T  > 0: tokens[j] = the race over p with (node f, purpose 2 + j), j = 0..k-1: k
 *           independent samples of p;
 *   conf[j] = p[tokens[j]]; probs[v] = p_v when probs is not NULL;
 *   near[j] = 1 when the decision is within `margin`: T == 0, the chosen logit and the next
 *   one below it differ by at most margin * max(1, |logit|); T > 0, the race's best and
 *   second keys are within margin (relative).
 * Outputs are [B, F, k] (probs [B, F, V]). */
void orc_draft_select(int B, int F, int V, int k, const float *logits, double T, uint64_t seed,
                      uint64_t offset, double margin, int32_t *tokens, double *conf, double *probs,
                      int32_t *near)
{
    double *p = malloc(sizeof(double) * (size_t)V);
    const double Tp = T > 0.0 ? T : 1.0;
    for (int b = 0; b < B; ++b) {
        for (int f = 0; f < F; ++f) {
            const size_t r = (size_t)b * F + f;
            const float *l = logits + r * V;
            double m = -INFINITY;
            for (int v = 0; v < V; ++v) m = fmax(m, (double)l[v] / Tp);
            double z = 0.0;
            for (int v = 0; v < V; ++v) z += exp((double)l[v] / Tp - m);
            for (int v = 0; v < V; ++v) p[v] = exp((double)l[v] / Tp - m) / z;
            if (probs) memcpy(probs + r * V, p, sizeof(double) * (size_t)V);
            int32_t *tok = tokens + r * k;
            for (int j = 0; j < k; ++j) {
                int32_t arg = -1;
                int is_near = 0;
                if (T > 0.0) {
                    double gap;
                    arg = orc_race_purpose(V, p, seed, offset, b, f, 2 + j, &gap);
                    is_near = gap <= margin;
                } else {
                    /* the best logit not taken yet: strictly below the previous pick in
                     * (value descending, index ascending) order */
                    for (int v = 0; v < V; ++v) {
                        if (l[v] != l[v]) continue; /* NaN is never a child */
                        if (j > 0) {
                            const float pv = l[tok[j - 1]];
                            if (!(l[v] < pv || (l[v] == pv && v > tok[j - 1]))) continue;
                        }
                        if (arg < 0 || l[v] > l[arg]) arg = v;
                    }
                    if (arg >= 0) {
                        /* next value below the pick, for the margin */
                        double nextv = -INFINITY;
                        for (int v = 0; v < V; ++v)
                            if (v != arg && (l[v] < l[arg] || (l[v] == l[arg] && v > arg)))
                                nextv = fmax(nextv, l[v]);
                        is_near = (double)l[arg] - nextv <= margin * fmax(1.0, fabs((double)l[arg]));
                    }
                }
                tok[j] = arg;
                conf[r * k + j] = arg >= 0 ? p[arg] : 0.0;
                if (near) near[r * k + j] = is_near;
            }
        }
    }
    free(p);
}

/* O7: siblings drawn without replacement (EAGLE summary, appendix A.1 "Tree Structure": k
 * tokens are sampled for a node's children; sampling them without replacement keeps the
 * siblings distinct).  Row (b, f) as in O6, p = softmax(logits / T') in float64:
 *   T == 0: the k largest logits (as O6: distinct by construction);
 *   T  > 0: the k smallest clocks E_v / p_v, E_v = -ln U(b, f, v, purpose 2), in increasing
 *           order, over the tokens with p_v > 0 (fewer than k such tokens: -1 after them).
 *           The clocks of independent exponentials come out in the order of successive draws
 *           without replacement: the first is a draw from p, each later one a draw from p
 *           restricted to the tokens not drawn yet.
 *   conf[j] = p[tokens[j]]; probs = p when not NULL;
 *   near[j] = 1 when clock j is within `margin` (relative) of clock j + 1 or of clock j - 1
 *   (T == 0: O6's rule). */
static int orc_cmp_clock(const void *a, const void *b)
{
    const double *x = (const double *)a, *y = (const double *)b;
    if (x[0] < y[0]) return -1;
    if (x[0] > y[0]) return 1;
    return x[1] < y[1] ? -1 : (x[1] > y[1] ? 1 : 0);
}

void orc_draft_select_distinct(int B, int F, int V, int k, const float *logits, double T,
                               uint64_t seed, uint64_t offset, double margin, int32_t *tokens,
                               double *conf, double *probs, int32_t *near)
{
    if (!(T > 0.0)) {
        orc_draft_select(B, F, V, k, logits, T, seed, offset, margin, tokens, conf, probs, near);
        return;
    }
    double *p = malloc(sizeof(double) * (size_t)V);
    double *clk = malloc(sizeof(double) * 2 * (size_t)V); /* (clock, token) pairs */
    for (int b = 0; b < B; ++b) {
        for (int f = 0; f < F; ++f) {
            const size_t r = (size_t)b * F + f;
            const float *l = logits + r * V;
            double m = -INFINITY;
            for (int v = 0; v < V; ++v) m = fmax(m, (double)l[v] / T);
            double z = 0.0;
            for (int v = 0; v < V; ++v) z += exp((double)l[v] / T - m);
            for (int v = 0; v < V; ++v) p[v] = exp((double)l[v] / T - m) / z;
            if (probs) memcpy(probs + r * V, p, sizeof(double) * (size_t)V);
            int n = 0;
            for (int v = 0; v < V; ++v) {
                if (!(p[v] > 0.0)) continue;
                clk[2 * n] = -log(orc_uniform(seed, offset, b, f, v, 2)) / p[v];
                clk[2 * n + 1] = v;
                ++n;
            }
            qsort(clk, (size_t)n, 2 * sizeof(double), orc_cmp_clock);
            for (int j = 0; j < k; ++j) {
                const int have = j < n;
                tokens[r * k + j] = have ? (int32_t)clk[2 * j + 1] : -1;
                conf[r * k + j] = have ? p[(int)clk[2 * j + 1]] : 0.0;
                if (near) {
                    int is_near = 0;
                    if (have && j + 1 < n) is_near |= (clk[2 * j + 2] - clk[2 * j]) <= margin * clk[2 * j];
                    if (have && j > 0) is_near |= (clk[2 * j] - clk[2 * j - 2]) <= margin * clk[2 * j - 2];
                    near[r * k + j] = is_near;
                }
            }
        }
    }
    free(clk);
    free(p);
}

/* O7: the row each sibling was drawn from.  Child j of row (b, f) was drawn from p with the
 * earlier siblings' tokens removed, so its row is
 *   q_j(v) = p_v / R_j for v not in {t_0 .. t_{j-1}}, 0 otherwise,  R_j = the sum of p over
 *   the tokens not removed (summed directly, not as 1 minus the removed mass);
 * q_0 = p, and a row with R_j = 0 (or a token -1 before it) is all zeros.  probs [B, F, V],
 * tokens [B, F, k] -> child [B, F, k, V], float64. */
void orc_draft_child_rows(int B, int F, int V, int k, const double *probs, const int32_t *tokens,
                          double *child)
{
    unsigned char *gone = malloc((size_t)V);
    for (size_t r = 0; r < (size_t)B * F; ++r) {
        const double *p = probs + r * V;
        memset(gone, 0, (size_t)V);
        int dead = 0;
        for (int j = 0; j < k; ++j) {
            double *q = child + (r * k + j) * V;
            double R = 0.0;
            if (!dead)
                for (int v = 0; v < V; ++v)
                    if (!gone[v]) R += p[v];
            for (int v = 0; v < V; ++v) q[v] = (!dead && !gone[v] && R > 0.0) ? p[v] / R : 0.0;
            const int32_t t = tokens[r * k + j];
            if (t < 0 || t >= V) dead = 1;
            else gone[t] = 1;
        }
    }
    free(gone);
}

/* Uniforms U(b, node, v, purpose) for v = 0..n-1 (test helper for the generator pins). */
void orc_fill_uniforms(uint64_t seed, uint64_t offset, int32_t b, int32_t node, int32_t purpose,
                       int32_t n, double *out)
{
    for (int32_t v = 0; v < n; ++v) out[v] = orc_uniform(seed, offset, b, node, v, purpose);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
