/*
 * h2o_oracle.c -- fp64 CPU oracle of one chunked H2O sparse-attention step.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library and
 * its Python binding) may include, link or call this file. Only the tests,
 * the smoke check and the CPU-baseline leg of the benchmark use it. It shares
 * no code, header, table or constant with the CUDA path.
 *
 * What it computes follows "Learning how to Forget: Fine-tuning for
 * Long-Context Sparse Attention" (arXiv 2608.19920), as summarised on its
 * paper page (m.montaan.com/papers/2608.19920):
 *   - section "Improvements to Heavy-Hitter Oracle (H2O)": a slot's H2O score
 *     accumulates the attention weights the slot receives, and new content is
 *     written by overwriting the slots with the smallest scores;
 *   - section "Kernel Support Needs": the score increment is the sum over
 *     query rows i of the softmax weights w[b,h,i,j], and keys are masked by
 *     position, (b,h,i,j) -> -inf * I[P + i < t(b,h,j)].
 * Readings where the pages are silent (all stated, none invented here):
 *   - softmax scale 1/sqrt(d); GQA: query head h reads KV head h / G;
 *   - the score of a KV slot sums the weights from all G query heads of its
 *     group;
 *   - eviction candidates are the valid cache slots plus the T chunk tokens;
 *     the C largest survive under (score desc, position desc); scores are
 *     updated with this step's weights before selecting;
 *   - kept cache entries stay in their slots; the kept chunk tokens, in
 *     ascending position, fill the free slots (empty or evicted) in ascending
 *     slot order.
 * Eviction policies (the ranking key; the stored score is phi in both):
 *   - sum (policy 0): phi itself;
 *   - normalized (policy 1), the same section's improved score: phi divided
 *     by the candidate's age, (t - t_j)^-1 * phi, read with t = P + T the
 *     token count after the step and t_j the candidate's position, so every
 *     age is at least 1 (the page's superscript is garbled; this is the
 *     plainest reading).
 *
 * h2o_oracle_step_insert is the insert-always variant of the same section
 * (evict before the chunk attends, every chunk token enters; see there).
 * h2o_oracle_backward is the gradient of the chunk SDPA with the kept set
 * fixed (the paper's fine-tuning trains through the sparse cache; the
 * eviction itself is replayed, not differentiated).
 *
 * Everything is fp64, plain loops, exp()/log() from libm. OpenMP only splits
 * independent (batch, KV head) groups or independent query rows; no result
 * depends on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_OOM (-3)

/* ------------------------------------------------------------------------ */
/* Candidate ordering for eviction: larger score first, and for equal scores
 * the larger (more recent) position first. Positions are unique, so this is a
 * strict total order. Returns 1 when candidate a ranks above candidate b. */
static int ranks_above(double score_a, int64_t pos_a, double score_b, int64_t pos_b)
{
    if (score_a > score_b) return 1;
    if (score_a < score_b) return 0;
    return pos_a > pos_b;
}

/*
 * Eviction for one (batch, KV head) group (steps 4 and 5 of the step).
 *   C          cache size
 *   T          chunk length
 *   n_cand     number of candidates = (valid cache slots) + T
 *   cand_score [n_cand] updated score of each candidate
 *   cand_pos   [n_cand] position of each candidate (unique)
 *   cand_slot  [n_cand] cache slot of a cache candidate, -1 for chunk tokens;
 *              the chunk tokens are the last T candidates, in position order
 * Outputs:
 *   kept       [n_cand] 1 if the candidate survives
 *   token_slot [T]      slot that chunk token t is written to, -1 if dropped
 * A candidate is kept iff fewer than C candidates rank above it. That is the
 * plain definition of "the C largest", evaluated by counting (O(n^2)).
 */
int h2o_oracle_select_group(int C, int T, int n_cand,
                            const double *cand_score, const int64_t *cand_pos,
                            const int32_t *cand_slot,
                            uint8_t *kept, int32_t *token_slot)
{
    if (C <= 0 || T < 0 || n_cand < T || n_cand - T > C) return ORACLE_ERR_ARG;
    for (int a = 0; a < n_cand; ++a) {
        if (n_cand <= C) { kept[a] = 1; continue; }
        int above = 0;
        for (int b = 0; b < n_cand; ++b)
            if (b != a && ranks_above(cand_score[b], cand_pos[b], cand_score[a], cand_pos[a]))
                ++above;
        kept[a] = (uint8_t)(above < C);
    }
    /* Free slots: slots holding no kept cache candidate (empty before the
     * step, or evicted now), listed in ascending slot order. */
    uint8_t *occupied = (uint8_t *)calloc((size_t)C, 1);
    if (!occupied) return ORACLE_ERR_OOM;
    for (int a = 0; a < n_cand - T; ++a) {
        int s = cand_slot[a];
        if (s < 0 || s >= C) { free(occupied); return ORACLE_ERR_ARG; }
        if (kept[a]) occupied[s] = 1;
    }
    int next_free = 0;
    for (int t = 0; t < T; ++t) {
        int a = n_cand - T + t;
        token_slot[t] = -1;
        if (!kept[a]) continue;
        while (next_free < C && occupied[next_free]) ++next_free;
        if (next_free >= C) { free(occupied); return ORACLE_ERR_ARG; }
        token_slot[t] = next_free;
        occupied[next_free] = 1;
    }
    free(occupied);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Logit of query row qrow against key krow: scale * <q, k>. */
static double logit(const double *qrow, const double *krow, int d, double scale)
{
    double acc = 0.0;
    for (int x = 0; x < d; ++x) acc += qrow[x] * krow[x];
    return scale * acc;
}

/*
 * One step for one (batch b, KV head g) group. Shapes are those of the group:
 *   Kc, Vc  [C, d]       cache keys / values            (in/out)
 *   phi     [C]          H2O scores, 0 for empty slots  (in/out)
 *   pos     [C]          slot positions, -1 = empty     (in/out)
 *   q       [G, T, d]    the group's query heads for this chunk
 *   k, v    [T, d]       this chunk's keys / values for KV head g
 *   P       position of the chunk's first token
 * Outputs:
 *   out     [G, T, d]    attention output
 *   lse     [G, T]       natural-log sum of exp of each row's visible logits
 *   cand_*  [C + T]      candidates (valid cache slots in slot order, then the
 *                        chunk tokens); *n_cand receives their count
 *   token_slot [T]       where each chunk token went, -1 if dropped
 */
static int group_step(int G, int d, int C, int T, int64_t P, int policy,
                      double *Kc, double *Vc, double *phi, int64_t *pos,
                      const double *q, const double *k, const double *v,
                      double *out, double *lse,
                      double *cand_score, int64_t *cand_pos, int32_t *cand_slot,
                      uint8_t *cand_kept, int32_t *n_cand_out, int32_t *token_slot)
{
    const double scale = 1.0 / sqrt((double)d);

    /* Step 1: the candidate list and, for each candidate, its key/value row. */
    int n_valid = 0;
    for (int j = 0; j < C; ++j) {
        if (pos[j] < 0) continue;
        cand_score[n_valid] = phi[j];
        cand_pos[n_valid] = pos[j];
        cand_slot[n_valid] = j;
        ++n_valid;
    }
    const int n_cand = n_valid + T;
    for (int t = 0; t < T; ++t) {
        cand_score[n_valid + t] = 0.0;
        cand_pos[n_valid + t] = P + t;
        cand_slot[n_valid + t] = -1;
    }
    *n_cand_out = n_cand;
    const double **krow = (const double **)malloc(sizeof(double *) * (size_t)(n_cand > 0 ? n_cand : 1));
    const double **vrow = (const double **)malloc(sizeof(double *) * (size_t)(n_cand > 0 ? n_cand : 1));
    double *delta = (double *)calloc((size_t)(n_cand > 0 ? n_cand : 1), sizeof(double));
    double *w = (double *)malloc(sizeof(double) * (size_t)(n_cand > 0 ? n_cand : 1));
    double *rank_key = (double *)malloc(sizeof(double) * (size_t)(n_cand > 0 ? n_cand : 1));
    if (!krow || !vrow || !delta || !w || !rank_key) {
        free(krow); free(vrow); free(delta); free(w); free(rank_key);
        return ORACLE_ERR_OOM;
    }
    for (int c = 0; c < n_valid; ++c) {
        krow[c] = Kc + (size_t)cand_slot[c] * d;
        vrow[c] = Vc + (size_t)cand_slot[c] * d;
    }
    for (int t = 0; t < T; ++t) {
        krow[n_valid + t] = k + (size_t)t * d;
        vrow[n_valid + t] = v + (size_t)t * d;
    }

    /* Step 2: softmax attention of every row of every query head in the
     * group. Row i (position P+i) sees key c iff pos(c) <= P + i: all valid
     * cache slots (their positions are below P) and chunk tokens t <= i. */
    for (int h = 0; h < G; ++h) {
        for (int i = 0; i < T; ++i) {
            const double *qrow = q + ((size_t)h * T + i) * d;
            int n_vis = 0;
            double m = -INFINITY;
            for (int c = 0; c < n_cand; ++c) {
                if (cand_pos[c] > P + i) { w[c] = 0.0; continue; }
                w[c] = logit(qrow, krow[c], d, scale);
                if (w[c] > m) m = w[c];
                ++n_vis;
            }
            double Z = 0.0;
            for (int c = 0; c < n_cand; ++c)
                if (cand_pos[c] <= P + i) Z += exp(w[c] - m);
            double *orow = out + ((size_t)h * T + i) * d;
            for (int x = 0; x < d; ++x) orow[x] = 0.0;
            for (int c = 0; c < n_cand; ++c) {
                if (cand_pos[c] > P + i) continue;
                double wc = exp(w[c] - m) / Z;
                for (int x = 0; x < d; ++x) orow[x] += wc * vrow[c][x];
                delta[c] += wc;
            }
            lse[(size_t)h * T + i] = (n_vis > 0) ? m + log(Z) : -INFINITY;
        }
    }

    /* Step 3: updated scores (old score plus this step's weight sum). */
    for (int c = 0; c < n_cand; ++c) cand_score[c] += delta[c];

    /* Steps 4 and 5: eviction (ranked by the policy's key) and slot placement. */
    const int64_t t_after = P + T;
    for (int c = 0; c < n_cand; ++c)
        rank_key[c] = policy == 1 ? cand_score[c] / (double)(t_after - cand_pos[c]) : cand_score[c];
    int rc = h2o_oracle_select_group(C, T, n_cand, rank_key, cand_pos, cand_slot,
                                     cand_kept, token_slot);
    if (rc == ORACLE_OK) {
        for (int c = 0; c < n_valid; ++c) {
            int j = cand_slot[c];
            if (cand_kept[c]) {
                phi[j] = cand_score[c];
            } else {
                phi[j] = 0.0;
                pos[j] = -1;
            }
        }
        for (int t = 0; t < T; ++t) {
            int j = token_slot[t];
            if (j < 0) continue;
            memcpy(Kc + (size_t)j * d, k + (size_t)t * d, sizeof(double) * (size_t)d);
            memcpy(Vc + (size_t)j * d, v + (size_t)t * d, sizeof(double) * (size_t)d);
            phi[j] = cand_score[n_valid + t];
            pos[j] = P + t;
        }
    }
    free(krow); free(vrow); free(delta); free(w); free(rank_key);
    return rc;
}

/*
 * One step for the whole batch. Layouts (row-major, contiguous):
 *   Kc, Vc [B,Hkv,C,d]  phi, pos [B,Hkv,C]  q, out [B,Hq,T,d]  k, v [B,Hkv,T,d]
 *   lse [B,Hq,T]  cand_score, cand_pos, cand_slot, cand_kept [B,Hkv,C+T]
 *   n_cand [B,Hkv]  token_slot [B,Hkv,T]
 * Query head h belongs to KV head h / (Hq/Hkv). Groups run in parallel.
 */
int h2o_oracle_step_policy(int B, int Hq, int Hkv, int d, int C, int T, int64_t P, int policy,
                           double *Kc, double *Vc, double *phi, int64_t *pos,
                           const double *q, const double *k, const double *v,
                           double *out, double *lse,
                           double *cand_score, int64_t *cand_pos, int32_t *cand_slot,
                           uint8_t *cand_kept, int32_t *n_cand, int32_t *token_slot,
                           int nthreads)
{
    if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0 || d <= 0 || C <= 0 || T <= 0 || P < 0 ||
        (policy != 0 && policy != 1))
        return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const int groups = B * Hkv;
    int rc_all = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int bg = 0; bg < groups; ++bg) {
        const int b = bg / Hkv;
        const int g = bg % Hkv;
        const size_t cs = (size_t)bg * C;
        const size_t ct = (size_t)bg * (C + T);
        const size_t qo = ((size_t)b * Hq + (size_t)g * G) * T;
        int rc = group_step(G, d, C, T, P, policy,
                            Kc + cs * d, Vc + cs * d, phi + cs, pos + cs,
                            q + qo * d, k + (size_t)bg * T * d, v + (size_t)bg * T * d,
                            out + qo * d, lse + qo,
                            cand_score + ct, cand_pos + ct, cand_slot + ct, cand_kept + ct,
                            n_cand + bg, token_slot + (size_t)bg * T);
        if (rc != ORACLE_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
            rc_all = rc;
        }
    }
    return rc_all;
}

/* The step under the sum policy (policy 0). */
int h2o_oracle_step(int B, int Hq, int Hkv, int d, int C, int T, int64_t P,
                    double *Kc, double *Vc, double *phi, int64_t *pos,
                    const double *q, const double *k, const double *v,
                    double *out, double *lse,
                    double *cand_score, int64_t *cand_pos, int32_t *cand_slot,
                    uint8_t *cand_kept, int32_t *n_cand, int32_t *token_slot,
                    int nthreads)
{
    return h2o_oracle_step_policy(B, Hq, Hkv, d, C, T, P, 0, Kc, Vc, phi, pos, q, k, v, out, lse,
                                  cand_score, cand_pos, cand_slot, cand_kept, n_cand, token_slot,
                                  nthreads);
}

/* ------------------------------------------------------------------------ */
/* Insert-always variant ("Learning how to Forget", paper page, section
 * "Improvements to Heavy-Hitter Oracle (H2O)": new content overwrites the
 * slots with the smallest scores; section "Kernel Support Needs": attention
 * under the position mask). Reading taken: before the chunk attends, if the
 * cache cannot hold the n valid entries plus the T chunk tokens, the
 * n + T - C valid slots with the lowest pre-step scores are evicted (lowest
 * score first, the older position first among equal scores); the chunk
 * tokens, in position order, fill the empty and evicted slots in ascending
 * slot order with score 0; then every row attends to the C-slot buffer,
 * slot j visible to row i iff pos(j) <= P + i, and every valid slot's score
 * grows by the weights it receives. No chunk token is dropped, so T <= C. */
static int group_step_insert(int G, int d, int C, int T, int64_t P,
                             double *Kc, double *Vc, double *phi, int64_t *pos,
                             const double *q, const double *k, const double *v,
                             double *out, double *lse, int32_t *token_slot)
{
    if (T > C) return ORACLE_ERR_ARG;
    const double scale = 1.0 / sqrt((double)d);
    int n = 0;
    for (int j = 0; j < C; ++j) n += pos[j] >= 0;
    const int need = n + T - C;  /* valid slots to evict, if positive */
    uint8_t *evict = (uint8_t *)calloc((size_t)C, 1);
    double *w = (double *)malloc(sizeof(double) * (size_t)C);
    double *delta = (double *)calloc((size_t)C, sizeof(double));
    if (!evict || !w || !delta) { free(evict); free(w); free(delta); return ORACLE_ERR_OOM; }
    /* a valid slot goes iff fewer than `need` valid slots rank below it */
    for (int a = 0; need > 0 && a < C; ++a) {
        if (pos[a] < 0) continue;
        int below = 0;
        for (int b = 0; b < C; ++b)
            if (b != a && pos[b] >= 0 && ranks_above(phi[a], pos[a], phi[b], pos[b])) ++below;
        evict[a] = (uint8_t)(below < need);
    }
    /* free slots (empty or evicted) in ascending order take the chunk tokens */
    int t = 0;
    for (int j = 0; j < C && t < T; ++j) {
        if (pos[j] >= 0 && !evict[j]) continue;
        memcpy(Kc + (size_t)j * d, k + (size_t)t * d, sizeof(double) * (size_t)d);
        memcpy(Vc + (size_t)j * d, v + (size_t)t * d, sizeof(double) * (size_t)d);
        phi[j] = 0.0;
        pos[j] = P + t;
        token_slot[t] = j;
        ++t;
    }
    for (int j = 0; j < C; ++j)  /* evicted slots no chunk token took */
        if (evict[j] && pos[j] < P) { pos[j] = -1; phi[j] = 0.0; }
    /* attention over the buffer under the position mask */
    for (int h = 0; h < G; ++h) {
        for (int i = 0; i < T; ++i) {
            const double *qrow = q + ((size_t)h * T + i) * d;
            double m = -INFINITY;
            for (int j = 0; j < C; ++j) {
                if (pos[j] < 0 || pos[j] > P + i) continue;
                w[j] = logit(qrow, Kc + (size_t)j * d, d, scale);
                if (w[j] > m) m = w[j];
            }
            double Z = 0.0;
            for (int j = 0; j < C; ++j)
                if (pos[j] >= 0 && pos[j] <= P + i) Z += exp(w[j] - m);
            double *orow = out + ((size_t)h * T + i) * d;
            for (int x = 0; x < d; ++x) orow[x] = 0.0;
            for (int j = 0; j < C; ++j) {
                if (pos[j] < 0 || pos[j] > P + i) continue;
                const double wj = exp(w[j] - m) / Z;
                for (int x = 0; x < d; ++x) orow[x] += wj * Vc[(size_t)j * d + x];
                delta[j] += wj;
            }
            lse[(size_t)h * T + i] = m + log(Z);
        }
    }
    for (int j = 0; j < C; ++j)
        if (pos[j] >= 0) phi[j] += delta[j];
    free(evict); free(w); free(delta);
    return ORACLE_OK;
}

/* The insert-always step for the whole batch (layouts as h2o_oracle_step;
 * token_slot [B,Hkv,T] receives each chunk token's slot). */
int h2o_oracle_step_insert(int B, int Hq, int Hkv, int d, int C, int T, int64_t P,
                           double *Kc, double *Vc, double *phi, int64_t *pos,
                           const double *q, const double *k, const double *v,
                           double *out, double *lse, int32_t *token_slot, int nthreads)
{
    if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0 || d <= 0 || C <= 0 || T <= 0 || T > C || P < 0)
        return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const int groups = B * Hkv;
    int rc_all = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int bg = 0; bg < groups; ++bg) {
        const int b = bg / Hkv, g = bg % Hkv;
        const size_t cs = (size_t)bg * C;
        const size_t qo = ((size_t)b * Hq + (size_t)g * G) * T;
        int rc = group_step_insert(G, d, C, T, P, Kc + cs * d, Vc + cs * d, phi + cs, pos + cs,
                                   q + qo * d, k + (size_t)bg * T * d, v + (size_t)bg * T * d,
                                   out + qo * d, lse + qo, token_slot + (size_t)bg * T);
        if (rc != ORACLE_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
            rc_all = rc;
        }
    }
    return rc_all;
}

/* ------------------------------------------------------------------------ */
/* Backward of the chunk SDPA with the kept set fixed (the eviction is a
 * discrete choice, replayed, not differentiated): given dL/dO, the gradients
 * of L with respect to q, the chunk's k and v, and the cache's K and V, for
 * the same key set and mask as the forward (valid cache slots all visible,
 * chunk token t visible to row i iff t <= i), scale 1/sqrt(d). Per row:
 *   p = softmax(s), s_j = scale q.k_j;  dv_j += p_j dO;  dp_j = dO.v_j;
 *   ds_j = p_j (dp_j - sum_l p_l dp_l);  dq = scale sum_j ds_j k_j;
 *   dk_j += scale ds_j q.
 * Gradients of one KV head sum over the query heads of its group. Empty
 * cache slots get zero gradients. */
static int group_backward(int G, int d, int C, int T, int64_t P,
                          const double *Kc, const double *Vc, const int64_t *pos,
                          const double *q, const double *k, const double *v, const double *dout,
                          double *dq, double *dKc, double *dVc, double *dk, double *dv)
{
    const double scale = 1.0 / sqrt((double)d);
    const int nk = C + T;  /* key index j: cache slot j < C, chunk token j - C */
    double *p = (double *)malloc(sizeof(double) * (size_t)nk);
    double *dp = (double *)malloc(sizeof(double) * (size_t)nk);
    if (!p || !dp) { free(p); free(dp); return ORACLE_ERR_OOM; }
    memset(dKc, 0, sizeof(double) * (size_t)C * d);
    memset(dVc, 0, sizeof(double) * (size_t)C * d);
    memset(dk, 0, sizeof(double) * (size_t)T * d);
    memset(dv, 0, sizeof(double) * (size_t)T * d);
    for (int h = 0; h < G; ++h) {
        for (int i = 0; i < T; ++i) {
            const double *qrow = q + ((size_t)h * T + i) * d;
            const double *go = dout + ((size_t)h * T + i) * d;
            double *gq = dq + ((size_t)h * T + i) * d;
            double m = -INFINITY;
            for (int j = 0; j < nk; ++j) {
                const int vis = j < C ? pos[j] >= 0 : (j - C) <= i;
                if (!vis) { p[j] = -INFINITY; continue; }
                const double *kr = j < C ? Kc + (size_t)j * d : k + (size_t)(j - C) * d;
                p[j] = logit(qrow, kr, d, scale);
                if (p[j] > m) m = p[j];
            }
            double Z = 0.0;
            for (int j = 0; j < nk; ++j)
                if (p[j] != -INFINITY) Z += exp(p[j] - m);
            double pdp = 0.0;
            for (int j = 0; j < nk; ++j) {
                if (p[j] == -INFINITY) { p[j] = 0.0; dp[j] = 0.0; continue; }
                p[j] = exp(p[j] - m) / Z;
                const double *vr = j < C ? Vc + (size_t)j * d : v + (size_t)(j - C) * d;
                double acc = 0.0;
                for (int x = 0; x < d; ++x) acc += go[x] * vr[x];
                dp[j] = acc;
                pdp += p[j] * acc;
            }
            for (int x = 0; x < d; ++x) gq[x] = 0.0;
            for (int j = 0; j < nk; ++j) {
                if (p[j] == 0.0 && dp[j] == 0.0) continue;
                const double ds = p[j] * (dp[j] - pdp);
                const double *kr = j < C ? Kc + (size_t)j * d : k + (size_t)(j - C) * d;
                double *gk = j < C ? dKc + (size_t)j * d : dk + (size_t)(j - C) * d;
                double *gv = j < C ? dVc + (size_t)j * d : dv + (size_t)(j - C) * d;
                for (int x = 0; x < d; ++x) {
                    gq[x] += scale * ds * kr[x];
                    gk[x] += scale * ds * qrow[x];
                    gv[x] += p[j] * go[x];
                }
            }
        }
    }
    (void)P;
    free(p); free(dp);
    return ORACLE_OK;
}

/* Backward for the whole batch. Layouts: as h2o_oracle_step for Kc, Vc, pos,
 * q, k, v; dout and dq [B,Hq,T,d]; dKc, dVc [B,Hkv,C,d]; dk, dv [B,Hkv,T,d]. */
int h2o_oracle_backward(int B, int Hq, int Hkv, int d, int C, int T, int64_t P,
                        const double *Kc, const double *Vc, const int64_t *pos,
                        const double *q, const double *k, const double *v, const double *dout,
                        double *dq, double *dKc, double *dVc, double *dk, double *dv, int nthreads)
{
    if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0 || d <= 0 || C <= 0 || T <= 0 || P < 0)
        return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const int groups = B * Hkv;
    int rc_all = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int bg = 0; bg < groups; ++bg) {
        const int b = bg / Hkv, g = bg % Hkv;
        const size_t cs = (size_t)bg * C;
        const size_t qo = ((size_t)b * Hq + (size_t)g * G) * T;
        int rc = group_backward(G, d, C, T, P, Kc + cs * d, Vc + cs * d, pos + cs,
                                q + qo * d, k + (size_t)bg * T * d, v + (size_t)bg * T * d, dout + qo * d,
                                dq + qo * d, dKc + cs * d, dVc + cs * d, dk + (size_t)bg * T * d,
                                dv + (size_t)bg * T * d);
        if (rc != ORACLE_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
            rc_all = rc;
        }
    }
    return rc_all;
}

/*
 * Attention outputs of selected rows only, for checks at sizes where the full
 * step is too slow. For each requested (b, h, i): O and LSE of that row,
 * given the pre-step cache (valid slots = pos >= 0) and this chunk's k, v.
 * rows [n_rows, 3] int32 triples (b, h, i). out_rows [n_rows, d], lse_rows [n_rows].
 * Parallel over rows.
 */
int h2o_oracle_rows(int B, int Hq, int Hkv, int d, int C, int T, int64_t P,
                    const double *Kc, const double *Vc, const int64_t *pos,
                    const double *q, const double *k, const double *v,
                    int n_rows, const int32_t *rows,
                    double *out_rows, double *lse_rows, int nthreads)
{
    if (B <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || C <= 0 || T <= 0) return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const double scale = 1.0 / sqrt((double)d);
    int rc_all = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int r = 0; r < n_rows; ++r) {
        const int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= T) {
#ifdef _OPENMP
#pragma omp critical
#endif
            rc_all = ORACLE_ERR_ARG;
            continue;
        }
        const int g = h / G;
        const size_t bg = (size_t)b * Hkv + g;
        const double *qrow = q + (((size_t)b * Hq + h) * T + i) * d;
        const int n_keys = C + i + 1;
        double *l = (double *)malloc(sizeof(double) * (size_t)n_keys);
        if (!l) {
#ifdef _OPENMP
#pragma omp critical
#endif
            rc_all = ORACLE_ERR_OOM;
            continue;
        }
        double m = -INFINITY;
        for (int c = 0; c < n_keys; ++c) {
            const double *krow;
            if (c < C) {
                if (pos[bg * C + c] < 0) { l[c] = NAN; continue; }
                krow = Kc + (bg * C + c) * d;
            } else {
                krow = k + (bg * T + (c - C)) * d;
            }
            l[c] = logit(qrow, krow, d, scale);
            if (l[c] > m) m = l[c];
        }
        double Z = 0.0;
        for (int c = 0; c < n_keys; ++c)
            if (!isnan(l[c])) Z += exp(l[c] - m);
        double *orow = out_rows + (size_t)r * d;
        for (int x = 0; x < d; ++x) orow[x] = 0.0;
        for (int c = 0; c < n_keys; ++c) {
            if (isnan(l[c])) continue;
            const double *vr = (c < C) ? Vc + (bg * C + c) * d : v + (bg * T + (c - C)) * d;
            const double wc = exp(l[c] - m) / Z;
            for (int x = 0; x < d; ++x) orow[x] += wc * vr[x];
        }
        lse_rows[r] = m + log(Z);
        free(l);
    }
    return rc_all;
}
