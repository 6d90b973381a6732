/*
 * fp_oracle.c -- plain, slow fp64 CPU oracle for FlashPrefill-style block-sparse causal prefill.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU-baseline /
 * reference legs may load this library. The product path (the CUDA library) never calls it,
 * and this file shares no code, header, table or helper with the CUDA side.
 *
 * What it computes, step by step, in the order of the pages:
 *
 *   pool    FlashPrefill ("FlashPrefill: Instantaneous Pattern Discovery ...", skill summary page,
 *           "Stage 1: Block-Level Attention Approximation"): block b of a sequence of length L
 *           spans tokens [b*B, min((b+1)*B, L)); its pooled query/key is the MEAN over the tokens
 *           it actually holds; the number of blocks is ceil(L/B).
 *   score   same section: block score = (pooled q) . (pooled k) / sqrt(d), d = head dim.
 *           Causal (j <= i), per q-head, GQA kv-head = h / (Hq/Hkv): from the problem statement
 *           this repository implements (the pages only give the per-head form).
 *   keep    same page, "Core Concept" item 3 ("Dynamic Thresholding": a single max reduction
 *           instead of sorting / cumulative sums) and the abstract's "max-based dynamic
 *           thresholding": p_ij = softmax over j <= i of the block scores; keep j iff
 *           p_ij >= tau * max_j p_ij; the sink block j = 0 and the diagonal block j = i are
 *           always kept.
 *   emit    "Architecture Overview", "Physical Index Jumping": kept block indices per
 *           (head, query block), ascending.
 *   attn    exact softmax attention of each query token over the keys of its kept blocks that
 *           are at or before it (causal), in fp64.
 *
 * Readings where the pages are silent:
 *   - the garbled Stage-1 snippet is read as mean over the token axis, num_blocks = ceil(L/B),
 *     d = last dim of Q;
 *   - "uniformly distributed query probes" is read as the block mean of all queries;
 *   - no mean-correction term (FlashPrefill V2 names one but gives no formula): parity for that
 *     variant is unpinned and it is not implemented;
 *   - varlen: blocks, the sink and block ids restart at each sequence; no cross-sequence keys;
 *   - token attention uses the same 1/sqrt(d) scale unless the caller passes another.
 *
 * Index-list layout (an interface, restated independently on the CUDA side):
 *   counts[h * NB + gb]                     gb = global block id = cu_blocks[s] + i
 *   indices[base_s + h*nb_s(nb_s+1)/2 + i(i+1)/2 + n]   n-th kept block (local id) of row (s,h,i)
 *   base_s = sum over s' < s of Hq * nb_s'(nb_s'+1)/2
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bits -> double, exact (bf16 is the top half of an IEEE float32). */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int64_t blocks_of(int64_t len, int B) { return (len + B - 1) / B; }

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Total number of blocks over all sequences. */
int64_t orc_total_blocks(const int32_t* cu, int S, int B) {
    int64_t nb = 0;
    for (int s = 0; s < S; ++s) nb += blocks_of(cu[s + 1] - cu[s], B);
    return nb;
}

/* Number of int32 entries of the triangular index buffer. */
int64_t orc_index_elems(const int32_t* cu, int S, int B, int Hq) {
    int64_t n = 0;
    for (int s = 0; s < S; ++s) {
        int64_t nb = blocks_of(cu[s + 1] - cu[s], B);
        n += (int64_t)Hq * nb * (nb + 1) / 2;
    }
    return n;
}

/* ---------------------------------------------------------------- pool ----------------------- */
/* x: bf16 bits [T, H, d]; out: [NB, H, d] block means. Returns 0. */
int orc_pool(const uint16_t* x, const int32_t* cu, int S, int H, int d, int B, double* out) {
    int64_t gb0 = 0;
    for (int s = 0; s < S; ++s) {
        int64_t start = cu[s], L = cu[s + 1] - cu[s];
        int64_t nb = blocks_of(L, B);
#pragma omp parallel for schedule(static)
        for (int64_t b = 0; b < nb; ++b) {
            int64_t gb = gb0 + b;
            int64_t t0 = start + b * B;
            int64_t t1 = start + ((b + 1) * B < L ? (b + 1) * B : L); /* partial last block */
            double n = (double)(t1 - t0);
            for (int h = 0; h < H; ++h) {
                for (int c = 0; c < d; ++c) {
                    double sum = 0.0;
                    for (int64_t t = t0; t < t1; ++t) sum += bf16_to_double(x[(t * H + h) * d + c]);
                    out[(gb * H + h) * d + c] = sum / n;
                }
            }
        }
        gb0 += nb;
    }
    return 0;
}

/* ------------------------------------------------------- pooled softmax row ------------------ */
/* For one (sequence s, q-head h, query block i): scores, softmax p and ratio p/max p over j<=i.
 * qbar: [NB, Hq, d], kbar: [NB, Hkv, d]. p and ratio have i+1 entries. gb0 = first global block
 * of the sequence. */
static void pooled_row(const double* qbar, const double* kbar, int64_t gb0, int Hq, int Hkv, int d,
                       int h, int64_t i, double* score, double* p, double* ratio) {
    int G = Hq / Hkv;
    int g = h / G;
    double inv_sqrt_d = 1.0 / sqrt((double)d);
    const double* qv = qbar + ((gb0 + i) * Hq + h) * d;
    double m = -INFINITY;
    for (int64_t j = 0; j <= i; ++j) {
        const double* kv = kbar + ((gb0 + j) * Hkv + g) * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qv[c] * kv[c];
        score[j] = dot * inv_sqrt_d;
        if (score[j] > m) m = score[j];
    }
    double z = 0.0;
    for (int64_t j = 0; j <= i; ++j) z += exp(score[j] - m);
    double pmax = 0.0;
    for (int64_t j = 0; j <= i; ++j) {
        p[j] = exp(score[j] - m) / z;
        if (p[j] > pmax) pmax = p[j];
    }
    for (int64_t j = 0; j <= i; ++j) ratio[j] = p[j] / pmax;
}

/* Expose one pooled softmax row (for the tests' invariants). Returns 0, or -1 on bad args. */
int orc_pooled_row(const double* qbar, const double* kbar, const int32_t* cu, int S, int B, int Hq,
                   int Hkv, int d, int s, int h, int64_t i, double* score, double* p, double* ratio) {
    if (s < 0 || s >= S || h < 0 || h >= Hq || Hq % Hkv) return -1;
    int64_t gb0 = 0;
    for (int t = 0; t < s; ++t) gb0 += blocks_of(cu[t + 1] - cu[t], B);
    if (i < 0 || i >= blocks_of(cu[s + 1] - cu[s], B)) return -1;
    pooled_row(qbar, kbar, gb0, Hq, Hkv, d, h, i, score, p, ratio);
    return 0;
}

/* ------------------------------------------------------ top-p search (comparison) ------------ */
/* The cumulative-probability selector that FlashPrefill sets its threshold against (FlashPrefill
 * skill summary page, "The Problem": Top-k / Top-p need score computation, sorting and cumulative
 * sums; FlexPrefill abstract, "Cumulative-Attention Based Index Selection": the selected indexes'
 * attention scores must sum to a preset threshold). On the same pooled scores and causal softmax
 * p_ij as orc_search: rank the blocks by p (largest first) and keep the smallest leading set whose
 * probability sum reaches gamma. Written without an order among equal p values: with
 *     D_j = sum of p_l over the blocks l with p_l > p_j   (the mass ranked strictly before j),
 * block j is kept iff D_j < gamma, so blocks tied at the cut are kept together. The sink block 0
 * and the diagonal block i are kept as in orc_search. gamma <= 0 keeps only those two; gamma >= 1
 * keeps every causal block. band (optional): 1 where the decision is within reach of rounding:
 * |D_j - gamma| <= band_rel * max(gamma, 1e-300), or a block with p within 1e-5 (relative) of p_j
 * could change D_j across gamma. */
static int cmp_desc(const void* a, const void* b) {
    double x = *(const double*)a, y = *(const double*)b;
    return (x < y) - (x > y);
}

int orc_search_topp(const double* qbar, const double* kbar, const int32_t* cu, int S, int B, int Hq,
                    int Hkv, int d, double gamma, double band_rel, int32_t* counts, int32_t* indices,
                    uint8_t* band) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return -1;
    int64_t NB = orc_total_blocks(cu, S, B);
    int64_t gb0 = 0, base = 0;
    for (int s = 0; s < S; ++s) {
        int64_t nb = blocks_of(cu[s + 1] - cu[s], B);
        int64_t tri = nb * (nb + 1) / 2;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
        for (int h = 0; h < Hq; ++h) {
            for (int64_t i = 0; i < nb; ++i) {
                int64_t n = i + 1;
                double* score = (double*)malloc(sizeof(double) * (size_t)(6 * n + 1));
                double* p = score + n;
                double* ratio = p + n;
                double* sorted = ratio + n;
                double* dmass = sorted + n;
                double* prefix = dmass + n; /* n + 1 entries: prefix[r] = sorted[0] + ... + sorted[r-1] */
                pooled_row(qbar, kbar, gb0, Hq, Hkv, d, h, i, score, p, ratio);
                memcpy(sorted, p, sizeof(double) * (size_t)n);
                qsort(sorted, (size_t)n, sizeof(double), cmp_desc);
                prefix[0] = 0.0;
                for (int64_t r = 0; r < n; ++r) prefix[r + 1] = prefix[r] + sorted[r];
                int64_t row = base + (int64_t)h * tri + i * (i + 1) / 2;
                int32_t cnt = 0;
                for (int64_t j = 0; j <= i; ++j) {
                    /* lo = number of sorted entries strictly greater than p_j; hi = those >= p_j */
                    int64_t lo = 0, hi = n;
                    while (lo < hi) {
                        int64_t mid = (lo + hi) / 2;
                        if (sorted[mid] > p[j]) lo = mid + 1; else hi = mid;
                    }
                    int64_t eq_end = lo;
                    while (eq_end < n && sorted[eq_end] == p[j]) ++eq_end;
                    dmass[j] = prefix[lo]; /* D_j: mass ranked strictly before j */
                    int keep = gamma >= 1.0 || dmass[j] < gamma || j == 0 || j == i;
                    if (band) {
                        int amb = fabs(dmass[j] - gamma) <= band_rel * (gamma > 1e-300 ? gamma : 1e-300);
                        /* a value within 1e-5 (relative) of p_j on either side, or an exact tie */
                        int near = (eq_end - lo) > 1 || (lo > 0 && sorted[lo - 1] - p[j] <= 1e-5 * sorted[lo - 1]) ||
                                   (eq_end < n && p[j] - sorted[eq_end] <= 1e-5 * p[j]);
                        if (near && fabs(dmass[j] - gamma) <= 2.00002 * p[j] + 1e-300) amb = 1;
                        band[row + j] = (uint8_t)(gamma > 0.0 && gamma < 1.0 && amb);
                    }
                    if (keep) indices[row + cnt++] = (int32_t)j;
                }
                counts[(int64_t)h * NB + gb0 + i] = cnt;
                free(score);
            }
        }
        gb0 += nb;
        base += (int64_t)Hq * tri;
    }
    return 0;
}

/* ------------------------------------------------------------- search ------------------------ */
/* Threshold + emission. counts: [Hq, NB]; indices: triangular layout above; band (optional, same
 * layout as indices, one byte per causal (row, j)): 1 where |ratio - tau| <= band_rel * tau,
 * i.e. the block sits within the stated tie band of the threshold. Returns 0, -1 on bad args. */
int orc_search(const double* qbar, const double* kbar, const int32_t* cu, int S, int B, int Hq,
               int Hkv, int d, double tau, double band_rel, int32_t* counts, int32_t* indices,
               uint8_t* band) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return -1;
    int64_t NB = orc_total_blocks(cu, S, B);
    int64_t gb0 = 0, base = 0;
    for (int s = 0; s < S; ++s) {
        int64_t nb = blocks_of(cu[s + 1] - cu[s], B);
        int64_t tri = nb * (nb + 1) / 2;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
        for (int h = 0; h < Hq; ++h) {
            for (int64_t i = 0; i < nb; ++i) {
                double* score = (double*)malloc(sizeof(double) * (size_t)(3 * (i + 1)));
                double* p = score + (i + 1);
                double* ratio = p + (i + 1);
                pooled_row(qbar, kbar, gb0, Hq, Hkv, d, h, i, score, p, ratio);
                double pmax = 0.0;
                for (int64_t j = 0; j <= i; ++j)
                    if (p[j] > pmax) pmax = p[j];
                int64_t row = base + (int64_t)h * tri + i * (i + 1) / 2;
                int32_t n = 0;
                for (int64_t j = 0; j <= i; ++j) {
                    int keep = (p[j] >= tau * pmax) || j == 0 || j == i;
                    if (band) band[row + j] = (tau > 0.0 && fabs(ratio[j] - tau) <= band_rel * tau);
                    if (keep) indices[row + n++] = (int32_t)j;
                }
                counts[(int64_t)h * NB + gb0 + i] = n;
                free(score);
            }
        }
        gb0 += nb;
        base += (int64_t)Hq * tri;
    }
    return 0;
}

/* ------------------------------------------------------------- attention --------------------- */
/* Exact attention for a list of (token, q-head) rows. If counts == NULL every causal block is
 * kept (dense causal attention). q: [T, Hq, d], k/v: [T, Hkv, d] bf16 bits. out: [nrows, d],
 * lse (optional): [nrows], natural log of sum_u exp(scale * q.k_u). scale <= 0 means 1/sqrt(d).
 * Returns 0, or -1 on bad args. */
int orc_attn_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu, int S,
                  int B, int Hq, int Hkv, int d, double scale, const int32_t* counts,
                  const int32_t* indices, int64_t nrows, const int64_t* row_tok,
                  const int32_t* row_head, double* out, double* lse) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    int64_t NB = orc_total_blocks(cu, S, B);
    int64_t T = cu[S];
    int G = Hq / Hkv;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = row_tok[r];
        int h = row_head[r];
        if (t < 0 || t >= T || h < 0 || h >= Hq) { bad |= 1; continue; }
        /* locate the sequence of token t and its block bases */
        int s = 0;
        int64_t gb0 = 0, base = 0;
        while (!(cu[s] <= t && t < cu[s + 1])) {
            int64_t nbs = blocks_of(cu[s + 1] - cu[s], B);
            gb0 += nbs;
            base += (int64_t)Hq * nbs * (nbs + 1) / 2;
            ++s;
        }
        int64_t start = cu[s], L = cu[s + 1] - cu[s];
        int64_t nb = blocks_of(L, B);
        int64_t pos = t - start, i = pos / B;
        int g = h / G;

        int64_t nkept = counts ? counts[(int64_t)h * NB + gb0 + i] : i + 1;
        const int32_t* list = counts ? indices + base + (int64_t)h * (nb * (nb + 1) / 2) + i * (i + 1) / 2 : NULL;

        double* logit = (double*)malloc(sizeof(double) * (size_t)(pos + 1));
        int64_t* key = (int64_t*)malloc(sizeof(int64_t) * (size_t)(pos + 1));
        int64_t nk = 0;
        const uint16_t* qv = q + (t * Hq + h) * d;
        double m = -INFINITY;
        for (int64_t n = 0; n < nkept; ++n) {
            int64_t j = list ? list[n] : n;
            if (j < 0 || j > i) { bad |= 2; continue; }
            for (int64_t u = j * B; u < (j + 1) * B && u < L && u <= pos; ++u) {
                const uint16_t* kv = k + ((start + u) * Hkv + g) * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += bf16_to_double(qv[c]) * bf16_to_double(kv[c]);
                logit[nk] = dot * scale;
                key[nk] = start + u;
                if (logit[nk] > m) m = logit[nk];
                ++nk;
            }
        }
        double z = 0.0;
        for (int64_t n = 0; n < nk; ++n) z += exp(logit[n] - m);
        double* o = out + r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int64_t n = 0; n < nk; ++n) {
            double w = exp(logit[n] - m) / z;
            const uint16_t* vv = v + (key[n] * Hkv + g) * d;
            for (int c = 0; c < d; ++c) o[c] += w * bf16_to_double(vv[c]);
        }
        if (lse) lse[r] = (nk > 0) ? m + log(z) : -INFINITY;
        free(logit);
        free(key);
    }
    return bad ? -1 : 0;
}
