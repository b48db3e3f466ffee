/*
 * dsa_oracle.c -- plain, slow CPU oracle for the DeepSeek Sparse Attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's CPU
 * baseline leg may load this library.  It shares no code, header, table or helper
 * with the CUDA path in sparse_attention_17_b200/, and it includes nothing from it.
 *
 * Every value is computed in IEEE double from the exact float32 images of the
 * inputs (bf16 and fp32 inputs both convert to float32, and from there to double,
 * without rounding).  No blocking, fusion or reordering beyond the definitions:
 *
 *   1. Lightning indexer score (DSA ablation model card, "Attention" bullet: a ReLU
 *      lightning indexer with a few heads scores keys per query).  The pages do not
 *      print the formula; this file takes the standard DSA reading
 *          I(t,s) = sum_j w[t,j] * max(0, sum_d q_idx[t,j,d] * k_idx[s,d])
 *      with ONE indexer key per token shared by all indexer heads and a per-query,
 *      per-head weight w.  The same card's parameter count (1,530,496 with indexers,
 *      1,498,496 without: 32,000 over 5 layers of hidden 128) is exactly
 *      5 * (128*2*16 + 128*16 + 128*2), i.e. this shape with one shared key.
 *   2. Causality (DSV2-Lite-IndexCache-Sparse-1250 card, first paragraph: "causal key
 *      selection"): query t may select keys s <= t, itself included.  In decode the
 *      new token's row is already in the cache, so a sequence of length L offers
 *      keys 0..L-1.
 *   3. Top-k selection (DSA ablation card, "Attention" bullet: top-512 keys per query;
 *      DSV2-Lite-IndexCache card: budget 2048).  Of the n valid keys, take the k
 *      highest scores; equal scores go to the lower index.  If n <= k every key is
 *      selected (ablation card, closing note: at prompts no longer than k DSA equals
 *      dense attention).  Indices are returned ascending and padded with -1.
 *   4. Sparse attention over the selected keys only (DSV2-Lite-IndexCache card,
 *      attention_mode="sparse"; its "portable runtime" is masked SDPA, i.e. a softmax
 *      restricted to the selected keys).  For MLA in absorbed form the key is the
 *      576-dim latent row (512 kv_lora + 64 RoPE, DeepSeek-V2-Lite-Chat SIQ card,
 *      "MLA attention (kvlorarank 512 ...)", 576 B/token at fp8) shared by all heads,
 *      and the value is its first 512 dims.
 *   5. Decode reads cache rows through a page table: token s of sequence b lives in
 *      pool row page_table[b][s / page_size] * page_size + s % page_size.
 *
 * The IndexCache layer loop (vLLM IndexCache docs, "How It Works") is a loop over
 * these functions and lives in oracle.py.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- deliberate mistakes, compiled in only for the mutation tests -------------
 * tests/test_oracle_mutants.py builds this file with -DORACLE_MUTANT=<n> and checks
 * that each such build fails at least one pin.  The default build has none. */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int oracle_mutant_id(void) { return ORACLE_MUTANT; }

/* One indexer score (definition 1) for query vectors qt[H_I][D_I], weights wt[H_I]
 * and key ks[D_I]. */
static double indexer_score(const float* qt, const float* wt, const float* ks, int H_I, int D_I) {
    double total = 0.0;
    for (int j = 0; j < H_I; ++j) {
        double dot = 0.0;
#if ORACLE_MUTANT == 4
        for (int d = 0; d < D_I - 1; ++d)          /* mutant: drops the last dim */
#else
        for (int d = 0; d < D_I; ++d)
#endif
            dot += (double)qt[(long)j * D_I + d] * (double)ks[d];
#if ORACLE_MUTANT == 1
        double r = dot;                             /* mutant: no ReLU */
#else
        double r = dot > 0.0 ? dot : 0.0;
#endif
#if ORACLE_MUTANT == 2
        total += r;                                 /* mutant: head weight dropped */
#else
        total += (double)wt[j] * r;
#endif
    }
    return total;
}

/* Prefill scores (definitions 1, 2).  Row r is query t = q_begin + r.  Entries
 * s > t are causally invalid and are written as -INFINITY; columns run 0..S-1. */
void oracle_indexer_scores_prefill(const float* q_idx, const float* k_idx, const float* w,
                                   int H_I, int D_I, int q_begin, int rows, int S,
                                   double* scores) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < rows; ++r) {
        long t = (long)q_begin + r;
        const float* qt = q_idx + t * H_I * D_I;
        const float* wt = w + t * H_I;
        double* out = scores + (long)r * S;
        for (int s = 0; s < S; ++s) {
#if ORACLE_MUTANT == 3
            int valid = s < t;                      /* mutant: diagonal excluded */
#else
            int valid = s <= t;
#endif
            out[s] = valid ? indexer_score(qt, wt, k_idx + (long)s * D_I, H_I, D_I) : -INFINITY;
        }
    }
}

/* Row of the cache pool that holds token s of sequence b (definition 5). */
static long paged_row(const int* page_table, int max_pages, int page_size, int b, long s) {
    return (long)page_table[(long)b * max_pages + s / page_size] * page_size + s % page_size;
}

/* Decode scores (definitions 1, 2, 5): row b scores keys 0..seq_lens[b]-1 of its own
 * paged key cache; columns seq_lens[b]..S-1 are written as -INFINITY. */
void oracle_indexer_scores_decode(const float* q_idx, const float* k_pool, const float* w,
                                  int H_I, int D_I, int B, const int* page_table,
                                  int max_pages, int page_size, const int* seq_lens,
                                  int S, double* scores) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        const float* qt = q_idx + (long)b * H_I * D_I;
        const float* wt = w + (long)b * H_I;
        double* out = scores + (long)b * S;
        for (int s = 0; s < S; ++s) {
            if (s < seq_lens[b]) {
                long row = paged_row(page_table, max_pages, page_size, b, s);
                out[s] = indexer_score(qt, wt, k_pool + row * D_I, H_I, D_I);
            } else {
                out[s] = -INFINITY;
            }
        }
    }
}

typedef struct { double score; int index; } scored_key;

/* Order of definition 3: higher score first, then lower index first. */
static int by_score_then_index(const void* a, const void* b) {
    const scored_key* x = (const scored_key*)a;
    const scored_key* y = (const scored_key*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
#if ORACLE_MUTANT == 5
    return (x->index < y->index) ? 1 : (x->index > y->index) ? -1 : 0;   /* mutant: ties to the higher index */
#else
    return (x->index < y->index) ? -1 : (x->index > y->index) ? 1 : 0;
#endif
}

static int ascending_int(const void* a, const void* b) {
    int x = *(const int*)a, y = *(const int*)b;
    return (x > y) - (x < y);
}

/* Top-k (definition 3) of each row: row r has n_valid[r] valid scores in columns
 * 0..n_valid[r]-1 of scores[r*ld ...].  Writes idx[r*k .. r*k+k-1]. */
void oracle_topk_rows(const double* scores, long ld, int rows, const int* n_valid, int k,
                      int* idx) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        int n = n_valid[r];
        const double* row = scores + (long)r * ld;
        scored_key* keys = (scored_key*)malloc(sizeof(scored_key) * (size_t)(n > 0 ? n : 1));
        for (int s = 0; s < n; ++s) { keys[s].score = row[s]; keys[s].index = s; }
        qsort(keys, (size_t)n, sizeof(scored_key), by_score_then_index);
        int take = n < k ? n : k;
        int* out = idx + (long)r * k;
        for (int i = 0; i < take; ++i) out[i] = keys[i].index;
        qsort(out, (size_t)take, sizeof(int), ascending_int);
        for (int i = take; i < k; ++i) out[i] = -1;
        free(keys);
    }
}

/* Sparse attention (definition 4) for NQ queries with H heads each.
 *   query n, head h:       q + n*q_stride_tok + h*q_stride_head, D_qk values
 *   key s, head h:         k + row(s)*kv_stride_tok + h*kv_stride_head, D_qk values
 *   value s, head h:       v + row(s)*kv_stride_tok + h*kv_stride_head, first D_v values
 * with row(s) = s, or the paged row of definition 5 when page_table is not NULL
 * (query n is then sequence n).  MLA passes v == k, kv_stride_head == 0, D_v = 512.
 * Selected keys are idx[n*ld_idx + i], i < k_sel; entries < 0 are padding.
 *   logit_s = scale * q . k_s ;  m = max logit ;  p_s = exp(logit_s - m)
 *   out = sum_s p_s v_s / sum_s p_s ;  lse = m + log(sum_s p_s)
 * A query with no selected key gets out = 0 and lse = -INFINITY. */
void oracle_sparse_attention(const float* q, long q_stride_tok, long q_stride_head,
                             const float* k, const float* v, long kv_stride_tok,
                             long kv_stride_head, int NQ, int H, int D_qk, int D_v,
                             double scale, const int* idx, long ld_idx, int k_sel,
                             const int* page_table, int max_pages, int page_size,
                             double* out, double* lse) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NQ; ++n) {
        const int* sel = idx + (long)n * ld_idx;
        double* logits = (double*)malloc(sizeof(double) * (size_t)(k_sel > 0 ? k_sel : 1));
        long* rows = (long*)malloc(sizeof(long) * (size_t)(k_sel > 0 ? k_sel : 1));
        int count = 0;
        for (int i = 0; i < k_sel; ++i) {
            if (sel[i] < 0) continue;
            rows[count++] = page_table ? paged_row(page_table, max_pages, page_size, n, sel[i])
                                       : (long)sel[i];
        }
        for (int h = 0; h < H; ++h) {
            const float* qh = q + (long)n * q_stride_tok + (long)h * q_stride_head;
            double* o = out + ((long)n * H + h) * D_v;
            for (int d = 0; d < D_v; ++d) o[d] = 0.0;
            if (count == 0) { lse[(long)n * H + h] = -INFINITY; continue; }
            double m = -INFINITY;
            for (int i = 0; i < count; ++i) {
                const float* kr = k + rows[i] * kv_stride_tok + (long)h * kv_stride_head;
                double dot = 0.0;
                for (int d = 0; d < D_qk; ++d) dot += (double)qh[d] * (double)kr[d];
#if ORACLE_MUTANT == 6
                logits[i] = dot;                    /* mutant: softmax scale dropped */
#else
                logits[i] = scale * dot;
#endif
                if (logits[i] > m) m = logits[i];
            }
            double denom = 0.0;
            for (int i = 0; i < count; ++i) {
                double p = exp(logits[i] - m);
                denom += p;
#if ORACLE_MUTANT == 7
                const float* vr = v + rows[i] * kv_stride_tok + (long)h * kv_stride_head + 64;  /* mutant: wrong value slice */
#else
                const float* vr = v + rows[i] * kv_stride_tok + (long)h * kv_stride_head;
#endif
                for (int d = 0; d < D_v; ++d) o[d] += p * (double)vr[d];
            }
            for (int d = 0; d < D_v; ++d) o[d] /= denom;
#if ORACLE_MUTANT == 8
            lse[(long)n * H + h] = log(denom);      /* mutant: max not added back */
#else
            lse[(long)n * H + h] = m + log(denom);
#endif
        }
        free(logits);
        free(rows);
    }
}
