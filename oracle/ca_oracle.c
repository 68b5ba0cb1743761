/*
 * ca_oracle.c — plain, slow CPU oracle for the CompactAttention chunked-prefill
 * hot path. TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; the CUDA library never does, and the
 * two share no source.
 *
 * Source: "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
 * Selection" (arXiv 2605.16839), as summarised on its gist.science,
 * hotpaper.ai and fugumt.com pages:
 *   - Selection stage ("Methodology", step 1): a per-head 2D block mask is
 *     reduced by a Q-block union over the chunk's query blocks and an
 *     intra-group union over the query heads that share a KV head, giving the
 *     minimal per-(batch, KV-group) table T_{b,g} that keeps every block any
 *     head or Q-block of the group selected (coverage preservation).
 *   - Execution stage ("Methodology", step 2): dense attention of every query
 *     head of the group over the selected blocks, read in place from the
 *     KV-head-major cache [B, H_kv, L, D]; the tables travel as
 *     kv_indptr / kv_indices.
 * Readings where the pages are silent (each is listed in the design notes):
 *   - query head h uses KV head floor(h / G), G = H_q / H_kv;
 *   - tables are ascending, padded with -1;
 *   - causality is bottom-right aligned: chunk row r of sequence b sits at
 *     position p = chunk_start[b] + r and sees key k iff k <= p, inside every
 *     selected block;
 *   - LSE is the natural log of the softmax denominator of the scaled logits;
 *     a row that sees no key has O = 0 and LSE = -inf.
 *
 * Everything is the plain definition, evaluated in fp64 from the exact bf16
 * inputs. The only concurrency is independent rows spread over pthreads; the
 * arithmetic of each row is unchanged by it.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ETABLE (-2)
#define ORACLE_ENOMEM (-3)

/* bf16 is the top half of an IEEE binary32: widening is exact. */
/* FP8 E4M3 (the OCP 8-bit format without infinities): sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits. Exponent field 0 holds the subnormals
 * m/8 * 2^-6; the code with every exponent and mantissa bit set is NaN;
 * everything else is (1 + m/8) * 2^(e - 7). The largest finite value is 448. */
static double e4m3_to_f64(uint8_t bits) {
    const int sign = bits >> 7, e = (bits >> 3) & 15, m = bits & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

double oracle_e4m3_decode(int bits) { return e4m3_to_f64((uint8_t)(bits & 0xFF)); }

static double bf16_to_f64(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Block-Union table construction (selection stage).
 *   U[b,g,j] = OR over heads h of group g, OR over Q-blocks i, of M[b,h,i,j]
 *   T_{b,g}  = { j : U[b,g,j] } in ascending order, tail padded with -1
 *   counts   = |T_{b,g}|
 *   indptr   = exclusive prefix sum of counts over (b, g) row-major,
 *   indices  = the tables concatenated (the kv_indptr / kv_indices form).
 * indptr / indices may be NULL.
 */
int oracle_block_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int group,
                        int32_t *tables, int32_t *counts, int32_t *indptr, int32_t *indices) {
    if (!mask || !tables || !counts || B <= 0 || H_q <= 0 || nQ <= 0 || nKVmax <= 0 ||
        group <= 0 || H_q % group != 0)
        return ORACLE_EINVAL;
    const int H_kv = H_q / group;
    for (int b = 0; b < B; ++b) {
        for (int g = 0; g < H_kv; ++g) {
            int32_t *T = tables + ((size_t)b * H_kv + g) * nKVmax;
            int n = 0;
            for (int j = 0; j < nKVmax; ++j) {
                int selected = 0;
                for (int hl = 0; hl < group; ++hl) {
                    const int h = g * group + hl;
                    for (int i = 0; i < nQ; ++i) {
                        if (mask[(((size_t)b * H_q + h) * nQ + i) * nKVmax + j] != 0)
                            selected = 1;
                    }
                }
                if (selected) T[n++] = j;
            }
            counts[b * H_kv + g] = n;
            for (int t = n; t < nKVmax; ++t) T[t] = -1;
        }
    }
    if (indptr) {
        indptr[0] = 0;
        for (int bg = 0; bg < B * H_kv; ++bg) indptr[bg + 1] = indptr[bg] + counts[bg];
        if (indices) {
            for (int bg = 0; bg < B * H_kv; ++bg)
                for (int t = 0; t < counts[bg]; ++t)
                    indices[indptr[bg] + t] = tables[(size_t)bg * nKVmax + t];
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Attention over the selected blocks (execution stage).                   */
/* ---------------------------------------------------------------------- */

typedef struct {
    const void *Q, *K, *V;           /* bf16 bits, or e4m3 bytes (fp8) */
    int fp8;                         /* inputs are e4m3, value = descale * code */
    double q_descale, k_descale, v_descale;
    const int32_t *tables, *counts;  /* NULL tables: dense, T = [0, nKV_b) */
    const uint8_t *tile_mask;        /* non-NULL: per-tile block-sparse key sets */
    int nQ;                          /* Q-blocks per chunk (tile_mask only) */
    const int32_t *chunk_start;
    int B, H_q, H_kv, C, L_max, D, blk;
    double scale;
    const int64_t *rows;             /* flat (b*H_q + h)*C + r, or NULL = all */
    int64_t n_rows;
    double *O, *LSE;                 /* [n_rows, D], [n_rows] */
    int64_t begin, end;              /* this worker's slice of rows */
    int status;
} attn_job;

static int attention_over_keys(const attn_job *J, int b, int h, int g, int r,
                               const int32_t *keys, int64_t nk, double *s, double *o,
                               double *lse);

/* Element i of an input tensor as a real number: a bf16 value, or an e4m3
 * code times the tensor's descale factor. */
static double elem(const void *base, size_t i, int fp8, double descale) {
    if (fp8) return descale * e4m3_to_f64(((const uint8_t *)base)[i]);
    return bf16_to_f64(((const uint16_t *)base)[i]);
}

/* One query row: the definition written out.
 *   K_set = { k : floor(k / blk) in T_{b,g}, k <= p }
 *   s_k   = scale * sum_d Q[b,h,r,d] K[b,g,k,d]
 *   LSE   = log sum_{k in K_set} exp(s_k)          (max-subtracted)
 *   O[d]  = sum_{k in K_set} exp(s_k - LSE) V[b,g,k,d]                    */
static int attention_row(const attn_job *J, int64_t flat, double *s, int32_t *keys,
                         double *o, double *lse) {
    const int C = J->C, blk = J->blk;
    const int r = (int)(flat % C);
    const int h = (int)((flat / C) % J->H_q);
    const int b = (int)(flat / ((int64_t)C * J->H_q));
    const int G = J->H_q / J->H_kv;
    const int g = h / G;
    const int64_t p = (int64_t)J->chunk_start[b] + r;
    const int nKVmax = J->L_max / blk;

    int64_t nk = 0;
    if (J->tile_mask) {
        /* Per-tile block-sparse baseline: row r of head h uses only the blocks
         * its own Q-block i = floor(r / blk) selected in its own mask row,
         *   K_set = { k : M[b,h,i,floor(k / blk)] != 0, k <= p }.         */
        const uint8_t *mrow =
            J->tile_mask + (((size_t)b * J->H_q + h) * J->nQ + r / blk) * (size_t)nKVmax;
        for (int j = 0; j < nKVmax; ++j) {
            if (mrow[j] == 0) continue;
            for (int c = 0; c < blk; ++c) {
                const int64_t k = (int64_t)j * blk + c;
                if (k <= p) keys[nk++] = (int32_t)k;
            }
        }
        return attention_over_keys(J, b, h, g, r, keys, nk, s, o, lse);
    }

    int n_entries;
    const int32_t *T = NULL;
    if (J->tables) {
        n_entries = J->counts[b * J->H_kv + g];
        if (n_entries < 0 || n_entries > nKVmax) return ORACLE_ETABLE;
        T = J->tables + ((size_t)b * J->H_kv + g) * nKVmax;
    } else {
        n_entries = (J->chunk_start[b] + C + blk - 1) / blk;  /* nKV_b */
    }

    for (int t = 0; t < n_entries; ++t) {
        const int j = T ? T[t] : t;
        if (j < 0 || j >= nKVmax) return ORACLE_ETABLE;
        for (int c = 0; c < blk; ++c) {
            const int64_t k = (int64_t)j * blk + c;
            if (k <= p) keys[nk++] = (int32_t)k;
        }
    }
    return attention_over_keys(J, b, h, g, r, keys, nk, s, o, lse);
}

/* Softmax attention of query row (b, h, r) over the key positions keys[0, nk)
 * of KV head g, in fp64: s_k = scale * q . K[k]; LSE = log sum exp(s_k)
 * (max-subtracted); O = sum exp(s_k - LSE) V[k]. No key: O = 0, LSE = -inf. */
static int attention_over_keys(const attn_job *J, int b, int h, int g, int r,
                               const int32_t *keys, int64_t nk, double *s, double *o,
                               double *lse) {
    const int C = J->C, D = J->D;
    const size_t q0 = (((size_t)b * J->H_q + h) * C + r) * D;
    const size_t kv0 = ((size_t)b * J->H_kv + g) * (size_t)J->L_max * D;

    if (nk == 0) {
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return ORACLE_OK;
    }
    double m = -INFINITY;
    for (int64_t i = 0; i < nk; ++i) {
        const size_t k0 = kv0 + (size_t)keys[i] * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += elem(J->Q, q0 + d, J->fp8, J->q_descale) * elem(J->K, k0 + d, J->fp8, J->k_descale);
        s[i] = J->scale * dot;
        if (s[i] > m) m = s[i];
    }
    double sum = 0.0;
    for (int64_t i = 0; i < nk; ++i) sum += exp(s[i] - m);
    const double L = m + log(sum);
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t i = 0; i < nk; ++i) {
        const double w = exp(s[i] - L);
        const size_t v0 = kv0 + (size_t)keys[i] * D;
        for (int d = 0; d < D; ++d) o[d] += w * elem(J->V, v0 + d, J->fp8, J->v_descale);
    }
    *lse = L;
    return ORACLE_OK;
}

static void *attn_worker(void *arg) {
    attn_job *J = (attn_job *)arg;
    double *s = (double *)malloc(sizeof(double) * (size_t)J->L_max);
    int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)J->L_max);
    if (!s || !keys) {
        J->status = ORACLE_ENOMEM;
        free(s);
        free(keys);
        return NULL;
    }
    for (int64_t i = J->begin; i < J->end; ++i) {
        const int64_t flat = J->rows ? J->rows[i] : i;
        const int st = attention_row(J, flat, s, keys, J->O + (size_t)i * J->D, J->LSE + i);
        if (st != ORACLE_OK) {
            J->status = st;
            break;
        }
    }
    free(s);
    free(keys);
    return NULL;
}

/*
 * Attention for a list of query rows (or all B*H_q*C rows when rows == NULL).
 * Q: bf16 [B, H_q, C, D]; K, V: bf16 [B, H_kv, L_max, D];
 * tables [B, H_kv, L_max/blk] + counts [B, H_kv], or tables == NULL for the
 * dense reference (every block of the sequence's visible length).
 * Writes O (fp64, [n_rows, D]) and LSE (fp64, [n_rows]).
 */
static int run_rows(const void *Q, const void *K, const void *V, int fp8, const double *descale,
                    const int32_t *tables, const int32_t *counts, const uint8_t *tile_mask,
                    int nQ, const int32_t *chunk_start, int B, int H_q, int H_kv, int C,
                    int L_max, int D, int blk, double scale, const int64_t *rows,
                    int64_t n_rows, double *O, double *LSE, int n_threads) {
    if (!Q || !K || !V || !chunk_start || !O || !LSE || B <= 0 || H_q <= 0 || H_kv <= 0 ||
        H_q % H_kv != 0 || C <= 0 || L_max <= 0 || D <= 0 || blk <= 0 || L_max % blk != 0)
        return ORACLE_EINVAL;
    if (tables && !counts) return ORACLE_EINVAL;
    if (tile_mask && (nQ <= 0 || (int64_t)nQ * blk < C)) return ORACLE_EINVAL;
    for (int b = 0; b < B; ++b)
        if (chunk_start[b] < 0 || (int64_t)chunk_start[b] + C > L_max)
            return ORACLE_EINVAL;
    if (!rows) n_rows = (int64_t)B * H_q * C;
    for (int64_t i = 0; rows && i < n_rows; ++i)
        if (rows[i] < 0 || rows[i] >= (int64_t)B * H_q * C) return ORACLE_EINVAL;
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_rows) n_threads = (int)(n_rows > 0 ? n_rows : 1);

    attn_job *jobs = (attn_job *)calloc((size_t)n_threads, sizeof(attn_job));
    pthread_t *tid = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!jobs || !tid) {
        free(jobs);
        free(tid);
        return ORACLE_ENOMEM;
    }
    for (int w = 0; w < n_threads; ++w) {
        attn_job *J = &jobs[w];
        J->Q = Q; J->K = K; J->V = V;
        J->fp8 = fp8;
        J->q_descale = fp8 ? descale[0] : 1.0;
        J->k_descale = fp8 ? descale[1] : 1.0;
        J->v_descale = fp8 ? descale[2] : 1.0;
        J->tables = tables; J->counts = counts; J->chunk_start = chunk_start;
        J->tile_mask = tile_mask; J->nQ = nQ;
        J->B = B; J->H_q = H_q; J->H_kv = H_kv; J->C = C; J->L_max = L_max;
        J->D = D; J->blk = blk; J->scale = scale;
        J->rows = rows; J->n_rows = n_rows; J->O = O; J->LSE = LSE;
        J->begin = n_rows * w / n_threads;
        J->end = n_rows * (w + 1) / n_threads;
        J->status = ORACLE_OK;
    }
    /* A job whose thread cannot be started runs on this thread instead, so
     * every row is computed whatever the process's thread limit. */
    char *started = (char *)calloc((size_t)n_threads, 1);
    if (!started) {
        free(jobs);
        free(tid);
        return ORACLE_ENOMEM;
    }
    for (int w = 1; w < n_threads; ++w)
        started[w] = pthread_create(&tid[w], NULL, attn_worker, &jobs[w]) == 0;
    attn_worker(&jobs[0]);
    for (int w = 1; w < n_threads; ++w)
        if (!started[w]) attn_worker(&jobs[w]);
    int status = jobs[0].status;
    for (int w = 1; w < n_threads; ++w) {
        if (started[w]) pthread_join(tid[w], NULL);
        if (jobs[w].status != ORACLE_OK) status = jobs[w].status;
    }
    free(started);
    free(jobs);
    free(tid);
    return status;
}

int oracle_attention_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                          const int32_t *tables, const int32_t *counts,
                          const int32_t *chunk_start, int B, int H_q, int H_kv, int C,
                          int L_max, int D, int blk, double scale, const int64_t *rows,
                          int64_t n_rows, double *O, double *LSE, int n_threads) {
    return run_rows(Q, K, V, 0, NULL, tables, counts, NULL, 0, chunk_start, B, H_q, H_kv, C,
                    L_max, D, blk, scale, rows, n_rows, O, LSE, n_threads);
}

/*
 * The same attention on FP8 inputs: Q, K, V hold e4m3 codes and the real
 * inputs are descale[0] * Q, descale[1] * K, descale[2] * V (per-tensor
 * scale factors), each decoded exactly and then used in fp64 as above.
 */
int oracle_attention_rows_e4m3(const uint8_t *Q, const uint8_t *K, const uint8_t *V,
                               const double *descale, const int32_t *tables,
                               const int32_t *counts, const int32_t *chunk_start, int B, int H_q,
                               int H_kv, int C, int L_max, int D, int blk, double scale,
                               const int64_t *rows, int64_t n_rows, double *O, double *LSE,
                               int n_threads) {
    if (!descale) return ORACLE_EINVAL;
    return run_rows(Q, K, V, 1, descale, tables, counts, NULL, 0, chunk_start, B, H_q, H_kv, C,
                    L_max, D, blk, scale, rows, n_rows, O, LSE, n_threads);
}

/*
 * Per-tile block-sparse attention (the ablation baseline the pages set
 * against the Block-Union path: every head and Q-block keeps its own mask
 * row, no union). mask: uint8 [B, H_q, nQ, L_max / blk]; everything else as
 * in oracle_attention_rows.
 */
int oracle_attention_tile_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                               const uint8_t *mask, int nQ, const int32_t *chunk_start, int B,
                               int H_q, int H_kv, int C, int L_max, int D, int blk,
                               double scale, const int64_t *rows, int64_t n_rows, double *O,
                               double *LSE, int n_threads) {
    if (!mask) return ORACLE_EINVAL;
    return run_rows(Q, K, V, 0, NULL, NULL, NULL, mask, nQ, chunk_start, B, H_q, H_kv, C, L_max,
                    D, blk, scale, rows, n_rows, O, LSE, n_threads);
}

/*
 * Merge of two attention results over disjoint key sets of the same query
 * rows (the identity the split-KV path rests on): with w_x = exp(LSE_x - L),
 *     L = ln(exp(LSE_a) + exp(LSE_b)),   O = w_a O_a + w_b O_b,
 * evaluated with the larger LSE subtracted first; two empty inputs (LSE =
 * -inf) give O = 0, LSE = -inf. O_a, O_b, O fp64 [rows, D]; LSE fp64 [rows].
 */
int oracle_merge_states(const double *O_a, const double *LSE_a, const double *O_b,
                        const double *LSE_b, int64_t rows, int D, double *O, double *LSE) {
    if (!O_a || !LSE_a || !O_b || !LSE_b || !O || !LSE || rows < 0 || D <= 0)
        return ORACLE_EINVAL;
    for (int64_t r = 0; r < rows; ++r) {
        const double la = LSE_a[r], lb = LSE_b[r];
        const double m = la > lb ? la : lb;
        if (m == -INFINITY) {
            for (int d = 0; d < D; ++d) O[r * D + d] = 0.0;
            LSE[r] = -INFINITY;
            continue;
        }
        const double wa = exp(la - m), wb = exp(lb - m);
        const double sum = wa + wb;
        for (int d = 0; d < D; ++d)
            O[r * D + d] = (wa * O_a[r * D + d] + wb * O_b[r * D + d]) / sum;
        LSE[r] = m + log(sum);
    }
    return ORACLE_OK;
}

/*
 * Span tables for the per-tile path. The chunk's Q-blocks are taken in spans
 * of `span` consecutive Q-blocks (the last span may be short); for each
 * (b, h, span) the table lists, ascending, every KV block j that some
 * Q-block of the span selects, as the entry
 *     j | (bit u set iff Q-block span * span_index + u selects j) << 24,
 * padded with -1; counts[b, h, span] is the number of entries. Shapes:
 * tables int32 [B, H_q, nS, nKVmax], counts int32 [B, H_q, nS], nS =
 * ceil(nQ / span). Requires nKVmax < 2^24 and 1 <= span <= 7.
 */
int oracle_tile_span_tables(const uint8_t *mask, int B, int H_q, int nQ, int nKVmax, int span,
                            int32_t *tables, int32_t *counts) {
    if (!mask || !tables || !counts || B <= 0 || H_q <= 0 || nQ <= 0 || nKVmax <= 0 ||
        nKVmax >= (1 << 24) || span < 1 || span > 7)
        return ORACLE_EINVAL;
    const int nS = (nQ + span - 1) / span;
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H_q; ++h) {
            for (int sp = 0; sp < nS; ++sp) {
                const size_t item = ((size_t)b * H_q + h) * nS + sp;
                int32_t *T = tables + item * nKVmax;
                int n = 0;
                for (int j = 0; j < nKVmax; ++j) {
                    int bits = 0;
                    for (int u = 0; u < span; ++u) {
                        const int i = sp * span + u;
                        if (i < nQ && mask[(((size_t)b * H_q + h) * nQ + i) * nKVmax + j] != 0)
                            bits |= 1 << u;
                    }
                    if (bits) T[n++] = j | (bits << 24);
                }
                counts[item] = n;
                for (int t = n; t < nKVmax; ++t) T[t] = -1;
            }
        }
    }
    return ORACLE_OK;
}

/* Number of (row, key) pairs the attention above touches, per row list: the
 * "effective" work count of the selected blocks (4*D flops per pair). */
int64_t oracle_visible_pairs(const int32_t *tables, const int32_t *counts,
                             const int32_t *chunk_start, int B, int H_q, int H_kv, int C,
                             int L_max, int blk) {
    const int nKVmax = L_max / blk;
    int64_t total = 0;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H_q; ++h) {
            const int g = h / (H_q / H_kv);
            const int n = tables ? counts[b * H_kv + g] : (chunk_start[b] + C + blk - 1) / blk;
            const int32_t *T = tables ? tables + ((size_t)b * H_kv + g) * nKVmax : NULL;
            for (int r = 0; r < C; ++r) {
                const int64_t p = (int64_t)chunk_start[b] + r;
                for (int t = 0; t < n; ++t) {
                    const int64_t j = T ? T[t] : t;
                    for (int c = 0; c < blk; ++c)
                        if (j * blk + c <= p) ++total;
                }
            }
        }
    return total;
}
