/*
 * qsa_oracle.c -- plain, slow CPU statement of Qwen Sparse Attention (QSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
 * baseline load this file.  It shares no code, header, table or helper with the CUDA
 * library in block_sparse_attention_40_b200/csrc, and it never calls it.
 *
 * What it computes (one query row at a time, no blocking, no fusion):
 *
 *   Sources on the pages:
 *   - "Long context became an architecture problem", section "Linear attention carries
 *     the stream; sparse attention retrieves detail": a small indexer scores compressed
 *     key blocks; the budget is 512 blocks = 2,048 tokens; the final incomplete block
 *     stays uncompressed.
 *   - "unsloth Qwen3.8-Flash-Next GGUF" (axbrief), section "Shifting from Tokens to
 *     Micro-Blocks": micro-blocks; 24 query heads paired with 2 key-value heads.
 *   - "Qwen3.8-Flash-Next Previews Qwen4.x Architecture", "Context & Analysis" and
 *     "FAQ": the micro-blocks are 4 tokens long.
 *   - aiany.app "Qwen3.8-Flash-Next", section "Key Capabilities": the indexer is an
 *     MQA indexer (one key head shared by the indexer's query heads).
 *
 *   Parameters the pages leave open, fixed for this implementation: head_dim 128;
 *   block compression = fp32 mean of the block's per-token indexer keys; 16 indexer
 *   query heads of width 64; score s(t,b) = sum_h w[t,h] * ReLU(q_idx[t,h] . kbar[b]);
 *   one selection per token shared by all 24 heads; ties go to the lower block index.
 *
 *   Readings of the open points (each listed in the design notes):
 *   - compression order: ((k0 + k1) + k2) + k3 in fp32, times 0.25 (exact), then the
 *     stored compressed key is the bf16 round-to-nearest-even of that fp32 value;
 *   - candidates of token t are the complete blocks 0 .. floor(t/4)-1 of its own
 *     sequence ("strictly before the query's own block"), even when t's block is full;
 *   - the tail is tokens 4*floor(t/4) .. t, attended raw and causally;
 *   - when there are at most k candidates all are taken;
 *   - softmax scale 1/sqrt(128); query head h uses key/value head floor(h/12).
 *
 * Everything after the compression step is fp64.  bf16 inputs arrive as raw 16-bit
 * patterns (uint16_t) and are widened exactly.
 *
 * Pins (tests/test_oracle_*.py): a pure-Python brute force on tiny inputs, dense causal
 * GQA attention from torch's scaled_dot_product_attention when n_c <= k, exact integer
 * scores, constant-score and monotone-score closed forms, V == 1, planted needles, and
 * torch's own fp32 -> bf16 rounding for the compression.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define NH 24     /* query heads */
#define NKV 2     /* key/value heads */
#define GRP 12    /* query heads per key/value head */
#define HD 128    /* head dim */
#define NHI 16    /* indexer query heads */
#define DI 64     /* indexer width */
#define BLK 4     /* tokens per micro-block */

static float bf16_bits_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static double bf(uint16_t b) { return (double)bf16_bits_to_float(b); }

/* Round an fp32 value to the nearest bf16, ties to even (NaN kept quiet). */
static uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/*
 * Step 1: block compression.  For every sequence s (tokens cu[s] .. cu[s+1]-1) and
 * every complete block b < floor(L_s/4):
 *     kbar[off_s + b][d] = bf16_rne( fl32( fl32( fl32(k0 + k1) + k2 ) + k3 ) * 0.25 )
 * where kj = k_idx[cu[s] + 4b + j][d].  off_s = sum of floor(L_j/4) over j < s.
 */
void qsa_oracle_compress(const uint16_t *k_idx, const int64_t *cu, int32_t num_seqs,
                         uint16_t *kbar) {
    int64_t off = 0;
    for (int32_t s = 0; s < num_seqs; ++s) {
        int64_t L = cu[s + 1] - cu[s];
        int64_t nb = L / BLK;
        for (int64_t b = 0; b < nb; ++b) {
            const uint16_t *base = k_idx + (cu[s] + BLK * b) * DI;
            for (int d = 0; d < DI; ++d) {
                float a = bf16_bits_to_float(base[0 * DI + d]);
                float x1 = bf16_bits_to_float(base[1 * DI + d]);
                float x2 = bf16_bits_to_float(base[2 * DI + d]);
                float x3 = bf16_bits_to_float(base[3 * DI + d]);
                float s01 = a + x1;
                float s012 = s01 + x2;
                float s0123 = s012 + x3;
                float mean = s0123 * 0.25f;
                kbar[(off + b) * DI + d] = float_to_bf16_rne(mean);
            }
        }
        off += nb;
    }
}

/*
 * Step 2: indexer score of one block for one query token, fp64:
 *     s = sum_h w[h] * max(0, sum_d q_idx[h][d] * kbar[d])
 */
static double score_one(const uint16_t *qi, const uint16_t *w, const uint16_t *kb) {
    double s = 0.0;
    for (int h = 0; h < NHI; ++h) {
        double dot = 0.0;
        for (int d = 0; d < DI; ++d) dot += bf(qi[h * DI + d]) * bf(kb[d]);
        double r = dot > 0.0 ? dot : 0.0;
        s += bf(w[h]) * r;
    }
    return s;
}

/* Scores of explicit (row, block) pairs; used by the tests' tie-band checks. */
void qsa_oracle_score_pairs(const uint16_t *q_idx_rows, const uint16_t *w_rows,
                            const uint16_t *kbar, const int64_t *kbar_off,
                            const int64_t *row_seq, const int64_t *pair_row,
                            const int64_t *pair_block, int64_t n_pairs, double *out) {
    for (int64_t i = 0; i < n_pairs; ++i) {
        int64_t r = pair_row[i];
        int64_t s = row_seq[r];
        const uint16_t *kb = kbar + (kbar_off[s] + pair_block[i]) * DI;
        out[i] = score_one(q_idx_rows + r * NHI * DI, w_rows + r * NHI, kb);
    }
}

typedef struct { double s; int64_t b; } cand_t;

/* Order: larger score first; among equal scores the lower block index first. */
static int cand_cmp(const void *pa, const void *pb) {
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->b < b->b) ? -1 : (a->b > b->b);
}

static int idx_cmp(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * Step 3: selection.  Sort all n_c candidates by (-score, block) and keep the first
 * min(k, n_c); return them in ascending block order.  *kth receives the score of the
 * last kept block when n_c > k (the selection boundary), else -1.
 */
static int32_t select_blocks(const uint16_t *qi, const uint16_t *w, const uint16_t *kbar_seq,
                             int64_t n_c, int32_t k, int32_t *idx, double *kth) {
    if (n_c <= k) {
        for (int64_t b = 0; b < n_c; ++b) idx[b] = (int32_t)b;
        *kth = -1.0;
        return (int32_t)n_c;
    }
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)n_c);
    for (int64_t b = 0; b < n_c; ++b) {
        c[b].s = score_one(qi, w, kbar_seq + b * DI);
        c[b].b = b;
    }
    qsort(c, (size_t)n_c, sizeof(cand_t), cand_cmp);
    for (int32_t i = 0; i < k; ++i) idx[i] = (int32_t)c[i].b;
    *kth = c[k - 1].s;
    free(c);
    qsort(idx, (size_t)k, sizeof(int32_t), idx_cmp);
    return k;
}

/*
 * Step 4: attention of one query token at position t (within its sequence) over
 *     J(t) = { 4b .. 4b+3 : b selected }  U  { 4*floor(t/4) .. t },
 * one softmax over all of J(t), per query head h with key/value head floor(h/12):
 *     o[h] = sum_j softmax_j( q[h] . k[j] / sqrt(128) ) v[j]
 * k_seq, v_seq: the sequence's tokens, layout [L][2][128].
 */
static void attend_row(const uint16_t *q_row, const uint16_t *k_seq, const uint16_t *v_seq,
                       int64_t t, const int32_t *idx, int32_t cnt, double *out) {
    int64_t c = t / BLK;
    int64_t tail0 = BLK * c;
    int64_t nj = (int64_t)cnt * BLK + (t - tail0 + 1);
    int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)nj);
    int64_t n = 0;
    for (int32_t i = 0; i < cnt; ++i)
        for (int j = 0; j < BLK; ++j) tok[n++] = (int64_t)idx[i] * BLK + j;
    for (int64_t j = tail0; j <= t; ++j) tok[n++] = j;
    double *sc = (double *)malloc(sizeof(double) * (size_t)nj);
    const double scale = 1.0 / sqrt((double)HD);
    for (int h = 0; h < NH; ++h) {
        int g = h / GRP;
        double m = -INFINITY;
        for (int64_t j = 0; j < nj; ++j) {
            const uint16_t *kr = k_seq + (tok[j] * NKV + g) * HD;
            double dot = 0.0;
            for (int d = 0; d < HD; ++d) dot += bf(q_row[h * HD + d]) * bf(kr[d]);
            sc[j] = dot * scale;
            if (sc[j] > m) m = sc[j];
        }
        double z = 0.0;
        for (int64_t j = 0; j < nj; ++j) {
            sc[j] = exp(sc[j] - m);
            z += sc[j];
        }
        for (int d = 0; d < HD; ++d) {
            double acc = 0.0;
            for (int64_t j = 0; j < nj; ++j) acc += sc[j] * bf(v_seq[(tok[j] * NKV + g) * HD + d]);
            out[h * HD + d] = acc / z;
        }
    }
    free(sc);
    free(tok);
}

/*
 * Whole path for a list of query rows.  Row r is token row_pos[r] of sequence
 * row_seq[r].  Per-row inputs: q_rows [n][24][128], q_idx_rows [n][16][64],
 * w_rows [n][16].  Per-sequence inputs: k, v token-major [sum L][2][128] with
 * sequence s starting at token cu[s]; kbar packed [sum floor(L/4)][64] with sequence s
 * starting at block kbar_off[s] (as written by qsa_oracle_compress).
 *
 * If forced_idx is non-NULL the selection is not computed: row r uses
 * forced_idx[r*k .. r*k+forced_cnt[r]-1] (ascending).  Otherwise idx_out/cnt_out/kth_out
 * receive the selection (idx rows padded with -1).  If q_rows is NULL no attention is
 * computed.  Rows are independent; they are spread over n_threads OpenMP threads.
 */
void qsa_oracle_rows(const uint16_t *q_rows, const uint16_t *q_idx_rows,
                     const uint16_t *w_rows, const int64_t *row_seq,
                     const int64_t *row_pos, int64_t n_rows, const uint16_t *k,
                     const uint16_t *v, const uint16_t *kbar, const int64_t *cu,
                     const int64_t *kbar_off, int32_t topk, const int32_t *forced_idx,
                     const int32_t *forced_cnt, int32_t *idx_out, int32_t *cnt_out,
                     double *kth_out, double *out, int32_t n_threads) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t s = row_seq[r];
        int64_t t = row_pos[r];
        int64_t n_c = t / BLK;
        int32_t *idx;
        int32_t cnt;
        int32_t *own = NULL;
        if (forced_idx) {
            idx = (int32_t *)(forced_idx + r * topk);
            cnt = forced_cnt[r];
        } else {
            own = (int32_t *)malloc(sizeof(int32_t) * (size_t)topk);
            double kth;
            cnt = select_blocks(q_idx_rows + r * NHI * DI, w_rows + r * NHI,
                                kbar + kbar_off[s] * DI, n_c, topk, own, &kth);
            for (int32_t i = 0; i < topk; ++i) idx_out[r * topk + i] = i < cnt ? own[i] : -1;
            cnt_out[r] = cnt;
            kth_out[r] = kth;
            idx = own;
        }
        if (q_rows) {
            const uint16_t *ks = k + cu[s] * NKV * HD;
            const uint16_t *vs = v + cu[s] * NKV * HD;
            attend_row(q_rows + r * NH * HD, ks, vs, t, idx, cnt, out + r * NH * HD);
        }
        free(own);
    }
}

/* Geometry constants, so that the Python side can check what it was built with. */
int32_t qsa_oracle_constant(int32_t which) {
    switch (which) {
        case 0: return NH;
        case 1: return NKV;
        case 2: return HD;
        case 3: return NHI;
        case 4: return DI;
        case 5: return BLK;
        default: return -1;
    }
}
