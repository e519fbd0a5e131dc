/*
 * pspec_oracle.c -- the CPU oracle for the speculative-decoding step (TEST INFRASTRUCTURE).
 *
 * This file is test infrastructure, not product code.  Only the test suite, the
 * package's smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header, table or helper with the CUDA library: it is written from the pages'
 * statement of the method, in plain C, one obviously-correct loop per definition, with
 * every floating-point quantity carried in double precision.
 *
 * Sources (page title, section):
 *   [P1] "Eagle parallel speculative decoding, vLLM, TorchSpec" (blog.hotdry.top),
 *        section "Parallel architecture": the drafter input pairs prompt tokens with their
 *        hidden states, the first prediction slot (NTP) with h_context, and prediction
 *        slots 2..K with the mask embedding and the shared hidden state h_shared.
 *   [P1] same page, section "TorchSpec integration": the batch metadata (copy, scatter,
 *        insert, pad, mask, remap) is rebuilt on the GPU; h_shared is broadcast into the
 *        mask slots by a separate copy; rejected tokens map to PADDING_SLOT_ID = -1.
 *   [P3] "Capstone 14: speculative decoding inference server", section "Concept": the
 *        target checks all k drafts in one forward pass and any accepted prefix replaces
 *        the greedy path; section "Architecture": accept the prefix, resample the rejected
 *        suffix.
 *   [P2] rskf.cn article, section 2.2 (table row "target model"): the output must be
 *        identical to plain autoregressive decoding.
 * The acceptance rule itself (accept draft t with probability min(1, p(t)/q(t)); at the
 * first rejection draw from norm(max(0, p - q)); when all K drafts pass draw the bonus
 * from the target's last row) is the standard rule that meets [P2]'s losslessness
 * requirement; the pages do not print it.
 *
 * Readings taken where the pages are silent (each is also listed in the design notes):
 *   R1  accept iff u < p/q, with u in [0,1); when q = 0 accept iff p > 0.
 *   R2  an accept decision with |u - p/q| < tie_eps is flagged (bit 0 of flags).
 *   R3  the resample is an inverse CDF in token-id order: the smallest t with
 *       sum_{v<=t} r_v > u_K * Z.  If rounding leaves no such t, the last t with r_t > 0.
 *       If Z = 0 the draw falls back to the target row p itself.  A draw whose u_K*Z lies
 *       within tie_eps*Z of a CDF boundary is flagged (bit 1 of flags).
 *   R4  greedy argmax takes the lowest token id among equal maxima.
 *   R5  a draft token outside [0, V) is never accepted (p = q = 0 for it) and raises
 *       error bit 0x1.
 *   R6  draft-batch layout per sequence i with L_i verify rows, a_i accepted drafts and
 *       c_i = L_i - K + a_i surviving rows: [c_i - 1 context rows | 1 NTP row | K-1 MASK
 *       rows | K - a_i rejected rows].  Context row j carries token j+1 with hidden j (the
 *       EAGLE pairing), the NTP row carries the bonus token with hidden c_i - 1
 *       (h_context), MASK row m carries mask_id with h_shared at position NTP + m, and the
 *       rejected rows carry pad_id, their old verify position and slot -1.  Padding rows
 *       after the last span carry pad_id, position 0 and slot -1.
 *   R8  draft sampling draws each of the drafter's K output rows by the same inverse-CDF
 *       convention as R3 (u in [0,1), token-id order) from softmax(row); without uniforms
 *       it takes the argmax (R4).  A draw within tie_eps of a CDF boundary is flagged.
 *   R7  invalid values never stop the oracle: accepted counts are clamped into [0, K]
 *       (error bit 0x2), out-of-range block lookups give slot -1 (error bit 0x4), a
 *       sequence with L_i < K+1 keeps its span as padding rows with seq_len 0 and sample
 *       index -1 (error bit 0x8), and a qsl_in that is not an offset array (qsl_in[0] != 0,
 *       decreasing, or past T_in) rejects the whole batch (error bit 0x8; every row padding).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "pspec_oracle.h"

/* ---- element access: logits are fp32 or bf16 (upper half of an IEEE fp32) ---- */
static double logit_at(const void *base, int dtype, long long idx)
{
    if (dtype == ORACLE_F32) {
        return (double)((const float *)base)[idx];
    }
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* max over a row (used as the shift of the log-sum-exp) */
static double row_max(const void *base, int dtype, long long off, int V)
{
    double m = -INFINITY;
    for (int t = 0; t < V; ++t) {
        double x = logit_at(base, dtype, off + t);
        if (x > m) m = x;
    }
    return m;
}

/* log sum_t exp(x_t), the softmax normaliser of one row */
static double row_logsumexp(const void *base, int dtype, long long off, int V)
{
    double m = row_max(base, dtype, off, V);
    if (m == -INFINITY) return -INFINITY;
    double s = 0.0;
    for (int t = 0; t < V; ++t) s += exp(logit_at(base, dtype, off + t) - m);
    return m + log(s);
}

/* softmax probability of token t in a row with normaliser lse */
static double row_prob(const void *base, int dtype, long long off, int t, double lse)
{
    if (lse == -INFINITY) return 0.0;
    return exp(logit_at(base, dtype, off + t) - lse);
}

/* argmax with the lowest id winning ties (R4): a strict '>' scan */
static int row_argmax(const void *base, int dtype, long long off, int V)
{
    int best = 0;
    double bv = logit_at(base, dtype, off);
    for (int t = 1; t < V; ++t) {
        double x = logit_at(base, dtype, off + t);
        if (x > bv) { bv = x; best = t; }
    }
    return best;
}

/* R14: sequence i's own draft count K_i (k_len[i]; K when k_len is NULL), clamped into
   [0, K] with error bit 0x20 when outside */
static int draft_count(const int *k_len, int i, int K, int *e)
{
    if (!k_len) return K;
    int k = k_len[i];
    if (k < 0 || k > K) { *e |= 0x20; k = k < 0 ? 0 : K; }
    return k;
}

int oracle_verify_greedy(int B, int K, int V, long long ld, int dtype,
                         const void *target_logits, const int *draft_tokens,
                         const int *k_len,
                         int *out_tokens, int *accepted_len, int *bonus,
                         double *target_lse, int *err)
{
    if (B < 0 || K < 1 || V < 1 || ld < V) return 1;
    int e = 0;
    int *amax = (int *)malloc(sizeof(int) * (size_t)(K + 1));
    if (!amax) return 1;
    for (int i = 0; i < B; ++i) {
        /* target argmax of every verify row k = 0..K */
        for (int k = 0; k <= K; ++k) {
            long long off = ((long long)i * (K + 1) + k) * ld;
            amax[k] = row_argmax(target_logits, dtype, off, V);
            if (target_lse) target_lse[(long long)i * (K + 1) + k] =
                row_logsumexp(target_logits, dtype, off, V);
        }
        /* accepted prefix: drafts that equal the greedy choice, in order [P3 Concept];
           only the sequence's own K_i drafts are tested (R14) */
        const int Ki = draft_count(k_len, i, K, &e);
        int a = 0;
        while (a < Ki) {
            int d = draft_tokens[(long long)i * K + a];
            if (d < 0 || d >= V) { e |= 0x1; break; }
            if (d != amax[a]) break;
            ++a;
        }
        for (int k = a; k < Ki; ++k) {    /* R5: range errors past the prefix count too */
            int d = draft_tokens[(long long)i * K + k];
            if (d < 0 || d >= V) e |= 0x1;
        }
        int *out = out_tokens + (long long)i * (K + 1);
        for (int k = 0; k < a; ++k) out[k] = draft_tokens[(long long)i * K + k];
        out[a] = amax[a];                 /* the bonus: greedy token after the prefix */
        for (int k = a + 1; k <= K; ++k) out[k] = -1;
        accepted_len[i] = a;
        bonus[i] = amax[a];
    }
    free(amax);
    if (err) *err |= e;
    return 0;
}

int oracle_verify_rejection(int B, int K, int V, long long ld, int dtype,
                            const void *target_logits, const void *draft_logits,
                            const int *draft_tokens, const float *uniforms,
                            const int *k_len, int *out_tokens, int *accepted_len, int *bonus,
                            double *p_at_draft, double *q_at_draft,
                            double *target_lse, double *draft_lse,
                            double *residual_mass, int *flags, double tie_eps, int *err)
{
    if (B < 0 || K < 1 || V < 1 || ld < V) return 1;
    int e = 0;
    double *lse_t = (double *)malloc(sizeof(double) * (size_t)(K + 1));
    double *lse_q = (double *)malloc(sizeof(double) * (size_t)K);
    double *pk = (double *)malloc(sizeof(double) * (size_t)K);
    double *qk = (double *)malloc(sizeof(double) * (size_t)K);
    double *r = (double *)malloc(sizeof(double) * (size_t)V);
    if (!lse_t || !lse_q || !pk || !qk || !r) {
        free(lse_t); free(lse_q); free(pk); free(qk); free(r);
        return 1;
    }

    for (int i = 0; i < B; ++i) {
        const int *d = draft_tokens + (long long)i * K;
        const float *u = uniforms + (long long)i * (K + 1);
        int flag = 0;
        const int Ki = draft_count(k_len, i, K, &e);       /* R14 */

        /* softmax normalisers of the K+1 target rows and the K draft rows */
        for (int k = 0; k <= K; ++k) {
            lse_t[k] = row_logsumexp(target_logits, dtype, ((long long)i * (K + 1) + k) * ld, V);
            if (target_lse) target_lse[(long long)i * (K + 1) + k] = lse_t[k];
        }
        for (int k = 0; k < K; ++k) {
            lse_q[k] = row_logsumexp(draft_logits, dtype, ((long long)i * K + k) * ld, V);
            if (draft_lse) draft_lse[(long long)i * K + k] = lse_q[k];
        }

        /* p(d_k) and q(d_k) for every draft position */
        for (int k = 0; k < K; ++k) {
            pk[k] = 0.0;
            qk[k] = 0.0;
            if (d[k] >= 0 && d[k] < V) {
                pk[k] = row_prob(target_logits, dtype, ((long long)i * (K + 1) + k) * ld, d[k], lse_t[k]);
                qk[k] = row_prob(draft_logits, dtype, ((long long)i * K + k) * ld, d[k], lse_q[k]);
            } else if (k < Ki) {
                e |= 0x1;                 /* R5 (the sequence's own drafts only) */
            }
            if (p_at_draft) p_at_draft[(long long)i * K + k] = pk[k];
            if (q_at_draft) q_at_draft[(long long)i * K + k] = qk[k];
        }

        /* accept drafts in order with probability min(1, p/q); stop at the first rejection */
        int a = Ki;
        for (int k = 0; k < Ki; ++k) {
            int accept;
            if (qk[k] > 0.0) {
                double ratio = pk[k] / qk[k];
                accept = (double)u[k] < ratio;                      /* R1 */
                if (fabs((double)u[k] - ratio) < tie_eps) flag |= 1; /* R2 */
            } else {
                accept = pk[k] > 0.0;
            }
            if (!accept) { a = k; break; }
        }

        /* the distribution to draw from: norm(max(0, p_a - q_a)) after a rejection,
           the target's row K_i when every draft passed */
        long long toff = ((long long)i * (K + 1) + a) * ld;
        double Z = 0.0;
        if (a < Ki) {
            long long qoff = ((long long)i * K + a) * ld;
            for (int t = 0; t < V; ++t) {
                double diff = row_prob(target_logits, dtype, toff, t, lse_t[a]) -
                              row_prob(draft_logits, dtype, qoff, t, lse_q[a]);
                r[t] = diff > 0.0 ? diff : 0.0;
                Z += r[t];
            }
        }
        if (a == Ki || Z == 0.0) {       /* R3: Z = 0 falls back to p itself */
            Z = 0.0;
            for (int t = 0; t < V; ++t) {
                r[t] = row_prob(target_logits, dtype, toff, t, lse_t[a]);
                Z += r[t];
            }
        }
        if (residual_mass) residual_mass[i] = Z;

        /* inverse CDF in token-id order (R3), driven by uniform column K_i (R4, R14) */
        double thr = (double)u[Ki] * Z;
        double cum = 0.0, prev = 0.0;
        int tok = -1, last_pos = -1;
        for (int t = 0; t < V; ++t) {
            if (r[t] > 0.0) last_pos = t;
            prev = cum;
            cum += r[t];
            if (cum > thr) { tok = t; break; }
        }
        if (tok < 0) {
            tok = last_pos >= 0 ? last_pos : 0;
            flag |= 2;
        } else if (thr - prev < tie_eps * Z || cum - thr < tie_eps * Z) {
            flag |= 2;
        }

        int *out = out_tokens + (long long)i * (K + 1);
        for (int k = 0; k < a; ++k) out[k] = d[k];
        out[a] = tok;
        for (int k = a + 1; k <= K; ++k) out[k] = -1;
        accepted_len[i] = a;
        bonus[i] = tok;
        if (flags) flags[i] = flag;
    }
    free(lse_t);
    free(lse_q);
    free(pk);
    free(qk);
    free(r);
    if (err) *err |= e;
    return 0;
}

int oracle_sample_rows(int N, int V, long long ld, int dtype, const void *logits,
                       const float *uniforms, int *tokens, double *probs, int *flags,
                       double tie_eps)
{
    if (N < 0 || V < 1 || ld < V) return 1;
    for (int n = 0; n < N; ++n) {
        long long off = (long long)n * ld;
        double lse = row_logsumexp(logits, dtype, off, V);
        int tok, flag = 0;
        if (!uniforms) {
            tok = row_argmax(logits, dtype, off, V);
        } else {
            /* inverse CDF of the softmax in token-id order (R3, R8) */
            double Z = 0.0;
            for (int t = 0; t < V; ++t) Z += row_prob(logits, dtype, off, t, lse);
            double thr = (double)uniforms[n] * Z, cum = 0.0, prev = 0.0;
            int last_pos = -1;
            tok = -1;
            for (int t = 0; t < V; ++t) {
                double p = row_prob(logits, dtype, off, t, lse);
                if (p > 0.0) last_pos = t;
                prev = cum;
                cum += p;
                if (cum > thr) { tok = t; break; }
            }
            if (tok < 0) {
                tok = last_pos >= 0 ? last_pos : 0;
                flag = 2;
            } else if (thr - prev < tie_eps * Z || cum - thr < tie_eps * Z) {
                flag = 2;
            }
        }
        tokens[n] = tok;
        if (probs) probs[n] = row_prob(logits, dtype, off, tok, lse);
        if (flags) flags[n] = flag;
    }
    return 0;
}

/* slot of token position pos of sequence i in the paged KV cache:
   block_table[i][pos / bs] * bs + pos % bs, or -1 when the lookup is out of range */
static long long kv_slot(const int *block_table, int max_blocks, int block_size, int i,
                         int pos, int *e)
{
    if (pos < 0) { *e |= 0x4; return -1; }
    int blk = pos / block_size;
    if (blk >= max_blocks) { *e |= 0x4; return -1; }
    int id = block_table[(long long)i * max_blocks + blk];
    if (id < 0) { *e |= 0x4; return -1; }
    return (long long)id * block_size + pos % block_size;
}

int oracle_build_draft_batch(int B, int K, int H, int hidden_elem_bytes,
                             int block_size, int max_blocks, int mask_id, int pad_id,
                             int T_in, int T_cap,
                             const int *qsl_in, const int *verify_tokens, const int *verify_pos,
                             const int *accepted_len, const int *bonus, const int *k_len,
                             const int *block_table,
                             const void *verify_hidden, const void *h_shared,
                             int *draft_tokens, int *draft_pos, long long *slot_mapping,
                             unsigned char *row_kind, int *hidden_src,
                             int *qsl_out, int *seq_lens_out, int *sample_idx,
                             void *draft_hidden, int *err)
{
    if (B < 0 || K < 1 || H < 1 || block_size < 1 || max_blocks < 1 || T_in < 0) return 1;
    if ((long long)T_cap < (long long)T_in + (long long)B * (K - 1)) return 1;
    int e = 0;
    size_t row_bytes = (size_t)H * (size_t)hidden_elem_bytes;
    unsigned char *dh = (unsigned char *)draft_hidden;
    const unsigned char *vh = (const unsigned char *)verify_hidden;

    /* every row starts as padding; the spans below overwrite their own rows */
    for (int row = 0; row < T_cap; ++row) {
        draft_tokens[row] = pad_id;
        draft_pos[row] = 0;
        slot_mapping[row] = -1;
        row_kind[row] = ORACLE_ROW_PAD;
        hidden_src[row] = -1;
    }

    /* the verify layout must be offsets: qsl_in[0] = 0, non-decreasing, qsl_in[B] <= T_in.
       Otherwise the batch is rejected as a whole (error bit 0x8) and left as padding. */
    int layout_ok = 1;
    if (B > 0 && qsl_in[0] != 0) layout_ok = 0;
    for (int i = 0; i < B; ++i)
        if (qsl_in[i + 1] < qsl_in[i]) layout_ok = 0;
    if (B > 0 && qsl_in[B] > T_in) layout_ok = 0;
    if (!layout_ok) {
        for (int i = 0; i <= B; ++i) qsl_out[i] = 0;
        for (int i = 0; i < B; ++i) {
            seq_lens_out[i] = 0;
            for (int k = 0; k < K; ++k) sample_idx[(long long)i * K + k] = -1;
        }
        if (err) *err |= 0x8;
        return 0;
    }

    /* output offsets: each span holds its L_i verify rows plus K-1 inserted mask rows */
    int off = 0;
    for (int i = 0; i < B; ++i) {
        qsl_out[i] = off;
        off += (qsl_in[i + 1] - qsl_in[i]) + K - 1;
    }
    qsl_out[B] = off;

    for (int i = 0; i < B; ++i) {
        int s = qsl_in[i];
        int L = qsl_in[i + 1] - qsl_in[i];
        int o = qsl_out[i];
        /* R14: the span's last K_i verify rows held this step's drafts; the next step still
           gets K-1 mask slots */
        const int Ki = draft_count(k_len, i, K, &e);
        if (L < Ki + 1) {                 /* R7: too short to hold its drafts; stays padding */
            e |= 0x8;
            seq_lens_out[i] = 0;
            for (int k = 0; k < K; ++k) sample_idx[(long long)i * K + k] = -1;
            continue;
        }
        int a = accepted_len[i];
        if (a < 0 || a > Ki) { e |= 0x2; a = a < 0 ? 0 : Ki; }
        int c = L - Ki + a;               /* surviving verify rows; the last one is h_context */
        int ntp_pos = verify_pos[s + c - 1];

        for (int j = 0; j < L + K - 1; ++j) {
            int row = o + j;
            int tok, pos, src, kind;
            long long slot;
            if (j < c - 1) {              /* context: token j+1 paired with hidden j */
                tok = verify_tokens[s + j + 1];
                pos = verify_pos[s + j];
                src = s + j;
                kind = ORACLE_ROW_CTX;
                slot = kv_slot(block_table, max_blocks, block_size, i, pos, &e);
            } else if (j == c - 1) {      /* NTP: bonus token paired with h_context */
                tok = bonus[i];
                pos = ntp_pos;
                src = s + j;
                kind = ORACLE_ROW_NTP;
                slot = kv_slot(block_table, max_blocks, block_size, i, pos, &e);
            } else if (j < c + K - 1) {   /* MASK m = 1..K-1: mask token with h_shared */
                int m = j - (c - 1);
                tok = mask_id;
                pos = ntp_pos + m;
                src = -1;
                kind = ORACLE_ROW_MASK;
                slot = kv_slot(block_table, max_blocks, block_size, i, pos, &e);
            } else {                      /* rejected verify rows, kept at the tail */
                int v = c + (j - (c + K - 1));
                tok = pad_id;
                pos = verify_pos[s + v];
                src = -1;
                kind = ORACLE_ROW_REJ;
                slot = -1;                /* PADDING_SLOT_ID */
            }
            draft_tokens[row] = tok;
            draft_pos[row] = pos;
            slot_mapping[row] = slot;
            row_kind[row] = (unsigned char)kind;
            hidden_src[row] = src;
            if (draft_hidden) {
                if (kind == ORACLE_ROW_CTX || kind == ORACLE_ROW_NTP)
                    memcpy(dh + (size_t)row * row_bytes, vh + (size_t)src * row_bytes, row_bytes);
                else if (kind == ORACLE_ROW_MASK)
                    memcpy(dh + (size_t)row * row_bytes, h_shared, row_bytes);
            }
        }
        seq_lens_out[i] = ntp_pos + K;    /* last mask position + 1 */
        for (int k = 0; k < K; ++k) sample_idx[(long long)i * K + k] = o + c - 1 + k;
    }
    if (err) *err |= e;
    return 0;
}
