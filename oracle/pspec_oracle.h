/*
 * pspec_oracle.h -- declarations of the CPU oracle (TEST INFRASTRUCTURE ONLY).
 *
 * Only the test suite, the package smoke check and the benchmark's CPU-baseline leg may
 * load this library.  It shares nothing with the CUDA library's headers.  Every pointer
 * is host memory owned by the caller; every function returns 0 on success and 1 on a
 * malformed call (negative sizes, too small a capacity).  Invalid *values* (tokens out of
 * range, accepted counts out of range, block lookups past the table) never stop it: they
 * OR bits into *err (0x1 token range, 0x2 accepted count, 0x4 block lookup, 0x8 layout,
 * 0x20 draft count).
 *
 * k_len (every function that takes it; NULL = K for every sequence): sequence i's own draft
 * count K_i in [0, K] (R14).  Sequence i is then verified exactly as if it were alone with
 * K = K_i: drafts 0..K_i-1 are tested (with uniforms 0..K_i-1), the bonus after K_i
 * acceptances comes from target row K_i, the draw uses uniform column K_i, and only those
 * drafts are range-checked; out_tokens keeps K+1 columns (-1 after the bonus).  In the
 * draft batch K_i sets how many of the span's verify rows were drafts (c_i = L_i - K_i +
 * a_i survive); every span still gets K-1 mask rows.
 */
#ifndef PSPEC_ORACLE_H
#define PSPEC_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };
enum { ORACLE_ROW_CTX = 0, ORACLE_ROW_NTP = 1, ORACLE_ROW_MASK = 2, ORACLE_ROW_REJ = 3,
       ORACLE_ROW_PAD = 4 };

/* Greedy verify.  target_logits: [B, K+1, ld] (V valid columns); draft_tokens: [B, K].
   Outputs out_tokens [B, K+1] (-1 after the bonus), accepted_len [B], bonus [B] and,
   when non-NULL, target_lse [B, K+1] in double. */
int oracle_verify_greedy(int B, int K, int V, long long ld, int dtype,
                         const void *target_logits, const int *draft_tokens,
                         const int *k_len, int *out_tokens, int *accepted_len, int *bonus,
                         double *target_lse, int *err);

/* Rejection-rule verify.  draft_logits: [B, K, ld]; uniforms: [B, K+1] in [0,1), column K
   drives the resample or bonus draw.  Optional double outputs (NULL skips): p_at_draft and
   q_at_draft [B, K], target_lse [B, K+1], draft_lse [B, K], residual_mass [B].  flags [B]
   (optional): bit 0 = an accept decision within tie_eps of u, bit 1 = a resample draw
   within tie_eps*Z of a CDF boundary. */
int oracle_verify_rejection(int B, int K, int V, long long ld, int dtype,
                            const void *target_logits, const void *draft_logits,
                            const int *draft_tokens, const float *uniforms,
                            const int *k_len, int *out_tokens, int *accepted_len, int *bonus,
                            double *p_at_draft, double *q_at_draft,
                            double *target_lse, double *draft_lse,
                            double *residual_mass, int *flags, double tie_eps, int *err);

/* Draft sampling from the drafter's output rows: N rows of logits [N, ld] (V valid).
   With uniforms [N] in [0,1): tokens[n] = the smallest t whose cumulative softmax exceeds
   u_n (token-id order; if rounding leaves none, the last t with positive probability);
   flags[n] bit 1 marks a draw within tie_eps of a boundary.  With uniforms NULL: the
   argmax, lowest id on ties.  probs[n] (optional) = softmax probability of the token. */
int oracle_sample_rows(int N, int V, long long ld, int dtype, const void *logits,
                       const float *uniforms, int *tokens, double *probs, int *flags,
                       double tie_eps);

/* P-EAGLE draft-batch construction.  Inputs: qsl_in [B+1], verify_tokens [T_in],
   verify_pos [T_in], accepted_len [B], bonus [B], block_table [B, max_blocks],
   verify_hidden [T_in, H] and h_shared [H] (hidden_elem_bytes per element; NULL
   draft_hidden skips the hidden rows).  Outputs for T_cap rows: draft_tokens, draft_pos,
   slot_mapping (int64), row_kind (u8), hidden_src; qsl_out [B+1], seq_lens_out [B],
   sample_idx [B, K], draft_hidden [T_cap, H] (rejected and padding rows left as they were). */
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
                             void *draft_hidden, int *err);

#ifdef __cplusplus
}
#endif
#endif
