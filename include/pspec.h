/*
 * pspec.h -- C ABI of libpspec: the per-step hot path of speculative decoding with
 * P-EAGLE parallel drafting, on one NVIDIA B200 (sm_100a).
 *
 * Three operations, each one or two hand-written CUDA kernels:
 *
 *   pspec_verify_greedy       target verification, greedy rule
 *   pspec_verify_rejection    target verification, rejection rule
 *   pspec_build_draft_batch   parallel-draft batch construction
 *
 * Sources (page title, section):
 *   "Capstone 14: speculative decoding inference server", section "Concept": the target
 *     checks the k drafts in one forward pass and an accepted prefix replaces the greedy
 *     path; section "Architecture": accept the prefix, resample for the rejected suffix.
 *   rskf.cn speculative-decoding article, section 2.2 (table row "target model"): the
 *     output must be identical to plain autoregressive decoding.  Section 2.1 names the
 *     vocabulary-wide softmax and the memory-bandwidth bound of decode.
 *   "Eagle parallel speculative decoding, vLLM, TorchSpec", section "Parallel
 *     architecture": drafter inputs pair context tokens with their hidden states, the
 *     next-token slot with h_context and prediction slots 2..K with a mask token and the
 *     shared hidden state h_shared; section "TorchSpec integration": the draft batch
 *     metadata (copy, scatter, insert, pad, mask, remap) is rebuilt on the GPU, h_shared
 *     is broadcast into the mask slots by a separate copy, and rejected tokens take
 *     PADDING_SLOT_ID = -1 in the KV slot mapping.
 *
 * Conventions shared by every entry point:
 *   - Every array pointer is caller-owned DEVICE memory (cudaMalloc / torch tensors).  The
 *     argument structs themselves are host memory and are read before the call returns.
 *   - Calls are asynchronous on the caller's stream: the library never synchronises the
 *     host, never allocates, and launches nothing outside the given stream.
 *   - Host-side checks (null pointers, sizes, alignment, capacity) return an error status
 *     and launch nothing.  Invalid VALUES found on the device (a token outside [0, V), an
 *     accepted count outside [0, K], a block lookup outside the table, a malformed query
 *     offset array) never trap: the kernel ORs a PSPEC_DEVERR_* bit into *err and writes a
 *     documented safe output instead.  *err is only ever OR-ed, so zero it before a call
 *     whose bits you want to read alone.
 *   - Results are deterministic: repeated calls on the same inputs give bit-identical
 *     outputs (segment partials are merged in a fixed order; no floating-point atomics).
 */
#ifndef PSPEC_H
#define PSPEC_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define PSPEC_API __attribute__((visibility("default")))
#else
#define PSPEC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PSPEC_OK = 0,
  PSPEC_ERR_INVALID_ARG = 1,  /* a host-side check failed; nothing was launched */
  PSPEC_ERR_UNSUPPORTED = 2,  /* a valid but unsupported request (e.g. K > 31) */
  PSPEC_ERR_CUDA = 3,         /* a launch failed; cudaGetLastError() has the cause */
  PSPEC_ERR_WORKSPACE = 4     /* workspace pointer NULL, misaligned or too small */
} pspec_status;

typedef enum { PSPEC_F32 = 0, PSPEC_BF16 = 1 } pspec_dtype;

/* Bits OR-ed into the device error word. */
#define PSPEC_DEVERR_TOKEN_RANGE 0x1   /* draft token outside [0, V): never accepted */
#define PSPEC_DEVERR_ACCEPT_RANGE 0x2  /* accepted_len outside [0, K]: clamped into it */
#define PSPEC_DEVERR_BLOCK_RANGE 0x4   /* position < 0, pos/block_size >= max_blocks or a
                                          negative block id: that row's slot is -1 */
#define PSPEC_DEVERR_LAYOUT 0x8        /* qsl_in not an offset array, or a sequence with
                                          fewer than K+1 verify rows */
#define PSPEC_DEVERR_KLEN_RANGE 0x20   /* k_len[i] outside [0, K]: clamped into it */

/* Row kinds written to pspec_build_args.row_kind. */
#define PSPEC_ROW_CTX 0   /* context row: accepted token paired with its target hidden */
#define PSPEC_ROW_NTP 1   /* next-token row: bonus token paired with h_context */
#define PSPEC_ROW_MASK 2  /* prediction slot 2..K: mask token paired with h_shared */
#define PSPEC_ROW_REJ 3   /* rejected verify row: pad token, slot -1, hidden unwritten */
#define PSPEC_ROW_PAD 4   /* capacity padding: pad token, position 0, slot -1 */

#define PSPEC_PADDING_SLOT_ID (-1)
#define PSPEC_MAX_K 31    /* the accept decisions of one sequence live in one 32-bit mask */

/*
 * Tuning of one call (the pages have no counterpart: these choose among equivalent
 * implementations and never change a result).  A verify or step call whose
 * pspec_verify_args.options is non-NULL runs with exactly these values; with NULL it runs
 * with the process-wide defaults that the pspec_set_* functions below change.  The struct
 * is read before the call returns.  0 in any field means the automatic choice; values
 * outside the documented range read as 0.
 */
typedef struct {
  int verify_path;           /* 0 automatic, 1 full sweep, 2 early exit (see
                                pspec_set_verify_path) */
  int cluster_size;          /* early exit: CTAs per cluster, 2, 4, 8, 12 or 16; 0 automatic */
  int tail_split;            /* early exit: sequences of the second, wider launch; 0 automatic,
                                -1 never, n > 0 that many (at most half the batch) */
  int step_fusion;           /* pspec_step_*: 0 automatic, 1 always one launch, 2 never */
  long long segment_elems;   /* full sweep: elements of one row per CTA (rounded up to a
                                multiple of 8); 0 automatic.  Changes the workspace size:
                                see pspec_verify_workspace_bytes_opt. */
} pspec_options;

/*
 * Verification arguments.
 *
 * Layout: logits rows are row-major with a row stride of `ld` elements (ld >= V); row k of
 * sequence i is at base + (i*(K+1) + k)*ld for the target and base + (i*K + k)*ld for the
 * draft.  Bases need only element alignment; V and ld may be anything.  Rows are streamed
 * with 16-byte loads from their first 16-byte boundary on; an unaligned head and a ragged
 * tail (fewer than 8 bf16 / 4 fp32 elements each) are read with scalar loads, so rows
 * that start on a 16-byte boundary (base 16-byte aligned, ld*sizeof(elem) a multiple of
 * 16) are read fastest.
 */
typedef struct {
  int B;                       /* sequences; B = 0 is a no-op */
  int K;                       /* drafts per sequence, 1 <= K <= PSPEC_MAX_K */
  int V;                       /* vocabulary size, >= 1 */
  long long ld;                /* row stride of the logits in elements, >= V */
  pspec_dtype dtype;           /* logits dtype (both sides) */
  const void *target_logits;   /* [B, K+1, ld] target rows; row k scores position k */
  const void *draft_logits;    /* [B, K, ld] draft rows (rejection only; else NULL) */
  const int32_t *draft_tokens; /* [B, K] drafted token ids */
  const float *uniforms;       /* [B, K+1] in [0,1) (rejection only): column k < K is the
                                  accept test of draft k, column K drives the resample or
                                  bonus draw.  The caller owns the random numbers, so
                                  results do not depend on any generator in the library. */
  int32_t *out_tokens;         /* [B, K+1] out: accepted drafts, then the bonus token, then
                                  -1 up to K+1 entries */
  int32_t *accepted_len;       /* [B] out: a_i in [0, K] */
  int32_t *bonus;              /* [B] out: the token emitted after the accepted prefix */
  /* Optional fp32 diagnostics (NULL skips each): */
  float *target_lse;           /* [B, K+1] log-sum-exp of each target row */
  float *draft_lse;            /* [B, K]   log-sum-exp of each draft row (rejection) */
  float *p_at_draft;           /* [B, K]   target softmax probability of draft k (rejection) */
  float *q_at_draft;           /* [B, K]   draft softmax probability of draft k (rejection) */
  float *residual_mass;        /* [B]      Z = sum max(0, p - q) of the resampled row, or
                                           sum p of the bonus row (rejection) */
  int32_t *err;                /* device error word (required); bits are OR-ed in */
  const int32_t *k_len;        /* [B] per-sequence draft counts K_i in [0, K], or NULL for K
                                  everywhere ("dynamic draft length", rskf.cn article,
                                  section 3.2, MTP): sequence i is verified as if it were
                                  alone with K = K_i -- drafts 0..K_i-1 tested with uniforms
                                  0..K_i-1, the bonus after K_i acceptances from target row
                                  K_i, the draw on uniform column K_i, only those drafts
                                  range-checked; rows past K_i are never needed (the
                                  early-exit path never reads them). */
  const pspec_options *options; /* tuning of this call, or NULL for the process-wide
                                  defaults (pspec_set_*) */
} pspec_verify_args;

/*
 * Workspace for the verify calls: scratch device memory owned by the caller, at least
 * pspec_verify_workspace_bytes(B, K, V, rejection) bytes, 256-byte aligned.  It must be
 * zero-filled once (cudaMemsetAsync) before its first use; every call leaves its
 * counters back at zero, so later calls need no re-initialisation.  The counters sit at
 * the end of the workspace (the address plus the byte count passed with each call, so
 * pass the same count every time), at addresses that depend on neither B nor K: a
 * workspace sized for B sequences serves every later call with at most B sequences, on
 * any verify path.  Calls that share one workspace must not overlap on the GPU (use one
 * workspace per stream).
 */
PSPEC_API size_t pspec_verify_workspace_bytes(int B, int K, int V, int rejection);

/* The same for calls made with `options` (NULL: the process-wide defaults); only
   options->segment_elems changes the size. */
PSPEC_API size_t pspec_verify_workspace_bytes_opt(int B, int K, int V, int rejection,
                                                  const pspec_options *options);

/*
 * Greedy verification ("any accepted prefix replaces the greedy path").
 * For each sequence i: g_k = argmax over the vocabulary of target row k (the lowest id
 * wins ties); a_i = the number of leading drafts with d_k == g_k; bonus = g_{a_i};
 * out_tokens = [d_0 .. d_{a_i-1}, bonus, -1 ...].  target_lse is written when non-NULL.
 * One kernel launch (two when the early-exit path splits a large batch).  Full sweep: all
 * B*(K+1) target rows, the last CTA of each sequence combining its row partials.  Early
 * exit (see pspec_set_verify_path): one cluster of CTAs per sequence reads rows 0, 1, ...
 * in order and stops at the first mismatch.  Errors: PSPEC_ERR_INVALID_ARG for bad
 * arguments; a draft token outside [0, V) is treated as a mismatch and sets
 * PSPEC_DEVERR_TOKEN_RANGE.
 */
PSPEC_API pspec_status pspec_verify_greedy(const pspec_verify_args *args, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream);

/*
 * Rejection-rule verification ("accept prefix; resample for rejected suffix", lossless).
 * p_k = softmax(target row k), q_k = softmax(draft row k).  Draft k is accepted iff
 * u_k * q_k(d_k) < p_k(d_k) (that is, with probability min(1, p/q)); a_i is the first
 * rejected position, K if none.  The emitted token after the prefix is drawn by inverse
 * CDF in token-id order with u_K: from r = max(0, p_{a_i} - q_{a_i}) after a rejection,
 * from r = p_K when every draft passed; token = the smallest t with
 * sum_{v<=t} r_v > u_K * sum r (if rounding leaves none, the last t with r_t > 0; if the
 * residual sums to zero, the draw uses p_{a_i} itself).  Full sweep: two launches, a
 * vocabulary sweep over the 2K+1 rows of every sequence (softmax statistics and the
 * accept mask), then a chunked inverse-CDF draw over each sequence's row a_i.  Early exit
 * (see pspec_set_verify_path): one launch (two when a large batch is split), one cluster of
 * CTAs per sequence streaming the target and draft rows of positions 0, 1, ... and stopping
 * at the first rejection, where it re-reads that position's rows for the draw.  A draft
 * token outside [0, V) has p = q = 0, is rejected, and sets PSPEC_DEVERR_TOKEN_RANGE.
 */
PSPEC_API pspec_status pspec_verify_rejection(const pspec_verify_args *args, void *workspace,
                                    size_t workspace_bytes, cudaStream_t stream);

/*
 * Draft-token sampling ("Eagle parallel speculative decoding, vLLM, TorchSpec", section
 * "Parallel architecture": the P-EAGLE drafter predicts its K draft tokens from K output
 * rows of one forward pass).  For every row (i, k) of logits [B, K, ld] (V valid, any
 * alignment of the base to its element size): with uniforms, draft_tokens[i][k] = the
 * smallest token t whose cumulative softmax probability exceeds u_{i,k} (token-id order;
 * if rounding leaves none, the last token with positive probability), the same inverse-CDF
 * convention as the verify draw; with uniforms NULL, the argmax (lowest id on ties).
 * q_at_draft (optional) receives each drafted token's softmax probability.  One launch,
 * one pass over the logits: per chunk of 2048 (bf16) or 1024 (fp32) elements the sweep
 * keeps (max, sum exp) or (max, first index); the CTA finishing a row turns the chunk
 * partials into the token and rescans one chunk.  Workspace:
 * pspec_sample_workspace_bytes(B, K, V) bytes (enough for either dtype), 256-byte aligned,
 * zero-filled once before first use (each call leaves its counters at zero; they sit at
 * the end of the workspace, one per row, so a workspace sized for B*K rows serves any
 * call with fewer rows when the same byte count is passed).  Returns
 * PSPEC_ERR_INVALID_ARG for bad sizes, pointers or dtype, PSPEC_ERR_WORKSPACE for a
 * missing, misaligned or short workspace, PSPEC_ERR_CUDA when the launch fails.
 */
typedef struct {
  int B;                       /* sequences; B = 0 is a no-op */
  int K;                       /* drafter output rows per sequence, >= 1 */
  int V;                       /* vocabulary size, >= 1 */
  long long ld;                /* row stride in elements, >= V */
  pspec_dtype dtype;
  const void *logits;          /* [B, K, ld] */
  const float *uniforms;       /* [B, K] in [0,1), or NULL for the argmax */
  int32_t *draft_tokens;       /* [B, K] out */
  float *q_at_draft;           /* [B, K] out, optional */
  int32_t *err;                /* device error word (required) */
} pspec_sample_args;

PSPEC_API size_t pspec_sample_workspace_bytes(int B, int K, int V);
PSPEC_API pspec_status pspec_sample_drafts(const pspec_sample_args *args, void *workspace,
                                           size_t workspace_bytes, cudaStream_t stream);

/*
 * Draft-batch construction arguments.
 *
 * Verify batch: sequence i owns rows [qsl_in[i], qsl_in[i+1]) of the verify arrays, with
 * L_i = qsl_in[i+1] - qsl_in[i] >= K+1 rows whose last K are its drafts.  After
 * verification a_i drafts were accepted, so c_i = L_i - K + a_i verify rows survive and
 * the last survivor's target hidden state is h_context.  Output span of sequence i, at
 * qsl_out[i] = qsl_in[i] + i*(K-1), length L_i + K - 1, in this order:
 *   rows 0 .. c_i-2     CTX  token verify_tokens[s+j+1], hidden verify row s+j,
 *                            position verify_pos[s+j]                    (s = qsl_in[i])
 *   row  c_i-1          NTP  token bonus[i], hidden verify row s+c_i-1 (h_context),
 *                            position P = verify_pos[s+c_i-1]
 *   rows c_i .. c_i+K-2 MASK token mask_id, hidden h_shared, position P + m (m = 1..K-1)
 *   last K - a_i rows   REJ  token pad_id, position of the rejected verify row, slot -1
 * Rows [qsl_out[B], T_cap) are PAD rows (pad_id, position 0, slot -1).
 * Slots of CTX/NTP/MASK rows: block_table[i][pos / block_size] * block_size
 * + pos % block_size.  seq_lens_out[i] = P + K (last mask position + 1).
 * sample_idx[i*K + k] = qsl_out[i] + c_i - 1 + k (the NTP row and the mask rows).
 * hidden_src[row] = the verify row copied into draft_hidden[row] (CTX/NTP), else -1.
 * draft_hidden rows of kind REJ and PAD are not written.
 */
typedef struct {
  int B;                          /* sequences; B = 0 writes only the PAD rows */
  int K;                          /* drafts per sequence, 1 <= K <= PSPEC_MAX_K */
  int H;                          /* hidden size (elements) */
  pspec_dtype hidden_dtype;       /* element type of verify_hidden / h_shared / draft_hidden */
  int block_size;                 /* KV block size in tokens, >= 1 */
  int max_blocks;                 /* columns of block_table, >= 1 */
  int mask_id;                    /* token id of the mask placeholder */
  int pad_id;                     /* token id written to REJ and PAD rows */
  int T_in;                       /* verify rows */
  int T_cap;                      /* output rows, >= T_in + B*(K-1) */
  const int32_t *qsl_in;          /* [B+1] verify query offsets, qsl_in[0] = 0 */
  const int32_t *verify_tokens;   /* [T_in] */
  const int32_t *verify_pos;      /* [T_in] */
  const int32_t *accepted_len;    /* [B] a_i from the verify step */
  const int32_t *bonus;           /* [B] bonus token from the verify step */
  const int32_t *block_table;     /* [B, max_blocks] KV block ids */
  const void *verify_hidden;      /* [T_in, H] target hidden states (16-byte aligned rows) */
  const void *h_shared;           /* [H] learned shared hidden state (16-byte aligned) */
  int32_t *draft_tokens;          /* [T_cap] out */
  int32_t *draft_pos;             /* [T_cap] out */
  int64_t *slot_mapping;          /* [T_cap] out, PSPEC_PADDING_SLOT_ID for REJ/PAD rows */
  uint8_t *row_kind;              /* [T_cap] out, PSPEC_ROW_* */
  int32_t *hidden_src;            /* [T_cap] out */
  int32_t *qsl_out;               /* [B+1] out */
  int32_t *seq_lens_out;          /* [B] out */
  int32_t *sample_idx;            /* [B, K] out */
  void *draft_hidden;             /* [T_cap, H] out (16-byte aligned rows) */
  int32_t *err;                   /* device error word (required) */
  const int32_t *k_len;           /* [B] per-sequence draft counts K_i in [0, K], or NULL for
                                     K everywhere: the last K_i verify rows of span i held
                                     this step's drafts, so c_i = L_i - K_i + a_i rows survive
                                     (L_i >= K_i + 1); every span still gets K-1 mask rows */
} pspec_build_args;

/*
 * Greedy verification with no allocation by anyone (the pages have no counterpart: this
 * serves callers that cannot provide device memory).  Some callers cannot hand this
 * library a workspace: a serving engine that reserves nearly all HBM for its KV cache at
 * start-up and gives memory out only through its own pool, a program that links only this
 * C library and has no device allocator, or a latency-critical path that cannot afford
 * cudaMalloc's implicit device synchronisation.  This entry point gives the same outputs as
 * pspec_verify_greedy (and runs the same argument checks), but always runs the full-sweep
 * greedy kernel -- whatever path pspec_verify_greedy would choose -- with its scratch in a
 * fixed array of PSPEC_NOALLOC_SCRATCH_BYTES inside the library's device image, so neither
 * side calls cudaMalloc, cudaFree or any allocating routine.
 *   - Every GPU that loads the library holds that array until the process exits.
 *   - Every call looks the array's device address up for the current device and context
 *     (cudaGetSymbolAddress, which allocates nothing), so the address stays right after
 *     cudaDeviceReset and in any context the caller makes current.  The first call on a
 *     device may load the library's device code there; make it before any stream capture.
 *   - All calls on a device share the array, which keeps the last call's contents: each
 *     call clears its tickets first (an asynchronous memset on `stream`), and calls whose
 *     executions overlap on the GPU race on it, so order them (one stream, or events).
 *   - It always uses the automatic segment length (options and pspec_set_segment_elems do
 *     not apply).  A call needs pspec_verify_workspace_bytes(B, K, V, 0) bytes with the
 *     automatic segment length; above PSPEC_NOALLOC_SCRATCH_BYTES it returns
 *     PSPEC_ERR_UNSUPPORTED and launches nothing (B = 1024, K = 7, V = 201088 needs about
 *     0.5 MiB).
 *   - pspec_last_launches() then reports 1 (0 for B = 0) and pspec_last_verify_path() 1.
 * Arguments, layout, outputs and device error bits are those of pspec_verify_greedy.
 */
#define PSPEC_NOALLOC_SCRATCH_BYTES (4u << 20)
PSPEC_API pspec_status pspec_verify_greedy_noalloc(const pspec_verify_args *args,
                                                   cudaStream_t stream);

/*
 * Parallel-draft batch construction: one launch.  Its CTAs take one of two roles: the
 * metadata role writes every per-row and per-sequence output, the hidden role copies the
 * CTX/NTP hidden rows and broadcasts h_shared into the MASK rows with 16-byte stores.
 * H * sizeof(elem) must be a multiple of 16 and the hidden bases 16-byte aligned
 * (PSPEC_ERR_INVALID_ARG otherwise).  Invalid values on the device: accepted_len outside
 * [0, K] is clamped (PSPEC_DEVERR_ACCEPT_RANGE); an out-of-table lookup gives slot -1
 * (PSPEC_DEVERR_BLOCK_RANGE); a sequence with L_i < K+1 keeps its span as PAD rows with
 * seq_lens_out 0 and sample_idx -1 (PSPEC_DEVERR_LAYOUT); a qsl_in that is not an offset
 * array (qsl_in[0] != 0, decreasing, or qsl_in[B] > T_in) sets PSPEC_DEVERR_LAYOUT and
 * leaves the outputs unspecified but every access in bounds.  The launch is a programmatic
 * dependent of the stream's previous kernel (its CTAs may be placed while that kernel's
 * last CTAs run, and wait for its completion before reading anything), which ordinary
 * stream order already implies; after a non-kernel operation it is an ordinary launch.
 */
PSPEC_API pspec_status pspec_build_draft_batch(const pspec_build_args *args, cudaStream_t stream);

/*
 * One speculative-decoding step: target verification followed by the P-EAGLE draft-batch
 * construction for the next step ("Eagle parallel speculative decoding, vLLM, TorchSpec",
 * sections "Parallel architecture" and "TorchSpec integration": the batch metadata and the
 * hidden-state fill are rebuilt on the GPU right after verification).  Computes exactly
 * pspec_verify_greedy / pspec_verify_rejection(v, ...) followed by
 * pspec_build_draft_batch(b) with b's accepted_len and bonus taken from v's outputs
 * (b->accepted_len and b->bonus must be NULL or v->accepted_len and v->bonus; b->B and b->K
 * must equal v->B and v->K).  When fusion is on (pspec_set_step_fusion; automatic: fewer
 * than 256 sequences, where the saved launch measured faster than building each span at the
 * end of the work that decides it), the verify's own last launch also builds: on the
 * early-exit path the cluster that decides sequence i, on the full sweep the CTA that
 * decides it (greedy) or draws its token (rejection), writes sequence i's span of the draft
 * batch (its metadata and its hidden rows), and the one of the last sequence writes the
 * padding rows; otherwise the verify launches are followed by the build launch.
 * pspec_last_launches() reports which.  Errors: those of the two calls it stands for; the
 * build's device-side error bits go to b->err, the verify's to v->err.
 */
PSPEC_API pspec_status pspec_step_greedy(const pspec_verify_args *v, const pspec_build_args *b,
                                         void *workspace, size_t workspace_bytes,
                                         cudaStream_t stream);
PSPEC_API pspec_status pspec_step_rejection(const pspec_verify_args *v, const pspec_build_args *b,
                                            void *workspace, size_t workspace_bytes,
                                            cudaStream_t stream);

/* Human-readable name of a status code (static storage). */
PSPEC_API const char *pspec_status_string(pspec_status status);

/* Number of kernel launches the most recent successful call made on this host thread
   issued (0 for an empty batch).  Used to count launches per decode step. */
PSPEC_API int pspec_last_launches(void);

/* The functions below set the PROCESS-WIDE DEFAULTS of the tuning options: they apply to
   every call whose arguments carry no pspec_options (options == NULL), and they are not
   synchronised with calls running on other host threads -- a program that tunes calls on
   several threads or streams passes its own pspec_options with each call instead.
   pspec_get_options() copies the current defaults. */
PSPEC_API void pspec_get_options(pspec_options *out);

/* Verify path selection (default of pspec_options.verify_path):
   0 (default) automatic -- the early-exit path when no per-row diagnostic is requested
     (target_lse, draft_lse, p_at_draft, q_at_draft all NULL), V is a multiple of 8 and
     the logits rows start on 16-byte boundaries, and the batch is large enough for the
     early exit to pay: B >= 160 for the rejection rule, B >= 64 for the greedy rule (below,
     the full sweep measured faster: it reads every row at once, while the early exit walks
     each sequence's positions one after another); otherwise the full sweep;
   1 always the full sweep;
   2 always the early-exit path (PSPEC_ERR_UNSUPPORTED when the arguments do not allow it).
   Both paths give the same outputs; they differ in which rows they read. */
PSPEC_API void pspec_set_verify_path(int path);

/* Tuning (default of pspec_options.cluster_size): CTAs per thread-block cluster on the
   early-exit path (2, 4, 8, 12 or 16; each CTA streams a 1/G slice of a row); 0 restores
   the automatic choice: a fixed width from 128 sequences on (16 when its slices would
   exceed 262144 elements); below, for the rejection rule the widest of 16, 12 and 8 with
   which the clusters of all sequences fit on the GPU at once
   (cudaOccupancyMaxActiveClusters, asked once per device and kernel variant), for the
   greedy rule 8 (16 below 16 sequences). */
PSPEC_API void pspec_set_cluster_size(int G);

/* Tuning (default of pspec_options.tail_split): on the early-exit path with the large-batch
   cluster width, the last n sequences of the batch are verified by a second launch of
   wider clusters, queued with programmatic dependent launch so that it starts while the
   first launch drains (the CTAs of the first launch release it when they are placed; CTA 0
   of the second waits for the first grid before it ends, so work queued later on the
   stream sees all outputs).  0 automatic (from 128 sequences on: the last B/8, at most 96
   for the rejection rule and 64 for the greedy rule), -1 never, n > 0 that many sequences (at
   most half the batch).  Outputs are the same either way; pspec_last_launches then reports
   2.  Every early-exit CTA also releases the stream's next programmatic launch when it is
   placed: the draft-batch build of pspec_step_* and pspec_build_draft_batch is launched
   that way and waits for the verify grid's completion before it reads anything. */
PSPEC_API void pspec_set_tail_split(int n);

/* Tuning (default of pspec_options.step_fusion): fusion of the build of pspec_step_* into
   the verify's last launch (either path): 0 automatic (fewer than 256 sequences), 1
   always, 2 never. */
PSPEC_API void pspec_set_step_fusion(int mode);

/* The path the most recent successful verify call on this host thread took: 1 full sweep,
   2 early exit, 0 none yet (or an empty batch). */
PSPEC_API int pspec_last_verify_path(void);

/* CTAs per cluster of the first (or only) launch of the last early-exit verify on this
   thread (the automatic choice or pspec_set_cluster_size's); 0 before any. */
PSPEC_API int pspec_last_cluster_size(void);

/* Tuning (default of pspec_options.segment_elems): force the full sweep's segment length
   (elements of one row handled by one CTA; rounded up to a multiple of 8).  0 restores the
   automatic choice, which aims at about 4 CTAs per SM with 8192 to 65536 elements per CTA.
   The segment length changes pspec_verify_workspace_bytes, so size workspaces after
   setting it. */
PSPEC_API void pspec_set_segment_elems(long long elems);

/* Profiling hook: while `event` is non-NULL, every pspec_verify_rejection call records it
   on the call's stream between its two launches (after the statistics sweep, before the
   draw; after the single launch of the early-exit path), so that a caller can time each
   launch with CUDA events.  NULL turns it off.  Process-wide; the caller owns the event. */
PSPEC_API void pspec_set_split_event(cudaEvent_t event);

#ifdef __cplusplus
}
#endif
#endif /* PSPEC_H */
