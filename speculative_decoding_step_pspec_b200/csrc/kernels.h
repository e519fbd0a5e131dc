// kernels.h -- launch descriptors passed by value to the libpspec kernels.
//
// The C entry points (api.cu) validate the caller's arguments, build one of these from the
// argument struct and the workspace plan, and call the matching launcher.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pspec.h"

namespace pspec {

struct GreedyLaunch {
  int B, K, V;
  long long ld;
  pspec_dtype dtype;
  int S;                 // segments per row
  long long seg;         // elements per segment
  const void* target;
  const int32_t* draft_tokens;
  int32_t* out_tokens;
  int32_t* accepted_len;
  int32_t* bonus;
  float* target_lse;     // optional
  int32_t* err;
  const int32_t* k_len;  // optional per-sequence draft counts
  int* cnt;              // zero area: ticket column (entry i = zcol(cnt, i))
  void* part;            // workspace: GreedyPart [B*(K+1)*S]
  int fuse_build;        // 1: the CTA that decides a sequence also builds its draft span
  pspec_build_args b;    // draft-batch arguments (accepted_len / bonus = this launch's outputs)
  long long row_vecs;    // 16-byte vectors per hidden row of b
};

struct RejectionLaunch {
  int B, K, V;
  long long ld;
  pspec_dtype dtype;
  int S;
  long long seg;
  int tiles, tiles_per_chunk, C;
  const void* target;
  const void* draft;
  const int32_t* draft_tokens;
  const float* uniforms;
  int32_t* out_tokens;
  int32_t* accepted_len;
  int32_t* bonus;
  float* target_lse;     // optional
  float* draft_lse;      // optional
  float* p_at_draft;     // optional
  float* q_at_draft;     // optional
  float* residual_mass;  // optional
  int32_t* err;
  const int32_t* k_len;  // optional per-sequence draft counts
  int* cnt;              // zero area: sweep ticket column (zcol)
  int* cnt2;             // zero area: resample ticket column (zcol)
  void* part;            // workspace: RejPart [B*(2K+1)*S]
  void* seq;             // workspace: SeqInfo [B]
  double* tile_sums;     // workspace: [B*tiles] sums of r over 256-element tiles
  int fuse_build;        // 1: the draw's last CTA of a sequence also builds its draft span
  pspec_build_args b;    // draft-batch arguments (accepted_len / bonus = this launch's outputs)
  long long row_vecs;    // 16-byte vectors per hidden row of b
};

struct EarlyExitLaunch {
  int B, K, V;
  long long ld;
  pspec_dtype dtype;
  int rejection;         // 1: rejection rule, 0: greedy
  int G;                 // CTAs per cluster (one cluster per sequence): 2, 4, 8, 12 or 16
  int seq0, nseq;        // this launch's sequences [seq0, seq0 + nseq) of the batch's B
  int pdl;               // split batch: 1 first launch, 2 second launch (a programmatic
                         // dependent of the first; its CTA 0 ends after the first grid)
  long long vs;          // slice of each row per CTA (elements, multiple of 8)
  const void* target;
  const void* draft;
  const int32_t* draft_tokens;
  const float* uniforms;
  int32_t* out_tokens;
  int32_t* accepted_len;
  int32_t* bonus;
  float* residual_mass;  // optional
  int32_t* err;
  const int32_t* k_len;  // optional per-sequence draft counts
  int fuse_build;        // 1: each cluster also builds its sequence's draft span (below)
  pspec_build_args b;    // draft-batch arguments; accepted_len / bonus = this launch's outputs
  long long row_vecs;    // 16-byte vectors per hidden row of b
};

struct SampleLaunch {
  long long rows;        // B*K drafter rows
  int V;
  long long ld;
  pspec_dtype dtype;
  int tiles;             // chunks per row (2048 bf16 / 1024 fp32 elements)
  int tiles_per_seg;     // chunks per CTA
  int S;                 // CTAs per row
  const void* logits;
  const float* uniforms; // NULL: argmax
  int32_t* tokens;
  float* probs;          // optional
  int32_t* err;
  int* cnt;              // end of the workspace: ticket of row r = zrow(cnt, r)
  void* parts;           // workspace: (m, s) per chunk [rows*tiles]
  void* maxes;           // workspace: (max, index) per chunk [rows*tiles]
};

struct BuildLaunch {
  pspec_build_args a;
  long long row_vecs;    // 16-byte vectors per hidden row
  int meta_blocks;       // CTAs of the metadata role (the rest copy hidden rows)
  int hid_rows;          // rows the hidden role inspects: T_in + B*(K-1)
};

cudaError_t launch_greedy(const GreedyLaunch& L, cudaStream_t stream);
// split_event (may be null) is recorded between the statistics sweep and the draw.
cudaError_t launch_rejection(const RejectionLaunch& L, cudaStream_t stream, cudaEvent_t split_event);
cudaError_t launch_build(const BuildLaunch& L, cudaStream_t stream);
cudaError_t launch_early_exit(const EarlyExitLaunch& L, cudaStream_t stream);
// Clusters of the variant L names (G, dtype, rule, fusion) that fit on the
// current device at once; 0 when the query fails.  Cached per device and variant.
int early_exit_max_clusters(const EarlyExitLaunch& L);
cudaError_t launch_sample(const SampleLaunch& L, cudaStream_t stream);
// Host helpers of the entry points (api.cu), shared by every verify entry point: the
// argument checks of a verify call, and the per-thread record behind pspec_last_launches()
// and pspec_last_verify_path().
pspec_status check_verify_host(const pspec_verify_args* a, bool rejection);
void record_last_call(int launches, int path);

}  // namespace pspec
