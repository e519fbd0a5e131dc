// build_batch.cu -- P-EAGLE parallel-draft batch construction (one launch).
//
// "Eagle parallel speculative decoding, vLLM, TorchSpec", section "Parallel architecture":
// the drafter's single forward pass takes the accepted context tokens paired with their
// target hidden states, one next-token (NTP) slot paired with h_context, and K-1 mask
// slots paired with the learned h_shared.  Section "TorchSpec integration": the batch
// metadata (copy, scatter, insert, pad, mask, remap) is rebuilt on the GPU in one launch,
// the hidden states are moved by a separate broadcast copy because they dominate the
// bytes, and rejected tokens take PADDING_SLOT_ID = -1 so they cannot write the KV cache.
//
// Here both jobs share one launch, organised by sequence: P CTAs per sequence, CTA p owning
// R consecutive rows of the sequence's output span (R P covers the uniform span of 2K rows;
// longer spans are walked in further steps of R P rows).  Each CTA reads the sequence's
// offsets, accepted count and bonus token once -- in parallel, not as a chain per row --
// then writes the metadata of its rows (one thread per row) and copies their hidden states
// as one flat block of 16-byte vectors (context / NTP rows from consecutive verify rows,
// mask rows from h_shared).  The first CTA of a sequence also writes its per-sequence
// outputs, and a few more CTAs write the padding rows after the last span and the end
// offset.  No CTA waits on another.
#include "build_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace pspec {

namespace {

__global__ void __launch_bounds__(kBuildThreads) build_kernel(const BuildLaunch L) {
  const pspec_build_args& a = L.a;
  const long long blk = blockIdx.x;
  const long long seq_blocks = (long long)a.B * L.parts;
  int eb = 0;
  if (blk < seq_blocks) {
    // part p of sequence i: span rows [p R, p R + R), then every parts * R rows further for
    // spans longer than the uniform 2K rows
    const int i = (int)(blk / L.parts);
    const int part = (int)(blk - (long long)i * L.parts);
    int eb_k = 0;
    const int Ki = draft_count(a.k_len, i, a.K, &eb_k);
    const int acc = __ldg(a.accepted_len + i);
    const int bonus = __ldg(a.bonus + i);
    const long long span_rows = (long long)__ldg(a.qsl_in + i + 1) - __ldg(a.qsl_in + i) + a.K - 1;
    const long long R = L.rows_per_part;
    for (long long j0 = part * R; j0 < span_rows; j0 += (long long)L.parts * R) {
      build_span_meta(a, i, acc, Ki, bonus, j0, j0 + R, &eb);
      if (a.draft_hidden)
        build_span_copy(a, L.row_vecs, i, acc, Ki, j0 * L.row_vecs, (j0 + R) * L.row_vecs);
    }
    if (part == 0) {
      eb |= eb_k;
      if (threadIdx.x == 0) build_write_seq(a, i, acc, Ki, &eb);
    }
  } else {
    // padding rows [0, qsl_out[0]) and [qsl_out[B], T_cap), and the end offset
    build_tail_pad(a, (int)(blk - seq_blocks), L.pad_blocks, &eb);
  }
  set_err(a.err, eb);
}

}  // namespace

cudaError_t launch_build(const BuildLaunch& L, cudaStream_t stream) {
  const long long grid = (long long)L.a.B * L.parts + L.pad_blocks;
  build_kernel<<<(unsigned)grid, kBuildThreads, 0, stream>>>(L);
  return cudaGetLastError();
}

}  // namespace pspec
