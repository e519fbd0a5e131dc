// build_common.cuh -- the per-row and per-sequence pieces of P-EAGLE draft-batch
// construction, shared by the build launch and the fused verify + build launch.
//
// "Eagle parallel speculative decoding, vLLM, TorchSpec", section "Parallel architecture":
// the drafter's single forward pass takes the accepted context tokens paired with their
// target hidden states, one next-token (NTP) slot paired with h_context, and K-1 mask
// slots paired with the learned h_shared; section "TorchSpec integration": rejected tokens
// take PADDING_SLOT_ID = -1 so they cannot write the KV cache.
//
// Sequence i's span of the draft batch starts at qsl_out[i] = qsl_in[i] + i(K-1) and holds
// L_i + K - 1 rows, L_i = qsl_in[i+1] - qsl_in[i] verify rows of which the last K_i held this
// step's drafts (K_i = K unless per-sequence counts are given) and c_i = L_i - K_i + a_i
// survive:  [c_i - 1 context rows | NTP | K - 1 mask rows | K_i - a_i rejected rows].
// The accepted count and the bonus token are passed as values, so a kernel that has just
// computed them can build the span without reading them back.
#pragma once

#include "common.cuh"
#include "pspec.h"

namespace pspec {

struct BuildRow {
  int kind;
  int seq;
  int tok;
  int pos;
  int src;
};

__device__ __forceinline__ long long build_qout(const pspec_build_args& a, int i) {
  return (long long)__ldg(a.qsl_in + i) + (long long)i * (a.K - 1);
}

// Row j of sequence i's span, for the sequence's draft count Ki (its last Ki verify rows
// held drafts), accepted count acc (clamped into [0, Ki]) and bonus token.
__device__ __forceinline__ BuildRow build_classify(const pspec_build_args& a, int i, long long j,
                                                   int acc, int Ki, int bonus) {
  BuildRow row{PSPEC_ROW_PAD, -1, a.pad_id, 0, -1};
  const int K = a.K;
  const int s = __ldg(a.qsl_in + i);
  const int e = __ldg(a.qsl_in + i + 1);
  const long long L = (long long)e - s;
  if (s < 0 || e > a.T_in || L < Ki + 1 || j < 0 || j >= L + K - 1) return row;
  acc = acc < 0 ? 0 : (acc > Ki ? Ki : acc);
  const int c = (int)L - Ki + acc;       // surviving verify rows, c >= 1
  row.seq = i;
  if (j < c - 1) {                       // context: token j+1 with hidden j
    row.kind = PSPEC_ROW_CTX;
    row.tok = __ldg(a.verify_tokens + s + j + 1);
    row.pos = __ldg(a.verify_pos + s + j);
    row.src = s + (int)j;
  } else if (j == c - 1) {               // NTP: bonus with h_context
    row.kind = PSPEC_ROW_NTP;
    row.tok = bonus;
    row.pos = __ldg(a.verify_pos + s + j);
    row.src = s + (int)j;
  } else if (j < c + K - 1) {            // MASK m = j - c + 1
    row.kind = PSPEC_ROW_MASK;
    row.tok = a.mask_id;
    row.pos = __ldg(a.verify_pos + s + c - 1) + (int)(j - c + 1);
  } else {                               // rejected verify row j - K + 1
    row.kind = PSPEC_ROW_REJ;
    row.tok = a.pad_id;
    row.pos = __ldg(a.verify_pos + s + (j - K + 1));
  }
  return row;
}

__device__ __forceinline__ long long build_kv_slot(const pspec_build_args& a, int i, int pos, int* eb) {
  if (pos < 0) { *eb |= PSPEC_DEVERR_BLOCK_RANGE; return PSPEC_PADDING_SLOT_ID; }
  const int blk = pos / a.block_size;
  if (blk >= a.max_blocks) { *eb |= PSPEC_DEVERR_BLOCK_RANGE; return PSPEC_PADDING_SLOT_ID; }
  const int id = __ldg(a.block_table + (long long)i * a.max_blocks + blk);
  if (id < 0) { *eb |= PSPEC_DEVERR_BLOCK_RANGE; return PSPEC_PADDING_SLOT_ID; }
  return (long long)id * a.block_size + pos % a.block_size;
}

// The metadata of output row t.
__device__ __forceinline__ void build_write_row(const pspec_build_args& a, long long t,
                                                const BuildRow& row, int* eb) {
  long long slot = PSPEC_PADDING_SLOT_ID;
  if (row.kind == PSPEC_ROW_CTX || row.kind == PSPEC_ROW_NTP || row.kind == PSPEC_ROW_MASK)
    slot = build_kv_slot(a, row.seq, row.pos, eb);
  a.draft_tokens[t] = row.tok;
  a.draft_pos[t] = row.pos;
  a.slot_mapping[t] = slot;
  a.row_kind[t] = (uint8_t)row.kind;
  a.hidden_src[t] = row.src;
}

// The per-sequence outputs of sequence i < B (acc as given, before clamping: a count outside
// [0, Ki] sets PSPEC_DEVERR_ACCEPT_RANGE), or the end offset and layout check for i == B.
__device__ __forceinline__ void build_write_seq(const pspec_build_args& a, int i, int acc, int Ki,
                                                int* eb) {
  const int K = a.K;
  const int s = __ldg(a.qsl_in + i);
  a.qsl_out[i] = (int)build_qout(a, i);
  if (i == a.B) {
    if (__ldg(a.qsl_in) != 0 || s > a.T_in) *eb |= PSPEC_DEVERR_LAYOUT;
    return;
  }
  const int e = __ldg(a.qsl_in + i + 1);
  const long long L = (long long)e - s;
  if (e < s) *eb |= PSPEC_DEVERR_LAYOUT;
  if (s < 0 || e > a.T_in || L < Ki + 1) {
    *eb |= PSPEC_DEVERR_LAYOUT;
    a.seq_lens_out[i] = 0;
    for (int k = 0; k < K; ++k) a.sample_idx[(long long)i * K + k] = -1;
    return;
  }
  if (acc < 0 || acc > Ki) {
    *eb |= PSPEC_DEVERR_ACCEPT_RANGE;
    acc = acc < 0 ? 0 : Ki;
  }
  const int c = (int)L - Ki + acc;
  const int P = __ldg(a.verify_pos + s + c - 1);
  a.seq_lens_out[i] = P + K;
  const int base = (int)build_qout(a, i) + c - 1;
  for (int k = 0; k < K; ++k) a.sample_idx[(long long)i * K + k] = base + k;
}

// One warp: the hidden state of output row r (a verify row for CTX / NTP, h_shared for
// MASK; rejected and padding rows keep their contents), 16-byte vectors, four in flight.
__device__ __forceinline__ void build_copy_hidden(const pspec_build_args& a, long long row_vecs,
                                                  long long r, const BuildRow& row) {
  const uint4* src;
  if (row.kind == PSPEC_ROW_CTX || row.kind == PSPEC_ROW_NTP)
    src = static_cast<const uint4*>(a.verify_hidden) + (long long)row.src * row_vecs;
  else if (row.kind == PSPEC_ROW_MASK)
    src = static_cast<const uint4*>(a.h_shared);
  else
    return;
  uint4* dst = static_cast<uint4*>(a.draft_hidden) + r * row_vecs;
  const int lane = threadIdx.x & 31;
  constexpr int U = 4;
  for (long long v0 = lane; v0 < row_vecs; v0 += 32 * U) {
    uint4 buf[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long v = v0 + 32LL * u;
      if (v < row_vecs) buf[u] = __ldg(src + v);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long v = v0 + 32LL * u;
      if (v < row_vecs) dst[v] = buf[u];
    }
  }
}

}  // namespace pspec
