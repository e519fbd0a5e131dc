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

// The hidden rows of sequence i's span, as flat 16-byte vectors: the span's first c rows
// (CTX and NTP) copy the c consecutive verify rows s .. s+c-1, the next K-1 rows (MASK)
// repeat h_shared, and rejected rows are not written.  This call copies the vectors
// [f0, f1) of that sequence (clamped to the span's vectors) with all threads of the CTA,
// kCopyUnroll vectors in flight per thread.  A span whose offsets build_classify rejects
// (every row PAD) gets no hidden rows, and rows outside [0, T_cap) are skipped, as in the
// per-row classification.
constexpr int kCopyUnroll = 4;

__device__ __forceinline__ void build_span_copy(const pspec_build_args& a, long long row_vecs,
                                                int i, int acc, int Ki, long long f0, long long f1) {
  const long long q0 = build_qout(a, i);
  const int nthr = (int)blockDim.x, tid = (int)threadIdx.x;
  const int s = __ldg(a.qsl_in + i);
  const int e = __ldg(a.qsl_in + i + 1);
  const long long L = (long long)e - s;
  if (s < 0 || e > a.T_in || L < Ki + 1) return;          // every row of the span is PAD
  const int ac = acc < 0 ? 0 : (acc > Ki ? Ki : acc);
  const long long c = L - Ki + ac;                        // CTX + NTP rows
  const long long total = (c + a.K - 1) * row_vecs;       // and the MASK rows after them
  if (f1 > total) f1 = total;
  if (f0 < 0) f0 = 0;
  if (f0 + tid >= f1) return;
  const uint4* vh = static_cast<const uint4*>(a.verify_hidden);
  const uint4* hs = static_cast<const uint4*>(a.h_shared);
  uint4* dh = static_cast<uint4*>(a.draft_hidden);
  // (row j of the span, vector v of the row) of this thread's vectors, stepped by nthr
  long long f = f0 + tid;
  long long j = f / row_vecs, v = f - j * row_vecs;
  const long long dj = nthr / row_vecs, dv = nthr - dj * row_vecs;
  for (; f < f1; f += (long long)kCopyUnroll * nthr) {
    uint4 buf[kCopyUnroll];
    long long dst[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const long long r = q0 + j;                         // output row
      dst[u] = (f + (long long)u * nthr < f1 && r >= 0 && r < a.T_cap) ? r * row_vecs + v : -1;
      if (dst[u] >= 0) buf[u] = __ldg(j < c ? vh + (long long)(s + j) * row_vecs + v : hs + v);
      v += dv;
      j += dj;
      if (v >= row_vecs) { v -= row_vecs; ++j; }
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u)
      if (dst[u] >= 0) dh[dst[u]] = buf[u];
  }
}

// The metadata of rows [j0, j1) of sequence i's span (clamped to the span and to
// [0, T_cap)), one thread per row.
__device__ __forceinline__ void build_span_meta(const pspec_build_args& a, int i, int acc, int Ki,
                                                int bonus, long long j0, long long j1, int* eb) {
  const long long q0 = build_qout(a, i), q1 = build_qout(a, i + 1);
  long long lo = q0 + j0, hi = q0 + j1;
  if (lo < q0) lo = q0;
  if (lo < 0) lo = 0;
  if (hi > q1) hi = q1;
  if (hi > a.T_cap) hi = a.T_cap;
  for (long long t = lo + threadIdx.x; t < hi; t += blockDim.x)
    build_write_row(a, t, build_classify(a, i, t - q0, acc, Ki, bonus), eb);
}

// Sequence i's whole span by one group of `parts` CTAs: the metadata of every row and the
// per-sequence outputs (the CTA with `meta`), and an equal share of the hidden vectors
// (part `part`).
__device__ __forceinline__ void build_span(const pspec_build_args& a, long long row_vecs, int i,
                                           int acc, int Ki, int bonus, bool meta, int part,
                                           int parts, int* eb) {
  if (meta) {
    build_span_meta(a, i, acc, Ki, bonus, 0, 0x7fffffffffffLL, eb);
    if (threadIdx.x == 0) build_write_seq(a, i, acc, Ki, eb);
  }
  if (!a.draft_hidden) return;
  const long long span_vecs = ((long long)__ldg(a.qsl_in + i + 1) - __ldg(a.qsl_in + i) + a.K - 1) * row_vecs;
  if (span_vecs <= 0) return;
  const long long per = (span_vecs + parts - 1) / parts;
  build_span_copy(a, row_vecs, i, acc, Ki, (long long)part * per, (long long)part * per + per);
}

// The padding rows after the last span (and before the first, for an offset array that
// does not start at 0) and the end offset, shared by `parts` CTAs of blockDim.x threads.
__device__ __forceinline__ void build_tail_pad(const pspec_build_args& a, int part, int parts,
                                               int* eb) {
  const BuildRow pad{PSPEC_ROW_PAD, -1, a.pad_id, 0, -1};
  const long long first = build_qout(a, 0), last = build_qout(a, a.B);
  const long long head = first < 0 ? 0 : (first > a.T_cap ? (long long)a.T_cap : first);
  const long long tail = last < 0 ? 0 : last;
  const long long step = (long long)parts * blockDim.x;
  for (long long t = (long long)part * blockDim.x + threadIdx.x; t < head; t += step)
    build_write_row(a, t, pad, eb);
  for (long long t = tail + (long long)part * blockDim.x + threadIdx.x; t < a.T_cap; t += step)
    build_write_row(a, t, pad, eb);
  if (part == 0 && threadIdx.x == 0) build_write_seq(a, a.B, 0, a.K, eb);
}

}  // namespace pspec
