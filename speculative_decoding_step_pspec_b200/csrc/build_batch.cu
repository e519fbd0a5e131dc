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
// Here both jobs share one launch with two CTA roles that never wait for each other:
//   metadata role: one thread per output row (token, position, slot, kind, hidden source)
//                  plus one thread per sequence (offsets, sequence length, sample index);
//   hidden role:   one warp per output row, copying the row's hidden state with 16-byte
//                  loads and stores (verify row for CTX/NTP, h_shared for MASK).
// Each role derives a row's sequence on its own: the uniform layout (every L_i = K+1) is
// checked with two loads, anything else falls back to a binary search over the offsets.
#include "common.cuh"
#include "kernels.h"

namespace pspec {

namespace {

struct Row {
  int kind;
  int seq;
  int tok;
  int pos;
  int src;
};

__device__ __forceinline__ long long qout(const int32_t* qsl_in, int i, int K) {
  return (long long)__ldg(qsl_in + i) + (long long)i * (K - 1);
}

// The sequence whose output span holds row r: the largest i in [0, B] with
// qsl_out[i] <= r, or -1 when none.  Bounded for any contents of qsl_in.
__device__ __forceinline__ int find_seq(const pspec_build_args& a, long long r) {
  const int B = a.B, K = a.K;
  const long long span = 2LL * K;
  const long long g = r / span;
  if (g < B && qout(a.qsl_in, (int)g, K) <= r && r < qout(a.qsl_in, (int)g + 1, K)) return (int)g;
  if (qout(a.qsl_in, 0, K) > r) return -1;
  int lo = 0, hi = B;                    // qsl_out[lo] <= r
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (qout(a.qsl_in, mid, K) <= r) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ Row classify(const pspec_build_args& a, long long r) {
  Row row{PSPEC_ROW_PAD, -1, a.pad_id, 0, -1};
  const int K = a.K;
  const int i = find_seq(a, r);
  if (i < 0 || i >= a.B) return row;
  const int s = __ldg(a.qsl_in + i);
  const int e = __ldg(a.qsl_in + i + 1);
  const long long L = (long long)e - s;
  const long long j = r - qout(a.qsl_in, i, K);
  if (s < 0 || e > a.T_in || L < K + 1 || j < 0 || j >= L + K - 1) return row;
  int acc = __ldg(a.accepted_len + i);
  acc = acc < 0 ? 0 : (acc > K ? K : acc);
  const int c = (int)L - K + acc;        // surviving verify rows, c >= 1
  row.seq = i;
  if (j < c - 1) {                       // context: token j+1 with hidden j
    row.kind = PSPEC_ROW_CTX;
    row.tok = __ldg(a.verify_tokens + s + j + 1);
    row.pos = __ldg(a.verify_pos + s + j);
    row.src = s + (int)j;
  } else if (j == c - 1) {               // NTP: bonus with h_context
    row.kind = PSPEC_ROW_NTP;
    row.tok = __ldg(a.bonus + i);
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

__device__ __forceinline__ long long kv_slot(const pspec_build_args& a, int i, int pos, int* eb) {
  if (pos < 0) { *eb |= PSPEC_DEVERR_BLOCK_RANGE; return PSPEC_PADDING_SLOT_ID; }
  const int blk = pos / a.block_size;
  if (blk >= a.max_blocks) { *eb |= PSPEC_DEVERR_BLOCK_RANGE; return PSPEC_PADDING_SLOT_ID; }
  const int id = __ldg(a.block_table + (long long)i * a.max_blocks + blk);
  if (id < 0) { *eb |= PSPEC_DEVERR_BLOCK_RANGE; return PSPEC_PADDING_SLOT_ID; }
  return (long long)id * a.block_size + pos % a.block_size;
}

__device__ void meta_role(const pspec_build_args& a, long long t) {
  const int K = a.K;
  int eb = 0;
  if (t < a.T_cap) {                     // one output row
    const Row row = classify(a, t);
    long long slot = PSPEC_PADDING_SLOT_ID;
    if (row.kind == PSPEC_ROW_CTX || row.kind == PSPEC_ROW_NTP || row.kind == PSPEC_ROW_MASK)
      slot = kv_slot(a, row.seq, row.pos, &eb);
    a.draft_tokens[t] = row.tok;
    a.draft_pos[t] = row.pos;
    a.slot_mapping[t] = slot;
    a.row_kind[t] = (uint8_t)row.kind;
    a.hidden_src[t] = row.src;
  } else if (t < (long long)a.T_cap + a.B + 1) {  // one sequence (or the end offset)
    const int i = (int)(t - a.T_cap);
    const int s = __ldg(a.qsl_in + i);
    a.qsl_out[i] = (int)qout(a.qsl_in, i, K);
    if (i == a.B) {
      if (__ldg(a.qsl_in) != 0 || s > a.T_in) eb |= PSPEC_DEVERR_LAYOUT;
    } else {
      const int e = __ldg(a.qsl_in + i + 1);
      const long long L = (long long)e - s;
      if (e < s) eb |= PSPEC_DEVERR_LAYOUT;
      if (s < 0 || e > a.T_in || L < K + 1) {
        eb |= PSPEC_DEVERR_LAYOUT;
        a.seq_lens_out[i] = 0;
        for (int k = 0; k < K; ++k) a.sample_idx[(long long)i * K + k] = -1;
      } else {
        int acc = __ldg(a.accepted_len + i);
        if (acc < 0 || acc > K) {
          eb |= PSPEC_DEVERR_ACCEPT_RANGE;
          acc = acc < 0 ? 0 : K;
        }
        const int c = (int)L - K + acc;
        const int P = __ldg(a.verify_pos + s + c - 1);
        a.seq_lens_out[i] = P + K;
        const int base = (int)qout(a.qsl_in, i, K) + c - 1;
        for (int k = 0; k < K; ++k) a.sample_idx[(long long)i * K + k] = base + k;
      }
    }
  }
  set_err(a.err, eb);
}

__device__ void hidden_role(const BuildLaunch& L, long long r) {
  const pspec_build_args& a = L.a;
  const Row row = classify(a, r);
  const uint4* src;
  if (row.kind == PSPEC_ROW_CTX || row.kind == PSPEC_ROW_NTP)
    src = static_cast<const uint4*>(a.verify_hidden) + (long long)row.src * L.row_vecs;
  else if (row.kind == PSPEC_ROW_MASK)
    src = static_cast<const uint4*>(a.h_shared);
  else
    return;                              // REJ / PAD rows keep their contents
  uint4* dst = static_cast<uint4*>(a.draft_hidden) + r * L.row_vecs;
  const int lane = threadIdx.x & 31;
  constexpr int U = 4;
  for (long long v0 = lane; v0 < L.row_vecs; v0 += 32 * U) {
    uint4 buf[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      long long v = v0 + 32LL * u;
      if (v < L.row_vecs) buf[u] = __ldg(src + v);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      long long v = v0 + 32LL * u;
      if (v < L.row_vecs) dst[v] = buf[u];
    }
  }
}

__global__ void __launch_bounds__(kThreads) build_kernel(const BuildLaunch L) {
  if ((int)blockIdx.x < L.meta_blocks) {
    meta_role(L.a, (long long)blockIdx.x * kThreads + threadIdx.x);
  } else {
    const long long r =
        (long long)(blockIdx.x - L.meta_blocks) * kWarps + (threadIdx.x >> 5);
    if (r < L.hid_rows) hidden_role(L, r);
  }
}

}  // namespace

cudaError_t launch_build(const BuildLaunch& L, cudaStream_t stream) {
  long long hid_blocks = L.a.draft_hidden ? (L.hid_rows + kWarps - 1) / kWarps : 0;
  long long grid = L.meta_blocks + hid_blocks;
  build_kernel<<<(unsigned)grid, kThreads, 0, stream>>>(L);
  return cudaGetLastError();
}

}  // namespace pspec
