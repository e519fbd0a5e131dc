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
#include "build_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace pspec {

namespace {

// The sequence whose output span holds row r: the largest i in [0, B] with
// qsl_out[i] <= r, or -1 when none.  Bounded for any contents of qsl_in.
__device__ __forceinline__ int find_seq(const pspec_build_args& a, long long r) {
  const int B = a.B;
  const long long span = 2LL * a.K;
  const long long g = r / span;
  if (g < B && build_qout(a, (int)g) <= r && r < build_qout(a, (int)g + 1)) return (int)g;
  if (build_qout(a, 0) > r) return -1;
  int lo = 0, hi = B;                    // qsl_out[lo] <= r
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (build_qout(a, mid) <= r) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Row r's classification.  Under the uniform layout (every L_i = K+1) row r belongs to
// sequence g = r / 2K, so its offsets, accepted count, draft count and bonus token are all
// requested at once and the row waits for one round trip instead of a chain of two; a row
// outside span g (any other layout) takes the binary search.
__device__ __forceinline__ BuildRow classify(const pspec_build_args& a, long long r) {
  const long long g = r / (2LL * a.K);
  int i = -1, acc = 0, kl = a.K, bon = 0;
  if (g < a.B) {
    const int q0 = __ldg(a.qsl_in + g), q1 = __ldg(a.qsl_in + g + 1);
    const int acc_g = __ldg(a.accepted_len + g);
    const int kl_g = a.k_len ? __ldg(a.k_len + g) : a.K;
    const int bon_g = __ldg(a.bonus + g);
    if ((long long)q0 + g * (a.K - 1) <= r && r < (long long)q1 + (g + 1) * (a.K - 1)) {
      i = (int)g;
      acc = acc_g;
      kl = kl_g;
      bon = bon_g;
    }
  }
  if (i < 0) {
    i = find_seq(a, r);
    if (i < 0 || i >= a.B) return BuildRow{PSPEC_ROW_PAD, -1, a.pad_id, 0, -1};
    acc = __ldg(a.accepted_len + i);
    kl = a.k_len ? __ldg(a.k_len + i) : a.K;
    bon = __ldg(a.bonus + i);
  }
  const int Ki = kl < 0 ? 0 : (kl > a.K ? a.K : kl);      // as draft_count clamps it
  return build_classify(a, i, r - build_qout(a, i), acc, Ki, bon);
}

__device__ void meta_role(const pspec_build_args& a, long long t) {
  int eb = 0;
  if (t < a.T_cap) {                     // one output row
    build_write_row(a, t, classify(a, t), &eb);
  } else if (t < (long long)a.T_cap + a.B + 1) {  // one sequence (or the end offset)
    const int i = (int)(t - a.T_cap);
    const int Ki = i < a.B ? draft_count(a.k_len, i, a.K, &eb) : a.K;
    build_write_seq(a, i, i < a.B ? __ldg(a.accepted_len + i) : 0, Ki, &eb);
  }
  set_err(a.err, eb);
}

__global__ void __launch_bounds__(kThreads) build_kernel(const BuildLaunch L) {
  // Launched as a programmatic dependent of the stream's previous kernel: the CTAs may be
  // placed while that kernel's last CTAs still run (the verify launches allow it once all
  // their CTAs have started), and wait here until it has finished and its writes are
  // visible.  After any other kernel this returns at once.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if ((int)blockIdx.x < L.meta_blocks) {
    meta_role(L.a, (long long)blockIdx.x * kThreads + threadIdx.x);
  } else {
    const long long r =
        (long long)(blockIdx.x - L.meta_blocks) * kWarps + (threadIdx.x >> 5);
    if (r < L.hid_rows) build_copy_hidden(L.a, L.row_vecs, r, classify(L.a, r));
  }
}

}  // namespace

cudaError_t launch_build(const BuildLaunch& L, cudaStream_t stream) {
  long long hid_blocks = L.a.draft_hidden ? (L.hid_rows + kWarps - 1) / kWarps : 0;
  long long grid = L.meta_blocks + hid_blocks;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, build_kernel, L);
}

}  // namespace pspec
