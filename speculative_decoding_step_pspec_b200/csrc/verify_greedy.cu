// verify_greedy.cu -- greedy target verification (one launch).
//
// "Any accepted prefix replaces the greedy path" ("Capstone 14: speculative decoding
// inference server", section "Concept"): for each sequence the target's argmax over the
// vocabulary is taken on each of its K+1 rows, the accepted prefix is the run of leading
// drafts equal to it, and the token after the prefix is the argmax of the next row.
//
// Design: the grid is B*(K+1) rows x S segments, one CTA per segment, 16-byte streaming
// loads with four vectors in flight per thread.  The bf16 max of each vector is taken
// on packed pairs (max.bf16x2), and only a vector that beats the running best is
// unpacked to find the first position of its maximum.  The optional log-sum-exp uses the
// base-2 online normaliser of verify_common.cuh.  Each CTA writes one partial;
// an atomic ticket per sequence elects the CTA that finishes the sequence last, and that
// CTA merges the partials in segment order (deterministic, lowest id wins ties) and
// writes the accepted length, the bonus token and the output tokens.  No CTA waits.
#include "build_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "verify_common.cuh"

namespace pspec {

namespace {

template <typename Tag, bool kLse, bool kFuse>
__global__ void __launch_bounds__(kThreads)
greedy_sweep_kernel(const GreedyLaunch L) {
  using elem = typename Tag::elem;
  // the stream's next programmatic launch (the step's build) may be placed once every CTA
  // of this grid has started; it waits for this grid's completion before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long item = blockIdx.x;
  const int s = (int)(item % L.S);
  const long long rowg = item / L.S;                 // i*(K+1) + k
  const int i = (int)(rowg / (L.K + 1));
  const elem* row = static_cast<const elem*>(L.target) + rowg * L.ld;
  const long long lo = (long long)s * L.seg;
  const long long hi = min((long long)L.V, lo + L.seg);

  VI best{-INFINITY, kNoIndex};
  MSAcc acc = msacc_init();
  sweep_segment<Tag, 4>(
      row, lo, hi,
      [&](const uint4& v, long long idx0) {
        consume_argmax<Tag>(v, idx0, best);
        if (kLse) consume_ms<Tag>(v, acc);
      },
      [&](float x, long long t) {
        if (x > best.v) { best.v = x; best.i = (int)t; }
        if (kLse) consume_one(x, acc);
      });
  MS ms = msacc_final(acc);

  // CTA reduction
  __shared__ VI s_vi[kWarps];
  __shared__ MS s_ms[kWarps];
  __shared__ int s_last;
  best = warp_argmax(best);
  if (kLse) ms = warp_merge_ms(ms);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) { s_vi[warp] = best; s_ms[warp] = ms; }
  __syncthreads();
  if (warp == 0) {
    best = lane < kWarps ? s_vi[lane] : VI{-INFINITY, kNoIndex};
    ms = lane < kWarps ? s_ms[lane] : MS{-INFINITY, 0.f};
    best = warp_argmax(best);
    if (kLse) ms = warp_merge_ms(ms);
    if (lane == 0) {
      GreedyPart* part = reinterpret_cast<GreedyPart*>(L.part);
      part[item] = GreedyPart{best.v, best.i, ms.m, ms.s};
      __threadfence();
      int t = atomicAdd(zcol(L.cnt, i), 1);
      s_last = (t == L.S * (L.K + 1) - 1);
    }
  }
  __syncthreads();
  if (!s_last) return;

  // This CTA finished sequence i last: merge its (K+1) x S partials, warp w taking rows
  // w, w + 8, ... and lane t segments t, t + 32, ... (argmax: largest value, lowest id).
  __threadfence();
  const int K = L.K;
  const GreedyPart* part =
      reinterpret_cast<const GreedyPart*>(L.part) + (long long)i * (K + 1) * L.S;
  __shared__ int s_g[PSPEC_MAX_K + 1];
  __shared__ double s_lse[PSPEC_MAX_K + 1];
  for (int r = warp; r <= K; r += kWarps) {
    VI b{-INFINITY, kNoIndex};
    float M = -INFINITY;
    for (int t = lane; t < L.S; t += 32) {
      const GreedyPart q = ld_cg(part + (long long)r * L.S + t);
      if (vi_better(VI{q.v, q.i}, b)) b = VI{q.v, q.i};
      M = fmaxf(M, q.m);
    }
    b = warp_argmax(b);
    if (kLse) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      double S = 0.0;
      if (M != -INFINITY)
        for (int t = lane; t < L.S; t += 32) {
          const GreedyPart q = ld_cg(part + (long long)r * L.S + t);
          if (q.m != -INFINITY) S += (double)q.s * exp2((double)q.m - (double)M);
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
      if (lane == 0) s_lse[r] = M == -INFINITY ? -INFINITY : ((double)M + log2(S)) / (double)kLog2e;
    }
    if (lane == 0) s_g[r] = b.i == kNoIndex ? 0 : b.i;   // a row of -inf / NaN only: token 0
  }
  __syncthreads();
  __shared__ int s_fin[3];                           // (a, K_i, bonus) for the fused build
  if (warp == 0) {
  const int g = lane <= K ? s_g[lane] : 0;           // argmax of row `lane`
  const double lse = (kLse && lane <= K) ? s_lse[lane] : 0.0;
  int eb = 0;
  const int Ki = draft_count(L.k_len, i, K, &eb);    // the sequence's own drafts
  int d = -1;
  bool bad = false;
  if (lane < Ki) {
    d = L.draft_tokens[(long long)i * K + lane];
    bad = d < 0 || d >= L.V;
  }
  unsigned match = __ballot_sync(0xffffffffu, lane < Ki && !bad && d == g);
  unsigned anybad = __ballot_sync(0xffffffffu, bad);
  int a = __ffs(~match) - 1;             // first mismatch
  if (a > Ki) a = Ki;
  int bonus = __shfl_sync(0xffffffffu, g, a);
  if (lane <= K) {
    L.out_tokens[(long long)i * (K + 1) + lane] = lane < a ? d : (lane == a ? bonus : -1);
    if (kLse) L.target_lse[(long long)i * (K + 1) + lane] = (float)lse;
  }
  if (lane == 0) {
    L.accepted_len[i] = a;
    L.bonus[i] = bonus;
    set_err(L.err, eb | (anybad ? PSPEC_DEVERR_TOKEN_RANGE : 0));
    *zcol(L.cnt, i) = 0;                       // ticket back to zero for the next call
    s_fin[0] = a;
    s_fin[1] = Ki;
    s_fin[2] = bonus;
  }
  }  // warp 0
  if constexpr (kFuse) {
    // the whole step in this launch: the sequence's draft span, built by this CTA
    __syncthreads();
    int ebb = 0;
    build_span(L.b, L.row_vecs, i, s_fin[0], s_fin[1], s_fin[2], true, 0, 1, &ebb);
    if (i == L.b.B - 1) build_tail_pad(L.b, 0, 1, &ebb);
    set_err(L.b.err, ebb);
  }
}

}  // namespace

cudaError_t launch_greedy(const GreedyLaunch& L, cudaStream_t stream) {
  const long long grid = (long long)L.B * (L.K + 1) * L.S;
  const bool lse = L.target_lse != nullptr;
  const bool f = L.fuse_build != 0;
  if (L.dtype == PSPEC_BF16) {
    if (lse) {
      if (f) greedy_sweep_kernel<BF16Tag, true, true><<<(unsigned)grid, kThreads, 0, stream>>>(L);
      else greedy_sweep_kernel<BF16Tag, true, false><<<(unsigned)grid, kThreads, 0, stream>>>(L);
    } else {
      if (f) greedy_sweep_kernel<BF16Tag, false, true><<<(unsigned)grid, kThreads, 0, stream>>>(L);
      else greedy_sweep_kernel<BF16Tag, false, false><<<(unsigned)grid, kThreads, 0, stream>>>(L);
    }
  } else {
    if (lse) {
      if (f) greedy_sweep_kernel<F32Tag, true, true><<<(unsigned)grid, kThreads, 0, stream>>>(L);
      else greedy_sweep_kernel<F32Tag, true, false><<<(unsigned)grid, kThreads, 0, stream>>>(L);
    } else {
      if (f) greedy_sweep_kernel<F32Tag, false, true><<<(unsigned)grid, kThreads, 0, stream>>>(L);
      else greedy_sweep_kernel<F32Tag, false, false><<<(unsigned)grid, kThreads, 0, stream>>>(L);
    }
  }
  return cudaGetLastError();
}

}  // namespace pspec
