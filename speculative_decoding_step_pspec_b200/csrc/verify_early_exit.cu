// verify_early_exit.cu -- target verification that stops at the first rejection.
//
// The accept rule is sequential ("Capstone 14: speculative decoding inference server",
// section "Architecture": accept the prefix, resample for the rejected suffix): once
// draft k is rejected, rows k+1..K of that sequence do not influence the result.  This
// path reads only rows 0..a_i (and row K when every draft passes), which at the pages'
// 60-80 % acceptance is well under half of the full sweep's bytes, and its outputs are
// the full sweep's outputs.
//
// Design (one thread-block cluster of G CTAs per sequence, G = 2, 4, 8, 12 or 16):
//   * position k = 0, 1, ...: each CTA streams its 1/G slice of target row k (and of draft
//     row k for the rejection rule) with 16-byte loads through registers, and every warp
//     reduces its share to one partial -- (max, sum exp) per row, or (max, first index);
//   * the warp writes its partial to shared memory and ARRIVES at the cluster barrier, then
//     WAITS for it: no block barrier and no single-thread merge stand between the loads of
//     one position and the decision.  After the wait every warp of the cluster reads the
//     G x 8 warp partials of the position over distributed shared memory, merges them in a
//     fixed order (bit-identical in every warp) and takes the decision itself (u q < p, or
//     draft == argmax), so no broadcast follows.  Partials are double-buffered by position
//     parity: a warp writing position k+1 has passed the barrier of position k, which every
//     reader of position k-1 had reached first;
//   * the draft tokens sit in lane registers from the start (lane k holds d_k), the
//     uniforms u_0..u_K in shared memory, and the logits at d_k are requested when position
//     k starts, so nothing in the decision waits on a global load.  The decision u q < p is
//     taken in fp32 when the two sides differ by more than 1e-4 (the fp32 error is a few
//     1e-6), else in double as before: the same decisions, without two double exponentials
//     and divisions at every position;
//   * rejection rule: at the stop position each CTA sums r = max(0, p - q) over
//     256-element warp tiles of its slice, re-read right after the statistics pass and
//     backwards (the most recently streamed lines first, while L2 still holds them), two
//     tiles' loads in flight per warp and kept packed as loaded until they are summed; the
//     slice totals are prefix-summed in rank order on every CTA, and the CTA whose slice
//     holds u_K * Z rescans one tile.
//     When the draw is from the target row itself (all drafts passed), the slice totals
//     follow from the statistics already merged and only the CTA holding u_K * Z goes over
//     its slice.
// A large batch may be split over two launches of this kernel (seq0, nseq): the last
// sequences go to wider clusters queued with programmatic dependent launch, which shortens
// the end of the launch, where the last sequences' chains of positions run alone.
#include <cooperative_groups.h>

#include <atomic>

#include "build_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "verify_common.cuh"

namespace cg = cooperative_groups;

namespace pspec {

namespace {

#ifndef PSPEC_EE_REJ_UNROLL
#define PSPEC_EE_REJ_UNROLL 2
#endif
#ifndef PSPEC_EE_MIN_BLOCKS
#define PSPEC_EE_MIN_BLOCKS 6
#endif
// Greedy rule: six vectors per row at five CTAs per SM on the large-batch width, where the
// clusters fill the GPU many times over (b1024: 0.185 ms against 0.191-0.208 for 4-8
// vectors at 4-6 CTAs per SM); eight vectors at four CTAs per SM on the wider clusters of
// small batches and of the tail launch, whose chains of positions are latency-bound (c64:
// 0.033 ms against 0.039 with six vectors).
#ifndef PSPEC_EE_GREEDY_UNROLL
#define PSPEC_EE_GREEDY_UNROLL 6
#endif
#ifndef PSPEC_EE_GREEDY_MIN_BLOCKS
#define PSPEC_EE_GREEDY_MIN_BLOCKS 5
#endif
#ifndef PSPEC_EE_GREEDY_WIDE_UNROLL
#define PSPEC_EE_GREEDY_WIDE_UNROLL 8
#endif
#ifndef PSPEC_EE_GREEDY_WIDE_MIN_BLOCKS
#define PSPEC_EE_GREEDY_WIDE_MIN_BLOCKS 4
#endif

constexpr int kEERejUnroll = PSPEC_EE_REJ_UNROLL;   // vectors per row in flight (rejection)
constexpr int kEEMinBlocks = PSPEC_EE_MIN_BLOCKS;   // CTAs per SM the register budget targets

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Eight consecutive logits [e0, e0+8) of this CTA's slice of the draw rows (global memory,
// usually still in L2 from the statistics pass); -inf at or past the slice end n.
template <typename Tag>
__device__ __forceinline__ void slice_x8(const DrawRow& D, long long lo, int n, int e0,
                                         float (&xt)[8], float (&xq)[8]) {
  if (e0 >= n) {
#pragma unroll
    for (int j = 0; j < 8; ++j) xt[j] = xq[j] = -INFINITY;
    return;
  }
  using elem = typename Tag::elem;
  const elem* tp = static_cast<const elem*>(D.trow) + lo + e0;
  const elem* qp = static_cast<const elem*>(D.qrow) + lo + e0;
  if constexpr (Tag::kVec == 8) {
    unpack(ld_stream(tp), xt, BF16Tag{});
    if (D.resid) unpack(ld_stream(qp), xq, BF16Tag{});
  } else {
    float a[4], b[4];
    unpack(ld_stream(tp), a, F32Tag{});
    unpack(ld_stream(tp + 4), b, F32Tag{});
#pragma unroll
    for (int j = 0; j < 4; ++j) { xt[j] = a[j]; xt[4 + j] = b[j]; }
    if (D.resid) {
      unpack(ld_stream(qp), a, F32Tag{});
      unpack(ld_stream(qp + 4), b, F32Tag{});
#pragma unroll
      for (int j = 0; j < 4; ++j) { xq[j] = a[j]; xq[4 + j] = b[j]; }
    }
  }
}

// Lane sum of r over eight consecutive bf16 logits still packed as loaded: the arithmetic
// of draw_r8 followed by a sequential sum, in the same order, so that the tile sums agree
// bit for bit with the rescans that go through draw_r8.
__device__ __forceinline__ float draw_sum8_bf16(const DrawRow& D, const uint4& wt, const uint4& wq) {
  if (D.mt == -INFINITY) return 0.f;
  const uint32_t tw[4] = {wt.x, wt.y, wt.z, wt.w};
  const uint32_t qw[4] = {wq.x, wq.y, wq.z, wq.w};
  const bool use_q = D.resid && D.mq != -INFINITY;
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float a0, a1;
    ffma2(a0, a1, bf16_lo(tw[k]), bf16_hi(tw[k]), kLog2e, -D.mt);
    float p0, p1;
    fmul2(p0, p1, ex2(a0), ex2(a1), D.inv_st);
    float r0 = p0, r1 = p1;
    if (use_q) {
      float b0, b1, q0, q1;
      ffma2(b0, b1, bf16_lo(qw[k]), bf16_hi(qw[k]), kLog2e, -D.mq);
      fmul2(q0, q1, ex2(b0), ex2(b1), D.inv_sq);
      r0 = fmaxf(p0 - q0, 0.f);
      r1 = fmaxf(p1 - q1, 0.f);
    }
    s += r0;
    s += r1;
  }
  return s;
}

// Warp-wide float max in one redux instruction: the float's bits mapped to an unsigned key
// that orders like the value (negatives inverted, positives with the sign bit set).
__device__ __forceinline__ unsigned float_key(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float warp_max_redux(float v) {
  const unsigned k = __reduce_max_sync(0xffffffffu, float_key(v));
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
// (value, index) argmax over the warp: the largest value, then the lowest index among the
// lanes equal to it (-0 and +0 count as equal, as in vi_better).
__device__ __forceinline__ VI warp_argmax_redux(VI a) {
  const float M = warp_max_redux(a.v);
  const unsigned i = __reduce_min_sync(0xffffffffu, a.v == M ? (unsigned)a.i : 0xffffffffu);
  return VI{M, i == 0xffffffffu ? kNoIndex : (int)i};
}

// A warp's (m, s) partials merged max first: one exponential per lane instead of one per
// shuffle step.
__device__ __forceinline__ MS warp_merge_ms_maxfirst(MS v) {
  const float M = warp_max_redux(v.m);
  float s = (v.m == -INFINITY) ? 0.f : v.s * ex2(v.m - M);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return MS{M, M == -INFINITY ? 0.f : s};
}

// Whole-step fusion: the draft span of sequence i (output rows [qsl_out[i], qsl_out[i+1]),
// clamped into [0, T_cap)), built by the cluster that has just decided a_i and the bonus
// token.  The CTA holding the token (`meta`) writes the rows' metadata and the sequence's
// outputs; every CTA of the cluster copies its share of the hidden rows (the same
// per-sequence code as the build launch, with the cluster's G CTAs as the parts).  The
// cluster of the last sequence also writes the padding rows and the end offset.  The rows
// are exactly those pspec_build_draft_batch writes for a valid offset array; for an invalid
// one every write stays in bounds and the layout bit is set, as there.
__device__ __forceinline__ void ee_build_span(const pspec_build_args& b, long long row_vecs, int i,
                                              int a, int Ki, int token, bool meta, int g, int G) {
  int eb = 0;
  build_span(b, row_vecs, i, a, Ki, token, meta, g, G, &eb);
  if (i == b.B - 1) build_tail_pad(b, g, G, &eb);       // padding rows and the end offset
  set_err(b.err, eb);
}

template <typename Tag, int G, bool kRej, bool kFuse>
__global__ void __launch_bounds__(kThreads, kRej ? kEEMinBlocks
                                                 : (G <= 4 ? PSPEC_EE_GREEDY_MIN_BLOCKS
                                                           : PSPEC_EE_GREEDY_WIDE_MIN_BLOCKS))
ee_kernel(const EarlyExitLaunch L) {
  using elem = typename Tag::elem;
  constexpr int W = Tag::kVec;
  constexpr int U = kRej ? kEERejUnroll                              // vectors in flight per row
                         : (G <= 4 ? PSPEC_EE_GREEDY_UNROLL : PSPEC_EE_GREEDY_WIDE_UNROLL);
  constexpr int BV = U * kThreads;                                  // vectors per row and batch
  constexpr int NP = G * kWarps;                                    // warp partials per position
  constexpr int PL = (NP + 31) / 32;                                // of them per lane
  cg::cluster_group cluster = cg::this_cluster();
  const int g = (int)cluster.block_rank();
  const int i = L.seq0 + (int)(blockIdx.x / G);
  // Every CTA lets the stream's next programmatic launch begin once it has started: the
  // second launch of a split batch, or the draft-batch build, whose CTAs are then placed
  // as this grid's finish and wait (griddepcontrol.wait) for its completion.  A dependent
  // grid launches only after all of this grid's CTAs have started, so none of them can be
  // kept from a slot by the waiting CTAs.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = L.K;
  int ebk = 0;
  const int Ki = draft_count(L.k_len, i, K, &ebk);          // the sequence's own drafts
  if (g == 0 && tid == 0) set_err(L.err, ebk);

  // warp partials by position parity: rejection (mt, st, mq, sq), greedy (value, index bits)
  __shared__ float4 s_part[2][kWarps];
  __shared__ double tot_slice;                               // draw: sum of r over the slice
  __shared__ double tsum[kMaxSliceTiles];
  __shared__ double s_tot[16];                               // per-slice draw totals
  __shared__ int s_tile;
  __shared__ double s_base;
  __shared__ double s_wt[kWarps];                            // draw: per-warp sums of tile sums
  __shared__ int s_found, s_last;
  __shared__ int s_tok;                                      // the emitted token (build)

  const long long lo = (long long)g * L.vs;                 // this CTA's slice [lo, lo + n)
  const int n = (int)max(0LL, min((long long)L.V, lo + L.vs) - lo);
  const int nvec = n / W;                                   // n is a multiple of 8
  // this CTA's slice of target row k / draft row k (recomputed where needed rather than
  // kept in registers through the stream)
  auto trow_of = [&](int kk) {
    return static_cast<const elem*>(L.target) + ((long long)i * (K + 1) + kk) * L.ld + lo;
  };
  auto qrow_of = [&](int kk) {
    return static_cast<const elem*>(L.draft) + ((long long)i * K + kk) * L.ld + lo;
  };

  // lane k of every warp holds draft k of the sequence (-1 past K_i)
  const int dreg = lane < Ki ? __ldg(L.draft_tokens + (long long)i * K + lane) : -1;
  // the uniforms of positions 0..K, read from shared memory at each decision
  __shared__ float s_u[32];
  if (kRej && tid <= K) s_u[tid] = __ldg(L.uniforms + (long long)i * (K + 1) + tid);
  __syncthreads();

  // decision state of the stop position: every warp computes the same values and warp 0
  // leaves them in shared memory for the draw, so none of them occupies registers while
  // the rows stream
  __shared__ float s_dM[2];                                  // (Mt, Mq)
  __shared__ double s_dS[2];                                 // (St, Sq)
  int gk = 0;                                                // greedy: argmax of the stop row
  int k = 0;
  for (;; ++k) {
    const bool has_q = kRej && k < Ki;
    const elem* trow = trow_of(k);
    const elem* qrow = has_q ? qrow_of(k) : trow;
    // the draft token of this position and (rejection) the logits there, wanted at the
    // decision: requested now, so the stream below hides their latency
    const int d = k < Ki ? __shfl_sync(0xffffffffu, dreg, k & 31) : -1;
    float xt_d = 0.f, xq_d = 0.f;
    if (kRej && lane == 0 && d >= 0 && d < L.V) {
      xt_d = load_scalar(trow - lo, d);
      xq_d = load_scalar(qrow - lo, d);
    }
    // ---- stream this CTA's slice of the position's rows
    MSAcc at = msacc_init(), aq = msacc_init();
    VI best{-INFINITY, kNoIndex};
    {
      const uint4* tv = reinterpret_cast<const uint4*>(trow);
      const uint4* qv = reinterpret_cast<const uint4*>(qrow);
      int v0 = tid;
      for (; v0 + (U - 1) * kThreads < nvec; v0 += BV) {            // full batches
        uint4 bt[U], bq[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          bt[u] = ld_stream(tv + v0 + u * kThreads);
          if (has_q) bq[u] = ld_stream(qv + v0 + u * kThreads);
        }
        if constexpr (kRej) {
          consume_ms_batch<Tag, U>(bt, at);
          if (has_q) consume_ms_batch<Tag, U>(bq, aq);
        } else {
#pragma unroll
          for (int u = 0; u < U; ++u) consume_argmax<Tag>(bt[u], lo + (long long)(v0 + u * kThreads) * W, best);
        }
      }
      for (; v0 < nvec; v0 += kThreads) {                            // the rest, one by one
        const uint4 x = ld_stream(tv + v0);
        if constexpr (kRej) {
          consume_ms<Tag>(x, at);
          if (has_q) consume_ms<Tag>(ld_stream(qv + v0), aq);
        } else {
          consume_argmax<Tag>(x, lo + (long long)v0 * W, best);
        }
      }
    }
    // ---- this warp's partial, then the cluster barrier in two halves
    if constexpr (kRej) {
      const MS mt = warp_merge_ms_maxfirst(msacc_final(at));
      const MS mq = warp_merge_ms_maxfirst(msacc_final(aq));
      if (lane == 0) s_part[k & 1][warp] = make_float4(mt.m, mt.s, mq.m, mq.s);
    } else {
      best = warp_argmax_redux(best);
      if (lane == 0) s_part[k & 1][warp] = make_float4(best.v, __int_as_float(best.i), 0.f, 0.f);
    }
    __syncwarp();
    cluster_arrive();
    cluster_wait();

    // ---- every warp takes the same decision from the same partials, merged in one fixed
    // order (lane l holds partials l, l + 32, ...: CTA p / 8, warp p % 8)
    float4 pr[PL];
#pragma unroll
    for (int j = 0; j < PL; ++j) {
      const int p = lane + 32 * j;
      if (p < NP) {
        pr[j] = *cluster.map_shared_rank(&s_part[k & 1][p % kWarps], (unsigned)(p / kWarps));
      } else {
        pr[j] = kRej ? make_float4(-INFINITY, 0.f, -INFINITY, 0.f)
                     : make_float4(-INFINITY, __int_as_float(kNoIndex), 0.f, 0.f);
      }
    }
    bool stop;
    if constexpr (kRej) {
      float Mt = pr[0].x, Mq = pr[0].z;
#pragma unroll
      for (int j = 1; j < PL; ++j) { Mt = fmaxf(Mt, pr[j].x); Mq = fmaxf(Mq, pr[j].z); }
      Mt = warp_max_redux(Mt);
      Mq = warp_max_redux(Mq);
      // each warp partial s * 2^(m - M) scaled in fp32 (the SFU exponential: a double exp2
      // per partial cost ~2 % of the verify), the terms summed in double
      double st = 0.0, sq = 0.0;
#pragma unroll
      for (int j = 0; j < PL; ++j) {
        if (pr[j].x != -INFINITY) st += (double)(pr[j].y * ex2(pr[j].x - Mt));
        if (has_q && pr[j].z != -INFINITY) sq += (double)(pr[j].w * ex2(pr[j].z - Mq));
      }
      st = warp_sum_d(st);
      sq = warp_sum_d(sq);
      xt_d = __shfl_sync(0xffffffffu, xt_d, 0);
      xq_d = __shfl_sync(0xffffffffu, xq_d, 0);
      bool accept = false;
      if (k < Ki && d >= 0 && d < L.V) {
        const float uf = s_u[k];
        // fp32 first; the double form decides whenever the two sides are within 1e-4
        const float p32 = (Mt != -INFINITY && xt_d != -INFINITY)
                              ? ex2(fmaf(xt_d, kLog2e, -Mt)) / (float)st : 0.f;
        const float q32 = (Mq != -INFINITY && xq_d != -INFINITY)
                              ? ex2(fmaf(xq_d, kLog2e, -Mq)) / (float)sq : 0.f;
        const float lhs = uf * q32;
        if (p32 > 1e-30f && q32 > 1e-30f && fabsf(lhs - p32) > 1e-4f * fmaxf(lhs, p32)) {
          accept = lhs < p32;
        } else {
          const double pp = (Mt != -INFINITY && xt_d != -INFINITY)
                                ? exp2((double)xt_d * (double)kLog2e - (double)Mt) / st : 0.0;
          const double qq = (Mq != -INFINITY && xq_d != -INFINITY)
                                ? exp2((double)xq_d * (double)kLog2e - (double)Mq) / sq : 0.0;
          const double u = (double)uf;
          accept = qq > 0.0 ? (u * qq < pp) : (pp > 0.0);
        }
      }
      stop = !accept;
      if (stop && warp == 0 && lane == 0) {
        s_dM[0] = Mt; s_dM[1] = Mq;
        s_dS[0] = st; s_dS[1] = sq;
      }
    } else {
      VI b{pr[0].x, __float_as_int(pr[0].y)};
#pragma unroll
      for (int j = 1; j < PL; ++j) {
        const VI c{pr[j].x, __float_as_int(pr[j].y)};
        if (vi_better(c, b)) b = c;
      }
      b = warp_argmax_redux(b);           // largest value, lowest index among equals
      gk = b.i == kNoIndex ? 0 : b.i;
      stop = !(k < Ki && d >= 0 && d < L.V && d == gk);
    }
    if (stop) {
      if (g == 0 && warp == 0) {
        // outputs the two rules share: accepted drafts, the -1 tail, the count, range errors
        const int bad = lane < Ki && (dreg < 0 || dreg >= L.V);
        if (lane < k) L.out_tokens[(long long)i * (K + 1) + lane] = dreg;
        if (lane <= K && lane > k) L.out_tokens[(long long)i * (K + 1) + lane] = -1;
        if (__any_sync(0xffffffffu, bad) && lane == 0) set_err(L.err, PSPEC_DEVERR_TOKEN_RANGE);
        if (lane == 0) {
          L.accepted_len[i] = k;
          if constexpr (!kRej) { L.bonus[i] = gk; L.out_tokens[(long long)i * (K + 1) + k] = gk; }
        }
      }
      break;
    }
  }

  int meta_g = 0;                                            // the CTA that knows the token
  int token = gk;
  if constexpr (kRej) {
    // ---- the draw at the stop position a = k: r = max(0, p_a - q_a), or p_K after K passes
    const int a = k;
    __syncthreads();                                         // the stop position's state
    const float dMt = s_dM[0], dMq = s_dM[1];
    const double dSt = s_dS[0], dSq = s_dS[1];
    DrawRow D;
    D.trow = trow_of(a) - lo;
    D.resid = a < Ki;
    D.qrow = D.resid ? qrow_of(a) - lo : D.trow;
    D.mt = dMt; D.inv_st = dSt > 0.0 ? (float)(1.0 / dSt) : 0.f;
    D.mq = dMq; D.inv_sq = dSq > 0.0 ? (float)(1.0 / dSq) : 0.f;
    const int ntiles = (n + 255) / 256;
    const double u = (double)L.uniforms[(long long)i * (K + 1) + Ki];
    // Sums of r over this CTA's tiles, from the last one down (bf16: the warps take
    // adjacent pairs, every 8th pair; fp32: every 8th tile): the statistics pass streamed
    // the slice from its start, so its end is the part
    // most likely still in L2, and going backwards the re-read meets the freshest lines
    // before the other clusters' streams evict them.
    auto tile_pass = [&]() {
      if constexpr (Tag::kVec == 8) {
        // two adjacent tiles' loads in flight per warp, kept packed until they are summed,
        // and the two tile sums reduced across the warp together
        const uint16_t* tp = static_cast<const uint16_t*>(D.trow) + lo;
        const uint16_t* qp = static_cast<const uint16_t*>(D.qrow) + lo;
        double wsum = 0.0;
        for (int t = ntiles - 1 - 2 * warp; t >= 0; t -= 2 * kWarps) {
          const int t2 = t - 1;
          const int e0 = t * 256 + lane * 8, e1 = t2 * 256 + lane * 8;
          const bool in0 = e0 < n, in1 = t2 >= 0 && e1 < n;
          uint4 a = make_uint4(0, 0, 0, 0), aq = a, b = a, bq = a;
          if (in0) {
            a = ld_stream(tp + e0);
            if (D.resid) aq = ld_stream(qp + e0);
          }
          if (in1) {
            b = ld_stream(tp + e1);
            if (D.resid) bq = ld_stream(qp + e1);
          }
          double d0 = (double)(in0 ? draw_sum8_bf16(D, a, aq) : 0.f);
          double d1 = (double)(in1 ? draw_sum8_bf16(D, b, bq) : 0.f);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            d0 += __shfl_xor_sync(0xffffffffu, d0, o);
            d1 += __shfl_xor_sync(0xffffffffu, d1, o);
          }
          if (lane == 0) {
            tsum[t] = d0;
            if (t2 >= 0) tsum[t2] = d1;
          }
          wsum += d0;
          if (t2 >= 0) wsum += d1;
        }
        if (lane == 0) s_wt[warp] = wsum;
      } else {
        double wsum = 0.0;
        for (int t = ntiles - 1 - warp; t >= 0; t -= kWarps) {
          float xt[8], xq[8], r[8];
          slice_x8<Tag>(D, lo, n, t * 256 + lane * 8, xt, xq);
          draw_r8(D, xt, xq, r);
          float sum = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) sum += r[j];
          const double ts = warp_sum_d((double)sum);
          if (lane == 0) tsum[t] = ts;
          wsum += ts;
        }
        if (lane == 0) s_wt[warp] = wsum;
      }
    };
    bool own_pass_done = false;
    if (D.resid) {
      tile_pass();
      __syncthreads();
      if (tid == 0) {
        double tt = 0.0;
        for (int w = 0; w < kWarps; ++w) tt += s_wt[w];
        tot_slice = tt;
      }
      cluster.sync();                                        // slice totals in place
      if (tid < G) s_tot[tid] = *cluster.map_shared_rank(&tot_slice, (unsigned)tid);
      __syncthreads();
      double Z0 = 0.0;
      for (int h = 0; h < G; ++h) Z0 += s_tot[h];
      own_pass_done = true;
      if (Z0 == 0.0) {                                       // residual vanished: draw from p
        D.resid = false;
        D.qrow = D.trow;
        own_pass_done = false;
      }
    }
    if (!D.resid) {
      // Drawing from the target row itself (all K drafts passed, or the residual was
      // empty): slice h's total sum_w s_w 2^(m_w - M) / S follows from the statistics
      // already merged, so only the CTA that holds u*Z has to go over its slice again.
      if (tid < G) {
        double tot = 0.0;
        if (dSt > 0.0)
          for (int w = 0; w < kWarps; ++w) {
            const float4 ph = *cluster.map_shared_rank(&s_part[a & 1][w], (unsigned)tid);
            if (ph.x != -INFINITY) tot += (double)(ph.y * ex2(ph.x - dMt));   // as St's terms
          }
        s_tot[tid] = tot / (dSt > 0.0 ? dSt : 1.0);
      }
      __syncthreads();
    }
    double Z = 0.0;
    for (int h = 0; h < G; ++h) Z += s_tot[h];
    const double thr = u * Z;
    int owner = -1, last_pos = -1;
    double base = 0.0, run = 0.0;
    for (int h = 0; h < G; ++h) {
      const double th = s_tot[h];
      if (th > 0.0) last_pos = h;
      if (owner < 0 && th > 0.0 && run + th > thr) { owner = h; base = run; }
      run += th;
    }
    const bool crossing = owner >= 0;
    if (!crossing && Z > 0.0) owner = last_pos;              // rounding: last slice with mass
    meta_g = owner >= 0 ? owner : 0;
    if (g == owner) {
      if (!own_pass_done) {
        tile_pass();
        __syncthreads();
      }
      {
        // the tile holding u*Z: every thread takes a run of consecutive tile sums, one
        // block-wide exclusive scan gives each run its base, the run holding the crossing
        // (or the last positive tile, when rounding leaves none) reports it
        if (tid == 0) { s_found = 0x7fffffff; s_last = -1; }
        const int per = (ntiles + kThreads - 1) / kThreads;
        const int t0 = min(tid * per, ntiles), t1 = min(t0 + per, ntiles);
        double loc = 0.0;
        for (int t = t0; t < t1; ++t) loc += tsum[t];
        double incl = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (lane == 31) s_wt[warp] = incl;
        __syncthreads();
        double b2 = base + incl - loc;
        for (int w = 0; w < warp; ++w) b2 += s_wt[w];
        int mine = 0x7fffffff, lastp = -1;
        double mb = 0.0;
        for (int t = t0; t < t1; ++t) {
          const double ts = tsum[t];
          if (ts > 0.0) lastp = t;
          if (mine == 0x7fffffff && crossing && ts > 0.0 && b2 + ts > thr) { mine = t; mb = b2; }
          b2 += ts;
        }
        if (mine != 0x7fffffff) atomicMin(&s_found, mine);
        if (lastp >= 0) atomicMax(&s_last, lastp);
        __syncthreads();
        if (s_found != 0x7fffffff) {
          if (mine == s_found) { s_tile = mine; s_base = mb; }
        } else if (tid == 0) {
          s_tile = s_last;                                   // no crossing: its last positive r
          s_base = -INFINITY;
        }
      }
      __syncthreads();
      if (warp == 0) {
        int tok = 0;
        const int tile = s_tile;
        if (tile >= 0) {
          const int e0 = tile * 256 + lane * 8;
          float xt[8], xq[8], r[8];
          slice_x8<Tag>(D, lo, n, e0, xt, xq);
          draw_r8(D, xt, xq, r);
          float incl[8], acc = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) { acc += r[j]; incl[j] = acc; }
          double inc = acc;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const double v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
          }
          const double ex = inc - (double)acc;
          const double tb = s_base;
          int cand = 0x7fffffff, lastp = -1;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (r[j] > 0.f) lastp = (int)(lo + e0 + j);
            if (cand == 0x7fffffff && r[j] > 0.f && tb + ex + (double)incl[j] > thr)
              cand = (int)(lo + e0 + j);             // only a token with mass can cross
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            cand = min(cand, __shfl_xor_sync(0xffffffffu, cand, o));
            lastp = max(lastp, __shfl_xor_sync(0xffffffffu, lastp, o));
          }
          tok = cand != 0x7fffffff ? cand : (lastp >= 0 ? lastp : 0);
        }
        if (lane == 0) {
          L.out_tokens[(long long)i * (K + 1) + a] = tok;
          L.bonus[i] = tok;
          if (L.residual_mass) L.residual_mass[i] = (float)Z;
          s_tok = tok;
        }
      }
    } else if (owner < 0 && g == 0 && tid == 0) {            // no mass anywhere: token 0
      L.out_tokens[(long long)i * (K + 1) + a] = 0;
      L.bonus[i] = 0;
      if (L.residual_mass) L.residual_mass[i] = 0.f;
      s_tok = 0;
    }
    if constexpr (kFuse) {
      __syncthreads();
      token = g == meta_g ? s_tok : 0;
    }
  }
  cluster.sync();                                            // no remote reads after exit
  if constexpr (kFuse)                                       // the whole step in this launch
    ee_build_span(L.b, L.row_vecs, i, k, Ki, g == meta_g ? token : 0, g == meta_g, g, G);
  // second launch of a split batch: its completion implies the first grid's, so work queued
  // after it on the stream sees every sequence's outputs
  if (L.pdl == 2 && blockIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Launches the variant, or with max_clusters set only asks how many of its clusters can be
// resident at once (cudaOccupancyMaxActiveClusters) and launches nothing.
template <typename Tag, int G, bool kRej, bool kFuse>
cudaError_t launch_ee(const EarlyExitLaunch& L, cudaStream_t stream, int* max_clusters) {
  auto kern = ee_kernel<Tag, G, kRej, kFuse>;
  cudaError_t e = cudaSuccess;
  if (G > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)(L.nseq > 0 ? L.nseq : 1) * G), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = L.pdl == 2 ? 2 : 1;
  if (max_clusters) return cudaOccupancyMaxActiveClusters(max_clusters, kern, &cfg);
  return cudaLaunchKernelEx(&cfg, kern, L);
}

template <int G>
cudaError_t launch_ee_g(const EarlyExitLaunch& L, cudaStream_t s, int* m) {
  const bool bf = L.dtype == PSPEC_BF16;
  if (L.fuse_build) {
    if (L.rejection)
      return bf ? launch_ee<BF16Tag, G, true, true>(L, s, m) : launch_ee<F32Tag, G, true, true>(L, s, m);
    return bf ? launch_ee<BF16Tag, G, false, true>(L, s, m) : launch_ee<F32Tag, G, false, true>(L, s, m);
  }
  if (L.rejection)
    return bf ? launch_ee<BF16Tag, G, true, false>(L, s, m) : launch_ee<F32Tag, G, true, false>(L, s, m);
  return bf ? launch_ee<BF16Tag, G, false, false>(L, s, m) : launch_ee<F32Tag, G, false, false>(L, s, m);
}

cudaError_t dispatch_ee(const EarlyExitLaunch& L, cudaStream_t stream, int* m) {
  switch (L.G) {
    case 2: return launch_ee_g<2>(L, stream, m);
    case 4: return launch_ee_g<4>(L, stream, m);
    case 8: return launch_ee_g<8>(L, stream, m);
    case 12: return launch_ee_g<12>(L, stream, m);
    default: return launch_ee_g<16>(L, stream, m);
  }
}

}  // namespace

cudaError_t launch_early_exit(const EarlyExitLaunch& L, cudaStream_t stream) {
  return dispatch_ee(L, stream, nullptr);
}

int early_exit_max_clusters(const EarlyExitLaunch& L) {
  // cached per device and variant: 16 devices x 5 cluster sizes x dtype x rule x fusion
  static std::atomic<int> cache[16 * 5 * 8];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int gi = L.G == 2 ? 0 : L.G == 4 ? 1 : L.G == 8 ? 2 : L.G == 12 ? 3 : 4;
  const int idx = ((((dev & 15) * 5 + gi) * 2 + (L.dtype == PSPEC_BF16)) * 2 + (L.rejection != 0)) * 2 +
                  (L.fuse_build != 0);
  const int c = cache[idx].load(std::memory_order_relaxed);
  if (c > 0) return c - 1;
  int n = 0;
  if (dispatch_ee(L, nullptr, &n) != cudaSuccess) {
    cudaGetLastError();                                       // a failed query is not sticky
    return 0;
  }
  cache[idx].store(n + 1, std::memory_order_relaxed);
  return n;
}

}  // namespace pspec
