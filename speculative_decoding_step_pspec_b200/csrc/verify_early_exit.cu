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
//     row k for the rejection rule) with 16-byte loads -- two vectors per row in flight per
//     thread at six CTAs per SM for the rejection rule, eight at four CTAs per SM for the
//     greedy rule -- and reduces it to (max, sum exp) or to its argmax;
//   * one cluster barrier; then every CTA reads the G slice partials through distributed
//     shared memory in rank order and takes the same decision (u q < p, or draft ==
//     argmax), so no second barrier or broadcast is needed (partials are double-buffered
//     by position parity, so the next position cannot overwrite what a slower CTA reads);
//   * rejection rule: at the stop position each CTA sums r = max(0, p - q) over
//     256-element warp tiles of its slice, re-read right after the statistics pass (from
//     L2 while the clusters in flight hold less than it, from HBM at large batches); the
//     slice totals are prefix-summed in rank order on every CTA, and the CTA whose slice
//     holds u_K * Z rescans one tile.  When the draw is from the target row itself (all
//     drafts passed), the slice totals follow from the statistics already merged and only
//     the CTA holding u_K * Z goes over its slice.
// Rows are held in registers, not shared memory, so that six CTAs fit per SM and about 220
// sequences are in flight: measured on B200, caching each 100 KB slice pair in shared
// memory (two CTAs per SM) left HBM idle between positions, and streaming through per-warp
// rings of bulk copies (kRing, an option) was slower than registers at every batch tried.
// A large batch may be split over two launches of this kernel (seq0, nseq): the last
// sequences go to wider clusters queued with programmatic dependent launch, which shortens
// the end of the launch, where the last sequences' chains of positions run alone.
#include <cooperative_groups.h>

#include <atomic>

#include "build_common.cuh"
#include "bulk_ring.cuh"
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
// Greedy rule (one row per position): 4 CTAs per SM with 8 vectors in flight per thread
// measured 1.7 % faster at B=1024 than 6 CTAs with 4 (0.207 vs 0.210 ms); the rejection
// rule keeps 6 CTAs per SM with 2 vectors per row: fewer, deeper CTAs (3 x 4, 4 x 4,
// 2 x 8) were 5-50 % slower -- independent sequences hide the per-position latency better.
#ifndef PSPEC_EE_GREEDY_UNROLL
#define PSPEC_EE_GREEDY_UNROLL 8
#endif
#ifndef PSPEC_EE_GREEDY_MIN_BLOCKS
#define PSPEC_EE_GREEDY_MIN_BLOCKS 4
#endif

// Streaming through shared memory (kRing): each warp owns kRingStages stages of
// kRingBytes per row, filled by bulk asynchronous copies; CTAs per SM as the shared memory
// allows.
#ifndef PSPEC_EE_RING_BYTES
#define PSPEC_EE_RING_BYTES 2048
#endif
#ifndef PSPEC_EE_RING_STAGES
#define PSPEC_EE_RING_STAGES 2
#endif
#ifndef PSPEC_EE_RING_MIN_BLOCKS
#define PSPEC_EE_RING_MIN_BLOCKS 3
#endif
#ifndef PSPEC_EE_RING_GREEDY_MIN_BLOCKS
#define PSPEC_EE_RING_GREEDY_MIN_BLOCKS 5
#endif
constexpr int kRingBytes = PSPEC_EE_RING_BYTES;          // one row's share of a stage
constexpr int kRingStages = PSPEC_EE_RING_STAGES;
constexpr int kRingVecs = kRingBytes / 16;               // 16-byte vectors per row and stage
constexpr int kRingLaneVecs = kRingVecs / 32;
static_assert(kRingVecs % 32 == 0 && kRingLaneVecs >= 1, "ring stage: whole vectors per lane");

// Dynamic shared memory of the kRing variants: the warps' stages.
constexpr int ring_smem_bytes(bool rej) { return kWarps * kRingStages * (rej ? 2 : 1) * kRingBytes; }

constexpr int kEERejUnroll = PSPEC_EE_REJ_UNROLL;   // vectors per row in flight (rejection)
constexpr int kEEMinBlocks = PSPEC_EE_MIN_BLOCKS;   // CTAs per SM the register budget targets

// A CTA's contribution to one position.
struct EEPart {
  float mt, st;      // (max, sum exp) of its slice of the target row
  float mq, sq;      // the same for the draft row
  float bv;          // argmax value of its target slice (greedy)
  int bi;            // argmax index (global token id; kNoIndex when empty)
};

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

// The same eight elements in two steps, so that several groups' loads can be in flight
// before any of them is unpacked.
template <typename Tag>
struct SliceRaw {
  uint4 t[8 / Tag::kVec], q[8 / Tag::kVec];
  bool live;
};

template <typename Tag>
__device__ __forceinline__ void slice_load(const DrawRow& D, long long lo, int n, int e0,
                                           SliceRaw<Tag>& R) {
  R.live = e0 < n;
  if (!R.live) return;
  using elem = typename Tag::elem;
  const elem* tp = static_cast<const elem*>(D.trow) + lo + e0;
  const elem* qp = static_cast<const elem*>(D.qrow) + lo + e0;
#pragma unroll
  for (int k = 0; k < 8 / Tag::kVec; ++k) {
    R.t[k] = ld_stream(tp + k * Tag::kVec);
    if (D.resid) R.q[k] = ld_stream(qp + k * Tag::kVec);
  }
}

template <typename Tag>
__device__ __forceinline__ void slice_values(const DrawRow& D, const SliceRaw<Tag>& R,
                                             float (&xt)[8], float (&xq)[8]) {
  if (!R.live) {
#pragma unroll
    for (int j = 0; j < 8; ++j) xt[j] = xq[j] = -INFINITY;
    return;
  }
  if constexpr (Tag::kVec == 8) {
    unpack(R.t[0], xt, BF16Tag{});
    if (D.resid) unpack(R.q[0], xq, BF16Tag{});
  } else {
    float a[4], b[4];
    unpack(R.t[0], a, F32Tag{});
    unpack(R.t[1], b, F32Tag{});
#pragma unroll
    for (int j = 0; j < 4; ++j) { xt[j] = a[j]; xt[4 + j] = b[j]; }
    if (D.resid) {
      unpack(R.q[0], a, F32Tag{});
      unpack(R.q[1], b, F32Tag{});
#pragma unroll
      for (int j = 0; j < 4; ++j) { xq[j] = a[j]; xq[4 + j] = b[j]; }
    }
  }
}

#ifndef PSPEC_EE_DRAW_U
#define PSPEC_EE_DRAW_U 1
#endif

// Whole-step fusion: the draft span of sequence i (output rows [qsl_out[i], qsl_out[i+1]),
// clamped into [0, T_cap)), built by the cluster that has just decided a_i and the bonus
// token.  The CTA holding the token (`meta`) writes the rows' metadata and the sequence's
// outputs; every CTA of the cluster copies its share of the hidden rows (one warp per
// row).  The cluster of the last sequence also writes the padding rows and the end offset.
// The rows are exactly those pspec_build_draft_batch writes for a valid offset array; for
// an invalid one every write stays in bounds and the layout bit is set, as there.
__device__ __forceinline__ void ee_build_span(const pspec_build_args& b, long long row_vecs, int i,
                                           int a, int Ki, int token, bool meta, int g, int G) {
  const long long q0 = build_qout(b, i), q1 = build_qout(b, i + 1);
  const long long lo = q0 < 0 ? 0 : q0;
  const long long hi = q1 > b.T_cap ? (long long)b.T_cap : q1;
  int eb = 0;
  if (meta) {
    for (long long t = lo + threadIdx.x; t < hi; t += kThreads)
      build_write_row(b, t, build_classify(b, i, t - q0, a, Ki, token), &eb);
    if (threadIdx.x == 0) build_write_seq(b, i, a, Ki, &eb);
  }
  if (b.draft_hidden) {
    const int warp = threadIdx.x >> 5;
    for (long long t = lo + (long long)g * kWarps + warp; t < hi; t += (long long)G * kWarps)
      build_copy_hidden(b, row_vecs, t, build_classify(b, i, t - q0, a, Ki, token));
  }
  if (i == b.B - 1) {                                  // padding rows and the end offset
    const BuildRow pad{PSPEC_ROW_PAD, -1, b.pad_id, 0, -1};
    const long long first = build_qout(b, 0);
    const long long head = first < 0 ? 0 : (first > b.T_cap ? (long long)b.T_cap : first);
    const long long tail = q1 < 0 ? 0 : q1;
    const long long step = (long long)G * kThreads;
    for (long long t = (long long)g * kThreads + threadIdx.x; t < head; t += step)
      build_write_row(b, t, pad, &eb);
    for (long long t = tail + (long long)g * kThreads + threadIdx.x; t < b.T_cap; t += step)
      build_write_row(b, t, pad, &eb);
    if (g == 0 && threadIdx.x == 0) build_write_seq(b, b.B, 0, b.K, &eb);
  }
  set_err(b.err, eb);
}

template <typename Tag, int G, bool kRej, bool kFuse, bool kRing>
__global__ void __launch_bounds__(kThreads,
                                  kRing ? (kRej ? PSPEC_EE_RING_MIN_BLOCKS : PSPEC_EE_RING_GREEDY_MIN_BLOCKS)
                                        : (kRej ? kEEMinBlocks : PSPEC_EE_GREEDY_MIN_BLOCKS))
ee_kernel(const EarlyExitLaunch L) {
  using elem = typename Tag::elem;
  constexpr int W = Tag::kVec;
  constexpr int U = kRej ? kEERejUnroll : PSPEC_EE_GREEDY_UNROLL;  // vectors in flight per row
  cg::cluster_group cluster = cg::this_cluster();
  const int g = (int)cluster.block_rank();
  const int i = L.seq0 + (int)(blockIdx.x / G);
  if (L.pdl == 1) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = L.K;
  int ebk = 0;
  const int Ki = draft_count(L.k_len, i, K, &ebk);          // the sequence's own drafts
  if (g == 0 && tid == 0) set_err(L.err, ebk);

  __shared__ EEPart part[2];                                 // by position parity
  __shared__ double tot_slice;                               // draw: sum of r over the slice
  __shared__ double tsum[kMaxSliceTiles];
  __shared__ MS s_ms[2][kWarps];
  __shared__ VI s_vi[kWarps];
  __shared__ int s_stop;
  __shared__ float s_dec[4];
  __shared__ double s_St;                                    // target row's S at the stop
  __shared__ double s_tot[16];                               // per-slice draw totals
  __shared__ int s_tile;
  __shared__ double s_base;
  __shared__ int s_tok;                                      // the emitted token (build)

  const long long lo = (long long)g * L.vs;                 // this CTA's slice [lo, lo + n)
  const int n = (int)max(0LL, min((long long)L.V, lo + L.vs) - lo);
  const int nvec = n / W;                                   // n is a multiple of 8

  // kRing: warp w streams the run [wlo, wlo + wn) of the slice (multiples of 8 elements) in
  // chunks of SE elements through its own stages; gidx counts the chunks it has consumed,
  // which fixes each stage's mbarrier phase across positions.
  constexpr int kRows = kRej ? 2 : 1;
  constexpr int SE = kRingBytes / (int)sizeof(elem);
  __shared__ __align__(8) uint64_t s_bar[kRing ? kWarps * kRingStages : 1];
  extern __shared__ __align__(16) uint4 s_ring[];
  const int wper = ((n + kWarps - 1) / kWarps + 7) / 8 * 8;
  const int wlo = min(n, warp * wper);
  const int wn = min(n, wlo + wper) - wlo;
  const int nch = (wn + SE - 1) / SE;
  uint32_t gidx = 0;                                          // chunks consumed
  uint32_t issued = 0;                                        // chunks requested
  bool ring_ok = true;
  uint4* const ring = s_ring + (size_t)warp * kRingStages * kRows * kRingVecs;
  uint64_t* const bar = s_bar + (kRing ? warp * kRingStages : 0);
  if constexpr (kRing) {
    if (lane == 0) {
      for (int s = 0; s < kRingStages; ++s) mbar_init(&bar[s]);
      mbar_init_fence();
    }
    __syncwarp();
  }
  // chunk c of this warp's run of rows (tr, qr) into stage gi mod kRingStages (lane 0 only)
  auto issue = [&](const elem* tr, const elem* qr, bool hq, int c, uint32_t gi) {
    const int s = (int)(gi % kRingStages);
    const int e0 = wlo + c * SE;
    const unsigned bytes = (unsigned)(min(SE, wn - c * SE) * (int)sizeof(elem));
    uint4* st = ring + s * kRows * kRingVecs;
    fence_async_shared();
    mbar_arrive_expect(&bar[s], hq ? 2 * bytes : bytes);
    bulk_copy_g2s(st, tr + lo + e0, bytes, &bar[s]);
    if (hq) bulk_copy_g2s(st + kRingVecs, qr + lo + e0, bytes, &bar[s]);
  };

  int k = 0;
  for (; k <= Ki; ++k) {
    const bool has_q = kRej && k < Ki;
    const elem* trow = static_cast<const elem*>(L.target) + ((long long)i * (K + 1) + k) * L.ld;
    const elem* qrow = has_q ? static_cast<const elem*>(L.draft) + ((long long)i * K + k) * L.ld : trow;
    // the logits at the draft token, needed by every CTA's decision: in flight meanwhile
    float xt_d = 0.f, xq_d = 0.f;
    int d = -1;
    if (k < Ki && warp == 0) {
      d = L.draft_tokens[(long long)i * K + k];
      if (kRej && d >= 0 && d < L.V) {
        xt_d = load_scalar(trow, d);
        xq_d = load_scalar(qrow, d);
      }
    }
    // ---- stream this CTA's slice of the position's rows
    MSAcc at = msacc_init(), aq = msacc_init();
    VI best{-INFINITY, kNoIndex};
    if constexpr (kRing) {
      if (ring_ok)
        for (int c = 0; c < nch && c < kRingStages; ++c, ++issued)
          if (lane == 0) issue(trow, qrow, has_q, c, gidx + (uint32_t)c);
      for (int c = 0; c < nch; ++c, ++gidx) {
        const int s = (int)(gidx % kRingStages);
        if (ring_ok) {
          const bool ok =
              __all_sync(0xffffffffu, mbar_wait(&bar[s], (gidx / kRingStages) & 1u, L.spin_limit));
          if (!ok) {
            ring_ok = false;                             // no further copies from this warp
            if (lane == 0) set_err(L.err, PSPEC_DEVERR_TIMEOUT);
          }
        }
        const uint4* st = ring + s * kRows * kRingVecs;
        const int mv = min(SE, wn - c * SE) / W;
        const long long e0 = lo + wlo + (long long)c * SE;   // token id of the chunk's start
        if (mv == kRingVecs) {
          uint4 bt[kRingLaneVecs], bq[kRingLaneVecs];
#pragma unroll
          for (int u = 0; u < kRingLaneVecs; ++u) {
            bt[u] = st[lane + 32 * u];
            if (has_q) bq[u] = st[kRingVecs + lane + 32 * u];
          }
          if constexpr (kRej) {
            consume_ms_batch<Tag, kRingLaneVecs>(bt, at);
            if (has_q) consume_ms_batch<Tag, kRingLaneVecs>(bq, aq);
          } else {
#pragma unroll
            for (int u = 0; u < kRingLaneVecs; ++u)
              consume_argmax<Tag>(bt[u], e0 + (long long)(lane + 32 * u) * W, best);
          }
        } else {
          for (int v = lane; v < mv; v += 32) {
            if constexpr (kRej) {
              consume_ms<Tag>(st[v], at);
              if (has_q) consume_ms<Tag>(st[kRingVecs + v], aq);
            } else {
              consume_argmax<Tag>(st[v], e0 + (long long)v * W, best);
            }
          }
        }
        __syncwarp();                                        // the stage is read: refill it
        if (ring_ok && c + kRingStages < nch) {
          if (lane == 0) issue(trow, qrow, has_q, c + kRingStages, gidx + kRingStages);
          ++issued;
        }
      }
    } else {                                                 // through registers
      const uint4* tv = reinterpret_cast<const uint4*>(trow + lo);
      const uint4* qv = reinterpret_cast<const uint4*>(qrow + lo);
      int v0 = tid;
      for (; v0 + (U - 1) * kThreads < nvec; v0 += U * kThreads) {   // full batches
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
    MS mt = msacc_final(at), mq = msacc_final(aq);
    if constexpr (kRej) {
      mt = warp_merge_ms(mt);
      mq = warp_merge_ms(mq);
      if (lane == 0) { s_ms[0][warp] = mt; s_ms[1][warp] = mq; }
    } else {
      best = warp_argmax(best);
      if (lane == 0) s_vi[warp] = best;
    }
    __syncthreads();
    if (tid == 0) {
      EEPart& pp = part[k & 1];
      if constexpr (kRej) {
        MS a = s_ms[0][0], b = s_ms[1][0];
        for (int w = 1; w < kWarps; ++w) { a = ms_merge(a, s_ms[0][w]); b = ms_merge(b, s_ms[1][w]); }
        pp.mt = a.m; pp.st = a.s; pp.mq = b.m; pp.sq = b.s;
      } else {
        VI a = s_vi[0];
        for (int w = 1; w < kWarps; ++w)
          if (vi_better(s_vi[w], a)) a = s_vi[w];
        pp.bv = a.v; pp.bi = a.i;
      }
    }
    cluster.sync();                                          // A: this position's partials

    // ---- every CTA takes the same decision from the same partials (rank order, fixed
    // shuffle tree): no second barrier and no broadcast are needed
    if (warp == 0) {
      EEPart p{};
      if (lane < G) p = *cluster.map_shared_rank(&part[k & 1], (unsigned)lane);
      int stop = 0, a = k;
      if constexpr (kRej) {
        float Mt = lane < G ? p.mt : -INFINITY, Mq = lane < G ? p.mq : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          Mt = fmaxf(Mt, __shfl_xor_sync(0xffffffffu, Mt, o));
          Mq = fmaxf(Mq, __shfl_xor_sync(0xffffffffu, Mq, o));
        }
        double st = (lane < G && p.mt != -INFINITY) ? (double)p.st * exp2((double)p.mt - (double)Mt) : 0.0;
        double sq = (lane < G && has_q && p.mq != -INFINITY) ? (double)p.sq * exp2((double)p.mq - (double)Mq) : 0.0;
        st = warp_sum_d(st);
        sq = warp_sum_d(sq);
        d = __shfl_sync(0xffffffffu, d, 0);
        xt_d = __shfl_sync(0xffffffffu, xt_d, 0);
        xq_d = __shfl_sync(0xffffffffu, xq_d, 0);
        bool accept = false;
        if (k < Ki && d >= 0 && d < L.V) {
          const double pp = (Mt != -INFINITY && xt_d != -INFINITY)
                                ? exp2((double)xt_d * (double)kLog2e - (double)Mt) / st : 0.0;
          const double qq = (Mq != -INFINITY && xq_d != -INFINITY)
                                ? exp2((double)xq_d * (double)kLog2e - (double)Mq) / sq : 0.0;
          const double u = (double)L.uniforms[(long long)i * (K + 1) + k];
          accept = qq > 0.0 ? (u * qq < pp) : (pp > 0.0);
        }
        if (!accept) {
          stop = 1;
          if (lane == 0) {
            s_dec[0] = Mt;
            s_dec[1] = st > 0.0 ? (float)(1.0 / st) : 0.f;
            s_dec[2] = Mq;
            s_dec[3] = sq > 0.0 ? (float)(1.0 / sq) : 0.f;
            s_St = st;
          }
        }
      } else {
        VI b = lane < G ? VI{p.bv, p.bi} : VI{-INFINITY, kNoIndex};
        b = warp_argmax(b);                 // largest value, lowest index among equals
        const int gk = b.i == kNoIndex ? 0 : b.i;
        d = __shfl_sync(0xffffffffu, d, 0);
        const bool match = k < Ki && d >= 0 && d < L.V && d == gk;
        if (!match) {
          stop = 1;
          if (g == 0 && lane == 0) { L.bonus[i] = gk; L.out_tokens[(long long)i * (K + 1) + k] = gk; }
          if (lane == 0) s_tok = gk;
        }
      }
      if (stop && g == 0) {
        // outputs the two rules share: accepted drafts, the -1 tail, the count, range errors
        int bad = 0;
        if (lane < Ki) {
          const int dj = L.draft_tokens[(long long)i * K + lane];
          bad = dj < 0 || dj >= L.V;
          if (lane < a) L.out_tokens[(long long)i * (K + 1) + lane] = dj;
        }
        if (lane <= K && lane > a) L.out_tokens[(long long)i * (K + 1) + lane] = -1;
        if (__any_sync(0xffffffffu, bad) && lane == 0) set_err(L.err, PSPEC_DEVERR_TOKEN_RANGE);
        if (lane == 0) L.accepted_len[i] = a;
      }
      if (lane == 0) s_stop = stop;
    }
    __syncthreads();
    if (s_stop) break;
  }

  int meta_g = 0;                                            // the CTA that knows the token
  if constexpr (kRej) {
    // ---- the draw at the stop position a = k: r = max(0, p_a - q_a), or p_K after K passes
    const int a = k;
    DrawRow D;
    D.trow = static_cast<const elem*>(L.target) + ((long long)i * (K + 1) + a) * L.ld;
    D.resid = a < Ki;
    D.qrow = D.resid ? static_cast<const elem*>(L.draft) + ((long long)i * K + a) * L.ld : D.trow;
    D.mt = s_dec[0]; D.inv_st = s_dec[1]; D.mq = s_dec[2]; D.inv_sq = s_dec[3];
    const int ntiles = (n + 255) / 256;
    const double u = (double)L.uniforms[(long long)i * (K + 1) + Ki];

    // Sums of r over this CTA's tiles (all warps; tile t goes to warp t mod 8).  Measured on
    // B200 at B=1024: walking the slice last tile first (the part streamed most recently)
    // and two or four tiles in flight per warp were both slower or no faster, so the
    // defaults are first tile first, one tile per warp and iteration.
#ifndef PSPEC_EE_DRAW_REVERSE
#define PSPEC_EE_DRAW_REVERSE 0
#endif
    // PSPEC_EE_DRAW_U tiles per warp and iteration, all their loads issued first.
    auto tile_pass = [&]() {
      constexpr int U = PSPEC_EE_DRAW_U;
      for (int t0 = warp; t0 < ntiles; t0 += kWarps * U) {
        SliceRaw<Tag> R[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int tu = t0 + u * kWarps;
          const int t = PSPEC_EE_DRAW_REVERSE ? ntiles - 1 - tu : tu;
          R[u].live = false;
          if (tu < ntiles) slice_load<Tag>(D, lo, n, t * 256 + lane * 8, R[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int tu = t0 + u * kWarps;
          if (tu >= ntiles) break;                   // the same on every lane
          const int t = PSPEC_EE_DRAW_REVERSE ? ntiles - 1 - tu : tu;
          float xt[8], xq[8], r[8];
          slice_values<Tag>(D, R[u], xt, xq);
          draw_r8(D, xt, xq, r);
          float sum = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) sum += r[j];
          const double ts = warp_sum_d((double)sum);
          if (lane == 0) tsum[t] = ts;
        }
      }
    };
    bool own_pass_done = false;
    if (D.resid) {
      tile_pass();
      __syncthreads();
      if (tid == 0) {
        double tt = 0.0;
        for (int t = 0; t < ntiles; ++t) tt += tsum[t];
        tot_slice = tt;
      }
      cluster.sync();                                        // C: slice totals in place
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
      // empty): its slice totals s_g 2^(m_g - M) / S come from the statistics already
      // merged, so only the CTA that holds u*Z has to go over its slice again.
      if (tid < G) {
        const EEPart ph = *cluster.map_shared_rank(&part[a & 1], (unsigned)tid);
        const double Mt = (double)D.mt;
        s_tot[tid] = (ph.mt == -INFINITY || s_St <= 0.0) ? 0.0
                                                         : (double)ph.st * exp2((double)ph.mt - Mt) / s_St;
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
      if (tid == 0) {
        int tile = -1, last_tile = -1;
        double b2 = base, tb = base;
        for (int t = 0; t < ntiles; ++t) {
          if (tsum[t] > 0.0) last_tile = t;
          if (tile < 0 && crossing && tsum[t] > 0.0 && b2 + tsum[t] > thr) { tile = t; tb = b2; }
          b2 += tsum[t];
        }
        if (tile < 0) { tile = last_tile; tb = -INFINITY; } // no crossing: its last positive r
        s_tile = tile;
        s_base = tb;
      }
      __syncthreads();
      if (warp == 0) {
        int token = 0;
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
          token = cand != 0x7fffffff ? cand : (lastp >= 0 ? lastp : 0);
        }
        if (lane == 0) {
          L.out_tokens[(long long)i * (K + 1) + a] = token;
          L.bonus[i] = token;
          if (L.residual_mass) L.residual_mass[i] = (float)Z;
          s_tok = token;
        }
      }
    } else if (owner < 0 && g == 0 && tid == 0) {            // no mass anywhere: token 0
      L.out_tokens[(long long)i * (K + 1) + a] = 0;
      L.bonus[i] = 0;
      if (L.residual_mass) L.residual_mass[i] = 0.f;
      s_tok = 0;
    }
  }
  if constexpr (kRing) {
    // after a wait gave up, copies this warp requested may still be in flight: let them
    // land (each stage has at most one outstanding request; full poll budget) before the
    // CTA's shared memory is released
    if (!ring_ok)
      for (uint32_t u = issued > (uint32_t)kRingStages ? issued - kRingStages : 0; u < issued; ++u)
        mbar_wait(&bar[u % kRingStages], (u / kRingStages) & 1u);
  }
  cluster.sync();                                            // D: no remote reads after exit
  if constexpr (kFuse) {                                     // the whole step in this launch
    __syncthreads();
    ee_build_span(L.b, L.row_vecs, i, k, Ki, g == meta_g ? s_tok : 0, g == meta_g, g, G);
  }
  // second launch of a split batch: its completion implies the first grid's, so work queued
  // after it on the stream sees every sequence's outputs
  if (L.pdl == 2 && blockIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Shared-memory attributes of a kRing variant, set once per device.
template <typename Kern>
cudaError_t ring_attributes(Kern kern, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_relaxed) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

// Launches the variant, or with max_clusters set only asks how many of its clusters can be
// resident at once (cudaOccupancyMaxActiveClusters) and launches nothing.
template <typename Tag, int G, bool kRej, bool kFuse, bool kRing>
cudaError_t launch_ee(const EarlyExitLaunch& L, cudaStream_t stream, int* max_clusters) {
  auto kern = ee_kernel<Tag, G, kRej, kFuse, kRing>;
  cudaError_t e = cudaSuccess;
  if (G > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  const int dyn = kRing ? ring_smem_bytes(kRej) : 0;
  if constexpr (kRing) {
    static std::atomic<unsigned long long> done{0};
    e = ring_attributes(kern, dyn, done);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)(L.nseq > 0 ? L.nseq : 1) * G), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)dyn;
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

template <int G, bool kRing>
cudaError_t launch_ee_gr(const EarlyExitLaunch& L, cudaStream_t s, int* m) {
  const bool bf = L.dtype == PSPEC_BF16;
  if (L.fuse_build) {
    if (L.rejection)
      return bf ? launch_ee<BF16Tag, G, true, true, kRing>(L, s, m) : launch_ee<F32Tag, G, true, true, kRing>(L, s, m);
    return bf ? launch_ee<BF16Tag, G, false, true, kRing>(L, s, m) : launch_ee<F32Tag, G, false, true, kRing>(L, s, m);
  }
  if (L.rejection)
    return bf ? launch_ee<BF16Tag, G, true, false, kRing>(L, s, m) : launch_ee<F32Tag, G, true, false, kRing>(L, s, m);
  return bf ? launch_ee<BF16Tag, G, false, false, kRing>(L, s, m) : launch_ee<F32Tag, G, false, false, kRing>(L, s, m);
}

template <int G>
cudaError_t launch_ee_g(const EarlyExitLaunch& L, cudaStream_t s, int* m) {
  return L.ring ? launch_ee_gr<G, true>(L, s, m) : launch_ee_gr<G, false>(L, s, m);
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
  // cached per device and variant: 16 devices x 5 cluster sizes x dtype x rule x fusion x ring
  static std::atomic<int> cache[16 * 5 * 16];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int gi = L.G == 2 ? 0 : L.G == 4 ? 1 : L.G == 8 ? 2 : L.G == 12 ? 3 : 4;
  const int idx = (((((dev & 15) * 5 + gi) * 2 + (L.dtype == PSPEC_BF16)) * 2 + (L.rejection != 0)) * 2 +
                   (L.fuse_build != 0)) * 2 + (L.ring != 0);
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
