// verify_queue.cu -- position-major verification driven by an on-device work queue (one
// persistent launch per verify call, either rule).
//
// The accept rule is sequential ("Capstone 14: speculative decoding inference server",
// section "Architecture": accept the prefix, resample the rejected suffix; greedy: "any
// accepted prefix replaces the greedy path", section "Concept"): the rows of position k+1
// of a sequence matter only when its draft k was accepted.  The work here is the item
// (sequence i, position k).  An item is cut into units, one per segment of each of its
// rows (target row k, and draft row k under the rejection rule), and every CTA of a
// persistent grid pulls units from one queue:
//   - the queue starts with position 0 of every sequence, in sequence order;
//   - the CTA that completes the last unit of (i, k) (atomic ticket, nobody waits) merges
//     the segment partials and applies the rule; on acceptance it appends (i, k+1);
//   - greedy: on a mismatch (or after K matches) that CTA writes the outputs;
//   - rejection: on rejection at k (or after K acceptances) the draw over row k is
//     appended as C draw units to a second queue; the CTA finishing the last draw unit of
//     a sequence writes its outputs.  A CTA takes a draw unit when no stream unit is
//     ready for it (PSPEC_QUEUE_DRAW_FIRST=1 reverses the priority: measured slower on
//     B200, since the draws miss L2 either way and interrupt the streaming).
// The 2S units of an item run side by side, so an item takes about one segment's time,
// and the end of the launch is not held up by one long per-sequence chain.  Claims are
// atomicAdd tickets on the queue heads (a CAS loop serialised the claimers); a CTA holds
// at most one stream and one draw claim, taken ahead of use.  Waits (for a queue slot
// that is being published, or for work while other CTAs finish theirs) only wait on CTAs
// that are already running a unit, are bounded, and set PSPEC_DEVERR_TIMEOUT when the
// bound runs out.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "verify_common.cuh"
#include "verify_draw.cuh"

namespace pspec {

namespace {

enum : int { kQHeadS = 0, kQTailS = 1, kQHeadD = 2, kQTailD = 3, kQDone = 4, kQExit = 5 };
constexpr int kItemShift = 5;                            // item = i << 5 | k (K <= 31)

#ifndef PSPEC_QUEUE_MIN_BLOCKS
#define PSPEC_QUEUE_MIN_BLOCKS 5
#endif

#ifndef PSPEC_QUEUE_INLINE_DRAW
#define PSPEC_QUEUE_INLINE_DRAW 0
#endif
#ifndef PSPEC_QUEUE_DRAW_U
#define PSPEC_QUEUE_DRAW_U 4
#endif
#ifndef PSPEC_QUEUE_DRAW_FIRST
#define PSPEC_QUEUE_DRAW_FIRST 0
#endif

enum : int { kWorkExit = 0, kWorkDraw = 1, kWorkStream = 2 };

struct Work {
  int kind;
  int item;        // stream: i << 5 | k; draw: i
  int slot;        // queue slot the item came from (-1: an initial item)
  long long unit;  // unit within the item
};

__device__ __forceinline__ unsigned long long ld_volatile(const unsigned long long* p) {
  return *reinterpret_cast<const volatile unsigned long long*>(p);
}
__device__ __forceinline__ int ld_volatile(const int* p) {
  return *reinterpret_cast<const volatile int*>(p);
}

// Wait (bounded: `limit` polls) until a reserved queue slot is published; 0 on timeout.
__device__ __forceinline__ int wait_published(const int* slot, unsigned long long limit) {
  int v = ld_volatile(slot);
  for (unsigned long long w = 0; v == 0 && w < limit; ++w) {
    __nanosleep(32);
    v = ld_volatile(slot);
  }
  return v;
}

// Thread 0: the next unit for this CTA.  A CTA holds at most one claimed draw unit and one
// claimed stream unit (claims are plain atomicAdd tickets on the queue heads, taken ahead:
// a claim may point at a slot that is published later).  The stream claim is served once
// its item exists; otherwise the draw claim once its slot is published (or the other way
// round with PSPEC_QUEUE_DRAW_FIRST).
template <bool kRej>
__device__ Work pick_work(const QueueLaunch& L, long long& held, long long& held_d,
                          long long units_per_item, long long init_units) {
  unsigned long long* ctr = L.ctr;
  for (unsigned long long spin = 0;; ++spin) {
    if constexpr (kRej) {
      if (PSPEC_QUEUE_DRAW_FIRST) {
        if (held_d < 0) held_d = (long long)atomicAdd(ctr + kQHeadD, 1ull);
        const long long slot = held_d / L.C;
        if ((unsigned long long)slot < ld_volatile(ctr + kQTailD)) {
          const int v = wait_published(zcol(L.draws, slot), L.spin_limit);
          if (v == 0) {
            set_err(L.err, PSPEC_DEVERR_TIMEOUT);
            return Work{kWorkExit, 0, 0, 0};
          }
          __threadfence();
          const Work w{kWorkDraw, v - 1, (int)slot, held_d % L.C};
          held_d = -1;
          return w;
        }
      }
    }
    if (held < 0) held = (long long)atomicAdd(ctr + kQHeadS, 1ull);
    if (held < init_units) {
      const Work w{kWorkStream, (int)(held / units_per_item) << kItemShift, -1,
                   held % units_per_item};
      held = -1;
      return w;
    }
    const long long slot = (held - init_units) / units_per_item;
    if ((unsigned long long)slot < ld_volatile(ctr + kQTailS)) {
      const int v = wait_published(zitem(L.items, slot), L.spin_limit);
      if (v == 0) {
        set_err(L.err, PSPEC_DEVERR_TIMEOUT);
        return Work{kWorkExit, 0, 0, 0};
      }
      __threadfence();
      const Work w{kWorkStream, v - 1, (int)slot, (held - init_units) % units_per_item};
      held = -1;
      return w;
    }
    if constexpr (kRej) {
      if (!PSPEC_QUEUE_DRAW_FIRST) {                 // no stream unit ready: a draw unit
        if (held_d < 0) held_d = (long long)atomicAdd(ctr + kQHeadD, 1ull);
        const long long dslot = held_d / L.C;
        if ((unsigned long long)dslot < ld_volatile(ctr + kQTailD)) {
          const int v = wait_published(zcol(L.draws, dslot), L.spin_limit);
          if (v == 0) {
            set_err(L.err, PSPEC_DEVERR_TIMEOUT);
            return Work{kWorkExit, 0, 0, 0};
          }
          __threadfence();
          const Work w{kWorkDraw, v - 1, (int)dslot, held_d % L.C};
          held_d = -1;
          return w;
        }
      }
    }
    if (ld_volatile(ctr + kQDone) >= (unsigned long long)L.B) return Work{kWorkExit, 0, 0, 0};
    if (spin >= L.spin_limit) {
      set_err(L.err, PSPEC_DEVERR_TIMEOUT);
      return Work{kWorkExit, 0, 0, 0};
    }
    __nanosleep(64);
  }
}

struct QueueShared {
  Work work;
  int last;
  MS ms[kWarps];
  VI vi[kWarps];
  double M[2], Ssum[2];
  float dec_x[2], dec_u;
  int dec_d;
  int draw_now;
  SeqInfo si;
  DrawShared draw;
};

// Thread 0: append (i, k+1) to the stream queue.
__device__ __forceinline__ void append_item(const QueueLaunch& L, int i, int k) {
  const unsigned long long slot = atomicAdd(L.ctr + kQTailS, 1ull);
  atomicExch(zitem(L.items, (long long)slot), ((i << kItemShift) | k) + 1);
}

// Warp 0, once a sequence stops at a = k: accepted drafts, the -1 tail, the accepted count
// and the range check of the sequence's Ki draft tokens (as on the other paths).
__device__ __forceinline__ void write_prefix(const QueueLaunch& L, int i, int a, int Ki) {
  const int lane = threadIdx.x & 31;
  const int K = L.K;
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

// The end of a draw (all threads): the token from the tile sums ts of row a, then the
// sequence's outputs; `slot` >= 0 releases the draw slot the units came from.
template <typename Tag, typename Bar>
__device__ void finish_draw(const QueueLaunch& L, int i, int a, int Ki, DrawRow& D, double* ts,
                            QueueShared& sh, int slot) {
  const int K = L.K;
  double Z;
  const int token = draw_finish<Tag, Bar>(D, L.V, L.tiles, (double)L.uniforms[(long long)i * (K + 1) + Ki],
                                     ts, sh.draw, &Z);
  if ((threadIdx.x >> 5) == 0) {
    write_prefix(L, i, a, Ki);
    if ((threadIdx.x & 31) == 0) {
      L.out_tokens[(long long)i * (K + 1) + a] = token;
      L.bonus[i] = token;
      if (L.residual_mass) L.residual_mass[i] = (float)Z;
      if (slot >= 0) {
        atomicExch(zcol(L.cnt2, i), 0);
        atomicExch(zcol(L.draws, slot), 0);
      }
      __threadfence();
      atomicAdd(L.ctr + kQDone, 1ull);
    }
  }
}

// The whole draw of sequence i by this CTA (the one that just decided it), statistics in sh.si.
template <typename Tag, typename Bar>
__device__ __noinline__ void draw_whole(const QueueLaunch& L, int i, QueueShared& sh) {
  using elem = typename Tag::elem;
  const SeqInfo si = sh.si;
  DrawRow D = make_draw_row(L.target, L.draft, L.ld, L.K, si.kn, (int)sizeof(elem), i, si.a, si.mt,
                            si.st, si.mq, si.sq);
  double* ts = L.tile_sums + (long long)i * L.tiles;
  warp_tile_sums_wide<Tag, PSPEC_QUEUE_DRAW_U>(D, L.V, threadIdx.x >> 5, L.tiles, kWarps, ts);
  Bar::sync();
  finish_draw<Tag, Bar>(L, i, si.a, si.kn, D, ts, sh, -1);
}

// One draw unit of sequence i (rejection rule): tile sums over its chunk of row a_i; the CTA
// finishing the last unit draws the token and writes the sequence's outputs.
template <typename Tag, typename Bar>
__device__ __noinline__ void draw_unit(const QueueLaunch& L, const Work& w, QueueShared& sh) {
  using elem = typename Tag::elem;
  const int K = L.K;
  const int i = w.item;
  const int c = (int)w.unit;
  const int warp = threadIdx.x >> 5;
  const SeqInfo si = ld_cg(reinterpret_cast<const SeqInfo*>(L.seq) + i);
  DrawRow D = make_draw_row(L.target, L.draft, L.ld, K, si.kn, (int)sizeof(elem), i, si.a, si.mt,
                            si.st, si.mq, si.sq);
  double* ts = L.tile_sums + (long long)i * L.tiles;
  const long long t_lo = (long long)c * L.tiles_per_unit;
  const long long t_hi = min((long long)L.tiles, t_lo + L.tiles_per_unit);
  warp_tile_sums<Tag>(D, L.V, t_lo + warp, t_hi, kWarps, ts);
  Bar::sync();
  if (threadIdx.x == 0) {
    __threadfence();
    const int t = atomicAdd(zcol(L.cnt2, i), 1);
    sh.last = (t == L.C - 1);
  }
  Bar::sync();
  if (!sh.last) return;
  __threadfence();
  finish_draw<Tag, Bar>(L, i, si.a, si.kn, D, ts, sh, w.slot);
}

// One segment of one row of item (i, k); the CTA completing the item applies the rule.
template <typename Tag, bool kRej, typename Bar>
__device__ void stream_unit(const QueueLaunch& L, const Work& w, QueueShared& sh) {
  using elem = typename Tag::elem;
  const int K = L.K;
  const int i = w.item >> kItemShift;
  const int k = w.item & ((1 << kItemShift) - 1);
  const int r = (int)(w.unit / L.S);
  const int s = (int)(w.unit % L.S);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int R = kRej ? 2 : 1;
  int ebk = 0;
  const int Ki = draft_count(L.k_len, i, K, &ebk);    // the sequence's own drafts
  const bool live = !(kRej && r == 1 && k == Ki);     // no draft row at position K_i
  const long long lo = (long long)s * L.seg;
  const long long hi = min((long long)L.V, lo + L.seg);

  MS ms{-INFINITY, 0.f};
  VI best{-INFINITY, kNoIndex};
  if (live) {
    const elem* row = r == 0
        ? static_cast<const elem*>(L.target) + ((long long)i * (K + 1) + k) * L.ld
        : static_cast<const elem*>(L.draft) + ((long long)i * K + k) * L.ld;
    if constexpr (kRej) {
      MSAcc acc = msacc_init();
      sweep_segment_batched<Tag, 4>(
          row, lo, hi, [&](const uint4 (&v)[4]) { consume_ms_batch<Tag, 4>(v, acc); },
          [&](const uint4& v, long long) { consume_ms<Tag>(v, acc); },
          [&](float x, long long) { consume_one(x, acc); });
      ms = msacc_final(acc);
    } else {
      sweep_segment<Tag, 4>(
          row, lo, hi, [&](const uint4& v, long long idx0) { consume_argmax<Tag>(v, idx0, best); },
          [&](float x, long long t) {
            if (x > best.v) { best.v = x; best.i = (int)t; }
          });
    }
  }
  if constexpr (kRej) ms = warp_merge_ms(ms);
  else best = warp_argmax(best);
  if (lane == 0) {
    if constexpr (kRej) sh.ms[warp] = ms;
    else sh.vi[warp] = best;
  }
  Bar::sync();
  if (warp == 0) {
    if constexpr (kRej) {
      ms = lane < kWarps ? sh.ms[lane] : MS{-INFINITY, 0.f};
      ms = warp_merge_ms(ms);
    } else {
      best = lane < kWarps ? sh.vi[lane] : VI{-INFINITY, kNoIndex};
      best = warp_argmax(best);
    }
    if (lane == 0) {
      RejPart* part = reinterpret_cast<RejPart*>(L.part) + ((long long)i * R + r) * L.S + s;
      if constexpr (kRej) *part = RejPart{ms.m, ms.s};
      else *reinterpret_cast<VI*>(part) = best;
      __threadfence();
      const int t = atomicAdd(zcol(L.cnt, i), 1);
      sh.last = (t == R * L.S - 1);
    }
  }
  Bar::sync();
  if (!sh.last) return;
  __threadfence();

  // ---- this CTA completed item (i, k)
  const RejPart* part = reinterpret_cast<const RejPart*>(L.part) + (long long)i * R * L.S;
  if constexpr (kRej) {
    // warp r merges row r (lane t holds segments t, t+32, ...); warp 2 fetches the draft
    // token, the two logits at it and the uniform meanwhile
    if (warp < R && (warp == 0 || k < Ki)) {
      const RejPart* pr = part + (long long)warp * L.S;
      RejPart mine = lane < L.S ? ld_cg(pr + lane) : RejPart{-INFINITY, 0.f};
      float m = mine.m;
      for (int t = lane + 32; t < L.S; t += 32) m = fmaxf(m, ld_cg(&pr[t].m));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      double acc = 0.0;
      if (m != -INFINITY) {
        if (mine.m != -INFINITY) acc = (double)mine.s * exp2((double)mine.m - (double)m);
        for (int t = lane + 32; t < L.S; t += 32) {
          const RejPart q = ld_cg(pr + t);
          if (q.m != -INFINITY) acc += (double)q.s * exp2((double)q.m - (double)m);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        sh.M[warp] = m;
        sh.Ssum[warp] = acc;
      }
    } else if (warp == 2 && lane == 0 && k < Ki) {
      const int d = L.draft_tokens[(long long)i * K + k];
      float xt = -INFINITY, xq = -INFINITY;
      if (d >= 0 && d < L.V) {
        xt = load_scalar(static_cast<const elem*>(L.target) + ((long long)i * (K + 1) + k) * L.ld, d);
        xq = load_scalar(static_cast<const elem*>(L.draft) + ((long long)i * K + k) * L.ld, d);
      }
      sh.dec_d = d;
      sh.dec_x[0] = xt;
      sh.dec_x[1] = xq;
      sh.dec_u = L.uniforms[(long long)i * (K + 1) + k];
    }
    Bar::sync();
    if (tid == 0) {
      if (k == 0) set_err(L.err, ebk);
      const double Mt = sh.M[0], St = sh.Ssum[0];
      bool accept = false;
      double Mq = 0.0, Sq = 1.0;
      if (k < Ki) {
        Mq = sh.M[1];
        Sq = sh.Ssum[1];
        const int d = sh.dec_d;
        if (d >= 0 && d < L.V) {
          const float xt = sh.dec_x[0], xq = sh.dec_x[1];
          double p = 0.0, q = 0.0;
          if (Mt != -INFINITY && xt != -INFINITY) p = exp2((double)xt * (double)kLog2e - Mt) / St;
          if (Mq != -INFINITY && xq != -INFINITY) q = exp2((double)xq * (double)kLog2e - Mq) / Sq;
          const double u = (double)sh.dec_u;
          accept = q > 0.0 ? (u * q < p) : (p > 0.0);
        }
        if (accept) L.out_tokens[(long long)i * (K + 1) + k] = d;
      }
      atomicExch(zcol(L.cnt, i), 0);                     // ticket back to zero for the next item
      if (w.slot >= 0) atomicExch(zitem(L.items, w.slot), 0);
      if (accept) {
        __threadfence();
        append_item(L, i, k + 1);
      } else {
        SeqInfo si;
        si.mt = Mt;
        si.st = St;
        si.mq = k < Ki ? Mq : 0.0;
        si.sq = k < Ki ? Sq : 1.0;
        si.a = k;
        si.kn = Ki;
        si.pad[0] = si.pad[1] = 0;
#if PSPEC_QUEUE_INLINE_DRAW
        sh.si = si;
#else
        reinterpret_cast<SeqInfo*>(L.seq)[i] = si;
        __threadfence();
        const unsigned long long slot = atomicAdd(L.ctr + kQTailD, 1ull);
        atomicExch(zcol(L.draws, (long long)slot), i + 1);
#endif
      }
      sh.draw_now = !accept;
    }
#if PSPEC_QUEUE_INLINE_DRAW
    Bar::sync();
    if (sh.draw_now) draw_whole<Tag, Bar>(L, i, sh);       // this CTA draws while the rows are fresh
#endif
  } else {
    if (warp == 0) {
      VI b{-INFINITY, kNoIndex};
      for (int t = lane; t < L.S; t += 32) {
        const VI q = ld_cg(reinterpret_cast<const VI*>(part) + t);
        if (vi_better(q, b)) b = q;
      }
      b = warp_argmax(b);                            // largest value, lowest index among equals
      const int gk = b.i == kNoIndex ? 0 : b.i;      // a row of -inf / NaN only: token 0
      int d = -1;
      if (lane == 0 && k < Ki) d = L.draft_tokens[(long long)i * K + k];
      d = __shfl_sync(0xffffffffu, d, 0);
      const bool match = k < Ki && d >= 0 && d < L.V && d == gk;
      if (lane == 0) {
        if (k == 0) set_err(L.err, ebk);
        atomicExch(zcol(L.cnt, i), 0);
        if (w.slot >= 0) atomicExch(zitem(L.items, w.slot), 0);
      }
      if (match) {
        if (lane == 0) {
          L.out_tokens[(long long)i * (K + 1) + k] = d;
          __threadfence();
          append_item(L, i, k + 1);
        }
      } else {
        write_prefix(L, i, k, Ki);
        if (lane == 0) {
          L.out_tokens[(long long)i * (K + 1) + k] = gk;
          L.bonus[i] = gk;
          __threadfence();
          atomicAdd(L.ctr + kQDone, 1ull);
        }
      }
    }
  }
}

template <typename Tag, bool kRej>
__global__ void __launch_bounds__(kThreads, PSPEC_QUEUE_MIN_BLOCKS) queue_kernel(const QueueLaunch L) {
  __shared__ QueueShared sh;
  constexpr int R = kRej ? 2 : 1;
  const long long units_per_item = (long long)R * L.S;
  const long long init_units = (long long)L.B * units_per_item;
  long long held = -1;                               // thread 0: stream unit claimed ahead
  long long held_d = -1;                             // thread 0: draw unit claimed ahead
  for (;;) {
    if (threadIdx.x == 0) sh.work = pick_work<kRej>(L, held, held_d, units_per_item, init_units);
    __syncthreads();
    const Work w = sh.work;
    __syncthreads();                                 // everyone has its copy of sh.work
    if (w.kind == kWorkExit) break;
    if (threadIdx.x == 0 && held < 0 && (!kRej || w.kind == kWorkStream))
      held = (long long)atomicAdd(L.ctr + kQHeadS, 1ull);   // claim ahead: overlaps the unit
    if constexpr (kRej) {
      if (w.kind == kWorkDraw) draw_unit<Tag, CtaBarrier>(L, w, sh);
      else stream_unit<Tag, kRej, CtaBarrier>(L, w, sh);
    } else {
      stream_unit<Tag, kRej, CtaBarrier>(L, w, sh);
    }
    __syncthreads();                                 // sh reused by the next unit
  }
  // the last CTA out puts the counters back to zero (and, after a timeout, the queue state)
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned long long e = atomicAdd(L.ctr + kQExit, 1ull);
    sh.last = (e == (unsigned long long)gridDim.x - 1);
  }
  __syncthreads();
  if (!sh.last) return;
  __threadfence();
  if (ld_volatile(L.err) & PSPEC_DEVERR_TIMEOUT) {
    for (long long t = threadIdx.x; t < (long long)L.B * L.K; t += kThreads) *zitem(L.items, t) = 0;
    for (int t = threadIdx.x; t < L.B; t += kThreads) {
      *zcol(L.draws, t) = 0;
      *zcol(L.cnt, t) = 0;
      *zcol(L.cnt2, t) = 0;
    }
  }
  if (threadIdx.x < 8) L.ctr[threadIdx.x] = 0;
}

template <typename Tag, bool kRej>
cudaError_t launch_q(const QueueLaunch& L, cudaStream_t stream) {
  auto kern = queue_kernel<Tag, kRej>;
  const int threads = kThreads;
  static int per_sm[8] = {0};                        // per device
  static int sms[8] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 8 || per_sm[dev] == 0) {
    int nb = 0, n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, threads, 0);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (nb < 1) nb = 1;
    if (dev >= 0 && dev < 8) { per_sm[dev] = nb; sms[dev] = n; }
    else { per_sm[0] = nb; sms[0] = n; dev = 0; }
  }
  const long long units = (long long)L.B * (kRej ? 2 : 1) * L.S;
  long long grid = (long long)per_sm[dev] * sms[dev];
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, threads, 0, stream>>>(L);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_queue(const QueueLaunch& L, cudaStream_t stream) {
  if (L.dtype == PSPEC_BF16)
    return L.rejection ? launch_q<BF16Tag, true>(L, stream) : launch_q<BF16Tag, false>(L, stream);
  return L.rejection ? launch_q<F32Tag, true>(L, stream) : launch_q<F32Tag, false>(L, stream);
}

}  // namespace pspec
