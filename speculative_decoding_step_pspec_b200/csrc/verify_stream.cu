// verify_stream.cu -- early-exit verification fed by bulk copies (the large-batch path).
//
// The accept rule is sequential ("Capstone 14: speculative decoding inference server",
// section "Architecture": accept the prefix, resample for the rejected suffix), so a
// sequence needs its rows 0..a_i only; the draw then needs row pair a_i once more.  This
// kernel gives each sequence one CTA (or a cluster of two) that owns a whole SM, so that
// few sequences are in flight and the row pair of each sequence's current position is
// still in L2 when the draw re-reads it:
//
//   producer warp  one thread issues cp.async.bulk copies of 4 KB chunks of the position's
//                  target and draft rows (this CTA's slice) into a ring of kNS shared-memory
//                  stages, completion counted in bytes on each stage's mbarrier; after the
//                  first kSpec chunks of position k+1 it waits for the decision of position
//                  k (so at most kSpec chunks per CTA are read for a position that turns out
//                  not to be needed), then issues the draw's chunks and the end markers;
//   consumer warps stage g goes to warp g mod kCW; the warp copies the stage to registers,
//                  releases it at once, and folds it into its partial (max, sum exp) of the
//                  position -- or its argmax, or for a draw chunk the chunk's sum of
//                  r = max(0, p - q); after its last chunk of a position it publishes the
//                  partial and arrives on the position's barrier;
//   decider warp   merges the consumer partials in a fixed order, exchanges the CTA partial
//                  with the other CTA of the cluster over distributed shared memory
//                  (remote store + remote mbarrier arrive), takes the decision (u q < p, or
//                  draft == argmax), and at the stop position runs the draw: slice totals,
//                  the slice and chunk holding u_K * Z, a rescan of that chunk.
//
// Every wait is bounded (kSpinLimit polls, or the launch's own limit); a wait that runs out
// sets PSPEC_DEVERR_TIMEOUT, the kernel stops issuing copies, lets those in flight land and
// ends.  Outputs are those of the other verify paths (decisions and draws merge their
// partials in a fixed order, so they are deterministic).
#include <cooperative_groups.h>

#include <atomic>

#include "build_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "mbar.cuh"
#include "plan.h"
#include "verify_common.cuh"

namespace cg = cooperative_groups;

namespace pspec {

namespace {

#ifndef PSPEC_SS_WARPS
#define PSPEC_SS_WARPS 8
#endif
#ifndef PSPEC_SS_STAGES
#define PSPEC_SS_STAGES 24
#endif
#ifndef PSPEC_SS_SPEC
#define PSPEC_SS_SPEC 8
#endif
#ifndef PSPEC_SS_MINB
#define PSPEC_SS_MINB 1
#endif
constexpr int kCW = PSPEC_SS_WARPS;            // consumer warps
constexpr int kProducer = kCW;                 // warp index of the producer
// warp kCW + 1: the decider
constexpr int kSThreads = (kCW + 2) * 32;
constexpr int kCB = 4096;                      // bytes of one row per stage
constexpr int kCV = kCB / 16;                  // 16-byte vectors of one row per stage
constexpr int kLV = kCV / 32;                  // of them per lane
constexpr int kNS = PSPEC_SS_STAGES;           // ring stages
constexpr int kSpec = PSPEC_SS_SPEC;           // chunks of position k+1 issued before decision k
constexpr int kMaxChunks = 512;                // chunks per slice at most

enum : int { kStats = 0, kDraw = 1, kEnd = 2 };

struct Hdr {
  int kind, k, c, q;                           // kind, position, chunk, draft row present
};

struct Smem {
  uint4 ring[kNS][2][kCV];                     // stage s: target chunk, draft chunk
  Hdr hdr[kNS];
  uint64_t full[kNS], empty[kNS];
  uint64_t posdone[2], dec[2], xch[2], drawdone, xch2;
  float4 part[2][kCW];                         // consumer partials by position parity
  float4 xpart[2][2];                          // CTA partials of both ranks by parity
  double xtot[2];                              // draw slice totals of both ranks
  double csum[kMaxChunks];                     // draw: sum of r over each chunk of the slice
  int stop[2];                                 // decision of position k (by parity)
  int plan;                                    // draw: 0 none here, 1 residual, 2 target row
  int a;                                       // stop position
  float dmt, dinv_st, dmq, dinv_sq;            // draw row parameters
  int tok;                                     // the emitted token (fused build)
  int owner;                                   // rank whose slice holds u_K * Z (-1: none)
};

// r of the W elements of one 16-byte vector pair, computed on packed fp32 pairs exactly as
// the other draw paths do (p = 2^(x log2 e - mt) / St, q likewise, r = max(0, p - q), or
// r = p without the draft row).  Every pass over the same elements goes through here, so
// chunk sums and the rescan see bit-identical values.
template <typename Tag>
__device__ __forceinline__ void draw_vec(const DrawRow& D, const uint4& vt, const uint4& vq,
                                         float (&r)[Tag::kVec]) {
  constexpr int W = Tag::kVec;
  float xt[W], xq[W];
  unpack(vt, xt, Tag{});
  unpack(vq, xq, Tag{});
  if (D.mt == -INFINITY) {
#pragma unroll
    for (int j = 0; j < W; ++j) r[j] = 0.f;
    return;
  }
#pragma unroll
  for (int j = 0; j < W; j += 2) {
    float a0, a1;
    ffma2(a0, a1, xt[j], xt[j + 1], kLog2e, -D.mt);
    float p0, p1;
    fmul2(p0, p1, ex2(a0), ex2(a1), D.inv_st);
    if (D.resid && D.mq != -INFINITY) {
      float b0, b1, q0, q1;
      ffma2(b0, b1, xq[j], xq[j + 1], kLog2e, -D.mq);
      fmul2(q0, q1, ex2(b0), ex2(b1), D.inv_sq);
      r[j] = fmaxf(p0 - q0, 0.f);
      r[j + 1] = fmaxf(p1 - q1, 0.f);
    } else {
      r[j] = p0;
      r[j + 1] = p1;
    }
  }
}

// A lane's running (max, sum) of one row over a position, its sum kept in double: each
// chunk is reduced in fp32 against the chunk's own maximum and then folded in, so the fp32
// rounding covers one chunk's terms at a time.
struct MSD {
  float m;
  double s;
};

__device__ __forceinline__ void msd_add(MSD& d, const MS& c) {
  if (c.m == -INFINITY) return;
  if (d.m == -INFINITY) {
    d.m = c.m;
    d.s = (double)c.s;
  } else if (c.m > d.m) {
    d.s = d.s * (double)ex2(d.m - c.m) + (double)c.s;
    d.m = c.m;
  } else {
    d.s += (double)c.s * (double)ex2(c.m - d.m);
  }
}

__device__ __forceinline__ double warp_sum_dd(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The decider's rescan of chunk c of this CTA's slice of the draw rows (global memory,
// usually in L2): the smallest token whose running sum base + prefix exceeds thr (only a
// token with r > 0 can), else the last token with r > 0 in the chunk (-1 when none).
// Lane l takes the chunk's l-th run of kLV consecutive vectors, so prefixes run in
// token-id order.
template <typename Tag>
__device__ __forceinline__ void chunk_rescan(const DrawRow& D, const typename Tag::elem* trow,
                                             const typename Tag::elem* qrow, long long lo, int c,
                                             int nvec, double base, double thr, bool crossing,
                                             int* cand_out, int* last_out) {
  constexpr int W = Tag::kVec;
  constexpr int CE = kCB / (int)sizeof(typename Tag::elem);
  const int lane = threadIdx.x & 31;
  const uint4* tv = reinterpret_cast<const uint4*>(trow + (long long)c * CE);
  const uint4* qv = reinterpret_cast<const uint4*>(qrow + (long long)c * CE);
  float incl[kLV * W];                             // inclusive within each vector (fp32)
  double vbase[kLV];                               // the lane's sum before each vector
  unsigned long long pos = 0;                      // bit j: r > 0 at the lane's element j
  double acc = 0.0;
  int lastp = -1;
#pragma unroll
  for (int j = 0; j < kLV; ++j) {
    const int v = lane * kLV + j;
    float r[W];
    if (v < nvec) {
      draw_vec<Tag>(D, ld_stream(tv + v), D.resid ? ld_stream(qv + v) : make_uint4(0, 0, 0, 0), r);
    } else {
#pragma unroll
      for (int e = 0; e < W; ++e) r[e] = 0.f;
    }
    vbase[j] = acc;
    float vs = 0.f;
#pragma unroll
    for (int e = 0; e < W; ++e) {
      vs += r[e];
      incl[j * W + e] = vs;
      if (r[e] > 0.f) {
        pos |= 1ull << (j * W + e);
        lastp = (int)(lo + (long long)c * CE + (long long)v * W + e);
      }
    }
    acc += (double)vs;
  }
  double inc = acc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  const double ex = inc - acc;
  int cand = 0x7fffffff;
  if (crossing) {
#pragma unroll
    for (int j = 0; j < kLV * W; ++j)
      if (cand == 0x7fffffff && ((pos >> j) & 1ull) && base + ex + vbase[j / W] + (double)incl[j] > thr)
        cand = (int)(lo + (long long)c * CE + (long long)(lane * kLV) * W + j);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cand = min(cand, __shfl_xor_sync(0xffffffffu, cand, o));
    lastp = max(lastp, __shfl_xor_sync(0xffffffffu, lastp, o));
  }
  *cand_out = cand == 0x7fffffff ? -1 : cand;
  *last_out = lastp;
}

template <typename Tag, int G, bool kRej, bool kFuse>
__global__ void __launch_bounds__(kSThreads, PSPEC_SS_MINB) stream_kernel(const EarlyExitLaunch L) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  using elem = typename Tag::elem;
  constexpr int W = Tag::kVec;
  constexpr int CE = kCB / (int)sizeof(elem);          // elements of one row per chunk
  const int rank = G > 1 ? (int)cg::this_cluster().block_rank() : 0;
  const int i = (int)(blockIdx.x / G);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = L.K;
  const unsigned spin = L.spin_limit ? L.spin_limit : kSpinLimit;
  int ebk = 0;
  const int Ki = draft_count(L.k_len, i, K, &ebk);
  const long long lo = (long long)rank * L.vs;          // this CTA's slice [lo, lo + n)
  const int n = (int)max(0LL, min((long long)L.V, lo + L.vs) - lo);
  const long long nbytes = (long long)n * (long long)sizeof(elem);
  const int N = (int)((nbytes + kCB - 1) / kCB);         // chunks per position (>= kCW + kSpec)
  const elem* const tbase = static_cast<const elem*>(L.target) + (long long)i * (K + 1) * L.ld + lo;
  const elem* const qbase = kRej ? static_cast<const elem*>(L.draft) + (long long)i * K * L.ld + lo : tbase;

  if (tid == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int p = 0; p < 2; ++p) {
      mbar_init(&S.posdone[p], kCW);
      mbar_init(&S.dec[p], 1);
      mbar_init(&S.xch[p], G);
    }
    mbar_init(&S.drawdone, kCW);
    mbar_init(&S.xch2, G);
    S.plan = 0;
    S.a = 0;
    S.owner = -1;
    S.tok = 0;
    mbar_init_fence();
  }
  __syncthreads();
  if constexpr (G > 1) cg::this_cluster().sync();       // peers' barriers exist before any remote arrive

  int err = 0;
  if (warp < kCW) {
    // ------------------------------------------------------------------ consumer warps
    MSD dt{-INFINITY, 0.0}, dq{-INFINITY, 0.0};
    VI best{-INFINITY, kNoIndex};
    int cur_k = -1;
    for (unsigned g = warp;; g += kCW) {
      const int s = (int)(g % kNS);
      if (!mbar_wait(&S.full[s], (g / kNS) & 1u, spin)) { err |= PSPEC_DEVERR_TIMEOUT; break; }
      const Hdr h = S.hdr[s];
      if (h.kind == kEnd) break;
      const int nv = (int)(min((long long)kCB, nbytes - (long long)h.c * kCB) / 16);
      uint4 bt[kLV], bq[kLV];
#pragma unroll
      for (int j = 0; j < kLV; ++j) {
        const int v = lane + 32 * j;
        bt[j] = v < nv ? S.ring[s][0][v] : make_uint4(0, 0, 0, 0);
        bq[j] = (h.q && v < nv) ? S.ring[s][1][v] : make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[s]);          // the stage is free again
      const bool last = h.c + kCW >= N;                 // this warp's last chunk of the pass
      if (h.kind == kStats) {
        if (h.k != cur_k) {
          dt = MSD{-INFINITY, 0.0};
          dq = MSD{-INFINITY, 0.0};
          best = VI{-INFINITY, kNoIndex};
          cur_k = h.k;
        }
        if constexpr (kRej) {
          MSAcc at = msacc_init(), aq = msacc_init();
          if (nv == kCV) {
            consume_ms_batch<Tag, kLV>(bt, at);
            if (h.q) consume_ms_batch<Tag, kLV>(bq, aq);
          } else {
#pragma unroll
            for (int j = 0; j < kLV; ++j)
              if (lane + 32 * j < nv) {
                consume_ms<Tag>(bt[j], at);
                if (h.q) consume_ms<Tag>(bq[j], aq);
              }
          }
          msd_add(dt, msacc_final(at));
          if (h.q) msd_add(dq, msacc_final(aq));
        } else {
#pragma unroll
          for (int j = 0; j < kLV; ++j)
            if (lane + 32 * j < nv)
              consume_argmax<Tag>(bt[j], lo + (long long)h.c * CE + (long long)(lane + 32 * j) * W, best);
        }
        if (last) {
          if constexpr (kRej) {
            const MS mt = warp_merge_ms(MS{dt.m, (float)dt.s});
            const MS mq = warp_merge_ms(MS{dq.m, (float)dq.s});
            if (lane == 0) S.part[h.k & 1][warp] = make_float4(mt.m, mt.s, mq.m, mq.s);
          } else {
            const VI b = warp_argmax(best);
            if (lane == 0) S.part[h.k & 1][warp] = make_float4(b.v, __int_as_float(b.i), 0.f, 0.f);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.posdone[h.k & 1]);
        }
      } else {                                          // a draw chunk
        DrawRow D;
        D.trow = nullptr;
        D.qrow = nullptr;
        D.mt = S.dmt; D.inv_st = S.dinv_st; D.mq = S.dmq; D.inv_sq = S.dinv_sq;
        D.resid = h.q != 0;
        double sum = 0.0;                               // per vector in fp32, then double
#pragma unroll
        for (int j = 0; j < kLV; ++j) {
          if (lane + 32 * j < nv) {
            float r[W], vs = 0.f;
            draw_vec<Tag>(D, bt[j], bq[j], r);
#pragma unroll
            for (int e = 0; e < W; ++e) vs += r[e];
            sum += (double)vs;
          }
        }
        const double cs = warp_sum_dd(sum);
        if (lane == 0) S.csum[h.c] = cs;
        if (last) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.drawdone);
        }
      }
    }
  } else if (warp == kProducer) {
    // ------------------------------------------------------------------ producer warp
    if (lane == 0) {
      unsigned g = 0;
      bool ok = true;
      auto issue = [&](int kind, int k, int c, bool q, const elem* tr, const elem* qr) -> bool {
        const int s = (int)(g % kNS);
        // the stage's consumer released it (its reads happened before its arrive)
        if (g >= (unsigned)kNS && !mbar_wait(&S.empty[s], ((g / kNS) - 1u) & 1u, spin)) return false;
        S.hdr[s] = Hdr{kind, k, c, q ? 1 : 0};
        if (kind == kEnd) {
          mbar_arrive(&S.full[s]);
        } else {
          const unsigned bytes = (unsigned)min((long long)kCB, nbytes - (long long)c * kCB);
          mbar_arrive_expect(&S.full[s], q ? 2 * bytes : bytes);
          bulk_g2s(&S.ring[s][0][0], tr + (long long)c * CE, bytes, &S.full[s]);
          if (q) bulk_g2s(&S.ring[s][1][0], qr + (long long)c * CE, bytes, &S.full[s]);
        }
        ++g;
        return true;
      };
      for (int k = 0; ok; ++k) {
        const bool q = kRej && k < Ki;
        const elem* tr = tbase + (long long)k * L.ld;
        const elem* qr = q ? qbase + (long long)k * L.ld : tr;
        bool stop = false;
        for (int c = 0; c < N && ok; ++c) {
          if (k > 0 && c == kSpec) {
            if (!mbar_wait(&S.dec[(k - 1) & 1], ((unsigned)(k - 1) >> 1) & 1u, spin)) { ok = false; break; }
            if (S.stop[(k - 1) & 1]) { stop = true; break; }
          }
          ok = issue(kStats, k, c, q, tr, qr);
        }
        if (!ok || stop) break;
        if (k == Ki) {                                  // the last position: a stop
          if (!mbar_wait(&S.dec[k & 1], ((unsigned)k >> 1) & 1u, spin)) ok = false;
          break;
        }
      }
      if (ok && S.plan != 0) {                          // the draw's chunks
        const int a = S.a;
        const bool q = S.plan == 1;
        const elem* tr = tbase + (long long)a * L.ld;
        const elem* qr = q ? qbase + (long long)a * L.ld : tr;
        for (int c = 0; c < N && ok; ++c) ok = issue(kDraw, a, c, q, tr, qr);
      }
      for (int w = 0; w < kCW && ok; ++w) ok = issue(kEnd, 0, 0, false, tbase, tbase);
      if (!ok) {
        err |= PSPEC_DEVERR_TIMEOUT;
        // let every copy already requested land before the CTA's shared memory goes away
        // (with the full poll budget, whatever limit the call set for its other waits)
        const unsigned first = g > (unsigned)kNS ? g - kNS : 0;
        for (unsigned u = first; u < g; ++u) mbar_wait(&S.full[u % kNS], (u / kNS) & 1u, kSpinLimit);
      }
    }
  } else {
    // ------------------------------------------------------------------ decider warp
    const int dreg = lane < Ki ? __ldg(L.draft_tokens + (long long)i * K + lane) : -1;
    float Mt = -INFINITY, Mq = -INFINITY;
    double St = 0.0, Sq = 0.0;
    float4 xp[2] = {make_float4(-INFINITY, 0.f, -INFINITY, 0.f), make_float4(-INFINITY, 0.f, -INFINITY, 0.f)};
    int gk = 0, a = -1;
    bool ok = true;
    for (int k = 0;; ++k) {
      const bool has_q = kRej && k < Ki;
      const int d = k < Ki ? __shfl_sync(0xffffffffu, dreg, k & 31) : -1;
      float xt_d = 0.f, xq_d = 0.f;
      if (kRej && lane == 0 && d >= 0 && d < L.V) {
        xt_d = load_scalar(tbase + (long long)k * L.ld - lo, d);
        xq_d = load_scalar(qbase + (long long)k * L.ld - lo, d);
      }
      if (!mbar_wait(&S.posdone[k & 1], ((unsigned)k >> 1) & 1u, spin)) { ok = false; break; }
      // this CTA's partial: the consumer partials merged in one fixed order
      float4 p = lane < kCW ? S.part[k & 1][lane]
                            : (kRej ? make_float4(-INFINITY, 0.f, -INFINITY, 0.f)
                                    : make_float4(-INFINITY, __int_as_float(kNoIndex), 0.f, 0.f));
      float4 cp;
      if constexpr (kRej) {
        const MS t = warp_merge_ms(MS{p.x, p.y});
        const MS u = warp_merge_ms(MS{p.z, p.w});
        cp = make_float4(t.m, t.s, u.m, u.s);
      } else {
        const VI b = warp_argmax(VI{p.x, __float_as_int(p.y)});
        cp = make_float4(b.v, __int_as_float(b.i), 0.f, 0.f);
      }
      if constexpr (G > 1) {
        // both CTAs' partials, over distributed shared memory
        if (lane < G) {
          if (lane == rank) S.xpart[k & 1][rank] = cp;
          else st_remote_f4(&S.xpart[k & 1][rank], (unsigned)lane, cp);
        }
        __syncwarp();
        if (lane < G) {
          if (lane == rank) mbar_arrive(&S.xch[k & 1]);
          else mbar_arrive_remote(&S.xch[k & 1], (unsigned)lane);
        }
        if (!mbar_wait(&S.xch[k & 1], ((unsigned)k >> 1) & 1u, spin)) { ok = false; break; }
        xp[0] = S.xpart[k & 1][0];
        xp[1] = S.xpart[k & 1][1];
      } else {
        xp[0] = cp;
      }
      bool stop;
      if constexpr (kRej) {
        Mt = G > 1 ? fmaxf(xp[0].x, xp[1].x) : xp[0].x;
        Mq = G > 1 ? fmaxf(xp[0].z, xp[1].z) : xp[0].z;
        St = 0.0;
        Sq = 0.0;
        for (int r = 0; r < G; ++r) {
          if (xp[r].x != -INFINITY) St += (double)xp[r].y * exp2((double)xp[r].x - (double)Mt);
          if (has_q && xp[r].z != -INFINITY) Sq += (double)xp[r].w * exp2((double)xp[r].z - (double)Mq);
        }
        xt_d = __shfl_sync(0xffffffffu, xt_d, 0);
        xq_d = __shfl_sync(0xffffffffu, xq_d, 0);
        bool accept = false;
        if (k < Ki && d >= 0 && d < L.V) {
          const double pp = (Mt != -INFINITY && xt_d != -INFINITY)
                                ? exp2((double)xt_d * (double)kLog2e - (double)Mt) / St : 0.0;
          const double qq = (Mq != -INFINITY && xq_d != -INFINITY)
                                ? exp2((double)xq_d * (double)kLog2e - (double)Mq) / Sq : 0.0;
          const double u = (double)L.uniforms[(long long)i * (K + 1) + k];
          accept = qq > 0.0 ? (u * qq < pp) : (pp > 0.0);
        }
        stop = !accept;
      } else {
        VI b{xp[0].x, __float_as_int(xp[0].y)};
        if (G > 1) {
          const VI c{xp[1].x, __float_as_int(xp[1].y)};
          if (vi_better(c, b)) b = c;
        }
        gk = b.i == kNoIndex ? 0 : b.i;
        stop = !(k < Ki && d >= 0 && d < L.V && d == gk);
      }
      if (stop) {
        a = k;
        if (lane == 0) {
          S.a = k;
          if constexpr (kRej) {
            S.dmt = Mt;
            S.dinv_st = St > 0.0 ? (float)(1.0 / St) : 0.f;
            S.dmq = Mq;
            S.dinv_sq = Sq > 0.0 ? (float)(1.0 / Sq) : 0.f;
            if (k < Ki) {
              S.plan = 1;                              // residual: every CTA re-reads its slice
            } else {
              // the bonus draw from p_K: slice totals from the statistics already merged;
              // only the CTA holding u_K * 1 re-reads its slice of the target row
              const double u = (double)L.uniforms[(long long)i * (K + 1) + Ki];
              double tr[2] = {0.0, 0.0}, Z = 0.0, run = 0.0;
              for (int r = 0; r < G; ++r) {
                tr[r] = (St > 0.0 && xp[r].x != -INFINITY)
                            ? (double)xp[r].y * exp2((double)xp[r].x - (double)Mt) / St : 0.0;
                Z += tr[r];
              }
              int owner = -1, lastp = -1;
              for (int r = 0; r < G; ++r) {
                if (tr[r] > 0.0) lastp = r;
                if (owner < 0 && tr[r] > 0.0 && run + tr[r] > u * Z) owner = r;
                run += tr[r];
              }
              if (owner < 0 && Z > 0.0) owner = lastp;
              S.owner = owner;
              S.plan = owner == rank ? 2 : 0;
            }
          } else {
            S.plan = 0;
          }
        }
      }
      if (lane == 0) S.stop[k & 1] = stop ? 1 : 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.dec[k & 1]);
      if (stop) break;
    }
    if (ok) {
      // ---- the shared outputs (rank 0): accepted drafts, the -1 tail, the count, errors
      if (rank == 0) {
        const int bad = lane < Ki && (dreg < 0 || dreg >= L.V);
        if (lane < a) L.out_tokens[(long long)i * (K + 1) + lane] = dreg;
        if (lane <= K && lane > a) L.out_tokens[(long long)i * (K + 1) + lane] = -1;
        if (__any_sync(0xffffffffu, bad) && lane == 0) err |= PSPEC_DEVERR_TOKEN_RANGE;
        if (lane == 0) {
          L.accepted_len[i] = a;
          if constexpr (!kRej) {
            L.bonus[i] = gk;
            L.out_tokens[(long long)i * (K + 1) + a] = gk;
            S.tok = gk;
          }
          err |= ebk;
        }
      }
      if constexpr (kRej) {
        // ---- the draw at the stop position a
        DrawRow D;
        D.trow = tbase + (long long)a * L.ld - lo;
        D.resid = a < Ki;
        D.qrow = D.resid ? qbase + (long long)a * L.ld - lo : D.trow;
        D.mt = Mt; D.inv_st = St > 0.0 ? (float)(1.0 / St) : 0.f;
        D.mq = Mq; D.inv_sq = Sq > 0.0 ? (float)(1.0 / Sq) : 0.f;
        const double u = (double)L.uniforms[(long long)i * (K + 1) + Ki];
        double tot[2] = {0.0, 0.0};
        int owner = -1;
        bool have_sums = false;                         // csum holds this CTA's chunk sums
        if (D.resid) {
          if (!mbar_wait(&S.drawdone, 0u, spin)) ok = false;
          have_sums = true;
          double tt = 0.0;
          for (int c = lane; c < N; c += 32) tt += S.csum[c];
          tt = warp_sum_dd(tt);
          if constexpr (G > 1) {
            if (ok) {
              if (lane < G) {
                if (lane == rank) S.xtot[rank] = tt;
                else st_remote_f64(&S.xtot[rank], (unsigned)lane, tt);
              }
              __syncwarp();
              if (lane < G) {
                if (lane == rank) mbar_arrive(&S.xch2);
                else mbar_arrive_remote(&S.xch2, (unsigned)lane);
              }
              if (!mbar_wait(&S.xch2, 0u, spin)) ok = false;
              tot[0] = S.xtot[0];
              tot[1] = S.xtot[1];
            }
          } else {
            tot[0] = tt;
          }
          double Z0 = 0.0;
          for (int r = 0; r < G; ++r) Z0 += tot[r];
          if (Z0 == 0.0) {                              // residual vanished: draw from p
            D.resid = false;
            D.qrow = D.trow;
            have_sums = false;
          }
        }
        if (ok && !D.resid) {
          // slice totals of p from the statistics already merged
          for (int r = 0; r < G; ++r)
            tot[r] = (St > 0.0 && xp[r].x != -INFINITY)
                         ? (double)xp[r].y * exp2((double)xp[r].x - (double)Mt) / St : 0.0;
          if (S.plan == 2) {                            // this CTA's target row was re-read
            if (!mbar_wait(&S.drawdone, 0u, spin)) ok = false;
            have_sums = true;
          }
        }
        double Z = 0.0;
        for (int r = 0; r < G; ++r) Z += tot[r];
        const double thr = u * Z;
        double base = 0.0, run = 0.0;
        int last_pos = -1;
        for (int r = 0; r < G; ++r) {
          if (tot[r] > 0.0) last_pos = r;
          if (owner < 0 && tot[r] > 0.0 && run + tot[r] > thr) { owner = r; base = run; }
          run += tot[r];
        }
        const bool crossing = owner >= 0;
        if (!crossing && Z > 0.0) owner = last_pos;     // rounding: last slice with mass
        if (ok && owner == rank) {
          // chunk sums of this slice: from the draw pass, or (a residual that vanished, so
          // the draw is from p) computed here, grouped per lane as the consumers group them
          if (!have_sums)
            for (int c = 0; c < N; ++c) {
              const uint4* tv = reinterpret_cast<const uint4*>(static_cast<const elem*>(D.trow) + lo + (long long)c * CE);
              const int nv = (int)(min((long long)kCB, nbytes - (long long)c * kCB) / 16);
              double sum = 0.0;
#pragma unroll
              for (int j = 0; j < kLV; ++j) {
                const int v = lane + 32 * j;
                if (v < nv) {
                  float r[W], vs = 0.f;
                  draw_vec<Tag>(D, ld_stream(tv + v), make_uint4(0, 0, 0, 0), r);
#pragma unroll
                  for (int e = 0; e < W; ++e) vs += r[e];
                  sum += (double)vs;
                }
              }
              const double cs = warp_sum_dd(sum);
              if (lane == 0) S.csum[c] = cs;
              __syncwarp();
            }
          int chunk = -1, last_chunk = -1;
          double b2 = base, cb = base;
          for (int c = 0; c < N; ++c) {
            const double cs = S.csum[c];
            if (cs > 0.0) last_chunk = c;
            if (chunk < 0 && crossing && cs > 0.0 && b2 + cs > thr) { chunk = c; cb = b2; }
            b2 += cs;
          }
          int tok = 0;
          if (chunk < 0 && last_chunk >= 0) { chunk = last_chunk; cb = -INFINITY; }
          if (chunk >= 0) {
            int cand, lastp;
            chunk_rescan<Tag>(D, static_cast<const elem*>(D.trow) + lo,
                              static_cast<const elem*>(D.qrow) + lo, lo, chunk,
                              (int)(min((long long)kCB, nbytes - (long long)chunk * kCB) / 16), cb, thr,
                              crossing && cb != -INFINITY, &cand, &lastp);
            tok = cand >= 0 ? cand : (lastp >= 0 ? lastp : 0);
          }
          if (lane == 0) {
            L.out_tokens[(long long)i * (K + 1) + a] = tok;
            L.bonus[i] = tok;
            if (L.residual_mass) L.residual_mass[i] = (float)Z;
            S.tok = tok;
          }
        } else if (ok && owner < 0 && rank == 0 && lane == 0) {   // no mass anywhere: token 0
          L.out_tokens[(long long)i * (K + 1) + a] = 0;
          L.bonus[i] = 0;
          if (L.residual_mass) L.residual_mass[i] = 0.f;
          S.tok = 0;
        }
        if (lane == 0) S.owner = owner < 0 ? 0 : owner;
      } else {
        if (lane == 0) S.owner = 0;
      }
    }
    if (!ok && lane == 0) err |= PSPEC_DEVERR_TIMEOUT;
  }
  if (err) set_err(L.err, err);
  __syncthreads();
  if constexpr (G > 1) cg::this_cluster().sync();       // no remote traffic after this point
  if constexpr (kFuse) {                                // the whole step in this launch
    const int meta = S.owner;
    int eb = 0;
    build_span(L.b, L.row_vecs, i, S.a, Ki, rank == meta ? S.tok : 0, rank == meta, rank, G, &eb);
    if (i == L.b.B - 1) build_tail_pad(L.b, rank, G, &eb);
    set_err(L.b.err, eb);
  }
}

template <typename Kern>
cudaError_t smem_attribute(Kern kern, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_relaxed) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem));
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

template <typename Tag, int G, bool kRej, bool kFuse>
cudaError_t launch_one(const EarlyExitLaunch& L, cudaStream_t stream) {
  auto kern = stream_kernel<Tag, G, kRej, kFuse>;
  static std::atomic<unsigned long long> done{0};
  cudaError_t e = smem_attribute(kern, done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)L.nseq * G), 1, 1);
  cfg.blockDim = dim3(kSThreads, 1, 1);
  cfg.dynamicSmemBytes = sizeof(Smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = G > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, L);
}

template <int G>
cudaError_t launch_g(const EarlyExitLaunch& L, cudaStream_t s) {
  const bool bf = L.dtype == PSPEC_BF16;
  if (L.fuse_build) {
    if (L.rejection)
      return bf ? launch_one<BF16Tag, G, true, true>(L, s) : launch_one<F32Tag, G, true, true>(L, s);
    return bf ? launch_one<BF16Tag, G, false, true>(L, s) : launch_one<F32Tag, G, false, true>(L, s);
  }
  if (L.rejection)
    return bf ? launch_one<BF16Tag, G, true, false>(L, s) : launch_one<F32Tag, G, true, false>(L, s);
  return bf ? launch_one<BF16Tag, G, false, false>(L, s) : launch_one<F32Tag, G, false, false>(L, s);
}

}  // namespace

bool stream_shape_ok(int V, int G, pspec_dtype dtype) {
  if (V % 8 != 0 || (G != 1 && G != 2)) return false;
  const long long eb = dtype == PSPEC_BF16 ? 2 : 4;
  const long long vs = ((long long)V + G - 1) / G;
  const long long vs8 = (vs + 7) / 8 * 8;
  // every CTA's slice: at least kCW + kSpec chunks (so that no consumer warp's last chunk of
  // a position is among the chunks issued before the previous decision), at most kMaxChunks
  const long long last = (long long)V - (long long)(G - 1) * vs8;    // the shortest slice
  const long long n_min = last < vs8 ? last : vs8;
  const long long chunks_min = (n_min * eb + kCB - 1) / kCB;
  const long long chunks_max = (vs8 * eb + kCB - 1) / kCB;
  return n_min > 0 && chunks_min >= kCW + kSpec && chunks_max <= kMaxChunks;
}

long long stream_slice(int V, int G) {
  const long long vs = ((long long)V + G - 1) / G;
  return (vs + 7) / 8 * 8;
}

cudaError_t launch_stream(const EarlyExitLaunch& L, cudaStream_t stream) {
  return L.G == 2 ? launch_g<2>(L, stream) : launch_g<1>(L, stream);
}

}  // namespace pspec
