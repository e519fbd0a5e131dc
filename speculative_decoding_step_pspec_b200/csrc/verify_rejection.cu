// verify_rejection.cu -- rejection-rule target verification (two launches).
//
// "Accept prefix; resample for rejected suffix" ("Capstone 14: speculative decoding
// inference server", section "Architecture") with output identical in law to plain
// autoregressive decoding (rskf.cn article, section 2.2).  Draft k is accepted with
// probability min(1, p_k(d_k) / q_k(d_k)); at the first rejection a_i the emitted token is
// drawn from norm(max(0, p_{a_i} - q_{a_i})), and when every draft passes it is drawn from
// the target's row K.
//
// Launch 1 (stats sweep): grid B*(2K+1) rows x S segments.  Each CTA streams one segment
// of one target or draft row with 16-byte loads and keeps an online (max, sum exp) pair.
// The CTA that finishes a sequence last (atomic ticket, no waiting) merges the partials
// in segment order in double, evaluates p(d_k) and q(d_k), builds the accept bitmask
// (one bit per draft, so the first rejection is one find-first-set), and stores the
// statistics of row a_i for the draw.
//
// Launch 2 (draw): grid B x C chunks over row a_i of every sequence.  Each CTA sums
// r = max(0, p - q) (or p) over its 2048-element tiles and stores one double per tile.
// The last CTA of the sequence prefix-sums the tile sums, picks the tile that holds
// u_K * Z, and rescans only that tile with a block-wide scan to find the token.
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace pspec {

namespace {

template <typename Tag>
__device__ __forceinline__ void consume_ms(const uint4& v, MS& ms) {
  constexpr int W = Tag::kVec;
  float x[W];
  unpack(v, x, Tag{});
  float vmax = x[0];
#pragma unroll
  for (int t = 1; t < W; ++t) vmax = fmaxf(vmax, x[t]);
  if (vmax == -INFINITY) return;
  if (vmax > ms.m) {
    ms.s = ms.m == -INFINITY ? 0.f : ms.s * ex2((ms.m - vmax) * kLog2e);
    ms.m = vmax;
  }
  float acc = 0.f;
#pragma unroll
  for (int t = 0; t < W; ++t) acc += ex2((x[t] - ms.m) * kLog2e);
  ms.s += acc;
}

// Row r of sequence i in the sweep order: target rows 0..K, then draft rows 0..K-1.
template <typename elem>
__device__ __forceinline__ const elem* sweep_row(const RejectionLaunch& L, int i, int r) {
  if (r <= L.K)
    return static_cast<const elem*>(L.target) + ((long long)i * (L.K + 1) + r) * L.ld;
  return static_cast<const elem*>(L.draft) + ((long long)i * L.K + (r - L.K - 1)) * L.ld;
}

template <typename Tag>
__global__ void __launch_bounds__(kThreads)
rej_stats_kernel(const RejectionLaunch L) {
  using elem = typename Tag::elem;
  const int K = L.K;
  const int R = 2 * K + 1;
  const long long item = blockIdx.x;
  const int s = (int)(item % L.S);
  const long long rowg = item / L.S;                 // i*R + r
  const int i = (int)(rowg / R);
  const int r = (int)(rowg % R);
  const elem* row = sweep_row<elem>(L, i, r);
  const long long lo = (long long)s * L.seg;
  const long long hi = min((long long)L.V, lo + L.seg);

  MS ms{-INFINITY, 0.f};
  sweep_segment<Tag, 4>(
      row, lo, hi, [&](const uint4& v, long long) { consume_ms<Tag>(v, ms); },
      [&](float x, long long) {
        if (x != -INFINITY) ms = ms_merge(ms, MS{x, 1.f});
      });

  __shared__ MS s_ms[kWarps];
  __shared__ int s_last;
  ms = warp_merge_ms(ms);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s_ms[warp] = ms;
  __syncthreads();
  if (warp == 0) {
    ms = lane < kWarps ? s_ms[lane] : MS{-INFINITY, 0.f};
    ms = warp_merge_ms(ms);
    if (lane == 0) {
      reinterpret_cast<RejPart*>(L.part)[item] = RejPart{ms.m, ms.s};
      __threadfence();
      int t = atomicAdd(L.cnt + i, 1);
      s_last = (t == L.S * R - 1);
    }
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA of sequence i: merge partials (double), accept test, stats of row a_i
  __shared__ double s_M[2 * PSPEC_MAX_K + 1];
  __shared__ double s_S[2 * PSPEC_MAX_K + 1];
  const RejPart* part = reinterpret_cast<const RejPart*>(L.part) + (long long)i * R * L.S;
  if (threadIdx.x < R) {
    const RejPart* pr = part + (long long)threadIdx.x * L.S;
    float M = -INFINITY;
    for (int t = 0; t < L.S; ++t) M = fmaxf(M, ld_cg(&pr[t].m));
    double S = 0.0;
    if (M != -INFINITY)
      for (int t = 0; t < L.S; ++t) {
        RejPart q = ld_cg(pr + t);
        if (q.m != -INFINITY) S += (double)q.s * exp((double)q.m - (double)M);
      }
    s_M[threadIdx.x] = M;
    s_S[threadIdx.x] = S;
  }
  __syncthreads();
  if (warp != 0) return;

  int d = -1;
  bool bad = false, accept = false;
  double p = 0.0, q = 0.0;
  if (lane < K) {
    d = L.draft_tokens[(long long)i * K + lane];
    bad = d < 0 || d >= L.V;
    if (!bad) {
      const double Mt = s_M[lane], St = s_S[lane];
      const double Mq = s_M[K + 1 + lane], Sq = s_S[K + 1 + lane];
      const float xt = load_scalar(sweep_row<elem>(L, i, lane), d);
      const float xq = load_scalar(sweep_row<elem>(L, i, K + 1 + lane), d);
      if (Mt != -INFINITY && xt != -INFINITY) p = exp((double)xt - Mt) / St;
      if (Mq != -INFINITY && xq != -INFINITY) q = exp((double)xq - Mq) / Sq;
      const double u = (double)L.uniforms[(long long)i * (K + 1) + lane];
      accept = q > 0.0 ? (u * q < p) : (p > 0.0);
    }
  }
  const unsigned mask = __ballot_sync(0xffffffffu, accept);
  const unsigned anybad = __ballot_sync(0xffffffffu, bad);
  int a = __ffs(~mask) - 1;              // first rejected draft
  if (a > K) a = K;
  if (lane < K) {
    if (L.p_at_draft) L.p_at_draft[(long long)i * K + lane] = (float)p;
    if (L.q_at_draft) L.q_at_draft[(long long)i * K + lane] = (float)q;
    if (L.draft_lse) {
      const double M = s_M[K + 1 + lane];
      L.draft_lse[(long long)i * K + lane] = (float)(M == -INFINITY ? M : M + log(s_S[K + 1 + lane]));
    }
  }
  if (lane <= K) {
    if (L.target_lse) {
      const double M = s_M[lane];
      L.target_lse[(long long)i * (K + 1) + lane] = (float)(M == -INFINITY ? M : M + log(s_S[lane]));
    }
    if (lane != a) L.out_tokens[(long long)i * (K + 1) + lane] = lane < a ? d : -1;
  }
  if (lane == 0) {
    SeqInfo si;
    si.mt = s_M[a];
    si.st = s_S[a];
    si.mq = a < K ? s_M[K + 1 + a] : 0.0;
    si.sq = a < K ? s_S[K + 1 + a] : 1.0;
    si.a = a;
    si.pad[0] = si.pad[1] = si.pad[2] = 0;
    reinterpret_cast<SeqInfo*>(L.seq)[i] = si;
    L.accepted_len[i] = a;
    if (anybad) set_err(L.err, PSPEC_DEVERR_TOKEN_RANGE);
    L.cnt[i] = 0;
  }
}

// ---------------------------------------------------------------------------------------
// The draw.  r(t) for t in [0, V): max(0, p(t) - q(t)) (kResid) or p(t) (target only),
// each probability computed in fp32 as 2^((x - M) log2 e) / S.  The chunk pass and the
// rescan call the same function, so both see bit-identical r values.
struct DrawRow {
  const void* trow;
  const void* qrow;
  float mt, inv_st, mq, inv_sq;
  bool resid;
};

template <typename Tag>
__device__ __forceinline__ void load8(const typename Tag::elem* row, int V, long long t0,
                                      float (&x)[8]) {
  if (t0 + 8 <= V && (reinterpret_cast<uintptr_t>(row + t0) & 15u) == 0) {
    if constexpr (Tag::kVec == 8) {
      unpack(ld_stream(row + t0), x, BF16Tag{});
    } else {
      float lo[4], hi[4];
      unpack(ld_stream(row + t0), lo, F32Tag{});
      unpack(ld_stream(row + t0 + 4), hi, F32Tag{});  // 32 bytes: both halves aligned
#pragma unroll
      for (int j = 0; j < 4; ++j) { x[j] = lo[j]; x[4 + j] = hi[j]; }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = t0 + j < V ? load_scalar(row, t0 + j) : -INFINITY;
  }
}

template <typename Tag>
__device__ __forceinline__ void tile_values(const DrawRow& D, int V, long long t0, float (&r)[8]) {
  using elem = typename Tag::elem;
  float xt[8], xq[8];
  load8<Tag>(static_cast<const elem*>(D.trow), V, t0, xt);
  if (D.resid) load8<Tag>(static_cast<const elem*>(D.qrow), V, t0, xq);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float pt = (D.mt == -INFINITY || xt[j] == -INFINITY) ? 0.f
                                                         : ex2((xt[j] - D.mt) * kLog2e) * D.inv_st;
    if (D.resid) {
      float pq = (D.mq == -INFINITY || xq[j] == -INFINITY)
                     ? 0.f
                     : ex2((xq[j] - D.mq) * kLog2e) * D.inv_sq;
      r[j] = fmaxf(pt - pq, 0.f);
    } else {
      r[j] = pt;
    }
  }
}

__device__ __forceinline__ double block_sum(double v, double* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += s_red[w];
  return t;
}

// Exclusive prefix over the CTA of one double per thread; returns the prefix and sets *total.
__device__ __forceinline__ double block_exclusive_scan(double v, double* s_red, double* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  __syncthreads();
  if (lane == 31) s_red[warp] = incl;
  __syncthreads();
  double base = 0.0, all = 0.0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) base += s_red[w];
    all += s_red[w];
  }
  *total = all;
  return base + incl - v;
}

template <typename Tag>
__device__ double tile_sum(const DrawRow& D, int V, int tile, double* s_red) {
  float r[8];
  tile_values<Tag>(D, V, (long long)tile * kTile + threadIdx.x * 8, r);
  float th = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) th += r[j];
  return block_sum((double)th, s_red);
}

template <typename Tag>
__global__ void __launch_bounds__(kThreads)
rej_draw_kernel(const RejectionLaunch L) {
  const int K = L.K;
  const int i = blockIdx.x / L.C;
  const int c = blockIdx.x % L.C;
  __shared__ double s_red[kWarps];
  __shared__ int s_last;
  __shared__ int s_tok;

  const SeqInfo si = reinterpret_cast<const SeqInfo*>(L.seq)[i];  // previous launch
  const int a = si.a;
  DrawRow D;
  D.trow = static_cast<const typename Tag::elem*>(L.target) + ((long long)i * (K + 1) + a) * L.ld;
  D.resid = a < K;
  D.qrow = D.resid ? static_cast<const typename Tag::elem*>(L.draft) + ((long long)i * K + a) * L.ld
                   : D.trow;
  D.mt = (float)si.mt;
  D.inv_st = si.st > 0.0 ? (float)(1.0 / si.st) : 0.f;
  D.mq = (float)si.mq;
  D.inv_sq = si.sq > 0.0 ? (float)(1.0 / si.sq) : 0.f;

  double* ts = L.tile_sums + (long long)i * L.tiles;
  const int t_lo = c * L.tiles_per_chunk;
  const int t_hi = min(L.tiles, t_lo + L.tiles_per_chunk);
  for (int t = t_lo; t < t_hi; ++t) {
    double v = tile_sum<Tag>(D, L.V, t, s_red);
    if (threadIdx.x == 0) ts[t] = v;
  }
  if (threadIdx.x == 0) {
    __threadfence();
    int t = atomicAdd(L.cnt2 + i, 1);
    s_last = (t == L.C - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA: Z, the tile holding u*Z, and the token inside it
  const double u = (double)L.uniforms[(long long)i * (K + 1) + K];
  double Z = 0.0;
  for (int t0 = 0; t0 < L.tiles; t0 += kThreads) {
    double v = t0 + (int)threadIdx.x < L.tiles ? ld_cg(ts + t0 + threadIdx.x) : 0.0;
    Z += block_sum(v, s_red);
  }
  if (Z == 0.0 && D.resid) {
    // max(0, p - q) vanished everywhere: draw from p itself
    D.resid = false;
    D.qrow = D.trow;
    Z = 0.0;
    for (int t = 0; t < L.tiles; ++t) {
      double v = tile_sum<Tag>(D, L.V, t, s_red);
      if (threadIdx.x == 0) ts[t] = v;
      Z += v;
    }
    __syncthreads();
    __threadfence_block();
  }
  const double thr = u * Z;

  // first tile whose inclusive prefix exceeds thr
  int tile = -1;
  double tile_base = 0.0;
  {
    double base = 0.0;
    if (threadIdx.x == 0) s_tok = 0x7fffffff;
    for (int t0 = 0; t0 < L.tiles && tile < 0; t0 += kThreads) {
      const int t = t0 + threadIdx.x;
      double v = t < L.tiles ? ld_cg(ts + t) : 0.0;
      double tot;
      double ex = block_exclusive_scan(v, s_red, &tot);
      if (t < L.tiles && base + ex + v > thr) atomicMin(&s_tok, t);
      __syncthreads();
      int found = s_tok;
      if (found != 0x7fffffff) {
        tile = found;
        // base of the found tile: re-read the prefix from the owning thread
        if (t == found) s_red[0] = base + ex;
        __syncthreads();
        tile_base = s_red[0];
      }
      base += tot;
      __syncthreads();
    }
  }

  int token = 0;
  if (tile >= 0) {
    float r[8];
    const long long t0 = (long long)tile * kTile + threadIdx.x * 8;
    tile_values<Tag>(D, L.V, t0, r);
    float incl[8];
    float run = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) { run += r[j]; incl[j] = run; }
    double tot;
    double ex = block_exclusive_scan((double)run, s_red, &tot);
    int cand = 0x7fffffff, lastpos = -1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (r[j] > 0.f) lastpos = (int)(t0 + j);
      if (cand == 0x7fffffff && tile_base + ex + (double)incl[j] > thr) cand = (int)(t0 + j);
    }
    __syncthreads();
    if (threadIdx.x == 0) { s_tok = 0x7fffffff; }
    __syncthreads();
    if (cand != 0x7fffffff) atomicMin(&s_tok, cand);
    __syncthreads();
    token = s_tok;
    if (token == 0x7fffffff) {
      // rounding left the crossing outside the rescan: the last positive r of the tile
      __syncthreads();
      if (threadIdx.x == 0) s_tok = -1;
      __syncthreads();
      if (lastpos >= 0) atomicMax(&s_tok, lastpos);
      __syncthreads();
      token = s_tok < 0 ? 0 : s_tok;
    }
  }
  if (threadIdx.x == 0) {
    L.out_tokens[(long long)i * (K + 1) + a] = token;
    L.bonus[i] = token;
    if (L.residual_mass) L.residual_mass[i] = (float)Z;
    L.cnt2[i] = 0;
  }
}

}  // namespace

cudaError_t launch_rejection(const RejectionLaunch& L, cudaStream_t stream,
                             cudaEvent_t split_event) {
  const long long grid1 = (long long)L.B * (2 * L.K + 1) * L.S;
  const long long grid2 = (long long)L.B * L.C;
  if (L.dtype == PSPEC_BF16)
    rej_stats_kernel<BF16Tag><<<(unsigned)grid1, kThreads, 0, stream>>>(L);
  else
    rej_stats_kernel<F32Tag><<<(unsigned)grid1, kThreads, 0, stream>>>(L);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (split_event) {
    e = cudaEventRecord(split_event, stream);
    if (e != cudaSuccess) return e;
  }
  if (L.dtype == PSPEC_BF16)
    rej_draw_kernel<BF16Tag><<<(unsigned)grid2, kThreads, 0, stream>>>(L);
  else
    rej_draw_kernel<F32Tag><<<(unsigned)grid2, kThreads, 0, stream>>>(L);
  return cudaGetLastError();
}

}  // namespace pspec
