// verify_rejection.cu -- rejection-rule target verification (two launches).
//
// "Accept prefix; resample for rejected suffix" ("Capstone 14: speculative decoding
// inference server", section "Architecture") with output identical in law to plain
// autoregressive decoding (rskf.cn article, section 2.2).  Draft k is accepted with
// probability min(1, p_k(d_k) / q_k(d_k)); at the first rejection a_i the emitted token is
// drawn from norm(max(0, p_{a_i} - q_{a_i})), and when every draft passes it is drawn from
// the target's row K.
//
// Stats sweep: grid B*(2K+1) rows x S segments.  Each CTA streams one segment
// of one target or draft row with 16-byte loads and keeps an online (max, sum exp) pair.
// The CTA that finishes a sequence last (atomic ticket, no waiting) merges the partials
// in segment order in double, evaluates p(d_k) and q(d_k), and builds the accept bitmask
// (one bit per draft, so the first rejection is one find-first-set).
//
// Draw launch: grid B x C CTAs over 256-element warp tiles of each sequence's row a_i.
// Each warp sums r = max(0, p - q) (or p) over its own tiles, with no block barrier per
// tile, and stores one double per tile; the CTA that finishes a sequence last prefix-sums
// the tile sums, picks the tile holding u_K * Z and rescans that tile with one warp.
#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "verify_common.cuh"

namespace pspec {

namespace {

// Row r of sequence i in the sweep order: target rows 0..K, then draft rows 0..K-1.
template <typename elem>
__device__ __forceinline__ const elem* sweep_row(const RejectionLaunch& L, int i, int r) {
  if (r <= L.K)
    return static_cast<const elem*>(L.target) + ((long long)i * (L.K + 1) + r) * L.ld;
  return static_cast<const elem*>(L.draft) + ((long long)i * L.K + (r - L.K - 1)) * L.ld;
}

// ---------------------------------------------------------------------------------------
// The draw.  r(t) for t in [0, V): max(0, p(t) - q(t)) (resid) or p(t) (target only),
// each probability computed in fp32 as 2^((x - M) log2 e) / S.  The tile sums and the
// rescan compute r through the same code, so both see bit-identical values.
constexpr int kWTile = 256;   // one warp tile: 32 lanes x 8 consecutive elements

__device__ __forceinline__ DrawRow make_draw_row(const RejectionLaunch& L, int elem_bytes, int i,
                                                 int a, double mt, double st, double mq,
                                                 double sq) {
  DrawRow D;
  const char* t = static_cast<const char*>(L.target);
  const char* q = static_cast<const char*>(L.draft);
  D.trow = t + ((long long)i * (L.K + 1) + a) * L.ld * elem_bytes;
  D.resid = a < L.K;
  D.qrow = D.resid ? q + ((long long)i * L.K + a) * L.ld * elem_bytes : D.trow;
  D.mt = (float)mt;
  D.inv_st = st > 0.0 ? (float)(1.0 / st) : 0.f;
  D.mq = (float)mq;
  D.inv_sq = sq > 0.0 ? (float)(1.0 / sq) : 0.f;
  return D;
}

// Eight consecutive elements [t0, t0+8) of a row: 16-byte loads when the group lies inside
// the row on a 16-byte boundary, else scalar loads (-inf past V) when the values are read.
template <typename Tag>
struct Raw8 {
  uint4 v[8 / Tag::kVec];
  bool fast;
};

template <typename Tag>
__device__ __forceinline__ void raw8_load(const void* rowp, int V, long long t0, Raw8<Tag>& R) {
  const typename Tag::elem* row = static_cast<const typename Tag::elem*>(rowp);
  R.fast = t0 + 8 <= V && (reinterpret_cast<uintptr_t>(row + t0) & 15u) == 0;
  if (R.fast) {
#pragma unroll
    for (int k = 0; k < 8 / Tag::kVec; ++k) R.v[k] = ld_stream(row + t0 + k * Tag::kVec);
  }
}

template <typename Tag>
__device__ __forceinline__ void raw8_values(const void* rowp, int V, long long t0,
                                            const Raw8<Tag>& R, float (&x)[8]) {
  const typename Tag::elem* row = static_cast<const typename Tag::elem*>(rowp);
  if (R.fast) {
    if constexpr (Tag::kVec == 8) {
      unpack(R.v[0], x, BF16Tag{});
    } else {
      float lo[4], hi[4];
      unpack(R.v[0], lo, F32Tag{});
      unpack(R.v[1], hi, F32Tag{});
#pragma unroll
      for (int j = 0; j < 4; ++j) { x[j] = lo[j]; x[4 + j] = hi[j]; }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = t0 + j < V ? load_scalar(row, t0 + j) : -INFINITY;
  }
}

template <typename Tag>
__device__ __forceinline__ void r8(const DrawRow& D, int V, long long t0, float (&r)[8]) {
  Raw8<Tag> T, Q;
  raw8_load<Tag>(D.trow, V, t0, T);
  if (D.resid) raw8_load<Tag>(D.qrow, V, t0, Q);
  float xt[8], xq[8];
  raw8_values<Tag>(D.trow, V, t0, T, xt);
  if (D.resid) raw8_values<Tag>(D.qrow, V, t0, Q, xq);
  draw_r8(D, xt, xq, r);
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// This warp's share of the tile sums: tiles t_begin, t_begin + stride, ... below t_end,
// two tiles per iteration with all their loads issued before any arithmetic.
template <typename Tag>
__device__ void warp_tile_sums(const DrawRow& D, int V, long long t_begin, long long t_end,
                               long long stride, double* ts) {
  const int lane = threadIdx.x & 31;
  for (long long t = t_begin; t < t_end; t += 2 * stride) {
    const long long t2 = t + stride;
    const bool two = t2 < t_end;
    const long long e1 = t * kWTile + lane * 8, e2 = t2 * kWTile + lane * 8;
    Raw8<Tag> T1, Q1, T2, Q2;
    raw8_load<Tag>(D.trow, V, e1, T1);
    if (D.resid) raw8_load<Tag>(D.qrow, V, e1, Q1);
    if (two) {
      raw8_load<Tag>(D.trow, V, e2, T2);
      if (D.resid) raw8_load<Tag>(D.qrow, V, e2, Q2);
    }
    float x[8], y[8], r[8];
    float s1 = 0.f, s2 = 0.f;
    raw8_values<Tag>(D.trow, V, e1, T1, x);
    if (D.resid) raw8_values<Tag>(D.qrow, V, e1, Q1, y);
    draw_r8(D, x, y, r);
#pragma unroll
    for (int j = 0; j < 8; ++j) s1 += r[j];
    if (two) {
      raw8_values<Tag>(D.trow, V, e2, T2, x);
      if (D.resid) raw8_values<Tag>(D.qrow, V, e2, Q2, y);
      draw_r8(D, x, y, r);
#pragma unroll
      for (int j = 0; j < 8; ++j) s2 += r[j];
    }
    const double d1 = warp_sum((double)s1);
    const double d2 = warp_sum((double)s2);
    if (lane == 0) {
      ts[t] = d1;
      if (two) ts[t2] = d2;
    }
  }
}

__device__ __forceinline__ double block_sum(double v, double* s_red) {
  v = warp_sum(v);
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

struct DrawShared {
  double red[kWarps + 1];
  int found;
  int token;
};

// One CTA, all threads, once the tile sums ts[0..tiles) of row a_i are in place: Z, the
// first tile whose inclusive prefix exceeds u*Z, and the first token of that tile whose
// running sum does (the last positive r of the tile if rounding leaves none; token 0 if
// the row holds no mass at all).  A residual that sums to zero is redrawn from p itself.
template <typename Tag>
__device__ int draw_finish(DrawRow& D, int V, int tiles, double u, double* ts, DrawShared& sh,
                           double* Zout) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double Z = 0.0;
  for (int t0 = 0; t0 < tiles; t0 += kThreads)
    Z += block_sum(t0 + tid < tiles ? ld_cg(ts + t0 + tid) : 0.0, sh.red);
  if (Z == 0.0 && D.resid) {
    D.resid = false;                       // max(0, p - q) vanished: draw from p
    D.qrow = D.trow;
    __syncthreads();
    warp_tile_sums<Tag>(D, V, warp, tiles, kWarps, ts);
    __syncthreads();
    Z = 0.0;
    for (int t0 = 0; t0 < tiles; t0 += kThreads)
      Z += block_sum(t0 + tid < tiles ? ld_cg(ts + t0 + tid) : 0.0, sh.red);
  }
  const double thr = u * Z;

  int tile = -1;
  double tile_base = 0.0;
  double base = 0.0;
  for (int t0 = 0; t0 < tiles; t0 += kThreads) {
    const int t = t0 + tid;
    const double v = t < tiles ? ld_cg(ts + t) : 0.0;
    double tot;
    const double ex = block_exclusive_scan(v, sh.red, &tot);
    if (tid == 0) sh.found = 0x7fffffff;
    __syncthreads();
    if (t < tiles && v > 0.0 && base + ex + v > thr) atomicMin(&sh.found, t);
    __syncthreads();
    const int f = sh.found;
    if (f != 0x7fffffff) {
      if (t == f) sh.red[kWarps] = base + ex;
      __syncthreads();
      tile = f;
      tile_base = sh.red[kWarps];
      break;                               // f is the same on every thread
    }
    base += tot;
  }
  if (tile < 0 && Z > 0.0) {
    // rounding kept every prefix at or below u*Z: the last tile holding any mass
    if (tid == 0) sh.found = -1;
    __syncthreads();
    for (int t = tid; t < tiles; t += kThreads)
      if (ld_cg(ts + t) > 0.0) atomicMax(&sh.found, t);
    __syncthreads();
    tile = sh.found;
    if (tile >= 0) {
      tile_base = thr;                     // no crossing inside: take its last positive r
    }
  }
  if (warp == 0) {
    int token = 0;
    if (tile >= 0) {
      const long long e0 = (long long)tile * kWTile + lane * 8;
      float r[8];
      r8<Tag>(D, V, e0, r);
      float incl[8], run = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) { run += r[j]; incl[j] = run; }
      double inc = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
      }
      const double ex = inc - (double)run;
      int cand = 0x7fffffff, lastpos = -1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (r[j] > 0.f) lastpos = (int)(e0 + j);
        if (cand == 0x7fffffff && tile_base + ex + (double)incl[j] > thr) cand = (int)(e0 + j);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        cand = min(cand, __shfl_xor_sync(0xffffffffu, cand, o));
        lastpos = max(lastpos, __shfl_xor_sync(0xffffffffu, lastpos, o));
      }
      token = cand != 0x7fffffff ? cand : (lastpos >= 0 ? lastpos : 0);
    }
    if (lane == 0) sh.token = token;
  }
  __syncthreads();
  *Zout = Z;
  return sh.token;
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

  MSAcc acc = msacc_init();
  sweep_segment_batched<Tag, 4>(
      row, lo, hi, [&](const uint4 (&v)[4]) { consume_ms_batch<Tag, 4>(v, acc); },
      [&](const uint4& v, long long) { consume_ms<Tag>(v, acc); },
      [&](float x, long long) { consume_one(x, acc); });
  MS ms = msacc_final(acc);

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

  // ---- last CTA of sequence i: merge partials (double), accept test, stats of row a_i.
  // Partials are in base-2 units (MS); p(d) uses the same kLog2e, so the normaliser and
  // the numerator describe one and the same softmax.
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
        if (q.m != -INFINITY) S += (double)q.s * exp2((double)q.m - (double)M);
      }
    s_M[threadIdx.x] = M;
    s_S[threadIdx.x] = S;
  }
  __syncthreads();
  if (warp != 0) return;

  {
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
      if (Mt != -INFINITY && xt != -INFINITY) p = exp2((double)xt * (double)kLog2e - Mt) / St;
      if (Mq != -INFINITY && xq != -INFINITY) q = exp2((double)xq * (double)kLog2e - Mq) / Sq;
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
      L.draft_lse[(long long)i * K + lane] =
          (float)(M == -INFINITY ? M : (M + log2(s_S[K + 1 + lane])) / (double)kLog2e);
    }
  }
  if (lane <= K) {
    if (L.target_lse) {
      const double M = s_M[lane];
      L.target_lse[(long long)i * (K + 1) + lane] =
          (float)(M == -INFINITY ? M : (M + log2(s_S[lane])) / (double)kLog2e);
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
  }  // warp 0
}

// The draw launch: B x C CTAs over the warp tiles of each sequence's row a_i.
template <typename Tag>
__global__ void __launch_bounds__(kThreads)
rej_draw_kernel(const RejectionLaunch L) {
  using elem = typename Tag::elem;
  const int K = L.K;
  const int i = blockIdx.x / L.C;
  const int c = blockIdx.x % L.C;
  const int warp = threadIdx.x >> 5;
  __shared__ int s_last;
  __shared__ DrawShared sh;

  const SeqInfo si = reinterpret_cast<const SeqInfo*>(L.seq)[i];  // previous launch
  DrawRow D = make_draw_row(L, sizeof(elem), i, si.a, si.mt, si.st, si.mq, si.sq);
  double* ts = L.tile_sums + (long long)i * L.tiles;
  const long long t_lo = (long long)c * L.tiles_per_chunk;
  const long long t_hi = min((long long)L.tiles, t_lo + L.tiles_per_chunk);
  warp_tile_sums<Tag>(D, L.V, t_lo + warp, t_hi, kWarps, ts);
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int t = atomicAdd(L.cnt2 + i, 1);
    s_last = (t == L.C - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  double Z;
  const int token = draw_finish<Tag>(D, L.V, L.tiles, (double)L.uniforms[(long long)i * (K + 1) + K],
                                     ts, sh, &Z);
  if (threadIdx.x == 0) {
    L.out_tokens[(long long)i * (K + 1) + si.a] = token;
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
