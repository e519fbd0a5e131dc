// verify_draw.cuh -- the rejection rule's draw over one row pair, used by the full sweep's
// draw launch.
//
// "Accept prefix; resample for rejected suffix" ("Capstone 14: speculative decoding
// inference server", section "Architecture"): at the first rejection a_i the emitted token
// is drawn from norm(max(0, p_{a_i} - q_{a_i})), and when every draft passes from the
// target's row K; the draw is the inverse CDF in token-id order at u_K * Z.
//
// The row is cut into 256-element warp tiles: warps sum r over their tiles (no block
// barrier per tile) into one double per tile, then one CTA prefix-sums the tile sums,
// picks the tile holding u * Z and rescans that tile with one warp.
#pragma once

#include "common.cuh"
#include "verify_common.cuh"

namespace pspec {

// ---------------------------------------------------------------------------------------
// The draw.  r(t) for t in [0, V): max(0, p(t) - q(t)) (resid) or p(t) (target only),
// each probability computed in fp32 as 2^((x - M) log2 e) / S.  The tile sums and the
// rescan compute r through the same code, so both see bit-identical values.
constexpr int kWTile = 256;   // one warp tile: 32 lanes x 8 consecutive elements

// The draw row of sequence i at stop position a: target row a against draft row a (the
// residual) when a < K_i, the target row K_i alone when all of the sequence's K_i drafts
// passed.  Rows are [B, K+1, ld] (target) and [B, K, ld] (draft).
__device__ __forceinline__ DrawRow make_draw_row(const void* target, const void* draft,
                                                 long long ld, int K, int Ki, int elem_bytes,
                                                 int i, int a, double mt, double st, double mq,
                                                 double sq) {
  DrawRow D;
  const char* t = static_cast<const char*>(target);
  const char* q = static_cast<const char*>(draft);
  D.trow = t + ((long long)i * (K + 1) + a) * ld * elem_bytes;
  D.resid = a < Ki;
  D.qrow = D.resid ? q + ((long long)i * K + a) * ld * elem_bytes : D.trow;
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

// The same walk with U tiles per iteration (2U loads of 16 bytes in flight per lane), for a
// single CTA that sums the tiles of a whole row on its own.
template <typename Tag, int U>
__device__ void warp_tile_sums_wide(const DrawRow& D, int V, long long t_begin, long long t_end,
                                    long long stride, double* ts) {
  const int lane = threadIdx.x & 31;
  for (long long t = t_begin; t < t_end; t += U * stride) {
    Raw8<Tag> T[U], Q[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long tu = t + u * stride;
      T[u].fast = Q[u].fast = false;
      if (tu < t_end) {
        raw8_load<Tag>(D.trow, V, tu * kWTile + lane * 8, T[u]);
        if (D.resid) raw8_load<Tag>(D.qrow, V, tu * kWTile + lane * 8, Q[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long tu = t + u * stride;
      if (tu >= t_end) break;                         // the same on every lane
      const long long e = tu * kWTile + lane * 8;
      float x[8], y[8], r[8];
      raw8_values<Tag>(D.trow, V, e, T[u], x);
      if (D.resid) raw8_values<Tag>(D.qrow, V, e, Q[u], y);
      else {
#pragma unroll
        for (int j = 0; j < 8; ++j) y[j] = x[j];
      }
      draw_r8(D, x, y, r);
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) sum += r[j];
      const double d = warp_sum((double)sum);
      if (lane == 0) ts[tu] = d;
    }
  }
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
  // Each thread owns a run of consecutive tiles: one pass of loads and one block-wide scan
  // give Z and every run's starting prefix, and the run holding u*Z finds its tile alone.
  const int per = (tiles + kThreads - 1) / kThreads;
  const int t_begin = tid * per;
  const int t_end = t_begin + per < tiles ? t_begin + per : tiles;
  double loc = 0.0;
  for (int t = t_begin; t < t_end; ++t) loc += ld_cg(ts + t);
  double Z;
  double base = block_exclusive_scan(loc, sh.red, &Z);
  if (Z == 0.0 && D.resid) {
    D.resid = false;                       // max(0, p - q) vanished: draw from p
    D.qrow = D.trow;
    __syncthreads();
    warp_tile_sums<Tag>(D, V, warp, tiles, kWarps, ts);
    __syncthreads();
    loc = 0.0;
    for (int t = t_begin; t < t_end; ++t) loc += ld_cg(ts + t);
    base = block_exclusive_scan(loc, sh.red, &Z);
  }
  const double thr = u * Z;

  // the first tile with mass whose inclusive prefix exceeds u*Z
  if (tid == 0) sh.found = 0x7fffffff;
  __syncthreads();
  int mine = 0x7fffffff;
  double mine_base = 0.0, run = base;
  for (int t = t_begin; t < t_end; ++t) {
    const double v = ld_cg(ts + t);
    if (v > 0.0 && run + v > thr) { mine = t; mine_base = run; break; }
    run += v;
  }
  if (mine != 0x7fffffff) atomicMin(&sh.found, mine);
  __syncthreads();
  int tile = sh.found;
  double tile_base = 0.0;
  if (tile != 0x7fffffff) {
    if (mine == tile) sh.red[kWarps] = mine_base;
    __syncthreads();
    tile_base = sh.red[kWarps];
  } else {
    tile = -1;
  }
  if (tile < 0 && Z > 0.0) {
    // rounding kept every prefix at or below u*Z: the last tile holding any mass
    __syncthreads();                       // every thread has read sh.found
    if (tid == 0) sh.found = -1;
    __syncthreads();
    for (int t = tid; t < tiles; t += kThreads)
      if (ld_cg(ts + t) > 0.0) atomicMax(&sh.found, t);
    __syncthreads();
    tile = sh.found;
    tile_base = -INFINITY;                 // no crossing inside: its last positive r
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
        // only a token with mass can cross (keeps padding past V out of reach)
        if (cand == 0x7fffffff && r[j] > 0.f && tile_base + ex + (double)incl[j] > thr)
          cand = (int)(e0 + j);
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

}  // namespace pspec
