// sample_drafts.cu -- draft tokens from the drafter's K output rows (one launch).
//
// "Eagle parallel speculative decoding, vLLM, TorchSpec", section "Parallel architecture":
// the P-EAGLE drafter predicts its K draft tokens from K output rows in one forward pass.
// Each row's token is drawn from softmax(row) by inverse CDF in token-id order with a
// caller-supplied uniform (the same convention as the verify draw), or taken as the argmax
// (lowest id on ties) when no uniforms are given.
//
// One pass over the logits: the grid is rows x S segments of chunks, a chunk being what one
// warp holds after eight 16-byte loads per lane (2048 bf16 or 1024 fp32 elements, lane l
// taking elements g*256 + 8l .. g*256 + 8l + 7 of group g).  Warp w of a CTA owns every
// eighth chunk of its segment and reduces each to one partial: the chunk max (base-2 units)
// and the sum of 2^(x log2e - max) over the chunk, or the chunk's (max, first index).  With
// the max taken first, every exponent is <= 0 and no running rescale is needed.  Because the
// draw is from the softmax itself, the chunk totals s 2^(m - M) / S that the CTA finishing a
// row derives from these partials ARE the row's CDF at chunk granularity; that CTA finds the
// chunk holding u and rescans it, one warp per group.  No CTA waits for another.
#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "verify_common.cuh"

namespace pspec {

namespace {

#ifndef PSPEC_SAMPLE_MIN_BLOCKS
#define PSPEC_SAMPLE_MIN_BLOCKS 5
#endif
constexpr int kSampleMinBlocks = PSPEC_SAMPLE_MIN_BLOCKS;   // CTAs per SM the registers target

struct TileMS {
  float m, s;
};

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---- a chunk in registers: 8 vectors, vector k = group k / VPG, part k % VPG -----------
template <typename Tag>
struct ChunkShape {
  static constexpr int VPG = 8 / Tag::kVec;           // 16-byte vectors per group of 8
  static constexpr int G = Tag::kVec;                 // groups per chunk (8 vectors in all)
};

// kVec consecutive elements from e with -inf past V, by scalar loads (ragged tails and
// rows whose base is not 16-byte aligned).
__device__ __forceinline__ uint4 ld_padded(const uint16_t* row, int V, long long e) {
  const unsigned short* r = reinterpret_cast<const unsigned short*>(row);
  uint32_t w[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const uint32_t lo = e + 2 * h < V ? (uint32_t)__ldg(r + e + 2 * h) : 0xFF80u;
    const uint32_t hi = e + 2 * h + 1 < V ? (uint32_t)__ldg(r + e + 2 * h + 1) : 0xFF80u;
    w[h] = lo | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 ld_padded(const float* row, int V, long long e) {
  uint32_t w[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) w[h] = e + h < V ? __float_as_uint(__ldg(row + e + h)) : 0xFF800000u;
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// The lane's part of group g starts at element c0 + 256 g (c0 = chunk start + 8 lane).
template <typename Tag, int N>
__device__ __forceinline__ void load_groups(const typename Tag::elem* row, int V, long long c0,
                                            bool fast, uint4 (&v)[N]) {
  constexpr int VPG = ChunkShape<Tag>::VPG;
  if (fast) {
#pragma unroll
    for (int k = 0; k < N; ++k) v[k] = ld_stream(row + c0 + (k / VPG) * 256 + (k % VPG) * Tag::kVec);
  } else {
#pragma unroll
    for (int k = 0; k < N; ++k) v[k] = ld_padded(row, V, c0 + (k / VPG) * 256 + (k % VPG) * Tag::kVec);
  }
}

template <typename Tag>
__device__ __forceinline__ float group_max(const uint4* v) {
  if constexpr (ChunkShape<Tag>::VPG == 1) return vec_max(v[0], Tag{});
  else return fmaxf(vec_max(v[0], Tag{}), vec_max(v[1], Tag{}));
}

template <typename Tag>
__device__ __forceinline__ void group_values(const uint4* v, float (&x)[8]) {
  if constexpr (ChunkShape<Tag>::VPG == 1) {
    unpack(v[0], x, BF16Tag{});
  } else {
    float lo[4], hi[4];
    unpack(v[0], lo, F32Tag{});
    unpack(v[1], hi, F32Tag{});
#pragma unroll
    for (int j = 0; j < 4; ++j) { x[j] = lo[j]; x[4 + j] = hi[j]; }
  }
}

template <typename Tag>
__global__ void __launch_bounds__(kThreads, kSampleMinBlocks) sample_kernel(const SampleLaunch L) {
  using elem = typename Tag::elem;
  constexpr int G = ChunkShape<Tag>::G;                 // groups of 8 elements per chunk
  constexpr int VPG = ChunkShape<Tag>::VPG;
  constexpr long long kChunk = 256LL * G;
  const long long item = blockIdx.x;
  const int seg = (int)(item % L.S);
  const long long row = item / L.S;
  const elem* rowp = static_cast<const elem*>(L.logits) + row * L.ld;
  const bool row_fast = (reinterpret_cast<uintptr_t>(rowp) & 15u) == 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool want_ms = L.uniforms != nullptr || L.probs != nullptr;
  const bool want_max = L.uniforms == nullptr;
  TileMS* parts = reinterpret_cast<TileMS*>(L.parts) + row * L.tiles;
  VI* maxes = reinterpret_cast<VI*>(L.maxes) + row * L.tiles;

  // ---- this CTA's chunks [t_lo, t_hi), warp w taking t_lo + w, t_lo + w + 8, ...
  const int t_lo = seg * L.tiles_per_seg;
  const int t_hi = min(L.tiles, t_lo + L.tiles_per_seg);
  for (int t = t_lo + warp; t < t_hi; t += kWarps) {
    const long long c0 = (long long)t * kChunk + lane * 8;
    uint4 v[8];
    load_groups<Tag>(rowp, L.V, c0, row_fast && (long long)(t + 1) * kChunk <= L.V, v);
    float gm[G];
#pragma unroll
    for (int g = 0; g < G; ++g) gm[g] = group_max<Tag>(v + g * VPG);
    if (want_max) {                                       // groups in increasing index order
      VI best{-INFINITY, kNoIndex};
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (gm[g] > best.v) {
          float x[8];
          group_values<Tag>(v + g * VPG, x);
          int jj = 0;
#pragma unroll
          for (int j = 7; j >= 0; --j)
            if (x[j] == gm[g]) jj = j;
          best = VI{gm[g], (int)(c0 + g * 256 + jj)};
        }
      }
      best = warp_argmax(best);
      if (lane == 0) maxes[t] = best;
    }
    if (want_ms) {
      float lm = gm[0];
#pragma unroll
      for (int g = 1; g < G; ++g) lm = fmaxf(lm, gm[g]);
      const float cmax = warp_max_f(lm);
      const float m = cmax == -INFINITY ? -INFINITY : cmax * kLog2e;
      float gs[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x[8];
        group_values<Tag>(v + g * VPG, x);
        float a0 = 0.f, a1 = 0.f;
        if (m != -INFINITY) {
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            float e0, e1;
            ffma2(e0, e1, x[j], x[j + 1], kLog2e, -m);
            fadd2(a0, a1, ex2(e0), ex2(e1));
          }
        }
        gs[g] = a0 + a1;
      }
#pragma unroll
      for (int w = 1; w < G; w <<= 1)                     // pairwise over the groups
#pragma unroll
        for (int g = 0; g + w < G; g += 2 * w) gs[g] += gs[g + w];
      const float cs = warp_sum_f(gs[0]);
      if (lane == 0) parts[t] = TileMS{m, cs};
    }
  }

  // ---- the CTA that finishes the row last turns the tile partials into the token
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int tk = atomicAdd(zrow(L.cnt, row), 1);
    s_last = (tk == L.S - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  __shared__ double s_red[kWarps + 1];
  __shared__ VI s_vi[kWarps];
  __shared__ float s_M;
  __shared__ int s_found, s_tok;
  const int tid = threadIdx.x;
  const int T = L.tiles;
  double S = 0.0;
  float M = -INFINITY;
  if (want_ms) {
    float mm = -INFINITY;
    for (int t = tid; t < T; t += kThreads) mm = fmaxf(mm, ld_cg(&parts[t].m));
    mm = warp_max_f(mm);
    if (lane == 0) s_red[warp] = mm;
    __syncthreads();
    if (tid == 0) {
      float a = -INFINITY;
      for (int w = 0; w < kWarps; ++w) a = fmaxf(a, (float)s_red[w]);
      s_M = a;
    }
    __syncthreads();
    M = s_M;
    double acc = 0.0;
    if (M != -INFINITY)
      for (int t = tid; t < T; t += kThreads) {
        const TileMS p = ld_cg(parts + t);
        if (p.m != -INFINITY) acc += (double)p.s * exp2((double)p.m - (double)M);
      }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    __syncthreads();
    if (lane == 0) s_red[warp] = acc;
    __syncthreads();
    for (int w = 0; w < kWarps; ++w) S += s_red[w];
  }

  int token = 0;
  if (want_max) {
    VI best{-INFINITY, kNoIndex};
    for (int t = tid; t < T; t += kThreads) {
      const VI v = ld_cg(maxes + t);
      if (vi_better(v, best)) best = v;
    }
    best = warp_argmax(best);
    __syncthreads();
    if (lane == 0) s_vi[warp] = best;
    __syncthreads();
    if (tid == 0) {
      VI b = s_vi[0];
      for (int w = 1; w < kWarps; ++w)
        if (vi_better(s_vi[w], b)) b = s_vi[w];
      s_tok = b.i == kNoIndex ? 0 : b.i;                 // a row of -inf / NaN only: token 0
    }
    __syncthreads();
    token = s_tok;
  } else {
    // chunk totals s 2^(m - M) / S are the CDF at chunk granularity: the first chunk whose
    // inclusive prefix exceeds u * Z (Z = their sum, 1 up to rounding) holds the token
    const double u = (double)L.uniforms[row];
    auto tile_total = [&](int t) -> double {
      if (t >= T || M == -INFINITY || S <= 0.0) return 0.0;
      const TileMS p = ld_cg(parts + t);
      return p.m == -INFINITY ? 0.0 : (double)p.s * exp2((double)p.m - (double)M) / S;
    };
    double Z = 0.0;
    {
      double z = 0.0;
      for (int t = tid; t < T; t += kThreads) z += tile_total(t);
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      __syncthreads();
      if (lane == 0) s_red[warp] = z;
      __syncthreads();
      for (int w = 0; w < kWarps; ++w) Z += s_red[w];
    }
    const double thr = u * Z;
    int tile = -1;
    double tile_base = 0.0, base = 0.0;
    for (int t0 = 0; t0 < T; t0 += kThreads) {
      const int t = t0 + tid;
      const double v = tile_total(t);
      double incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      __syncthreads();
      if (lane == 31) s_red[warp] = incl;
      if (tid == 0) s_found = 0x7fffffff;
      __syncthreads();
      double wb = 0.0, all = 0.0;
      for (int w = 0; w < kWarps; ++w) {
        if (w < warp) wb += s_red[w];
        all += s_red[w];
      }
      const double ex = wb + incl - v;
      if (t < T && v > 0.0 && base + ex + v > thr) atomicMin(&s_found, t);
      __syncthreads();
      const int f = s_found;
      if (f != 0x7fffffff) {
        if (t == f) s_red[kWarps] = base + ex;
        __syncthreads();
        tile = f;
        tile_base = s_red[kWarps];
        break;
      }
      base += all;
    }
    if (tile < 0 && Z > 0.0) {                           // rounding: the last chunk with mass
      __syncthreads();                                   // every thread has read s_found
      if (tid == 0) s_found = -1;
      __syncthreads();
      for (int t = tid; t < T; t += kThreads)
        if (tile_total(t) > 0.0) atomicMax(&s_found, t);
      __syncthreads();
      tile = s_found;
      tile_base = -INFINITY;                             // no crossing: its last positive p
    }
    // rescan the chunk: warp g < G takes group g, the groups' totals order the warps
    __shared__ double s_gtot[kWarps];
    __shared__ int s_cand[kWarps], s_lastp[kWarps];
    if (tile >= 0) {
      const long long e0 = (long long)tile * kChunk + warp * 256 + lane * 8;
      float r[8], incl[8];
      double ex = 0.0;
      if (warp < G) {
        uint4 gv[VPG];
        float x[8];
        load_groups<Tag>(rowp, L.V, e0, row_fast && e0 + 8 <= L.V, gv);
        group_values<Tag>(gv, x);
        const float inv_s = (float)(1.0 / S);
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          r[j] = ex2(fmaf(x[j], kLog2e, -M)) * inv_s;    // -inf and padding give 0
          acc += r[j];
          incl[j] = acc;
        }
        double inc = acc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double n = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += n;
        }
        ex = inc - (double)acc;
        if (lane == 31) s_gtot[warp] = inc;
      }
      __syncthreads();
      if (warp < G) {
        double gb = tile_base;
        for (int w = 0; w < warp; ++w) gb += s_gtot[w];
        int cand = 0x7fffffff, lastp = -1;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (r[j] > 0.f) lastp = (int)(e0 + j);
          // only a token with mass can cross (keeps padding past V out of reach)
          if (cand == 0x7fffffff && r[j] > 0.f && gb + ex + (double)incl[j] > thr) cand = (int)(e0 + j);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          cand = min(cand, __shfl_xor_sync(0xffffffffu, cand, o));
          lastp = max(lastp, __shfl_xor_sync(0xffffffffu, lastp, o));
        }
        if (lane == 0) {
          s_cand[warp] = cand;
          s_lastp[warp] = lastp;
        }
      }
      __syncthreads();
      if (tid == 0) {
        int cand = 0x7fffffff, lastp = -1;
        for (int w = 0; w < G; ++w) {
          cand = min(cand, s_cand[w]);
          lastp = max(lastp, s_lastp[w]);
        }
        s_tok = cand != 0x7fffffff ? cand : (lastp >= 0 ? lastp : 0);
      }
    } else if (tid == 0) {
      s_tok = 0;                                         // a row without mass
    }
    __syncthreads();
    token = s_tok;
  }
  if (tid == 0) {
    L.tokens[row] = token;
    if (L.probs) {
      const float x = load_scalar(rowp, token);
      L.probs[row] = (M == -INFINITY || x == -INFINITY || S <= 0.0)
                         ? 0.f
                         : (float)(exp2((double)x * (double)kLog2e - (double)M) / S);
    }
    *zrow(L.cnt, row) = 0;
  }
}

}  // namespace

cudaError_t launch_sample(const SampleLaunch& L, cudaStream_t stream) {
  const long long grid = L.rows * L.S;
  if (L.dtype == PSPEC_BF16)
    sample_kernel<BF16Tag><<<(unsigned)grid, kThreads, 0, stream>>>(L);
  else
    sample_kernel<F32Tag><<<(unsigned)grid, kThreads, 0, stream>>>(L);
  return cudaGetLastError();
}

}  // namespace pspec
