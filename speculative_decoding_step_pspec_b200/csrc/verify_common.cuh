// verify_common.cuh -- per-logit arithmetic shared by the verify kernels (full sweeps and
// the early-exit cluster kernel): the online softmax normaliser of 16-byte vectors, the
// argmax of 16-byte vectors, and the residual r = max(0, p - q) of the draw.
//
// The sweeps are bound by instruction issue as much as by HBM, so each vector is handled
// with as few instructions as the arithmetic allows: one running-max check per batch of
// vectors, exponent arguments as one fused multiply-add per element issued as packed fp32
// pairs, pairwise accumulation, packed bf16 max.
#pragma once

#include "common.cuh"

namespace pspec {

// ---- vector maxima ----------------------------------------------------------------------
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float vec_max(const uint4& v, BF16Tag) {
  uint32_t m = bmax2(bmax2(v.x, v.y), bmax2(v.z, v.w));
  return fmaxf(bf16_lo(m), bf16_hi(m));
}

__device__ __forceinline__ float vec_max(const uint4& v, F32Tag) {
  return fmaxf(fmax3(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z)),
               __uint_as_float(v.w));
}

// ---- online softmax normaliser (base-2 units, see MS) ------------------------------------

// Terms 2^(x * kLog2e - m) of one vector, added pairwise into (a0, a1).
template <typename Tag>
__device__ __forceinline__ void add_terms(const uint4& v, float m, float& a0, float& a1) {
  constexpr int W = Tag::kVec;
  float x[W];
  unpack(v, x, Tag{});
#pragma unroll
  for (int j = 0; j < W; j += 2) {
    float t0, t1;
    ffma2(t0, t1, x[j], x[j + 1], kLog2e, -m);
    fadd2(a0, a1, ex2(t0), ex2(t1));
  }
}

// Running state of one thread: (m, s) plus two pending accumulators that share m.
struct MSAcc {
  MS ms;
  float a0, a1;
};

__device__ __forceinline__ MSAcc msacc_init() { return MSAcc{MS{-INFINITY, 0.f}, 0.f, 0.f}; }

// Raise the reference m to cover a batch whose largest logit is bmax; false when the batch
// holds nothing but -inf.  Raises are rare once the first vectors are in.
__device__ __forceinline__ bool msacc_raise(MSAcc& st, float bmax) {
  if (bmax == -INFINITY) return false;
  const float cand = bmax * kLog2e;
  if (cand > st.ms.m) {
    st.ms.s = st.ms.m == -INFINITY ? 0.f : (st.ms.s + st.a0 + st.a1) * ex2(st.ms.m - cand);
    st.a0 = st.a1 = 0.f;
    st.ms.m = cand;
  }
  return true;
}

// Fold U vectors: one reference check for the whole batch, then the terms.
template <typename Tag, int U>
__device__ __forceinline__ void consume_ms_batch(const uint4 (&v)[U], MSAcc& st) {
  float bm = vec_max(v[0], Tag{});
#pragma unroll
  for (int u = 1; u < U; ++u) bm = fmaxf(bm, vec_max(v[u], Tag{}));
  if (!msacc_raise(st, bm)) return;
#pragma unroll
  for (int u = 0; u < U; ++u) add_terms<Tag>(v[u], st.ms.m, st.a0, st.a1);
}

template <typename Tag>
__device__ __forceinline__ void consume_ms(const uint4& v, MSAcc& st) {
  if (!msacc_raise(st, vec_max(v, Tag{}))) return;
  add_terms<Tag>(v, st.ms.m, st.a0, st.a1);
}

// One scalar logit (unaligned heads, ragged tails).
__device__ __forceinline__ void consume_one(float x, MSAcc& st) {
  if (!msacc_raise(st, x)) return;
  st.a0 += ex2(fmaf(x, kLog2e, -st.ms.m));
}

__device__ __forceinline__ MS msacc_final(const MSAcc& st) {
  return MS{st.ms.m, st.ms.m == -INFINITY ? 0.f : st.ms.s + (st.a0 + st.a1)};
}

// ---- the draw ---------------------------------------------------------------------------
// The row a draw samples from: r(t) = max(0, p(t) - q(t)) when resid, else p(t), with
// p = 2^(x * kLog2e - mt) * inv_st and q likewise (fp32; mt and mq in base-2 units).
struct DrawRow {
  const void* trow;
  const void* qrow;
  float mt, inv_st, mq, inv_sq;
  bool resid;
};


// r of eight consecutive elements, computed on packed fp32 pairs.  Every pass over the
// same elements (tile sums, rescans) goes through this function, so all of them see
// bit-identical values.
__device__ __forceinline__ void fmul2(float& d0, float& d1, float a0, float a1, float b) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b));
}

__device__ __forceinline__ void draw_r8(const DrawRow& D, const float (&xt)[8], const float (&xq)[8],
                                        float (&r)[8]) {
  if (D.mt == -INFINITY) {
#pragma unroll
    for (int j = 0; j < 8; ++j) r[j] = 0.f;
    return;
  }
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    float a0, a1;
    ffma2(a0, a1, xt[j], xt[j + 1], kLog2e, -D.mt);        // -inf logits give 2^-inf = 0
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

// ---- argmax over 16-byte vectors: the vector's max on packed pairs, and only a vector
// that beats the running best is unpacked to find the first position of its max.
template <typename Tag>
__device__ __forceinline__ void take_first_max(const uint4& v, float vmax, long long idx0, VI& best) {
  constexpr int W = Tag::kVec;
  float x[W];
  unpack(v, x, Tag{});
  int j = 0;
#pragma unroll
  for (int t = W - 1; t >= 0; --t)
    if (x[t] == vmax) j = t;
  best.v = vmax;
  best.i = (int)(idx0 + j);
}

// Fold one vector starting at element idx0 into a running argmax (lowest index on ties,
// provided the caller feeds each thread's vectors in increasing index order).
template <typename Tag>
__device__ __forceinline__ void consume_argmax(const uint4& v, long long idx0, VI& best) {
  const float vmax = vec_max(v, Tag{});
  if (vmax > best.v) take_first_max<Tag>(v, vmax, idx0, best);
}

}  // namespace pspec
