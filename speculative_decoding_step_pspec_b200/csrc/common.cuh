// common.cuh -- device helpers shared by the libpspec kernels (sm_100a).
//
// Streaming loads, bf16 unpacking, the base-2 exponential used by the softmax sweeps, and
// the warp / CTA reductions.  Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pspec.h"

namespace pspec {

constexpr int kThreads = 256;            // CTA size of every sweep kernel
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kNoIndex = 0x7fffffff;     // "no element seen" in an argmax partial

// ---------------------------------------------------------------------------------------
// Loads.  Logits are read exactly once per sweep: the non-coherent path with no L1
// allocation keeps L1 free for the small per-sequence tables.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// Reads of data written by other CTAs of the same launch (L2 only, bypassing L1).
// Trivially-copyable records of 8 or 16*n bytes are moved as 64/128-bit words.
template <typename T>
__device__ __forceinline__ T ld_cg(const T* p) {
  static_assert(sizeof(T) == 4 || sizeof(T) == 8 || sizeof(T) % 16 == 0, "ld_cg size");
  T out;
  if constexpr (sizeof(T) == 4) {
    unsigned w = __ldcg(reinterpret_cast<const unsigned*>(p));
    memcpy(&out, &w, 4);
  } else if constexpr (sizeof(T) == 8) {
    unsigned long long w = __ldcg(reinterpret_cast<const unsigned long long*>(p));
    memcpy(&out, &w, 8);
  } else {
    int4 w[sizeof(T) / 16];
#pragma unroll
    for (int k = 0; k < (int)(sizeof(T) / 16); ++k) w[k] = __ldcg(reinterpret_cast<const int4*>(p) + k);
    memcpy(&out, w, sizeof(T));
  }
  return out;
}

// The thread-block cluster barrier in two halves: arrive (release: this thread's earlier
// shared-memory writes become visible to the cluster) and wait (acquire), so that a thread
// can issue independent work between them.  Every thread of every CTA of the cluster
// alternates arrive and wait, whole warps at a time.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// Element access.
struct F32Tag { using elem = float; static constexpr int kVec = 4; };
struct BF16Tag { using elem = uint16_t; static constexpr int kVec = 8; };

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float load_scalar(const float* base, long long idx) {
  return __ldg(base + idx);
}
__device__ __forceinline__ float load_scalar(const uint16_t* base, long long idx) {
  return __uint_as_float(((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(base) + idx)) << 16);
}

// Unpack one 16-byte vector into kVec floats (exact for both dtypes).
__device__ __forceinline__ void unpack(const uint4& v, float (&x)[4], F32Tag) {
  x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
  x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ void unpack(const uint4& v, float (&x)[8], BF16Tag) {
  x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
  x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z); x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}

// ---------------------------------------------------------------------------------------
// 2^x on the SFU (the hardware ex2.approx instruction, flush-to-zero below 2^-126).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------------------
// Packed fp32 pairs (sm_100): (d0, d1) = (a0, a1) * b + c and (d0, d1) += (a0, a1), one
// instruction each.
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}

__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(d0), "f"(d1), "f"(a0), "f"(a1));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ---------------------------------------------------------------------------------------
// Softmax normaliser partials in base-2 units: (m, s) stands for s * 2^m with
// s = sum over its elements of 2^(x * kLog2e - m).  Forming every exponent as one fused
// multiply-add x * kLog2e - m (instead of (x - m) * log2 e) halves the arithmetic per
// logit; the double-precision merges convert back with the same constant, so the result
// is the softmax of x * (kLog2e ln 2), within 1.4e-8 of the softmax of x.  A pair with
// m = -inf holds no mass.
struct MS {
  float m;
  float s;
};

__device__ __forceinline__ MS ms_merge(MS a, MS b) {
  float M = fmaxf(a.m, b.m);
  if (M == -INFINITY) return MS{-INFINITY, 0.f};
  float sa = a.m == -INFINITY ? 0.f : a.s * ex2(a.m - M);
  float sb = b.m == -INFINITY ? 0.f : b.s * ex2(b.m - M);
  return MS{M, sa + sb};
}

__device__ __forceinline__ MS warp_merge_ms(MS v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    MS w{__shfl_xor_sync(0xffffffffu, v.m, o), __shfl_xor_sync(0xffffffffu, v.s, o)};
    v = ms_merge(v, w);
  }
  return v;
}

// (value, index) argmax pairs: larger value wins, the lower index wins ties.
struct VI {
  float v;
  int i;
};

__device__ __forceinline__ bool vi_better(VI a, VI b) {
  return a.v > b.v || (a.v == b.v && a.i < b.i);
}

__device__ __forceinline__ VI warp_argmax(VI a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    VI b{__shfl_xor_sync(0xffffffffu, a.v, o), __shfl_xor_sync(0xffffffffu, a.i, o)};
    if (vi_better(b, a)) a = b;
  }
  return a;
}

__device__ __forceinline__ void set_err(int32_t* err, int bits) {
  if (bits) atomicOr(reinterpret_cast<int*>(err), bits);
}

// Sequence i's own draft count K_i ("dynamic draft length"): k_len[i], or K when k_len is
// NULL; a value outside [0, K] is clamped into it and sets PSPEC_DEVERR_KLEN_RANGE in *eb.
__device__ __forceinline__ int draft_count(const int32_t* k_len, int i, int K, int* eb) {
  if (!k_len) return K;
  int k = __ldg(k_len + i);
  if (k < 0 || k > K) {
    *eb |= PSPEC_DEVERR_KLEN_RANGE;
    k = k < 0 ? 0 : K;
  }
  return k;
}

// ---------------------------------------------------------------------------------------
// One segment [lo, hi) of a row, in element order per thread: an unaligned head with
// scalar loads (up to kVec-1 elements, only when the row does not start on 16 bytes), the
// 16-byte vectors with kUnroll loads in flight, then the ragged tail with scalar loads.
// vec(v, idx0) gets a vector starting at element idx0; one(x, idx) a single element.
// Each thread sees its elements in increasing index order.
template <typename Tag, int kUnroll, typename FVec, typename FOne>
__device__ __forceinline__ void sweep_segment(const typename Tag::elem* row, long long lo,
                                              long long hi, FVec vec, FOne one) {
  using elem = typename Tag::elem;
  constexpr int W = Tag::kVec;
  const int mis = (int)((reinterpret_cast<uintptr_t>(row + lo) & 15u) / sizeof(elem));
  const long long head = mis == 0 ? 0 : min((long long)(W - mis), hi - lo);
  if ((long long)threadIdx.x < head) one(load_scalar(row, lo + threadIdx.x), lo + threadIdx.x);
  const long long a0 = lo + head;
  const long long nvec = (hi - a0) / W;
  const uint4* vp = reinterpret_cast<const uint4*>(row + a0);
  for (long long v0 = threadIdx.x; v0 < nvec; v0 += (long long)kUnroll * kThreads) {
    uint4 buf[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long v = v0 + (long long)u * kThreads;
      if (v < nvec) buf[u] = ld_stream(vp + v);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long v = v0 + (long long)u * kThreads;
      if (v < nvec) vec(buf[u], a0 + v * W);
    }
  }
  const long long t = a0 + nvec * W + threadIdx.x;
  if (t < hi) one(load_scalar(row, t), t);
}

// The same walk with the vectors handed over in batches of U (one batch = the U vectors a
// thread has in flight together); a last incomplete batch goes vector by vector.
template <typename Tag, int U, typename FBatch, typename FVec, typename FOne>
__device__ __forceinline__ void sweep_segment_batched(const typename Tag::elem* row, long long lo,
                                                      long long hi, FBatch batch, FVec vec,
                                                      FOne one) {
  using elem = typename Tag::elem;
  constexpr int W = Tag::kVec;
  const int mis = (int)((reinterpret_cast<uintptr_t>(row + lo) & 15u) / sizeof(elem));
  const long long head = mis == 0 ? 0 : min((long long)(W - mis), hi - lo);
  if ((long long)threadIdx.x < head) one(load_scalar(row, lo + threadIdx.x), lo + threadIdx.x);
  const long long a0 = lo + head;
  const long long nvec = (hi - a0) / W;
  const uint4* vp = reinterpret_cast<const uint4*>(row + a0);
  long long v0 = threadIdx.x;
  for (; v0 + (long long)(U - 1) * kThreads < nvec; v0 += (long long)U * kThreads) {
    uint4 buf[U];
#pragma unroll
    for (int u = 0; u < U; ++u) buf[u] = ld_stream(vp + v0 + (long long)u * kThreads);
    batch(buf);
  }
  for (; v0 < nvec; v0 += kThreads) vec(ld_stream(vp + v0), a0 + v0 * W);
  const long long t = a0 + nvec * W + threadIdx.x;
  if (t < hi) one(load_scalar(row, t), t);
}

// Round x up to a multiple of a.
__host__ __device__ __forceinline__ long long round_up(long long x, long long a) {
  return (x + a - 1) / a * a;
}

}  // namespace pspec
