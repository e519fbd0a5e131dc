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
#include "build_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "verify_common.cuh"
#include "verify_draw.cuh"

namespace pspec {

namespace {

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
  // the draw launch is a programmatic dependent of this one: its CTAs may be placed once
  // every CTA of this grid has started, and wait for this grid's completion
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
      int t = atomicAdd(zcol(L.cnt, i), 1);
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
  // warp w merges rows w, w + 8, ...: lane t takes segments t, t + 32, ... (a fixed tree
  // order); the loads of all lanes are in flight together
  for (int r = warp; r < R; r += kWarps) {
    const RejPart* pr = part + (long long)r * L.S;
    float M = -INFINITY;
    for (int t = lane; t < L.S; t += 32) M = fmaxf(M, ld_cg(&pr[t].m));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    double S = 0.0;
    if (M != -INFINITY)
      for (int t = lane; t < L.S; t += 32) {
        const RejPart q = ld_cg(pr + t);
        if (q.m != -INFINITY) S += (double)q.s * exp2((double)q.m - (double)M);
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    if (lane == 0) {
      s_M[r] = M;
      s_S[r] = S;
    }
  }
  __syncthreads();
  if (warp != 0) return;

  {
  int eb = 0;
  const int Ki = draft_count(L.k_len, i, K, &eb);    // the sequence's own drafts
  int d = -1;
  bool bad = false, accept = false;
  double p = 0.0, q = 0.0;
  if (lane < K) {
    d = L.draft_tokens[(long long)i * K + lane];
    bad = lane < Ki && (d < 0 || d >= L.V);
    if (d >= 0 && d < L.V) {
      const double Mt = s_M[lane], St = s_S[lane];
      const double Mq = s_M[K + 1 + lane], Sq = s_S[K + 1 + lane];
      const float xt = load_scalar(sweep_row<elem>(L, i, lane), d);
      const float xq = load_scalar(sweep_row<elem>(L, i, K + 1 + lane), d);
      if (Mt != -INFINITY && xt != -INFINITY) p = exp2((double)xt * (double)kLog2e - Mt) / St;
      if (Mq != -INFINITY && xq != -INFINITY) q = exp2((double)xq * (double)kLog2e - Mq) / Sq;
      const double u = (double)L.uniforms[(long long)i * (K + 1) + lane];
      accept = lane < Ki && (q > 0.0 ? (u * q < p) : (p > 0.0));
    }
  }
  const unsigned mask = __ballot_sync(0xffffffffu, accept);
  const unsigned anybad = __ballot_sync(0xffffffffu, bad);
  int a = __ffs(~mask) - 1;              // first rejected draft
  if (a > Ki) a = Ki;
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
    si.mq = a < Ki ? s_M[K + 1 + a] : 0.0;
    si.sq = a < Ki ? s_S[K + 1 + a] : 1.0;
    si.a = a;
    si.kn = Ki;
    si.pad[0] = si.pad[1] = 0;
    reinterpret_cast<SeqInfo*>(L.seq)[i] = si;
    L.accepted_len[i] = a;
    set_err(L.err, eb | (anybad ? PSPEC_DEVERR_TOKEN_RANGE : 0));
    *zcol(L.cnt, i) = 0;
  }
  }  // warp 0
}

// The draw launch: B x C CTAs over the warp tiles of each sequence's row a_i.  With kFuse
// the CTA that draws a sequence's token also builds its draft span (the whole step).
template <typename Tag, bool kFuse>
__global__ void __launch_bounds__(kThreads)
rej_draw_kernel(const RejectionLaunch L) {
  using elem = typename Tag::elem;
  // the statistics launch's outputs (SeqInfo, tile plans) are read only after it completed;
  // then the stream's next programmatic launch (the step's build) may be placed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int K = L.K;
  const int i = blockIdx.x / L.C;
  const int c = blockIdx.x % L.C;
  const int warp = threadIdx.x >> 5;
  __shared__ int s_last;
  __shared__ DrawShared sh;

  const SeqInfo si = reinterpret_cast<const SeqInfo*>(L.seq)[i];  // previous launch
  DrawRow D = make_draw_row(L.target, L.draft, L.ld, K, si.kn, (int)sizeof(elem), i, si.a, si.mt,
                            si.st, si.mq, si.sq);
  double* ts = L.tile_sums + (long long)i * L.tiles;
  const long long t_lo = (long long)c * L.tiles_per_chunk;
  const long long t_hi = min((long long)L.tiles, t_lo + L.tiles_per_chunk);
  warp_tile_sums<Tag>(D, L.V, t_lo + warp, t_hi, kWarps, ts);
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int t = atomicAdd(zcol(L.cnt2, i), 1);
    s_last = (t == L.C - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  double Z;
  const int token = draw_finish<Tag>(D, L.V, L.tiles,
                                     (double)L.uniforms[(long long)i * (K + 1) + si.kn], ts, sh, &Z);
  __shared__ int s_tok;
  if (threadIdx.x == 0) {
    L.out_tokens[(long long)i * (K + 1) + si.a] = token;
    L.bonus[i] = token;
    if (L.residual_mass) L.residual_mass[i] = (float)Z;
    *zcol(L.cnt2, i) = 0;
    s_tok = token;
  }
  if constexpr (kFuse) {
    __syncthreads();
    int eb = 0;
    build_span(L.b, L.row_vecs, i, si.a, si.kn, s_tok, true, 0, 1, &eb);
    if (i == L.b.B - 1) build_tail_pad(L.b, 0, 1, &eb);
    set_err(L.b.err, eb);
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (L.fuse_build) {
    if (L.dtype == PSPEC_BF16) return cudaLaunchKernelEx(&cfg, rej_draw_kernel<BF16Tag, true>, L);
    return cudaLaunchKernelEx(&cfg, rej_draw_kernel<F32Tag, true>, L);
  }
  if (L.dtype == PSPEC_BF16) return cudaLaunchKernelEx(&cfg, rej_draw_kernel<BF16Tag, false>, L);
  return cudaLaunchKernelEx(&cfg, rej_draw_kernel<F32Tag, false>, L);
}

}  // namespace pspec
