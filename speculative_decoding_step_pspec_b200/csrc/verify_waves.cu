// verify_waves.cu -- rejection-rule verify in position waves (path 4).
//
// "Accept prefix; resample for rejected suffix" ("Capstone 14: speculative decoding
// inference server", section "Architecture"): rows after a sequence's first rejection
// never matter, so they are never read.  Where the early-exit path walks each sequence's
// positions inside one cluster, this path walks the positions of the whole batch in step:
//
//   wave k (one persistent launch per position k = 0..K): the sequences still undecided
//   at position k (all of them for k = 0, else the list wave k-1 appended) are cut into
//   units (sequence, row, segment) -- target row k and, while k < K_i, draft row k -- and
//   every CTA sweeps units with 16-byte loads into (max, sum exp) partials, like the full
//   sweep's statistics pass.  The CTA that completes a sequence's last unit (atomic ticket)
//   merges the partials in double and applies the rule at position k: an accepted draft is
//   written and the sequence appended to wave k+1's list; a rejection (or k = K_i) stops it
//   and records what the draw needs.  The segment length of a wave follows the number of
//   sequences in it, so that late waves with few sequences still fill the GPU.
//
//   the draw: the full sweep's draw launch, one flat pass over every sequence's row a_i.
//
// Waves are queued with programmatic dependent launch: each wave lets the next be placed
// while it runs, and every wave after the first waits (griddepcontrol.wait, the hardware
// grid dependency) for the previous one before reading its list.  No wave waits on another
// CTA.
#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "verify_common.cuh"

namespace pspec {

namespace {

struct WaveShared {
  MS ms[kWarps];
  double M[2], S[2];
  int last;
};

template <typename Tag>
__global__ void __launch_bounds__(kThreads) wave_kernel(const WaveLaunch L, const int k) {
  using elem = typename Tag::elem;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (k > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ WaveShared sh;
  const int K = L.K;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // sequences in this wave (each sequence is appended to a wave at most once, so at most B)
  const unsigned cnt = k == 0 ? (unsigned)L.B : *reinterpret_cast<volatile const unsigned*>(L.wave_cnt + k);
  const int n = cnt < (unsigned)L.B ? (int)cnt : L.B;
  // segments per row for this wave's n sequences (at least L.seg_min elements each)
  long long S = n > 0 ? (L.target_units + 2LL * n - 1) / (2LL * n) : 1;
  if (S > L.S_max) S = L.S_max;
  if (S < 1) S = 1;
  const long long seg = round_up((L.V + S - 1) / S, 8);
  S = (L.V + seg - 1) / seg;
  const long long units = 2LL * n * S;
  const int* list = L.lists + (long long)k * L.B;

  for (long long u = blockIdx.x; u < units; u += gridDim.x) {
    const int j = (int)(u / (2 * S));
    const int r = (int)((u / S) & 1);                        // 0: target row, 1: draft row
    const long long s = u % S;
    const int i = k == 0 ? j : list[j];
    int unused = 0;
    const int Ki = draft_count(L.k_len, i, K, &unused);
    MS ms{-INFINITY, 0.f};
    if (r == 0 || k < Ki) {                                  // draft row k exists for k < K_i
      const elem* row = r == 0
          ? static_cast<const elem*>(L.target) + ((long long)i * (K + 1) + k) * L.ld
          : static_cast<const elem*>(L.draft) + ((long long)i * K + k) * L.ld;
      const long long lo = s * seg;
      const long long hi = min((long long)L.V, lo + seg);
      MSAcc acc = msacc_init();
      sweep_segment_batched<Tag, 4>(
          row, lo, hi, [&](const uint4 (&v)[4]) { consume_ms_batch<Tag, 4>(v, acc); },
          [&](const uint4& v, long long) { consume_ms<Tag>(v, acc); },
          [&](float x, long long) { consume_one(x, acc); });
      ms = msacc_final(acc);
    }
    ms = warp_merge_ms(ms);
    if (lane == 0) sh.ms[warp] = ms;
    __syncthreads();
    if (warp == 0) {
      ms = lane < kWarps ? sh.ms[lane] : MS{-INFINITY, 0.f};
      ms = warp_merge_ms(ms);
      if (lane == 0) {
        reinterpret_cast<RejPart*>(L.part)[((long long)j * 2 + r) * L.S_max + s] = RejPart{ms.m, ms.s};
        __threadfence();
        const int t = atomicAdd(zcol(L.cnt, i), 1);
        sh.last = (t == 2 * S - 1);
      }
    }
    __syncthreads();
    if (sh.last) {
      __threadfence();
      // ---- the sequence's last unit: merge each row's partials (warp r, lanes over
      // segments, in double) and apply the rule at position k
      if (warp < 2) {
        const RejPart* pr = reinterpret_cast<const RejPart*>(L.part) + ((long long)j * 2 + warp) * L.S_max;
        float M = -INFINITY;
        for (long long t = lane; t < S; t += 32) M = fmaxf(M, ld_cg(&pr[t].m));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        double Sd = 0.0;
        if (M != -INFINITY)
          for (long long t = lane; t < S; t += 32) {
            const RejPart q = ld_cg(pr + t);
            if (q.m != -INFINITY) Sd += (double)q.s * exp2((double)q.m - (double)M);
          }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Sd += __shfl_xor_sync(0xffffffffu, Sd, o);
        if (lane == 0) {
          sh.M[warp] = M;
          sh.S[warp] = Sd;
        }
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int eb = 0;
        const int Kd = draft_count(L.k_len, i, K, &eb);
        bool accept = false;
        int d = -1;
        if (k < Kd) {
          d = L.draft_tokens[(long long)i * K + k];
          if (d >= 0 && d < L.V) {
            const elem* trow = static_cast<const elem*>(L.target) + ((long long)i * (K + 1) + k) * L.ld;
            const elem* qrow = static_cast<const elem*>(L.draft) + ((long long)i * K + k) * L.ld;
            const float xt = load_scalar(trow, d), xq = load_scalar(qrow, d);
            const double Mt = sh.M[0], St = sh.S[0], Mq = sh.M[1], Sq = sh.S[1];
            const double p = (Mt != -INFINITY && xt != -INFINITY)
                                 ? exp2((double)xt * (double)kLog2e - Mt) / St : 0.0;
            const double q = (Mq != -INFINITY && xq != -INFINITY)
                                 ? exp2((double)xq * (double)kLog2e - Mq) / Sq : 0.0;
            const double uu = (double)L.uniforms[(long long)i * (K + 1) + k];
            accept = q > 0.0 ? (uu * q < p) : (p > 0.0);
          }
        }
        if (accept) {
          L.out_tokens[(long long)i * (K + 1) + k] = d;
          const unsigned slot = atomicAdd(L.wave_cnt + k + 1, 1u);
          if (slot < (unsigned)L.B) L.lists[(long long)(k + 1) * L.B + slot] = i;
        } else {
          // stop at a_i = k: the draw samples the residual of row pair k, or the target
          // row K_i when every draft passed
          SeqInfo si;
          si.mt = sh.M[0];
          si.st = sh.S[0];
          si.mq = k < Kd ? sh.M[1] : 0.0;
          si.sq = k < Kd ? sh.S[1] : 1.0;
          si.a = k;
          si.kn = Kd;
          si.pad[0] = si.pad[1] = 0;
          reinterpret_cast<SeqInfo*>(L.seq)[i] = si;
          L.accepted_len[i] = k;
          for (int t = k + 1; t <= K; ++t) L.out_tokens[(long long)i * (K + 1) + t] = -1;
          for (int t = 0; t < Kd; ++t) {
            const int dt = L.draft_tokens[(long long)i * K + t];
            if (dt < 0 || dt >= L.V) eb |= PSPEC_DEVERR_TOKEN_RANGE;
          }
        }
        set_err(L.err, eb);
        *zcol(L.cnt, i) = 0;
      }
    }
    __syncthreads();                                         // sh is reused by the next unit
  }
  // the last CTA out of the last wave puts the wave counts back to zero
  if (k == K) {
    if (threadIdx.x == 0) {
      __threadfence();
      const unsigned e = atomicAdd(L.wave_cnt + K + 1, 1u);
      sh.last = (e == gridDim.x - 1);
    }
    __syncthreads();
    if (sh.last && threadIdx.x <= K + 1) L.wave_cnt[threadIdx.x] = 0;
  }
}

template <typename Tag>
cudaError_t launch_w(const WaveLaunch& L, cudaStream_t stream) {
  auto kern = wave_kernel<Tag>;
  static int per_sm[8] = {0};                                // per device
  static int sms[8] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int slot = dev >= 0 && dev < 8 ? dev : 0;
  if (per_sm[slot] == 0) {
    int nb = 0, n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, 0);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    per_sm[slot] = nb < 1 ? 1 : nb;
    sms[slot] = n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(per_sm[slot] * sms[slot]), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  for (int k = 0; k <= L.K; ++k) {
    cfg.attrs = attr;
    cfg.numAttrs = k == 0 ? 0 : 1;                           // wave 0 follows the stream
    e = cudaLaunchKernelEx(&cfg, kern, L, k);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_waves(const WaveLaunch& L, cudaStream_t stream) {
  return L.dtype == PSPEC_BF16 ? launch_w<BF16Tag>(L, stream) : launch_w<F32Tag>(L, stream);
}

}  // namespace pspec
