// noalloc.cu -- greedy verification for callers that cannot allocate device memory.
//
// pspec_verify_greedy needs a caller-provided scratch workspace (per-sequence tickets and
// per-segment partials).  Some callers have no way to provide one: a serving engine that
// reserves nearly all of HBM for its KV cache at start-up and hands memory out only
// through its own block pool, a host program that links only this C library and has no
// device allocator of its own, or a latency-critical path where cudaMalloc's implicit
// device synchronisation is not acceptable.  This file gives them the same kernel with
// its scratch in a fixed file-scope device array, so nobody allocates anything per call.
//
// The array is kNoAllocScratchBytes (4 MiB).  Every GPU that loads the library keeps it
// until the process exits.  All calls on a device share it and it keeps the last call's
// contents, so the tickets are cleared at the start of every call, and two calls whose
// executions overlap on the GPU (on different streams, or on different host threads
// with no ordering between them) race on it.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace pspec {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// In host code `g_noalloc_scratch` names a host-side stand-in, not device memory: its
// device address has to be looked up once per device, with that device current.
constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

cudaError_t scratch_of_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace pspec

extern "C" pspec_status pspec_verify_greedy_noalloc(const pspec_verify_args* a,
                                                    cudaStream_t stream) {
  using namespace pspec;
  if (!a) return PSPEC_ERR_INVALID_ARG;
  if (a->B < 0 || a->K < 1 || a->V < 1 || a->ld < a->V) return PSPEC_ERR_INVALID_ARG;
  if (a->K > PSPEC_MAX_K) return PSPEC_ERR_UNSUPPORTED;
  if (a->dtype != PSPEC_F32 && a->dtype != PSPEC_BF16) return PSPEC_ERR_INVALID_ARG;
  if (!a->err) return PSPEC_ERR_INVALID_ARG;
  if (a->B == 0) return PSPEC_OK;
  if (!a->target_logits || !a->draft_tokens || !a->out_tokens || !a->accepted_len || !a->bonus)
    return PSPEC_ERR_INVALID_ARG;
  if (!aligned_to(a->target_logits, a->dtype == PSPEC_BF16 ? 2 : 4)) return PSPEC_ERR_INVALID_ARG;

  // Always the automatic segment length: the scratch bound must not move with tuning.
  const VerifyPlan p = make_verify_plan(a->B, a->K, a->V, 0, 0);
  if (align256(p.bytes) + zero_area_bytes(a->B) > kNoAllocScratchBytes) return PSPEC_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  if (scratch_of_current_device(&scratch) != cudaSuccess) return PSPEC_ERR_CUDA;
  char* ws = static_cast<char*>(scratch);
  const ZeroArea z = zero_area(scratch, kNoAllocScratchBytes, a->B);
  // the tickets (the zero area's lines of sequences 0..B-1) must start at zero whatever an
  // earlier call left behind
  if (cudaMemsetAsync(z.lowest, 0, kLineBytes * (size_t)a->B, stream) != cudaSuccess)
    return PSPEC_ERR_CUDA;

  GreedyLaunch L{};
  L.B = a->B; L.K = a->K; L.V = a->V; L.ld = a->ld; L.dtype = a->dtype;
  L.S = p.S; L.seg = p.seg;
  L.target = a->target_logits;
  L.draft_tokens = a->draft_tokens;
  L.out_tokens = a->out_tokens;
  L.accepted_len = a->accepted_len;
  L.bonus = a->bonus;
  L.target_lse = a->target_lse;
  L.err = a->err;
  L.k_len = a->k_len;
  L.cnt = z.line0 + kZwSCnt;
  L.part = ws + p.off_part;
  return launch_greedy(L, stream) == cudaSuccess ? PSPEC_OK : PSPEC_ERR_CUDA;
}
