// noalloc.cu -- greedy verification for callers that cannot allocate device memory.
//
// pspec_verify_greedy needs a caller-provided scratch workspace (per-sequence tickets and
// per-segment partials).  Some callers have no way to provide one: a serving engine that
// reserves nearly all of HBM for its KV cache at start-up and hands memory out only
// through its own block pool, a host program that links only this C library and has no
// device allocator of its own, or a latency-critical path where cudaMalloc's implicit
// device synchronisation is not acceptable.  This file gives them the full-sweep greedy
// kernel with its scratch in a fixed file-scope device array, so nobody allocates anything
// per call.  The outputs are those of pspec_verify_greedy; the kernel is always the full
// sweep, whichever path pspec_verify_greedy would take.
//
// The array is kNoAllocScratchBytes (4 MiB).  Every GPU that loads the library keeps it
// until the process exits.  All calls on a device share it and it keeps the last call's
// contents, so the tickets are cleared at the start of every call, and two calls whose
// executions overlap on the GPU (on different streams, or on different host threads
// with no ordering between them) race on it.
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace pspec {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// In host code `g_noalloc_scratch` names a host-side stand-in, not device memory.  Its
// device address is looked up on every call, for the device and context current at the
// call: the lookup allocates nothing and is cheap, and an address cached across calls
// would go stale after cudaDeviceReset (which reloads the module) or under another context
// on the same device.
cudaError_t scratch_of_current_context(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace pspec

extern "C" pspec_status pspec_verify_greedy_noalloc(const pspec_verify_args* a,
                                                    cudaStream_t stream) {
  using namespace pspec;
  const pspec_status st = check_verify_host(a, false);
  if (st != PSPEC_OK) return st;
  if (a->B == 0) {
    record_last_call(0, 0);
    return PSPEC_OK;
  }

  // Always the automatic segment length: the scratch bound must not move with tuning.
  const VerifyPlan p = make_verify_plan(a->B, a->K, a->V, 0, 0);
  if (align256(p.bytes) + zero_area_bytes(a->B) > kNoAllocScratchBytes) return PSPEC_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  if (scratch_of_current_context(&scratch) != cudaSuccess) return PSPEC_ERR_CUDA;
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
  if (launch_greedy(L, stream) != cudaSuccess) return PSPEC_ERR_CUDA;
  record_last_call(1, 1);
  return PSPEC_OK;
}
