// api.cu -- the C entry points of libpspec: host-side validation, workspace planning and
// kernel launches.  Every check here runs before any launch; a failed check returns a
// status and touches no device memory.
#include <stdint.h>
#include <stdlib.h>

#include "build_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"
#include "pspec.h"

namespace {

using namespace pspec;

// Process-wide defaults of the tuning options (pspec_set_*), used by calls whose arguments
// carry no pspec_options of their own.
pspec_options g_defaults = {0, 0, 0, 0, 0};
cudaEvent_t g_split_event = nullptr;
thread_local int t_last_launches = 0;
thread_local int t_last_path = 0;
thread_local int t_last_cluster = 0;   // CTAs per cluster of the last early-exit launch

// The options one call runs with: its own, or the process-wide defaults; out-of-range
// values read as automatic.
pspec_options resolve(const pspec_options* o) {
  pspec_options r = o ? *o : g_defaults;
  if (r.verify_path < 0 || r.verify_path > 2) r.verify_path = 0;
  if (!(r.cluster_size == 2 || r.cluster_size == 4 || r.cluster_size == 8 ||
        r.cluster_size == 12 || r.cluster_size == 16))
    r.cluster_size = 0;
  if (r.tail_split < 0) r.tail_split = -1;
  if (r.step_fusion < 0 || r.step_fusion > 2) r.step_fusion = 0;
  if (r.segment_elems < 0) r.segment_elems = 0;
  return r;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t elem_bytes(pspec_dtype d) { return d == PSPEC_BF16 ? 2 : 4; }

bool dtype_ok(pspec_dtype d) { return d == PSPEC_F32 || d == PSPEC_BF16; }

}  // namespace

namespace pspec {

pspec_status check_verify_host(const pspec_verify_args* a, bool rejection) {
  if (!a) return PSPEC_ERR_INVALID_ARG;
  if (a->B < 0 || a->K < 1 || a->V < 1 || a->ld < a->V) return PSPEC_ERR_INVALID_ARG;
  if (a->K > PSPEC_MAX_K) return PSPEC_ERR_UNSUPPORTED;
  if (!dtype_ok(a->dtype)) return PSPEC_ERR_INVALID_ARG;
  if (!a->err) return PSPEC_ERR_INVALID_ARG;
  if (a->B == 0) return PSPEC_OK;
  if (!a->target_logits || !a->draft_tokens || !a->out_tokens || !a->accepted_len || !a->bonus)
    return PSPEC_ERR_INVALID_ARG;
  if (rejection && (!a->draft_logits || !a->uniforms)) return PSPEC_ERR_INVALID_ARG;
  const size_t eb = elem_bytes(a->dtype);
  if (!aligned_to(a->target_logits, eb)) return PSPEC_ERR_INVALID_ARG;
  if (rejection && !aligned_to(a->draft_logits, eb)) return PSPEC_ERR_INVALID_ARG;
  // grid size: rows x segments must fit one launch
  const long long rows = (long long)a->B * (rejection ? 2 * a->K + 1 : a->K + 1);
  if (rows * ((a->V + kSegMin - 1) / kSegMin) >= 0x7fffffffLL) return PSPEC_ERR_UNSUPPORTED;
  return PSPEC_OK;
}

void record_last_call(int launches, int path) {
  t_last_launches = launches;
  t_last_path = path;
}

}  // namespace pspec

namespace {

// Host checks of a draft-batch construction; fills the launch descriptor on success.
pspec_status check_build(const pspec_build_args* a, BuildLaunch* L) {
  if (!a) return PSPEC_ERR_INVALID_ARG;
  if (a->B < 0 || a->K < 1 || a->H < 1 || a->block_size < 1 || a->max_blocks < 1 ||
      a->T_in < 0 || a->T_cap < 0)
    return PSPEC_ERR_INVALID_ARG;
  if (a->K > PSPEC_MAX_K) return PSPEC_ERR_UNSUPPORTED;
  if (!dtype_ok(a->hidden_dtype)) return PSPEC_ERR_INVALID_ARG;
  if ((long long)a->T_cap < (long long)a->T_in + (long long)a->B * (a->K - 1))
    return PSPEC_ERR_INVALID_ARG;
  if (!a->qsl_in || !a->err || !a->draft_tokens || !a->draft_pos || !a->slot_mapping ||
      !a->row_kind || !a->hidden_src || !a->qsl_out)
    return PSPEC_ERR_INVALID_ARG;
  if (a->B > 0 && (!a->verify_tokens || !a->verify_pos || !a->accepted_len || !a->bonus ||
                   !a->block_table || !a->seq_lens_out || !a->sample_idx))
    return PSPEC_ERR_INVALID_ARG;
  const bool hidden = a->draft_hidden != nullptr;
  if (hidden) {
    if (!a->h_shared || (a->T_in > 0 && !a->verify_hidden)) return PSPEC_ERR_INVALID_ARG;
    if (((long long)a->H * (long long)elem_bytes(a->hidden_dtype)) % 16 != 0)
      return PSPEC_ERR_INVALID_ARG;
    if (!aligned16(a->draft_hidden) || !aligned16(a->h_shared) ||
        (a->verify_hidden && !aligned16(a->verify_hidden)))
      return PSPEC_ERR_INVALID_ARG;
  }
  const long long meta_threads = (long long)a->T_cap + a->B + 1;
  const long long hid_rows = (long long)a->T_in + (long long)a->B * (a->K - 1);
  if ((meta_threads + kThreads - 1) / kThreads + (hid_rows + kWarps - 1) / kWarps >= 0x7fffffffLL)
    return PSPEC_ERR_UNSUPPORTED;
  *L = BuildLaunch{};
  L->a = *a;
  L->row_vecs = (long long)a->H * (long long)elem_bytes(a->hidden_dtype) / 16;
  L->meta_blocks = (int)((meta_threads + kThreads - 1) / kThreads);
  L->hid_rows = (int)hid_rows;
  return PSPEC_OK;
}

// Whether the automatic selection takes the early-exit path: from kEarlyExitMinB sequences on
// for the rejection rule, from kEarlyExitGreedyMinB on for the greedy rule (plan.h gives the
// measurements behind both).
bool early_exit_wanted(int B, bool rejection) {
  return B >= (rejection ? kEarlyExitMinB : kEarlyExitGreedyMinB);
}

// The early-exit cluster path, when the arguments allow it and the selection asks for it:
// returns true and sets *st when it handled the call.  With `fuse` non-null the same launch
// also builds the draft batch described there (from this call's accepted counts and bonus
// tokens).
bool try_early_exit(const pspec_verify_args* a, bool rejection, const pspec_options& o,
                    cudaStream_t stream, pspec_status* st, const BuildLaunch* fuse = nullptr) {
  const bool diagnostics = a->target_lse || a->draft_lse || a->p_at_draft || a->q_at_draft;
  if (o.verify_path == 1) return false;
  if (o.verify_path == 0 && (!early_exit_wanted(a->B, rejection) || diagnostics)) return false;
  const int eb = (int)elem_bytes(a->dtype);
  const bool aligned = aligned16(a->target_logits) && (!rejection || aligned16(a->draft_logits)) &&
                       (a->ld * eb) % 16 == 0;
  const bool v_ok = a->V % 8 == 0 && make_early_exit_plan(a->V, 16).ok;
  if (!v_ok || !aligned || diagnostics) {
    if (o.verify_path == 0) return false;
    *st = PSPEC_ERR_UNSUPPORTED;            // early exit forced on arguments it cannot take
    return true;
  }
  EarlyExitLaunch L{};
  L.B = a->B; L.K = a->K; L.V = a->V; L.ld = a->ld; L.dtype = a->dtype;
  L.rejection = rejection;
  L.target = a->target_logits;
  L.draft = a->draft_logits;
  L.draft_tokens = a->draft_tokens;
  L.uniforms = a->uniforms;
  L.out_tokens = a->out_tokens;
  L.accepted_len = a->accepted_len;
  L.bonus = a->bonus;
  L.residual_mass = rejection ? a->residual_mass : nullptr;
  L.err = a->err;
  L.k_len = a->k_len;
  if (fuse) {
    L.fuse_build = 1;
    L.b = fuse->a;
    L.row_vecs = fuse->row_vecs;
  }
  // Cluster size: kEarlyExitCluster from kEarlyExitSmallB sequences on.  Below, the rejection
  // rule takes the widest cluster (16, 12, 8) with which every sequence's cluster is
  // resident at once (a batch that needs a second round of clusters costs a second chain of
  // positions); the greedy rule, with less work per element, 8 (16 below 16 sequences).
  L.seq0 = 0;
  L.nseq = a->B;
  int G = o.cluster_size;
  if (G == 0) {
    G = kEarlyExitCluster;
    if (a->B < kEarlyExitSmallB && !rejection) {
      G = a->B < 16 ? 16 : 8;
    } else if (a->B < kEarlyExitSmallB) {
      for (const int cand : {16, 12, 8}) {
        const EarlyExitPlan pc = make_early_exit_plan(a->V, cand);
        if (!pc.ok) continue;
        L.G = cand;
        L.vs = pc.vs;
        if (early_exit_max_clusters(L) >= a->B) { G = cand; break; }
      }
    }
  }
  EarlyExitPlan ep = make_early_exit_plan(a->V, G);
  if (!ep.ok && o.cluster_size == 0) ep = make_early_exit_plan(a->V, 16);   // slices too long
  if (!ep.ok) {
    if (o.verify_path == 0) return false;
    *st = PSPEC_ERR_UNSUPPORTED;
    return true;
  }
  L.G = ep.G;
  L.vs = ep.vs;
  // The last X sequences go to a second launch of wider clusters that starts as the first
  // launch's clusters finish (programmatic dependent launch): the sequences that start last
  // then run their chains of rows twice as wide, which shortens the launch's tail.
  // Automatic: large batches on the large-batch width; a forced count: any narrower width.
  int X = 0;
  if (ep.G < kEarlyExitTailCluster && o.tail_split >= 0)
    X = o.tail_split > 0 ? o.tail_split
                         : (ep.G == kEarlyExitCluster && a->B >= kEarlyExitSmallB
                                ? early_exit_tail(a->B, rejection) : 0);
  X = X < a->B / 2 ? X : a->B / 2;
  const EarlyExitPlan et = make_early_exit_plan(a->V, kEarlyExitTailCluster);
  int launches = 1;
  cudaError_t ce;
  if (X > 0 && et.ok) {
    EarlyExitLaunch L2 = L;
    L.nseq = a->B - X;
    L.pdl = 1;
    L2.seq0 = a->B - X;
    L2.nseq = X;
    L2.G = kEarlyExitTailCluster;
    L2.vs = et.vs;
    L2.pdl = 2;
    ce = launch_early_exit(L, stream);
    if (ce == cudaSuccess) ce = launch_early_exit(L2, stream);
    launches = 2;
  } else {
    ce = launch_early_exit(L, stream);
  }
  if (ce != cudaSuccess) {
    *st = PSPEC_ERR_CUDA;
    return true;
  }
  if (rejection && g_split_event) cudaEventRecord(g_split_event, stream);
  t_last_launches = launches;
  t_last_path = 2;
  t_last_cluster = L.G;
  *st = PSPEC_OK;
  return true;
}

// The caller's workspace: 256-byte aligned, `scratch` bytes from its start and the zero area
// of B sequences below its (aligned) end; *z receives the zero area.
pspec_status check_workspace(void* ws, size_t bytes, size_t scratch, long long B, ZeroArea* z) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PSPEC_ERR_WORKSPACE;
  if (bytes < align256(scratch) + zero_area_bytes(B)) return PSPEC_ERR_WORKSPACE;
  *z = zero_area(ws, bytes, B);
  if (static_cast<char*>(ws) + scratch > z->lowest) return PSPEC_ERR_WORKSPACE;
  return PSPEC_OK;
}

// Scratch the verify calls need below the zero area: the full sweep's plan (the early-exit
// path needs none), so that a workspace of pspec_verify_workspace_bytes serves every path
// and every call checks against the one size that function reports.
size_t verify_scratch_bytes(int B, int K, int V, int rejection, const pspec_options& o) {
  return align256(make_verify_plan(B, K, V, rejection, o.segment_elems).bytes);
}

}  // namespace

extern "C" {

size_t pspec_verify_workspace_bytes_opt(int B, int K, int V, int rejection,
                                        const pspec_options* options) {
  if (B < 0 || K < 1 || K > PSPEC_MAX_K || V < 1) return 0;
  return verify_scratch_bytes(B, K, V, rejection, resolve(options)) + zero_area_bytes(B);
}

size_t pspec_verify_workspace_bytes(int B, int K, int V, int rejection) {
  return pspec_verify_workspace_bytes_opt(B, K, V, rejection, nullptr);
}

}  // extern "C"

namespace {

// The greedy verify behind both entry points; `fuse` (may be null) is passed to the
// early-exit path, and *fused tells whether that launch also built the draft batch.
pspec_status verify_greedy_impl(const pspec_verify_args* a, void* workspace,
                                size_t workspace_bytes, cudaStream_t stream,
                                const BuildLaunch* fuse, bool* fused) {
  *fused = false;
  pspec_status st = check_verify_host(a, false);
  if (st != PSPEC_OK) return st;
  if (a->B == 0) { record_last_call(0, 0); return st; }
  const pspec_options o = resolve(a->options);
  const VerifyPlan p = make_verify_plan(a->B, a->K, a->V, 0, o.segment_elems);
  ZeroArea z;
  st = check_workspace(workspace, workspace_bytes, verify_scratch_bytes(a->B, a->K, a->V, 0, o), a->B, &z);
  if (st != PSPEC_OK) return st;
  if (try_early_exit(a, false, o, stream, &st, fuse)) {
    *fused = fuse != nullptr && st == PSPEC_OK;
    return st;
  }
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
  char* ws = static_cast<char*>(workspace);
  L.cnt = z.line0 + kZwSCnt;
  L.part = ws + p.off_part;
  if (fuse) {                                 // the deciding CTA of each sequence builds too
    L.fuse_build = 1;
    L.b = fuse->a;
    L.row_vecs = fuse->row_vecs;
  }
  if (launch_greedy(L, stream) != cudaSuccess) return PSPEC_ERR_CUDA;
  *fused = fuse != nullptr;
  record_last_call(1, 1);
  return PSPEC_OK;
}

// The rejection-rule verify behind both entry points (see verify_greedy_impl).
pspec_status verify_rejection_impl(const pspec_verify_args* a, void* workspace,
                                   size_t workspace_bytes, cudaStream_t stream,
                                   const BuildLaunch* fuse, bool* fused) {
  *fused = false;
  pspec_status st = check_verify_host(a, true);
  if (st != PSPEC_OK) return st;
  if (a->B == 0) { record_last_call(0, 0); return st; }
  const pspec_options o = resolve(a->options);
  const VerifyPlan p = make_verify_plan(a->B, a->K, a->V, 1, o.segment_elems);
  ZeroArea z;
  st = check_workspace(workspace, workspace_bytes, verify_scratch_bytes(a->B, a->K, a->V, 1, o), a->B, &z);
  if (st != PSPEC_OK) return st;
  if (try_early_exit(a, true, o, stream, &st, fuse)) {
    *fused = fuse != nullptr && st == PSPEC_OK;
    return st;
  }
  RejectionLaunch L{};
  L.B = a->B; L.K = a->K; L.V = a->V; L.ld = a->ld; L.dtype = a->dtype;
  L.S = p.S; L.seg = p.seg;
  L.tiles = p.tiles; L.tiles_per_chunk = p.tiles_per_chunk; L.C = p.C;
  L.target = a->target_logits;
  L.draft = a->draft_logits;
  L.draft_tokens = a->draft_tokens;
  L.uniforms = a->uniforms;
  L.out_tokens = a->out_tokens;
  L.accepted_len = a->accepted_len;
  L.bonus = a->bonus;
  L.target_lse = a->target_lse;
  L.draft_lse = a->draft_lse;
  L.p_at_draft = a->p_at_draft;
  L.q_at_draft = a->q_at_draft;
  L.residual_mass = a->residual_mass;
  L.err = a->err;
  L.k_len = a->k_len;
  char* ws = static_cast<char*>(workspace);
  L.cnt = z.line0 + kZwSCnt;
  L.cnt2 = z.line0 + kZwSCnt2;
  L.part = ws + p.off_part;
  L.seq = ws + p.off_seq;
  L.tile_sums = reinterpret_cast<double*>(ws + p.off_tiles);
  if (fuse) {                                 // the draw's deciding CTA builds too
    L.fuse_build = 1;
    L.b = fuse->a;
    L.row_vecs = fuse->row_vecs;
  }
  if (launch_rejection(L, stream, g_split_event) != cudaSuccess) return PSPEC_ERR_CUDA;
  *fused = fuse != nullptr;
  record_last_call(2, 1);
  return PSPEC_OK;
}

// One step: verify, then the draft batch from the verify's own accepted counts and bonus
// tokens (b's accepted_len / bonus must be NULL or those same arrays).
pspec_status step_impl(const pspec_verify_args* v, const pspec_build_args* b, bool rejection,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!v || !b) return PSPEC_ERR_INVALID_ARG;
  if (b->B != v->B || b->K != v->K) return PSPEC_ERR_INVALID_ARG;
  if ((b->accepted_len && b->accepted_len != v->accepted_len) || (b->bonus && b->bonus != v->bonus) ||
      (b->k_len && b->k_len != v->k_len))
    return PSPEC_ERR_INVALID_ARG;
  pspec_build_args bb = *b;
  bb.accepted_len = v->accepted_len;
  bb.bonus = v->bonus;
  bb.k_len = v->k_len;
  BuildLaunch BL;
  pspec_status st = check_build(&bb, &BL);
  if (st != PSPEC_OK) return st;
  // one launch for both halves where that measured faster: below kStepFuseMaxB sequences
  // the saved launch outweighs building each span at the end of its cluster's work
  const pspec_options o = resolve(v->options);
  const bool want_fuse = o.step_fusion == 1 || (o.step_fusion == 0 && v->B < kStepFuseMaxB);
  const BuildLaunch* fuse = want_fuse ? &BL : nullptr;
  bool fused = false;
  st = rejection ? verify_rejection_impl(v, workspace, workspace_bytes, stream, fuse, &fused)
                 : verify_greedy_impl(v, workspace, workspace_bytes, stream, fuse, &fused);
  if (st != PSPEC_OK || fused) return st;
  const int verify_launches = t_last_launches;
  if (launch_build(BL, stream) != cudaSuccess) return PSPEC_ERR_CUDA;
  t_last_launches = verify_launches + 1;
  return PSPEC_OK;
}

}  // namespace

extern "C" {

pspec_status pspec_verify_greedy(const pspec_verify_args* a, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
  bool fused;
  return verify_greedy_impl(a, workspace, workspace_bytes, stream, nullptr, &fused);
}

pspec_status pspec_verify_rejection(const pspec_verify_args* a, void* workspace,
                                    size_t workspace_bytes, cudaStream_t stream) {
  bool fused;
  return verify_rejection_impl(a, workspace, workspace_bytes, stream, nullptr, &fused);
}

pspec_status pspec_step_greedy(const pspec_verify_args* v, const pspec_build_args* b,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return step_impl(v, b, false, workspace, workspace_bytes, stream);
}

pspec_status pspec_step_rejection(const pspec_verify_args* v, const pspec_build_args* b,
                                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return step_impl(v, b, true, workspace, workspace_bytes, stream);
}

pspec_status pspec_build_draft_batch(const pspec_build_args* a, cudaStream_t stream) {
  BuildLaunch L;
  const pspec_status st = check_build(a, &L);
  if (st != PSPEC_OK) return st;
  if (launch_build(L, stream) != cudaSuccess) return PSPEC_ERR_CUDA;
  t_last_launches = 1;
  return PSPEC_OK;
}

size_t pspec_sample_workspace_bytes(int B, int K, int V) {
  if (B < 0 || K < 1 || V < 1) return 0;
  // sized for the smaller fp32 chunks, so one workspace serves either dtype
  return make_sample_plan((long long)B * K, V, sample_chunk_elems(PSPEC_F32)).bytes;
}

pspec_status pspec_sample_drafts(const pspec_sample_args* a, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
  if (!a) return PSPEC_ERR_INVALID_ARG;
  if (a->B < 0 || a->K < 1 || a->V < 1 || a->ld < a->V) return PSPEC_ERR_INVALID_ARG;
  if (!dtype_ok(a->dtype) || !a->err) return PSPEC_ERR_INVALID_ARG;
  if (a->B == 0) { t_last_launches = 0; return PSPEC_OK; }
  if (!a->logits || !a->draft_tokens) return PSPEC_ERR_INVALID_ARG;
  if (!aligned_to(a->logits, elem_bytes(a->dtype))) return PSPEC_ERR_INVALID_ARG;
  const long long rows = (long long)a->B * a->K;
  const SamplePlan p = make_sample_plan(rows, a->V, sample_chunk_elems(a->dtype));
  if (rows * p.S >= 0x7fffffffLL) return PSPEC_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < p.bytes)
    return PSPEC_ERR_WORKSPACE;
  // tickets at the aligned end, one per row, so calls with other batch sizes find them at 0
  int32_t* tickets_end = reinterpret_cast<int32_t*>(
      (reinterpret_cast<uintptr_t>(workspace) + workspace_bytes) & ~uintptr_t(255));
  SampleLaunch L{};
  L.rows = rows; L.V = a->V; L.ld = a->ld; L.dtype = a->dtype;
  L.tiles = p.tiles; L.tiles_per_seg = p.tiles_per_seg; L.S = p.S;
  L.logits = a->logits;
  L.uniforms = a->uniforms;
  L.tokens = a->draft_tokens;
  L.probs = a->q_at_draft;
  L.err = a->err;
  char* ws = static_cast<char*>(workspace);
  L.cnt = tickets_end;
  L.parts = ws + p.off_parts;
  L.maxes = ws + p.off_maxes;
  if (launch_sample(L, stream) != cudaSuccess) return PSPEC_ERR_CUDA;
  t_last_launches = 1;
  return PSPEC_OK;
}

const char* pspec_status_string(pspec_status s) {
  switch (s) {
    case PSPEC_OK: return "PSPEC_OK";
    case PSPEC_ERR_INVALID_ARG: return "PSPEC_ERR_INVALID_ARG";
    case PSPEC_ERR_UNSUPPORTED: return "PSPEC_ERR_UNSUPPORTED";
    case PSPEC_ERR_CUDA: return "PSPEC_ERR_CUDA";
    case PSPEC_ERR_WORKSPACE: return "PSPEC_ERR_WORKSPACE";
  }
  return "PSPEC_ERR_UNKNOWN";
}

int pspec_last_launches(void) { return t_last_launches; }

int pspec_last_verify_path(void) { return t_last_path; }
int pspec_last_cluster_size(void) { return t_last_cluster; }

void pspec_set_verify_path(int path) { g_defaults.verify_path = (path == 1 || path == 2) ? path : 0; }

void pspec_set_cluster_size(int G) {
  g_defaults.cluster_size = (G == 2 || G == 4 || G == 8 || G == 12 || G == 16) ? G : 0;
}

void pspec_set_step_fusion(int mode) { g_defaults.step_fusion = (mode == 1 || mode == 2) ? mode : 0; }
void pspec_set_tail_split(int n) { g_defaults.tail_split = n < 0 ? -1 : n; }

void pspec_set_segment_elems(long long elems) { g_defaults.segment_elems = elems > 0 ? elems : 0; }

void pspec_get_options(pspec_options* out) {
  if (out) *out = g_defaults;
}

void pspec_set_split_event(cudaEvent_t event) { g_split_event = event; }

}  // extern "C"
