// plan.h -- launch plans and workspace layout of the verify kernels (host + device).
//
// A verify call sweeps rows x segments CTAs.  The plan fixes the segment length (a
// multiple of 8 elements, so every segment starts on a 16-byte boundary for both dtypes),
// the resample tiling, and the byte offsets of each region of the caller's workspace.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace pspec {

constexpr int kNumSMs = 148;             // B200
constexpr int kDrawTile = 256;           // draw tile: one warp, 32 lanes x 8 elements
// Segments of at least 8192 elements (four 16-byte vectors per thread for bf16): at small
// batches the sweep then launches a few CTAs per SM instead of many one-vector CTAs
// (measured on B200, one sequence of V=201088: 2.5 CTAs/SM of 16 KB each beat 10 of 4 KB).
constexpr long long kSegMin = 8192;
constexpr long long kSegMax = 65536;     // bounds the tail of the last wave
#ifndef PSPEC_TARGET_CTAS_PER_SM
#define PSPEC_TARGET_CTAS_PER_SM 32         // draft sampling: segments per row
#endif
// The verify sweep aims at about four CTAs per SM: fewer, longer segments cost fewer CTA
// starts and fewer partials for each sequence's last CTA to merge.  Measured on B200 (step
// time, L2 flushed): 4 sequences 0.038 -> 0.034 ms, 16 sequences 0.058 -> 0.052 ms, 64
// sequences 0.093 -> 0.087 ms against 32 CTAs per SM; one sequence unchanged (the 8192-
// element minimum decides there) and 1024 sequences unchanged (the 65536-element maximum).
#ifndef PSPEC_SWEEP_CTAS_PER_SM
#define PSPEC_SWEEP_CTAS_PER_SM 4
#endif
#ifndef PSPEC_DRAW_CTAS_PER_SM
#define PSPEC_DRAW_CTAS_PER_SM 1      // separate draw launch: about one CTA per SM, at least
#endif                                // kDrawTilesPerCta tiles per CTA (batches of one: 6)
constexpr int kTargetCtas = kNumSMs * PSPEC_TARGET_CTAS_PER_SM;
constexpr int kSweepTargetCtas = kNumSMs * PSPEC_SWEEP_CTAS_PER_SM;
constexpr int kResampleTargetCtas = kNumSMs * PSPEC_DRAW_CTAS_PER_SM;
constexpr int kDrawTilesPerCta = 64;     // separate draw launch: at most 8 tiles per warp
// Automatic path selection: the early exit from kEarlyExitMinB sequences on for the
// rejection rule and from kEarlyExitGreedyMinB on for the greedy rule, the full sweep below.
// A small batch reads few bytes either way; there the early exit's chain of positions (one
// round of loads, a cluster barrier and a decision per position, ~9 us each on a 16-CTA
// cluster) costs more than the sweep, which reads every row at once on all SMs.  Measured
// crossovers (prepared step calls, L2 flushed): rejection between 128 and 192 sequences
// (V = 201088) and between 128 and 160 (V = 151936); greedy at 64-96 and 48-64.  At one
// sequence the sweep's 0.032 ms is constant while the early exit's runs from 0.029 ms (a
// rejection at position 0) to 0.070 ms (five acceptances): 0.044 ms averaged over 16 seeds.
constexpr int kEarlyExitMinB = 160;
constexpr int kEarlyExitGreedyMinB = 64;
// CTAs per sequence on the early-exit path from kEarlyExitSmallB sequences on.
#ifndef PSPEC_EE_CLUSTER
#define PSPEC_EE_CLUSTER 4
#endif
constexpr int kEarlyExitCluster = PSPEC_EE_CLUSTER;
// Below this many sequences the automatic cluster is wider (16, 12 or 8; see the rule in
// api.cu): with 4, a batch of 64 fills only 256 CTA slots of ~900.
constexpr int kEarlyExitSmallB = 128;
constexpr int kStepFuseMaxB = 256;       // automatic step fusion below this many sequences

// Early exit, large batches: the last B/8 sequences, at most 96 for the rejection rule and
// 64 for the greedy rule's shorter chains, go to a second launch of
// kEarlyExitTailCluster-CTA clusters that fills the SMs as the first launch drains.
// (Measured: at 1024 sequences 96 against 64 or 160; at 256, where the first launch's
// clusters nearly all fit at once, 32 against 64 or 96.)
#ifndef PSPEC_EE_TAIL_SEQS
#define PSPEC_EE_TAIL_SEQS 96
#endif
#ifndef PSPEC_EE_GREEDY_TAIL_SEQS
#define PSPEC_EE_GREEDY_TAIL_SEQS 64
#endif
#ifndef PSPEC_EE_TAIL_CLUSTER
#define PSPEC_EE_TAIL_CLUSTER 8
#endif
constexpr int kEarlyExitTailCluster = PSPEC_EE_TAIL_CLUSTER;
inline int early_exit_tail(long long B, bool rejection) {
  const long long X = rejection ? PSPEC_EE_TAIL_SEQS : PSPEC_EE_GREEDY_TAIL_SEQS;
  return (int)(B / 8 < X ? B / 8 : X);
}

// Per-(row, segment) partial of the greedy sweep.
struct GreedyPart {
  float v;   // best value
  int i;     // its token id (kNoIndex when the segment is empty)
  float m;   // running max of the segment (lse)
  float s;   // sum of exp(x - m) over the segment (lse)
};

// Per-(row, segment) partial of the rejection sweep.
struct RejPart {
  float m;
  float s;
};

// Per-sequence result of the rejection sweep, read by the resample kernel.
struct SeqInfo {
  double mt, st;   // max and sum-exp of target row a_i
  double mq, sq;   // the same for draft row a_i (unused when a_i = K)
  int a;           // accepted drafts a_i
  int kn;          // the sequence's own draft count K_i
  int pad[2];
};

struct VerifyPlan {
  int rows;               // rows swept per sequence: K+1 (greedy) or 2K+1 (rejection)
  int S;                  // segments per row
  long long seg;          // elements per segment
  int tiles;              // draw tiles per row
  int tiles_per_chunk;    // draw tiles per CTA of the separate draw launch
  int C;                  // CTAs per sequence of the separate draw launch
  size_t off_part;        // partials [B*rows*S]
  size_t off_seq;         // SeqInfo[B]
  size_t off_tiles;       // double[B*tiles]
  size_t bytes;           // scratch bytes (the zero area comes on top, see zero_area)
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Words that must be zero when a call starts (the sweep's per-sequence tickets) live at
// the END of the caller's workspace, and scratch (partials, statistics, tile sums) grows
// from its start.  The tickets are laid out backwards from the end, one line of
// kLineWords words per sequence, so that their addresses depend on neither B nor K: a call
// with a smaller batch finds every ticket a larger call left at zero, and its scratch never
// reaches them.
constexpr int kLineWords = 2;
constexpr size_t kLineBytes = kLineWords * sizeof(int32_t);
enum : int {
  kZwSCnt = 0,      // sweep ticket
  kZwSCnt2 = 1,     // sweep draw ticket
};

// Bytes of zero area for B sequences (with slack for aligning the end down to 256 bytes).
inline size_t zero_area_bytes(long long B) {
  return ((size_t)B * kLineBytes + 255) / 256 * 256 + 256;
}

struct ZeroArea {
  int32_t* line0;            // word 0 of line 0; line j starts kLineWords * j words lower
  char* lowest;              // first byte of line B-1 (scratch must end at or below it)
};

inline ZeroArea zero_area(void* ws, size_t bytes, long long B) {
  const uintptr_t end = (reinterpret_cast<uintptr_t>(ws) + bytes) & ~uintptr_t(255);
  ZeroArea z;
  z.line0 = reinterpret_cast<int32_t*>(end - kLineBytes);
  z.lowest = reinterpret_cast<char*>(end) - (size_t)(B > 0 ? B : 1) * kLineBytes;
  return z;
}

// Entry i of a zero-area column (col = line0 + word): entries run backwards, a line apart.
__host__ __device__ __forceinline__ int32_t* zcol(int32_t* col, long long i) {
  return col - i * kLineWords;
}
// Entry r of a plain backward array ending at `end` (the sampling tickets).
__host__ __device__ __forceinline__ int32_t* zrow(int32_t* end, long long r) { return end - 1 - r; }

// seg_override > 0 forces the segment length (rounded up to a multiple of 8).
inline VerifyPlan make_verify_plan(int B, int K, int V, int rejection, long long seg_override) {
  VerifyPlan p{};
  p.rows = rejection ? 2 * K + 1 : K + 1;
  long long rows_total = (long long)B * p.rows;
  long long s_lo = (V + kSegMax - 1) / kSegMax;
  long long s_hi = (V + kSegMin - 1) / kSegMin;
  if (s_hi < 1) s_hi = 1;
  long long S = rows_total > 0 ? (kSweepTargetCtas + rows_total - 1) / rows_total : 1;
  if (S < s_lo) S = s_lo;
  if (S > s_hi) S = s_hi;
  if (S < 1) S = 1;
  long long seg = (V + S - 1) / S;
  if (seg_override > 0) seg = seg_override;
  seg = (seg + 7) / 8 * 8;
  p.seg = seg;
  p.S = (int)((V + seg - 1) / seg);
  p.tiles = (V + kDrawTile - 1) / kDrawTile;
  int C = B > 0 ? (kResampleTargetCtas + B - 1) / B : 1;
  int c_lo = (p.tiles + kDrawTilesPerCta - 1) / kDrawTilesPerCta;
  if (C < c_lo) C = c_lo;
  if (C > p.tiles) C = p.tiles;
  if (C < 1) C = 1;
  p.tiles_per_chunk = (p.tiles + C - 1) / C;
  p.C = (p.tiles + p.tiles_per_chunk - 1) / p.tiles_per_chunk;

  size_t off = 0;
  p.off_part = off;
  size_t part_sz = rejection ? sizeof(RejPart) : sizeof(GreedyPart);
  off = align256(off + part_sz * (size_t)B * p.rows * p.S);
  p.off_seq = off;
  off = align256(off + (rejection ? sizeof(SeqInfo) * (size_t)B : 0));
  p.off_tiles = off;
  off = align256(off + (rejection ? sizeof(double) * (size_t)B * p.tiles : 0));
  p.bytes = off;
  return p;
}

// Early-exit verify: one cluster of G CTAs per sequence, each CTA streaming a 1/G slice
// of the position's rows.  Needs V a multiple of 8 and 16-byte aligned rows; the slice
// must hold at most kMaxSliceTiles 256-element tiles.
constexpr int kMaxSliceTiles = 1024;

struct EarlyExitPlan {
  bool ok;
  int G;
  long long vs;
};

inline EarlyExitPlan make_early_exit_plan(int V, int G) {
  EarlyExitPlan p{};
  if (V % 8 != 0) return p;
  p.G = G;
  p.vs = ((long long)V + G - 1) / G;
  p.vs = (p.vs + 7) / 8 * 8;
  p.ok = (p.vs + 255) / 256 <= kMaxSliceTiles;
  return p;
}

// Draft sampling: rows x S CTAs over chunks of 32 lanes x kSampleGroups(dtype) groups of 8
// elements (2048 bf16 / 1024 fp32 elements: eight 16-byte loads per lane), each warp taking
// every eighth chunk of its CTA's segment; workspace = tickets + two partials per chunk.
inline int sample_chunk_elems(pspec_dtype dt) { return dt == PSPEC_BF16 ? 2048 : 1024; }

struct SamplePlan {
  int tiles, tiles_per_seg, S;    // chunks per row, chunks per CTA, CTAs per row
  size_t off_parts, off_maxes;    // scratch, from the start of the workspace
  size_t scratch;                 // scratch bytes
  size_t bytes;                   // scratch + tickets at the end (one int per row) + slack
};

inline SamplePlan make_sample_plan(long long rows, int V, int chunk_elems) {
  SamplePlan p{};
  p.tiles = (int)(((long long)V + chunk_elems - 1) / chunk_elems);
  long long S = rows > 0 ? (kTargetCtas + rows - 1) / rows : 1;
  const long long s_hi = (p.tiles + kWarps - 1) / kWarps;   // at least one chunk per warp
  if (S > s_hi) S = s_hi;
  if (S < 1) S = 1;
  p.tiles_per_seg = (int)((p.tiles + S - 1) / S);
  p.S = (p.tiles + p.tiles_per_seg - 1) / p.tiles_per_seg;
  size_t off = 0;
  p.off_parts = off;
  off = align256(off + 8 * (size_t)rows * p.tiles);
  p.off_maxes = off;
  off = align256(off + 8 * (size_t)rows * p.tiles);
  p.scratch = off;
  p.bytes = off + (sizeof(int32_t) * (size_t)rows + 255) / 256 * 256 + 256;
  return p;
}

}  // namespace pspec
