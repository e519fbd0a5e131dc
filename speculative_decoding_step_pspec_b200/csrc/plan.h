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
constexpr long long kSegMin = 2048;      // one 16-byte vector per thread (bf16)
constexpr long long kSegMax = 65536;     // bounds the tail of the last wave
constexpr int kTargetCtas = kNumSMs * 32;
constexpr int kResampleTargetCtas = kNumSMs * 8;
constexpr int kDrawTilesPerCta = 64;     // separate draw launch: at most 8 tiles per warp
constexpr int kEarlyExitMinB = 64;       // automatic path: early exit from this many sequences
constexpr int kEarlyExitCluster = 4;     // CTAs per sequence on the early-exit path

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
  int pad[3];
};

struct VerifyPlan {
  int rows;               // rows swept per sequence: K+1 (greedy) or 2K+1 (rejection)
  int S;                  // segments per row
  long long seg;          // elements per segment
  int tiles;              // draw tiles per row
  int tiles_per_chunk;    // draw tiles per CTA of the separate draw launch
  int C;                  // CTAs per sequence of the separate draw launch
  size_t off_cnt;         // int32[B]  sweep tickets
  size_t off_cnt2;        // int32[B]  resample tickets
  size_t off_part;        // partials [B*rows*S]
  size_t off_seq;         // SeqInfo[B]
  size_t off_tiles;       // double[B*tiles]
  size_t bytes;           // total
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// seg_override > 0 forces the segment length (rounded up to a multiple of 8).
inline VerifyPlan make_verify_plan(int B, int K, int V, int rejection, long long seg_override) {
  VerifyPlan p{};
  p.rows = rejection ? 2 * K + 1 : K + 1;
  long long rows_total = (long long)B * p.rows;
  long long s_lo = (V + kSegMax - 1) / kSegMax;
  long long s_hi = (V + kSegMin - 1) / kSegMin;
  if (s_hi < 1) s_hi = 1;
  long long S = rows_total > 0 ? (kTargetCtas + rows_total - 1) / rows_total : 1;
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
  p.off_cnt = off;
  off = align256(off + sizeof(int32_t) * (size_t)B);
  p.off_cnt2 = off;
  off = align256(off + (rejection ? sizeof(int32_t) * (size_t)B : 0));
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
  size_t off_cnt, off_parts, off_maxes, bytes;
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
  p.off_cnt = off;
  off = align256(off + sizeof(int32_t) * (size_t)rows);
  p.off_parts = off;
  off = align256(off + 8 * (size_t)rows * p.tiles);
  p.off_maxes = off;
  off = align256(off + 8 * (size_t)rows * p.tiles);
  p.bytes = off;
  return p;
}

}  // namespace pspec
