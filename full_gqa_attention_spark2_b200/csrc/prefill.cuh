// Prefill (flash attention over a chunk of queries): tile schedule, masks and
// constants shared by the sm_100a kernel in prefill2.cuh.
//
// A block owns one (sequence b, query head h, 128-query tile).  K/V tiles of
// 128 keys are visited in order: history tiles from the cache, then the
// chunk's own tiles.  Tiles that no query of the block can see are never
// loaded; only tiles that straddle a mask boundary are masked element by
// element ("Spark-X2.6-4B-Base" page §滑动窗口 512 and §36 层混合注意力排布: full
// layers key kp visible to query qp iff kp <= qp; sliding layers also need
// kp > qp - 512).
//
// Tensor memory per block (512 columns x 128 lanes, fp32):
//   [0, 256)    O accumulator, one lane per query row
//   [256, 384)  S buffer 0 (QK^T of even tiles; P as bf16 pairs in its first 64 columns)
//   [384, 512)  S buffer 1 (odd tiles)
#pragma once
#include <cuda.h>
#include "ptx.cuh"
#include "rope_append.cuh"

namespace spark {

constexpr int kPfM = 128;                      // query rows per block
constexpr int kPfN = 128;                      // keys per KV tile
constexpr int kPfQBytes = kPfM * kHeadDim * 2; // 64 KB
constexpr int kPfThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0;
constexpr uint32_t kSCol = 256;

struct PrefillParams {
  __nv_bfloat16* out;            // [B][T][16][256]
  const __nv_bfloat16* gate;     // [B][T][16]
  const int* pos0;               // [B]
  int B, T, cap, sliding, has_cache, n_qt;
  int rope, rot;                 // rope: q is raw and is rotated in shared memory
  double log2_theta;
  unsigned long long timeout_ns;
  RopeFreq freq;
  // Ragged batches: sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of
  // the packed q, k, v, gate and out (T is then the longest sequence), and its
  // history comes from a paged pool: logical row r in page
  // block_table[b * max_pages + r / page] at row r % page (block_table null:
  // no paged history).
  const int* cu_seqlens;
  const int* block_table;
  int max_pages, page_shift, n_pages;
};

// Which KV tiles a block visits.  Tile j < n_hist comes from the cache and
// covers absolute positions [a0 + 128 j, +128); later tiles come from the
// chunk and cover positions pos0 + 128 (c_lo + j - n_hist) + [0, 128).
struct PfSchedule {
  int pos0, T, qp0, q_last, need_lo, a0, n_hist, c_lo, n_tiles;
};

// T: this sequence's chunk length (P.T for a dense batch).
__device__ __forceinline__ PfSchedule pf_schedule(const PrefillParams& P, int qt, int pos0, int T) {
  PfSchedule S;
  S.pos0 = pos0;
  S.T = T;
  S.qp0 = pos0 + qt * kPfM;
  S.q_last = min(pos0 + T, S.qp0 + kPfM) - 1;
  S.need_lo = P.sliding ? max(0, S.qp0 - (kWindow - 1)) : 0;
  S.n_hist = 0;
  S.a0 = 0;
  if (P.has_cache && pos0 > S.need_lo) {
    S.a0 = (S.need_lo / kPfN) * kPfN;
    S.n_hist = (pos0 - 1) / kPfN - S.a0 / kPfN + 1;
  }
  S.c_lo = S.need_lo > pos0 ? (S.need_lo - pos0) / kPfN : 0;
  S.n_tiles = S.n_hist + (qt - S.c_lo + 1);
  return S;
}

struct PfTile {
  int hist;        // 1: from the cache
  int kt0;         // absolute position of the tile's first key
  int row;         // cache row (hist) or chunk token index of the first key
  int v_lo, v_hi;  // keys with positions in [v_lo, v_hi) exist
};

__device__ __forceinline__ PfTile pf_tile(const PfSchedule& S, const PrefillParams& P, int j) {
  PfTile t;
  if (j < S.n_hist) {
    t.hist = 1;
    t.kt0 = S.a0 + j * kPfN;
    t.v_lo = S.need_lo;
    t.v_hi = S.pos0;
    // Cache rows at and past pos0 may never have been written, and a masked
    // score does not cancel a NaN there (0 * NaN).  So the last history tile
    // is moved back to end exactly at pos0, and the keys it shares with the
    // tile before it are masked.  Rows before 0 are the TMA's zero fill.  A
    // ring that has wrapped (pos0 >= 512) holds written rows everywhere.
    // Paged history keeps its tiles page-aligned instead (a moved tile would
    // straddle pages): there the rows of the last page past pos0 must be finite.
    if (j == S.n_hist - 1 && t.kt0 + kPfN > S.pos0 && (!P.sliding || S.pos0 < kWindow) &&
        P.block_table == nullptr) {
      t.v_lo = max(S.need_lo, t.kt0);
      t.kt0 = S.pos0 - kPfN;
    }
    t.row = (P.sliding && t.kt0 >= 0) ? (t.kt0 & (kWindow - 1)) : t.kt0;
  } else {
    const int c = S.c_lo + (j - S.n_hist);
    t.hist = 0;
    t.kt0 = S.pos0 + c * kPfN;
    t.row = c * kPfN;
    t.v_lo = S.pos0;
    t.v_hi = S.pos0 + S.T;
  }
  return t;
}

}  // namespace spark
