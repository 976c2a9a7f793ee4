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

// RoPE at load: rotate the block's raw Q tile in shared memory (four 128-byte
// swizzled [128 x 64] boxes) in place, shared by kRopeThreads threads (warps 2..7).
// Thread t takes four adjacent pairs (dims 4 qd .. 4 qd + 3 and their partners
// half later) on every n_grp-th row from row rg: four independent recurrences
// and 8-byte accesses, two rows loaded before either is stored.  The first
// row's angles are exact (fp64 product and reduction); the next rows advance by
// the rotation by n_grp * f_i.
constexpr int kRopeThreads = 192;

// n_thr: the threads sharing the tile (a multiple of 32 that n_qd divides).
__device__ __forceinline__ void rope_q_tile(uint8_t* qg, const PrefillParams& P, int qp0, int t,
                                            int n_thr = kRopeThreads) {
  const int half = P.rot >> 1;
  const int n_qd = half >> 2;                   // quads per row: 32 (sliding) or 8 (full)
  const int n_grp = n_thr / n_qd;               // row stride: 6 or 24 for 192 threads
  const int qd = t % n_qd;
  const int rg = t / n_qd;
  float c[4], sn[4], cf[4], sf[4];
  const double r1 = P.freq.f[1];                // the same word for every lane
  double f = pow_u8(r1, 4 * qd);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    rope_angle(qp0 + rg, f, c[e], sn[e]);
    rope_angle(n_grp, f, cf[e], sf[e]);
    f *= r1;
  }
  const int dlo = 4 * qd, dhi = 4 * qd + half;
  auto addr = [&](int d, int row) -> uint2* {
    return reinterpret_cast<uint2*>(qg + (d >> 6) * 16384 + row * 128 + ((((d & 63) >> 3) ^ (row & 7)) << 4) +
                                    (d & 7) * 2);
  };
  auto rotate = [&](const uint2& lo, const uint2& hi, int row) {
    const float l[4] = {bf16_lo(lo.x), bf16_hi(lo.x), bf16_lo(lo.y), bf16_hi(lo.y)};
    const float h[4] = {bf16_lo(hi.x), bf16_hi(hi.x), bf16_lo(hi.y), bf16_hi(hi.y)};
    uint2 ol, oh;
    ol.x = pack_bf16(l[0] * c[0] - h[0] * sn[0], l[1] * c[1] - h[1] * sn[1]);
    ol.y = pack_bf16(l[2] * c[2] - h[2] * sn[2], l[3] * c[3] - h[3] * sn[3]);
    oh.x = pack_bf16(h[0] * c[0] + l[0] * sn[0], h[1] * c[1] + l[1] * sn[1]);
    oh.y = pack_bf16(h[2] * c[2] + l[2] * sn[2], h[3] * c[3] + l[3] * sn[3]);
    *addr(dlo, row) = ol;
    *addr(dhi, row) = oh;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float cn = c[e] * cf[e] - sn[e] * sf[e];
      sn[e] = sn[e] * cf[e] + c[e] * sf[e];
      c[e] = cn;
    }
  };
  int row = rg;
  for (; row + n_grp < kPfM; row += 2 * n_grp) {
    const uint2 lo0 = *addr(dlo, row), hi0 = *addr(dhi, row);
    const uint2 lo1 = *addr(dlo, row + n_grp), hi1 = *addr(dhi, row + n_grp);
    rotate(lo0, hi0, row);
    rotate(lo1, hi1, row + n_grp);
  }
  if (row < kPfM) {
    const uint2 lo0 = *addr(dlo, row), hi0 = *addr(dhi, row);
    rotate(lo0, hi0, row);
  }
}


// One KV tile of the online softmax for this thread's query row (its tensor-memory lane), shared by
// the two prefill kernels.  The tile's scores are read from tensor memory (scol) and masked on a
// boundary tile (keys outside [v_lo, v_hi), after the query, or out of its window).  The running
// max and sum are updated.  The reference max moves only when the max grows by more than 2^8; then
// O in tensor memory (ocol) is rescaled once the previous P.V has completed (barrier o_bar,
// parity o_parity).  P = 2^(s log2(e) / 16 - m) is written back over the scores as bf16 pairs.
// kPacked: the elementwise work in sm_100 packed fp32 pairs and the three-input max.  Returns
// false when a wait ran out.
template <bool kPacked>
__device__ __forceinline__ bool pf_softmax_tile(uint32_t scol, uint32_t ocol, const PfTile& t, const PfSchedule& S,
                                                const PrefillParams& P, int qp, float& m_ref, float& l_run,
                                                uint32_t o_bar, uint32_t o_parity, volatile int* abort_flag,
                                                unsigned where) {
  const float c_scale = 0.0625f * 1.4426950408889634f;    // 1/sqrt(256) * log2(e)
  uint32_t sv[128];
  tmem_ld32(scol, sv);
  tmem_ld32(scol + 32, sv + 32);
  tmem_ld32(scol + 64, sv + 64);
  tmem_ld32(scol + 96, sv + 96);
  tmem_wait_ld();

  const bool full_tile = t.kt0 >= t.v_lo && t.kt0 + kPfN <= t.v_hi && t.kt0 + kPfN - 1 <= S.qp0 &&
                         (!P.sliding || t.kt0 > S.qp0 + kPfM - 1 - kWindow);
  // row max over the raw scores in four independent chains (scale applied after: c_scale > 0)
  float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  if (full_tile) {
    if constexpr (!kPacked) {
#pragma unroll
      for (int i = 0; i < 128; ++i) m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(sv[i]));
    } else {
#pragma unroll
      for (int i = 0; i < 128; i += 2)
        m4[(i >> 1) & 3] = fmax3(m4[(i >> 1) & 3], __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
    }
  } else {
    const int lo = max(t.v_lo, P.sliding ? qp - (kWindow - 1) : t.v_lo) - t.kt0;
    const int hi = min(t.v_hi - 1, qp) - t.kt0;
    if constexpr (!kPacked) {
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        const float x = (i >= lo && i <= hi) ? __uint_as_float(sv[i]) : -INFINITY;
        sv[i] = __float_as_uint(x);
        m4[i & 3] = fmaxf(m4[i & 3], x);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 128; i += 2) {
        const float x0 = (i >= lo && i <= hi) ? __uint_as_float(sv[i]) : -INFINITY;
        const float x1 = (i + 1 >= lo && i + 1 <= hi) ? __uint_as_float(sv[i + 1]) : -INFINITY;
        sv[i] = __float_as_uint(x0);
        sv[i + 1] = __float_as_uint(x1);
        m4[(i >> 1) & 3] = fmax3(m4[(i >> 1) & 3], x0, x1);
      }
    }
  }
  const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c_scale;
  float factor = 1.f;
  const bool resc = mx > m_ref + 8.f;
  if (resc) {
    factor = fast_exp2(m_ref - mx);
    m_ref = mx;
  }
  const bool need_o = resc && l_run > 0.f;
  if (__any_sync(0xffffffffu, need_o)) {
    if (!__all_sync(0xffffffffu, mbar_wait(o_bar, o_parity, abort_flag, P.timeout_ns, where))) return false;
    tc_fence_after();
    const float f = need_o ? factor : 1.f;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t ov[32];
      tmem_ld32(ocol + 32 * c, ov);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
      tmem_st32(ocol + 32 * c, ov);
    }
    tmem_wait_st();
  }
  l_run *= factor;
  const float nmr = (m_ref == -INFINITY) ? 0.f : -m_ref;
  uint32_t pk[64];
  if constexpr (!kPacked) {
    float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * i]), c_scale, nmr));
      const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * i + 1]), c_scale, nmr));
      l4[i & 3] += p0 + p1;
      pk[i] = pack_bf16(p0, p1);
    }
    l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
  } else {
    // p = 2^(s c - m) for pairs of columns with packed FMAs; row sums in two packed accumulators
    const unsigned long long c2 = f2_pack(c_scale, c_scale), n2 = f2_pack(nmr, nmr);
    unsigned long long l2[2] = {0ull, 0ull};
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), c2, n2), x0, x1);
      const float p0 = fast_exp2(x0);
      const float p1 = fast_exp2(x1);
      l2[i & 1] = f2_add(l2[i & 1], f2_pack(p0, p1));
      pk[i] = pack_bf16(p0, p1);
    }
    float la, lb, lc, ld;
    f2_unpack(l2[0], la, lb);
    f2_unpack(l2[1], lc, ld);
    l_run += (la + lb) + (lc + ld);
  }
  tmem_st32(scol, pk);
  tmem_st32(scol + 32, pk + 32);
  tmem_wait_st();
  return true;
}

}  // namespace spark
