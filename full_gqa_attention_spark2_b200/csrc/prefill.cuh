// Flash-attention prefill for sm_100a: TMA-staged tiles, tcgen05 UMMA into
// tensor memory, fp32 online softmax, sigmoid gate in the epilogue.
//
// One block = one (sequence b, query head h, 128-query tile).  Q (128 x 256
// bf16, 64 KB) stays in shared memory; K and V stream through a ring of ten
// 16 KB slots: a K tile of 128 keys is four slots (one per 64-dim box, 128 B
// swizzle), a V tile is four slots of 32 keys each (all 256 dims).
//
// Tensor memory (512 columns x 128 lanes, fp32):
//   [0, 256)    O accumulator, one lane per query row
//   [256, 384)  S buffer 0 (QK^T of even tiles; P as bf16 pairs in its first 64 columns)
//   [384, 512)  S buffer 1 (odd tiles)
//
// Warp roles (256 threads):
//   warp 0  lane 0: TMA producer (Q once, then K/V slots in MMA order)
//   warp 1  lane 0: MMA issuer; the whole warp allocates / frees TMEM
//   warps 4..7     : softmax, one thread per query row (= TMEM lane); they
//                    also rescale O when the running max grows by more than
//                    2^8 and run the epilogue out = O / l * sigmoid(gate)
// MMA order S_0, S_1, PV_0, S_2, PV_1, ... keeps the tensor core on S_{j+1}
// while the softmax warps turn S_j into P_j.
//
// Masks ("Spark-X2.6-4B-Base" page §滑动窗口 512 and §36 层混合注意力排布): full
// layers key kp visible to query qp iff kp <= qp; sliding layers also need
// kp > qp - 512.  Tiles that no query of the block can see are never loaded;
// only tiles that straddle a boundary are masked element by element.
#pragma once
#include <cuda.h>
#include "ptx.cuh"
#include "rope_append.cuh"

namespace spark {

constexpr int kPfM = 128;                      // query rows per block
constexpr int kPfN = 128;                      // keys per KV tile
constexpr int kPfSlots = 10;
constexpr int kPfSlotBytes = 16384;
constexpr int kPfQBytes = kPfM * kHeadDim * 2; // 64 KB
constexpr int kPfThreads = 256;
constexpr int kPfSmemBytes = 1024 + kPfQBytes + kPfSlots * kPfSlotBytes + 512;
constexpr uint32_t kIdescQK = umma_idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 256, false, true);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0;
constexpr uint32_t kSCol = 256;

struct PrefillParams {
  __nv_bfloat16* out;            // [B][T][16][256]
  const __nv_bfloat16* gate;     // [B][T][16]
  const int* pos0;               // [B]
  int B, T, cap, sliding, has_cache, n_qt;
  unsigned long long timeout_ns;
};

// Which KV tiles a block visits.  Tile j < n_hist comes from the cache and
// covers absolute positions [a0 + 128 j, +128); later tiles come from the
// chunk and cover positions pos0 + 128 (c_lo + j - n_hist) + [0, 128).
struct PfSchedule {
  int pos0, qp0, q_last, need_lo, a0, n_hist, c_lo, n_tiles;
};

__device__ __forceinline__ PfSchedule pf_schedule(const PrefillParams& P, int qt, int pos0) {
  PfSchedule S;
  S.pos0 = pos0;
  S.qp0 = pos0 + qt * kPfM;
  S.q_last = min(pos0 + P.T, S.qp0 + kPfM) - 1;
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
    t.row = P.sliding ? (t.kt0 & (kWindow - 1)) : t.kt0;
    t.v_lo = S.need_lo;
    t.v_hi = S.pos0;
  } else {
    const int c = S.c_lo + (j - S.n_hist);
    t.hist = 0;
    t.kt0 = S.pos0 + c * kPfN;
    t.row = c * kPfN;
    t.v_lo = S.pos0;
    t.v_hi = S.pos0 + P.T;
  }
  return t;
}

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kcmap,
                   const __grid_constant__ CUtensorMap vcmap, const PrefillParams P) {
  extern __shared__ uint8_t dsmem[];
  const uint32_t raw = smem_u32(dsmem);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = dsmem + (base - raw);
  const uint32_t q_s = base;
  const uint32_t slots = base + kPfQBytes;
  uint8_t* gmisc = gbase + kPfQBytes + kPfSlots * kPfSlotBytes;
  const uint32_t misc = smem_u32(gmisc);
  const uint32_t bar_slot_full = misc;              // [10]
  const uint32_t bar_slot_empty = misc + 80;        // [10]
  const uint32_t bar_q = misc + 160;
  const uint32_t bar_s = misc + 168;                // [2]
  const uint32_t bar_p = misc + 184;                // [2]
  const uint32_t bar_o = misc + 200;                // [2]
  const uint32_t bar_done = misc + 216;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gmisc + 224);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gmisc + 228);

  // block -> (head within group, query tile (heaviest first), KV head, sequence)
  int id = blockIdx.x;
  const int hh = id & 3;
  id >>= 2;
  const int qt = P.n_qt - 1 - (id % P.n_qt);
  id /= P.n_qt;
  const int kvh = id & 3;
  const int b = id >> 2;
  const int h = kvh * 4 + hh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int pos0 = P.pos0[b];
  const bool bad = pos0 < 0 || pos0 > kMaxPos - P.T || (P.has_cache && !P.sliding && pos0 > P.cap);
  PfSchedule S = pf_schedule(P, qt, bad ? 0 : pos0);
  if (bad) {
    S.n_tiles = 0;
    if (threadIdx.x == 0 && qt == 0 && h == 0) raise_error(kErrPosition, 0x400u | (unsigned)b);
  }
  const int n = S.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPfSlots; ++s) {
      mbar_init(bar_slot_full + 8 * s, 1);
      mbar_init(bar_slot_empty + 8 * s, 1);
    }
    mbar_init(bar_q, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_s + 8 * x, 1);
      mbar_init(bar_p + 8 * x, 4);
      mbar_init(bar_o + 8 * x, 1);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (n > 0 && warp == 0) {
    // ----------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      if (P.has_cache) {
        tma_prefetch_desc(&kcmap);
        tma_prefetch_desc(&vcmap);
      }
      mbar_arrive_expect_tx(bar_q, kPfQBytes);
      for (int d = 0; d < 4; ++d) tma_load_4d(q_s + d * 16384, &qmap, bar_q, d * 64, h, qt * kPfM, b);
      const int plane = b * kNkv + kvh;
      int li = 0;
      bool ok = true;
      // load order = MMA consumption order: K_0, then (K_{j+1}, V_j) for each j
      for (int step = 0; step <= n && ok; ++step) {
        for (int part = 0; part < 2 && ok; ++part) {
          const bool is_k = (part == 0);
          const int j = is_k ? step : step - 1;
          if (j < 0 || j >= n) continue;
          const PfTile t = pf_tile(S, P, j);
          for (int x = 0; x < 4; ++x) {
            const int s = li % kPfSlots;
            if (li >= kPfSlots &&
                !mbar_wait(bar_slot_empty + 8 * s, ((li / kPfSlots) - 1) & 1, abort_flag, P.timeout_ns, 0x20u)) {
              ok = false;
              break;
            }
            const uint32_t dst = slots + s * kPfSlotBytes;
            const uint32_t full = bar_slot_full + 8 * s;
            mbar_arrive_expect_tx(full, kPfSlotBytes);
            if (is_k) {        // x = 64-dim box, 128 keys
              if (t.hist) tma_load_3d(dst, &kcmap, full, x * 64, t.row, plane);
              else tma_load_4d(dst, &kmap, full, x * 64, kvh, t.row, b);
            } else {           // x = 32-key sub-tile, all four 64-dim boxes
              for (int d = 0; d < 4; ++d) {
                if (t.hist) tma_load_3d(dst + d * 4096, &vcmap, full, d * 64, t.row + 32 * x, plane);
                else tma_load_4d(dst + d * 4096, &vmap, full, d * 64, kvh, t.row + 32 * x, b);
              }
            }
            ++li;
          }
        }
      }
      // never leave with copies in flight
      if (mbar_drain(bar_q, 0, 200000000ull)) {
        for (int i = max(0, li - kPfSlots); i < li; ++i)
          if (!mbar_drain(bar_slot_full + 8 * (i % kPfSlots), (i / kPfSlots) & 1, 200000000ull)) break;
      }
    }
    __syncwarp();
  } else if (n > 0 && warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dq = smem_desc_sw128(q_s, 16, 1024);
      bool ok = mbar_wait(bar_q, 0, abort_flag, P.timeout_ns, 0x30u);
      tc_fence_after();
      int li = 0;
      auto issue_s = [&](int j) -> bool {
        const uint32_t dcol = tmem + kSCol + 128u * (j & 1);
        for (int d = 0; d < 4; ++d) {
          const int s = li % kPfSlots;
          if (!mbar_wait(bar_slot_full + 8 * s, (li / kPfSlots) & 1, abort_flag, P.timeout_ns, 0x31u))
            return false;
          tc_fence_after();
          const uint64_t dk = smem_desc_sw128(slots + s * kPfSlotBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(dcol, dq + (uint64_t)((d * 16384 + kk * 32) >> 4), dk + (uint64_t)((kk * 32) >> 4),
                    kIdescQK, (d | kk) != 0);
          umma_commit(bar_slot_empty + 8 * s);
          ++li;
        }
        umma_commit(bar_s + 8 * (j & 1));
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(bar_p + 8 * (j & 1), (j >> 1) & 1, abort_flag, P.timeout_ns, 0x32u)) return false;
        tc_fence_after();
        const uint32_t pcol = tmem + kSCol + 128u * (j & 1);
        for (int v = 0; v < 4; ++v) {
          const int s = li % kPfSlots;
          if (!mbar_wait(bar_slot_full + 8 * s, (li / kPfSlots) & 1, abort_flag, P.timeout_ns, 0x33u))
            return false;
          tc_fence_after();
          const uint64_t dv = smem_desc_sw128(slots + s * kPfSlotBytes, 4096, 1024);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_ts(tmem + kOCol, pcol + 16u * v + 8u * kk, dv + (uint64_t)((kk * 2048) >> 4), kIdescPV,
                    (j > 0 || v > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar_slot_empty + 8 * s);
          ++li;
        }
        umma_commit(bar_o + 8 * (j & 1));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
      // every MMA issued so far has completed before TMEM is released
      umma_commit(bar_done);
      mbar_drain(bar_done, 0, 200000000ull);
    }
    __syncwarp();
  } else if (n > 0 && warp >= 4) {
    // ------------------------------------------------------ softmax warps
    const int r = threadIdx.x - 128;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ocol = tmem + lane_base + kOCol;
    const int qp = S.qp0 + r;
    const bool row_valid = qp < S.pos0 + P.T;
    const float c_scale = 0.0625f * 1.4426950408889634f;    // 1/sqrt(256) * log2(e)
    float m_ref = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      // warp-uniform outcomes: tcgen05.ld / st below need every lane of the warp
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s + 8 * (j & 1), (j >> 1) & 1, abort_flag, P.timeout_ns, 0x40u))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t scol = tmem + lane_base + kSCol + 128u * (j & 1);
      uint32_t sv[128];
      tmem_ld32(scol, sv);
      tmem_ld32(scol + 32, sv + 32);
      tmem_ld32(scol + 64, sv + 64);
      tmem_ld32(scol + 96, sv + 96);
      tmem_wait_ld();

      const PfTile t = pf_tile(S, P, j);
      // the whole tile is visible to every row of the block?
      const bool full_tile = t.kt0 >= t.v_lo && t.kt0 + kPfN <= t.v_hi && t.kt0 + kPfN - 1 <= S.qp0 &&
                             (!P.sliding || t.kt0 > S.qp0 + kPfM - 1 - kWindow);
      float mx = -INFINITY;
      if (full_tile) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const float x = __uint_as_float(sv[i]) * c_scale;
          sv[i] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      } else {
        const int lo = max(t.v_lo, P.sliding ? qp - (kWindow - 1) : t.v_lo) - t.kt0;
        const int hi = min(t.v_hi - 1, qp) - t.kt0;
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const float x = (i >= lo && i <= hi) ? __uint_as_float(sv[i]) * c_scale : -INFINITY;
          sv[i] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      }
      // conditional rescaling: move the reference max only when it grows by > 2^8
      float factor = 1.f;
      const bool resc = mx > m_ref + 8.f;
      if (resc) {
        factor = fast_exp2(m_ref - mx);        // 0 when m_ref = -inf
        m_ref = mx;
      }
      const bool need_o = resc && l_run > 0.f;
      if (__any_sync(0xffffffffu, need_o)) {
        // O must hold PV_{j-1} before it is rescaled
        if (!__all_sync(0xffffffffu,
                        mbar_wait(bar_o + 8 * ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, P.timeout_ns, 0x41u))) {
          ok = false;
          break;
        }
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
      const float mr = (m_ref == -INFINITY) ? 0.f : m_ref;
      float ls = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float p0 = fast_exp2(__uint_as_float(sv[2 * i]) - mr);
        const float p1 = fast_exp2(__uint_as_float(sv[2 * i + 1]) - mr);
        ls += p0 + p1;
        pk[i] = pack_bf16(p0, p1);
      }
      l_run += ls;
      tmem_st32(scol, pk);
      tmem_st32(scol + 32, pk + 32);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p + 8 * (j & 1));
    }
    if (ok && __all_sync(0xffffffffu,
                         mbar_wait(bar_o + 8 * ((n - 1) & 1), ((n - 1) >> 1) & 1, abort_flag, P.timeout_ns, 0x42u))) {
      tc_fence_after();
      float scale = 0.f;
      __nv_bfloat16* dst = nullptr;
      if (row_valid) {
        const long long tok = (long long)b * P.T + (qp - S.pos0);
        const float gl = __bfloat162float(P.gate[tok * kNq + h]);
        scale = (l_run > 0.f ? 1.f / l_run : 0.f) * (1.f / (1.f + expf(-gl)));
        dst = P.out + (tok * kNq + h) * kHeadDim;
      }
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t ov[32];
        tmem_ld32(ocol + 32 * c, ov);
        tmem_wait_ld();
        if (row_valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(ov[8 * e + 0]) * scale, __uint_as_float(ov[8 * e + 1]) * scale);
            w.y = pack_bf16(__uint_as_float(ov[8 * e + 2]) * scale, __uint_as_float(ov[8 * e + 3]) * scale);
            w.z = pack_bf16(__uint_as_float(ov[8 * e + 4]) * scale, __uint_as_float(ov[8 * e + 5]) * scale);
            w.w = pack_bf16(__uint_as_float(ov[8 * e + 6]) * scale, __uint_as_float(ov[8 * e + 7]) * scale);
            d4[e] = w;
          }
        }
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace spark
