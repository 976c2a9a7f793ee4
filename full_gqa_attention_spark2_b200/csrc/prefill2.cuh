// Flash-attention prefill on a pair of SMs (tcgen05 cta_group::2, M = 256).
//
// A cluster of two blocks computes two query heads of the same KV group over
// the same 128-query tile, so both need exactly the same K/V tiles and masks.
// Each UMMA instruction of the pair is issued once, by the even block, with
// M = 256 rows: rows 0..127 (block 0's head) come from block 0's shared memory
// and tensor memory, rows 128..255 from block 1's, and the B operand is split
// in halves between the two blocks.  So each block stages only half of every
// K tile (64 of its 128 keys) and half of every V tile (128 of its 256 dims):
// 64 KB of K/V per 128-key tile per SM instead of 128 KB, which doubles the
// loads in flight that the shared-memory ring can hold and halves the L2->SM
// traffic.
//
// Per block: Q tile 64 KB; ring of 5 slots of 32 KB.  A K slot holds this
// block's 64 keys of a K tile (four 64-dim boxes); a V slot holds this block's
// 128 dims of a V tile (four 32-key sub-tiles of two 64-dim boxes).  One
// barrier wait per slot keeps the single MMA-issuing thread ahead of the
// tensor core.  TMEM per
// block as in the single-SM kernel: O [0,256), S buffers [256,384) and
// [384,512), P (bf16 pairs) over the first 64 columns of its S buffer.
//
// Synchronisation of the pair:
//   - both producers load into their own shared memory; their TMA bytes complete
//     on the even block's slot barrier, which only the even producer arms;
//   - the even block's MMA thread commits with a two-block multicast to the
//     slot-empty, S-ready and O-ready barriers of both blocks;
//   - both blocks' softmax warps arrive on the even block's P-ready barrier.
#pragma once
#include <cuda.h>
#include "prefill.cuh"
#include "ptx.cuh"

namespace spark {

constexpr int kP2Slots = 5;
constexpr int kP2SlotBytes = 32768;
constexpr int kP2SmemBytes = 1024 + kPfQBytes + kP2Slots * kP2SlotBytes + 1024;
constexpr uint32_t kIdescQK2 = umma_idesc_bf16(256, 128, false, false);
constexpr uint32_t kIdescPV2 = umma_idesc_bf16(256, 256, false, true);

// Page-entry prefetch of a ragged batch: tiles ahead, and ring slots (2 ints each).
constexpr int kPgAhead = 3;
constexpr int kPgRing = 8;

// kRagged: packed sequences of different lengths (cu_seqlens) with history
// from a paged pool; q, k, v, gate and out are [total][heads][256] views
// (4-D maps with a batch extent of 1), the pool maps 4-D (dim, row in page,
// head, page).  Otherwise a dense batch [B][T] with a dense cache.
template <bool kRagged>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPfThreads, 1)
    prefill2_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kcmap,
                    const __grid_constant__ CUtensorMap vcmap, const __grid_constant__ CUtensorMap omap,
                    const PrefillParams P) {
  extern __shared__ uint8_t dsmem[];
  const uint32_t raw = smem_u32(dsmem);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = dsmem + (base - raw);
  const uint32_t q_s = base;
  const uint32_t slots = base + kPfQBytes;
  uint8_t* gmisc = gbase + kPfQBytes + kP2Slots * kP2SlotBytes;
  const uint32_t misc = smem_u32(gmisc);
  const uint32_t bar_slot_full = misc;              // [5], even block's are used
  const uint32_t bar_slot_empty = misc + 40;        // [5], both blocks
  const uint32_t bar_q = misc + 80;                 // this block's Q landed (each block's own)
  const uint32_t bar_s = misc + 88;                 // [2], both
  const uint32_t bar_p = misc + 104;                // [2], even block's is used
  const uint32_t bar_o = misc + 120;                // [2], both
  const uint32_t bar_done = misc + 136;             // even block's
  const uint32_t bar_q_ready = misc + 144;          // both blocks' Q rotated / checked (even block's)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gmisc + 160);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gmisc + 164);

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  // cluster -> (head pair, query tile (heaviest first), KV head, sequence)
  int id = blockIdx.x >> 1;
  const int hp = id & 1;
  id >>= 1;
  const int qt = P.n_qt - 1 - (id % P.n_qt);
  id /= P.n_qt;
  const int kvh = id & 3;
  const int b = id >> 2;
  const int h = kvh * 4 + hp * 2 + (int)rank;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int pos0 = P.pos0[b];
  // this sequence's first packed row and chunk length
  const int tok0 = kRagged ? P.cu_seqlens[b] : 0;
  const int T_b = kRagged ? P.cu_seqlens[b + 1] - tok0 : P.T;
  const bool bad = pos0 < 0 || T_b < 0 || T_b > P.T || pos0 > kMaxPos - T_b ||
                   (P.has_cache && !P.sliding && pos0 > P.cap);
  PfSchedule S = pf_schedule(P, qt, bad ? 0 : pos0, bad ? 0 : T_b);
  if (bad) {
    S.n_tiles = 0;
    if (threadIdx.x == 0 && qt == 0 && h == 0) raise_error(kErrPosition, 0x500u | (unsigned)b);
  } else if (kRagged && qt * kPfM >= T_b) {
    S.n_tiles = 0;                    // a shorter sequence: this query tile is past its end
  }
  const int n = S.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kP2Slots; ++s) {
      mbar_init(bar_slot_full + 8 * s, 1);
      mbar_init(bar_slot_empty + 8 * s, 1);
    }
    mbar_init(bar_q, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_s + 8 * x, 1);
      mbar_init(bar_p + 8 * x, 8);        // 4 softmax warps of each block
      mbar_init(bar_o + 8 * x, 1);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_q_ready, P.rope ? 12 : 8);   // softmax warps (and RoPE helper warps 2, 3) of each block
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (n > 0 && warp == 0 && !kRagged) {
    // ------------------------------------------------------ producers (both)
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      if (P.has_cache) {
        tma_prefetch_desc(&kcmap);
        tma_prefetch_desc(&vcmap);
      }
      // Q lands on this block's own barrier: its softmax warps rotate it (RoPE at load) or
      // just see it arrive, then tell the even block's MMA thread
      mbar_arrive_expect_tx(bar_q, kPfQBytes);
      for (int d = 0; d < 4; ++d) tma_load_4d(q_s + d * 16384, &qmap, bar_q, d * 64, h, qt * kPfM, b);
      const int plane = b * kNkv + kvh;
      const int key_half = 64 * (int)rank;       // this block's keys of a K tile
      const int dim_half = 128 * (int)rank;      // this block's dims of a V tile
      int li = 0;
      bool ok = true;
      for (int step = 0; step <= n && ok; ++step) {
        for (int part = 0; part < 2 && ok; ++part) {
          const bool is_k = (part == 0);
          const int j = is_k ? step : step - 1;
          if (j < 0 || j >= n) continue;
          const PfTile t = pf_tile(S, P, j);
          const int s = li % kP2Slots;
          if (li >= kP2Slots &&
              !mbar_wait(bar_slot_empty + 8 * s, ((li / kP2Slots) - 1) & 1, abort_flag, P.timeout_ns, 0x50u)) {
            ok = false;
            break;
          }
          const uint32_t dst = slots + s * kP2SlotBytes;
          const uint32_t full0 = mapa_shared(bar_slot_full + 8 * s, 0);
          if (leader) mbar_arrive_expect_tx(bar_slot_full + 8 * s, 2 * kP2SlotBytes);
          if (is_k) {          // four 64-dim boxes of this block's 64 keys, 8 KB each
            for (int x = 0; x < 4; ++x) {
              if (t.hist) tma2_load_3d(dst + x * 8192, &kcmap, full0, x * 64, t.row + key_half, plane);
              else tma2_load_4d(dst + x * 8192, &kmap, full0, x * 64, kvh, t.row + key_half, b);
            }
          } else {             // four 32-key sub-tiles x this block's two 64-dim boxes, 4 KB each
            for (int x = 0; x < 4; ++x)
              for (int d = 0; d < 2; ++d) {
                const int dim = dim_half + 64 * d;
                const uint32_t o = dst + x * 8192 + d * 4096;
                if (t.hist) tma2_load_3d(o, &vcmap, full0, dim, t.row + 32 * x, plane);
                else tma2_load_4d(o, &vmap, full0, dim, kvh, t.row + 32 * x, b);
              }
          }
          ++li;
        }
      }
      const bool q_landed = mbar_drain(bar_q, 0, 200000000ull);
      if (leader) {
        // the even block's slot barriers count both blocks' bytes: wait for all copies in flight
        if (q_landed) {
          for (int i = max(0, li - kP2Slots); i < li; ++i)
            if (!mbar_drain(bar_slot_full + 8 * (i % kP2Slots), (i / kP2Slots) & 1, 200000000ull)) break;
        }
      } else if (!ok) {
        __nanosleep(200000);   // aborted: let this block's last copies land before the pair leaves
      }
    }
    __syncwarp();
  } else if (n > 0 && warp == 0) {
    // ------------------------------------------------- producers (both), ragged batch
    const int key_half = 64 * (int)rank;       // this block's keys of a K tile
    const int dim_half = 128 * (int)rank;      // this block's dims of a V tile
    int li = 0;
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      if (P.has_cache) {
        tma_prefetch_desc(&kcmap);
        tma_prefetch_desc(&vcmap);
      }
      mbar_arrive_expect_tx(bar_q, kPfQBytes);
      for (int d = 0; d < 4; ++d) tma_load_4d(q_s + d * 16384, &qmap, bar_q, d * 64, h, tok0 + qt * kPfM, 0);
    }
    {
      // Ragged batch.  A history tile's rows [row, row + 128) lie in at most two pages (pages of
      // 64 rows or more): those of rows `row` and `row + 64`.  Their table entries are fetched
      // kPgAhead tiles ahead with 4-byte asynchronous copies into a small ring in shared memory,
      // one commit group per tile, so the producer never waits on a table load in a register.
      // Both blocks of the pair read the same table, so both stop at the same tile on a bad index.
      if (lane == 0) {
        const uint32_t ring = misc + 192;          // [kPgRing][2] int
        int* ring_gen = reinterpret_cast<int*>(gmisc + 192);
        auto fetch = [&](int j) {                  // entries of tile j (nothing for chunk tiles)
          if (j < n) {
            const PfTile t = pf_tile(S, P, j);
            if (t.hist) {
              // rows row + 64 .. may lie past the table's last page (then they are past the
              // history and masked): read the first page's entry again instead
              const int n_lp = P.sliding ? (kWindow >> P.page_shift) : P.max_pages;
              const int lp_lo = t.row >> P.page_shift;
              const int lp_hi = (t.row + 64) >> P.page_shift;
              const int* row_tab = P.block_table + (long long)b * P.max_pages;
              const int slot = j % kPgRing;
              cp_async4(ring + 8 * slot, row_tab + lp_lo);
              cp_async4(ring + 8 * slot + 4, row_tab + (lp_hi < n_lp ? lp_hi : lp_lo));
            }
          }
          cp_async_commit();
        };
        for (int j = 0; j < kPgAhead; ++j) fetch(j);
        const int pmask = (1 << P.page_shift) - 1;
        for (int step = 0; step <= n && ok; ++step) {
          if (step < n) {                          // tile `step` is next needed: fetch one more
            fetch(step + kPgAhead);
            cp_async_wait<kPgAhead>();             // ... and the groups up to tile `step` are in
          }
          for (int part = 0; part < 2 && ok; ++part) {
            const bool is_k = (part == 0);
            const int j = is_k ? step : step - 1;
            if (j < 0 || j >= n) continue;
            const PfTile t = pf_tile(S, P, j);
            const int s = li % kP2Slots;
            int pg_lo = 0, pg_hi = 0;
            if (t.hist) {
              pg_lo = ring_gen[2 * (j % kPgRing)];
              pg_hi = ring_gen[2 * (j % kPgRing) + 1];
              if (pg_lo < 0 || pg_lo >= P.n_pages || pg_hi < 0 || pg_hi >= P.n_pages) {
                raise_error(kErrPosition, 0xA00u | (unsigned)b);
                *abort_flag = 1;
                ok = false;
                break;
              }
            }
            if (li >= kP2Slots &&
                !mbar_wait(bar_slot_empty + 8 * s, ((li / kP2Slots) - 1) & 1, abort_flag, P.timeout_ns, 0x50u)) {
              ok = false;
              break;
            }
            const uint32_t dst = slots + s * kP2SlotBytes;
            const uint32_t full0 = mapa_shared(bar_slot_full + 8 * s, 0);
            if (leader) mbar_arrive_expect_tx(bar_slot_full + 8 * s, 2 * kP2SlotBytes);
            if (is_k) {
              const int kr = t.row + key_half;
              const int pk = key_half ? pg_hi : pg_lo;
              for (int x = 0; x < 4; ++x) {
                if (t.hist) tma2_load_4d(dst + x * 8192, &kcmap, full0, x * 64, kr & pmask, kvh, pk);
                else tma2_load_4d(dst + x * 8192, &kmap, full0, x * 64, kvh, tok0 + kr, 0);
              }
            } else {
              for (int x = 0; x < 4; ++x)
                for (int d = 0; d < 2; ++d) {
                  const int dim = dim_half + 64 * d;
                  const int vr = t.row + 32 * x;
                  const uint32_t o = dst + x * 8192 + d * 4096;
                  if (t.hist) tma2_load_4d(o, &vcmap, full0, dim, vr & pmask, kvh, x < 2 ? pg_lo : pg_hi);
                  else tma2_load_4d(o, &vmap, full0, dim, kvh, tok0 + vr, 0);
                }
            }
            ++li;
          }
        }
        cp_async_wait<0>();                        // no copy into the ring may outlive the block
      }
    }
    if (lane == 0) {
      const bool q_landed = mbar_drain(bar_q, 0, 200000000ull);
      if (leader) {
        if (q_landed) {
          for (int i = max(0, li - kP2Slots); i < li; ++i)
            if (!mbar_drain(bar_slot_full + 8 * (i % kP2Slots), (i / kP2Slots) & 1, 200000000ull)) break;
        }
      } else if (!ok) {
        __nanosleep(200000);   // aborted: let this block's last copies land before the pair leaves
      }
    }
    __syncwarp();
  } else if (n > 0 && warp == 1) {
    // --------------------------------------------------- MMA issuer (even block)
    if (lane == 0 && leader) {
      const uint64_t dq = smem_desc_sw128(q_s, 16, 1024);
      bool ok = mbar_wait_cluster(bar_q_ready, 0, abort_flag, P.timeout_ns, 0x60u);
      tc_fence_after();
      int li = 0;
      auto issue_s = [&](int j) -> bool {
        const uint32_t dcol = tmem + kSCol + 128u * (j & 1);
        const int s = li % kP2Slots;
        if (!mbar_wait(bar_slot_full + 8 * s, (li / kP2Slots) & 1, abort_flag, P.timeout_ns, 0x61u)) return false;
        tc_fence_after();
        const uint64_t dk = smem_desc_sw128(slots + s * kP2SlotBytes, 16, 1024);
#pragma unroll
        for (int d = 0; d < 4; ++d)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma2_ss(dcol, dq + (uint64_t)((d * 16384 + kk * 32) >> 4), dk + (uint64_t)((d * 8192 + kk * 32) >> 4),
                     kIdescQK2, (d | kk) != 0);
        umma2_commit_mc(bar_slot_empty + 8 * s, 3);
        umma2_commit_mc(bar_s + 8 * (j & 1), 3);
        ++li;
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait_cluster(bar_p + 8 * (j & 1), (j >> 1) & 1, abort_flag, P.timeout_ns, 0x62u)) return false;
        const int s = li % kP2Slots;
        if (!mbar_wait(bar_slot_full + 8 * s, (li / kP2Slots) & 1, abort_flag, P.timeout_ns, 0x63u)) return false;
        tc_fence_after();
        const uint32_t pcol = tmem + kSCol + 128u * (j & 1);
        const uint64_t dv = smem_desc_sw128(slots + s * kP2SlotBytes, 4096, 1024);
#pragma unroll
        for (int v = 0; v < 4; ++v)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma2_ts(tmem + kOCol, pcol + 16u * v + 8u * kk, dv + (uint64_t)((v * 8192 + kk * 2048) >> 4), kIdescPV2,
                     (j > 0 || v > 0 || kk > 0) ? 1u : 0u);
        umma2_commit_mc(bar_slot_empty + 8 * s, 3);
        umma2_commit_mc(bar_o + 8 * (j & 1), 3);
        ++li;
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
      umma2_commit_mc(bar_done, 1);
      mbar_drain(bar_done, 0, 200000000ull);
    }
    __syncwarp();
  } else if (n > 0 && warp >= 2 && warp < 4 && P.rope) {
    // ------------------------------------------- RoPE helpers (both): their share of Q
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, abort_flag, P.timeout_ns, 0x74u));
    if (ok) {
      rope_q_tile(gbase, P, S.qp0, threadIdx.x - 64);
      fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0 && ok) {
      if (leader) mbar_arrive(bar_q_ready);
      else mbar_arrive_remote_cluster(mapa_shared(bar_q_ready, 0));
    }
  } else if (n > 0 && warp >= 4) {
    // ------------------------------------------------- softmax warps (both)
    const int r = threadIdx.x - 128;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ocol = tmem + lane_base + kOCol;
    const int qp = S.qp0 + r;
    const bool row_valid = qp < S.pos0 + S.T;
    const uint32_t p_ready0 = mapa_shared(bar_p, 0);
    bool ok = true;
    {
      // Q: wait for this block's tile, rotate it in place when q is raw (with warps 2 and 3),
      // hand it to the MMA thread.
      ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, abort_flag, P.timeout_ns, 0x73u));
      if (ok && P.rope) {
        rope_q_tile(gbase, P, S.qp0, threadIdx.x - 64);
        fence_proxy_async_smem();                         // the tensor core reads Q next
      }
      __syncwarp();
      if (lane == 0 && ok) {
        if (leader) mbar_arrive(bar_q_ready);
        else mbar_arrive_remote_cluster(mapa_shared(bar_q_ready, 0));
      }
    }
    float m_ref = -INFINITY, l_run = 0.f;
    for (int j = 0; j < n && ok; ++j) {
      // warp-uniform outcomes: tcgen05.ld / st below need every lane of the warp
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s + 8 * (j & 1), (j >> 1) & 1, abort_flag, P.timeout_ns, 0x70u))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t scol = tmem + lane_base + kSCol + 128u * (j & 1);
      const PfTile t = pf_tile(S, P, j);
      // the previous P.V (tile j-1) must be complete before O is rescaled
      if (!pf_softmax_tile<kRagged>(scol, ocol, t, S, P, qp, m_ref, l_run, bar_o + 8 * ((j - 1) & 1),
                               ((j - 1) >> 1) & 1, abort_flag, 0x71u)) {
        ok = false;
        break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(bar_p + 8 * (j & 1));
        else mbar_arrive_remote(p_ready0 + 8 * (j & 1));
      }
    }
    const bool ep_ok = ok && __all_sync(0xffffffffu, mbar_wait(bar_o + 8 * ((n - 1) & 1), ((n - 1) >> 1) & 1,
                                                               abort_flag, P.timeout_ns, 0x72u));
    if (ep_ok) {
      tc_fence_after();
      // out = O / l * sigmoid(gate) in bf16, staged in the Q buffer (free: every S
      // MMA has completed) in the 128-byte swizzled layout of four [128 x 64] boxes,
      // then written with TMA tensor stores (rows past the chunk are clipped)
      float scale = 0.f;
      if (row_valid) {
        const long long tok = kRagged ? (long long)tok0 + (qp - S.pos0) : (long long)b * P.T + (qp - S.pos0);
        const float gl = __bfloat162float(P.gate[tok * kNq + h]);
        scale = (l_run > 0.f ? 1.f / l_run : 0.f) * (1.f / (1.f + expf(-gl)));
      }
      uint8_t* q_gen = gbase;                     // generic view of the Q buffer
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t ov[32];
        tmem_ld32(ocol + 32 * c, ov);
        tmem_wait_ld();
        uint8_t* box = q_gen + (c >> 1) * 16384 + r * 128;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint4 w;
          w.x = pack_bf16(__uint_as_float(ov[8 * e + 0]) * scale, __uint_as_float(ov[8 * e + 1]) * scale);
          w.y = pack_bf16(__uint_as_float(ov[8 * e + 2]) * scale, __uint_as_float(ov[8 * e + 3]) * scale);
          w.z = pack_bf16(__uint_as_float(ov[8 * e + 4]) * scale, __uint_as_float(ov[8 * e + 5]) * scale);
          w.w = pack_bf16(__uint_as_float(ov[8 * e + 6]) * scale, __uint_as_float(ov[8 * e + 7]) * scale);
          const int chunk = (c & 1) * 4 + e;      // 16-byte chunk within the 128-byte row of the box
          *reinterpret_cast<uint4*>(box + ((chunk ^ (r & 7)) << 4)) = w;
        }
      }
      fence_proxy_async_smem();                   // make the generic writes visible to TMA
    }
    // every softmax thread reaches this barrier, aborted or not; store only if all staged their row
    uint32_t all_ok;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(all_ok)
        : "r"((uint32_t)ep_ok)
        : "memory");
    const bool full_rows = !kRagged || (qt + 1) * kPfM <= S.T;
    if (all_ok && full_rows && threadIdx.x == 128) {
      for (int d = 0; d < 4; ++d) {
        if (kRagged) tma_store_4d(&omap, q_s + d * 16384, d * 64, h, tok0 + qt * kPfM, 0);
        else tma_store_4d(&omap, q_s + d * 16384, d * 64, h, qt * kPfM, b);
      }
      bulk_commit_group();
      bulk_wait_group0();
    }
    if (kRagged && all_ok && !full_rows && row_valid) {
      // the sequence ends inside this tile: the rows after it belong to the next sequence, so
      // each row is stored by its own thread (the box store would cover all 128)
      const uint8_t* q_gen = gbase;
      uint4* dst = reinterpret_cast<uint4*>(P.out + ((long long)(tok0 + (qp - S.pos0)) * kNq + h) * kHeadDim);
#pragma unroll
      for (int bx = 0; bx < 4; ++bx)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          dst[bx * 8 + ch] = *reinterpret_cast<const uint4*>(q_gen + bx * 16384 + r * 128 + ((ch ^ (r & 7)) << 4));
    }
    __syncwarp();
  }

  // both blocks: no TMEM, shared memory or barrier of either block is in use past this point
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, kTmemCols);
  }
}

}  // namespace spark
