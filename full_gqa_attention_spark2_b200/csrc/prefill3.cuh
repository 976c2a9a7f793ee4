// Persistent flash-attention prefill on SM pairs (tcgen05 cta_group::2, M = 256).
//
// The same unit of work as prefill2_kernel (a cluster of two blocks computes
// two query heads of one KV group over one 128-query tile, each block staging
// half of every K/V tile), but each cluster stays resident and walks a list of
// units.  What a short unit pays once per block in prefill2 is paid once per
// launch or hidden behind the previous unit:
//   - barrier setup, TMEM allocation and the cluster handshake: once;
//   - the next unit's Q tile loads as soon as the previous unit's last S MMA
//     has read the Q buffer (a commit on `q_free`), and is rotated (RoPE at
//     load) while the previous unit finishes its P.V and epilogue;
//   - the epilogue stages the output in the ring slots of the unit's last two
//     K/V tiles (kept from the producer until the store has read them) and a
//     Q warp issues its TMA store, so the softmax warps go on to the next unit
//     as soon as O is staged; the next unit's first P.V (which overwrites O)
//     waits only until the epilogue has read O out of tensor memory (`o_free`);
//   - the slot ring, the S buffers and all barrier phases continue across units.
// History tiles (the chunk's earlier keys in a sliding ring or a full cache)
// load through the cache's tensor maps, as in prefill2_kernel.
// The grid has one cluster per unit, in the order of pf_unit_of (per sequence
// and KV head, the heaviest query tiles first).  A resident cluster takes more
// units by cancelling clusters that have not started yet (cluster launch
// control): the even block's producer asks for the next unit while it loads the
// current one and hands the answer to every role of both blocks through a small
// queue in shared memory.  Every unit runs exactly once, either in its own
// cluster or in the one that cancelled it, and the hardware hands out units in
// launch order, so the load balances like a non-persistent grid.
#pragma once
#include <cuda.h>
#include "prefill.cuh"
#include "prefill2.cuh"

namespace spark {

struct PfUnit {
  int hp, qt, kvh, b;
};

// Unit u (a cluster id): head pair hp of KV head kvh of sequence b over query
// tile qt, with u = ((b * 4 + kvh) * n_qt + (n_qt - 1 - qt)) * 2 + hp.  The
// ~74 units in flight at a time read the K/V of about one KV head (it stays in
// L2), and the long (causal: late) query tiles of each come first.
__device__ __forceinline__ void pf_unit_of(const PrefillParams& P, int u, PfUnit& x) {
  x.hp = u & 1;
  int id = u >> 1;
  x.qt = P.n_qt - 1 - id % P.n_qt;
  id /= P.n_qt;
  x.kvh = id & 3;
  x.b = id >> 2;
}

// The sequence of unit u.
__device__ __forceinline__ int pf_batch_of(const PrefillParams& P, int u) { return ((u >> 1) / P.n_qt) >> 2; }

constexpr int kUq = 8;          // unit queue entries
constexpr int kUqReaders = 14;  // per entry: MMA thread, 2 Q warps, 4 softmax warps (even block);
                                // producer, 2 Q warps, 4 softmax warps (odd block)

// kHist: history tiles from the cache (sliding layers with a ring); a separate instantiation, so
// the kernel without one keeps its smaller code (it is sensitive to instruction-fetch stalls).
template <bool kHist>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPfThreads, 1)
    prefill3_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
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
  const uint32_t bar_q = misc + 80;                 // this block's Q landed (one phase per unit)
  const uint32_t bar_s = misc + 88;                 // [2], both
  const uint32_t bar_p = misc + 104;                // [2], even block's is used
  const uint32_t bar_o = misc + 120;                // [2], both
  const uint32_t bar_done = misc + 136;             // even block's
  const uint32_t bar_q_ready = misc + 144;          // both blocks' Q rotated (even block's)
  const uint32_t bar_q_free = misc + 152;           // the unit's S MMAs have read Q (both)
  const uint32_t bar_o_free = misc + 160;           // the epilogue has read O (even block's)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gmisc + 168);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gmisc + 172);
  const uint32_t bar_o_staged = misc + 176;         // this block's output staged (one phase per unit)
  const uint32_t bar_uq_full = misc + 184;          // [kUq] unit queue entry written (both)
  const uint32_t bar_uq_empty = misc + 248;         // [kUq] entry read by every role (even block's)
  const uint32_t bar_clc = misc + 312;              // cancellation answer landed (even block's)
  const uint32_t clc_resp = misc + 320;             // 16-byte cancellation answer
  // [kUq] entries of (unit id, -1: none left; the first position of its sequence)
  volatile int* uq = reinterpret_cast<volatile int*>(gmisc + 384);

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Unit u (its sequence's first position pos0, read once by the scheduler) and its schedule:
  // returns its tile count (0: a bad position, which is flagged).
  auto unit_schedule = [&](int u, int pos0, PfUnit& x, PfSchedule& S) -> int {
    pf_unit_of(P, u, x);
    const bool bad = pos0 < 0 || pos0 > kMaxPos - P.T || (P.has_cache && !P.sliding && pos0 > P.cap);
    S = pf_schedule(P, x.qt, bad ? 0 : pos0, bad ? 0 : P.T);
    if (bad) {
      S.n_tiles = 0;
      if (threadIdx.x == 0 && x.qt == 0 && x.hp == 0 && x.kvh == 0) raise_error(kErrPosition, 0x500u | (unsigned)x.b);
    }
    return S.n_tiles;
  };
  // The k-th unit id of this cluster from the queue (every lane of a warp, or one thread), and
  // the hand-back of its entry (one thread per reader).
  auto uq_get = [&](int k, int& u, int& pos0, unsigned where) -> bool {
    if (!mbar_wait_cluster(bar_uq_full + 8 * (k % kUq), (k / kUq) & 1, abort_flag, P.timeout_ns, where)) return false;
    u = uq[2 * (k % kUq)];
    pos0 = uq[2 * (k % kUq) + 1];
    return true;
  };
  auto uq_release = [&](int k) {
    if (leader) mbar_arrive(bar_uq_empty + 8 * (k % kUq));
    else mbar_arrive_remote_cluster(mapa_shared(bar_uq_empty + 8 * (k % kUq), 0));
  };

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
    mbar_init(bar_q_ready, 4);          // the Q warps (2, 3) of each block
    mbar_init(bar_q_free, 1);
    mbar_init(bar_o_free, 8);           // 4 softmax warps of each block
    mbar_init(bar_o_staged, 4);         // this block's 4 softmax warps
    for (int e = 0; e < kUq; ++e) {
      mbar_init(bar_uq_full + 8 * e, 1);
      mbar_init(bar_uq_empty + 8 * e, kUqReaders);
    }
    mbar_init(bar_clc, 1);
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

  if (warp == 0) {
    // ------------------------------------------------------ producers (both)
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      if constexpr (kHist) {
        tma_prefetch_desc(&kcmap);
        tma_prefetch_desc(&vcmap);
      }
      const int key_half = 64 * (int)rank;       // this block's keys of a K tile
      const int dim_half = 128 * (int)rank;      // this block's dims of a V tile
      int li = 0;
      bool ok = true;
      // even block: the scheduler.  Entry k of both blocks' queues gets unit k's id and its
      // sequence's first position.
      auto publish = [&](int k, int u, int pos0) -> bool {
        const int e = k % kUq;
        if (k >= kUq &&
            !mbar_wait_cluster(bar_uq_empty + 8 * e, ((k / kUq) - 1) & 1, abort_flag, P.timeout_ns, 0x8Du))
          return false;
        uq[2 * e] = u;
        uq[2 * e + 1] = pos0;
        mbar_arrive(bar_uq_full + 8 * e);
        const uint32_t peer = mapa_shared(smem_u32((const void*)(uq + 2 * e)), 1);
        asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(peer), "r"(u), "r"(pos0) : "memory");
        mbar_arrive_remote_cluster(mapa_shared(bar_uq_full + 8 * e, 1));
        return true;
      };
      int clc_asked = 0, clc_got = 0;        // cancellation requests issued / answered
      bool clc_more = true;                  // no request has come back empty yet
      int u_next = (int)(blockIdx.x >> 1);   // this cluster's own unit first
      int pos0_next = P.pos0[pf_batch_of(P, u_next)];
      if (leader) ok = publish(0, u_next, pos0_next);
      for (int k = 0; ok; ++k) {
        int u = u_next, pos0 = pos0_next;
        if (!leader) {
          ok = uq_get(k, u, pos0, 0x8Eu);
          if (!ok) break;
          uq_release(k);
        }
        if (u < 0) break;
        if (leader && clc_more) {
          // ask now for the unit after this one: a cluster that has not started gives up its own
          mbar_arrive_expect_tx(bar_clc, 16);
          asm volatile(
              "clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128 [%0], [%1];" ::"r"(
                  clc_resp),
              "r"(bar_clc)
              : "memory");
          ++clc_asked;
        }
        PfUnit x;
        PfSchedule S;
        const int n = unit_schedule(u, pos0, x, S);
        for (int step = 0; step <= n && ok; ++step) {
          for (int part = 0; part < 2 && ok; ++part) {
            const bool is_k = (part == 0);
            const int j = is_k ? step : step - 1;
            if (j < 0 || j >= n) continue;
            const PfTile t = pf_tile(S, P, j);
            const int s = li % kP2Slots;
            if (li >= kP2Slots &&
                !mbar_wait(bar_slot_empty + 8 * s, ((li / kP2Slots) - 1) & 1, abort_flag, P.timeout_ns, 0x81u)) {
              ok = false;
              break;
            }
            const uint32_t dst = slots + s * kP2SlotBytes;
            const uint32_t full0 = mapa_shared(bar_slot_full + 8 * s, 0);
            if (leader) mbar_arrive_expect_tx(bar_slot_full + 8 * s, 2 * kP2SlotBytes);
            if (is_k) {
              for (int xx = 0; xx < 4; ++xx)
                if (kHist && t.hist)
                  tma2_load_3d(dst + xx * 8192, &kcmap, full0, xx * 64, t.row + key_half, x.b * kNkv + x.kvh);
                else
                  tma2_load_4d(dst + xx * 8192, &kmap, full0, xx * 64, x.kvh, t.row + key_half, x.b);
            } else {
              for (int xx = 0; xx < 4; ++xx)
                for (int d = 0; d < 2; ++d) {
                  if (kHist && t.hist)
                    tma2_load_3d(dst + xx * 8192 + d * 4096, &vcmap, full0, dim_half + 64 * d, t.row + 32 * xx,
                                 x.b * kNkv + x.kvh);
                  else
                    tma2_load_4d(dst + xx * 8192 + d * 4096, &vmap, full0, dim_half + 64 * d, x.kvh, t.row + 32 * xx,
                                 x.b);
                }
            }
            ++li;
          }
        }
        if (leader && ok) {
          u_next = -1;
          pos0_next = 0;
          if (clc_more) {
            ok = mbar_wait(bar_clc, clc_got & 1, abort_flag, P.timeout_ns, 0x8Fu);
            if (!ok) break;
            ++clc_got;
            uint32_t cx, valid;
            asm volatile(
                "{\n\t.reg .pred p;\n\t.reg .b128 r;\n\t"
                "ld.shared.b128 r, [%2];\n\t"
                "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, r;\n\t"
                "selp.u32 %1, 1, 0, p;\n\t"
                "mov.u32 %0, 0;\n\t"
                "@p clusterlaunchcontrol.query_cancel.get_first_ctaid::x.b32.b128 %0, r;\n\t}"
                : "=r"(cx), "=r"(valid)
                : "r"(clc_resp)
                : "memory");
            fence_proxy_async_smem();      // the next answer overwrites the buffer
            if (valid) u_next = (int)(cx >> 1);
            else clc_more = false;
          }
          if (u_next >= 0) pos0_next = P.pos0[pf_batch_of(P, u_next)];
          ok = publish(k + 1, u_next, pos0_next);
        }
      }
      // an unanswered cancellation request must land before the block leaves
      if (leader && clc_asked > clc_got) mbar_drain(bar_clc, clc_got & 1, 200000000ull);
      // never leave with copies in flight: (even block) every slot's bytes
      if (leader) {
        for (int i = max(0, li - kP2Slots); i < li; ++i)
          if (!mbar_drain(bar_slot_full + 8 * (i % kP2Slots), (i / kP2Slots) & 1, 200000000ull)) break;
      } else if (!ok) {
        __nanosleep(200000);   // aborted: let this block's last copies land before the pair leaves
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------- MMA issuer (even block)
    if (lane == 0 && leader) {
      int li = 0, jg = 0, qu = 0, li_end = 0;
      bool ok = true;
      const uint64_t dq = smem_desc_sw128(q_s, 16, 1024);
      // the unit's last two tiles' slots are released by the output store, not here
      auto issue_s = [&](int jgl) -> bool {
        const uint32_t dcol = tmem + kSCol + 128u * (jgl & 1);
        const int s = li % kP2Slots;
        if (!mbar_wait(bar_slot_full + 8 * s, (li / kP2Slots) & 1, abort_flag, P.timeout_ns, 0x82u)) return false;
        tc_fence_after();
        const uint64_t dk = smem_desc_sw128(slots + s * kP2SlotBytes, 16, 1024);
#pragma unroll
        for (int d = 0; d < 4; ++d)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma2_ss(dcol, dq + (uint64_t)((d * 16384 + kk * 32) >> 4), dk + (uint64_t)((d * 8192 + kk * 32) >> 4),
                     kIdescQK2, (d | kk) != 0);
        if (li < li_end - 2) umma2_commit_mc(bar_slot_empty + 8 * s, 3);
        umma2_commit_mc(bar_s + 8 * (jgl & 1), 3);
        ++li;
        return true;
      };
      auto issue_pv = [&](int jgl, bool first) -> bool {
        if (!mbar_wait_cluster(bar_p + 8 * (jgl & 1), (jgl >> 1) & 1, abort_flag, P.timeout_ns, 0x83u)) return false;
        const int s = li % kP2Slots;
        if (!mbar_wait(bar_slot_full + 8 * s, (li / kP2Slots) & 1, abort_flag, P.timeout_ns, 0x84u)) return false;
        tc_fence_after();
        const uint32_t pcol = tmem + kSCol + 128u * (jgl & 1);
        const uint64_t dv = smem_desc_sw128(slots + s * kP2SlotBytes, 4096, 1024);
#pragma unroll
        for (int v = 0; v < 4; ++v)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma2_ts(tmem + kOCol, pcol + 16u * v + 8u * kk, dv + (uint64_t)((v * 8192 + kk * 2048) >> 4), kIdescPV2,
                     (!first || v > 0 || kk > 0) ? 1u : 0u);
        if (li < li_end - 2) umma2_commit_mc(bar_slot_empty + 8 * s, 3);
        umma2_commit_mc(bar_o + 8 * (jgl & 1), 3);
        ++li;
        return true;
      };
      for (int k = 0; ok; ++k) {
        int u, pos0;
        if (!uq_get(k, u, pos0, 0x90u)) break;
        uq_release(k);
        if (u < 0) break;
        PfUnit x;
        PfSchedule S;
        const int n = unit_schedule(u, pos0, x, S);
        if (n == 0) continue;
        li_end = li + 2 * n;
        ok = mbar_wait_cluster(bar_q_ready, qu & 1, abort_flag, P.timeout_ns, 0x85u);
        tc_fence_after();
        if (ok) ok = issue_s(jg);
        if (ok && n == 1) umma2_commit_mc(bar_q_free, 3);      // the unit's last S is issued
        for (int j = 0; j < n && ok; ++j) {
          if (j + 1 < n) {
            ok = issue_s(jg + j + 1);
            if (ok && j + 2 == n) umma2_commit_mc(bar_q_free, 3);
          }
          // the first P.V of a unit overwrites O: the previous unit's epilogue must have read it
          if (ok && j == 0 && qu > 0) ok = mbar_wait_cluster(bar_o_free, (qu - 1) & 1, abort_flag, P.timeout_ns, 0x86u);
          if (ok) ok = issue_pv(jg + j, j == 0);
        }
        jg += n;
        ++qu;
      }
      umma2_commit_mc(bar_done, 1);
      mbar_drain(bar_done, 0, 200000000ull);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ---------------------------------- Q warps (both): each unit's Q loaded (thread 64, as soon as
    // the previous unit's S MMAs have read the Q buffer, so the producer never waits for that),
    // rotated (RoPE at load, the whole tile: these warps are otherwise idle, so the rotation of
    // the next unit's Q overlaps the current unit's work), handed to the MMA thread; then (thread
    // 64) the TMA store of the previous unit's staged output, after which its two slots go back to
    // the producer.  In time, unit k+1's Q lands before unit k's output is staged.
    int qu = 0, li = 0, q_issued = 0;
    bool ok = true;
    PfUnit px{0, 0, 0, 0};      // the unit whose output is to be stored
    int p_end = -1;             // its slot counter past its last tile (-1: none)
    auto store_prev = [&]() -> bool {
      if (p_end < 0) return true;
      bool good = true;
      if (threadIdx.x == 64) {
        good = mbar_wait(bar_o_staged, (qu - 2) & 1, abort_flag, P.timeout_ns, 0x8Cu);
        if (good) {
          const int h = px.kvh * 4 + px.hp * 2 + (int)rank;
          for (int d = 0; d < 4; ++d) {
            const int s = (p_end - 2 + (d >> 1)) % kP2Slots;
            tma_store_4d(&omap, slots + s * kP2SlotBytes + (d & 1) * 16384, d * 64, h, px.qt * kPfM, px.b);
          }
          bulk_commit_group();
          bulk_wait_group_read0();
          mbar_arrive(bar_slot_empty + 8 * ((p_end - 2) % kP2Slots));
          mbar_arrive(bar_slot_empty + 8 * ((p_end - 1) % kP2Slots));
        }
      }
      p_end = -1;
      return __all_sync(0xffffffffu, good);
    };
    for (int k = 0; ok; ++k) {
      int u, pos0;
      if (!__all_sync(0xffffffffu, uq_get(k, u, pos0, 0x91u))) {
        ok = false;
        break;
      }
      __syncwarp();
      if (lane == 0) uq_release(k);
      if (u < 0) break;
      PfUnit x;
      PfSchedule S;
      const int n = unit_schedule(u, pos0, x, S);
      if (n == 0) continue;
      if (threadIdx.x == 64) {
        // this block's Q tile, once the previous unit's S MMAs have read the buffer
        if (qu > 0 && !mbar_wait(bar_q_free, (qu - 1) & 1, abort_flag, P.timeout_ns, 0x80u)) {
          ok = false;
        } else {
          const int h = x.kvh * 4 + x.hp * 2 + (int)rank;
          mbar_arrive_expect_tx(bar_q, kPfQBytes);
          for (int d = 0; d < 4; ++d) tma_load_4d(q_s + d * 16384, &qmap, bar_q, d * 64, h, x.qt * kPfM, x.b);
          ++q_issued;
        }
      }
      if (!__all_sync(0xffffffffu, ok) ||
          !__all_sync(0xffffffffu, mbar_wait(bar_q, qu & 1, abort_flag, P.timeout_ns, 0x87u))) {
        ok = false;
        break;
      }
      if (P.rope) {
        rope_q_tile(gbase, P, S.qp0, threadIdx.x - 64, 64);
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(bar_q_ready);
        else mbar_arrive_remote_cluster(mapa_shared(bar_q_ready, 0));
      }
      ++qu;
      if (warp == 2) ok = store_prev();
      li += 2 * n;
      px = x;
      p_end = li;
    }
    if (warp == 2 && ok) {
      ++qu;                     // the last unit's phase of bar_o_staged is qu - 1
      store_prev();
    }
    if (threadIdx.x == 64) {
      bulk_wait_group0();       // never leave with a store in flight,
      // nor with a Q load in flight (only after an abort: otherwise every issued Q was waited for)
      if (!ok && q_issued > 0) mbar_drain(bar_q, (q_issued - 1) & 1, 200000000ull);
    }
  } else {
    // ------------------------------------------------- softmax warps (both)
    const int r = threadIdx.x - 128;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ocol = tmem + lane_base + kOCol;
    const uint32_t p_ready0 = mapa_shared(bar_p, 0);
    const uint32_t o_free0 = mapa_shared(bar_o_free, 0);
    int jg = 0, qu = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int u, pos0;
      if (!__all_sync(0xffffffffu, uq_get(k, u, pos0, 0x91u))) {
        ok = false;
        break;
      }
      __syncwarp();
      if (lane == 0) uq_release(k);
      if (u < 0) break;
      PfUnit x;
      PfSchedule S;
      const int n = unit_schedule(u, pos0, x, S);
      if (n == 0) continue;
      const int h = x.kvh * 4 + x.hp * 2 + (int)rank;
      const int qp = S.qp0 + r;
      const bool row_valid = qp < S.pos0 + S.T;
      // the row's gate logit, read now (its latency hides behind the unit) and used at the epilogue
      const float gl =
          row_valid ? __bfloat162float(P.gate[((long long)x.b * P.T + (qp - S.pos0)) * kNq + h]) : 0.f;
      float m_ref = -INFINITY, l_run = 0.f;
      for (int j = 0; j < n && ok; ++j) {
        const int jgl = jg + j;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(bar_s + 8 * (jgl & 1), (jgl >> 1) & 1, abort_flag, P.timeout_ns, 0x89u))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t scol = tmem + lane_base + kSCol + 128u * (jgl & 1);
        const PfTile t = pf_tile(S, P, j);
        // the previous P.V (tile j-1) must be complete before O is rescaled
        if (!pf_softmax_tile<true>(scol, ocol, t, S, P, qp, m_ref, l_run, bar_o + 8 * ((jgl - 1) & 1),
                                 ((jgl - 1) >> 1) & 1, abort_flag, 0x8Au)) {
          ok = false;
          break;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader) mbar_arrive(bar_p + 8 * (jgl & 1));
          else mbar_arrive_remote(p_ready0 + 8 * (jgl & 1));
        }
      }
      if (!ok) break;
      // epilogue: out = O / l * sigmoid(gate) in bf16, staged in the slots of the unit's last two
      // tiles (dims 0-127, then 128-255: two [128 x 64] 128-byte-swizzled boxes each; both tiles'
      // MMAs have completed) for the Q warp's TMA store, which clips rows past the chunk
      const int jl = jg + n - 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_o + 8 * (jl & 1), (jl >> 1) & 1, abort_flag, P.timeout_ns, 0x8Bu))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float scale = row_valid ? (l_run > 0.f ? 1.f / l_run : 0.f) * (1.f / (1.f + expf(-gl))) : 0.f;
      const int li_end = 2 * (jg + n);
      uint8_t* const gslots = gbase + kPfQBytes;
      auto stage = [&](const uint32_t* ov, int cc) {
        uint8_t* box = gslots + ((li_end - 2 + (cc >> 2)) % kP2Slots) * kP2SlotBytes + ((cc >> 1) & 1) * 16384 + r * 128;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint4 w;
          w.x = pack_bf16(__uint_as_float(ov[8 * e + 0]) * scale, __uint_as_float(ov[8 * e + 1]) * scale);
          w.y = pack_bf16(__uint_as_float(ov[8 * e + 2]) * scale, __uint_as_float(ov[8 * e + 3]) * scale);
          w.z = pack_bf16(__uint_as_float(ov[8 * e + 4]) * scale, __uint_as_float(ov[8 * e + 5]) * scale);
          w.w = pack_bf16(__uint_as_float(ov[8 * e + 6]) * scale, __uint_as_float(ov[8 * e + 7]) * scale);
          const int chunk = (cc & 1) * 4 + e;     // 16-byte chunk within the 128-byte row of the box
          *reinterpret_cast<uint4*>(box + ((chunk ^ (r & 7)) << 4)) = w;
        }
      };
      // two 32-column reads of O in flight: chunk cc+1 loads while chunk cc is staged
      uint32_t ova[32], ovb[32];
      tmem_ld32(ocol, ova);
#pragma unroll 1
      for (int cc = 0; cc < 8; cc += 2) {
        tmem_wait_ld();
        tmem_ld32(ocol + 32 * (cc + 1), ovb);
        stage(ova, cc);
        tmem_wait_ld();
        if (cc + 2 < 8) {
          tmem_ld32(ocol + 32 * (cc + 2), ova);
        } else {
          // every read of O has landed: the next unit's first P.V may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (leader) mbar_arrive(bar_o_free);
            else mbar_arrive_remote(o_free0);
          }
        }
        stage(ovb, cc + 1);
      }
      fence_proxy_async_smem();                   // make the staged rows visible to the TMA store
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_o_staged);
      jg += n;
      ++qu;
    }
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
