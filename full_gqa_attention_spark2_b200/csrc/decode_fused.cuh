// One launch per decode layer: the append of the new token, the split-KV
// attention over the cache and the log-sum-exp combine of the splits.
//
// Work.  A block is (split s, KV head g, sequence b), as in
// decode_partial_kernel: the four query heads of the group against tiles
// [s * tiles_per_split, (s + 1) * tiles_per_split) of that head's cache rows,
// streamed through three TMA stages.  The consumers are kG groups of kW warps;
// group j takes tiles j, j + kG, .. (each warp 16 keys of a 16 kW key tile),
// so kG tiles are worked on at once.  Two shapes:
//   kW = 4, kG = 1: 64-key tiles (192 KB of stages: one block per SM) and a
//     producer warp that streams them;
//   kW = 2, kG = 2: 32-key tiles (96 KB: two blocks per SM) and no producer
//     warp: the group that frees a stage issues the load of the tile three
//     ahead into it.  Two blocks of four warps keep two warps per scheduler,
//     so a thread keeps its 255 registers (a fifth warp would cap it at 168).
// Sliding layers use the second: at B=64 their 256 units of 512 keys then run
// as one wave of 256 blocks on 148 SMs instead of 1.7 waves of one block per
// SM.  The hardware deals the blocks to the SMs as they free up, which keeps
// SMs of unequal speed busy to the end.
//
// The new token.  Its key and value are taken from the call's k and v
// (rotated here when asked), not read back from the cache: the block of a
// unit's last split adds the token to its running softmax and writes it into
// the cache row (full: row = position; sliding: the ring row position mod
// 512, whose old entry has just left the window and is masked in the tiles).
// Cache rows are visible when row < row_end and row != hole:
//   full:    row_end = p, no hole;
//   sliding: row_end = min(p, 512), hole = p mod 512 once the ring has wrapped.
// So attention sees exactly positions max(0, p - 511)..p (sliding) or 0..p
// (full), as append-then-attend does ("Spark-X2.6-4B-Base" page §滑动窗口 512
// and §36 层混合注意力排布).
//
// Combine.  With one split the block normalises, gates and writes the output
// itself.  Otherwise each block writes its partial (m, l, o[256] per query
// head) to the workspace and adds one to its unit's arrival counter; the block
// that brings the counter to the number of splits merges the unit's partials,
// writes the output and sets the counter back to zero.  No block waits for
// another.
//
// Launch order.  The kernel is launched with programmatic stream
// serialisation: a block sets up its barriers and prefetches its tensor maps,
// then waits (griddepcontrol.wait) for the previous kernel of the stream to
// finish before it reads an input or writes anything, and lets the next one
// be scheduled (griddepcontrol.launch_dependents), so a layer's launch and
// set-up overlap the previous layer's last blocks.
#pragma once
#include <cuda.h>
#include "decode.cuh"

namespace spark {

template <int kW, int kG>
struct DfShape {
  static constexpr int kNK = 16 * kW;                      // keys per tile
  static constexpr int kNW = kW * kG;                      // consumer warps
  static constexpr bool kProducer = kG == 1;               // a producer warp (else the groups issue)
  static constexpr int kThreads = (kNW + (kProducer ? 1 : 0)) * 32;
  static constexpr int kBoxBytes = kNK * 128;              // one 64-dim box of the tile
  static constexpr int kTileBytes = 4 * kBoxBytes;         // K (or V) of one tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kMiscBytes = 5120;                  // q rows, new k/v, RoPE angles, barriers, m/l, flags
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kDecStages * kStageBytes + kMiscBytes;
  // the warps' merge reuses the stages once every tile has been consumed
  static_assert(kNW * 4 * kHeadDim * 4 <= kDecStages * kStageBytes, "merge area");
  static_assert(kNW <= 4, "one query head per consumer warp in the merge");
};

struct DecodeFusedParams {
  const __nv_bfloat16* q;      // [B][16][256], sequence b at element b * q_sB
  const __nv_bfloat16* k_new;  // [B][4][256], sequence b at element b * kv_sB
  const __nv_bfloat16* v_new;  // [B][4][256], as k_new
  long long q_sB, kv_sB;
  const __nv_bfloat16* gate;   // [B][16]
  const int* pos;              // [B]
  __nv_bfloat16* out;          // [B][16][256]
  __nv_bfloat16* k_cache;      // [B][4][cap][256]
  __nv_bfloat16* v_cache;
  float* o_part;               // [B][16][splits][256]
  float* ml_part;              // [B][16][splits][2]
  int* cnt;                    // [B * 4], zero between calls
  int B, cap, sliding, n_splits, tiles_per_split, rope, rot;
  unsigned long long timeout_ns;
  RopeFreq freq;
};

// Named barrier of the consumer warps (barrier 1, n threads).
template <int kN>
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kN) : "memory");
}

template <int kW, int kG>
__global__ void __launch_bounds__(DfShape<kW, kG>::kThreads, kW == 2 ? 2 : 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                        const DecodeFusedParams P) {
  using S = DfShape<kW, kG>;
  constexpr int kNK = S::kNK;
  constexpr int kNW = S::kNW;
  constexpr int kNC = 32 * kNW;                // consumer threads
  extern __shared__ uint8_t dsmem[];
  const uint32_t raw = smem_u32(dsmem);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = dsmem + (base - raw);
  // layout: [stages x (K tile | V tile)] (the merge area once every tile is consumed) |
  //         q rows, new k/v, RoPE angles, barriers, abort, m, l, flag
  float* mrg_o = reinterpret_cast<float*>(gbase);
  uint8_t* misc = gbase + kDecStages * S::kStageBytes;
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(misc);            // [4][256], q / 16
  __nv_bfloat16* kn_s = reinterpret_cast<__nv_bfloat16*>(misc + 2048);   // [256], the new key (rotated)
  __nv_bfloat16* vn_s = reinterpret_cast<__nv_bfloat16*>(misc + 2560);   // [256], the new value
  float2* rtab = reinterpret_cast<float2*>(misc + 3072);                 // [128] angles of position p
  const uint32_t bar_full = smem_u32(misc + 4096);
  const uint32_t bar_empty = bar_full + 8 * kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4096 + 16 * kDecStages);
  volatile int* last_flag = abort_flag + 1;
  int* max_issued = const_cast<int*>(abort_flag) + 2;                  // last tile loaded (no producer)
  float* sm_m = reinterpret_cast<float*>(misc + 4096 + 16 * kDecStages + 16);
  float* sm_l = sm_m + 4 * kNW;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kW);      // the warps of the group that owns the tile
    }
    *abort_flag = 0;
    *max_issued = -1;
    fence_mbar_init();
  }
  if (threadIdx.x == (S::kProducer ? kNC : 0)) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  __syncthreads();
  // past this point the previous kernel of the stream has finished and its writes are visible; the
  // next one may be scheduled now (it waits the same way before it touches memory)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int p = P.pos[b];
  const bool bad = p < 0 || p >= kMaxPos || (!P.sliding && p >= P.cap);
  const int row_end = bad ? 0 : (P.sliding ? min(p, kWindow) : p);
  const int hole = (!bad && P.sliding && p >= kWindow) ? (p & (kWindow - 1)) : -1;
  const int t_lo = split * P.tiles_per_split;
  const int t_hi = min((split + 1) * P.tiles_per_split, (row_end + kNK - 1) / kNK);
  const int n_tiles = max(0, t_hi - t_lo);
  const bool last_split = split == P.n_splits - 1;      // adds and writes the new token
  if (bad && last_split && g == 0 && threadIdx.x == 0) raise_error(kErrPosition, 0x340u | (unsigned)b);

  // tile i of this block into stage i % 3 (one thread)
  auto load_tile = [&](int i) {
    const int s = i % kDecStages;
    const uint32_t full = bar_full + 8 * s;
    mbar_arrive_expect_tx(full, S::kStageBytes);
    const uint32_t kt = base + s * S::kStageBytes;
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      tma_load_3d(kt + d * S::kBoxBytes, &kmap, full, d * 64, (t_lo + i) * kNK, b * kNkv + g);
      tma_load_3d(kt + S::kTileBytes + d * S::kBoxBytes, &vmap, full, d * 64, (t_lo + i) * kNK, b * kNkv + g);
    }
  };
  if constexpr (!S::kProducer) {
    if (threadIdx.x == 0 && n_tiles > 0) {
      for (int i = 0; i < min(n_tiles, kDecStages); ++i) load_tile(i);
      atomicMax(max_issued, min(n_tiles, kDecStages) - 1);
    }
  }

  if (S::kProducer && warp == kNW) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_tiles > 0) {
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kDecStages;
        if (i >= kDecStages &&
            !mbar_wait(bar_empty + 8 * s, ((i / kDecStages) - 1) & 1, abort_flag, P.timeout_ns, 0x20u))
          break;
        load_tile(i);
        issued = i + 1;
      }
      // never leave with copies in flight
      for (int i = max(0, issued - kDecStages); i < issued; ++i)
        if (!mbar_drain(bar_full + 8 * (i % kDecStages), (i / kDecStages) & 1, 200000000ull)) break;
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = threadIdx.x;
  // the rotation of position p, for q and the new key
  if (P.rope && !bad) {
    dec_rope_table(rtab, p, P.rot, P.freq, tid, kNC);
    consumers_sync<kNC>();
  }
  dec_stage_q(qs, P.q + (long long)b * P.q_sB + g * 4 * kHeadDim, rtab, P.rope && !bad, P.rot, tid, kNC);
  if (last_split && !bad) {
    // the new token of (b, g): k rotated as the append kernel rotates it, v as it is; staged for its
    // score below and written into its cache row
    const long long src = (long long)b * P.kv_sB + g * kHeadDim;
    const int row = P.sliding ? (p & (kWindow - 1)) : p;
    const long long dst = (((long long)b * kNkv + g) * P.cap + row) * kHeadDim;
    for (int ch = tid; ch < 64; ch += kNC) {
      if (ch < 32) {
        const uint4 x = reinterpret_cast<const uint4*>(P.v_new + src)[ch];
        reinterpret_cast<uint4*>(vn_s)[ch] = x;
        reinterpret_cast<uint4*>(P.v_cache + dst)[ch] = x;
        continue;
      }
      const int c = ch - 32;                           // 16-byte chunk of k: dims 8 c .. 8 c + 7
      const int half = P.rot >> 1;
      const uint4* ks = reinterpret_cast<const uint4*>(P.k_new + src);
      if (!P.rope || c * 8 >= P.rot) {
        const uint4 x = ks[c];
        reinterpret_cast<uint4*>(kn_s)[c] = x;
        reinterpret_cast<uint4*>(P.k_cache + dst)[c] = x;
      } else if (c * 8 < half) {
        const int pc = c + (half >> 3);                // the chunk holding the partner dims
        uint4 lo = ks[c], hi = ks[pc];
        uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
        uint32_t* hv = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i0 = c * 8 + 2 * e;
          const float2 a0 = rtab[i0], a1 = rtab[i0 + 1];   // the append kernel's angles, bit for bit
          const float l0 = bf16_lo(l[e]), l1 = bf16_hi(l[e]), h0 = bf16_lo(hv[e]), h1 = bf16_hi(hv[e]);
          l[e] = pack_bf16(rope_lo(l0, h0, a0.x, a0.y), rope_lo(l1, h1, a1.x, a1.y));
          hv[e] = pack_bf16(rope_hi(l0, h0, a0.x, a0.y), rope_hi(l1, h1, a1.x, a1.y));
        }
        reinterpret_cast<uint4*>(kn_s)[c] = lo;
        reinterpret_cast<uint4*>(kn_s)[pc] = hi;
        reinterpret_cast<uint4*>(P.k_cache + dst)[c] = lo;
        reinterpret_cast<uint4*>(P.k_cache + dst)[pc] = hi;
      }
    }
  }
  consumers_sync<kNC>();
  uint32_t qa[16][2];
  dec_q_fragments(qs, lane, qa);

  float o[16][4];
#pragma unroll
  for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m_run = -INFINITY, l_part = 0.f;
  bool ok = true;
  const int grp = warp / kW, wl = warp % kW;    // tile group, warp within it
  for (int i = grp; i < n_tiles; i += kG) {
    const int s = i % kDecStages;
    // Without a producer, a stage serves the two groups in turn, so this group can reach tile i while
    // the stage's previous tile (the other group's) is still in flight; the full barrier's parity
    // would then name that earlier phase.  Waiting first until the other group has released the
    // stage (its empty phase cannot run ahead: the next one needs this group) makes the full wait
    // name this tile's phase.
    if (!S::kProducer && i >= kDecStages &&
        !__all_sync(0xffffffffu, mbar_wait(bar_empty + 8 * s, ((i / kDecStages) - 1) & 1, abort_flag,
                                           P.timeout_ns, 0x24u))) {
      ok = false;
      break;
    }
    if (!__all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, (i / kDecStages) & 1, abort_flag, P.timeout_ns,
                                           0x22u))) {
      ok = false;           // the other warps see the abort flag at their next wait
      break;
    }
    const uint32_t kt = base + s * S::kStageBytes;
    dec_consume_tile<kNK>(kt, kt + S::kTileBytes, qa, o, m_run, l_part, (t_lo + i) * kNK, row_end, hole, wl,
                          lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    if (!S::kProducer && wl == 0 && lane == 0 && i + kDecStages < n_tiles) {
      // the group's warps are done with the stage: load the tile three ahead into it
      if (mbar_wait(bar_empty + 8 * s, (i / kDecStages) & 1, abort_flag, P.timeout_ns, 0x23u)) {
        load_tile(i + kDecStages);
        atomicMax(max_issued, i + kDecStages);
      } else {
        ok = false;
      }
    }
    if (!S::kProducer && !__all_sync(0xffffffffu, ok)) break;
  }
  {
    // every consumer thread reaches this barrier; a wait that ran out in any warp ends the block here
    uint32_t all_ok;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(all_ok)
        : "r"((uint32_t)ok), "n"(kNC)
        : "memory");
    if (!all_ok) {
      if (!S::kProducer && tid == 0) {
        // never leave with copies in flight: only the last three loads can be outstanding
        const int mi = *max_issued;
        for (int j = max(0, mi - (kDecStages - 1)); j <= mi; ++j)
          mbar_drain(bar_full + 8 * (j % kDecStages), (j / kDecStages) & 1, 200000000ull);
      }
      return;
    }
  }

  // -------------------------------------------- merge the consumer warps
  float ms[4 / kNW], ls[4 / kNW], acc[4 / kNW][8];
  dec_merge_warps<kNW>(mrg_o, sm_m, sm_l, o, m_run, l_part, warp, lane, ms, ls, acc);
#pragma unroll
  for (int i = 0; i < 4 / kNW; ++i) {
    const int hh = warp + kNW * i;
    if (last_split && !bad) {
      // the new token: its score from the same bf16 q / 16 and rotated bf16 key, summed in fp32
      float sdot = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int d = lane + 32 * k;
        sdot = fmaf(__bfloat162float(qs[hh * kHeadDim + d]), __bfloat162float(kn_s[d]), sdot);
      }
#pragma unroll
      for (int sh = 16; sh > 0; sh >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, sh);
      const float s_new = sdot * 1.4426950408889634f;
      const float m2 = fmaxf(ms[i], s_new);
      const float e_old = (ms[i] == -INFINITY) ? 0.f : fast_exp2(ms[i] - m2);
      const float e_new = fast_exp2(s_new - m2);
      ls[i] = ls[i] * e_old + e_new;
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[i][k] = acc[i][k] * e_old + e_new * __bfloat162float(vn_s[lane + 32 * k]);
      ms[i] = m2;
    }
    const long long bh = (long long)b * kNq + g * 4 + hh;
    if (P.n_splits == 1) {
      const float scale = decode_out_scale(ls[i], P.gate[bh]);
#pragma unroll
      for (int k = 0; k < 8; ++k) P.out[bh * kHeadDim + lane + 32 * k] = __float2bfloat16_rn(acc[i][k] * scale);
    } else {
      float* dst = P.o_part + (bh * P.n_splits + split) * kHeadDim;
#pragma unroll
      for (int k = 0; k < 8; ++k) dst[lane + 32 * k] = acc[i][k];
      if (lane == 0) {
        P.ml_part[(bh * P.n_splits + split) * 2 + 0] = ms[i];
        P.ml_part[(bh * P.n_splits + split) * 2 + 1] = ls[i];
      }
    }
  }
  if (P.n_splits == 1) return;

  // ------------------------- arrival; the unit's last block merges the splits
  __threadfence();
  consumers_sync<kNC>();
  const int unit = b * kNkv + g;
  if (tid == 0) *last_flag = atomicAdd(P.cnt + unit, 1) == P.n_splits - 1;
  consumers_sync<kNC>();
  if (!*last_flag) return;
  __threadfence();
#pragma unroll
  for (int i = 0; i < 4 / kNW; ++i) {
    const int hh = warp + kNW * i;
    const long long bh = (long long)b * kNq + g * 4 + hh;
    const long long r0 = bh * P.n_splits;
    float mm = -INFINITY;
#pragma unroll 4
    for (int s = 0; s < P.n_splits; ++s) mm = fmaxf(mm, __ldcg(P.ml_part + (r0 + s) * 2));
    float L = 0.f, A[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int s = 0; s < P.n_splits; ++s) {
      const float m = __ldcg(P.ml_part + (r0 + s) * 2);
      const float e = (m == -INFINITY) ? 0.f : fast_exp2(m - mm);
      L += e * __ldcg(P.ml_part + (r0 + s) * 2 + 1);
      const float* ps = P.o_part + (r0 + s) * kHeadDim;
#pragma unroll
      for (int k = 0; k < 8; ++k) A[k] += e * __ldcg(ps + lane + 32 * k);
    }
    const float scale = decode_out_scale(L, P.gate[bh]);
#pragma unroll
    for (int k = 0; k < 8; ++k) P.out[bh * kHeadDim + lane + 32 * k] = __float2bfloat16_rn(A[k] * scale);
  }
  if (tid == 0) P.cnt[unit] = 0;         // ready for the next call
}

}  // namespace spark
