// Split-KV decode ("flash decoding") for one new token per sequence.
//
// Work unit: (sequence b, KV head g, split s).  The four query heads 4g..4g+3
// that share KV head g ("Spark-X2.6-4B-Base" page §配套效率设计: 16 query heads
// share 4 KV heads) are packed into one pass over that head's keys, so every
// K/V byte is read from HBM once per step.  The pass is HBM-bound: per key it
// reads 1 KB (K and V, 256 dims, bf16) and does 4 KFLOP.
//
// Data path per block: one producer warp streams 64-key K and V tiles with
// TMA (128-byte swizzled, 3 stages of 64 KB) into shared memory; four
// consumer warps each take 16 keys of a tile and do
//     S  = Q K^T        mma.m16n8k16, A = the 4 query rows (padded to 16),
//                       B = K straight from the swizzled tile (ldmatrix)
//     online softmax    fp32, exp2 domain
//     O^T += V^T P^T    A = V^T via ldmatrix.trans, B = P from S's registers
// then the four warps merge in shared memory and the block writes an
// unnormalised partial (m, l, o[256]) per query head.  A second kernel merges
// the splits with a log-sum-exp and applies the sigmoid gate.
#pragma once
#include <cuda.h>
#include "ptx.cuh"
#include "rope_append.cuh"

namespace spark {

constexpr int kDecNK = 64;                                   // keys per tile
constexpr int kDecStages = 3;
constexpr int kDecConsumerWarps = 4;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;    // + 1 producer warp
constexpr int kDecTileBytes = kDecNK * kHeadDim * 2;         // 32 KB (K or V)
constexpr int kDecBoxBytes = kDecNK * 128;                   // one 64-dim box: 8 KB
constexpr int kDecStageBytes = 2 * kDecTileBytes;
constexpr int kDecMergeBytes = kDecConsumerWarps * 4 * kHeadDim * 4;   // 16 KB
constexpr int kDecSmemBytes = 1024 /*align slack*/ + kDecStages * kDecStageBytes +
                              kDecMergeBytes + 1024 /*q, barriers, m/l*/;

struct DecodeParams {
  const __nv_bfloat16* q;     // [B][16][256], sequence b at element b * q_sB
  long long q_sB;
  const int* pos;             // [B]
  float* o_part;              // [B][16][splits][256]
  float* ml_part;             // [B][16][splits][2]
  __nv_bfloat16* out;         // [B][16][256], written here when n_splits == 1
  const __nv_bfloat16* gate;  // [B][16]
  int B, cap, sliding, n_splits, tiles_per_split;
  int rope, rot;
  double log2_theta;
  unsigned long long timeout_ns;
  RopeFreq freq;
  // paged caches only: pool [n_pages][4][page][256]; logical row r of sequence b
  // lives in page block_table[b * max_pages + r / page] at row r % page
  const int* block_table;
  int max_pages, page_shift, n_pages;
  // context parallelism (full layers): this cache holds positions key_off ..
  // key_off + cap - 1 of a cache sharded across ranks (row = position -
  // key_off); a query sees the rows up to its own position, none when it lies
  // before the shard.  The partials are always left for decode_cp_reduce_kernel.
  int key_off, shard;
};

// TMA coordinates of the 64 keys that start at logical row `row0` of
// (sequence b, KV head g): a dense cache is 3-D (dim, row, b * 4 + g), a paged
// pool 4-D (dim, row in page, head, page).  `ok` is false for a page index
// outside the pool.
struct KvTile {
  int c1, c2, c3;
  bool ok;
};

template <bool kPaged>
__device__ __forceinline__ KvTile kv_tile(const DecodeParams& P, int b, int g, int row0) {
  if (!kPaged) return KvTile{row0, b * kNkv + g, 0, true};
  const int pg = P.block_table[(long long)b * P.max_pages + (row0 >> P.page_shift)];
  return KvTile{row0 & ((1 << P.page_shift) - 1), g, pg, pg >= 0 && pg < P.n_pages};
}

template <bool kPaged>
__device__ __forceinline__ void kv_tile_load(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x,
                                             const KvTile& t) {
  if (kPaged)
    tma_load_4d(dst, map, bar, x, t.c1, t.c2, t.c3);
  else
    tma_load_3d(dst, map, bar, x, t.c1, t.c2);
}

// Factor of the merged numerator: 1 / (softmax denominator) times the
// sigmoid of the head's gate logit; 0 for a row that saw no key.
__device__ __forceinline__ float decode_out_scale(float l, __nv_bfloat16 gate_logit) {
  const float gl = __bfloat162float(gate_logit);
  return (l > 0.f) ? (1.f / l) * (1.f / (1.f + expf(-gl))) : 0.f;
}

// Byte address of (key, dim) in a tile of four [kNK keys x 128 B] boxes (one per 64 dims) with
// the 128-byte swizzle.
template <int kNK = kDecNK>
__device__ __forceinline__ uint32_t swz_addr(uint32_t tile, int key, int dim) {
  return tile + (uint32_t)(dim >> 6) * (uint32_t)(kNK * 128) + (uint32_t)key * 128u +
         ((uint32_t)(((dim & 63) >> 3) ^ (key & 7)) << 4);
}

// ----------------------------------------------- consumer steps, shared ----
// The decode kernels' consumer warps, kW of them, each take 16 keys of every kNK = 16 kW key tile.

// The rotation of position p: (cos, sin) of p f_i for the rot/2 frequencies, one angle per
// thread (an fp64 reduction and sincosf each, as the RoPE and append kernels compute them), into
// tab[rot/2] in shared memory.  A block's q rows and new key all turn by these rot/2 angles.
__device__ __forceinline__ void dec_rope_table(float2* tab, int p, int rot, const RopeFreq& freq, int tid,
                                               int nthr) {
  for (int i = tid; i < (rot >> 1); i += nthr) {
    float c, s;
    rope_angle(p, freq.f[i], c, s);
    tab[i] = make_float2(c, s);
  }
}

// Stage the four query rows of KV group g (qrow: [4][256]) as bf16 q / 16: rotated first when
// `rope` by the angles of tab (bf16 rounding of the rotated value, as the stand-alone RoPE kernel
// does), then scaled by 1/16 (exact) and rounded.  Thread tid of nthr; tab is complete.
__device__ __forceinline__ void dec_stage_q(__nv_bfloat16* qs, const __nv_bfloat16* qrow, const float2* tab,
                                            bool rope, int rot, int tid, int nthr) {
  const int half = rot >> 1;
  for (int e = tid; e < 4 * kHeadDim; e += nthr) {
    const int d = e & (kHeadDim - 1);
    float x = __bfloat162float(qrow[e]);
    if (rope && d < rot) {
      const float2 cs = tab[d < half ? d : d - half];
      const float xp = __bfloat162float(qrow[e + (d < half ? half : -half)]);
      x = __bfloat162float(
          __float2bfloat16_rn(d < half ? rope_lo(x, xp, cs.x, cs.y) : rope_hi(xp, x, cs.x, cs.y)));
    }
    qs[e] = __float2bfloat16_rn(x * 0.0625f);
  }
}

// A warp's A fragments of the staged q rows (rows 4..15 of the m16 tile are zero).
__device__ __forceinline__ void dec_q_fragments(const __nv_bfloat16* qs, int lane, uint32_t (&qa)[16][2]) {
  const int gq = lane >> 2, cq = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 16; ++ks) {
    if (gq < 4) {
      qa[ks][0] = *reinterpret_cast<const uint32_t*>(qs + gq * kHeadDim + 16 * ks + 2 * cq);
      qa[ks][1] = *reinterpret_cast<const uint32_t*>(qs + gq * kHeadDim + 16 * ks + 2 * cq + 8);
    } else {
      qa[ks][0] = 0u;
      qa[ks][1] = 0u;
    }
  }
}

// One K/V tile (kt, vt: its K and V halves in shared memory) for this warp's 16 keys: S = Q K^T
// (mma.m16n8k16, K from the swizzled tile by ldmatrix), the online softmax in the exp2 domain, and
// O^T += V^T P^T (V^T by ldmatrix.trans, P from S's registers).  The tile's key k is cache row
// row0 + k; rows < row_end other than `hole` are visible.  Invisible rows may hold anything, NaN
// included, and a zero probability does not cancel a NaN, so when the tile has any, this warp
// first clears the V rows of its own keys there; the clearing is ordered before the stage's next
// TMA load by a proxy fence.
template <int kNK>
__device__ __forceinline__ void dec_consume_tile(uint32_t kt, uint32_t vt, const uint32_t (&qa)[16][2],
                                                 float (&o)[16][4], float& m_run, float& l_part, int row0,
                                                 int row_end, int hole, int warp, int lane) {
  const int cq = lane & 3;
  const int mi = lane >> 3, r8 = lane & 7;             // ldmatrix: matrix index, row
  const int key_l = warp * 16 + (mi >> 1) * 8 + r8;    // key row this lane addresses
  const int dim_off = (mi & 1) * 8;
  const float kLog2e = 1.4426950408889634f;
  if (row0 + kNK > row_end || (hole >= row0 && hole < row0 + kNK)) {
    for (int e = lane; e < 16 * 32; e += 32) {
      const int key = warp * 16 + (e >> 5);
      const int row = row0 + key;
      if (row >= row_end || row == hole)
        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(swz_addr<kNK>(vt, key, (e & 31) * 8)), "r"(0)
                     : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
  }
  // S = Q K^T for this warp's 16 keys, two accumulation chains per n-tile
  float sa[2][2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int c = 0; c < 2; ++c) sa[a][c][0] = sa[a][c][1] = sa[a][c][2] = sa[a][c][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 16; ++ks) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4(swz_addr<kNK>(kt, key_l, 16 * ks + dim_off), b0, b1, b2, b3);
    mma_bf16_16816(sa[0][ks & 1], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
    mma_bf16_16816(sa[1][ks & 1], qa[ks][0], 0u, qa[ks][1], 0u, b2, b3);
  }
  // scores of row gq at keys (8*nt + 2*cq + j)
  const int rbase = row0 + warp * 16;
  float tv[2][2];
  float mx = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int row = rbase + nt * 8 + 2 * cq + j;
      const float sv = (sa[nt][0][j] + sa[nt][1][j]) * kLog2e;
      tv[nt][j] = (row < row_end && row != hole) ? sv : -INFINITY;
      mx = fmaxf(mx, tv[nt][j]);
    }
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const float m_new = fmaxf(m_run, mx);
  const float m_use = m_new == -INFINITY ? 0.f : m_new;
  const float alpha = fast_exp2(m_run - m_use);
  float pv[2][2], psum = 0.f;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      pv[nt][j] = fast_exp2(tv[nt][j] - m_use);
      psum += pv[nt][j];
    }
  l_part = l_part * alpha + psum;
  m_run = m_new;
  const float a_lo = __shfl_sync(0xffffffffu, alpha, (8 * cq) & 31);
  const float a_hi = __shfl_sync(0xffffffffu, alpha, (8 * cq + 4) & 31);
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    o[t][0] *= a_lo;
    o[t][1] *= a_hi;
    o[t][2] *= a_lo;
    o[t][3] *= a_hi;
  }
  const uint32_t pb0 = pack_bf16(pv[0][0], pv[0][1]);
  const uint32_t pb1 = pack_bf16(pv[1][0], pv[1][1]);
  // O^T += V^T P^T
#pragma unroll
  for (int mt = 0; mt < 16; ++mt) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4_t(swz_addr<kNK>(vt, key_l, 16 * mt + dim_off), a0, a1, a2, a3);
    mma_bf16_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
  }
}

// Merge of the kW consumer warps' (m, l, o) through shared memory (mrg_o: kW x 4 heads x 256 floats;
// sm_m, sm_l: kW x 4).  Afterwards thread (warp w, lane) holds, for each query head hh = w, w + kW,
// .. < 4 of the group, the merged max ms[i], sum ls[i] and numerator acc[i][k] at dims lane + 32 k.
// `bar`: the consumers' named barrier; the first one also orders the staged q's last reads.
template <int kW>
__device__ __forceinline__ void dec_merge_warps(float* mrg_o, float* sm_m, float* sm_l, const float (&o)[16][4],
                                                float m_run, float l_part, int warp, int lane,
                                                float (&ms)[4 / kW], float (&ls)[4 / kW],
                                                float (&acc)[4 / kW][8]) {
  const int gq = lane >> 2, cq = lane & 3;
  float l_row = l_part;
  l_row += __shfl_xor_sync(0xffffffffu, l_row, 1);
  l_row += __shfl_xor_sync(0xffffffffu, l_row, 2);
  if (cq == 0 && gq < 4) {
    sm_m[warp * 4 + gq] = m_run;
    sm_l[warp * 4 + gq] = l_row;
  }
  if (cq < 2) {
    float* w = mrg_o + warp * 4 * kHeadDim;
#pragma unroll
    for (int mt = 0; mt < 16; ++mt) {
      const int d0 = 16 * mt + gq;
      w[(2 * cq) * kHeadDim + d0] = o[mt][0];
      w[(2 * cq + 1) * kHeadDim + d0] = o[mt][1];
      w[(2 * cq) * kHeadDim + d0 + 8] = o[mt][2];
      w[(2 * cq + 1) * kHeadDim + d0 + 8] = o[mt][3];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kW) : "memory");
#pragma unroll
  for (int i = 0; i < 4 / kW; ++i) {
    const int hh = warp + kW * i;
    float mw[kW], ew[kW];
    ms[i] = -INFINITY;
    ls[i] = 0.f;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      mw[w] = sm_m[w * 4 + hh];
      ms[i] = fmaxf(ms[i], mw[w]);
    }
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      ew[w] = (ms[i] == -INFINITY) ? 0.f : fast_exp2(mw[w] - ms[i]);
      ls[i] += ew[w] * sm_l[w * 4 + hh];
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < kW; ++w) a += ew[w] * mrg_o[(w * 4 + hh) * kHeadDim + lane + 32 * k];
      acc[i][k] = a;
    }
  }
}

template <bool kPaged>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_partial_kernel(const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap, const DecodeParams P) {
  extern __shared__ uint8_t dsmem[];
  const uint32_t raw = smem_u32(dsmem);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = dsmem + (base - raw);
  // layout: [stages x (K tile | V tile)] | merge area (also q staging) | barriers, abort, m, l
  float* mrg_o = reinterpret_cast<float*>(gbase + kDecStages * kDecStageBytes);
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(mrg_o);        // [4][256], before the loop
  uint8_t* misc = gbase + kDecStages * kDecStageBytes + kDecMergeBytes;
  const uint32_t bar_full = smem_u32(misc);
  const uint32_t bar_empty = bar_full + 8 * kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 16 * kDecStages);
  float* sm_m = reinterpret_cast<float*>(misc + 16 * kDecStages + 16);
  float* sm_l = sm_m + 16;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int p = P.pos[b];
  const bool bad = p < 0 || p >= kMaxPos || (!P.sliding && !P.shard && p >= P.cap);
  const int n_keys = bad ? 0 : (P.sliding ? min(p + 1, kWindow) : min(max(p + 1 - P.key_off, 0), P.cap));
  const int key_begin = split * P.tiles_per_split * kDecNK;
  const int key_end = min(n_keys, key_begin + P.tiles_per_split * kDecNK);
  const int n_tiles = key_end > key_begin ? (key_end - key_begin + kDecNK - 1) / kDecNK : 0;
  if (bad && threadIdx.x == 0 && split == 0 && g == 0) raise_error(kErrPosition, 0x300u | (unsigned)b);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kDecConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kDecStages;
        if (i >= kDecStages &&
            !mbar_wait(bar_empty + 8 * s, ((i / kDecStages) - 1) & 1, abort_flag, P.timeout_ns, 0x10u))
          break;
        const KvTile t = kv_tile<kPaged>(P, b, g, key_begin + i * kDecNK);
        if (!t.ok) {                       // a page index outside the pool: flag it, stop the block
          raise_error(kErrPosition, 0x600u | (unsigned)b);
          *abort_flag = 1;
          break;
        }
        const uint32_t full = bar_full + 8 * s;
        mbar_arrive_expect_tx(full, kDecStageBytes);
        const uint32_t kt = base + s * kDecStageBytes;
#pragma unroll
        for (int d = 0; d < 4; ++d) {
          kv_tile_load<kPaged>(kt + d * kDecBoxBytes, &kmap, full, d * 64, t);
          kv_tile_load<kPaged>(kt + kDecTileBytes + d * kDecBoxBytes, &vmap, full, d * 64, t);
        }
        issued = i + 1;
      }
      // Never leave with copies in flight: wait for the last issued tiles to land.
      for (int i = max(0, issued - kDecStages); i < issued; ++i)
        if (!mbar_drain(bar_full + 8 * (i % kDecStages), (i / kDecStages) & 1, 200000000ull)) break;
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = threadIdx.x;                 // 0..127
  float2* rtab = reinterpret_cast<float2*>(mrg_o + 4 * kHeadDim);       // after qs, before the loop only
  if (P.rope && !bad) {
    dec_rope_table(rtab, p, P.rot, P.freq, tid, 128);
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
  dec_stage_q(qs, P.q + (long long)b * P.q_sB + g * 4 * kHeadDim, rtab, P.rope && !bad, P.rot, tid, 128);
  asm volatile("bar.sync 1, 128;" ::: "memory");
  uint32_t qa[16][2];
  dec_q_fragments(qs, lane, qa);

  float o[16][4];
#pragma unroll
  for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m_run = -INFINITY, l_part = 0.f;

  for (int i = 0; i < n_tiles; ++i) {
    const int s = i % kDecStages;
    // warp-uniform outcome: ldmatrix / mma.sync below need every lane
    if (!__all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, (i / kDecStages) & 1, abort_flag, P.timeout_ns, 0x12u)))
      break;
    const uint32_t kt = base + s * kDecStageBytes;
    dec_consume_tile<kDecNK>(kt, kt + kDecTileBytes, qa, o, m_run, l_part, key_begin + i * kDecNK, key_end, -1, warp,
                             lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);
  }

  // ----------------------------------------------------- merge the 4 warps
  asm volatile("bar.sync 1, 128;" ::: "memory");    // q staging area is free again
  float ms[1], ls[1], acc[1][8];
  dec_merge_warps<kDecConsumerWarps>(mrg_o, sm_m, sm_l, o, m_run, l_part, warp, lane, ms, ls, acc);
  const int hh = warp;                            // query head within the group
  const long long row = ((long long)b * kNq + g * 4 + hh) * P.n_splits + split;
  if (P.n_splits == 1 && !P.shard) {
    // a single split is the whole answer: normalise, gate and store it here
    const float scale = decode_out_scale(ls[0], P.gate[(long long)b * kNq + g * 4 + hh]);
    __nv_bfloat16* dst = P.out + ((long long)b * kNq + g * 4 + hh) * kHeadDim;
#pragma unroll
    for (int k = 0; k < 8; ++k) dst[lane + 32 * k] = __float2bfloat16_rn(acc[0][k] * scale);
    return;
  }
  float* dst = P.o_part + row * kHeadDim;
#pragma unroll
  for (int k = 0; k < 8; ++k) dst[lane + 32 * k] = acc[0][k];
  if (lane == 0) {
    P.ml_part[row * 2 + 0] = ms[0];
    P.ml_part[row * 2 + 1] = ls[0];
  }
}

// out[b][h][:] = gate-scaled log-sum-exp merge of the splits' partials.
__global__ void __launch_bounds__(64) decode_combine_kernel(__nv_bfloat16* __restrict__ out,
                                                            const __nv_bfloat16* __restrict__ gate,
                                                            const float* __restrict__ o_part,
                                                            const float* __restrict__ ml_part,
                                                            int n_splits) {
  const int h = blockIdx.x, b = blockIdx.y;
  const long long row0 = ((long long)b * kNq + h) * n_splits;
  float ms = -INFINITY;
#pragma unroll 4
  for (int s = 0; s < n_splits; ++s) ms = fmaxf(ms, ml_part[(row0 + s) * 2]);
  float ls = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int s = 0; s < n_splits; ++s) {
    const float m = ml_part[(row0 + s) * 2];
    const float e = (m == -INFINITY) ? 0.f : fast_exp2(m - ms);
    ls += e * ml_part[(row0 + s) * 2 + 1];
    const float4 v = reinterpret_cast<const float4*>(o_part + (row0 + s) * kHeadDim)[threadIdx.x];
    acc.x += e * v.x;
    acc.y += e * v.y;
    acc.z += e * v.z;
    acc.w += e * v.w;
  }
  const float scale = decode_out_scale(ls, gate[(long long)b * kNq + h]);
  uint2 packed;
  packed.x = pack_bf16(acc.x * scale, acc.y * scale);
  packed.y = pack_bf16(acc.z * scale, acc.w * scale);
  reinterpret_cast<uint2*>(out + ((long long)b * kNq + h) * kHeadDim)[threadIdx.x] = packed;
}

// ------------------------------------------------- context parallelism ----
// A rank's record of one layer's decode: for every (sequence b, q head h) its
// attention output over the keys it holds, normalised, and the log-sum-exp of
// those keys' logits in base 2 (logits scaled by log2(e)/16, the kernels'
// exponent domain; -inf when the rank holds none).  Layout: o [B][16][256]
// then lse [B][16], fp32, cp_record_floats(B) floats.
__host__ __device__ constexpr long long cp_record_floats(int B) { return (long long)B * kNq * (kHeadDim + 1); }

__global__ void __launch_bounds__(64) decode_cp_reduce_kernel(float* __restrict__ rec, const float* __restrict__ o_part,
                                                              const float* __restrict__ ml_part, int n_splits, int B) {
  const int h = blockIdx.x, b = blockIdx.y;
  const long long row0 = ((long long)b * kNq + h) * n_splits;
  float ms = -INFINITY;
#pragma unroll 4
  for (int s = 0; s < n_splits; ++s) ms = fmaxf(ms, ml_part[(row0 + s) * 2]);
  float ls = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int s = 0; s < n_splits; ++s) {
    const float m = ml_part[(row0 + s) * 2];
    const float e = (m == -INFINITY) ? 0.f : fast_exp2(m - ms);
    ls += e * ml_part[(row0 + s) * 2 + 1];
    const float4 v = reinterpret_cast<const float4*>(o_part + (row0 + s) * kHeadDim)[threadIdx.x];
    acc.x += e * v.x;
    acc.y += e * v.y;
    acc.z += e * v.z;
    acc.w += e * v.w;
  }
  const float inv = ls > 0.f ? 1.f / ls : 0.f;
  const long long bh = (long long)b * kNq + h;
  reinterpret_cast<float4*>(rec + bh * kHeadDim)[threadIdx.x] =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (threadIdx.x == 0) rec[(long long)B * kNq * kHeadDim + bh] = ls > 0.f ? ms + log2f(ls) : -INFINITY;
}

// out = (sum over ranks of 2^(lse_r - M) o_r) / (sum of 2^(lse_r - M)) * sigmoid(gate), M the
// largest lse; recs holds G records back to back (rank order, as an all-gather lays them out).
__global__ void __launch_bounds__(64) decode_cp_merge_kernel(__nv_bfloat16* __restrict__ out,
                                                             const __nv_bfloat16* __restrict__ gate,
                                                             const float* __restrict__ recs, int G, int B) {
  const int h = blockIdx.x, b = blockIdx.y;
  const long long bh = (long long)b * kNq + h;
  const long long stride = cp_record_floats(B);
  const long long lse_at = (long long)B * kNq * kHeadDim + bh;
  float M = -INFINITY;
  for (int r = 0; r < G; ++r) M = fmaxf(M, recs[r * stride + lse_at]);
  float W = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = 0; r < G; ++r) {
    const float l = recs[r * stride + lse_at];
    const float w = (l == -INFINITY) ? 0.f : fast_exp2(l - M);
    W += w;
    const float4 v = reinterpret_cast<const float4*>(recs + r * stride + bh * kHeadDim)[threadIdx.x];
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  const float scale = decode_out_scale(W, gate[bh]);
  uint2 packed;
  packed.x = pack_bf16(acc.x * scale, acc.y * scale);
  packed.y = pack_bf16(acc.z * scale, acc.w * scale);
  reinterpret_cast<uint2*>(out + bh * kHeadDim)[threadIdx.x] = packed;
}

}  // namespace spark
