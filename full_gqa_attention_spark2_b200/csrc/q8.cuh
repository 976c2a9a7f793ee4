// 8-bit block-quantised KV cache: append (quantise) and split-KV decode that
// reads the codes straight from shared memory into tensor-core fragments.
//
// The format is the GGML "q8_0" block that the "Sharp-Spark-X2.5-4B-GGUF"
// page §四 offers as the KV-cache type (36 -> 19 KB per token): 32
// consecutive values share one fp16 scale and each value is an 8-bit code.
// Per cache row (one key or value vector, 256 dims):
//   codes   u8[256]  offset binary: byte = c + 128, c in [-127, 127]
//   scales f16[8]    one per 32-dim block; the value is c * scale
// Quantising a block, all in float32: amax = max |x|, scale = f16(amax / 127),
// c = x * (127 / amax) rounded half away from zero; a block of zeros (or of
// values so small that 127 / amax overflows) gives c = 0 and scale 0.  Caches: codes [B][4][cap][256], scales [B][4][cap][8],
// rows placed as in the bf16 cache (a ring of 512 rows for sliding layers,
// the position for full layers).  K rows hold rotated keys.
//
// Decode reads 544 bytes per key (K and V codes and scales) instead of 1024.
// Dequantisation is folded into the fragments: the byte u of a code becomes
// the fp16 value 1536 + u with one byte permute (fp16 bits 0x66uu), and one
// fp16 subtraction of 1664 gives c exactly.
//   S = Q K^T   B fragments come from 8 bytes of one key per block; the 32
//               dims of a block are visited in an order that q's A fragments
//               share, so each pair of k16 steps covers exactly one block and
//               its fp32 partial product is multiplied by that block's scale.
//   O^T += V^T P^T   A fragments pair two keys of one dim: four keys' bytes
//               of the thread's own 32-dim block are interleaved with byte
//               permutes, turned into fp16 and multiplied by the two keys'
//               scales (fp16 products).
// q and P enter the products in fp16 (q keeps its bf16 value exactly; a row
// whose |q|/16 reaches 2^15 is scaled down by a power of two first, and the
// scores are scaled back in fp32).
#pragma once
#include <cuda_fp16.h>
#include "decode.cuh"

namespace spark {

constexpr int kQ8Block = 32;
constexpr int kQ8NK = 64;                                   // keys per tile
constexpr int kQ8Stages = 4;
// Two groups of four consumer warps take alternate tiles (a warp holds ~230
// registers, so one block per SM; two warps per scheduler hide latency).
constexpr int kQ8ConsumerWarps = 8;
constexpr int kQ8Threads = (kQ8ConsumerWarps + 1) * 32;     // + 1 producer warp
constexpr int kQ8MergeBytes = kQ8ConsumerWarps * 4 * kHeadDim * 4;   // 32 KB
constexpr int kQ8CodeTile = kQ8NK * kHeadDim;               // 16 KB: codes of 64 keys
constexpr int kQ8CodeBox = kQ8NK * 128;                     // 8 KB: one 128-dim box
constexpr int kQ8ScaleTile = kQ8NK * 8 * 2;                 // 1 KB: scales of 64 keys
constexpr int kQ8StageBytes = 2 * kQ8CodeTile + 2 * kQ8ScaleTile;
constexpr int kQ8QBytes = 4 * kHeadDim * 2;                 // staged q, fp16
constexpr int kQ8MiscBytes = 1536;   // barriers, flags, m/l; from byte 512 the RoPE angle table
constexpr int kQ8SmemBytes = 1024 /*align slack*/ + kQ8Stages * kQ8StageBytes + kQ8QBytes + kQ8MiscBytes;
static_assert(kQ8MergeBytes <= kQ8Stages * kQ8StageBytes, "the merge area reuses the stages");
static_assert(kQ8StageBytes % 1024 == 0, "128-byte swizzled boxes need 1024-byte alignment");

// ----------------------------------------------------------------- append ----
// k/v [B][T][4][256] bf16 -> q8 caches.  One block per written token; K is
// rotated first when `rope` is set (bf16 rounding of the rotated value, as in
// the bf16 append).  Staged values are padded by one float per 32 so that the
// two threads of a block and their neighbours read distinct banks.
__device__ __forceinline__ int q8_pad(int i) { return i + (i >> 5); }

__global__ void __launch_bounds__(128) kv_append_q8_kernel(
    uint8_t* __restrict__ k_codes, __half* __restrict__ k_scales, uint8_t* __restrict__ v_codes,
    __half* __restrict__ v_scales, int cap, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, int B, int T, long long sB, long long sT, int t_first,
    const int* __restrict__ pos0, int sliding,
    int rope, const RopeFreq rf, int rot, CachePages pages, const int* __restrict__ cu, int key_off, int shard) {
  __shared__ float xs[2][kNkv * kHeadDim + kNkv * kHeadDim / 32];
  const int b = blockIdx.y;
  const int tid = threadIdx.x;
  const TokenSpan sp = token_span(b, T, t_first, sliding, cu);
  const int t = sp.t_first + blockIdx.x;
  if (t >= sp.T) return;
  const int p0 = pos0[b];
  const bool bad = p0 < 0 || p0 > kMaxPos - sp.T || (!sliding && !shard && p0 + sp.T > cap) ||
                   (cu != nullptr && sp.T > T);    // ragged: longer than max_seqlen, the launch's T
  if (bad) {
    if (blockIdx.x == 0 && tid == 0) raise_error(kErrPosition, 0x400u | (unsigned)b);
    return;
  }
  const int pos = p0 + t;
  if (shard && (pos - key_off < 0 || pos - key_off >= cap)) return;   // another rank's position
  const long long src = token_offset(cu, b, t, sp.tok0, sB, sT);
  // thread = one 16-byte chunk (8 dims) of K and of V: head tid / 32, dims 8 (tid % 32) ..
  {
    const uint4 kr = reinterpret_cast<const uint4*>(k + src)[tid];
    const uint4 vr = reinterpret_cast<const uint4*>(v + src)[tid];
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(&kr);
    const uint32_t* vw = reinterpret_cast<const uint32_t*>(&vr);
    const int i0 = q8_pad(8 * tid);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      xs[0][i0 + 2 * e] = bf16_lo(kw[e]);
      xs[0][i0 + 2 * e + 1] = bf16_hi(kw[e]);
      xs[1][i0 + 2 * e] = bf16_lo(vw[e]);
      xs[1][i0 + 2 * e + 1] = bf16_hi(vw[e]);
    }
  }
  __syncthreads();
  if (rope) {
    const int half = rot >> 1;
    const int d0 = 8 * (tid & 31);
    float r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int d = d0 + e;
      const float x = xs[0][q8_pad(8 * tid + e)];
      r[e] = x;
      if (d < rot) {
        const bool lo = d < half;
        const int i = lo ? d : d - half;
        float c, s;
        rope_angle(pos, rf.f[i], c, s);
        const float xp = xs[0][q8_pad(8 * tid + e + (lo ? half : -half))];
        r[e] = __bfloat162float(__float2bfloat16_rn(lo ? rope_lo(x, xp, c, s) : rope_hi(xp, x, c, s)));
      }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) xs[0][q8_pad(8 * tid + e)] = r[e];
    __syncthreads();
  }
  // two threads per 32-value block: 4 heads x 8 blocks x (K, V) = 64 blocks
  const int blk = tid >> 1, hf = tid & 1;
  const int which = blk >> 5;            // 0: K, 1: V
  const int hb = blk & 31;               // head * 8 + block
  const float* x = &xs[which][hb * 33 + hf * 16];
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(x[e]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  // a block of denormal values (127 / amax overflows) quantises like a zero block
  float inv = __fdiv_rn(127.f, amax);
  if (!(amax > 0.f) || isinf(inv)) inv = 0.f;
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float y = __fmul_rn(x[e], inv);
    const int c = (int)roundf(y);          // round half away from zero, exact
    const uint32_t u = (uint32_t)(c + 128);
    w[e >> 2] |= u << (8 * (e & 3));
  }
  const int h = hb >> 3, bl = hb & 7;
  const int row = sliding ? (pos & (kWindow - 1)) : pos - key_off;
  const long long crow = cache_row(pages, b, h, cap, row);
  if (crow < 0) {                        // a page index outside the pool
    if (tid == 0) raise_error(kErrPosition, 0x800u | (unsigned)b);
    return;
  }
  uint8_t* codes = which ? v_codes : k_codes;
  *reinterpret_cast<uint4*>(codes + crow * kHeadDim + bl * kQ8Block + hf * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  if (hf == 0) (which ? v_scales : k_scales)[crow * 8 + bl] = __float2half_rn(__fdiv_rn(amax, 127.f));
}

// ----------------------------------------------------------------- decode ----
// Byte address of code (key, dim) in a code tile of two [64 keys x 128 B]
// boxes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t q8_addr(uint32_t tile, int key, int dim) {
  return tile + (uint32_t)(dim >> 7) * kQ8CodeBox + (uint32_t)key * 128u +
         ((uint32_t)(((dim & 127) >> 4) ^ (key & 7)) << 4) + (uint32_t)(dim & 15);
}

__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 r;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
  return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 r;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
  return r;
}

__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  unsigned short r;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(r) : "r"(a));
  return r;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ float half_of(const uint4& v, int b) {
  const uint32_t w = word_of(v, b >> 1);
  return __half2float(__ushort_as_half((unsigned short)((b & 1) ? (w >> 16) : (w & 0xFFFFu))));
}

constexpr uint32_t kQ8Magic = 0x66666666u;   // high byte of fp16 1536 + u
constexpr uint32_t kQ8Bias = 0x66806680u;    // fp16 1664 in both halves
constexpr uint32_t kSelLo = 0x5140u;         // bytes {a0, b0, a1, b1}
constexpr uint32_t kSelHi = 0x7362u;         // bytes {a2, b2, a3, b3}

__device__ __forceinline__ uint32_t q8_pair(uint32_t bytes, uint32_t sel) {
  return hsub2_u32(prmt(bytes, kQ8Magic, sel), kQ8Bias);
}

template <bool kPaged>
__global__ void __launch_bounds__(kQ8Threads, 1)
    decode_q8_partial_kernel(const __grid_constant__ CUtensorMap kcmap, const __grid_constant__ CUtensorMap ksmap,
                             const __grid_constant__ CUtensorMap vcmap, const __grid_constant__ CUtensorMap vsmap,
                             const DecodeParams P) {
  extern __shared__ uint8_t dsmem[];
  const uint32_t raw = smem_u32(dsmem);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = dsmem + (base - raw);
  // layout: [stages x (K codes | V codes | K scales | V scales)] | q (fp16) | barriers, abort, m, l
  float* mrg_o = reinterpret_cast<float*>(gbase);           // after the loop only: reuses the stages
  __half* qs = reinterpret_cast<__half*>(gbase + kQ8Stages * kQ8StageBytes);
  uint8_t* misc = gbase + kQ8Stages * kQ8StageBytes + kQ8QBytes;
  const uint32_t bar_full = smem_u32(misc);
  const uint32_t bar_empty = bar_full + 8 * kQ8Stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 16 * kQ8Stages);
  unsigned* row_amax = reinterpret_cast<unsigned*>(misc + 16 * kQ8Stages + 16);
  float* sm_m = reinterpret_cast<float*>(misc + 16 * kQ8Stages + 32);    // [8 warps][4 heads]
  float* sm_l = sm_m + 4 * kQ8ConsumerWarps;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int p = P.pos[b];
  const bool bad = p < 0 || p >= kMaxPos || (!P.sliding && !P.shard && p >= P.cap);
  const int n_keys = bad ? 0 : (P.sliding ? min(p + 1, kWindow) : min(max(p + 1 - P.key_off, 0), P.cap));
  const int key_begin = split * P.tiles_per_split * kQ8NK;
  const int key_end = min(n_keys, key_begin + P.tiles_per_split * kQ8NK);
  const int n_tiles = key_end > key_begin ? (key_end - key_begin + kQ8NK - 1) / kQ8NK : 0;
  if (bad && threadIdx.x == 0 && split == 0 && g == 0) raise_error(kErrPosition, 0x500u | (unsigned)b);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQ8Stages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 4);        // the four warps of the group that owns the tile
    }
    *abort_flag = 0;
    for (int r = 0; r < 4; ++r) row_amax[r] = 0u;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kQ8ConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&kcmap);
      tma_prefetch_desc(&ksmap);
      tma_prefetch_desc(&vcmap);
      tma_prefetch_desc(&vsmap);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kQ8Stages;
        if (i >= kQ8Stages &&
            !mbar_wait(bar_empty + 8 * s, ((i / kQ8Stages) - 1) & 1, abort_flag, P.timeout_ns, 0x20u))
          break;
        const KvTile t = kv_tile<kPaged>(P, b, g, key_begin + i * kQ8NK);
        if (!t.ok) {                       // a page index outside the pool: flag it, stop the block
          raise_error(kErrPosition, 0x700u | (unsigned)b);
          *abort_flag = 1;
          break;
        }
        const uint32_t full = bar_full + 8 * s;
        mbar_arrive_expect_tx(full, kQ8StageBytes);
        const uint32_t st = base + s * kQ8StageBytes;
        kv_tile_load<kPaged>(st, &kcmap, full, 0, t);
        kv_tile_load<kPaged>(st + kQ8CodeBox, &kcmap, full, 128, t);
        kv_tile_load<kPaged>(st + kQ8CodeTile, &vcmap, full, 0, t);
        kv_tile_load<kPaged>(st + kQ8CodeTile + kQ8CodeBox, &vcmap, full, 128, t);
        kv_tile_load<kPaged>(st + 2 * kQ8CodeTile, &ksmap, full, 0, t);
        kv_tile_load<kPaged>(st + 2 * kQ8CodeTile + kQ8ScaleTile, &vsmap, full, 0, t);
        issued = i + 1;
      }
      for (int i = max(0, issued - kQ8Stages); i < issued; ++i)
        if (!mbar_drain(bar_full + 8 * (i % kQ8Stages), (i / kQ8Stages) & 1, 200000000ull)) break;
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = threadIdx.x;                 // 0..255
  const int grp = warp >> 2, wl = warp & 3;    // tile group (alternate tiles) / warp in group
  const int gq = lane >> 2, cq = lane & 3;     // mma fragment row group / column pair
  {
    // the group's four query rows: rotate (optional), bf16-round, scale by
    // 1/16; then per row a power of two that keeps |q| below 2^15 in fp16
    const __nv_bfloat16* qrow = P.q + (long long)b * P.q_sB + g * 4 * kHeadDim;
    const int half = P.rot >> 1;
    float2* rtab = reinterpret_cast<float2*>(misc + 512);    // one angle per RoPE frequency
    if (P.rope && !bad) {
      dec_rope_table(rtab, p, P.rot, P.freq, tid, 256);
      asm volatile("bar.sync 1, 256;" ::: "memory");
    }
    float qv[4];
#pragma unroll
    for (int k8 = 0; k8 < 4; ++k8) {
      const int e = tid + 256 * k8;
      const int d = e & (kHeadDim - 1);
      float x = __bfloat162float(qrow[e]);
      if (P.rope && d < P.rot && !bad) {
        const float2 cs = rtab[d < half ? d : d - half];
        const float xp = __bfloat162float(qrow[e + (d < half ? half : -half)]);
        x = __bfloat162float(
            __float2bfloat16_rn(d < half ? rope_lo(x, xp, cs.x, cs.y) : rope_hi(xp, x, cs.x, cs.y)));
      }
      qv[k8] = x * 0.0625f;
      atomicMax(&row_amax[e >> 8], __float_as_uint(fabsf(qv[k8])));
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
#pragma unroll
    for (int k8 = 0; k8 < 4; ++k8) {
      const int e = tid + 256 * k8;
      const unsigned am = row_amax[e >> 8];
      const int ex = __uint_as_float(am) >= 32768.f ? (int)(am >> 23) - 127 - 14 : 0;
      qs[e] = __float2half_rn(qv[k8] * __uint_as_float((unsigned)(127 - ex) << 23));
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
  }
  // A fragments of q come from shared memory, block by block: k-step (block bl,
  // sub) covers dims 32 bl + 8 cq + 4 sub + {0,1 | 2,3} of row gq.  Rows 4..7
  // of the fragment repeat rows 0..3 (their results are never used).
  const uint32_t q_frag = smem_u32(qs) + (uint32_t)(gq & 3) * (kHeadDim * 2) + 16u * cq;
  const float kLog2e = 1.4426950408889634f;
  float s_row;
  {
    const unsigned am = row_amax[gq & 3];
    const int ex = __uint_as_float(am) >= 32768.f ? (int)(am >> 23) - 127 - 14 : 0;
    s_row = kLog2e * __uint_as_float((unsigned)(127 + ex) << 23);
  }

  float o[16][4];
#pragma unroll
  for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m_run = -INFINITY, l_part = 0.f;
  bool ok = true;

  for (int i = grp; i < n_tiles; i += 2) {
    const int s = i % kQ8Stages;
    if (!__all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, (i / kQ8Stages) & 1, abort_flag, P.timeout_ns, 0x22u))) {
      ok = false;
      break;
    }
    const uint32_t kc = base + s * kQ8StageBytes;
    const uint32_t vc = kc + kQ8CodeTile;
    const uint32_t ksc = kc + 2 * kQ8CodeTile;
    const uint32_t vsc = ksc + kQ8ScaleTile;
    const int tile_key0 = key_begin + i * kQ8NK;

    // ---- S = Q K^T, block by block, each block's partial times its scale
    float sc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    uint4 sk[2][2];                                       // K scales of this thread's score keys
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int key_s = wl * 16 + nt * 8 + 2 * cq;
      sk[nt][0] = lds128(ksc + key_s * 16);
      sk[nt][1] = lds128(ksc + (key_s + 1) * 16);
    }
#pragma unroll
    for (int bl = 0; bl < 8; ++bl) {
      const uint4 qf = lds128(q_frag + 64u * bl);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const uint2 w = lds64(q8_addr(kc, wl * 16 + nt * 8 + gq, 32 * bl + 8 * cq));   // B-fragment key
        float acc[4];
        mma_f16_16816_z(acc, qf.x, 0u, qf.y, 0u, q8_pair(w.x, kSelLo), q8_pair(w.x, kSelHi));
        mma_f16_16816(acc, qf.z, 0u, qf.w, 0u, q8_pair(w.y, kSelLo), q8_pair(w.y, kSelHi));
        sc[nt][0] = fmaf(half_of(sk[nt][0], bl), acc[0], sc[nt][0]);
        sc[nt][1] = fmaf(half_of(sk[nt][1], bl), acc[1], sc[nt][1]);
      }
    }

    // ---- online softmax (fp32, exp2 domain); keys past key_end are masked
    const int kbase = tile_key0 + wl * 16;
    float tv[2][2];
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int kidx = kbase + nt * 8 + 2 * cq + j;
        tv[nt][j] = kidx < key_end ? sc[nt][j] * s_row : -INFINITY;
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
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
      const float a_lo = __shfl_sync(0xffffffffu, alpha, (8 * cq) & 31);
      const float a_hi = __shfl_sync(0xffffffffu, alpha, (8 * cq + 4) & 31);
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        o[t][0] *= a_lo;
        o[t][1] *= a_hi;
        o[t][2] *= a_lo;
        o[t][3] *= a_hi;
      }
    }
    const uint32_t pb0 = pack_f16(pv[0][0], pv[0][1]);
    const uint32_t pb1 = pack_f16(pv[1][0], pv[1][1]);

    // ---- O^T += V^T P^T over the thread's 32-dim block gq and keys kA, kA+1, kA+8, kA+9
    const int kA = wl * 16 + 2 * cq;
    uint32_t sv[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int key = kA + (kk & 1) + 8 * (kk >> 1);
      // a key past the last one gets scale 0: its codes are finite, so its V is exactly 0
      sv[kk] = (tile_key0 + key < key_end) ? lds16(vsc + key * 16 + gq * 2) : 0u;
    }
    const uint32_t sAB = sv[0] | (sv[1] << 16);
    const uint32_t sCD = sv[2] | (sv[3] << 16);
#pragma unroll
    for (int hv = 0; hv < 2; ++hv) {                       // dims 32 gq + 16 hv .. + 15
      uint4 wv[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        wv[kk] = lds128(q8_addr(vc, kA + (kk & 1) + 8 * (kk >> 1), 32 * gq + 16 * hv));
#pragma unroll
      for (int mh = 0; mh < 8; ++mh) {
        const int mt = 8 * hv + mh;
        const int j = mh >> 1;                               // word: dims 32 gq + 16 hv + 4 j ..
        const uint32_t sel = (mh & 1) ? kSelHi : kSelLo;    // dims +0,+1 or +2,+3
        const uint32_t x = prmt(word_of(wv[0], j), word_of(wv[1], j), sel);
        const uint32_t z = prmt(word_of(wv[2], j), word_of(wv[3], j), sel);
        const uint32_t a0 = hmul2_u32(q8_pair(x, kSelLo), sAB);   // dim 32 gq + 2 mt,     keys kA, kA+1
        const uint32_t a1 = hmul2_u32(q8_pair(x, kSelHi), sAB);   // dim 32 gq + 2 mt + 1, keys kA, kA+1
        const uint32_t a2 = hmul2_u32(q8_pair(z, kSelLo), sCD);   // keys kA+8, kA+9
        const uint32_t a3 = hmul2_u32(q8_pair(z, kSelHi), sCD);
        mma_f16_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);
  }

  // ----------------------------------------------------- merge the 8 warps
  // Only when every tile arrived: then no copy is in flight and the stage
  // memory can hold the merge.  After a timeout the partials stay unwritten
  // (the error word reports it).
  uint32_t all_ok;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(all_ok)
      : "r"((uint32_t)ok)
      : "memory");
  if (!all_ok) return;
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
      const int d0 = 32 * gq + 2 * mt;
      w[(2 * cq) * kHeadDim + d0] = o[mt][0];
      w[(2 * cq + 1) * kHeadDim + d0] = o[mt][1];
      w[(2 * cq) * kHeadDim + d0 + 1] = o[mt][2];
      w[(2 * cq + 1) * kHeadDim + d0 + 1] = o[mt][3];
    }
  }
  asm volatile("bar.sync 1, 256;" ::: "memory");
  {
    const int hh = tid >> 6;                      // query head within the group
    float mw[kQ8ConsumerWarps], ms = -INFINITY;
#pragma unroll
    for (int w = 0; w < kQ8ConsumerWarps; ++w) {
      mw[w] = sm_m[w * 4 + hh];
      ms = fmaxf(ms, mw[w]);
    }
    float ew[kQ8ConsumerWarps], ls = 0.f;
#pragma unroll
    for (int w = 0; w < kQ8ConsumerWarps; ++w) {
      ew[w] = (ms == -INFINITY) ? 0.f : fast_exp2(mw[w] - ms);
      ls += ew[w] * sm_l[w * 4 + hh];
    }
    const long long row = ((long long)b * kNq + g * 4 + hh) * P.n_splits + split;
    if (P.n_splits == 1 && !P.shard) {
      // a single split is the whole answer: normalise, gate and store it here
      const float scale = decode_out_scale(ls, P.gate[(long long)b * kNq + g * 4 + hh]);
      __nv_bfloat16* dst = P.out + ((long long)b * kNq + g * 4 + hh) * kHeadDim;
      for (int d = (tid & 63); d < kHeadDim; d += 64) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kQ8ConsumerWarps; ++w) acc += ew[w] * mrg_o[(w * 4 + hh) * kHeadDim + d];
        dst[d] = __float2bfloat16_rn(acc * scale);
      }
      return;
    }
    float* dst = P.o_part + row * kHeadDim;
    for (int d = (tid & 63); d < kHeadDim; d += 64) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kQ8ConsumerWarps; ++w) acc += ew[w] * mrg_o[(w * 4 + hh) * kHeadDim + d];
      dst[d] = acc;
    }
    if ((tid & 63) == 0) {
      P.ml_part[row * 2 + 0] = ms;
      P.ml_part[row * 2 + 1] = ls;
    }
  }
}

// The history a prefill chunk reads from an 8-bit cache, as bf16 rows in the bf16 cache's layout
// ([B][4][cap][256]): rows [0, min(pos0[b], cap)) of sequence b (a full layer's positions; a
// sliding ring's rows, cap 512, which then hold every history position the chunk can see).  Rows
// past them, and every row of a sequence with a negative position, are left as they are (the
// prefill never reads them; it flags a bad position itself).  Each value is code * scale, exact in fp32
// (an 8-bit code times an 11-bit significand), then rounded once to bf16.  One warp per (row,
// tensor): lane i takes codes 8i .. 8i+7 of block i/4 (256 bytes read, 512 written per warp).
// Grid (ceil(cap / 4), 4 KV heads, B), 256 threads: warp w takes row 4 blockIdx.x + w/2, K (even
// w) or V (odd w).
__global__ void __launch_bounds__(256) q8_history_kernel(const uint8_t* __restrict__ k_codes,
                                                         const __half* __restrict__ k_scales,
                                                         const uint8_t* __restrict__ v_codes,
                                                         const __half* __restrict__ v_scales, int cap,
                                                         const int* __restrict__ pos0, __nv_bfloat16* __restrict__ k_out,
                                                         __nv_bfloat16* __restrict__ v_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + (warp >> 1);
  const int b = blockIdx.z;
  const int p = pos0[b];
  if (p < 0 || row >= min(p, cap)) return;
  const bool is_v = warp & 1;
  const long long r = ((long long)b * kNkv + blockIdx.y) * cap + row;
  const uint2 c8 = *reinterpret_cast<const uint2*>((is_v ? v_codes : k_codes) + r * kHeadDim + lane * 8);
  const float d = __half2float((is_v ? v_scales : k_scales)[r * (kHeadDim / 32) + (lane >> 2)]);
  auto val = [&](uint32_t w, int i) { return (float)((int)((w >> (8 * i)) & 0xFFu) - 128) * d; };
  uint4 o;
  o.x = pack_bf16(val(c8.x, 0), val(c8.x, 1));
  o.y = pack_bf16(val(c8.x, 2), val(c8.x, 3));
  o.z = pack_bf16(val(c8.y, 0), val(c8.y, 1));
  o.w = pack_bf16(val(c8.y, 2), val(c8.y, 3));
  *reinterpret_cast<uint4*>((is_v ? v_out : k_out) + r * kHeadDim + lane * 8) = o;
}

}  // namespace spark
