// RoPE and KV-cache append kernels (memory-bound, bf16 in / bf16 out).
//
// RoPE ("Spark-X2.6-4B config.json" page §1M 上下文如何做到 and "Spark-X2.6-4B-Base"
// page §全局注意力 5M 基频 RoPE): for i < rot/2 the pair (x_i, x_{i+rot/2}) turns
// by a = pos * theta^(-2i/rot); sliding layers rot = 256, theta = 1e4; full
// layers rot = 64, theta = 5e6 (dims 64..255 untouched).
//
// Angle accuracy: at pos ~ 2^20 the product pos * f_i in fp32 would carry an
// error of ~0.06 rad.  The product and its reduction into [-pi, pi] are done
// in fp64, then sincosf runs on the reduced fp32 angle (error ~1e-7 rad).
#pragma once
#include "ptx.cuh"

namespace spark {

constexpr int kHeadDim = 256;
constexpr int kNq = 16;
constexpr int kNkv = 4;
constexpr int kWindow = 512;
constexpr int kMaxPos = 1 << 20;

// Frequencies f_i = theta^(-2i/rot), i < rot/2, of one layer kind, computed
// once on the host in double precision and passed in the kernel parameters.
struct RopeFreq {
  double f[128];
};

// r^n for 0 <= n < 256 by binary powers (at most 14 fp64 products).  With
// r = f_1 = theta^(-2/rot), f_i = r^i: every lane of a warp reads the same
// f_1, where a lane-indexed table read of the parameters would be serialised.
__device__ __forceinline__ double pow_u8(double r, int n) {
  double y = 1.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (n & (1 << k)) y *= r;
    r *= r;
  }
  return y;
}

// A pair (lo, hi) = (x_i, x_{i+rot/2}) turned by the angle whose cosine and sine are c, s:
// lo' = lo c - hi s, hi' = hi c + lo s.  The rounding is pinned (the second product rounded,
// then one fused multiply-add), so every kernel that rotates the same value at the same
// position writes the same bits whatever the compiler would contract.
__device__ __forceinline__ float rope_lo(float lo, float hi, float c, float s) {
  return __fmaf_rn(lo, c, -__fmul_rn(hi, s));
}
__device__ __forceinline__ float rope_hi(float lo, float hi, float c, float s) {
  return __fmaf_rn(hi, c, __fmul_rn(lo, s));
}

// cos/sin of pos * f for an integer position, via an fp64 reduction mod 2*pi.
__device__ __forceinline__ void rope_angle(int pos, double f, float& c, float& s) {
  const double kTwoPi = 6.283185307179586476925286766559;
  const double kInvTwoPi = 0.15915494309189533576888376337251;
  double a = (double)pos * f;
  double k = rint(a * kInvTwoPi);
  double r = fma(-k, kTwoPi, a);
  sincosf((float)r, &s, &c);
}

// 16-head tensors (q): x [B][T][16][256] (dense, cu == nullptr) or packed [total][16][256] with
// sequence b at rows cu[b] .. cu[b+1]-1 (ragged), in place.  One thread per (token, two
// consecutive pairs), all sixteen heads' pairs loaded before any is stored, so sixteen loads are
// in flight together (3x faster on full layers than one head at a time; faster than the run kernel
// below, whose angle reuse matters less where sixteen heads share each angle).  A block walks
// kRopeIters groups of tokens, so that its frequency table serves many tokens.  Dense: a 1-D grid
// over the B*T tokens.  Ragged: grid.y = sequence, grid.x over its tokens (T = the longest).
constexpr int kRopeIters = 8;

// Token rows as for rope_kernel below.
__global__ void __launch_bounds__(128) rope16_kernel(__nv_bfloat16* __restrict__ x, int B, int T,
                                                     long long sB, long long sT, const int* __restrict__ pos0,
                                                     const RopeFreq rf, int rot, const int* __restrict__ cu) {
  __shared__ double freq[128];
  const int half = rot >> 1;
  for (int i = threadIdx.x; i < half; i += blockDim.x) freq[i] = rf.f[i];
  __syncthreads();

  const int per_tok = half >> 1;                  // threads per token
  const int tok_per_block = blockDim.x / per_tok;
  const int j = threadIdx.x % per_tok;
  if (threadIdx.x / per_tok >= tok_per_block) return;
  for (int it = 0; it < kRopeIters; ++it) {
    const long long slot = ((long long)blockIdx.x * kRopeIters + it) * tok_per_block + threadIdx.x / per_tok;
    long long n;                                  // packed row of the token
    int b, t, T_b;
    if (cu == nullptr) {
      n = slot;
      if (n >= (long long)B * T) return;
      b = (int)(n / T);
      t = (int)(n % T);
      T_b = T;
    } else {
      b = blockIdx.y;
      t = (int)slot;
      T_b = cu[b + 1] - cu[b];
      if (T_b < 0 || T_b > T) {                  // a sequence longer than max_seqlen: not rotated
        if (t == 0 && j == 0) raise_error(kErrPosition, 0x100u | (unsigned)b);
        return;
      }
      if (t >= T_b) return;
      n = (long long)cu[b] + t;
    }
    const int p0 = pos0[b];
    if (p0 < 0 || p0 > kMaxPos - T_b) {
      if (t == 0 && j == 0) raise_error(kErrPosition, 0x100u | (unsigned)b);
      continue;
    }
    const int pos = p0 + t;
    float c0, s0, c1, s1;
    rope_angle(pos, freq[2 * j], c0, s0);
    rope_angle(pos, freq[2 * j + 1], c1, s1);
    __nv_bfloat16* row = x + (cu == nullptr ? (long long)b * sB + (long long)t * sT : n * sT);
    {
      uint32_t lo[16], hi[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        lo[h] = *reinterpret_cast<const uint32_t*>(row + h * kHeadDim + 2 * j);
        hi[h] = *reinterpret_cast<const uint32_t*>(row + h * kHeadDim + half + 2 * j);
      }
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const float l0 = bf16_lo(lo[h]), l1 = bf16_hi(lo[h]), h0 = bf16_lo(hi[h]), h1 = bf16_hi(hi[h]);
        *reinterpret_cast<uint32_t*>(row + h * kHeadDim + 2 * j) =
            pack_bf16(rope_lo(l0, h0, c0, s0), rope_lo(l1, h1, c1, s1));
        *reinterpret_cast<uint32_t*>(row + h * kHeadDim + half + 2 * j) =
            pack_bf16(rope_hi(l0, h0, c0, s0), rope_hi(l1, h1, c1, s1));
      }
    }
  }
}

// One 32-bit word of a low chunk and its partner in the high chunk: two pairs rotated by the angles
// (c0, s0) and (c1, s1), each product rounded before the FMA that adds it (as in the append).
__device__ __forceinline__ void rope_word(uint32_t& l, uint32_t& u, float c0, float s0, float c1, float s1) {
  const float a0 = bf16_lo(l), a1 = bf16_hi(l), b0 = bf16_lo(u), b1 = bf16_hi(u);
  l = pack_bf16(rope_lo(a0, b0, c0, s0), rope_lo(a1, b1, c1, s1));
  u = pack_bf16(rope_hi(a0, b0, c0, s0), rope_hi(a1, b1, c1, s1));
}

// 4-head tensors (k): x [B][T][4][256] (dense, cu == nullptr) or packed [total][4][256] with
// sequence b at rows cu[b] .. cu[b+1]-1 (ragged), in place (H: a multiple of 4).  A thread takes one chunk of eight pairs (dims 8 c .. 8 c + 7 and
// their partners rot/2 later) in every head of kRopeRun consecutive tokens of one sequence: 16-byte
// accesses, four heads' loads in flight together.  Its first token's angles are exact (fp64
// product and reduction); each later token's advance by one position's rotation, so one angle
// serves H * kRopeRun rotations.  Dense: a 1-D grid over every sequence's runs of tokens.  Ragged:
// grid.y = sequence, grid.x over its runs (T = the longest).
// Token rows: dense batches put token t of sequence b at element b * sB + t * sT; packed rows
// (ragged) put row n at n * sT.  Within a token the H heads are contiguous rows of 256.
constexpr int kRopeRun = 4;

__global__ void __launch_bounds__(128) rope_kernel(__nv_bfloat16* __restrict__ x, int B, int T, int H, long long sB,
                                                   long long sT, const int* __restrict__ pos0, const RopeFreq rf,
                                                   int rot, const int* __restrict__ cu) {
  const int half = rot >> 1;
  const int n_ch = half >> 3;                      // chunks per head: 16 (sliding) or 4 (full)
  const int ch = threadIdx.x % n_ch;
  const long long run = (long long)blockIdx.x * (blockDim.x / n_ch) + threadIdx.x / n_ch;
  int b, t0, T_b;
  if (cu == nullptr) {
    const int runs_per_seq = (T + kRopeRun - 1) / kRopeRun;
    if (run >= (long long)B * runs_per_seq) return;
    b = (int)(run / runs_per_seq);
    t0 = (int)(run % runs_per_seq) * kRopeRun;
    T_b = T;
  } else {
    b = blockIdx.y;
    T_b = cu[b + 1] - cu[b];
    if (T_b < 0 || T_b > T) {                    // a sequence longer than max_seqlen: not rotated
      if (run == 0 && ch == 0) raise_error(kErrPosition, 0x100u | (unsigned)b);
      return;
    }
    if (run * kRopeRun >= T_b) return;
    t0 = (int)run * kRopeRun;
  }
  const int p0 = pos0[b];
  if (p0 < 0 || p0 > kMaxPos - T_b) {
    if (t0 == 0 && ch == 0) raise_error(kErrPosition, 0x100u | (unsigned)b);
    return;
  }
  float c[8], s[8], cs[8], ss[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const double f = rf.f[8 * ch + e];
    rope_angle(p0 + t0, f, c[e], s[e]);
    sincosf((float)f, &ss[e], &cs[e]);             // one position: 0 < f <= 1 needs no reduction
  }
  for (int i = 0; i < kRopeRun; ++i) {
    const int t = t0 + i;
    if (t >= T_b) break;
    __nv_bfloat16* row = x + (cu == nullptr ? (long long)b * sB + (long long)t * sT : ((long long)cu[b] + t) * sT);
    for (int h0 = 0; h0 < H; h0 += 4) {
      uint4 lo[4], hi[4];
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        lo[hh] = *reinterpret_cast<const uint4*>(row + (h0 + hh) * kHeadDim + 8 * ch);
        hi[hh] = *reinterpret_cast<const uint4*>(row + (h0 + hh) * kHeadDim + half + 8 * ch);
      }
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        rope_word(lo[hh].x, hi[hh].x, c[0], s[0], c[1], s[1]);
        rope_word(lo[hh].y, hi[hh].y, c[2], s[2], c[3], s[3]);
        rope_word(lo[hh].z, hi[hh].z, c[4], s[4], c[5], s[5]);
        rope_word(lo[hh].w, hi[hh].w, c[6], s[6], c[7], s[7]);
        *reinterpret_cast<uint4*>(row + (h0 + hh) * kHeadDim + 8 * ch) = lo[hh];
        *reinterpret_cast<uint4*>(row + (h0 + hh) * kHeadDim + half + 8 * ch) = hi[hh];
      }
    }
    // the next position: (c + i s)(cs + i ss)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float cn = c[e] * cs[e] - s[e] * ss[e];
      s[e] = s[e] * cs[e] + c[e] * ss[e];
      c[e] = cn;
    }
  }
}

// Where a cache row lives.  Dense caches: [B][4][cap][256].  Paged pools:
// [n_pages][4][page][256], logical row r of sequence b in page
// table[b * max_pages + r / page] at row r % page (table == nullptr: dense).
struct CachePages {
  const int* table;
  int max_pages, page_shift, n_pages;
};

// Index of the 256-element row holding (sequence b, KV head h, logical row),
// or -1 when the page index is outside the pool.
__device__ __forceinline__ long long cache_row(const CachePages& pg, int b, int h, int cap, int row) {
  if (pg.table == nullptr) return ((long long)b * kNkv + h) * cap + row;
  const int page = pg.table[(long long)b * pg.max_pages + (row >> pg.page_shift)];
  if (page < 0 || page >= pg.n_pages) return -1;
  return ((long long)page * kNkv + h) * (1 << pg.page_shift) + (row & ((1 << pg.page_shift) - 1));
}

// The tokens of sequence b an append writes.  Dense batches [B][T]: rows
// b*T + t, the launch's t_first.  Ragged (cu != nullptr): rows cu[b] + t of a
// sequence of cu[b+1] - cu[b] tokens; a sliding layer writes its last 512.
struct TokenSpan {
  long long tok0;
  int T, t_first;
};

__device__ __forceinline__ TokenSpan token_span(int b, int T, int t_first, int sliding, const int* cu) {
  if (cu == nullptr) return TokenSpan{(long long)b * T, T, t_first};
  const int T_b = cu[b + 1] - cu[b];
  return TokenSpan{(long long)cu[b], T_b, (sliding && T_b > kWindow) ? T_b - kWindow : 0};
}

// Element offset of token t of sequence b: dense batches b * sB + t * sT, packed rows (ragged)
// (tok0 + t) * sT, with tok0 the sequence's first packed row.
__device__ __forceinline__ long long token_offset(const int* cu, int b, int t, long long tok0, long long sB,
                                                  long long sT) {
  return cu == nullptr ? (long long)b * sB + (long long)t * sT : (tok0 + t) * sT;
}

// Append k/v [B][T][4][256] of T new tokens into caches [B][4][cap][256].
// One block per written token, thread = (head, 16-byte chunk of 8 dims).
// Sliding layers (ring of 512 rows) only write the last min(T, 512) tokens.
__global__ void __launch_bounds__(128) kv_append_kernel(
    __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache, int cap,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, int B, int T, long long sB,
    long long sT, int t_first, const int* __restrict__ pos0, int sliding, int rope, const RopeFreq rf, int rot,
    CachePages pages, const int* __restrict__ cu, int key_off, int shard) {
  const int b = blockIdx.y;
  const int h = threadIdx.x >> 5;
  const int ch = threadIdx.x & 31;
  const TokenSpan sp = token_span(b, T, t_first, sliding, cu);
  const int t = sp.t_first + blockIdx.x;
  if (t >= sp.T) return;
  const int p0 = pos0[b];
  // (ragged: a sequence longer than max_seqlen, the launch's T, is not written either)
  const bool bad = p0 < 0 || p0 > kMaxPos - sp.T || (!sliding && !shard && p0 + sp.T > cap) ||
                   (cu != nullptr && sp.T > T);
  if (bad) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(kErrPosition, 0x200u | (unsigned)b);
    return;
  }
  const int pos = p0 + t;
  // full layers: row = position - key_off (0 unless the cache is one rank's shard of positions)
  const int row = sliding ? (pos & (kWindow - 1)) : pos - key_off;
  if (shard && (row < 0 || row >= cap)) return;   // another rank's position
  const long long src = token_offset(cu, b, t, sp.tok0, sB, sT) + h * kHeadDim;
  const long long crow = cache_row(pages, b, h, cap, row);
  if (crow < 0) {                        // a page index outside the pool
    if (ch == 0) raise_error(kErrPosition, 0x900u | (unsigned)b);
    return;
  }
  const long long dst = crow * kHeadDim;

  const uint4* vs = reinterpret_cast<const uint4*>(v + src);
  reinterpret_cast<uint4*>(v_cache + dst)[ch] = vs[ch];

  const uint4* ks = reinterpret_cast<const uint4*>(k + src);
  uint4* kd = reinterpret_cast<uint4*>(k_cache + dst);
  const int half = rot >> 1;
  if (!rope || ch * 8 >= rot) {
    kd[ch] = ks[ch];
    return;
  }
  if (ch * 8 >= half) return;                    // the partner thread writes this chunk
  const int pc = ch + (half >> 3);               // chunk holding the partner dims
  uint4 lo = ks[ch], hi = ks[pc];
  uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* hh = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int i0 = ch * 8 + 2 * e;
    float c0, s0, c1, s1;
    rope_angle(pos, rf.f[i0], c0, s0);
    rope_angle(pos, rf.f[i0 + 1], c1, s1);
    float l0 = bf16_lo(l[e]), l1 = bf16_hi(l[e]), h0 = bf16_lo(hh[e]), h1 = bf16_hi(hh[e]);
    l[e] = pack_bf16(rope_lo(l0, h0, c0, s0), rope_lo(l1, h1, c1, s1));
    hh[e] = pack_bf16(rope_hi(l0, h0, c0, s0), rope_hi(l1, h1, c1, s1));
  }
  kd[ch] = lo;
  kd[pc] = hi;
}

}  // namespace spark
