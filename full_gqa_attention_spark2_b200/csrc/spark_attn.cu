// libspark_attn.so: host entry points of the C ABI declared in
// include/spark_attn.h.  One translation unit: the kernels live in the .cuh
// files included below, so the device error word is a single module symbol.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/spark_attn.h"
#include "decode.cuh"
#include "decode_fused.cuh"
#include "prefill.cuh"
#include "prefill2.cuh"
#include "prefill3.cuh"
#include "ptx.cuh"
#include "q8.cuh"
#include "rope_append.cuh"

namespace spark {
// One block waits, with the library's bounded wait, on a barrier phase that
// nothing ever completes: the wait must run out, set the device error word and
// let the kernel return.  Used to test the failure-detection path.
__global__ void selftest_wait_kernel(unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, timeout_ns, 0x7Fu);
}
}  // namespace spark

namespace {

thread_local char g_last_error[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SPARK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------- devices ---
constexpr int kMaxDevices = 64;
struct DeviceInfo {
  std::once_flag once;
  int ok = 0;          // 1: sm_100 and attributes set
  int sm_count = 148;
  char why[160] = "";
};
DeviceInfo g_dev[kMaxDevices];

int device_ready(int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SPARK_ERR_UNSUPPORTED, "device index %d", dev);
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&]() {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10 || minor != 0) {
      snprintf(d.why, sizeof(d.why), "device %d is sm_%d%d; this library is built for sm_100a", dev,
               major, minor);
      return;
    }
    d.sm_count = sms > 0 ? sms : 148;
    cudaError_t a = cudaFuncSetAttribute(spark::decode_partial_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         spark::kDecSmemBytes);
    if (a == cudaSuccess)
      a = cudaFuncSetAttribute(spark::decode_partial_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               spark::kDecSmemBytes);
    if (a == cudaSuccess)
      a = cudaFuncSetAttribute(spark::decode_fused_kernel<4, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               spark::DfShape<4, 1>::kSmemBytes);
    if (a == cudaSuccess)
      a = cudaFuncSetAttribute(spark::decode_fused_kernel<2, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               spark::DfShape<2, 2>::kSmemBytes);
    cudaError_t b = cudaFuncSetAttribute(spark::prefill2_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         spark::kP2SmemBytes);
    if (b == cudaSuccess)
      b = cudaFuncSetAttribute(spark::prefill2_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               spark::kP2SmemBytes);
    if (b == cudaSuccess)
      b = cudaFuncSetAttribute(spark::prefill3_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               spark::kP2SmemBytes);
    if (b == cudaSuccess)
      b = cudaFuncSetAttribute(spark::prefill3_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               spark::kP2SmemBytes);
    cudaError_t c = cudaFuncSetAttribute(spark::decode_q8_partial_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         spark::kQ8SmemBytes);
    if (c == cudaSuccess)
      c = cudaFuncSetAttribute(spark::decode_q8_partial_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               spark::kQ8SmemBytes);
    if (a != cudaSuccess || b != cudaSuccess || c != cudaSuccess) {
      snprintf(d.why, sizeof(d.why), "cudaFuncSetAttribute: %s",
               cudaGetErrorString(a != cudaSuccess ? a : b != cudaSuccess ? b : c));
      return;
    }
    d.ok = 1;
  });
  if (!d.ok) return fail(SPARK_ERR_UNSUPPORTED, "%s", d.why);
  *dev_out = dev;
  return SPARK_OK;
}

// Wait limit of the kernels' bounded waits.  SPARK_WAIT_TIMEOUT_NS overrides
// it (used by the tests that make a wait run out on purpose).
unsigned long long wait_timeout_ns() {
  static std::atomic<unsigned long long> cached{0};
  unsigned long long v = cached.load();
  if (v == 0) {
    const char* s = getenv("SPARK_WAIT_TIMEOUT_NS");
    v = s ? strtoull(s, nullptr, 10) : 0ull;
    if (v == 0) v = 1000000000ull;   // 1 s
    cached.store(v);
  }
  return v;
}

// ------------------------------------------------------------ tensor maps ---
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map, dims/strides innermost first (strides in bytes, rank-1 of them).
int make_map_t(CUtensorMap* m, CUtensorMapDataType dtype, CUtensorMapSwizzle swz, const void* ptr, int rank,
               const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SPARK_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, dtype, (cuuint32_t)rank, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SPARK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SPARK_OK;
}

// bf16 tensor map with the 128-byte swizzle
int make_map(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
             const cuuint32_t* box) {
  return make_map_t(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B, ptr, rank, dims, strides,
                    box);
}

// -------------------------------------------------------------- RoPE tables ----
// f_i = theta^(-2i/rot) of the two layer kinds, computed once on the host in
// double precision and passed in the kernel parameters (no device memory;
// safe to use while a stream is being captured).
struct RopeTables {
  spark::RopeFreq freq[2];
};

const RopeTables& rope_tables() {
  static RopeTables t;
  static std::once_flag once;
  std::call_once(once, []() {
    for (int k = 0; k < 2; ++k) {
      const int rot = k == 0 ? 256 : 64;
      const double theta = k == 0 ? 1.0e4 : 5.0e6;
      for (int i = 0; i < 128; ++i) t.freq[k].f[i] = i < rot / 2 ? exp2(-(2.0 * i / rot) * log2(theta)) : 0.0;
    }
  });
  return t;
}

int kind_index(const spark_layer_cfg* cfg) { return cfg->kind == SPARK_SLIDING ? 0 : 1; }

const spark::RopeFreq& rope_freq(const spark_layer_cfg* cfg) { return rope_tables().freq[kind_index(cfg)]; }

// -------------------------------------------------------------- checks -----
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Element strides of a token tensor [B][T][H][256] whose H heads of 256 are contiguous within a
// token (a view of a wider projection output is allowed).  sB = sT = 0 selects the dense layout.
// Otherwise: multiples of 8 elements (16-byte rows), a token's heads fit in sT, sequences do not
// overlap, and both stay below 2^36 elements (tensor-map strides are below 2^40 bytes).
int token_strides(int B, int T, int H, long long* sB, long long* sT, const char* what) {
  const long long row = (long long)H * SPARK_HEAD_DIM;
  if (*sB == 0 && *sT == 0) {
    *sT = row;
    *sB = (long long)T * row;
    return SPARK_OK;
  }
  if (*sT < row || (*sT & 7) || *sB < 0 || (*sB & 7) || *sT >= (1LL << 36) || *sB >= (1LL << 36) ||
      (B > 1 && *sB < (long long)(T - 1) * *sT + row))
    return fail(SPARK_ERR_INVALID_ARG, "%s: strides sB=%lld sT=%lld do not describe [%d][%d][%d][256] token rows",
                what, *sB, *sT, B, T, H);
  if (B == 1) *sB = (long long)T * *sT;      // unused: any value the tensor maps accept
  return SPARK_OK;
}

int check_cfg(const spark_layer_cfg* c) {
  if (!c) return fail(SPARK_ERR_INVALID_ARG, "cfg is NULL");
  if (c->n_q != 16 || c->n_kv != 4 || c->head_dim != 256)
    return fail(SPARK_ERR_UNSUPPORTED, "only n_q 16, n_kv 4, head_dim 256 are built");
  if (fabsf(c->scale - 0.0625f) > 0.0f) return fail(SPARK_ERR_UNSUPPORTED, "scale must be 1/16");
  if (c->kind == SPARK_SLIDING) {
    if (c->window != 512 || c->rot_dim != 256 || c->theta != 1.0e4)
      return fail(SPARK_ERR_INVALID_ARG, "sliding cfg must be window 512, rot 256, theta 1e4");
  } else if (c->kind == SPARK_FULL) {
    if (c->window != 0 || c->rot_dim != 64 || c->theta != 5.0e6)
      return fail(SPARK_ERR_INVALID_ARG, "full cfg must be window 0, rot 64, theta 5e6");
  } else {
    return fail(SPARK_ERR_INVALID_ARG, "unknown layer kind %d", c->kind);
  }
  return SPARK_OK;
}

// ---------------------------------------------------------- decode plan ----
struct DecodePlan {
  int n_splits;
  int tiles_per_split;
};

// Choose the number of key splits per (sequence, KV head): each block streams
// tiles_per_split 64-key tiles; the grid runs in waves of one block per SM.
// Minimise waves * (tiles per block + fixed per-block cost of ~2 tiles).
DecodePlan decode_plan(int B, int cap, int sliding, int sm_count) {
  const int max_keys = sliding ? spark::kWindow : cap;
  const int tiles = (max_keys + spark::kDecNK - 1) / spark::kDecNK;
  const long long units = (long long)B * spark::kNkv;
  DecodePlan best{1, tiles};
  double best_cost = 1e300;
  const int s_max = tiles < 4096 ? tiles : 4096;
  for (int s = 1; s <= s_max; ++s) {
    const int tps = (tiles + s - 1) / s;
    const int s_eff = (tiles + tps - 1) / tps;
    const long long ctas = units * s_eff;
    const long long waves = (ctas + sm_count - 1) / sm_count;
    const double cost = (double)waves * (tps + 2.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best.n_splits = s_eff;
      best.tiles_per_split = tps;
    }
  }
  return best;
}

size_t decode_ws_bytes(int B, const DecodePlan& pl) {
  const size_t rows = (size_t)B * spark::kNq * pl.n_splits;
  return rows * spark::kHeadDim * sizeof(float) + rows * 2 * sizeof(float);
}

// One q8 decode block per SM, like the bf16 one.
DecodePlan decode_q8_plan(int B, int cap, int sliding, int sm_count) {
  return decode_plan(B, cap, sliding, sm_count);
}

// ------------------------------------------------------------ cache views ----
// One layer's K/V storage as the kernels address it: dense [B][4][cap][256]
// or a paged pool [n_pages][4][page][256]; bf16 values, or 8-bit codes with
// fp16 scales ([...][8] per row) when ks/vs are set.
struct CacheView {
  void* k;
  void* v;
  void* ks;             // scales of the 8-bit K codes, nullptr for a bf16 cache
  void* vs;
  int cap;              // logical rows: dense capacity, 512 for a ring, max_pages * page when paged
  int page;             // rows per page (paged), 0 for a dense cache
  int n_pages;
  int max_pages;
  const int* table;     // paged: device int32 [B][max_pages]
  bool q8() const { return ks != nullptr; }
  bool paged() const { return page != 0; }
};

int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

spark::CachePages pages_of(const CacheView& c) {
  if (!c.paged()) return spark::CachePages{nullptr, 0, 0, 0};
  return spark::CachePages{c.table, c.max_pages, ilog2(c.page), c.n_pages};
}

CacheView dense_view(void* k, void* v, void* ks, void* vs, int cap) {
  return CacheView{k, v, ks, vs, cap, 0, 0, 0, nullptr};
}

int paged_view(const spark_paged_kv* kv, const spark_layer_cfg* cfg, CacheView* out) {
  if (!kv) return fail(SPARK_ERR_INVALID_ARG, "kv is NULL");
  if (!kv->k || !kv->v || !kv->block_table) return fail(SPARK_ERR_INVALID_ARG, "null pointer in spark_paged_kv");
  if ((kv->k_scales == nullptr) != (kv->v_scales == nullptr))
    return fail(SPARK_ERR_INVALID_ARG, "pass both scale pools or neither");
  const int P = kv->page_size;
  if (P < 64 || P > 512 || (P & (P - 1)))
    return fail(SPARK_ERR_INVALID_ARG, "page_size %d: a power of two from 64 to 512", P);
  if (kv->n_pages <= 0 || kv->max_pages <= 0)
    return fail(SPARK_ERR_INVALID_ARG, "n_pages %d, max_pages %d", kv->n_pages, kv->max_pages);
  const long long rows = (long long)kv->max_pages * P;
  int cap;
  if (cfg->kind == SPARK_SLIDING) {
    if (rows < SPARK_WINDOW)
      return fail(SPARK_ERR_INVALID_ARG, "a sliding ring needs 512 rows: max_pages * page_size = %lld", rows);
    cap = SPARK_WINDOW;
  } else {
    cap = (int)(rows < SPARK_MAX_POSITION ? rows : SPARK_MAX_POSITION);
  }
  *out = CacheView{kv->k, kv->v, kv->k_scales, kv->v_scales, cap, P, kv->n_pages, kv->max_pages,
                   kv->block_table};
  return SPARK_OK;
}

int check_view(const CacheView& c, const spark_layer_cfg* cfg) {
  if (!c.k || !c.v) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (c.cap <= 0) return fail(SPARK_ERR_INVALID_ARG, "bad cap %d", c.cap);
  const int sliding = cfg->kind == SPARK_SLIDING;
  if (sliding && c.cap != SPARK_WINDOW) return fail(SPARK_ERR_INVALID_ARG, "sliding caches hold 512 rows");
  if (!sliding && c.cap > SPARK_MAX_POSITION) return fail(SPARK_ERR_INVALID_ARG, "cap above 2^20");
  if (!aligned16(c.k) || !aligned16(c.v) || (c.q8() && (!aligned16(c.ks) || !aligned16(c.vs))))
    return fail(SPARK_ERR_INVALID_ARG, "caches must be 16-byte aligned");
  return SPARK_OK;
}

// cu_seqlens == nullptr: k/v [B][T][4][256].  Otherwise packed [total][4][256]
// with sequence b at rows cu_seqlens[b] .. cu_seqlens[b+1]-1 and T the longest.
// key_off / shard: the cache holds positions key_off .. key_off + cap - 1 of a
// full layer sharded across ranks; tokens outside that range are skipped.
// sB, sT: element strides of k and v (0, 0: dense; packed rows of a ragged batch are dense).
int append_impl(const CacheView& c, const void* k, const void* v, int B, int T, const int* pos0,
                const spark_layer_cfg* cfg, unsigned flags, void* stream, const int* cu_seqlens = nullptr,
                int key_off = 0, int shard = 0, long long sB = 0, long long sT = 0) {
  int rc = check_view(c, cfg);
  if (rc) return rc;
  if (!k || !v || !pos0) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || B > 65535 || T <= 0 || T > SPARK_MAX_POSITION)
    return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d T=%d", B, T);
  if ((rc = token_strides(B, T, SPARK_N_KV_HEADS, &sB, &sT, "k, v"))) return rc;
  if (cu_seqlens) sT = (long long)SPARK_N_KV_HEADS * SPARK_HEAD_DIM;
  if (flags & ~SPARK_ROPE_FUSED) return fail(SPARK_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (!aligned16(k) || !aligned16(v)) return fail(SPARK_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  int dev;
  if ((rc = device_ready(&dev))) return rc;
  const int sliding = cfg->kind == SPARK_SLIDING;
  const int t_first = sliding && T > SPARK_WINDOW ? T - SPARK_WINDOW : 0;
  dim3 grid(T - t_first, B);
  const int rope = (flags & SPARK_ROPE_FUSED) ? 1 : 0;
  if (c.q8()) {
    spark::kv_append_q8_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>(
        (uint8_t*)c.k, (__half*)c.ks, (uint8_t*)c.v, (__half*)c.vs, c.cap, (const __nv_bfloat16*)k,
        (const __nv_bfloat16*)v, B, T, sB, sT, t_first, pos0, sliding, rope, rope_freq(cfg), cfg->rot_dim,
        pages_of(c), cu_seqlens, key_off, shard);
  } else {
    spark::kv_append_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>(
        (__nv_bfloat16*)c.k, (__nv_bfloat16*)c.v, c.cap, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, B, T,
        sB, sT, t_first, pos0, sliding, rope, rope_freq(cfg), cfg->rot_dim, pages_of(c), cu_seqlens, key_off, shard);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPARK_OK : cuda_fail(e, c.q8() ? "kv_append_q8_kernel launch" : "kv_append_kernel launch");
}

int current_sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

DecodePlan plan_for(int B, const CacheView& c, int sliding, int sms) {
  return c.q8() ? decode_q8_plan(B, c.cap, sliding, sms) : decode_plan(B, c.cap, sliding, sms);
}

size_t decode_ws_for(int B, const CacheView& c, const spark_layer_cfg* cfg) {
  const int sliding = cfg->kind == SPARK_SLIDING;
  return decode_ws_bytes(B, plan_for(B, c, sliding, current_sm_count()));
}

// Tensor maps of one cache for the decode kernels: K, V (bf16 or codes) and,
// for 8-bit caches, the two scale arrays.
int decode_maps(const CacheView& c, int B, CUtensorMap* km, CUtensorMap* vm, CUtensorMap* ksm, CUtensorMap* vsm) {
  int rc;
  const cuuint64_t row_bytes = c.q8() ? 256 : 512;
  const CUtensorMapDataType dt = c.q8() ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint32_t box_x = c.q8() ? 128 : 64;              // 128 bytes per swizzled box row
  if (!c.paged()) {
    const cuuint64_t dims[3] = {256, (cuuint64_t)c.cap, (cuuint64_t)B * 4};
    const cuuint64_t str[2] = {row_bytes, (cuuint64_t)c.cap * row_bytes};
    const cuuint32_t box[3] = {box_x, 64, 1};
    if ((rc = make_map_t(km, dt, CU_TENSOR_MAP_SWIZZLE_128B, c.k, 3, dims, str, box))) return rc;
    if ((rc = make_map_t(vm, dt, CU_TENSOR_MAP_SWIZZLE_128B, c.v, 3, dims, str, box))) return rc;
    if (c.q8()) {
      const cuuint64_t sd[3] = {8, (cuuint64_t)c.cap, (cuuint64_t)B * 4};
      const cuuint64_t ss[2] = {16, (cuuint64_t)c.cap * 16};
      const cuuint32_t sb[3] = {8, 64, 1};
      if ((rc = make_map_t(ksm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, CU_TENSOR_MAP_SWIZZLE_NONE, c.ks, 3, sd, ss, sb)))
        return rc;
      if ((rc = make_map_t(vsm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, CU_TENSOR_MAP_SWIZZLE_NONE, c.vs, 3, sd, ss, sb)))
        return rc;
    }
  } else {
    const cuuint64_t P = (cuuint64_t)c.page;
    const cuuint64_t dims[4] = {256, P, 4, (cuuint64_t)c.n_pages};
    const cuuint64_t str[3] = {row_bytes, P * row_bytes, 4 * P * row_bytes};
    const cuuint32_t box[4] = {box_x, 64, 1, 1};
    if ((rc = make_map_t(km, dt, CU_TENSOR_MAP_SWIZZLE_128B, c.k, 4, dims, str, box))) return rc;
    if ((rc = make_map_t(vm, dt, CU_TENSOR_MAP_SWIZZLE_128B, c.v, 4, dims, str, box))) return rc;
    if (c.q8()) {
      const cuuint64_t sd[4] = {8, P, 4, (cuuint64_t)c.n_pages};
      const cuuint64_t ss[3] = {16, P * 16, 4 * P * 16};
      const cuuint32_t sb[4] = {8, 64, 1, 1};
      if ((rc = make_map_t(ksm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, CU_TENSOR_MAP_SWIZZLE_NONE, c.ks, 4, sd, ss, sb)))
        return rc;
      if ((rc = make_map_t(vsm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, CU_TENSOR_MAP_SWIZZLE_NONE, c.vs, 4, sd, ss, sb)))
        return rc;
    }
  }
  return SPARK_OK;
}

// The usual plan with fewer, longer splits when its partials would exceed
// max_bytes (at least one split's partials must fit: checked by the caller).
DecodePlan fit_plan(DecodePlan pl, int B, int tiles, size_t max_bytes) {
  if (decode_ws_bytes(B, pl) <= max_bytes) return pl;
  const size_t per_split = decode_ws_bytes(B, DecodePlan{1, tiles});
  const int s_fit = (int)(max_bytes / per_split);
  pl.tiles_per_split = (tiles + s_fit - 1) / s_fit;
  pl.n_splits = (tiles + pl.tiles_per_split - 1) / pl.tiles_per_split;
  return pl;
}

// record != nullptr: context parallelism (a full layer's cache is one rank's
// shard, positions key_off ..): no output, this rank's record is written instead.
// fit_ws: the workspace is a fixed array of ws_bytes; the plan is fitted to it.
// q_sB: element stride between sequences of q (0: dense [B][16][256]).
int decode_impl(void* out, const void* q, const void* gate, const CacheView& c, int B, const int* pos,
                const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes, unsigned flags, void* stream,
                int key_off = 0, float* record = nullptr, bool fit_ws = false, long long q_sB = 0) {
  int rc = check_view(c, cfg);
  if (rc) return rc;
  long long q_sT = q_sB ? (long long)SPARK_N_Q_HEADS * SPARK_HEAD_DIM : 0;     // one token per sequence
  if (B > 0 && B <= 65535 && (rc = token_strides(B, 1, SPARK_N_Q_HEADS, &q_sB, &q_sT, "q"))) return rc;
  if (record) {
    out = record;                      // checked below like an output
    gate = record;
  }
  if (!out || !q || !gate || !pos || !workspace) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || B > 65535) return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d", B);
  if (flags & ~SPARK_ROPE_FUSED) return fail(SPARK_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (!aligned16(out) || !aligned16(q) || !aligned16(workspace))
    return fail(SPARK_ERR_INVALID_ARG, "tensors and workspace must be 16-byte aligned");
  int dev;
  if ((rc = device_ready(&dev))) return rc;
  const int sliding = cfg->kind == SPARK_SLIDING;
  DecodePlan pl = plan_for(B, c, sliding, g_dev[dev].sm_count);
  if (fit_ws) pl = fit_plan(pl, B, ((sliding ? SPARK_WINDOW : c.cap) + spark::kDecNK - 1) / spark::kDecNK, ws_bytes);
  if (ws_bytes < decode_ws_bytes(B, pl))
    return fail(SPARK_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu needed", ws_bytes,
                decode_ws_bytes(B, pl));
  CUtensorMap km, vm, ksm, vsm;
  if ((rc = decode_maps(c, B, &km, &vm, &ksm, &vsm))) return rc;

  spark::DecodeParams P;
  P.q = (const __nv_bfloat16*)q;
  P.q_sB = q_sB;
  P.pos = pos;
  P.o_part = (float*)workspace;
  P.ml_part = (float*)workspace + (size_t)B * spark::kNq * pl.n_splits * spark::kHeadDim;
  P.out = (__nv_bfloat16*)out;
  P.gate = (const __nv_bfloat16*)gate;
  P.B = B;
  P.cap = c.cap;
  P.sliding = sliding;
  P.n_splits = pl.n_splits;
  P.tiles_per_split = pl.tiles_per_split;
  P.rope = (flags & SPARK_ROPE_FUSED) ? 1 : 0;
  P.rot = cfg->rot_dim;
  P.log2_theta = log2(cfg->theta);
  P.freq = rope_freq(cfg);
  P.timeout_ns = wait_timeout_ns();
  P.block_table = c.table;
  P.max_pages = c.max_pages;
  P.page_shift = c.paged() ? ilog2(c.page) : 0;
  P.n_pages = c.n_pages;
  P.key_off = key_off;
  P.shard = record ? 1 : 0;
  if (record) {
    P.out = nullptr;
    P.gate = nullptr;
  }
  dim3 grid(pl.n_splits, spark::kNkv, B);
  cudaStream_t st = (cudaStream_t)stream;
  const char* what;
  if (c.q8()) {
    what = "decode_q8_partial_kernel launch";
    if (c.paged())
      spark::decode_q8_partial_kernel<true><<<grid, spark::kQ8Threads, spark::kQ8SmemBytes, st>>>(km, ksm, vm, vsm, P);
    else
      spark::decode_q8_partial_kernel<false><<<grid, spark::kQ8Threads, spark::kQ8SmemBytes, st>>>(km, ksm, vm, vsm, P);
  } else {
    what = "decode_partial_kernel launch";
    if (c.paged())
      spark::decode_partial_kernel<true><<<grid, spark::kDecThreads, spark::kDecSmemBytes, st>>>(km, vm, P);
    else
      spark::decode_partial_kernel<false><<<grid, spark::kDecThreads, spark::kDecSmemBytes, st>>>(km, vm, P);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  if (record) {
    spark::decode_cp_reduce_kernel<<<dim3(spark::kNq, B), 64, 0, st>>>(record, P.o_part, P.ml_part, pl.n_splits, B);
    e = cudaGetLastError();
    return e == cudaSuccess ? SPARK_OK : cuda_fail(e, "decode_cp_reduce_kernel launch");
  }
  if (pl.n_splits == 1) return SPARK_OK;      // the split kernel wrote the output itself
  spark::decode_combine_kernel<<<dim3(spark::kNq, B), 64, 0, st>>>(
      (__nv_bfloat16*)out, (const __nv_bfloat16*)gate, P.o_part, P.ml_part, pl.n_splits);
  e = cudaGetLastError();
  return e == cudaSuccess ? SPARK_OK : cuda_fail(e, "decode_combine_kernel launch");
}

// ------------------------------------------------------- fused decode ----
// Split plan of spark_attn_decode_fused.  Full layers: the 64-key, one-block-per-SM shape and the
// plan of spark_attn_decode.  Sliding layers: the 32-key shape, two blocks per SM; the same cost
// model with twice the block slots and per-block overhead counted in 32-key tiles.
struct FusedPlan {
  int warps;           // consumer warps: 4 (64-key tiles) or 2 (32-key tiles)
  DecodePlan pl;
};

FusedPlan fused_plan(int B, int cap, int sliding, int sm_count) {
  if (!sliding) return FusedPlan{4, decode_plan(B, cap, 0, sm_count)};
  const int tiles = spark::kWindow / 32;
  const long long units = (long long)B * spark::kNkv;
  const int slots = 2 * sm_count;
  DecodePlan best{1, tiles};
  double best_cost = 1e300;
  for (int s = 1; s <= tiles; ++s) {
    const int tps = (tiles + s - 1) / s;
    const int s_eff = (tiles + tps - 1) / tps;
    const long long waves = (units * s_eff + slots - 1) / slots;
    const double cost = (double)waves * (tps + 4.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = DecodePlan{s_eff, tps};
    }
  }
  return FusedPlan{2, best};
}

// Workspace: the arrival counters first (B * 4 ints, at a fixed place whatever the plan, so one
// workspace can serve layers of both kinds in turn), then the partials.
size_t fused_cnt_bytes(int B) { return ((size_t)B * spark::kNkv * sizeof(int) + 255) & ~(size_t)255; }

size_t decode_fused_ws_bytes(int B, int cap, int sliding, int sm_count) {
  return fused_cnt_bytes(B) + decode_ws_bytes(B, fused_plan(B, cap, sliding, sm_count).pl);
}

template <int kW, int kG>
cudaError_t launch_fused(const CUtensorMap& km, const CUtensorMap& vm, const spark::DecodeFusedParams& P, int B,
                         cudaStream_t st) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)P.n_splits, spark::kNkv, (unsigned)B);
  lc.blockDim = dim3(spark::DfShape<kW, kG>::kThreads);
  lc.dynamicSmemBytes = spark::DfShape<kW, kG>::kSmemBytes;
  lc.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, spark::decode_fused_kernel<kW, kG>, km, vm, P);
}

int decode_fused_impl(void* out, const void* q, long long q_sB, const void* k, const void* v, long long kv_sB,
                      const void* gate, void* k_cache, void* v_cache, int cap, int B, const int* pos,
                      const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes, unsigned flags, void* stream) {
  const CacheView c = dense_view(k_cache, v_cache, nullptr, nullptr, cap);
  int rc = check_view(c, cfg);
  if (rc) return rc;
  if (!out || !q || !k || !v || !gate || !pos || !workspace) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || B > 65535) return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d", B);
  long long q_sT = q_sB ? (long long)SPARK_N_Q_HEADS * SPARK_HEAD_DIM : 0;      // one token per sequence
  long long kv_sT = kv_sB ? (long long)SPARK_N_KV_HEADS * SPARK_HEAD_DIM : 0;
  if ((rc = token_strides(B, 1, SPARK_N_Q_HEADS, &q_sB, &q_sT, "q"))) return rc;
  if ((rc = token_strides(B, 1, SPARK_N_KV_HEADS, &kv_sB, &kv_sT, "k, v"))) return rc;
  if (flags & ~SPARK_ROPE_FUSED) return fail(SPARK_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(workspace))
    return fail(SPARK_ERR_INVALID_ARG, "tensors and workspace must be 16-byte aligned");
  int dev;
  if ((rc = device_ready(&dev))) return rc;
  const int sliding = cfg->kind == SPARK_SLIDING;
  const int sms = g_dev[dev].sm_count;
  const FusedPlan fp = fused_plan(B, cap, sliding, sms);
  if (ws_bytes < decode_fused_ws_bytes(B, cap, sliding, sms))
    return fail(SPARK_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu needed", ws_bytes,
                decode_fused_ws_bytes(B, cap, sliding, sms));
  // K and V maps with boxes of the shape's tile (64-dim slabs of 16 * warps keys)
  CUtensorMap km, vm;
  {
    const cuuint64_t dims[3] = {256, (cuuint64_t)cap, (cuuint64_t)B * 4};
    const cuuint64_t str[2] = {512, (cuuint64_t)cap * 512};
    const cuuint32_t box[3] = {64, (cuuint32_t)(16 * fp.warps), 1};
    if ((rc = make_map(&km, k_cache, 3, dims, str, box))) return rc;
    if ((rc = make_map(&vm, v_cache, 3, dims, str, box))) return rc;
  }
  spark::DecodeFusedParams P;
  P.q = (const __nv_bfloat16*)q;
  P.k_new = (const __nv_bfloat16*)k;
  P.v_new = (const __nv_bfloat16*)v;
  P.q_sB = q_sB;
  P.kv_sB = kv_sB;
  P.gate = (const __nv_bfloat16*)gate;
  P.pos = pos;
  P.out = (__nv_bfloat16*)out;
  P.k_cache = (__nv_bfloat16*)k_cache;
  P.v_cache = (__nv_bfloat16*)v_cache;
  P.cnt = (int*)workspace;
  P.o_part = (float*)((char*)workspace + fused_cnt_bytes(B));
  P.ml_part = P.o_part + (size_t)B * spark::kNq * fp.pl.n_splits * spark::kHeadDim;
  P.B = B;
  P.cap = cap;
  P.sliding = sliding;
  P.n_splits = fp.pl.n_splits;
  P.tiles_per_split = fp.pl.tiles_per_split;
  P.rope = (flags & SPARK_ROPE_FUSED) ? 1 : 0;
  P.rot = cfg->rot_dim;
  P.timeout_ns = wait_timeout_ns();
  P.freq = rope_freq(cfg);
  const cudaError_t e = fp.warps == 2 ? launch_fused<2, 2>(km, vm, P, B, (cudaStream_t)stream)
                                      : launch_fused<4, 1>(km, vm, P, B, (cudaStream_t)stream);
  return e == cudaSuccess ? SPARK_OK : cuda_fail(e, "decode_fused_kernel launch");
}

// ------------------------------------------------- context parallelism ----
int check_cp_shard(int cap, int key_off, const spark_layer_cfg* cfg) {
  if (cfg->kind != SPARK_FULL)
    return fail(SPARK_ERR_UNSUPPORTED, "context parallelism shards full layers only (sliding layers hold 512 rows)");
  if (key_off < 0 || key_off >= SPARK_MAX_POSITION || cap <= 0 || cap > SPARK_MAX_POSITION - key_off)
    return fail(SPARK_ERR_INVALID_ARG, "shard of %d rows at %d outside [0, 2^20)", cap, key_off);
  return SPARK_OK;
}

// ------------------------------------------------- decode without workspace ----
// Some callers cannot allocate device memory when they run attention: a
// serving runtime that plans all of its memory at start-up and forbids any
// allocation afterwards, a host application that only lends the library its
// input and output buffers, or code that runs while a stream is being recorded
// into a CUDA graph, where cudaMalloc cannot be recorded.  For them
// spark_attn_decode_static keeps the split-KV partials in this fixed array of
// the library's own device memory instead of a caller workspace.  Every GPU
// that loads the library holds these 16 MiB until the process exits.
constexpr size_t kStaticScratchBytes = (size_t)SPARK_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is asked of the
// runtime once per device, with that device current; only a successful answer
// is kept (a failed lookup is retried by the next call).  The lookup is refused
// while `stream` is being captured into a graph: the first call on a device
// must come before any capture.
int static_scratch(int dev, cudaStream_t stream, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cs);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    if (cs != cudaStreamCaptureStatusNone)
      return fail(SPARK_ERR_INVALID_ARG,
                  "the first spark_attn_decode_static call on a device must come before any stream capture");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    if (p == nullptr) return fail(SPARK_ERR_CUDA, "cudaGetSymbolAddress(scratch) returned NULL");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SPARK_OK;
}

}  // namespace

extern "C" {

int spark_version(void) { return 100; }

const char* spark_last_error(void) { return g_last_error; }

int spark_layer_cfg_for_kind(int kind, spark_layer_cfg* out) {
  if (!out) return fail(SPARK_ERR_INVALID_ARG, "out is NULL");
  spark_layer_cfg c;
  c.kind = kind;
  c.n_q = 16;
  c.n_kv = 4;
  c.head_dim = 256;
  c.scale = 0.0625f;
  if (kind == SPARK_SLIDING) {
    c.window = 512;
    c.rot_dim = 256;
    c.theta = 1.0e4;
  } else if (kind == SPARK_FULL) {
    c.window = 0;
    c.rot_dim = 64;
    c.theta = 5.0e6;
  } else {
    return fail(SPARK_ERR_INVALID_ARG, "unknown layer kind %d", kind);
  }
  *out = c;
  return SPARK_OK;
}

int spark_layer_cfg_for_layer(int layer, spark_layer_cfg* out) {
  if (layer < 0 || layer >= SPARK_N_LAYERS) return fail(SPARK_ERR_INVALID_ARG, "layer %d outside [0, 36)", layer);
  return spark_layer_cfg_for_kind(layer % 4 == 3 ? SPARK_FULL : SPARK_SLIDING, out);
}

long long spark_kv_cache_bytes(const spark_layer_cfg* cfg, int B, long long cap) {
  if (check_cfg(cfg) != SPARK_OK || B <= 0 || cap <= 0) return -1;
  return 2LL * B * cfg->n_kv * cap * cfg->head_dim * 2LL;
}

long long spark_stack_kv_bytes(int B, long long ctx) {
  if (B <= 0 || ctx < 0) return -1;
  long long total = 0;
  for (int l = 0; l < SPARK_N_LAYERS; ++l) {
    const long long rows = (l % 4 == 3) ? ctx : (ctx < SPARK_WINDOW ? ctx : SPARK_WINDOW);
    total += 2LL * B * SPARK_N_KV_HEADS * rows * SPARK_HEAD_DIM * 2LL;
  }
  return total;
}

int spark_rope_apply(void* x, int B, int T, int H, long long sB, long long sT, const int* pos0,
                     const spark_layer_cfg* cfg, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!x || !pos0) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || T <= 0 || T > SPARK_MAX_POSITION || (H != 16 && H != 4))
    return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d T=%d H=%d", B, T, H);
  if ((rc = token_strides(B, T, H, &sB, &sT, "x"))) return rc;
  if (!aligned16(x)) return fail(SPARK_ERR_INVALID_ARG, "x must be 16-byte aligned");
  int dev;
  if ((rc = device_ready(&dev))) return rc;
  if (H == 16) {
    // a thread per (token, two pairs), kRopeIters tokens per thread
    const int tok_per_block = 128 / (cfg->rot_dim / 4) * spark::kRopeIters;
    const long long grid = ((long long)B * T + tok_per_block - 1) / tok_per_block;
    if (grid > 0x7FFFFFFFLL) return fail(SPARK_ERR_INVALID_ARG, "too many tokens");
    spark::rope16_kernel<<<(unsigned)grid, 128, 0, (cudaStream_t)stream>>>((__nv_bfloat16*)x, B, T, sB, sT, pos0,
                                                                           rope_freq(cfg), cfg->rot_dim, nullptr);
  } else {
    // a thread per (eight-pair chunk, run of kRopeRun tokens); 128 / chunks runs per block
    const int runs_per_block = 128 / (cfg->rot_dim / 16);
    const long long runs = (long long)B * ((T + spark::kRopeRun - 1) / spark::kRopeRun);
    const long long grid = (runs + runs_per_block - 1) / runs_per_block;
    if (grid > 0x7FFFFFFFLL) return fail(SPARK_ERR_INVALID_ARG, "too many tokens");
    spark::rope_kernel<<<(unsigned)grid, 128, 0, (cudaStream_t)stream>>>((__nv_bfloat16*)x, B, T, H, sB, sT, pos0,
                                                                         rope_freq(cfg), cfg->rot_dim, nullptr);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPARK_OK : cuda_fail(e, "rope_kernel launch");
}

int spark_kv_append(void* k_cache, void* v_cache, int cap, const void* k, const void* v, int B,
                    int T, long long sB, long long sT, const int* pos0, const spark_layer_cfg* cfg, unsigned flags,
                    void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  return append_impl(dense_view(k_cache, v_cache, nullptr, nullptr, cap), k, v, B, T, pos0, cfg, flags, stream,
                     nullptr, 0, 0, sB, sT);
}

size_t spark_decode_workspace_bytes(int B, int cap, const spark_layer_cfg* cfg) {
  if (check_cfg(cfg) != SPARK_OK || B <= 0 || cap <= 0) return 0;
  return decode_ws_for(B, dense_view((void*)1, (void*)1, nullptr, nullptr, cap), cfg);
}

int spark_attn_decode(void* out, const void* q, long long q_sB, const void* gate, const void* k_cache,
                      const void* v_cache, int cap, int B, const int* pos,
                      const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes,
                      unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  return decode_impl(out, q, gate, dense_view((void*)k_cache, (void*)v_cache, nullptr, nullptr, cap), B, pos, cfg,
                     workspace, ws_bytes, flags, stream, 0, nullptr, false, q_sB);
}

size_t spark_decode_fused_workspace_bytes(int B, int cap, const spark_layer_cfg* cfg) {
  if (check_cfg(cfg) != SPARK_OK || B <= 0 || B > 65535 || cap <= 0) return 0;
  return decode_fused_ws_bytes(B, cap, cfg->kind == SPARK_SLIDING, current_sm_count());
}

int spark_attn_decode_fused(void* out, const void* q, long long q_sB, const void* k, const void* v,
                            long long kv_sB, const void* gate, void* k_cache, void* v_cache, int cap, int B,
                            const int* pos, const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes,
                            unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  return decode_fused_impl(out, q, q_sB, k, v, kv_sB, gate, k_cache, v_cache, cap, B, pos, cfg, workspace,
                           ws_bytes, flags, stream);
}

long long spark_kv_cache_q8_bytes(const spark_layer_cfg* cfg, int B, long long cap) {
  if (check_cfg(cfg) != SPARK_OK || B <= 0 || cap <= 0) return -1;
  return 2LL * B * cfg->n_kv * cap * (cfg->head_dim + 2LL * (cfg->head_dim / 32));
}

int spark_kv_append_q8(void* k_codes, void* k_scales, void* v_codes, void* v_scales, int cap,
                       const void* k, const void* v, int B, int T, const int* pos0,
                       const spark_layer_cfg* cfg, unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!k_scales || !v_scales) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  return append_impl(dense_view(k_codes, v_codes, k_scales, v_scales, cap), k, v, B, T, pos0, cfg, flags,
                     stream);
}

size_t spark_decode_q8_workspace_bytes(int B, int cap, const spark_layer_cfg* cfg) {
  if (check_cfg(cfg) != SPARK_OK || B <= 0 || cap <= 0) return 0;
  return decode_ws_for(B, dense_view((void*)1, (void*)1, (void*)1, (void*)1, cap), cfg);
}

int spark_attn_decode_q8(void* out, const void* q, const void* gate, const void* k_codes,
                         const void* k_scales, const void* v_codes, const void* v_scales, int cap,
                         int B, const int* pos, const spark_layer_cfg* cfg, void* workspace,
                         size_t ws_bytes, unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!k_scales || !v_scales) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  return decode_impl(out, q, gate,
                     dense_view((void*)k_codes, (void*)v_codes, (void*)k_scales, (void*)v_scales, cap), B, pos,
                     cfg, workspace, ws_bytes, flags, stream);
}

int spark_kv_append_paged(const spark_paged_kv* kv, const void* k, const void* v, int B, int T,
                          const int* pos0, const spark_layer_cfg* cfg, unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  CacheView c;
  if ((rc = paged_view(kv, cfg, &c))) return rc;
  return append_impl(c, k, v, B, T, pos0, cfg, flags, stream);
}

size_t spark_decode_paged_workspace_bytes(int B, const spark_paged_kv* kv, const spark_layer_cfg* cfg) {
  CacheView c;
  if (check_cfg(cfg) != SPARK_OK || B <= 0 || paged_view(kv, cfg, &c) != SPARK_OK) return 0;
  return decode_ws_for(B, c, cfg);
}

int spark_attn_decode_paged(void* out, const void* q, const void* gate, const spark_paged_kv* kv, int B,
                            const int* pos, const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes,
                            unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  CacheView c;
  if ((rc = paged_view(kv, cfg, &c))) return rc;
  return decode_impl(out, q, gate, c, B, pos, cfg, workspace, ws_bytes, flags, stream);
}

// Everything a prefill needs before it launches: the arguments checked, the tensor maps encoded and
// the kernel parameters filled.  Nothing is launched until every check has passed.
struct PrefillPlan {
  CUtensorMap qm, km, vm, kcm, vcm, om;
  spark::PrefillParams P;
  long long blocks;
  bool has_cache, sliding;
  long long kv_sB, kv_sT;        // k, v element strides, dense ones filled in
};

int prefill_prepare(PrefillPlan& L, void* out, const void* q, const void* k, const void* v, const void* gate,
                    const void* k_cache, const void* v_cache, int cap, int B, int T, long long q_sB, long long q_sT,
                    long long kv_sB, long long kv_sT, const int* pos0, const spark_layer_cfg* cfg, unsigned flags) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!out || !q || !k || !v || !gate || !pos0) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if ((k_cache == nullptr) != (v_cache == nullptr))
    return fail(SPARK_ERR_INVALID_ARG, "pass both caches or neither");
  if (B <= 0 || B > 65535 || T <= 0 || T > SPARK_MAX_POSITION)
    return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d T=%d", B, T);
  if ((rc = token_strides(B, T, SPARK_N_Q_HEADS, &q_sB, &q_sT, "q"))) return rc;
  if ((rc = token_strides(B, T, SPARK_N_KV_HEADS, &kv_sB, &kv_sT, "k, v"))) return rc;
  if (flags & ~(SPARK_ROPE_FUSED | SPARK_APPEND_FUSED)) return fail(SPARK_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if ((flags & SPARK_APPEND_FUSED) && !k_cache)
    return fail(SPARK_ERR_INVALID_ARG, "SPARK_APPEND_FUSED needs the caches to append to");
  const int sliding = cfg->kind == SPARK_SLIDING;
  if (k_cache) {
    if (sliding && cap != SPARK_WINDOW) return fail(SPARK_ERR_INVALID_ARG, "sliding caches hold 512 rows");
    if (!sliding && (cap <= 0 || cap > SPARK_MAX_POSITION)) return fail(SPARK_ERR_INVALID_ARG, "bad cap %d", cap);
  }
  if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (k_cache && (!aligned16(k_cache) || !aligned16(v_cache))))
    return fail(SPARK_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  int dev;
  if ((rc = device_ready(&dev))) return rc;

  // Q, chunk K/V: [B][T][H][256] as 4-D (dim, head, token, batch) with the callers' token and
  // sequence strides; out dense; caches [B][4][cap][256] as 3-D (dim, row, batch*head).
  // 128-byte swizzled boxes of 64 dims.
  {
    const cuuint64_t dq[4] = {256, 16, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t sq[3] = {512, 2ull * (cuuint64_t)q_sT, 2ull * (cuuint64_t)q_sB};
    const cuuint64_t so[3] = {512, 512ull * 16, 512ull * 16 * T};
    const cuuint32_t bq[4] = {64, 1, (cuuint32_t)spark::kPfM, 1};
    if ((rc = make_map(&L.qm, q, 4, dq, sq, bq))) return rc;
    if ((rc = make_map(&L.om, out, 4, dq, so, bq))) return rc;
    const cuuint64_t dk[4] = {256, 4, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t sk[3] = {512, 2ull * (cuuint64_t)kv_sT, 2ull * (cuuint64_t)kv_sB};
    const cuuint32_t bk[4] = {64, 1, (cuuint32_t)(spark::kPfN / 2), 1};   // each block of the pair: 64 keys
    const cuuint32_t bv[4] = {64, 1, 32, 1};
    if ((rc = make_map(&L.km, k, 4, dk, sk, bk))) return rc;
    if ((rc = make_map(&L.vm, v, 4, dk, sk, bv))) return rc;
    if (k_cache) {
      const cuuint64_t dc[3] = {256, (cuuint64_t)cap, (cuuint64_t)B * 4};
      const cuuint64_t sc[2] = {512, (cuuint64_t)cap * 512};
      const cuuint32_t bkc[3] = {64, (cuuint32_t)(spark::kPfN / 2), 1};
      const cuuint32_t bvc[3] = {64, 32, 1};
      if ((rc = make_map(&L.kcm, k_cache, 3, dc, sc, bkc))) return rc;
      if ((rc = make_map(&L.vcm, v_cache, 3, dc, sc, bvc))) return rc;
    } else {
      L.kcm = L.km;
      L.vcm = L.vm;
    }
  }
  spark::PrefillParams& P = L.P;
  P.out = (__nv_bfloat16*)out;
  P.gate = (const __nv_bfloat16*)gate;
  P.pos0 = pos0;
  P.B = B;
  P.T = T;
  P.cap = k_cache ? cap : 0;
  P.sliding = sliding;
  P.has_cache = k_cache ? 1 : 0;
  P.n_qt = (T + spark::kPfM - 1) / spark::kPfM;
  P.rope = (flags & SPARK_ROPE_FUSED) ? 1 : 0;
  P.rot = cfg->rot_dim;
  P.log2_theta = log2(cfg->theta);
  P.freq = rope_freq(cfg);
  P.timeout_ns = wait_timeout_ns();
  P.cu_seqlens = nullptr;
  P.block_table = nullptr;
  P.max_pages = P.page_shift = P.n_pages = 0;
  L.blocks = (long long)B * spark::kNq * P.n_qt;
  if (L.blocks > 0x7FFFFFFFLL) return fail(SPARK_ERR_INVALID_ARG, "grid too large");
  L.has_cache = k_cache != nullptr;
  L.sliding = sliding != 0;
  L.kv_sB = kv_sB;
  L.kv_sT = kv_sT;
  return SPARK_OK;
}

int prefill_launch(const PrefillPlan& L, void* stream) {
  cudaError_t e;
  if (!L.has_cache || L.sliding) {
    // the persistent kernel: one cluster per unit (two query heads x one 128-query tile); resident
    // clusters take the units of clusters that have not started (cluster launch control).  Full
    // layers with a history (units of hundreds of KV tiles) measured 5-8 % faster in prefill2.
    if (L.has_cache)
      spark::prefill3_kernel<true><<<(unsigned)L.blocks, spark::kPfThreads, spark::kP2SmemBytes,
                                     (cudaStream_t)stream>>>(L.qm, L.km, L.vm, L.kcm, L.vcm, L.om, L.P);
    else
      spark::prefill3_kernel<false><<<(unsigned)L.blocks, spark::kPfThreads, spark::kP2SmemBytes,
                                      (cudaStream_t)stream>>>(L.qm, L.km, L.vm, L.kcm, L.vcm, L.om, L.P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prefill3_kernel launch");
  } else {
    // clusters of two blocks (an SM pair): two query heads of a KV group, same query tile
    spark::prefill2_kernel<false><<<(unsigned)L.blocks, spark::kPfThreads, spark::kP2SmemBytes,
                                    (cudaStream_t)stream>>>(L.qm, L.km, L.vm, L.kcm, L.vcm, L.om, L.P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prefill2_kernel launch");
  }
  return SPARK_OK;
}

int spark_attn_prefill(void* out, const void* q, const void* k, const void* v, const void* gate,
                       const void* k_cache, const void* v_cache, int cap, int B, int T, long long q_sB,
                       long long q_sT, long long kv_sB, long long kv_sT, const int* pos0, const spark_layer_cfg* cfg,
                       unsigned flags, void* stream) {
  PrefillPlan L;
  int rc = prefill_prepare(L, out, q, k, v, gate, k_cache, v_cache, cap, B, T, q_sB, q_sT, kv_sB, kv_sT, pos0, cfg,
                           flags);
  if (rc) return rc;
  if ((rc = prefill_launch(L, stream))) return rc;
  if (!(flags & SPARK_APPEND_FUSED)) return SPARK_OK;
  // the chunk's k (rotated) and v into the cache, after the attention on the same stream: a sliding
  // ring's rows are overwritten only once the attention has read them as history
  return append_impl(dense_view((void*)k_cache, (void*)v_cache, nullptr, nullptr, cap), k, v, B, T, pos0, cfg, 0,
                     stream, nullptr, 0, 0, L.kv_sB, L.kv_sT);
}

size_t spark_prefill_q8_workspace_bytes(int B, int cap, const spark_layer_cfg* cfg) {
  if (check_cfg(cfg) != SPARK_OK || B <= 0 || B > 65535 || cap <= 0 || cap > SPARK_MAX_POSITION) return 0;
  if (cfg->kind == SPARK_SLIDING && cap != SPARK_WINDOW) return 0;
  return 2ull * B * SPARK_N_KV_HEADS * (size_t)cap * SPARK_HEAD_DIM * 2;
}

int spark_attn_prefill_q8(void* out, const void* q, const void* k, const void* v, const void* gate,
                          const void* k_codes, const void* k_scales, const void* v_codes, const void* v_scales,
                          int cap, int B, int T, long long q_sB, long long q_sT, long long kv_sB, long long kv_sT,
                          const int* pos0, const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes,
                          unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!k_codes || !k_scales || !v_codes || !v_scales || !workspace || !pos0)
    return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (flags & ~(SPARK_ROPE_FUSED | SPARK_APPEND_FUSED)) return fail(SPARK_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (B <= 0 || B > 65535 || T <= 0 || T > SPARK_MAX_POSITION)
    return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d T=%d", B, T);
  const size_t need = spark_prefill_q8_workspace_bytes(B, cap, cfg);
  if (need == 0) return fail(SPARK_ERR_INVALID_ARG, "bad cap %d for this layer", cap);
  if (ws_bytes < need) return fail(SPARK_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  if (!aligned16(k_codes) || !aligned16(v_codes) || !aligned16(k_scales) || !aligned16(v_scales) ||
      !aligned16(workspace))
    return fail(SPARK_ERR_INVALID_ARG, "codes, scales and workspace must be 16-byte aligned");
  const CacheView q8c = dense_view((void*)k_codes, (void*)v_codes, (void*)k_scales, (void*)v_scales, cap);
  if ((rc = check_view(q8c, cfg))) return rc;
  __nv_bfloat16* hk = (__nv_bfloat16*)workspace;
  __nv_bfloat16* hv = hk + need / 4;
  // the bf16 prefill over the workspace, checked and set up before anything is launched
  PrefillPlan L;
  if ((rc = prefill_prepare(L, out, q, k, v, gate, hk, hv, cap, B, T, q_sB, q_sT, kv_sB, kv_sT, pos0, cfg,
                            flags & ~SPARK_APPEND_FUSED)))
    return rc;
  spark::q8_history_kernel<<<dim3((unsigned)((cap + 3) / 4), SPARK_N_KV_HEADS, (unsigned)B), 256, 0,
                             (cudaStream_t)stream>>>((const uint8_t*)k_codes, (const __half*)k_scales,
                                                     (const uint8_t*)v_codes, (const __half*)v_scales, cap, pos0,
                                                     hk, hv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "q8_history_kernel launch");
  if ((rc = prefill_launch(L, stream)) || !(flags & SPARK_APPEND_FUSED)) return rc;
  // the chunk's k (rotated) and v, quantised into the 8-bit cache after the attention
  return append_impl(q8c, k, v, B, T, pos0, cfg, 0, stream, nullptr, 0, 0, L.kv_sB, L.kv_sT);
}

int spark_rope_apply_varlen(void* x, int H, const int* cu_seqlens, int max_seqlen, const int* pos0, int B,
                            const spark_layer_cfg* cfg, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!x || !pos0 || !cu_seqlens) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || B > 65535 || max_seqlen <= 0 || max_seqlen > SPARK_MAX_POSITION || (H != 16 && H != 4))
    return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d max_seqlen=%d H=%d", B, max_seqlen, H);
  if (!aligned16(x)) return fail(SPARK_ERR_INVALID_ARG, "x must be 16-byte aligned");
  int dev;
  if ((rc = device_ready(&dev))) return rc;
  if (H == 16) {
    const int tok_per_block = 128 / (cfg->rot_dim / 4) * spark::kRopeIters;
    dim3 grid((max_seqlen + tok_per_block - 1) / tok_per_block, B);
    spark::rope16_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>((__nv_bfloat16*)x, B, max_seqlen, 0,
                                                                 (long long)H * SPARK_HEAD_DIM, pos0, rope_freq(cfg),
                                                                 cfg->rot_dim, cu_seqlens);
  } else {
    const int runs_per_block = 128 / (cfg->rot_dim / 16);
    const int runs = (max_seqlen + spark::kRopeRun - 1) / spark::kRopeRun;
    dim3 grid((runs + runs_per_block - 1) / runs_per_block, B);
    spark::rope_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>((__nv_bfloat16*)x, B, max_seqlen, H, 0,
                                                               (long long)H * SPARK_HEAD_DIM, pos0, rope_freq(cfg),
                                                               cfg->rot_dim, cu_seqlens);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPARK_OK : cuda_fail(e, "rope_kernel launch");
}

int spark_kv_append_varlen(const spark_paged_kv* kv, const void* k, const void* v, const int* cu_seqlens,
                           int max_seqlen, const int* pos0, int B, const spark_layer_cfg* cfg, unsigned flags,
                           void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!cu_seqlens) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  CacheView c;
  if ((rc = paged_view(kv, cfg, &c))) return rc;
  return append_impl(c, k, v, B, max_seqlen, pos0, cfg, flags, stream, cu_seqlens);
}

int spark_attn_prefill_varlen(void* out, const void* q, const void* k, const void* v, const void* gate,
                              const int* cu_seqlens, int total, int max_seqlen, const int* pos0,
                              const spark_paged_kv* history, int B, const spark_layer_cfg* cfg, unsigned flags,
                              void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!out || !q || !k || !v || !gate || !pos0 || !cu_seqlens) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || B > 65535 || total <= 0 || max_seqlen <= 0 || max_seqlen > SPARK_MAX_POSITION)
    return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d total=%d max_seqlen=%d", B, total, max_seqlen);
  if (flags & ~SPARK_ROPE_FUSED) return fail(SPARK_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(SPARK_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  CacheView c{};
  if (history) {
    if ((rc = paged_view(history, cfg, &c))) return rc;
    if (c.q8()) return fail(SPARK_ERR_UNSUPPORTED, "prefill reads bf16 history pages only");
    if ((rc = check_view(c, cfg))) return rc;
  }
  int dev;
  if ((rc = device_ready(&dev))) return rc;
  const int sliding = cfg->kind == SPARK_SLIDING;

  // packed q, out [total][16][256] and k, v [total][4][256] as 4-D (dim, head, row, 1);
  // the history pool [n_pages][4][page][256] as 4-D (dim, row in page, head, page)
  CUtensorMap qm, km, vm, kcm, vcm, om;
  {
    const cuuint64_t dq[4] = {256, 16, (cuuint64_t)total, 1};
    const cuuint64_t sq[3] = {512, 512ull * 16, 512ull * 16 * total};
    const cuuint32_t bq[4] = {64, 1, (cuuint32_t)spark::kPfM, 1};
    if ((rc = make_map(&qm, q, 4, dq, sq, bq))) return rc;
    if ((rc = make_map(&om, out, 4, dq, sq, bq))) return rc;
    const cuuint64_t dk[4] = {256, 4, (cuuint64_t)total, 1};
    const cuuint64_t sk[3] = {512, 512ull * 4, 512ull * 4 * total};
    const cuuint32_t bk[4] = {64, 1, (cuuint32_t)(spark::kPfN / 2), 1};
    const cuuint32_t bv[4] = {64, 1, 32, 1};
    if ((rc = make_map(&km, k, 4, dk, sk, bk))) return rc;
    if ((rc = make_map(&vm, v, 4, dk, sk, bv))) return rc;
    if (history) {
      const cuuint64_t Pg = (cuuint64_t)c.page;
      const cuuint64_t dc[4] = {256, Pg, 4, (cuuint64_t)c.n_pages};
      const cuuint64_t sc[3] = {512, Pg * 512, 4 * Pg * 512};
      const cuuint32_t bkc[4] = {64, (cuuint32_t)(spark::kPfN / 2), 1, 1};
      const cuuint32_t bvc[4] = {64, 32, 1, 1};
      if ((rc = make_map(&kcm, c.k, 4, dc, sc, bkc))) return rc;
      if ((rc = make_map(&vcm, c.v, 4, dc, sc, bvc))) return rc;
    } else {
      kcm = km;
      vcm = vm;
    }
  }
  spark::PrefillParams P;
  P.out = (__nv_bfloat16*)out;
  P.gate = (const __nv_bfloat16*)gate;
  P.pos0 = pos0;
  P.B = B;
  P.T = max_seqlen;
  P.cap = history ? c.cap : 0;
  P.sliding = sliding;
  P.has_cache = history ? 1 : 0;
  P.n_qt = (max_seqlen + spark::kPfM - 1) / spark::kPfM;
  P.rope = (flags & SPARK_ROPE_FUSED) ? 1 : 0;
  P.rot = cfg->rot_dim;
  P.log2_theta = log2(cfg->theta);
  P.freq = rope_freq(cfg);
  P.timeout_ns = wait_timeout_ns();
  P.cu_seqlens = cu_seqlens;
  P.block_table = history ? c.table : nullptr;
  P.max_pages = history ? c.max_pages : 0;
  P.page_shift = history ? ilog2(c.page) : 0;
  P.n_pages = history ? c.n_pages : 0;
  const long long blocks = (long long)B * spark::kNq * P.n_qt;
  if (blocks > 0x7FFFFFFFLL) return fail(SPARK_ERR_INVALID_ARG, "grid too large");
  spark::prefill2_kernel<true><<<(unsigned)blocks, spark::kPfThreads, spark::kP2SmemBytes, (cudaStream_t)stream>>>(
      qm, km, vm, kcm, vcm, om, P);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPARK_OK : cuda_fail(e, "prefill2_kernel launch");
}

int spark_attn_decode_static(void* out, const void* q, const void* gate, const void* k_cache,
                             const void* v_cache, int cap, int B, const int* pos,
                             const spark_layer_cfg* cfg, unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (B <= 0 || B > 65535) return fail(SPARK_ERR_INVALID_ARG, "bad shape B=%d", B);
  // one split needs a partial row (256 + 2 floats) per sequence and query head
  const size_t per_split = (size_t)B * spark::kNq * (spark::kHeadDim + 2) * sizeof(float);
  if (per_split > kStaticScratchBytes)
    return fail(SPARK_ERR_INVALID_ARG,
                "B=%d needs %zu bytes of scratch, above the %zu-byte static scratch (at most %zu sequences)",
                B, per_split, kStaticScratchBytes,
                kStaticScratchBytes / ((size_t)spark::kNq * (spark::kHeadDim + 2) * sizeof(float)));
  int dev;
  if ((rc = device_ready(&dev))) return rc;
  void* scratch = nullptr;
  if ((rc = static_scratch(dev, (cudaStream_t)stream, &scratch))) return rc;
  // the usual split plan, with fewer splits when its partials would not fit the array
  return decode_impl(out, q, gate, dense_view((void*)k_cache, (void*)v_cache, nullptr, nullptr, cap), B, pos, cfg,
                     scratch, kStaticScratchBytes, flags, stream, 0, nullptr, true);
}

// Split plan of spark_attn_decode_static (host only, for tests): writes n_splits and
// tiles_per_split for `sm_count` SMs; returns the partials' bytes, 0 on bad arguments.
size_t spark_decode_static_plan(int B, int cap, const spark_layer_cfg* cfg, int sm_count, int* n_splits,
                                int* tiles_per_split) {
  if (check_cfg(cfg) != SPARK_OK || B <= 0 || B > 65535 || cap <= 0 || sm_count <= 0) return 0;
  const size_t per_split = (size_t)B * spark::kNq * (spark::kHeadDim + 2) * sizeof(float);
  if (per_split > kStaticScratchBytes) return 0;
  const int sliding = cfg->kind == SPARK_SLIDING;
  const int tiles = ((sliding ? SPARK_WINDOW : cap) + spark::kDecNK - 1) / spark::kDecNK;
  const DecodePlan pl = fit_plan(decode_plan(B, cap, sliding, sm_count), B, tiles, kStaticScratchBytes);
  if (n_splits) *n_splits = pl.n_splits;
  if (tiles_per_split) *tiles_per_split = pl.tiles_per_split;
  return decode_ws_bytes(B, pl);
}

int spark_selftest_wait_timeout(unsigned long long timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull)
    return fail(SPARK_ERR_INVALID_ARG, "timeout_ns must be in (0, 10 s]");
  int rc, dev;
  if ((rc = device_ready(&dev))) return rc;
  spark::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(timeout_ns);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPARK_OK : cuda_fail(e, "selftest_wait_kernel launch");
}

int spark_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned word = 0, info = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, spark::g_error_word, sizeof(word));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&info, spark::g_error_info, sizeof(info));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(spark::g_error_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word & spark::kErrTimeout)
    return fail(SPARK_ERR_TIMEOUT, "a bounded device wait expired (site 0x%x)", info);
  if (word & spark::kErrPosition)
    return fail(SPARK_ERR_DEVICE_ARG, "a position failed its device-side check (site 0x%x)", info);
  return SPARK_OK;
}

// ------------------------------------------------- context parallelism ----
size_t spark_decode_cp_record_bytes(int B) {
  if (B <= 0 || B > 65535) return 0;
  return (size_t)spark::cp_record_floats(B) * sizeof(float);
}

int spark_kv_append_cp(void* k_cache, void* v_cache, int cap, int key_off, const void* k, const void* v, int B,
                       const int* pos, const spark_layer_cfg* cfg, unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if ((rc = check_cp_shard(cap, key_off, cfg))) return rc;
  return append_impl(dense_view(k_cache, v_cache, nullptr, nullptr, cap), k, v, B, 1, pos, cfg, flags, stream,
                     nullptr, key_off, 1);
}

int spark_attn_decode_cp_partial(void* record, const void* q, const void* k_cache, const void* v_cache, int cap,
                                 int key_off, int B, const int* pos, const spark_layer_cfg* cfg, void* workspace,
                                 size_t ws_bytes, unsigned flags, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if ((rc = check_cp_shard(cap, key_off, cfg))) return rc;
  if (!record) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  return decode_impl(nullptr, q, nullptr, dense_view((void*)k_cache, (void*)v_cache, nullptr, nullptr, cap), B, pos,
                     cfg, workspace, ws_bytes, flags, stream, key_off, (float*)record);
}

int spark_attn_decode_cp_merge(void* out, const void* gate, const void* records, int G, int B, void* stream) {
  if (!out || !gate || !records) return fail(SPARK_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || B > 65535 || G <= 0 || G > 1024) return fail(SPARK_ERR_INVALID_ARG, "bad shape G=%d B=%d", G, B);
  if (!aligned16(out) || !aligned16(records)) return fail(SPARK_ERR_INVALID_ARG, "out and records must be 16-byte aligned");
  int rc, dev;
  if ((rc = device_ready(&dev))) return rc;
  spark::decode_cp_merge_kernel<<<dim3(spark::kNq, B), 64, 0, (cudaStream_t)stream>>>(
      (__nv_bfloat16*)out, (const __nv_bfloat16*)gate, (const float*)records, G, B);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPARK_OK : cuda_fail(e, "decode_cp_merge_kernel launch");
}

}  // extern "C"
