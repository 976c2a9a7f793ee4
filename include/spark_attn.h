/*
 * spark_attn.h -- C ABI of libspark_attn.so, the attention core of the
 * Spark2_5 layer (Spark-X2.5 / X2.6 4B) on NVIDIA B200 (sm_100a).
 *
 * What it computes.  Causal grouped-query attention with 16 query heads that
 * share 4 KV heads (q head h reads KV head h / 4) at head_dim 256 and score
 * scale 1/sqrt(256), an fp32 softmax, and a per-head sigmoid output gate, over
 * a 36-layer stack that repeats three sliding-window layers and one full layer:
 *   - sliding layers: key j visible to query i iff i - 512 < j <= i; RoPE with
 *     theta 1e4 over all 256 dims;
 *   - full layers: key j visible iff j <= i; RoPE with theta 5e6 over the
 *     first 64 dims only (partial rotary factor 0.25).
 * Sources: "Spark-X2.6-4B-FP8 W8A8" page §一 (16/4 heads, head_dim 256,
 * 36 layers); "Spark-X2.6-4B config.json" page §混合注意力 and §1M 上下文如何做到
 * (3 sliding + 1 full, the two RoPE parameter sets); "Spark-X2.6-4B-Base"
 * hybrid attention page §36 层混合注意力排布, §滑动窗口 512, §全局注意力 5M 基频
 * RoPE, §配套效率设计 (masks, partial rotary, GQA, headwise gate);
 * "星火 X2.5-4B F16 与 Q4 实测对比" page §一 (KV cache per token) and §三 (fp32
 * softmax, sigmoid gate per head).
 *
 * RoPE convention (the pages give none): for i < rot/2 the pair
 * (x_i, x_{i+rot/2}) turns by angle pos * theta^(-2i/rot).
 *
 * Conventions shared by every call:
 *   - All tensors are bf16 (the q8 cache: uint8 codes and fp16 scales), in
 *     device memory, allocated and owned by the caller.  The library
 *     allocates and frees nothing.  Tensors are contiguous except the token
 *     tensors q, k, v of the calls that take element strides (sB, sT):
 *     there, token t of sequence b starts at element b * sB + t * sT and its
 *     heads are contiguous rows of 256, so q, k and v may be views of one
 *     fused projection output [B][T][16 + 4 + 4][256] ("Spark-X2.6-4B-FP8
 *     W8A8" page §三: one q_k_v_proj before attention).  Strides 0, 0 select
 *     the dense layout; otherwise both are multiples of 8 elements, a token's
 *     heads fit in sT, sequences do not overlap, and both are below 2^36.
 *   - Positions are absolute (0 <= pos < 2^20).  Per-sequence positions live
 *     in caller-owned device int32 arrays, so a captured CUDA graph can replay
 *     with new positions.  The T tokens a call takes for sequence b sit at
 *     consecutive positions pos0[b] .. pos0[b] + T - 1: a prompt chunk
 *     processed after a history of pos0[b] tokens, as the pages measure
 *     prefill ("Sharp-Spark-X2.5-4B-GGUF" page §三, prompt processing at a
 *     context depth).
 *   - Every call is asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *     default stream) and runs on the current device, which must be sm_100.
 *   - Host-side argument checks run before any launch; on failure nothing is
 *     launched.  Positions are device data, so they are checked on the device:
 *     a bad position makes the kernel skip that sequence and set the library's
 *     device error word, which spark_check() reports.
 *   - Layouts (element strides, innermost first):
 *       q, out   [B][T][16][256]      k, v (new tokens)  [B][T][4][256]
 *       gate     [B][T][16] (logits; the kernel applies the sigmoid)
 *       k_cache, v_cache [B][4][cap][256]
 *     Full layers use a linear cache: row = position, cap >= context.
 *     Sliding layers use a ring of cap = 512 rows: row = position mod 512.
 *   - Return value: SPARK_OK or a negative spark status.
 */
#ifndef SPARK_ATTN_H
#define SPARK_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPARK_OK                0
#define SPARK_ERR_INVALID_ARG  (-1)  /* null pointer, bad size, bad cfg */
#define SPARK_ERR_UNSUPPORTED  (-2)  /* not an sm_100 device, or dims other than 16/4/256 */
#define SPARK_ERR_CUDA         (-3)  /* a CUDA runtime call failed; see spark_last_error() */
#define SPARK_ERR_TIMEOUT      (-4)  /* a bounded device-side wait expired (reported by spark_check) */
#define SPARK_ERR_DEVICE_ARG   (-5)  /* a position checked on the device was out of range (spark_check) */

#define SPARK_N_LAYERS     36
#define SPARK_N_Q_HEADS    16
#define SPARK_N_KV_HEADS   4
#define SPARK_HEAD_DIM     256
#define SPARK_WINDOW       512
#define SPARK_MAX_POSITION (1 << 20)

typedef enum { SPARK_SLIDING = 0, SPARK_FULL = 1 } spark_kind;

/* Per-layer attention parameters.  Only the values the pages fix are
 * accepted: n_q 16, n_kv 4, head_dim 256, scale 1/16, and per kind
 * (window 512, rot_dim 256, theta 1e4) or (window 0, rot_dim 64, theta 5e6). */
typedef struct {
  int kind;       /* spark_kind */
  int window;     /* 512 for sliding layers, 0 (unbounded) for full layers */
  int rot_dim;    /* rotated leading dims: 256 sliding, 64 full */
  int n_q;        /* 16 */
  int n_kv;       /* 4 */
  int head_dim;   /* 256 */
  double theta;   /* RoPE base: 1e4 sliding, 5e6 full */
  float scale;    /* 1/sqrt(head_dim) = 0.0625 */
} spark_layer_cfg;

/* Flags */
#define SPARK_ROPE_FUSED 1u  /* the call rotates its raw q (prefill, decode) or k (kv_append) itself */
#define SPARK_APPEND_FUSED 2u  /* spark_attn_prefill also appends the chunk's k and v to the cache */

/* Parameters of 0-based layer `layer` of the 36-layer stack: layer l is full
 * iff l % 4 == 3 ("3 sliding + 1 full", the last layer full).
 * Errors: SPARK_ERR_INVALID_ARG for layer outside [0, 36) or out == NULL. */
int spark_layer_cfg_for_layer(int layer, spark_layer_cfg* out);

/* Parameters of a layer kind (SPARK_SLIDING or SPARK_FULL). */
int spark_layer_cfg_for_kind(int kind, spark_layer_cfg* out);

/* Bytes of one layer's K+V cache for B sequences of capacity cap rows:
 * 2 * B * 4 * cap * 256 * 2.  Per token and full layer this is the 4 KB the
 * "星火 X2.5-4B F16 与 Q4" page §一 derives.  Returns -1 on bad arguments. */
long long spark_kv_cache_bytes(const spark_layer_cfg* cfg, int B, long long cap);

/* Bytes of the whole 36-layer stack's caches at context ctx: 9 linear caches
 * of ctx rows plus 27 rings of min(ctx, 512) rows ("Sharp-Spark-X2.5-4B-GGUF"
 * page §三: only the 9 full layers grow).  Returns -1 on bad arguments. */
long long spark_stack_kv_bytes(int B, long long ctx);

/* Rotate x [B][T][H][256] (element strides sB, sT) in place; token t of
 * sequence b is at position pos0[b] + t (pos0: device int32 [B]).  H is 16
 * (queries) or 4 (keys).  Dims >= cfg->rot_dim are not touched. */
int spark_rope_apply(void* x, int B, int T, int H, long long sB, long long sT, const int* pos0,
                     const spark_layer_cfg* cfg, void* stream);

/* Append T new tokens per sequence to a layer's K/V cache.  k, v
 * [B][T][4][256], both with element strides sB, sT; token t of sequence b is
 * at position pos0[b] + t.
 * Full layer: row = position, requires pos0[b] + T <= cap.
 * Sliding layer: cap must be 512; row = position mod 512; only the last
 * min(T, 512) tokens are written (older ones would be overwritten anyway).
 * With SPARK_ROPE_FUSED, k is raw and is rotated on its way into the cache
 * (the k buffer itself is not modified); v is copied bit for bit. */
int spark_kv_append(void* k_cache, void* v_cache, int cap, const void* k, const void* v, int B,
                    int T, long long sB, long long sT, const int* pos0, const spark_layer_cfg* cfg,
                    unsigned flags, void* stream);

/* Attention of a chunk of T queries per sequence (prefill).
 *   q [B][T][16][256] (rotated, or raw with SPARK_ROPE_FUSED: the kernel then
 *   rotates each Q tile in shared memory after loading it; q itself is not
 *   modified; element strides q_sB, q_sT), k [B][T][4][256] rotated and
 *   v [B][T][4][256] (element strides kv_sB, kv_sT), gate [B][T][16];
 *   out [B][T][16][256] (dense).
 *   Token t of sequence b is at position pos0[b] + t (pos0: device int32 [B]).
 *   The chunk's own keys come from k/v.  Earlier keys (the history,
 *   positions < pos0[b]) come from the cache: full layers read rows
 *   [0, pos0[b]); sliding layers read the ring rows of positions
 *   [max(0, pos0[b] - 511), pos0[b]).  Pass k_cache = v_cache = NULL when no
 *   sequence has history.  Without SPARK_APPEND_FUSED the cache is only read:
 *   append the chunk after this call on sliding layers (the ring rows are
 *   still needed here), before or after it on full layers.
 * With SPARK_APPEND_FUSED (caches required) the call also appends the chunk's k
 * (as passed: rotated) and v to the cache, as spark_kv_append would, after the
 * attention on the same stream, so a sliding ring is overwritten only once it
 * has been read as history.  Without caches (no history) the call runs the
 * persistent kernel, which is faster on sliding layers; a first chunk is
 * therefore best attended without caches and appended by spark_kv_append.
 * Device requirements: sm_100a, about 225 KB of shared memory per block. */
int spark_attn_prefill(void* out, const void* q, const void* k, const void* v, const void* gate,
                       const void* k_cache, const void* v_cache, int cap, int B, int T, long long q_sB,
                       long long q_sT, long long kv_sB, long long kv_sT, const int* pos0,
                       const spark_layer_cfg* cfg, unsigned flags, void* stream);

/* Workspace bytes spark_attn_decode needs for B sequences and cache capacity
 * cap (split-KV partials: per sequence, query head and split, 256 + 2 fp32).
 * Returns 0 on bad arguments. */
size_t spark_decode_workspace_bytes(int B, int cap, const spark_layer_cfg* cfg);

/* Attention of one new token per sequence (decode, append-then-attend).
 *   q [B][16][256] (rotated, or raw with SPARK_ROPE_FUSED; sequence b at
 *   element b * q_sB, 0: dense), gate [B][16]; out [B][16][256].  The new
 *   token of sequence b is at position pos[b]
 *   (device int32 [B]) and its k/v must already be in the cache.
 *   Full layer: attends to cache rows 0..pos[b] (pos[b] < cap).
 *   Sliding layer (cap 512): attends to ring rows 0..min(pos[b], 511), which
 *   then hold exactly positions max(0, pos[b] - 511)..pos[b].
 *   workspace: caller-owned device scratch of at least
 *   spark_decode_workspace_bytes(B, cap, cfg) bytes, 16-byte aligned; calls
 *   that share a workspace must not overlap on the device.  When the split
 *   plan has one split per (sequence, KV head), as for sliding layers at
 *   B >= 37, one kernel writes `out` directly and the workspace is unused. */
int spark_attn_decode(void* out, const void* q, long long q_sB, const void* gate, const void* k_cache,
                      const void* v_cache, int cap, int B, const int* pos,
                      const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes,
                      unsigned flags, void* stream);

/* One decode layer in one launch: the append of the new token and the
 * attention of spark_attn_decode, fused (the two calls spark_kv_append +
 * spark_attn_decode give the same result up to fp32 rounding order).
 *   q [B][16][256] and k, v [B][4][256] (sequence b at elements b * q_sB and
 *   b * kv_sB, 0: dense): the new token of each sequence at
 *   position pos[b] (raw with SPARK_ROPE_FUSED: q and k are rotated at
 *   pos[b] here; k is written into the cache rotated and rounded to bf16,
 *   exactly as spark_kv_append writes it; v bit for bit).  gate [B][16];
 *   out [B][16][256].  k_cache, v_cache [B][4][cap][256] as for
 *   spark_kv_append / spark_attn_decode: the call writes row pos[b] (full,
 *   pos[b] < cap) or pos[b] mod 512 (sliding, cap 512) and attends to
 *   positions 0..pos[b] (full) or max(0, pos[b] - 511)..pos[b] (sliding), the
 *   new token's key and value taken from k and v.  Cache rows past the last
 *   cached position may hold anything.
 *   workspace: caller-owned device memory of at least
 *   spark_decode_fused_workspace_bytes(B, cap, cfg) bytes, 16-byte aligned,
 *   which must hold zeros before its first use (cudaMemsetAsync once after
 *   allocating it).  Its last B * 4 ints count, per (sequence, KV head), the
 *   blocks that have finished their share; every call that completes leaves
 *   them at zero again, so one workspace serves any number of calls and
 *   layers in turn.  After a call that spark_check() reported as failed
 *   (a wait that ran out), zero it again.  Calls that share a workspace must
 *   not overlap on the device.
 * The kernel is launched with programmatic stream serialisation: its blocks
 * may be scheduled while the previous kernel of the stream is still running,
 * but they read and write memory only after that kernel has completed. */
size_t spark_decode_fused_workspace_bytes(int B, int cap, const spark_layer_cfg* cfg);

int spark_attn_decode_fused(void* out, const void* q, long long q_sB, const void* k, const void* v,
                            long long kv_sB, const void* gate, void* k_cache, void* v_cache, int cap, int B,
                            const int* pos, const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes,
                            unsigned flags, void* stream);

/* Size of the fixed scratch array spark_attn_decode_static uses. */
#define SPARK_STATIC_SCRATCH_BYTES (16u << 20)

/* Decode for callers that cannot allocate device memory (no counterpart on the
 * pages; it exists for such callers).  Some hosts plan all device memory up
 * front and forbid allocation later, some only lend the library their inputs
 * and outputs, and code recording a CUDA graph cannot record cudaMalloc.  This
 * call computes exactly what spark_attn_decode computes, with the same
 * arguments minus q's stride (q is dense) and the workspace: the split-KV
 * partials go to a fixed
 * SPARK_STATIC_SCRATCH_BYTES array in the library's own device memory, which
 * every GPU that loads the library holds until the process exits.  It calls no
 * allocating routine.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, once per device, with that device current); make
 *     that first call before any stream capture.  A first call made while
 *     `stream` is being captured is refused with SPARK_ERR_INVALID_ARG and
 *     nothing is launched; a failed lookup is not remembered, the next call
 *     tries again.
 *   - One split needs B * 16 * 258 * 4 bytes, so B may be at most 1016; larger
 *     batches are rejected with SPARK_ERR_INVALID_ARG.  When the usual split
 *     plan does not fit, fewer splits are used.
 *   - All calls share the array and it keeps the last call's contents; nothing
 *     in it needs to start at zero, because every partial a call reads is
 *     written by the same call.  Calls that overlap on the device (other
 *     streams, or other host threads) race on it: serialise them. */
int spark_attn_decode_static(void* out, const void* q, const void* gate, const void* k_cache,
                             const void* v_cache, int cap, int B, const int* pos,
                             const spark_layer_cfg* cfg, unsigned flags, void* stream);

/* Split plan spark_attn_decode_static uses on a device of sm_count SMs (host
 * only, no device access): *n_splits key splits of *tiles_per_split 64-key
 * tiles per (sequence, KV head).  Returns the bytes of the array the partials
 * occupy (<= SPARK_STATIC_SCRATCH_BYTES), 0 on bad arguments or when B is above
 * the limit.  n_splits, tiles_per_split may be NULL. */
size_t spark_decode_static_plan(int B, int cap, const spark_layer_cfg* cfg, int sm_count, int* n_splits,
                                int* tiles_per_split);

/* ---- 8-bit block-quantised KV cache ("Sharp-Spark-X2.5-4B-GGUF" page §四:
 * the K/V cache stored as q8_0, 36 -> 19 KB per token).  The block format is
 * GGML's q8_0, which the page names but does not spell out: 32 consecutive
 * values of a row share one fp16 scale, each value is an 8-bit code.
 *   k_codes, v_codes    uint8 [B][4][cap][256]  byte = c + 128, c in [-127, 127]
 *   k_scales, v_scales  fp16  [B][4][cap][8]    value ~ c * scale of its block
 * Rows are placed as in the bf16 cache (ring of 512 for sliding layers).
 * Quantising a block (float32): amax = max |x|; scale = fp16(amax / 127);
 * c = x * (127 / amax) rounded half away from zero (IEEE single division and
 * product); an all-zero block, or one where 127 / amax overflows, gives c = 0,
 * scale 0.  Values are representable up to |x| = 127 * 65504 (fp16 scale).  Buffers are caller-owned
 * device memory: codes 16-byte aligned, scales 16-byte aligned. */

/* Bytes of one layer's q8 K and V caches (codes and scales), -1 on bad input. */
long long spark_kv_cache_q8_bytes(const spark_layer_cfg* cfg, int B, long long cap);

/* Quantise and append T new tokens per sequence (same positions, ring and
 * checks as spark_kv_append; k/v [B][T][4][256] bf16, not modified).  With
 * SPARK_ROPE_FUSED, k is rotated (and rounded to bf16) before quantisation. */
int spark_kv_append_q8(void* k_codes, void* k_scales, void* v_codes, void* v_scales, int cap,
                       const void* k, const void* v, int B, int T, const int* pos0,
                       const spark_layer_cfg* cfg, unsigned flags, void* stream);

/* Workspace bytes spark_attn_decode_q8 needs (0 on bad arguments). */
size_t spark_decode_q8_workspace_bytes(int B, int cap, const spark_layer_cfg* cfg);

/* spark_attn_decode over a q8 cache: same arguments, positions, visibility
 * and output as spark_attn_decode, with each cache given as codes + scales.
 * The products use q and the probabilities in fp16 (q keeps its bf16 value
 * exactly; a row with |q|/16 >= 2^15 is first scaled by a power of two) and
 * accumulate in fp32.  Rows past the last visible key are never used, so
 * they may hold anything. */
int spark_attn_decode_q8(void* out, const void* q, const void* gate, const void* k_codes,
                         const void* k_scales, const void* v_codes, const void* v_scales, int cap,
                         int B, const int* pos, const spark_layer_cfg* cfg, void* workspace,
                         size_t ws_bytes, unsigned flags, void* stream);

/* Workspace bytes spark_attn_prefill_q8 needs: the history as bf16, K and V
 * [B][4][cap][256] each (cap = 512 on sliding layers).  0 on bad arguments. */
size_t spark_prefill_q8_workspace_bytes(int B, int cap, const spark_layer_cfg* cfg);

/* spark_attn_prefill over a q8 cache history ("Sharp-Spark-X2.5-4B-GGUF" page
 * §四 runs the model with the K/V cache as q8_0, and §三 measures prefill at
 * 131072 tokens of context over it).  Same arguments, positions, visibility,
 * rotation and output as spark_attn_prefill, with the history's caches given
 * as codes + scales (the q8_0 layout above, cap rows) and a workspace.  The
 * history keys and values are code * scale rounded to bf16; the chunk's own
 * keys and values are the bf16 k/v passed in, as in spark_attn_prefill.
 * The call first writes the history rows each sequence reads (full layers:
 * rows [0, pos0[b]); sliding layers: the 512-row ring) into the workspace as
 * bf16, then runs the bf16 prefill over it, both on `stream`.
 *   workspace: caller-owned device memory of at least
 *   spark_prefill_q8_workspace_bytes(B, cap, cfg) bytes, 16-byte aligned,
 *   scratch only (its contents are undefined after the call, also after an
 *   argument error); calls sharing it must not overlap on the device.
 * With SPARK_APPEND_FUSED the chunk's k (as passed: rotated) and v are then
 * quantised into the 8-bit cache, as spark_kv_append_q8 would. */
int spark_attn_prefill_q8(void* out, const void* q, const void* k, const void* v, const void* gate,
                          const void* k_codes, const void* k_scales, const void* v_codes, const void* v_scales,
                          int cap, int B, int T, long long q_sB, long long q_sT, long long kv_sB, long long kv_sT,
                          const int* pos0, const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes,
                          unsigned flags, void* stream);

/* ---- Paged KV caches (the serving form; "Spark-X2.6-4B-Base" hybrid-attention
 * page §配套效率设计 serves the model through vLLM with prefix caching, whose
 * KV lives in fixed-size pages).  One layer's K and V live in pools of pages;
 * each sequence maps its logical pages to pool pages through a block table,
 * so sequences may share the pages of a common prefix.
 *   k, v           pools [n_pages][4][page_size][256]: bf16, or uint8 codes
 *                  when k_scales/v_scales are set (the q8_0 format above)
 *   k_scales, ...  NULL for bf16 pools, else fp16 [n_pages][4][page_size][8]
 *   block_table    device int32 [B][max_pages]; logical row r of sequence b
 *                  is row r % page_size of pool page block_table[b][r / page_size]
 *   page_size      64, 128, 256 or 512
 * Logical rows: full layers, row = position (positions < max_pages *
 * page_size); sliding layers, row = position mod 512 (a ring over the first
 * 512 / page_size table entries).  A page index outside [0, n_pages) that a
 * call needs is a device-side argument error (spark_check: SPARK_ERR_DEVICE_ARG)
 * and the affected sequence is not written.  Pages shared by several
 * sequences are only read by decode; appending into a shared page is the
 * caller's decision (copy it first to keep the other sequences' rows). */
typedef struct {
  void* k;
  void* v;
  void* k_scales;
  void* v_scales;
  const int* block_table;
  int page_size;
  int n_pages;
  int max_pages;
} spark_paged_kv;

/* spark_kv_append / spark_kv_append_q8 into a paged pool (same arguments,
 * positions, rotation and checks otherwise). */
int spark_kv_append_paged(const spark_paged_kv* kv, const void* k, const void* v, int B, int T,
                          const int* pos0, const spark_layer_cfg* cfg, unsigned flags, void* stream);

/* Workspace bytes spark_attn_decode_paged needs (0 on bad arguments). */
size_t spark_decode_paged_workspace_bytes(int B, const spark_paged_kv* kv, const spark_layer_cfg* cfg);

/* spark_attn_decode / spark_attn_decode_q8 over a paged pool: same
 * arguments, positions, visibility and output. */
int spark_attn_decode_paged(void* out, const void* q, const void* gate, const spark_paged_kv* kv, int B,
                            const int* pos, const spark_layer_cfg* cfg, void* workspace, size_t ws_bytes,
                            unsigned flags, void* stream);

/* ---- Ragged batches (packed sequences of different lengths), the serving
 * form of prefill.  Sequence b's new tokens are rows cu_seqlens[b] ..
 * cu_seqlens[b+1]-1 (device int32 [B+1], non-decreasing, cu_seqlens[0] = 0)
 * of packed tensors with `total` rows: q, out [total][16][256], k, v
 * [total][4][256], gate [total][16]; its first new token is at position
 * pos0[b].  max_seqlen (host) bounds every cu_seqlens[b+1] - cu_seqlens[b];
 * a longer sequence is a device-side argument error. */

/* spark_rope_apply on packed rows: x [total][H][256], H = 16 or 4. */
int spark_rope_apply_varlen(void* x, int H, const int* cu_seqlens, int max_seqlen, const int* pos0, int B,
                            const spark_layer_cfg* cfg, void* stream);

/* spark_kv_append_paged for packed k, v [total][4][256] (sliding layers write
 * each sequence's last 512 tokens). */
int spark_kv_append_varlen(const spark_paged_kv* kv, const void* k, const void* v, const int* cu_seqlens,
                           int max_seqlen, const int* pos0, int B, const spark_layer_cfg* cfg, unsigned flags,
                           void* stream);

/* spark_attn_prefill for a ragged batch: each sequence's chunk attends to
 * itself and to its history in the paged pool `history` (NULL: no history),
 * which must hold positions [0, pos0[b]) for full layers and the ring of the
 * last 512 for sliding layers (bf16 pools only; an 8-bit pool is
 * SPARK_ERR_UNSUPPORTED here: a dense 8-bit history goes through
 * spark_attn_prefill_q8).  History tiles stay page-aligned, so the rows
 * of a sequence's last history page past pos0[b] must hold finite values (a
 * zero-initialised pool, or rows an earlier append wrote). */
int spark_attn_prefill_varlen(void* out, const void* q, const void* k, const void* v, const void* gate,
                              const int* cu_seqlens, int total, int max_seqlen, const int* pos0,
                              const spark_paged_kv* history, int B, const spark_layer_cfg* cfg, unsigned flags,
                              void* stream);

/* Context-parallel decode of a full layer (no counterpart on the pages, which
 * give the 1M-position context, "Spark-X2.6-4B-FP8 W8A8" page §一, and note
 * that decode is bound by reading the KV cache, "星火 X2.5-4B F16 与 Q4 实测对比"
 * page §三; splitting one sequence's cache across GPUs is this library's way to
 * read it with several GPUs' bandwidth).  The cache of a full layer is sharded
 * by position: a rank's k_cache / v_cache [B][4][cap][256] holds positions
 * key_off .. key_off + cap - 1 (row = position - key_off).  Sliding layers are
 * not sharded (SPARK_ERR_UNSUPPORTED): each rank keeps the whole 512-row ring
 * and runs spark_attn_decode.  One decode step of a full layer on G ranks:
 *   1. spark_kv_append_cp on every rank (only the rank holding pos[b] writes
 *      token b; the others skip it);
 *   2. spark_attn_decode_cp_partial on every rank: its record;
 *   3. all-gather of the records (rank order, back to back);
 *   4. spark_attn_decode_cp_merge on every rank (or on the one that needs out).
 * The result equals spark_attn_decode over the whole cache up to rounding. */

/* Bytes of one rank's record for B sequences: fp32 o [B][16][256] (the rank's
 * attention output over its keys, normalised) followed by fp32 lse [B][16] (the
 * log-sum-exp of those keys' logits in base 2, of q.k / 16 * log2(e); -inf when
 * the rank holds none of a sequence's visible keys).  0 on bad B. */
size_t spark_decode_cp_record_bytes(int B);

/* spark_kv_append of one token per sequence (k, v [B][4][256], position
 * pos[b]) into a rank's shard: written at row pos[b] - key_off when that row is
 * in [0, cap), skipped otherwise.  With SPARK_ROPE_FUSED k is rotated at
 * pos[b].  0 <= key_off, key_off + cap <= 2^20. */
int spark_kv_append_cp(void* k_cache, void* v_cache, int cap, int key_off, const void* k, const void* v,
                       int B, const int* pos, const spark_layer_cfg* cfg, unsigned flags, void* stream);

/* A rank's part of spark_attn_decode: q [B][16][256] (raw with
 * SPARK_ROPE_FUSED, rotated at pos[b]) against the shard's rows for positions
 * key_off .. min(pos[b], key_off + cap - 1) (none when pos[b] < key_off);
 * writes the record (spark_decode_cp_record_bytes(B) bytes, 16-byte aligned).
 * workspace: at least spark_decode_workspace_bytes(B, cap, cfg) bytes. */
int spark_attn_decode_cp_partial(void* record, const void* q, const void* k_cache, const void* v_cache,
                                 int cap, int key_off, int B, const int* pos, const spark_layer_cfg* cfg,
                                 void* workspace, size_t ws_bytes, unsigned flags, void* stream);

/* Merge the records of G ranks (records: G records back to back, 16-byte
 * aligned) into out [B][16][256] bf16: the log-sum-exp weighted mean of the
 * ranks' outputs, times sigmoid(gate [B][16]). */
int spark_attn_decode_cp_merge(void* out, const void* gate, const void* records, int G, int B, void* stream);

/* Self-test of the failure-detection path: launches one block that waits,
 * with the same bounded wait every kernel of the library uses, on a barrier
 * phase that nothing completes.  The wait runs out after timeout_ns
 * (0 < timeout_ns <= 10 s), the block returns, and the next spark_check()
 * reports SPARK_ERR_TIMEOUT.  The GPU context stays usable. */
int spark_selftest_wait_timeout(unsigned long long timeout_ns, void* stream);

/* Synchronise `stream`, then read and clear the library's device error word
 * on the current device.  Returns SPARK_OK, SPARK_ERR_TIMEOUT,
 * SPARK_ERR_DEVICE_ARG or SPARK_ERR_CUDA. */
int spark_check(void* stream);

/* Text of the last error of the calling thread ("" if none). */
const char* spark_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int spark_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARK_ATTN_H */
