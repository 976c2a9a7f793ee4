"""Plain fp64 CPU oracle for the Spark2_5 hybrid GQA attention core.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA library (no kernels, headers, tables or helpers); the only thing both
sides use is the seeded input generator in ``synth/``, which holds none of the
attention arithmetic.

Everything here is written for a reader to check by eye against the pages:
every step is the plain definition, in float64, with no blocking, fusion or
reordering.  Page citations use the page's title and section:

* [FP8]    "Spark-X2.6-4B-FP8 ... W8A8" (nxmr.cn/news/148448)
* [F16-Q4] "量化精度怎么选？星火 X2.5-4B 的 F16 与 Q4 实测对比" (hotelren.com/news/5475707)
* [CONFIG] "Spark-X2.6-4B config.json" walkthrough (lqnn.cn/news/248463)
* [HYBRID] "Spark-X2.6-4B-Base" hybrid attention (eliteato.com/news/34565)
* [GGUF]   "Sharp-Spark-X2.5-4B-GGUF" on a 6 GB card (mpbf.cn/news/67460)

Readings taken where the pages are silent:
RoPE pairs dim i with dim i + rot/2 (the rotate-half convention of a
transformers modeling file); the partial-rotary inverse frequencies use the
rotated width as denominator, f_i = theta^(-2i/rot); the window of 512 counts
the query itself (key j visible to query i iff i-512 < j <= i); the score scale
is 1/sqrt(256); q head h reads KV head h // 4; the gate is one logit per
(token, head).

Every function below is pinned by ``tests/test_oracle_pins.py``; none is
"parity unpinned".
"""
from __future__ import annotations

import numpy as np

SLIDING = 0
FULL = 1

N_LAYERS = 36          # [FP8] §一 config table: num_hidden_layers 36
N_Q_HEADS = 16         # [FP8] §一: num_attention_heads 16
N_KV_HEADS = 4         # [FP8] §一: num_key_value_heads 4 (GQA)
HEAD_DIM = 256         # [FP8] §一: head_dim 256
WINDOW = 512           # [HYBRID] §滑动窗口 512 (config sliding_window: 512)
MAX_POSITION = 1 << 20  # [HYBRID] §全局注意力 5M 基频 RoPE: max_position_embeddings 1048576
GROUP = N_Q_HEADS // N_KV_HEADS


# ---------------------------------------------------------------------------
# Layer schedule and per-kind parameters
# ---------------------------------------------------------------------------

def layer_kind(layer: int) -> int:
    """Kind of 0-based layer ``layer`` in the 36-layer stack.

    [CONFIG] §混合注意力: 36 layers strictly cycle "3 sliding + 1 full";
    [HYBRID] §36 层混合注意力排布: 27 sliding, 9 full, and the last (36th)
    layer is a full-attention layer.  So layer l is full iff l % 4 == 3.
    """
    if not 0 <= layer < N_LAYERS:
        raise ValueError(f"layer {layer} outside [0, {N_LAYERS})")
    return FULL if layer % 4 == 3 else SLIDING


def layer_params(kind: int) -> dict:
    """RoPE base, rotated width and window of a layer kind.

    [CONFIG] §1M 上下文如何做到：RoPE 的"双参数"配置 and [HYBRID] §全局注意力 5M
    基频 RoPE: full layers use rope_theta 5e6 with partial_rotary_factor 0.25
    (only the first 64 of 256 dims rotate); sliding layers use rope_theta 1e4
    and rotate the whole head.  Full layers see the whole causal context;
    sliding layers at most 512 tokens back ([HYBRID] §滑动窗口 512).
    """
    if kind == FULL:
        return {"theta": 5.0e6, "rot": int(HEAD_DIM * 0.25), "window": None}
    if kind == SLIDING:
        return {"theta": 1.0e4, "rot": int(HEAD_DIM * 1.0), "window": WINDOW}
    raise ValueError(f"unknown layer kind {kind}")


# ---------------------------------------------------------------------------
# Rotary position embedding
# ---------------------------------------------------------------------------

def rope_inv_freq(kind: int) -> np.ndarray:
    """Inverse frequencies f_i = theta^(-2i/rot), i < rot/2, in float64.

    [CONFIG] §1M 上下文如何做到 and [HYBRID] §全局注意力 5M 基频 RoPE give theta and
    the rotated width; the exponent convention over the rotated width is the
    reading stated in the module docstring.
    """
    p = layer_params(kind)
    rot = p["rot"]
    i = np.arange(rot // 2, dtype=np.float64)
    return p["theta"] ** (-2.0 * i / rot)


def rope(x: np.ndarray, pos: np.ndarray, kind: int) -> np.ndarray:
    """Rotate ``x`` [T, H, 256] by absolute positions ``pos`` [T].

    For i < rot/2, the pair (x_i, x_{i+rot/2}) turns by angle pos * f_i:
        x'_i        = x_i cos a - x_{i+rot/2} sin a
        x'_{i+rot/2} = x_{i+rot/2} cos a + x_i sin a
    Dims >= rot pass through unchanged (the full layers' partial rotary,
    [HYBRID] §全局注意力 5M 基频 RoPE: "only the first 64 dims rotate").
    """
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.int64)
    if x.ndim != 3 or x.shape[-1] != HEAD_DIM or x.shape[0] != pos.shape[0]:
        raise ValueError("rope expects x [T, H, 256] and pos [T]")
    rot = layer_params(kind)["rot"]
    half = rot // 2
    f = rope_inv_freq(kind)
    a = pos.astype(np.float64)[:, None] * f[None, :]        # [T, half]
    c = np.cos(a)[:, None, :]
    s = np.sin(a)[:, None, :]
    out = x.copy()
    lo = x[:, :, :half]
    hi = x[:, :, half:rot]
    out[:, :, :half] = lo * c - hi * s
    out[:, :, half:rot] = hi * c + lo * s
    return out


# ---------------------------------------------------------------------------
# Masks and attention
# ---------------------------------------------------------------------------

def visible(qpos: np.ndarray, kpos: np.ndarray, kind: int) -> np.ndarray:
    """Boolean [Tq, Tk]: may the query at qpos see the key at kpos?

    Full layers: causal, kp <= qp ([HYBRID] §36 层混合注意力排布: full layers use
    a causal mask).  Sliding layers: qp - 512 < kp <= qp, a window of 512 keys
    that counts the query itself ([HYBRID] §滑动窗口 512).
    """
    qp = np.asarray(qpos, dtype=np.int64)[:, None]
    kp = np.asarray(kpos, dtype=np.int64)[None, :]
    vis = kp <= qp
    if kind == SLIDING:
        vis &= kp > qp - WINDOW
    return vis


def attention_probs(q: np.ndarray, k: np.ndarray, qpos, kpos, kind: int) -> np.ndarray:
    """Softmax weights P [16, Tq, Tk] for already-rotated q [Tq,16,256], k [Tk,4,256].

    Score s_ij = (q_i . k_j) / sqrt(256) for q head h against KV head h // 4
    (GQA: 16 query heads share 4 KV heads, [FP8] §一 and [HYBRID] §配套效率设计);
    invisible keys are dropped; the softmax is the max-subtracted exponential
    normalised over the visible keys ([F16-Q4] §三: softmax in fp32; here fp64).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    vis = visible(qpos, kpos, kind)
    scale = 1.0 / np.sqrt(HEAD_DIM)
    out = np.zeros((N_Q_HEADS, q.shape[0], k.shape[0]), dtype=np.float64)
    for h in range(N_Q_HEADS):
        g = h // GROUP
        s = (q[:, h, :] @ k[:, g, :].T) * scale
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.where(vis, np.exp(s - m), 0.0)
        out[h] = e / e.sum(axis=1, keepdims=True)
    return out


def sigmoid(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def attention(q, k, v, gate, qpos, kpos, kind: int) -> np.ndarray:
    """Gated attention output [Tq, 16, 256] for already-rotated q and k.

    o_i = sum_j P_ij v_j with v from KV head h // 4, then each head's output is
    multiplied by sigmoid(gate[i, h]) (the headwise sigmoid output gate,
    [F16-Q4] §三 and [HYBRID] §配套效率设计).
    """
    v = np.asarray(v, dtype=np.float64)
    p = attention_probs(q, k, qpos, kpos, kind)
    g = sigmoid(gate)                                      # [Tq, 16]
    out = np.zeros((p.shape[1], N_Q_HEADS, HEAD_DIM), dtype=np.float64)
    for h in range(N_Q_HEADS):
        out[:, h, :] = (p[h] @ v[:, h // GROUP, :]) * g[:, h][:, None]
    return out


def attention_group(q, k, v, gate, qpos, kpos, kind: int) -> np.ndarray:
    """The same gated attention for one GQA group only: the 4 query heads that share one KV head.

    q [Tq,4,256] and k [Tk,256] already rotated, v [Tk,256], gate [Tq,4];
    returns [Tq,4,256].  Identical, head by head, to ``attention`` restricted
    to heads 4g..4g+3 with KV head g; it exists so that long contexts need the
    keys of one KV head only.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    vis = visible(qpos, kpos, kind)
    scale = 1.0 / np.sqrt(HEAD_DIM)
    g = sigmoid(gate)
    out = np.zeros((q.shape[0], GROUP, HEAD_DIM), dtype=np.float64)
    for j in range(GROUP):
        s = (q[:, j, :] @ k.T) * scale
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.where(vis, np.exp(s - m), 0.0)
        p = e / e.sum(axis=1, keepdims=True)
        out[:, j, :] = (p @ v) * g[:, j][:, None]
    return out


def layer_prefill(q, k, v, gate, pos, kind: int, hist_k=None, hist_v=None, hist_pos=None):
    """One layer's attention for a chunk of tokens with raw (unrotated) q, k.

    q [T,16,256], k/v [T,4,256], gate [T,16], pos [T] absolute positions.  The
    optional history holds keys already in the cache (rotated k, v, positions).
    """
    pos = np.asarray(pos, dtype=np.int64)
    qr = rope(q, pos, kind)
    kr = rope(k, pos, kind)
    v = np.asarray(v, dtype=np.float64)
    if hist_k is not None and len(hist_pos) > 0:
        kr = np.concatenate([np.asarray(hist_k, dtype=np.float64), kr], axis=0)
        v = np.concatenate([np.asarray(hist_v, dtype=np.float64), v], axis=0)
        kpos = np.concatenate([np.asarray(hist_pos, dtype=np.int64), pos])
    else:
        kpos = pos
    return attention(qr, kr, v, gate, pos, kpos, kind)


def layer_prefill_rows(q_rows, k, v, gate_rows, pos, kind: int, rows, hist_k=None, hist_v=None, hist_pos=None):
    """``layer_prefill`` evaluated at the query rows ``rows`` only.

    q_rows [len(rows),16,256] and gate_rows [len(rows),16] are the raw queries
    and gate logits of those rows; k, v, pos are the whole chunk's.  Each
    selected query is computed exactly as in ``layer_prefill``: it sees the
    same keys and gets the same rotation; the other queries are simply not
    evaluated.  Used where the full oracle would take too long.
    """
    rows = np.asarray(rows, dtype=np.int64)
    pos = np.asarray(pos, dtype=np.int64)
    qr = rope(q_rows, pos[rows], kind)
    kr = rope(k, pos, kind)
    v = np.asarray(v, dtype=np.float64)
    if hist_k is not None and len(hist_pos) > 0:
        kr = np.concatenate([np.asarray(hist_k, dtype=np.float64), kr], axis=0)
        v = np.concatenate([np.asarray(hist_v, dtype=np.float64), v], axis=0)
        kpos = np.concatenate([np.asarray(hist_pos, dtype=np.int64), pos])
    else:
        kpos = pos
    return attention(qr, kr, v, gate_rows, pos[rows], kpos, kind)


def layer_decode(q, k_new, v_new, gate, p: int, kind: int, hist_k, hist_v, hist_pos):
    """Attention of one new token at position p (append-then-attend).

    q [16,256] and k_new [4,256] are raw and rotate at p; hist_k [n,4,256] holds
    already-rotated cached keys at positions hist_pos [n] (all < p).  The new
    key joins the visible set, so the query always sees itself.
    """
    qr = rope(np.asarray(q)[None], np.array([p]), kind)
    kr = rope(np.asarray(k_new)[None], np.array([p]), kind)
    ks = np.concatenate([np.asarray(hist_k, dtype=np.float64).reshape(-1, N_KV_HEADS, HEAD_DIM), kr], axis=0)
    vs = np.concatenate([np.asarray(hist_v, dtype=np.float64).reshape(-1, N_KV_HEADS, HEAD_DIM),
                         np.asarray(v_new, dtype=np.float64)[None]], axis=0)
    kpos = np.concatenate([np.asarray(hist_pos, dtype=np.int64), [p]])
    return attention(qr, ks, vs, np.asarray(gate)[None], np.array([p]), kpos, kind)[0]


# ---------------------------------------------------------------------------
# KV cache layout model and byte accounting
# ---------------------------------------------------------------------------

def cache_slot(pos: int, kind: int) -> int:
    """Cache row of absolute position ``pos``.

    Full layers keep every position (a linear cache that grows with the
    context); sliding layers keep only the last 512 ([F16-Q4] §一 and [CONFIG]
    §混合注意力: sliding-layer KV is capped by the 512 window), here as a ring
    of 512 rows indexed by pos mod 512.
    """
    return pos if kind == FULL else pos % WINDOW


def ring_contents_sequential(n_appended: int) -> np.ndarray:
    """Positions held by the 512 ring rows after appending 0..n-1 one by one (-1 = empty)."""
    ring = np.full(WINDOW, -1, dtype=np.int64)
    for p in range(n_appended):
        ring[cache_slot(p, SLIDING)] = p
    return ring


def kv_bytes_per_token_full_layer(bytes_per_elem: float = 2.0) -> float:
    """K+V x 4 heads x 256 dims x 2 bytes = 4 KB per token per full layer ([F16-Q4] §一)."""
    return 2 * N_KV_HEADS * HEAD_DIM * bytes_per_elem


Q8_0_BYTES_PER_ELEM = 34.0 / 32.0   # 32 int8 values + one fp16 scale per block


def stack_kv_bytes(n_ctx: int, bytes_per_elem: float = 2.0) -> float:
    """KV bytes of the 36-layer stack at context n_ctx.

    9 full layers grow with the context; the 27 sliding layers hold at most 512
    tokens each ([GGUF] §三: only the 9 full layers grow, the 27 window layers
    are a fixed ~57 MB).
    """
    n_full = sum(1 for l in range(N_LAYERS) if layer_kind(l) == FULL)
    n_slide = N_LAYERS - n_full
    per_tok = kv_bytes_per_token_full_layer(bytes_per_elem)
    return n_full * per_tok * n_ctx + n_slide * per_tok * min(n_ctx, WINDOW)


# ---------------------------------------------------------------------------
# 8-bit block-quantised KV cache (q8_0-style): 32-value blocks, one fp16 scale
# ---------------------------------------------------------------------------

Q8_BLOCK = 32


def quantize_q8(x):
    """Quantise rows of 256 values into 8 blocks of 32: codes and fp16 scales.

    [GGUF] §四: the KV cache can be stored as q8_0, 8-bit values in blocks that
    carry one scale each, cutting 36 KB per token to 19 KB.  The pages give the
    format's name and byte count only; the reading taken here: per block,
    amax = max |x|, scale d = fp16(amax / 127), code c = round-half-away-from-
    zero(x * (127 / amax)) in [-127, 127], stored offset by 128 as a byte.  The
    division and the product are float32 (the same operations the device
    performs); the rounding of the float32 product y is exact: it is done in
    float64, where |y| + 1/2 carries no rounding error.  A block
    whose 127 / amax is not a finite float32 (amax below ~3.7e-37, so its fp16
    scale is 0 anyway) gets code 0 throughout, like an all-zero block.
    Returns (u8 codes [..., 256], fp16 scales [..., 8]).
    """
    x = np.asarray(x, dtype=np.float32)
    blocks = x.reshape(x.shape[:-1] + (x.shape[-1] // Q8_BLOCK, Q8_BLOCK))
    amax = np.max(np.abs(blocks), axis=-1, keepdims=True).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        inv = (np.float32(127.0) / amax).astype(np.float32)
        inv = np.where((amax > 0) & np.isfinite(inv), inv, np.float32(0.0)).astype(np.float32)
    y = (blocks * inv).astype(np.float32).astype(np.float64)
    c = np.sign(y) * np.floor(np.abs(y) + 0.5)
    codes = (c + 128).astype(np.uint8).reshape(x.shape)
    scales = (amax[..., 0] / np.float32(127.0)).astype(np.float32).astype(np.float16)
    return codes, scales


def dequantize_q8(codes, scales):
    """Values of a quantised row: scale * code, in float64."""
    c = np.asarray(codes, dtype=np.float64) - 128.0
    d = np.asarray(scales, dtype=np.float64)
    blocks = c.reshape(c.shape[:-1] + (c.shape[-1] // Q8_BLOCK, Q8_BLOCK))
    return (blocks * d[..., None]).reshape(c.shape)


def q8_bytes_per_value() -> float:
    """34 bytes per 32 values: 32 codes and a 2-byte scale."""
    return (Q8_BLOCK + 2) / Q8_BLOCK
