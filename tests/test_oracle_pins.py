"""Pins of the fp64 oracle to facts fixed outside itself.

Each test checks the oracle against something other than its own formula: the
numbers the pages print (tests/golden/), closed forms and invariants of the
mathematics, brute-force loops on tiny inputs, and a library routine
(torch's scaled_dot_product_attention in float64) for the special case that
reduces to it.  A plausible slip in the oracle (a dropped term, a wrong sign,
index or head mapping, a transposed operand, an off-by-one window) fails at
least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import spark_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.rstrip("\n").split("\t")
            rows[parts[0]] = parts[1:]
    return rows


def _rand(*shape):
    return RNG.standard_normal(shape)


# ---------------------------------------------------------------- schedule ---

def test_layer_schedule_matches_pages():
    g = _golden("pages_numbers.txt")
    kinds = [O.layer_kind(l) for l in range(O.N_LAYERS)]
    assert O.N_LAYERS == int(g["n_layers"][0])
    assert kinds.count(O.SLIDING) == int(g["n_sliding"][0])
    assert kinds.count(O.FULL) == int(g["n_full"][0])
    assert (kinds[-1] == O.FULL) == bool(int(g["last_layer_full"][0]))
    # "3 sliding + 1 full", nine times
    assert kinds == [O.SLIDING, O.SLIDING, O.SLIDING, O.FULL] * 9
    with pytest.raises(ValueError):
        O.layer_kind(36)


def test_layer_params_match_pages():
    g = _golden("pages_numbers.txt")
    s, f = O.layer_params(O.SLIDING), O.layer_params(O.FULL)
    assert s["theta"] == float(g["theta_sliding"][0])
    assert f["theta"] == float(g["theta_full"][0])
    assert f["rot"] == int(g["rotated_dims_full"][0]) == O.HEAD_DIM * float(g["partial_rotary_full"][0])
    assert s["rot"] == O.HEAD_DIM * float(g["partial_rotary_sliding"][0])
    assert s["window"] == int(g["window"][0])
    assert O.N_Q_HEADS == int(g["n_q_heads"][0]) and O.N_KV_HEADS == int(g["n_kv_heads"][0])
    assert O.HEAD_DIM == int(g["head_dim"][0])
    assert O.MAX_POSITION == int(g["max_position"][0])


# -------------------------------------------------------------------- RoPE ---

@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_rope_position_zero_is_identity(kind):
    x = _rand(3, 5, 256)
    np.testing.assert_array_equal(O.rope(x, np.zeros(3, dtype=np.int64), kind), x)


def test_rope_full_leaves_dims_64_to_255_unchanged_and_sliding_moves_all():
    x = _rand(4, 3, 256)
    pos = np.array([1, 77, 4096, (1 << 20) - 1])
    yf = O.rope(x, pos, O.FULL)
    np.testing.assert_array_equal(yf[:, :, 64:], x[:, :, 64:])       # bit-unchanged
    assert np.all(np.abs(yf[1:, :, :64] - x[1:, :, :64]) > 0)
    ys = O.rope(x, pos, O.SLIDING)
    assert np.all(np.abs(ys[1:] - x[1:]) > 0)                         # every dim moves


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_rope_preserves_pair_norms(kind):
    rot = O.layer_params(kind)["rot"]
    h = rot // 2
    x = _rand(6, 4, 256)
    pos = np.array([0, 1, 511, 512, 99999, (1 << 20) - 1])
    y = O.rope(x, pos, kind)
    np.testing.assert_allclose(y[..., :h] ** 2 + y[..., h:rot] ** 2, x[..., :h] ** 2 + x[..., h:rot] ** 2,
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_rope_equals_complex_rotation(kind):
    """The pair (x_i, x_{i+rot/2}) as z = x_i + j x_{i+rot/2} is multiplied by exp(j p f_i)."""
    p = O.layer_params(kind)
    rot, theta = p["rot"], p["theta"]
    h = rot // 2
    x = _rand(5, 2, 256)
    pos = np.array([3, 100, 513, 65536, 1000003])
    y = O.rope(x, pos, kind)
    # frequencies from the geometric progression: f_0 = 1, f_{i+1} = f_i * theta^(-2/rot)
    f = np.cumprod(np.concatenate([[1.0], np.full(h - 1, theta ** (-2.0 / rot))]))
    z = (x[..., :h] + 1j * x[..., h:rot]) * np.exp(1j * np.outer(pos, f))[:, None, :]
    np.testing.assert_allclose(y[..., :h], z.real, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(y[..., h:rot], z.imag, rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_rope_composes_additively(kind):
    x = _rand(4, 2, 256)
    p1 = np.array([5, 1000, 77777, 300000])
    p2 = np.array([9, 24, 1, 700000])
    np.testing.assert_allclose(O.rope(O.rope(x, p1, kind), p2, kind), O.rope(x, p1 + p2, kind),
                               rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_rope_dot_depends_only_on_relative_position(kind):
    q = _rand(1, 1, 256)
    k = _rand(1, 1, 256)
    for (p, pp, s) in [(10, 3, 1000), (600, 0, 12345), (5, 5, 1 << 19)]:
        a = np.sum(O.rope(q, np.array([p + s]), kind) * O.rope(k, np.array([pp + s]), kind))
        b = np.sum(O.rope(q, np.array([p]), kind) * O.rope(k, np.array([pp]), kind))
        assert abs(a - b) < 1e-9 * (1 + abs(b))


def test_full_layer_frequencies_resolve_a_million_positions():
    """5e6 base over 64 rotated dims: the slowest pair's wavelength exceeds the 1M context."""
    f = O.rope_inv_freq(O.FULL)
    assert f[0] == 1.0 and f.shape == (32,)
    assert 2 * math.pi / f[-1] > O.MAX_POSITION
    fs = O.rope_inv_freq(O.SLIDING)
    assert fs.shape == (128,) and 2 * math.pi / fs[-1] > O.WINDOW


# --------------------------------------------------------------- attention ---

def _sdpa_reference(q, k, v, gate, qpos, kpos, kind):
    """torch float64 scaled_dot_product_attention with KV heads repeated 4x and an explicit mask."""
    qt = torch.tensor(q).permute(1, 0, 2)                     # [16, Tq, 256]
    kt = torch.tensor(k).permute(1, 0, 2).repeat_interleave(4, dim=0)
    vt = torch.tensor(v).permute(1, 0, 2).repeat_interleave(4, dim=0)
    qp = torch.tensor(qpos)[:, None]
    kp = torch.tensor(kpos)[None, :]
    mask = kp <= qp
    if kind == O.SLIDING:
        mask = mask & (kp > qp - 512)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)   # scale 1/sqrt(256)
    o = o.permute(1, 0, 2) * torch.sigmoid(torch.tensor(gate))[:, :, None]
    return o.numpy()


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("T,hist", [(7, 0), (64, 0), (600, 0), (100, 530)])
def test_attention_matches_torch_sdpa(kind, T, hist):
    n = T + hist
    kpos = np.arange(n)
    qpos = np.arange(hist, n)
    q = _rand(T, 16, 256)
    k = _rand(n, 4, 256)
    v = _rand(n, 4, 256)
    gate = _rand(T, 16)
    ours = O.attention(q, k, v, gate, qpos, kpos, kind)
    ref = _sdpa_reference(q, k, v, gate, qpos, kpos, kind)
    np.testing.assert_allclose(ours, ref, rtol=1e-10, atol=1e-12)


def test_attention_brute_force_loops():
    """Pure-Python loops over every (query, head, key) on a tiny case."""
    T = 6
    q, k, v, g = _rand(T, 16, 256), _rand(T, 4, 256), _rand(T, 4, 256), _rand(T, 16)
    pos = np.arange(T) + 509                 # window edge crosses the tiny sequence
    for kind in (O.SLIDING, O.FULL):
        ours = O.attention(q, k, v, g, pos, pos, kind)
        for i in range(T):
            for h in range(16):
                kv = h // 4
                scores = []
                for j in range(T):
                    ok = pos[j] <= pos[i] and (kind == O.FULL or pos[j] > pos[i] - 512)
                    if ok:
                        scores.append((j, sum(q[i, h, d] * k[j, kv, d] for d in range(256)) / 16.0))
                mx = max(s for _, s in scores)
                w = [(j, math.exp(s - mx)) for j, s in scores]
                z = sum(e for _, e in w)
                gate = 1.0 / (1.0 + math.exp(-g[i, h]))
                for d in (0, 1, 63, 64, 128, 255):
                    ref = sum(e * v[j, kv, d] for j, e in w) / z * gate
                    assert abs(ours[i, h, d] - ref) < 1e-12


def test_window_edge_query_512_loses_key_0():
    T = 513
    pos = np.arange(T)
    q, k, v, g = _rand(T, 16, 256), _rand(T, 4, 256), _rand(T, 4, 256), _rand(T, 16)
    s = O.attention(q, k, v, g, pos, pos, O.SLIDING)
    f = O.attention(q, k, v, g, pos, pos, O.FULL)
    np.testing.assert_array_equal(s[:512], f[:512])      # T <= 512: sliding == full
    assert np.max(np.abs(s[512] - f[512])) > 1e-6          # query 512 no longer sees key 0
    # sliding query i ignores key i-512: perturbing key 0 leaves query 512 unchanged
    k2, v2 = k.copy(), v.copy()
    k2[0] += 10.0
    v2[0] -= 5.0
    s2 = O.attention(q, k2, v2, g, pos, pos, O.SLIDING)
    np.testing.assert_array_equal(s2[512], s[512])
    assert np.max(np.abs(s2[511] - s[511])) > 1e-6        # but query 511 does see key 0


def test_gqa_head_mapping():
    T = 9
    pos = np.arange(T)
    q, k, v, g = _rand(T, 16, 256), _rand(T, 4, 256), _rand(T, 4, 256), _rand(T, 16)
    a = O.attention(q, k, v, g, pos, pos, O.FULL)
    k2, v2 = k.copy(), v.copy()
    k2[:, 1] = _rand(T, 256)
    v2[:, 1] = _rand(T, 256)
    b = O.attention(q, k2, v2, g, pos, pos, O.FULL)
    changed = [h for h in range(16) if np.max(np.abs(a[:, h] - b[:, h])) > 0]
    assert changed == [4, 5, 6, 7]


def test_softmax_rows_sum_to_one_and_v_ones_gives_the_gate():
    T = 700
    pos = np.arange(T)
    q, k, g = _rand(T, 16, 256), _rand(T, 4, 256), _rand(T, 16)
    for kind in (O.SLIDING, O.FULL):
        p = O.attention_probs(q, k, pos, pos, kind)
        np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-13)
        assert np.all(p[:, O.visible(pos, pos, kind) == False] == 0)  # noqa: E712
        out = O.attention(q, k, np.ones((T, 4, 256)), g, pos, pos, kind)
        np.testing.assert_allclose(out, np.broadcast_to((1 / (1 + np.exp(-g)))[:, :, None], out.shape),
                                   rtol=1e-13, atol=1e-14)


def test_gate_zero_halves_the_output():
    T = 40
    pos = np.arange(T)
    q, k, v = _rand(T, 16, 256), _rand(T, 4, 256), _rand(T, 4, 256)
    half = O.attention(q, k, v, np.zeros((T, 16)), pos, pos, O.FULL)
    full = O.attention(q, k, v, np.full((T, 16), 60.0), pos, pos, O.FULL)
    np.testing.assert_allclose(half, 0.5 * full, rtol=1e-13, atol=1e-15)


def test_single_key_returns_gated_value():
    q, k, v, g = _rand(1, 16, 256), _rand(1, 4, 256), _rand(1, 4, 256), _rand(1, 16)
    for kind in (O.SLIDING, O.FULL):
        out = O.layer_prefill(q, k, v, g, np.array([12345]), kind)
        for h in range(16):
            np.testing.assert_allclose(out[0, h], v[0, h // 4] / (1 + math.exp(-g[0, h])), rtol=1e-14)


# ------------------------------------------------ prefill / decode relations ---

@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_decode_equals_last_prefill_row(kind):
    T = 530
    pos = np.arange(T)
    q, k, v, g = _rand(T, 16, 256), _rand(T, 4, 256), _rand(T, 4, 256), _rand(T, 16)
    ref = O.layer_prefill(q, k, v, g, pos, kind)[-1]
    hist_k = O.rope(k[:-1], pos[:-1], kind)
    out = O.layer_decode(q[-1], k[-1], v[-1], g[-1], T - 1, kind, hist_k, v[:-1], pos[:-1])
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_chunked_prefill_equals_one_pass(kind):
    T, c = 900, 384
    pos = np.arange(T)
    q, k, v, g = _rand(T, 16, 256), _rand(T, 4, 256), _rand(T, 4, 256), _rand(T, 16)
    one = O.layer_prefill(q, k, v, g, pos, kind)
    hist_k = O.rope(k[:c], pos[:c], kind)
    two = O.layer_prefill(q[c:], k[c:], v[c:], g[c:], pos[c:], kind, hist_k, v[:c], pos[:c])
    np.testing.assert_allclose(two, one[c:], rtol=1e-12, atol=1e-13)
    rows = np.array([0, 1, 255, 511, 512, 513, T - 1])
    np.testing.assert_allclose(O.layer_prefill_rows(q[rows], k, v, g[rows], pos, kind, rows), one[rows],
                               rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------- KV cache -----

def test_cache_arithmetic_matches_pages():
    g = _golden("pages_numbers.txt")
    per_tok = O.kv_bytes_per_token_full_layer()
    assert per_tok == 4096 == int(g["kv_kb_per_token_full_layer"][0]) * 1024
    assert O.stack_kv_bytes(1) - O.stack_kv_bytes(0) == 36 * 4096      # below the window every layer grows
    assert O.stack_kv_bytes(1000) - O.stack_kv_bytes(999) == 9 * 4096   # past it only the 9 full layers
    assert (O.stack_kv_bytes(10 ** 6) - O.stack_kv_bytes(10 ** 6 - 1)) / 1024 == float(g["kv_kb_per_token_f16_stack"][0])
    q8 = (O.stack_kv_bytes(10 ** 6, O.Q8_0_BYTES_PER_ELEM) - O.stack_kv_bytes(10 ** 6 - 1, O.Q8_0_BYTES_PER_ELEM))
    assert round(q8 / 1024) == float(g["kv_kb_per_token_q8_0_stack"][0])
    gb_100k = 9 * per_tok * 100_000 / 1e9
    assert abs(gb_100k - float(g["kv_gb_100k_tokens_9_full_layers"][0])) < 0.1
    fixed = O.stack_kv_bytes(512) - 9 * per_tok * 512
    assert round(fixed / 1e6) == float(g["sliding_fixed_mb"][0])
    assert 9 * 0 + per_tok * O.MAX_POSITION == 4 * 2 ** 30          # 1M context: 4 GiB per full layer


def test_cache_size_table_matches_pages():
    for ctx, row in _golden("kv_cache_table.txt").items():
        n = int(ctx)
        f16 = O.stack_kv_bytes(n) / 1e9
        q8 = O.stack_kv_bytes(n, O.Q8_0_BYTES_PER_ELEM) / 1e9
        assert abs(q8 - float(row[1])) <= 0.01, (n, q8, row)
        if int(row[2]):
            assert abs(f16 - float(row[0])) <= 0.01, (n, f16, row)
        else:
            assert abs(f16 - float(row[0])) > 0.05, (n, f16, row)   # page error, recorded as such


@pytest.mark.parametrize("P", [0, 1, 300, 511, 512, 513, 1024, 1025, 5000])
def test_ring_holds_latest_position_per_slot(P):
    ring = O.ring_contents_sequential(P)
    for s in range(512):
        cands = [p for p in range(P) if p % 512 == s]
        assert ring[s] == (max(cands) if cands else -1)


@pytest.mark.parametrize("p", [0, 100, 511, 512, 513, 2047])
def test_ring_after_append_holds_exactly_the_sliding_window(p):
    ring = O.ring_contents_sequential(p + 1)
    held = set(int(x) for x in ring if x >= 0)
    window = set(int(j) for j in np.nonzero(O.visible(np.array([p]), np.arange(p + 1), O.SLIDING)[0])[0])
    assert held == window
    assert all(O.cache_slot(j, O.FULL) == j for j in (0, 5, (1 << 20) - 1))


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_group_attention_equals_the_full_form(kind):
    T = 530
    pos = np.arange(T) + 7
    q, k, v, g = _rand(T, 16, 256), _rand(T, 4, 256), _rand(T, 4, 256), _rand(T, 16)
    full = O.attention(q, k, v, g, pos, pos, kind)
    for grp in range(4):
        hs = slice(4 * grp, 4 * grp + 4)
        part = O.attention_group(q[:, hs], k[:, grp], v[:, grp], g[:, hs], pos, pos, kind)
        np.testing.assert_allclose(part, full[:, hs], rtol=1e-12, atol=1e-14)


# ----------------------------------------------------- 8-bit KV blocks -----

def test_q8_worked_example():
    """Hand-computed block: amax 1 -> scale 1/127; -0.5 * 127 = -63.5 rounds away from zero to -64."""
    x = np.zeros(256, dtype=np.float32)
    x[:4] = [1.0, -0.5, 0.25, -1.0]
    codes, scales = O.quantize_q8(x)
    assert list(codes[:4].astype(int) - 128) == [127, -64, 32, -127]
    assert np.all(codes[4:32] == 128)
    assert scales[0] == np.float16(1.0 / 127.0)
    assert np.all(scales[1:] == 0) and np.all(codes[32:] == 128)        # all-zero blocks


def test_q8_rounding_is_exact_half_away():
    """Codes are the float32 product y rounded half away from zero, exactly: with amax 127 the
    factor 127 / amax is 1, so y = x.  0.49999997f (the float just below 1/2) must give 0 even though
    0.49999997f + 0.5f rounds to 1.0f in float32; exact halves go away from zero."""
    x = np.zeros(256, dtype=np.float32)
    below_half = np.nextafter(np.float32(0.5), np.float32(0.0))
    assert below_half + np.float32(0.5) == np.float32(1.0)          # the float32 shortcut would give 1
    x[:9] = [127.0, below_half, -below_half, 0.5, -0.5, 2.5, -2.5, 126.5, -126.5]
    codes, scales = O.quantize_q8(x)
    assert list(codes[:9].astype(int) - 128) == [127, 0, 0, 1, -1, 3, -3, 127, -127]
    assert scales[0] == np.float16(1.0)


def test_q8_rounding_edge_unreachable_from_bf16():
    """The one float32 product where floor(|y| + 0.5f) in float32 differs from exact rounding,
    y = 0.5 - 2^-25, arises from no bf16 value x and bf16 block maximum amax >= |x| (the cache's
    inputs are bf16): for every amax, only the bf16 neighbours of y / (127 / amax) can round to y."""
    bits = np.arange(0x0080, 0x7F80, dtype=np.uint32)           # every positive normal bf16
    amax = (bits << 16).view(np.float32)
    with np.errstate(over="ignore"):
        inv = (np.float32(127.0) / amax).astype(np.float32)
    target = np.nextafter(np.float32(0.5), np.float32(0.0))
    x_near = ((target / inv.astype(np.float64)).astype(np.float32).view(np.uint32) >> 16).astype(np.int64)
    for d in range(-2, 3):
        cand = np.clip(x_near + d, 0x0080, 0x7F7F).astype(np.uint32)
        x = (cand << 16).view(np.float32)
        with np.errstate(over="ignore", invalid="ignore"):
            y = (x * inv).astype(np.float32)
        assert not np.any((y == target) & (x <= amax))


def test_q8_tiny_block_quantises_to_zero():
    """127 / amax overflows float32 for a block of denormal values: codes 0, scale 0 (no inf or NaN)."""
    x = np.zeros(256, dtype=np.float32)
    x[0] = np.float32(1e-40)
    x[40] = np.float32(-3e-38)
    codes, scales = O.quantize_q8(x)
    assert np.all(codes == 128) and np.all(scales == 0)
    assert np.all(O.dequantize_q8(codes, scales) == 0)
    # just above the overflow threshold the block still quantises normally
    x[64] = np.float32(1e-36)
    codes, scales = O.quantize_q8(x)
    assert codes[64] == 255 and scales[2] == 0          # the fp16 scale itself underflows


def test_q8_round_trip_bound_and_code_range():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 5, (64, 1))).astype(np.float32)
    codes, scales = O.quantize_q8(x)
    c = codes.astype(int) - 128
    assert c.min() >= -127 and c.max() <= 127
    blocks = np.abs(x).reshape(64, 8, 32)
    # the largest magnitude of every block maps to +-127
    arg = blocks.argmax(axis=-1)
    assert np.all(np.abs(np.take_along_axis(c.reshape(64, 8, 32), arg[..., None], -1)) == 127)
    # |x - dequant| <= half a step plus the fp16 rounding of the scale
    amax = blocks.max(axis=-1)
    step = amax / 127.0
    err = np.abs(x.astype(np.float64) - O.dequantize_q8(codes, scales)).reshape(64, 8, 32)
    bound = step[..., None] * 0.5 * (1 + 2 ** -10) + amax[..., None] * 2 ** -11
    assert np.all(err <= bound)


def test_q8_bytes_match_the_pages():
    g = _golden("pages_numbers.txt")
    per_tok_q8 = O.kv_bytes_per_token_full_layer(O.q8_bytes_per_value()) * 9
    assert round(per_tok_q8 / 1024) == float(g["kv_kb_per_token_q8_0_stack"][0])   # 36 KB -> 19 KB
