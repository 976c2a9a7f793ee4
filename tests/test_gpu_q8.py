"""GPU parity of the 8-bit block-quantised KV cache ("Sharp-Spark-X2.5-4B-GGUF"
page §四: the K/V cache stored as q8_0) against the oracle, through the C ABI.

Append without RoPE must give the oracle's codes and scales bit for bit (both
sides quantise the same bf16 values with the same float32 operations).  With
RoPE fused, the rotation may differ from the oracle's fp64 one in the last bf16
bit, so codes may move by one step; the dequantised keys must match the
oracle's rotated keys within the round-trip bound.  Decode over a q8 cache is
compared with the oracle's attention over the oracle's dequantised history, at
the usual tolerance |err| <= 2e-2 + 2e-2 |ref|.
"""
import numpy as np
import pytest
import torch

import full_gqa_attention_spark2_b200 as sa
import synth
from oracle import spark_oracle as O
from tests.helpers import assert_close, dev_to_f64, f64, tid, to_dev

pytestmark = pytest.mark.gpu
KIND_NAME = {O.SLIDING: "sliding", O.FULL: "full"}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import __graft_entry__
    __graft_entry__.build()
    sa._lib()
    yield


def _pos_tensor(vals):
    return torch.tensor(list(vals), dtype=torch.int32, device="cuda")


def _q8_cache(B, cap, fill_codes=0, fill_scales=0.0):
    codes = torch.full((B, 4, cap, 256), fill_codes, dtype=torch.uint8, device="cuda")
    scales = torch.full((B, 4, cap, 8), fill_scales, dtype=torch.float16, device="cuda")
    return codes, scales


def _host(t):
    return t.cpu().numpy()


# ------------------------------------------------------------------ append ----

@pytest.mark.parametrize("kind,T,pos0_list", [(O.SLIDING, 1, [0, 0]), (O.SLIDING, 5, [509, 509]),
                                              (O.SLIDING, 700, [0, 0]), (O.SLIDING, 513, [1000, 1000]),
                                              (O.FULL, 300, [0, 1700]), (O.FULL, 1, [4095, 7])])
def test_kv_append_q8_bit_exact(kind, T, pos0_list):
    B = len(pos0_list)
    pos = np.array([[p + t for t in range(T)] for p in pos0_list])
    cap = 512 if kind == O.SLIDING else int(pos.max()) + 11
    kb = synth.token_tensor(2, tid(3, synth.ROLE_K), B, 4, 256, pos)
    vb = synth.token_tensor(2, tid(3, synth.ROLE_V), B, 4, 256, pos, 4.0)
    kc, ks = _q8_cache(B, cap)
    vc, vs = _q8_cache(B, cap)
    cfg = sa.spark_layer_cfg_for_kind(kind)
    sa.spark_kv_append_q8(kc, ks, vc, vs, to_dev(kb), to_dev(vb), _pos_tensor(pos0_list), cfg)
    sa.spark_check()
    exp = {n: (np.zeros((B, 4, cap, 256), np.uint8), np.zeros((B, 4, cap, 8), np.float16)) for n in "kv"}
    for name, bits in (("k", kb), ("v", vb)):
        codes, scales = O.quantize_q8(f64(bits).astype(np.float32))     # [B, T, 4, 256]
        for b in range(B):
            for t in range(T):                       # sequential appends: later tokens overwrite
                s = O.cache_slot(pos[b, t], kind)
                exp[name][0][b, :, s] = codes[b, t]
                exp[name][1][b, :, s] = scales[b, t]
    for name, (c, sc) in (("k", (kc, ks)), ("v", (vc, vs))):
        np.testing.assert_array_equal(_host(c), exp[name][0], err_msg=f"{name} codes")
        np.testing.assert_array_equal(_host(sc).view(np.uint16), exp[name][1].view(np.uint16),
                                      err_msg=f"{name} scales")


def test_kv_append_q8_zero_and_extreme_blocks():
    """All-zero blocks give code 128 (c = 0) and scale 0; a block holding one huge value keeps it."""
    B, T = 1, 2
    kb = np.zeros((B, T, 4, 256), np.uint16)
    kb[0, 1, 2, 40] = 0x4780            # 65536.0 alone in its block
    kb[0, 1, 2, 41] = 0xC780            # -65536.0
    kb[0, 1, 3, 255] = 0x0001           # the smallest bf16 subnormal
    kc, ks = _q8_cache(B, 64, 7, 1.0)
    vc, vs = _q8_cache(B, 64, 7, 1.0)
    cfg = sa.spark_layer_cfg_for_kind(O.FULL)
    sa.spark_kv_append_q8(kc, ks, vc, vs, to_dev(kb), to_dev(kb), _pos_tensor([10]), cfg)
    sa.spark_check()
    codes, scales = O.quantize_q8(f64(kb).astype(np.float32))
    np.testing.assert_array_equal(_host(kc)[0, :, 10:12].transpose(1, 0, 2), codes[0])
    np.testing.assert_array_equal(_host(ks)[0, :, 10:12].transpose(1, 0, 2).view(np.uint16),
                                  scales[0].view(np.uint16))
    assert (_host(kc)[0, :, 10] == 128).all() and (_host(ks)[0, :, 10] == 0).all()
    assert (_host(kc)[0, :, 12:] == 7).all()                    # rows past the tokens untouched


def test_kv_append_q8_rounding_ties():
    """Exact halves round away from zero on the device as in the oracle: a block whose largest value
    is 127 (factor 127 / amax = 1) holding +-0.5, +-2.5, +-126.5 and the bf16 values next to 1/2."""
    B, T = 1, 1
    vals = np.zeros((B, T, 4, 256), np.float32)
    vals[0, 0, 1, 32:43] = [127.0, 0.5, -0.5, 2.5, -2.5, 126.5, -126.5, 0.498046875, -0.498046875,
                            0.50390625, 1.5]
    kb = (vals.view(np.uint32) >> 16).astype(np.uint16)      # all exact in bf16
    assert np.array_equal(f64(kb), vals.astype(np.float64))
    kc, ks = _q8_cache(B, 16)
    vc, vs = _q8_cache(B, 16)
    cfg = sa.spark_layer_cfg_for_kind(O.FULL)
    sa.spark_kv_append_q8(kc, ks, vc, vs, to_dev(kb), to_dev(kb), _pos_tensor([3]), cfg)
    sa.spark_check()
    codes, scales = O.quantize_q8(vals)
    assert list(codes[0, 0, 1, 32:43].astype(int) - 128) == [127, 1, -1, 3, -3, 127, -127, 0, 0, 1, 2]
    for c, sc in ((kc, ks), (vc, vs)):
        np.testing.assert_array_equal(_host(c)[0, :, 3], codes[0, 0])
        np.testing.assert_array_equal(_host(sc)[0, :, 3].view(np.uint16), scales[0, 0].view(np.uint16))


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_kv_append_q8_fused_rope(kind):
    B, T = 2, 200
    pos0_list = [0, 300] if kind == O.FULL else [900, 900]
    cap = 512 if kind == O.SLIDING else 1024
    pos = np.array([[p + t for t in range(T)] for p in pos0_list])
    kb = synth.token_tensor(6, tid(0, synth.ROLE_K), B, 4, 256, pos)
    vb = synth.token_tensor(6, tid(0, synth.ROLE_V), B, 4, 256, pos)
    kc, ks = _q8_cache(B, cap)
    vc, vs = _q8_cache(B, cap)
    kd = to_dev(kb)
    cfg = sa.spark_layer_cfg_for_kind(kind)
    sa.spark_kv_append_q8(kc, ks, vc, vs, kd, to_dev(vb), _pos_tensor(pos0_list), cfg, flags=sa.SPARK_ROPE_FUSED)
    sa.spark_check()
    assert np.array_equal(kd.view(torch.int16).cpu().numpy().view(np.uint16), kb)      # input untouched
    kch, ksh = _host(kc), _host(ks)
    for b in range(B):
        slots = np.array([O.cache_slot(p, kind) for p in pos[b]])
        got = O.dequantize_q8(kch[b][:, slots].transpose(1, 0, 2), ksh[b][:, slots].transpose(1, 0, 2))
        ref_rot = O.rope(f64(kb[b]), pos[b], kind)
        ref_codes, _ = O.quantize_q8(ref_rot.astype(np.float32))
        assert np.abs(kch[b][:, slots].transpose(1, 0, 2).astype(int) - ref_codes.astype(int)).max() <= 1
        assert_close(got, ref_rot, f"q8 fused-rope append {KIND_NAME[kind]} b={b}")


def test_q8_host_side_checks():
    cfg = sa.spark_layer_cfg_for_kind(O.SLIDING)
    kc, ks = _q8_cache(1, 256)                     # a ring must have 512 rows
    k = torch.ones(1, 1, 4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SparkError) as e:
        sa.spark_kv_append_q8(kc, ks, kc, ks, k, k, _pos_tensor([0]), cfg)
    assert e.value.status == -1
    kc, ks = _q8_cache(1, 512)
    with pytest.raises(ValueError):
        sa.spark_kv_append_q8(kc, ks[..., :4], kc, ks, k, k, _pos_tensor([0]), cfg)
    assert sa.spark_kv_cache_q8_bytes(cfg, 2, 512) == 2 * 2 * 4 * 512 * (256 + 16)


# ------------------------------------------------------------------ decode ----

def _decode_q8_case(kind, B, p_list, seed=31, layer=0, cap_extra=5, poison=False, sigma_q=1.0, sigma_v=1.0):
    """History appended as q8 without RoPE (keys taken as rotated), the new token with RoPE fused,
    then decode with RoPE fused on q.  Returns (out, reference)."""
    sliding = kind == O.SLIDING
    assert not sliding or len(set(p_list)) == 1
    cap = 512 if sliding else max(p_list) + 1 + cap_extra
    cfg = sa.spark_layer_cfg_for_kind(kind)
    kc, ks = _q8_cache(B, cap)
    vc, vs = _q8_cache(B, cap)
    n_hist = max(p_list)
    hp = np.broadcast_to(np.arange(n_hist), (B, n_hist))
    kh = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, hp)            # [B, n_hist, 4, 256]
    vh = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, hp, sigma_v)
    if n_hist > 0:
        sa.spark_kv_append_q8(kc, ks, vc, vs, to_dev(kh), to_dev(vh), _pos_tensor([0] * B), cfg)
    pnew = np.array(p_list)[:, None]
    qb = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pnew, sigma_q)[:, 0]
    kb = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pnew)
    vb = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pnew, sigma_v)
    gb = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pnew)[:, 0]
    pos = _pos_tensor(p_list)
    sa.spark_kv_append_q8(kc, ks, vc, vs, to_dev(kb), to_dev(vb), pos, cfg, flags=sa.SPARK_ROPE_FUSED)
    if poison:
        for b, p in enumerate(p_list):
            if not sliding or p < 511:
                kc[b, :, p + 1:] = 255
                vc[b, :, p + 1:] = 1
                ks[b, :, p + 1:] = float("nan")
                vs[b, :, p + 1:] = float("nan")
    out = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(sa.spark_decode_q8_workspace_bytes(B, cap, cfg), dtype=torch.uint8, device="cuda")
    sa.spark_attn_decode_q8(out, to_dev(qb), to_dev(gb), kc, ks, vc, vs, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
    sa.spark_check()
    got = dev_to_f64(out)
    refs = []
    for b, p in enumerate(p_list):
        hpos = np.arange(max(0, p - 511) if sliding else 0, p)
        kr = O.rope(f64(kb[b]), np.array([p]), kind)                     # [1, 4, 256]
        keys = np.concatenate([f64(kh[b, hpos]), kr]).astype(np.float32)
        vals = np.concatenate([f64(vh[b, hpos]), f64(vb[b])]).astype(np.float32)
        keys = O.dequantize_q8(*O.quantize_q8(keys))
        vals = O.dequantize_q8(*O.quantize_q8(vals))
        kpos = np.concatenate([hpos, [p]])
        qr = O.rope(f64(qb[b])[None], np.array([p]), kind)
        ref = np.concatenate([O.attention_group(qr[:, 4 * g:4 * g + 4], keys[:, g], vals[:, g],
                                                f64(gb[b])[None, 4 * g:4 * g + 4], np.array([p]), kpos, kind)[0]
                              for g in range(4)])
        refs.append(ref)
    return got, np.stack(refs)


@pytest.mark.parametrize("p", [0, 1, 63, 64, 65, 200, 511, 512, 513, 1000, 4097])
def test_decode_q8_sliding(p):
    got, ref = _decode_q8_case(O.SLIDING, 3, [p] * 3)
    assert_close(got, ref, f"q8 decode sliding p={p}")


@pytest.mark.parametrize("p_list", [[0], [5, 64, 65], [127, 128, 129, 3000], [20000, 1, 9999]])
def test_decode_q8_full(p_list):
    got, ref = _decode_q8_case(O.FULL, len(p_list), p_list)
    assert_close(got, ref, f"q8 decode full p={p_list}")


@pytest.mark.parametrize("kind,p_list", [(O.FULL, [5, 64, 65]), (O.FULL, [130, 3000]), (O.SLIDING, [0]),
                                         (O.SLIDING, [200])])
def test_decode_q8_ignores_garbage_past_the_last_key(kind, p_list):
    got, ref = _decode_q8_case(kind, len(p_list), p_list, cap_extra=100, poison=True)
    assert np.isfinite(got).all()
    assert_close(got, ref, f"q8 decode {KIND_NAME[kind]} p={p_list}, garbage past the last key")


def test_decode_q8_large_values():
    """V of scale 512 and q of scale 2^22 (|q|/16 far above 2^15, so q rows are scaled by a power of
    two before their fp16 products): the output still matches the oracle."""
    got, ref = _decode_q8_case(O.FULL, 2, [777, 2000], sigma_v=512.0)
    assert_close(got / 512.0, ref / 512.0, "q8 decode full, large V")
    got, ref = _decode_q8_case(O.SLIDING, 2, [700, 700], sigma_q=float(1 << 22))
    assert_close(got, ref, "q8 decode sliding, huge q")


# ----------------------------------------------------------------- prefill ----

def _prefill_q8_case(kind, T, pos0_list, seed=43, layer=0, cap_extra=9, flags=None, sigma_v=1.0):
    """A chunk of T tokens per sequence over an 8-bit history.  The history (keys taken as rotated)
    is quantised on the host by the oracle's quantiser and uploaded, so the comparison covers the
    prefill alone; cache rows that hold no history position, and the whole workspace, start as
    garbage (codes 255, NaN scales, NaN bf16).  Returns (out, reference, device tensors)."""
    sliding = kind == O.SLIDING
    B = len(pos0_list)
    cap = 512 if sliding else max(pos0_list) + T + cap_extra
    cfg = sa.spark_layer_cfg_for_kind(kind)
    codes = {n: np.full((B, 4, cap, 256), 255, np.uint8) for n in "kv"}
    scales = {n: np.full((B, 4, cap, 8), np.nan, np.float16) for n in "kv"}
    hist = {}
    for b, p0 in enumerate(pos0_list):
        hp = np.arange(max(0, p0 - 512) if sliding else 0, p0)
        rows = hp % 512 if sliding else hp
        for n, role, sig in (("k", synth.ROLE_K, 1.0), ("v", synth.ROLE_V, sigma_v)):
            x = np.stack([f64(synth.head_slice(seed, tid(layer, role), b, g, 4, 256, hp, sig)) for g in range(4)], 1)
            c, s = O.quantize_q8(x.astype(np.float32))                 # [n, 4, 256], [n, 4, 8]
            codes[n][b, :, rows] = c                               # (advanced index first: [n, 4, 256])
            scales[n][b, :, rows] = s
            hist[b, n] = O.dequantize_q8(c, s)
        hist[b, "pos"] = hp
    pos = np.array([[p + t for t in range(T)] for p in pos0_list])
    qb = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pos)
    kb = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pos)
    vb = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pos, sigma_v)
    gb = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pos)
    p0 = _pos_tensor(pos0_list)
    q, k, v, g = to_dev(qb), to_dev(kb), to_dev(vb), to_dev(gb)
    sa.spark_rope_apply(k, p0, cfg)
    dev = {n + "c": torch.from_numpy(codes[n]).cuda() for n in "kv"}
    dev.update({n + "s": torch.from_numpy(scales[n]).cuda() for n in "kv"})
    ws = torch.full((sa.spark_prefill_q8_workspace_bytes(B, cap, cfg),), 255, dtype=torch.uint8, device="cuda")
    out = torch.full((B, T, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.spark_attn_prefill_q8(out, q, k, v, g, dev["kc"], dev["ks"], dev["vc"], dev["vs"], p0, cfg, ws,
                             flags=sa.SPARK_ROPE_FUSED if flags is None else flags)
    sa.spark_check()
    refs = [O.layer_prefill(f64(qb[b]), f64(kb[b]), f64(vb[b]), f64(gb[b]), pos[b], kind,
                            hist.get((b, "k")), hist.get((b, "v")), hist[b, "pos"]) for b in range(B)]
    return dev_to_f64(out), np.stack(refs), dict(q=q, k=k, v=v, g=g, p0=p0, cfg=cfg, ws=ws, cap=cap, **dev)


@pytest.mark.parametrize("kind,T,pos0_list", [(O.SLIDING, 300, [0, 700, 1500]), (O.SLIDING, 129, [511, 512, 513]),
                                              (O.SLIDING, 1, [4097]), (O.FULL, 200, [0, 333, 1000]),
                                              (O.FULL, 129, [128, 1]), (O.FULL, 128, [4097])])
def test_prefill_q8_history(kind, T, pos0_list):
    """Every element against the oracle's attention over its own dequantised history, per-sequence
    positions, window edges and ring wraps, NaN in the workspace and garbage past the history."""
    got, ref, _ = _prefill_q8_case(kind, T, pos0_list)
    assert_close(got, ref, f"q8-history prefill {KIND_NAME[kind]} T={T} pos0={pos0_list}")


def test_prefill_q8_history_large_values():
    """V of scale 256 through fp16 scales and bf16 history rows."""
    got, ref, _ = _prefill_q8_case(O.FULL, 160, [900, 77], sigma_v=256.0)
    assert_close(got / 256.0, ref / 256.0, "q8-history prefill full, large V")


@pytest.mark.parametrize("kind,T,pos0_list", [(O.SLIDING, 300, [700, 0]), (O.FULL, 200, [333, 0])])
def test_prefill_q8_append_fused(kind, T, pos0_list):
    """SPARK_APPEND_FUSED: the same output, and the 8-bit cache afterwards bit-identical to
    spark_kv_append_q8 of the chunk after the call (a sliding ring's history rows are overwritten
    only after the attention has read them)."""
    got, _, d = _prefill_q8_case(kind, T, pos0_list)
    kc, ks, vc, vs = (d[n].clone() for n in ("kc", "ks", "vc", "vs"))
    out2 = torch.empty(len(pos0_list), T, 16, 256, dtype=torch.bfloat16, device="cuda")
    sa.spark_attn_prefill_q8(out2, d["q"], d["k"], d["v"], d["g"], kc, ks, vc, vs, d["p0"], d["cfg"], d["ws"],
                             flags=sa.SPARK_ROPE_FUSED | sa.SPARK_APPEND_FUSED)
    sa.spark_kv_append_q8(d["kc"], d["ks"], d["vc"], d["vs"], d["k"], d["v"], d["p0"], d["cfg"])
    sa.spark_check()
    assert np.array_equal(dev_to_f64(out2), got)
    assert torch.equal(kc, d["kc"]) and torch.equal(vc, d["vc"])
    assert torch.equal(ks.view(torch.int16), d["ks"].view(torch.int16))
    assert torch.equal(vs.view(torch.int16), d["vs"].view(torch.int16))


def test_prefill_q8_host_checks():
    cfg = sa.spark_layer_cfg_for_kind(O.SLIDING)
    full = sa.spark_layer_cfg_for_kind(O.FULL)
    assert sa.spark_prefill_q8_workspace_bytes(2, 512, cfg) == 2 * 2 * 4 * 512 * 256 * 2
    assert sa.spark_prefill_q8_workspace_bytes(2, 600, cfg) == 0
    assert sa.spark_prefill_q8_workspace_bytes(1, 1000, full) == 2 * 4 * 1000 * 256 * 2
    _, _, d = _prefill_q8_case(O.FULL, 64, [100])
    out = torch.empty(1, 64, 16, 256, dtype=torch.bfloat16, device="cuda")
    args = (out, d["q"], d["k"], d["v"], d["g"], d["kc"], d["ks"], d["vc"], d["vs"], d["p0"], d["cfg"])
    with pytest.raises(sa.SparkError):
        sa.spark_attn_prefill_q8(*args, d["ws"][:-16])              # workspace too small
    with pytest.raises(sa.SparkError):
        sa.spark_attn_prefill_q8(*args, d["ws"], flags=0x80)
    # an argument error of the prefill part (q's token stride not a multiple of 8 elements) is found
    # before anything is launched: the workspace is left as it was
    ws = d["ws"]
    ws.fill_(7)
    q_bad = torch.zeros(1, 64, 16 * 256 + 4, dtype=torch.bfloat16, device="cuda")[..., :16 * 256].view(1, 64, 16, 256)
    with pytest.raises(sa.SparkError) as e:
        sa.spark_attn_prefill_q8(out, q_bad, *args[2:], ws)
    assert e.value.status == -1
    torch.cuda.synchronize()
    assert bool((ws == 7).all())
