"""Parity at the full workload sizes, in the launch configurations bench.py times.

The device runs the whole workload; the fp64 oracle checks sampled outputs one
by one (chunk and tile boundaries, window edges, first/last rows, random rows),
regenerating exactly the inputs it needs from the seeded generator.  Tolerance
as everywhere: |err| <= 2e-2 + 2e-2 |ref|.
"""
import numpy as np
import pytest
import torch

import bench
import full_gqa_attention_spark2_b200 as sa
import synth
from oracle import spark_oracle as O
from tests.helpers import assert_close, dev_to_f64, f64, tid

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import __graft_entry__
    __graft_entry__.build()
    sa._lib()
    synth.load_lib()
    yield
    torch.cuda.empty_cache()


def _group_kv(seed, layer, b, g, pos, sigma_k=1.0):
    """K (as generated: raw for chunk tokens) and V of KV head g at positions pos: [n,256] each."""
    k = f64(synth.head_slice(seed, tid(layer, synth.ROLE_K), b, g, 4, 256, pos, sigma_k))
    v = f64(synth.head_slice(seed, tid(layer, synth.ROLE_V), b, g, 4, 256, pos))
    return k, v


def _rope1(x, pos, kind):
    """oracle RoPE of [n,256] rows (one head)."""
    return O.rope(x[:, None, :], pos, kind)[:, 0, :]


# ------------------------------------------------ B=4, T=8192 (headline) ----

def test_prefill_b4_t8192_sampled_rows():
    dev = torch.device("cuda")
    W, pos0 = bench.prefill_workload(torch, sa, synth, dev)
    T = bench.PREFILL_T
    pos = np.arange(T)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 129, 511, 512, 513, 4095, 4096, 8190, 8191],
                                     rng.integers(0, T, 4)]))
    for kind, layer in ((O.SLIDING, 0), (O.FULL, 3)):
        w = W[kind]
        w["out"].fill_(float("nan"))
        sa.spark_rope_apply(w["k"], pos0, w["cfg"])                  # as in bench.prefill_step:
        sa.spark_attn_prefill(w["out"], w["q"], w["k"], w["v"], w["g"], None, None, pos0, w["cfg"],
                              flags=sa.SPARK_ROPE_FUSED)              # q raw, rotated at load
        sa.spark_check()
        # every element written (no unit skipped or stored twice by the dynamic scheduling), and each
        # output a gated convex combination of v rows: |out| <= max |v|
        assert bool(torch.isfinite(w["out"]).all()), f"kind={kind}: unwritten or non-finite outputs"
        assert float(w["out"].abs().max()) <= float(w["v"].abs().max()) * (1 + 2 ** -7)
        for b in (0, 3):
            got = dev_to_f64(w["out"][b, torch.as_tensor(rows, device=dev)])
            for g in range(4):
                hs = slice(4 * g, 4 * g + 4)
                k, v = _group_kv(bench.PREFILL_SEED, layer, b, g, pos, 0.5)
                q = f64(synth.token_tensor(bench.PREFILL_SEED, tid(layer, synth.ROLE_Q), 4, 16, 256,
                                           np.broadcast_to(rows, (4, len(rows))))[b][:, hs])
                gate = f64(synth.token_tensor(bench.PREFILL_SEED, tid(layer, synth.ROLE_GATE), 4, 16, 1,
                                              np.broadcast_to(rows, (4, len(rows))), 2.0)[b][:, hs])
                ref = O.attention_group(O.rope(q, rows, kind), _rope1(k, pos, kind), v, gate, rows, pos, kind)
                assert_close(got[:, hs], ref, f"B=4 T=8192 kind={kind} b={b} group={g}")
    del W
    torch.cuda.empty_cache()


# ---------------------------------- decode: B=64 at 32768, and long context ----

@pytest.mark.parametrize("B,p,layer_ids,check_b,groups", [
    (64, 32768, (0, 3, 34, 35), (0, 31, 63), (0, 1, 2, 3)),      # the 36-layer step's launch configs
    (16, 131071, (0, 3), (0, 15), (1,)),                          # context 131072
    (1, (1 << 20) - 1, (0, 3), (0,), (0, 3)),                     # context 2^20
])
def test_decode_sampled(B, p, layer_ids, check_b, groups):
    dev = torch.device("cuda")
    layers = bench.decode_layers(torch, sa, synth, dev, B, p, layer_ids, seed=bench.DECODE_SEED)
    pos = torch.full((B,), p, dtype=torch.int32, device=dev)
    ws = torch.empty(max(sa.spark_decode_workspace_bytes(B, L["cap"], L["cfg"]) for L in layers),
                     dtype=torch.uint8, device=dev)
    bench.decode_step(sa, layers, pos, ws)
    sa.spark_check()
    seed = bench.DECODE_SEED
    for L in layers:
        kind, layer = L["kind"], L["layer"]
        got = dev_to_f64(L["out"])
        hist = np.arange(max(0, p - 511) if kind == O.SLIDING else 0, p)
        for b in check_b:
            qb = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, np.full((B, 1), p))[b, 0])
            gb = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, np.full((B, 1), p))[b, 0])
            for g in groups:
                hs = slice(4 * g, 4 * g + 4)
                hk, hv = _group_kv(seed, layer, b, g, hist)          # cached keys are taken as rotated
                kn, vn = _group_kv(seed, layer, b, g, np.array([p]))
                keys = np.concatenate([hk, _rope1(kn, np.array([p]), kind)])
                vals = np.concatenate([hv, vn])
                kpos = np.concatenate([hist, [p]])
                q = O.rope(qb[None, hs], np.array([p]), kind)
                ref = O.attention_group(q, keys, vals, gb[None, hs], np.array([p]), kpos, kind)[0]
                assert_close(got[b, hs], ref, f"decode B={B} p={p} layer={layer} b={b} group={g}")
    del layers, ws
    torch.cuda.empty_cache()


def test_decode_q8_b64_ctx32768_sampled():
    """The 8-bit-cache decode step in the launch configuration bench.py times (one sliding and one
    full layer), sampled sequences and groups against the oracle over its own quantised history."""
    dev = torch.device("cuda")
    B, p = bench.DECODE_B, bench.DECODE_CTX
    layers = bench.decode_q8_layers(torch, sa, synth, dev, B, p, (0, 3))
    pos = torch.full((B,), p, dtype=torch.int32, device=dev)
    ws = torch.empty(max(sa.spark_decode_q8_workspace_bytes(B, L["cap"], L["cfg"]) for L in layers),
                     dtype=torch.uint8, device=dev)
    bench.decode_q8_step(sa, layers, pos, ws)
    sa.spark_check()
    seed = bench.DECODE_SEED
    for L in layers:
        kind, layer = L["kind"], L["layer"]
        got = dev_to_f64(L["out"])
        hist = np.arange(max(0, p - 511) if kind == O.SLIDING else 0, p)
        for b in (0, 63):
            qb = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, np.full((B, 1), p))[b, 0])
            gb = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, np.full((B, 1), p))[b, 0])
            for g in (0, 3):
                hs = slice(4 * g, 4 * g + 4)
                hk, hv = _group_kv(seed, layer, b, g, hist)
                kn, vn = _group_kv(seed, layer, b, g, np.array([p]))
                keys = np.concatenate([hk, _rope1(kn, np.array([p]), kind)]).astype(np.float32)
                vals = np.concatenate([hv, vn]).astype(np.float32)
                keys = O.dequantize_q8(*O.quantize_q8(keys))
                vals = O.dequantize_q8(*O.quantize_q8(vals))
                kpos = np.concatenate([hist, [p]])
                q = O.rope(qb[None, hs], np.array([p]), kind)
                ref = O.attention_group(q, keys, vals, gb[None, hs], np.array([p]), kpos, kind)[0]
                assert_close(got[b, hs], ref, f"q8 decode B={B} p={p} layer={layer} b={b} group={g}")
    del layers, ws
    torch.cuda.empty_cache()


# ------------------------------------ long prefill, 8192-token chunks ------

def test_long_prefill_chunked_sampled_rows():
    """B=1, T=131072 in 16 chunks of 8192 over the growing cache, one full and one sliding layer.
    Every chunk: its first and last two rows, the rows at 510-513 (the window edge), and 8 seeded
    random rows; all 16 heads, against the oracle over every key the row sees."""
    dev = torch.device("cuda")
    seed, T, C = 4, 131072, 8192
    n_ch = T // C
    rng = np.random.default_rng(2024)
    rel = {c: np.unique(np.concatenate([[0, 1, 510, 511, 512, 513, C - 2, C - 1],
                                        rng.choice(C, 8, replace=False)])) for c in range(n_ch)}
    for kind, layer in ((O.SLIDING, 0), (O.FULL, 3)):
        cfg = sa.spark_layer_cfg_for_kind(kind)
        cap = 512 if kind == O.SLIDING else T
        kc = torch.zeros(1, 4, cap, 256, dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        q = torch.empty(1, C, 16, 256, dtype=torch.bfloat16, device=dev)
        k = torch.empty(1, C, 4, 256, dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        gt = torch.empty(1, C, 16, dtype=torch.bfloat16, device=dev)
        out = torch.empty_like(q)
        got = {}
        for c in range(n_ch):
            p0 = c * C
            synth.fill_tokens(q, seed, tid(layer, synth.ROLE_Q), p0)
            synth.fill_tokens(k, seed, tid(layer, synth.ROLE_K), p0)
            synth.fill_tokens(v, seed, tid(layer, synth.ROLE_V), p0)
            synth.fill_tokens(gt, seed, tid(layer, synth.ROLE_GATE), p0)
            pos0 = torch.full((1,), p0, dtype=torch.int32, device=dev)
            sa.spark_rope_apply(k, pos0, cfg)
            sa.spark_attn_prefill(out, q, k, v, gt, kc if c else None, vc if c else None, pos0, cfg,
                                  flags=sa.SPARK_ROPE_FUSED)
            sa.spark_kv_append(kc, vc, k, v, pos0, cfg)
            got[c] = dev_to_f64(out[0, torch.as_tensor(rel[c], device=dev)])
        sa.spark_check()
        del kc, vc, q, k, v, gt, out
        torch.cuda.empty_cache()
        all_pos = np.arange(T)
        for g in range(4):
            hs = slice(4 * g, 4 * g + 4)
            k_all, v_all = _group_kv(seed, layer, 0, g, all_pos)
            k_all = _rope1(k_all, all_pos, kind)
            for c in range(n_ch):
                rows = c * C + rel[c]
                q_rows = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_Q), 1, 16, 256, rows)[0][:, hs])
                g_rows = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), 1, 16, 1, rows)[0][:, hs])
                lo = max(0, rows.min() - 511) if kind == O.SLIDING else 0
                hi = rows.max() + 1
                ref = O.attention_group(O.rope(q_rows, rows, kind), k_all[lo:hi], v_all[lo:hi], g_rows, rows,
                                        all_pos[lo:hi], kind)
                assert_close(got[c][:, hs], ref, f"long prefill kind={kind} chunk={c} group={g}")
            del k_all, v_all
    torch.cuda.empty_cache()
