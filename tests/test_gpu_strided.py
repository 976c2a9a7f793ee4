"""q, k and v as views of one fused projection output, through the C ABI.

A layer's q_k_v_proj ("Spark-X2.6-4B-FP8 W8A8" page §三) produces one [B, T, 16 + 4 + 4, 256] tensor;
the calls take its slices as they are (element strides), with no copy.  Each call on the views must
give bit for bit what it gives on dense copies of them, and the prefill and decode outputs must match
the fp64 oracle at the usual tolerance |err| <= 2e-2 + 2e-2 |ref|.
"""
import numpy as np
import pytest
import torch

import full_gqa_attention_spark2_b200 as sa
import synth
from oracle import spark_oracle as O
from tests.helpers import assert_close, dev_to_f64, f64, tid, to_dev

pytestmark = pytest.mark.gpu
LAYER = {O.SLIDING: 0, O.FULL: 3}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import __graft_entry__
    __graft_entry__.build()
    sa._lib()
    yield


def _fused_buffer(kind, B, T, pos, seed):
    """x [B, T, 24, 256] holding q (heads 0-15), k (16-19) and v (20-23) from the generator, raw."""
    layer = LAYER[kind]
    q = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pos)
    k = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pos)
    v = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pos)
    x = to_dev(np.concatenate([q, k, v], axis=2))
    g_bits = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pos)
    return x, to_dev(g_bits), (q, k, v, g_bits)


def _bits(t):
    return t.contiguous().view(torch.int16)


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_prefill_and_append_on_projection_views(kind):
    """Two chunks (300 tokens, then 260 over the cached history) of B=2 sequences at different
    positions: RoPE on k's view, the prefill with q rotated at load, the append of k and v's views."""
    B, T1, T2 = 2, 300, 260
    seed = 61
    p0 = np.array([0, 777])
    pos1 = p0[:, None] + np.arange(T1)[None, :]
    pos2 = p0[:, None] + T1 + np.arange(T2)[None, :]
    cfg = sa.spark_layer_cfg_for_kind(kind)
    cap = 512 if kind == O.SLIDING else int(p0.max()) + T1 + T2
    caches = {}
    for name in ("view", "dense"):
        caches[name] = (torch.zeros(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda"),
                        torch.zeros(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda"))
    outs = {}
    host = []
    for c, (pos, T) in enumerate(((pos1, T1), (pos2, T2))):
        x, g, h = _fused_buffer(kind, B, T, pos, seed)
        host.append((pos, h))
        pos0 = torch.tensor(pos[:, 0], dtype=torch.int32, device="cuda")
        q, k, v = x[:, :, :16], x[:, :, 16:20], x[:, :, 20:24]
        assert not q.is_contiguous() and not k.is_contiguous() and not v.is_contiguous()
        qd, kd, vd = q.contiguous(), k.contiguous(), v.contiguous()
        for name, (qq, kk, vv) in (("view", (q, k, v)), ("dense", (qd, kd, vd))):
            kc, vc = caches[name]
            out = torch.full((B, T, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
            sa.spark_rope_apply(kk, pos0, cfg)
            sa.spark_attn_prefill(out, qq, kk, vv, g, kc if c else None, vc if c else None, pos0, cfg,
                                  flags=sa.SPARK_ROPE_FUSED)
            sa.spark_kv_append(kc, vc, kk, vv, pos0, cfg)
            outs[(name, c)] = out
        sa.spark_check()
        assert torch.equal(_bits(outs[("view", c)]), _bits(outs[("dense", c)])), f"chunk {c}: view != dense"
        assert torch.equal(_bits(k), _bits(kd)), "rotated k differs"
        assert torch.equal(_bits(x[:, :, :16]), _bits(to_dev(h[0]))), "q was modified"
    for a, b in zip(caches["view"], caches["dense"]):
        assert torch.equal(_bits(a), _bits(b)), "cache differs"
    # the second chunk against the oracle: keys of both chunks rotated by the oracle, and the cache's
    # zero rows for the positions before a sequence's first chunk (never written: zero keys and values)
    (pos_a, (qa, ka, va, ga)), (pos_b, (qb, kb, vb, gb)) = host
    got = dev_to_f64(outs[("view", 1)])
    for b in range(B):
        pre = np.arange(p0[b])
        kpos = np.concatenate([pre, pos_a[b], pos_b[b]])
        zeros = np.zeros((len(pre), 4, 256))
        keys = np.concatenate([zeros, O.rope(f64(ka[b]), pos_a[b], kind), O.rope(f64(kb[b]), pos_b[b], kind)])
        vals = np.concatenate([zeros, f64(va[b]), f64(vb[b])])
        ref = O.attention(O.rope(f64(qb[b]), pos_b[b], kind), keys, vals, f64(gb[b]), pos_b[b], kpos, kind)
        assert_close(got[b], ref, f"strided prefill kind={kind} b={b}")


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_decode_on_projection_views(kind):
    """One decode step of B=3 sequences whose new token's q, k, v are slices of [B, 1, 24, 256]: the
    two-call path and the fused call on the views equal the same calls on dense copies, bit for bit."""
    B, p = 3, 1500
    seed = 67
    cfg = sa.spark_layer_cfg_for_kind(kind)
    sliding = kind == O.SLIDING
    cap = 512 if sliding else p + 1
    layer = LAYER[kind]
    pos_np = np.full((B, 1), p)
    x, g, _ = _fused_buffer(kind, B, 1, pos_np, seed)
    q, k, v = x[:, 0, :16], x[:, 0, 16:20], x[:, 0, 20:24]
    gate = g[:, 0]
    pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
    res = {}
    for name, (qq, kk, vv) in (("view", (q, k, v)), ("dense", (q.contiguous(), k.contiguous(), v.contiguous()))):
        for path in ("two_call", "fused"):
            kc = torch.empty(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
            vc = torch.empty_like(kc)
            synth.fill_cache(kc, seed, tid(layer, synth.ROLE_K), p, sliding)
            synth.fill_cache(vc, seed, tid(layer, synth.ROLE_V), p, sliding)
            out = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
            if path == "two_call":
                sa.spark_kv_append(kc, vc, kk[:, None], vv[:, None], pos, cfg, flags=sa.SPARK_ROPE_FUSED)
                ws = torch.empty(sa.spark_decode_workspace_bytes(B, cap, cfg), dtype=torch.uint8, device="cuda")
                sa.spark_attn_decode(out, qq, gate, kc, vc, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
            else:
                ws = sa.spark_decode_fused_workspace(B, cap, cfg)
                sa.spark_attn_decode_fused(out, qq, kk, vv, gate, kc, vc, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
            sa.spark_check()
            res[(name, path)] = (out, kc, vc)
    for path in ("two_call", "fused"):
        for a, b in zip(res[("view", path)], res[("dense", path)]):
            assert torch.equal(_bits(a), _bits(b)), f"{path}: view != dense"
    assert_close(dev_to_f64(res[("view", "fused")][0]), dev_to_f64(res[("view", "two_call")][0]),
                 f"fused vs two-call on views, kind={kind}")
