"""Every output element at two full-size workloads, against the fp64 oracle.

- Prefill B=4, T=8192 (seed 1, k sigma 0.5, gate sigma 2), one sliding and one full layer, in the
  launch configuration bench.py times: all 4 x 8192 x 16 x 256 outputs of both layers.
- Decode B=64 with 32768 cached tokens (seed 3), layers 0 (sliding) and 3 (full), one step through
  the fused call bench.py times: all 64 x 16 x 256 outputs of both layers.
- Long-context decode, B=16 at 131072 and B=1 at 2^20 (seed 5), the same two layers and call: all
  outputs.

The oracle's inputs are the seeded generator's values.  The device generator filled the tensors;
they are read back before any library call touches them (and, for the decode caches, only at rows
the step does not write), and a sample of them is checked bit for bit against the host generator,
so the oracle never sees a value the library computed.  The oracle runs in query blocks of 1024
rows (a sliding layer's block sees only the 511 keys before it); the tolerance is the usual
|err| <= 2e-2 + 2e-2 |ref|.
"""
import numpy as np
import pytest
import torch

import bench
import full_gqa_attention_spark2_b200 as sa
import synth
from oracle import spark_oracle as O
from tests.helpers import assert_close, f64, tid

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import __graft_entry__
    __graft_entry__.build()
    sa._lib()
    synth.load_lib()
    yield
    torch.cuda.empty_cache()


def _host_f64(t):
    """A device bf16 tensor as float64 numpy (exact)."""
    return t.float().cpu().numpy().astype(np.float64)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_prefill_b4_t8192_every_element():
    dev = torch.device("cuda")
    B, T, seed = bench.PREFILL_B, bench.PREFILL_T, bench.PREFILL_SEED
    W, pos0 = bench.prefill_workload(torch, sa, synth, dev)
    pos = np.arange(T)
    blk = 1024
    for kind, layer in ((O.SLIDING, 0), (O.FULL, 3)):
        w = W[kind]
        # the generator's values, before the library touches them; one sequence's rows at a few
        # positions checked against the host generator
        rows = np.array([0, 511, 4097, T - 1])
        for name, role, H, sig in (("q", synth.ROLE_Q, 16, 1.0), ("k", synth.ROLE_K, 4, 0.5),
                                   ("v", synth.ROLE_V, 4, 1.0)):
            host = synth.token_tensor(seed, tid(layer, role), B, H, 256, np.broadcast_to(rows, (B, len(rows))), sig)
            assert np.array_equal(_bits(w[name][:, torch.as_tensor(rows, device=dev)]), host), name
        inputs = {n: w[n].cpu() for n in ("q", "k", "v", "g")}
        w["out"].fill_(float("nan"))
        sa.spark_rope_apply(w["k"], pos0, w["cfg"])                  # as in bench.prefill_step
        sa.spark_attn_prefill(w["out"], w["q"], w["k"], w["v"], w["g"], None, None, pos0, w["cfg"],
                              flags=sa.SPARK_ROPE_FUSED)
        sa.spark_check()
        out = w["out"].cpu()
        for b in range(B):
            qr = O.rope(inputs["q"][b].float().numpy().astype(np.float64), pos, kind)
            kr = O.rope(inputs["k"][b].float().numpy().astype(np.float64), pos, kind)
            vb = inputs["v"][b].float().numpy().astype(np.float64)
            gb = inputs["g"][b].float().numpy().astype(np.float64)
            for g in range(4):
                hs = slice(4 * g, 4 * g + 4)
                for r0 in range(0, T, blk):
                    r1 = min(T, r0 + blk)
                    k0 = max(0, r0 - (O.WINDOW - 1)) if kind == O.SLIDING else 0
                    ref = O.attention_group(qr[r0:r1, hs], kr[k0:r1, g], vb[k0:r1, g], gb[r0:r1, hs], pos[r0:r1],
                                            pos[k0:r1], kind)
                    got = out[b, r0:r1, hs].float().numpy().astype(np.float64)
                    assert_close(got, ref, f"prefill B=4 T=8192 kind={kind} b={b} group={g} rows {r0}..{r1 - 1}")
        del inputs, out
    del W
    torch.cuda.empty_cache()


def test_decode_b64_ctx32768_every_sequence():
    dev = torch.device("cuda")
    B, p, seed = bench.DECODE_B, bench.DECODE_CTX, bench.DECODE_SEED
    layers = bench.decode_layers(torch, sa, synth, dev, B, p, (0, 3), seed=seed)
    pos = torch.full((B,), p, dtype=torch.int32, device=dev)
    wsf = torch.zeros(max(sa.spark_decode_fused_workspace_bytes(B, L["cap"], L["cfg"]) for L in layers),
                      dtype=torch.uint8, device=dev)
    bench.decode_fused_step(sa, layers, pos, wsf)
    sa.spark_check()
    for L in layers:
        kind, layer = L["kind"], L["layer"]
        hist = np.arange(max(0, p - (O.WINDOW - 1)) if kind == O.SLIDING else 0, p)
        rows = hist % O.WINDOW if kind == O.SLIDING else hist      # cache rows the step did not write
        rows_d = torch.as_tensor(rows, device=dev)
        got = L["out"].float().cpu().numpy().astype(np.float64)
        pnew = np.full((B, 1), p)
        q_all = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pnew))[:, 0]
        g_all = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pnew))[:, 0]
        kn_all = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pnew))[:, 0]
        vn_all = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pnew))[:, 0]
        # the cached history is the generator's: a sample against the host generator
        for b, g in ((0, 0), (B - 1, 3)):
            sample = hist[[0, len(hist) // 2, -1]]
            host = synth.head_slice(seed, tid(layer, synth.ROLE_K), b, g, 4, 256, sample)
            srows = torch.as_tensor(rows[[0, len(rows) // 2, -1]], device=dev)
            assert np.array_equal(_bits(L["kc"][b, g][srows]), host)
        for b in range(B):
            kh = _host_f64(L["kc"][b][:, rows_d])                  # [4, n, 256]
            vh = _host_f64(L["vc"][b][:, rows_d])
            qr = O.rope(q_all[b][None], np.array([p]), kind)[0]
            knr = O.rope(kn_all[b][None], np.array([p]), kind)[0]
            kpos = np.concatenate([hist, [p]])
            for g in range(4):
                hs = slice(4 * g, 4 * g + 4)
                keys = np.concatenate([kh[g], knr[g][None]])
                vals = np.concatenate([vh[g], vn_all[b, g][None]])
                ref = O.attention_group(qr[None, hs], keys, vals, g_all[b][None, hs], np.array([p]), kpos, kind)[0]
                assert_close(got[b, hs], ref, f"decode B=64 p={p} layer={layer} b={b} group={g}")
    del layers, wsf
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,p", [(16, 131071), (1, (1 << 20) - 1)])
def test_long_decode_every_output(B, p):
    """Long-context decode with the new token at the end of the context (131072 at B=16, 2^20 at
    B=1; seed 5), one step of a sliding and a full layer through the fused call bench.py times:
    all B x 16 x 256 outputs of both layers, one (sequence, KV head) at a time."""
    dev = torch.device("cuda")
    seed = 5
    layers = bench.decode_layers(torch, sa, synth, dev, B, p, (0, 3), seed=seed)
    pos = torch.full((B,), p, dtype=torch.int32, device=dev)
    wsf = torch.zeros(max(sa.spark_decode_fused_workspace_bytes(B, L["cap"], L["cfg"]) for L in layers),
                      dtype=torch.uint8, device=dev)
    bench.decode_fused_step(sa, layers, pos, wsf)
    sa.spark_check()
    for L in layers:
        kind, layer = L["kind"], L["layer"]
        sliding = kind == O.SLIDING
        hist = np.arange(max(0, p - (O.WINDOW - 1)) if sliding else 0, p)
        rows = hist % O.WINDOW if sliding else hist                # cache rows the step did not write
        got = _host_f64(L["out"])
        pnew = np.full((B, 1), p)
        q_all = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pnew))[:, 0]
        g_all = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pnew))[:, 0]
        kn_all = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pnew))[:, 0]
        vn_all = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pnew))[:, 0]
        sample = np.array([0, len(hist) // 3, len(hist) // 2, len(hist) - 1])
        for b, g in ((0, 0), (B - 1, 3)):
            host = synth.head_slice(seed, tid(layer, synth.ROLE_K), b, g, 4, 256, hist[sample])
            assert np.array_equal(_bits(L["kc"][b, g][torch.as_tensor(rows[sample], device=dev)]), host)
        kpos = np.concatenate([hist, [p]])
        rows_d = None if not sliding else torch.as_tensor(rows, device=dev)
        for b in range(B):
            qr = O.rope(q_all[b][None], np.array([p]), kind)[0]
            knr = O.rope(kn_all[b][None], np.array([p]), kind)[0]
            for g in range(4):
                if sliding:
                    kh, vh = _host_f64(L["kc"][b, g][rows_d]), _host_f64(L["vc"][b, g][rows_d])
                else:
                    kh, vh = _host_f64(L["kc"][b, g, :p]), _host_f64(L["vc"][b, g, :p])
                hs = slice(4 * g, 4 * g + 4)
                keys = np.concatenate([kh, knr[g][None]])
                vals = np.concatenate([vh, vn_all[b, g][None]])
                del kh, vh
                ref = O.attention_group(qr[None, hs], keys, vals, g_all[b][None, hs], np.array([p]), kpos, kind)[0]
                assert_close(got[b, hs], ref, f"long decode B={B} p={p} layer={layer} b={b} group={g}")
                del keys, vals
    del layers, wsf
    torch.cuda.empty_cache()
