"""GPU parity of spark_attn_decode_fused (append + attention + combine in one launch) through the C ABI.

The output is compared with the fp64 oracle (cached keys as the generator writes them, the new
token's key rotated by the oracle's RoPE) at |err| <= 2e-2 + 2e-2 |ref|; the cache row the call
writes is compared bit for bit with what spark_kv_append writes; and the call is repeated on the
same workspace, whose arrival counters (its first B * 4 ints) must be back at zero after every call.  Window edges
(p = 0, 511, 512, 513), a wrapped ring whose outgoing row holds NaN, full layers with mixed
positions and NaN past the history, and the bench's B=64 x 32768 launch are covered.
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
    synth.load_lib()
    yield
    torch.cuda.empty_cache()


def _inputs(kind, B, p_list, seed, cap=None, poison=True):
    """Caches holding positions 0..p-1 of every sequence (the generator's values, taken as rotated),
    NaN in rows past each sequence's history (and in the ring row of the outgoing key), and the new
    token's raw q, k, v and gate logits at p."""
    sliding = kind == O.SLIDING
    layer = LAYER[kind]
    if sliding:
        assert len(set(p_list)) == 1          # one ring fill for the batch
    cap = 512 if sliding else (cap or max(p_list) + 1)
    kc = torch.empty(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    n_hist = p_list[0] if sliding else max(p_list)
    synth.fill_cache(kc, seed, tid(layer, synth.ROLE_K), n_hist, sliding)
    synth.fill_cache(vc, seed, tid(layer, synth.ROLE_V), n_hist, sliding)
    if poison:
        for b, p in enumerate(p_list):
            if sliding and p >= 512:
                kc[b, :, p % 512] = float("nan")     # the key that leaves the window
                vc[b, :, p % 512] = float("nan")
            else:
                kc[b, :, p:] = float("nan")
                vc[b, :, p:] = float("nan")
    pnew = np.array(p_list)[:, None]
    q = to_dev(synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pnew)[:, 0])
    kn = to_dev(synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pnew)[:, 0])
    vn = to_dev(synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pnew)[:, 0])
    g = to_dev(synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pnew)[:, 0])
    pos = torch.tensor(p_list, dtype=torch.int32, device="cuda")
    return dict(kc=kc, vc=vc, q=q, kn=kn, vn=vn, g=g, pos=pos, cfg=sa.spark_layer_cfg_for_kind(kind), cap=cap)


def _oracle(kind, B, p_list, seed, check_b):
    layer = LAYER[kind]
    out = {}
    for b in check_b:
        p = p_list[b]
        hist = np.arange(max(0, p - 511) if kind == O.SLIDING else 0, p)
        qb = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, np.full((B, 1), p))[b, 0])
        gb = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, np.full((B, 1), p))[b, 0])
        rows = np.zeros((16, 256))
        for grp in range(4):
            hs = slice(4 * grp, 4 * grp + 4)
            hk = f64(synth.head_slice(seed, tid(layer, synth.ROLE_K), b, grp, 4, 256, hist))
            hv = f64(synth.head_slice(seed, tid(layer, synth.ROLE_V), b, grp, 4, 256, hist))
            kn = f64(synth.head_slice(seed, tid(layer, synth.ROLE_K), b, grp, 4, 256, np.array([p])))
            vn = f64(synth.head_slice(seed, tid(layer, synth.ROLE_V), b, grp, 4, 256, np.array([p])))
            keys = np.concatenate([hk, O.rope(kn[:, None, :], np.array([p]), kind)[:, 0, :]])
            vals = np.concatenate([hv, vn])
            q = O.rope(qb[None, hs], np.array([p]), kind)
            rows[hs] = O.attention_group(q, keys, vals, gb[None, hs], np.array([p]),
                                         np.concatenate([hist, [p]]), kind)[0]
        out[b] = rows
    return out


def _row_of(kind, p):
    return p % 512 if kind == O.SLIDING else p


def _run_and_check(kind, B, p_list, seed, check_b=None, calls=2):
    x = _inputs(kind, B, p_list, seed)
    # what the unfused append writes into the new token's row (on copies of the caches)
    kc_ref, vc_ref = x["kc"].clone(), x["vc"].clone()
    sa.spark_kv_append(kc_ref, vc_ref, x["kn"].view(B, 1, 4, 256), x["vn"].view(B, 1, 4, 256), x["pos"], x["cfg"],
                       flags=sa.SPARK_ROPE_FUSED)
    ws = sa.spark_decode_fused_workspace(B, x["cap"], x["cfg"])
    n_cnt = B * 4
    check_b = list(range(B)) if check_b is None else check_b
    ref = _oracle(kind, B, p_list, seed, check_b)
    for call in range(calls):
        out = torch.full((B, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
        sa.spark_attn_decode_fused(out, x["q"], x["kn"], x["vn"], x["g"], x["kc"], x["vc"], x["pos"], x["cfg"], ws,
                                   flags=sa.SPARK_ROPE_FUSED)
        sa.spark_check()
        got = dev_to_f64(out)
        for b in check_b:
            assert_close(got[b], ref[b], f"fused decode kind={kind} p={p_list[b]} b={b} call={call + 1}")
        assert int(ws[:4 * n_cnt].view(torch.int32).abs().sum()) == 0, "arrival counters not back at zero"
        for b, p in enumerate(p_list):
            r = _row_of(kind, p)
            assert torch.equal(x["kc"][b, :, r].view(torch.int16), kc_ref[b, :, r].view(torch.int16)), (b, "k row")
            assert torch.equal(x["vc"][b, :, r].view(torch.int16), vc_ref[b, :, r].view(torch.int16)), (b, "v row")
    return x, got


@pytest.mark.parametrize("p", [0, 1, 63, 64, 300, 511, 512, 513, 1000, 4097, 32768])
def test_fused_decode_sliding(p):
    _run_and_check(O.SLIDING, 3, [p] * 3, seed=41)


@pytest.mark.parametrize("p_list", [[0, 1, 63, 64, 65, 700], [511, 512, 513, 2049], [32768, 32768]])
def test_fused_decode_full(p_list):
    _run_and_check(O.FULL, len(p_list), p_list, seed=43)


def test_fused_decode_matches_the_two_call_path():
    """Append + spark_attn_decode and the fused call agree within the tolerance on every element."""
    B, p = 5, 2000
    for kind in (O.SLIDING, O.FULL):
        x = _inputs(kind, B, [p] * B, seed=47, poison=False)
        kc2, vc2 = x["kc"].clone(), x["vc"].clone()
        ref = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
        sa.spark_kv_append(kc2, vc2, x["kn"].view(B, 1, 4, 256), x["vn"].view(B, 1, 4, 256), x["pos"], x["cfg"],
                           flags=sa.SPARK_ROPE_FUSED)
        ws = torch.empty(sa.spark_decode_workspace_bytes(B, x["cap"], x["cfg"]), dtype=torch.uint8, device="cuda")
        sa.spark_attn_decode(ref, x["q"], x["g"], kc2, vc2, x["pos"], x["cfg"], ws, flags=sa.SPARK_ROPE_FUSED)
        out = torch.empty_like(ref)
        wsf = sa.spark_decode_fused_workspace(B, x["cap"], x["cfg"])
        sa.spark_attn_decode_fused(out, x["q"], x["kn"], x["vn"], x["g"], x["kc"], x["vc"], x["pos"], x["cfg"], wsf,
                                   flags=sa.SPARK_ROPE_FUSED)
        sa.spark_check()
        assert_close(dev_to_f64(out), dev_to_f64(ref), f"fused vs two calls, kind={kind}")
        assert torch.equal(x["kc"].view(torch.int16), kc2.view(torch.int16))
        assert torch.equal(x["vc"].view(torch.int16), vc2.view(torch.int16))


def test_fused_decode_b64_ctx32768():
    """The bench's launch configuration: B=64 at p=32768, a sliding and a full layer; sampled
    sequences against the oracle, every sequence's cache row against the append's."""
    B, p = 64, 32768
    for kind in (O.SLIDING, O.FULL):
        x, got = _run_and_check(kind, B, [p] * B, seed=3, check_b=[0, 17, 63], calls=2)
        del x
        torch.cuda.empty_cache()


def test_fused_decode_long_context():
    """B=1 at p = 2^18 - 1 on a full layer: each of the 4 units spread over ~37 blocks of the grid,
    whose partials the last block to finish merges."""
    p = (1 << 18) - 1
    _run_and_check(O.FULL, 1, [p], seed=5, calls=1)
    torch.cuda.empty_cache()


def test_fused_decode_one_workspace_for_both_layer_kinds():
    """Layers of both kinds in turn on one workspace (sized for the larger), as a decode step runs them:
    every output matches the oracle and the counters are zero after each call."""
    B, p = 4, 3000
    xs = {kind: _inputs(kind, B, [p] * B, seed=53) for kind in (O.SLIDING, O.FULL)}
    ws = torch.zeros(max(sa.spark_decode_fused_workspace_bytes(B, x["cap"], x["cfg"]) for x in xs.values()),
                     dtype=torch.uint8, device="cuda")
    refs = {kind: _oracle(kind, B, [p] * B, 53, range(B)) for kind in xs}
    for kind in (O.FULL, O.SLIDING, O.FULL, O.SLIDING):
        x = xs[kind]
        out = torch.full((B, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
        sa.spark_attn_decode_fused(out, x["q"], x["kn"], x["vn"], x["g"], x["kc"], x["vc"], x["pos"], x["cfg"], ws,
                                   flags=sa.SPARK_ROPE_FUSED)
        sa.spark_check()
        assert int(ws[:4 * B * 4].view(torch.int32).abs().sum()) == 0
        got = dev_to_f64(out)
        for b in range(B):
            assert_close(got[b], refs[kind][b], f"shared workspace kind={kind} b={b}")


def test_fused_decode_bad_position_is_reported_and_the_workspace_stays_usable():
    B = 3
    x = _inputs(O.FULL, B, [10, 20, 30], seed=49)
    ws = sa.spark_decode_fused_workspace(B, x["cap"], x["cfg"])
    out = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    bad = torch.tensor([10, x["cap"], 30], dtype=torch.int32, device="cuda")      # row cap does not exist
    sa.spark_attn_decode_fused(out, x["q"], x["kn"], x["vn"], x["g"], x["kc"], x["vc"], bad, x["cfg"], ws)
    with pytest.raises(sa.SparkError) as e:
        sa.spark_check()
    assert e.value.status == -5
    assert int(ws[:4 * B * 4].view(torch.int32).abs().sum()) == 0
    assert bool(torch.isfinite(out[0]).all()) and bool((out[1] == 0).all())


def test_fused_decode_host_checks():
    B = 2
    x = _inputs(O.FULL, B, [5, 6], seed=51)
    out = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    small = torch.zeros(sa.spark_decode_fused_workspace_bytes(B, x["cap"], x["cfg"]) - 16, dtype=torch.uint8,
                        device="cuda")
    with pytest.raises(sa.SparkError) as e:
        sa.spark_attn_decode_fused(out, x["q"], x["kn"], x["vn"], x["g"], x["kc"], x["vc"], x["pos"], x["cfg"], small)
    assert e.value.status == -1
    ws = sa.spark_decode_fused_workspace(B, x["cap"], x["cfg"])
    with pytest.raises(sa.SparkError) as e:
        sa.spark_attn_decode_fused(out, x["q"], x["kn"], x["vn"], x["g"], x["kc"], x["vc"], x["pos"], x["cfg"], ws,
                                   flags=4)
    assert e.value.status == -1
