"""GPU parity of every kernel against the fp64 oracle, through the C ABI.

Inputs come from the seeded generator (synth): the device fills its buffers,
the host regenerates the same values bit for bit and hands them to the
oracle.  Floating-point outputs must satisfy |err| <= 2e-2 + 2e-2 |ref| per
bf16 element; cache contents and indexing must match bit for bit.
"""
import numpy as np
import pytest
import torch

import full_gqa_attention_spark2_b200 as sa
import synth
from oracle import spark_oracle as O
from tests.helpers import assert_close, dev_to_f64, f64, tid, to_dev

pytestmark = pytest.mark.gpu
KINDS = [O.SLIDING, O.FULL]
KIND_NAME = {O.SLIDING: "sliding", O.FULL: "full"}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import __graft_entry__
    __graft_entry__.build()
    sa._lib()
    yield


def _cfg(kind):
    return sa.spark_layer_cfg_for_kind(kind)


def _pos_tensor(vals):
    return torch.tensor(list(vals), dtype=torch.int32, device="cuda")


# ------------------------------------------------------------------ RoPE ----

@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("H", [16, 4])
def test_rope_apply(kind, H):
    B, T = 3, 37
    pos0 = [0, 777, (1 << 20) - T]
    pos = np.array([[p + t for t in range(T)] for p in pos0])
    bits = synth.token_tensor(5, tid(kind, synth.ROLE_Q), B, H, 256, pos)
    x = to_dev(bits)
    sa.spark_rope_apply(x, _pos_tensor(pos0), _cfg(kind))
    sa.spark_check()
    got = dev_to_f64(x)
    for b in range(B):
        ref = O.rope(f64(bits[b]), pos[b], kind)
        assert_close(got[b], ref, f"rope {KIND_NAME[kind]} b={b}")
    if kind == O.FULL:
        np.testing.assert_array_equal(x.view(torch.int16).cpu().numpy()[..., 64:].view(np.uint16), bits[..., 64:])


def test_rope_rejects_bad_position_on_device():
    x = to_dev(synth.token_tensor(1, 9, 1, 4, 256, np.arange(4)))
    before = x.clone()
    sa.spark_rope_apply(x, _pos_tensor([(1 << 20) - 2]), _cfg(O.FULL))
    with pytest.raises(sa.SparkError) as e:
        sa.spark_check()
    assert e.value.status == -5
    assert torch.equal(x, before)
    sa.spark_check()          # the error word was cleared


# ------------------------------------------------------------- KV append ----

@pytest.mark.parametrize("T,pos0", [(1, 0), (5, 509), (700, 0), (513, 1000), (1024, 3)])
def test_kv_append_ring_bit_exact(T, pos0):
    kind = O.SLIDING
    B = 2
    pos = np.array([[pos0 + t for t in range(T)]] * B)
    kb = synth.token_tensor(2, tid(0, synth.ROLE_K), B, 4, 256, pos)
    vb = synth.token_tensor(2, tid(0, synth.ROLE_V), B, 4, 256, pos)
    kc = torch.zeros(B, 4, 512, 256, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    sa.spark_kv_append(kc, vc, to_dev(kb), to_dev(vb), _pos_tensor([pos0] * B), _cfg(kind))
    sa.spark_check()
    exp_k = np.zeros((B, 4, 512, 256), np.uint16)
    exp_v = np.zeros_like(exp_k)
    for t in range(T):                       # sequential appends, later tokens overwrite
        s = O.cache_slot(pos0 + t, kind)
        exp_k[:, :, s] = kb[:, t]
        exp_v[:, :, s] = vb[:, t]
    np.testing.assert_array_equal(kc.view(torch.int16).cpu().numpy().view(np.uint16), exp_k)
    np.testing.assert_array_equal(vc.view(torch.int16).cpu().numpy().view(np.uint16), exp_v)


def test_kv_append_linear_bit_exact_and_fused_rope():
    kind = O.FULL
    B, T, cap = 2, 300, 2048
    pos0 = [0, 1700]
    pos = np.array([[p + t for t in range(T)] for p in pos0])
    kb = synth.token_tensor(3, tid(3, synth.ROLE_K), B, 4, 256, pos)
    vb = synth.token_tensor(3, tid(3, synth.ROLE_V), B, 4, 256, pos)
    kc = torch.zeros(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kd = to_dev(kb)
    sa.spark_kv_append(kc, vc, kd, to_dev(vb), _pos_tensor(pos0), _cfg(kind), flags=sa.SPARK_ROPE_FUSED)
    sa.spark_check()
    assert np.array_equal(kd.view(torch.int16).cpu().numpy().view(np.uint16), kb)      # input untouched
    vh = vc.view(torch.int16).cpu().numpy().view(np.uint16)
    kh = dev_to_f64(kc)
    for b in range(B):
        rows = pos[b]
        np.testing.assert_array_equal(vh[b][:, rows].transpose(1, 0, 2), vb[b])
        others = np.setdiff1d(np.arange(cap), rows)
        assert not vh[b][:, others].any()
        ref = O.rope(f64(kb[b]), pos[b], kind)
        assert_close(kh[b][:, rows].transpose(1, 0, 2), ref, f"fused rope append b={b}")


def test_kv_append_rejects_overflow_on_device():
    kc = torch.zeros(1, 4, 64, 256, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.ones(1, 8, 4, 256, dtype=torch.bfloat16, device="cuda")
    sa.spark_kv_append(kc, vc, k, k, _pos_tensor([60]), _cfg(O.FULL))
    with pytest.raises(sa.SparkError) as e:
        sa.spark_check()
    assert e.value.status == -5
    assert not kc.any()


def test_host_side_argument_checks():
    cfg = _cfg(O.SLIDING)
    kc = torch.zeros(1, 4, 256, 256, dtype=torch.bfloat16, device="cuda")      # ring must be 512 rows
    k = torch.ones(1, 1, 4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SparkError) as e:
        sa.spark_kv_append(kc, kc, k, k, _pos_tensor([0]), cfg)
    assert e.value.status == -1
    bad = sa.spark_layer_cfg_for_kind(sa.SPARK_SLIDING)
    bad.theta = 5e6
    with pytest.raises(sa.SparkError):
        sa.spark_rope_apply(k, _pos_tensor([0]), bad)


# ---------------------------------------------------------------- decode ----

def _decode_case(kind, B, p_list, seed=11, layer=0, fused_q=True, cap_extra=5, poison=False):
    """Append the new token (rope fused) and decode; return (out, reference).
    poison: cache rows past each sequence's new token hold NaN (memory the caller never wrote)."""
    sliding = kind == O.SLIDING
    assert not sliding or len(set(p_list)) == 1
    cap = 512 if sliding else max(p_list) + 1 + cap_extra
    n_hist = max(p_list) if not sliding else p_list[0]
    kc = torch.empty(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    synth.fill_cache(kc, seed, tid(layer, synth.ROLE_K), n_hist, sliding)
    synth.fill_cache(vc, seed, tid(layer, synth.ROLE_V), n_hist, sliding)
    # the new token of sequence b lives at p_list[b]
    pnew = np.array(p_list)[:, None]
    qb = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pnew)[:, 0]
    kb = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pnew)
    vb = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pnew)
    gb = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pnew)[:, 0]
    pos = _pos_tensor(p_list)
    cfg = _cfg(kind)
    sa.spark_kv_append(kc, vc, to_dev(kb), to_dev(vb), pos, cfg, flags=sa.SPARK_ROPE_FUSED)
    if poison:
        for b, p in enumerate(p_list):
            if not sliding or p < 511:
                kc[b, :, p + 1:] = float("nan")
                vc[b, :, p + 1:] = float("nan")
    q = to_dev(qb)
    if not fused_q:
        q4 = q.view(B, 1, 16, 256)
        sa.spark_rope_apply(q4, pos, cfg)
    out = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(sa.spark_decode_workspace_bytes(B, cap, cfg), dtype=torch.uint8, device="cuda")
    sa.spark_attn_decode(out, q, to_dev(gb), kc, vc, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED if fused_q else 0)
    sa.spark_check()
    got = dev_to_f64(out)
    refs = []
    for b, p in enumerate(p_list):
        hp = np.arange(max(0, p - 511) if sliding else 0, p)
        hist_k = np.stack([f64(synth.head_slice(seed, tid(layer, synth.ROLE_K), b, g, 4, 256, hp)) for g in range(4)], 1)
        hist_v = np.stack([f64(synth.head_slice(seed, tid(layer, synth.ROLE_V), b, g, 4, 256, hp)) for g in range(4)], 1)
        refs.append(O.layer_decode(f64(qb[b]), f64(kb[b, 0]), f64(vb[b, 0]), f64(gb[b]), p, kind,
                                   hist_k, hist_v, hp))
    return got, np.stack(refs)


@pytest.mark.parametrize("p", [0, 1, 63, 64, 200, 511, 512, 513, 1000, 4097])
def test_decode_sliding(p):
    got, ref = _decode_case(O.SLIDING, 3, [p] * 3)
    assert_close(got, ref, f"decode sliding p={p}")


@pytest.mark.parametrize("p_list", [[0], [5, 64, 65], [127, 128, 129, 3000], [20000, 1, 9999]])
def test_decode_full(p_list):
    got, ref = _decode_case(O.FULL, len(p_list), p_list)
    assert_close(got, ref, f"decode full p={p_list}")


@pytest.mark.parametrize("kind,p_list", [(O.FULL, [5, 64, 65]), (O.FULL, [127, 128, 129, 3000]),
                                         (O.SLIDING, [0]), (O.SLIDING, [63]), (O.SLIDING, [64]),
                                         (O.SLIDING, [200])])
def test_decode_ignores_nan_past_the_last_key(kind, p_list):
    """Rows the caller never wrote may hold NaN; a zero probability must not multiply them."""
    got, ref = _decode_case(kind, len(p_list), p_list, cap_extra=100, poison=True)
    assert np.isfinite(got).all()
    assert_close(got, ref, f"decode {KIND_NAME[kind]} p={p_list}, NaN past the last key")


def test_decode_unfused_q_matches_fused():
    got, ref = _decode_case(O.FULL, 2, [700, 1500], fused_q=False)
    assert_close(got, ref, "decode full, q rotated by spark_rope_apply")


def test_decode_rejects_position_beyond_cache():
    cfg = _cfg(O.FULL)
    kc = torch.zeros(1, 4, 100, 256, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(1, 16, 256, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(1, 16, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    ws = torch.empty(sa.spark_decode_workspace_bytes(1, 100, cfg), dtype=torch.uint8, device="cuda")
    sa.spark_attn_decode(out, q, g, kc, kc, _pos_tensor([100]), cfg, ws)
    with pytest.raises(sa.SparkError) as e:
        sa.spark_check()
    assert e.value.status == -5


# --------------------------------------------------------------- prefill ----

def _prefill_case(kind, B, T, pos0_list, seed=21, layer=0, sigma_k=1.0, sigma_g=1.0, fused_q=False,
                  history=True, poison=False, cap_extra=7):
    """history=False: positions start at pos0 but no cache is passed, so each chunk sees only itself.
    poison: cache rows that hold no history position are NaN (memory the caller never wrote)."""
    sliding = kind == O.SLIDING
    has_hist = history and max(pos0_list) > 0
    assert not (sliding and has_hist) or len(set(pos0_list)) == 1
    pos = np.array([[p + t for t in range(T)] for p in pos0_list])
    qb = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pos)
    kb = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pos, sigma_k)
    vb = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pos)
    gb = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pos, sigma_g)
    cfg = _cfg(kind)
    p0 = _pos_tensor(pos0_list)
    q, k = to_dev(qb), to_dev(kb)
    if not fused_q:
        sa.spark_rope_apply(q, p0, cfg)
    sa.spark_rope_apply(k, p0, cfg)
    kc = vc = None
    if has_hist:
        n_hist = max(pos0_list)
        cap = 512 if sliding else n_hist + cap_extra
        kc = torch.empty(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
        vc = torch.empty_like(kc)
        synth.fill_cache(kc, seed, tid(layer, synth.ROLE_K), n_hist, sliding, sigma_k)
        synth.fill_cache(vc, seed, tid(layer, synth.ROLE_V), n_hist, sliding)
        if poison:
            for b, p0b in enumerate(pos0_list):
                if not sliding or p0b < 512:
                    kc[b, :, p0b:] = float("nan")
                    vc[b, :, p0b:] = float("nan")
    out = torch.full((B, T, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.spark_attn_prefill(out, q, k, to_dev(vb), to_dev(gb), kc, vc, p0, cfg,
                          flags=sa.SPARK_ROPE_FUSED if fused_q else 0)
    sa.spark_check()
    got = dev_to_f64(out)
    refs = []
    for b, p0b in enumerate(pos0_list):
        hp = np.arange(max(0, p0b - 511) if sliding else 0, p0b) if has_hist else np.arange(0)
        hist_k = hist_v = None
        if len(hp):
            hist_k = np.stack([f64(synth.head_slice(seed, tid(layer, synth.ROLE_K), b, g, 4, 256, hp, sigma_k))
                               for g in range(4)], 1)
            hist_v = np.stack([f64(synth.head_slice(seed, tid(layer, synth.ROLE_V), b, g, 4, 256, hp))
                               for g in range(4)], 1)
        refs.append(O.layer_prefill(f64(qb[b]), f64(kb[b]), f64(vb[b]), f64(gb[b]), pos[b], kind,
                                    hist_k, hist_v, hp))
    return got, np.stack(refs)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("T", [1, 2, 127, 128, 129, 300, 640])
def test_prefill_no_history(kind, T):
    got, ref = _prefill_case(kind, 1, T, [0])
    assert_close(got, ref, f"prefill {KIND_NAME[kind]} T={T}")


@pytest.mark.parametrize("kind", KINDS)
def test_prefill_batch_of_two(kind):
    got, ref = _prefill_case(kind, 2, 333, [0, 0], seed=4)
    assert_close(got, ref, f"prefill {KIND_NAME[kind]} B=2")


@pytest.mark.parametrize("kind", KINDS)
def test_prefill_more_units_than_resident_clusters(kind):
    """B=5 x 773 tokens: 5 * 8 * 7 = 280 units (two query heads x one 128-query tile each) for about
    74 resident SM pairs, so most units run in clusters that took them from clusters that never
    started; every element is checked, with an odd tile count and a ragged last tile."""
    got, ref = _prefill_case(kind, 5, 773, [0] * 5, seed=21)
    assert_close(got, ref, f"prefill {KIND_NAME[kind]} B=5 T=773")


@pytest.mark.parametrize("kind,T,pos0_list", [(O.SLIDING, 300, [700, 0]), (O.FULL, 200, [333, 0])])
def test_prefill_append_fused(kind, T, pos0_list):
    """SPARK_APPEND_FUSED: the same output as without it, and the cache afterwards bit-identical to an
    explicit spark_kv_append after the call (sliding: ring rows that were history for this chunk get
    overwritten only after the attention)."""
    B = len(pos0_list)
    cfg = _cfg(kind)
    sliding = kind == O.SLIDING
    seed, layer = 9, 0
    pos = np.array([[p0 + t for t in range(T)] for p0 in pos0_list])
    q = to_dev(synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pos))
    k = to_dev(synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pos))
    v = to_dev(synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pos))
    g = to_dev(synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pos))
    p0 = _pos_tensor(pos0_list)
    sa.spark_rope_apply(k, p0, cfg)
    cap = 512 if sliding else max(pos0_list) + T + 3
    kc = torch.empty(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    synth.fill_cache(kc, seed, tid(layer, synth.ROLE_K), max(pos0_list), sliding)
    synth.fill_cache(vc, seed, tid(layer, synth.ROLE_V), max(pos0_list), sliding)
    kc2, vc2 = kc.clone(), vc.clone()
    out1 = torch.empty(B, T, 16, 256, dtype=torch.bfloat16, device="cuda")
    out2 = torch.empty_like(out1)
    sa.spark_attn_prefill(out1, q, k, v, g, kc, vc, p0, cfg, flags=sa.SPARK_ROPE_FUSED)
    sa.spark_kv_append(kc, vc, k, v, p0, cfg)
    sa.spark_attn_prefill(out2, q, k, v, g, kc2, vc2, p0, cfg, flags=sa.SPARK_ROPE_FUSED | sa.SPARK_APPEND_FUSED)
    sa.spark_check()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(kc.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vc2.view(torch.int16))
    with pytest.raises(sa.SparkError) as e:
        sa.spark_attn_prefill(out2, q, k, v, g, None, None, p0, cfg, flags=sa.SPARK_APPEND_FUSED)
    assert e.value.status == -1


@pytest.mark.parametrize("kind,T,pos0", [(O.SLIDING, 256, 512), (O.SLIDING, 200, 700), (O.SLIDING, 130, 1000),
                                         (O.FULL, 256, 512), (O.FULL, 100, 333), (O.FULL, 129, 1)])
def test_prefill_with_history(kind, T, pos0):
    got, ref = _prefill_case(kind, 1, T, [pos0])
    assert_close(got, ref, f"prefill {KIND_NAME[kind]} T={T} pos0={pos0}")


def test_prefill_full_history_per_sequence_positions():
    got, ref = _prefill_case(O.FULL, 3, 160, [0, 256, 900])
    assert_close(got, ref, "prefill full, per-sequence pos0")


@pytest.mark.parametrize("kind", KINDS)
def test_prefill_tiny_config_all_elements(kind):
    """B=1, T=1024, seed 0, q/k/v/gate ~N(0,1): the small prefill workload, every output element."""
    layer = 0 if kind == O.SLIDING else 3
    got, ref = _prefill_case(kind, 1, 1024, [0], seed=0, layer=layer)
    assert_close(got, ref, f"tiny prefill {KIND_NAME[kind]}")


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("T,pos0,history", [(1, 0, True), (129, 0, True), (640, 0, True), (200, 700, True),
                                            (256, (1 << 20) - 256, False), (300, 777777, False)])
def test_prefill_rope_fused_at_load(kind, T, pos0, history):
    """q is raw; the prefill block rotates its Q tile in shared memory before the first MMA.
    The cases near position 2^20 pass no cache (the chunk sees only itself) to keep the
    oracle's work small while still exercising the largest rotation angles."""
    got, ref = _prefill_case(kind, 1, T, [pos0], fused_q=True, history=history)
    assert_close(got, ref, f"prefill {KIND_NAME[kind]} fused RoPE T={T} pos0={pos0}")


def test_prefill_rope_fused_batch_positions():
    got, ref = _prefill_case(O.FULL, 3, 300, [0, 128, 5000], fused_q=True)
    assert_close(got, ref, "prefill full fused RoPE, per-sequence pos0")


@pytest.mark.parametrize("kind,T,pos0_list", [(O.FULL, 100, [333]), (O.FULL, 129, [1]), (O.FULL, 256, [256]),
                                              (O.FULL, 160, [0, 200, 900]), (O.SLIDING, 300, [200]),
                                              (O.SLIDING, 129, [1]), (O.SLIDING, 64, [130])])
def test_prefill_ignores_nan_past_the_history(kind, T, pos0_list):
    """Cache rows at and past pos0 may hold NaN; the last history tile must not read them."""
    got, ref = _prefill_case(kind, len(pos0_list), T, pos0_list, poison=True, cap_extra=200)
    assert np.isfinite(got).all()
    assert_close(got, ref, f"prefill {KIND_NAME[kind]} T={T} pos0={pos0_list}, NaN past the history")


@pytest.mark.parametrize("kind", KINDS)
def test_prefill_step_in_a_cuda_graph(kind):
    """The prefill step (RoPE on k, the prefill with q rotated at load, the append) captured in a CUDA
    graph and replayed gives the eager step's output and cache bit for bit (the persistent kernel's
    cluster launch control and tensor maps inside a graph)."""
    B, T, seed, layer = 1, 1024, 0, 0
    cfg = _cfg(kind)
    pos = np.broadcast_to(np.arange(T), (B, T))
    qb = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pos)
    kb = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pos)
    vb = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pos)
    gb = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pos)
    p0 = _pos_tensor([0])
    cap = 512 if kind == O.SLIDING else T
    runs = []
    for graph in (False, True):
        q, k, v, g = to_dev(qb), to_dev(kb), to_dev(vb), to_dev(gb)
        kc = torch.zeros(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        out = torch.empty(B, T, 16, 256, dtype=torch.bfloat16, device="cuda")

        def step():
            sa.spark_rope_apply(k, p0, cfg)
            sa.spark_attn_prefill(out, q, k, v, g, None, None, p0, cfg, flags=sa.SPARK_ROPE_FUSED)
            sa.spark_kv_append(kc, vc, k, v, p0, cfg)
        if graph:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=s):
                step()
            gr.replay()
        else:
            step()
        sa.spark_check()
        runs.append((out.view(torch.int16).clone(), kc.view(torch.int16).clone(), vc.view(torch.int16).clone()))
    for a, b in zip(*runs):
        assert torch.equal(a, b)
