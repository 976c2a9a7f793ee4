"""GPU parity of ragged batches (packed sequences of different lengths) through the C ABI.

Sequence b's new tokens are rows cu_seqlens[b]..cu_seqlens[b+1]-1 of packed
tensors; their positions start at pos0[b].  RoPE and appends are checked
against the oracle and a host model of page placement, and the ragged
prefill (history from a paged pool) against the oracle's layer_prefill per
sequence, at |err| <= 2e-2 + 2e-2 |ref|: lengths that are 0, 1, and on both
sides of the 128-row tile, sliding chunks longer than the window, history
lengths that are not multiples of the tile, rings not yet full and wrapped.
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


def _i32(vals):
    return torch.tensor(list(vals), dtype=torch.int32, device="cuda")


def _packed(seed, layer, role, lens, pos0, H, D, sigma=1.0):
    """bf16 bits of the packed rows [total, H, D] (D=1 squeezed) and the per-sequence slices."""
    parts = [synth.token_tensor(seed, tid(layer, role), len(lens), H, D,
                                np.array([[p0 + t for t in range(max(lens))] for p0 in pos0]), sigma)[b, :n]
             for b, n in enumerate(lens)]
    return np.concatenate(parts), parts


def test_rope_varlen():
    lens, pos0 = [1, 0, 37, 200], [0, 5, 900, (1 << 20) - 200]
    cu = np.concatenate([[0], np.cumsum(lens)])
    for kind in (O.SLIDING, O.FULL):
        bits, parts = _packed(5, 0, synth.ROLE_Q, lens, pos0, 16, 256)
        x = to_dev(bits)
        sa.spark_rope_apply_varlen(x, _i32(cu), max(lens), _i32(pos0), sa.spark_layer_cfg_for_kind(kind))
        sa.spark_check()
        got = dev_to_f64(x)
        for b, n in enumerate(lens):
            if n:
                ref = O.rope(f64(parts[b]), pos0[b] + np.arange(n), kind)
                assert_close(got[cu[b]:cu[b + 1]], ref, f"rope varlen {KIND_NAME[kind]} b={b}")


@pytest.mark.parametrize("q8", [False, True])
@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_append_varlen_paged(kind, q8):
    lens, pos0 = [3, 0, 700, 129], [10, 0, 0, 400]
    P = 128
    cu = np.concatenate([[0], np.cumsum(lens)])
    B = len(lens)
    max_pages = 512 // P if kind == O.SLIDING else 1024 // P
    n_pages = B * max_pages + 2
    rng = np.random.default_rng(3)
    table = torch.from_numpy(rng.permutation(n_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)).cuda()
    dt = torch.uint8 if q8 else torch.bfloat16
    kp = torch.zeros(n_pages, 4, P, 256, dtype=dt, device="cuda")
    vp = torch.zeros_like(kp)
    ks = vs = None
    if q8:
        ks = torch.zeros(n_pages, 4, P, 8, dtype=torch.float16, device="cuda")
        vs = torch.zeros_like(ks)
    kv = sa.paged_kv(kp, vp, table, ks, vs)
    kb, kparts = _packed(7, 3, synth.ROLE_K, lens, pos0, 4, 256)
    vb, vparts = _packed(7, 3, synth.ROLE_V, lens, pos0, 4, 256)
    sa.spark_kv_append_varlen(kv, to_dev(kb), to_dev(vb), _i32(cu), max(lens), _i32(pos0),
                              sa.spark_layer_cfg_for_kind(kind))
    sa.spark_check()
    tab = table.cpu().numpy()
    host = {n: t.cpu() for n, t in (("k", kp), ("v", vp), ("ks", ks), ("vs", vs)) if t is not None}
    for b, n in enumerate(lens):
        last = {}
        for t in range(n):
            last[O.cache_slot(pos0[b] + t, kind)] = t
        for row, t in last.items():
            page, slot = tab[b, row // P], row % P
            for name, parts in (("k", kparts), ("v", vparts)):
                want = parts[b][t]
                if q8:
                    codes, scales = O.quantize_q8(f64(want).astype(np.float32))
                    assert np.array_equal(host[name][page, :, slot].numpy(), codes)
                    assert np.array_equal(host[name + "s"][page, :, slot].numpy().view(np.uint16),
                                          scales.view(np.uint16))
                else:
                    got = host[name][page, :, slot].view(torch.int16).numpy().view(np.uint16)
                    assert np.array_equal(got, want), (b, t, name)


def _prefill_varlen_case(kind, lens, pos0, P=64, seed=13, layer=0, fused_q=True, tight=False):
    """History 0..pos0[b]-1 appended (RoPE fused) into a zero-initialised paged pool; the chunk's k
    rotated by spark_rope_apply_varlen; q raw (RoPE at load) unless fused_q is False."""
    B = len(lens)
    cfg = sa.spark_layer_cfg_for_kind(kind)
    sliding = kind == O.SLIDING
    cu = np.concatenate([[0], np.cumsum(lens)])
    # tight: the table ends with the last page any position needs (a history tile may reach past it)
    max_pages = 512 // P if sliding else -(-(max(p + n for p, n in zip(pos0, lens)) + (0 if tight else 1)) // P)
    n_pages = B * max_pages + 3
    rng = np.random.default_rng(5)
    table = torch.from_numpy(rng.permutation(n_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)).cuda()
    kp = torch.zeros(n_pages, 4, P, 256, dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    kv = sa.paged_kv(kp, vp, table)
    hist = None
    if max(pos0) > 0:
        hl = list(pos0)
        hk, hkp = _packed(seed, layer, synth.ROLE_K, hl, [0] * B, 4, 256)
        hv, hvp = _packed(seed, layer, synth.ROLE_V, hl, [0] * B, 4, 256)
        hcu = np.concatenate([[0], np.cumsum(hl)])
        sa.spark_kv_append_varlen(kv, to_dev(hk), to_dev(hv), _i32(hcu), max(hl), _i32([0] * B), cfg,
                                  flags=sa.SPARK_ROPE_FUSED)
        hist = kv
    qb, qparts = _packed(seed, layer, synth.ROLE_Q, lens, pos0, 16, 256)
    kb, kparts = _packed(seed, layer, synth.ROLE_K, lens, pos0, 4, 256)
    vb, vparts = _packed(seed, layer, synth.ROLE_V, lens, pos0, 4, 256)
    gb, gparts = _packed(seed, layer, synth.ROLE_GATE, lens, pos0, 16, 1)
    total = int(cu[-1])
    q, k = to_dev(qb), to_dev(kb)
    cu_d, p0_d = _i32(cu), _i32(pos0)
    if not fused_q:
        sa.spark_rope_apply_varlen(q, cu_d, max(lens), p0_d, cfg)
    sa.spark_rope_apply_varlen(k, cu_d, max(lens), p0_d, cfg)
    out = torch.full((total, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.spark_attn_prefill_varlen(out, q, k, to_dev(vb), to_dev(gb), cu_d, max(lens), p0_d, hist, cfg,
                                 flags=sa.SPARK_ROPE_FUSED if fused_q else 0)
    sa.spark_check()
    got = dev_to_f64(out)
    for b, n in enumerate(lens):
        if n == 0:
            continue
        p0 = pos0[b]
        hp = np.arange(max(0, p0 - 511) if sliding else 0, p0)
        hist_k = hist_v = None
        if len(hp):
            raw_k = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, np.broadcast_to(hp, (B, len(hp))))[b]
            hist_k = O.rope(f64(raw_k), hp, kind)
            hist_v = f64(synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256,
                                            np.broadcast_to(hp, (B, len(hp))))[b])
        ref = O.layer_prefill(f64(qparts[b]), f64(kparts[b]), f64(vparts[b]), f64(gparts[b]), p0 + np.arange(n),
                              kind, hist_k, hist_v, hp)
        assert_close(got[cu[b]:cu[b + 1]], ref, f"varlen prefill {KIND_NAME[kind]} b={b} len={n} pos0={p0}")
    return got


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("lens", [[1, 127, 128, 129, 300], [0, 640, 2]])
def test_prefill_varlen_no_history(kind, lens):
    _prefill_varlen_case(kind, lens, [0] * len(lens))


@pytest.mark.parametrize("kind,lens,pos0,P", [
    (O.FULL, [100, 257, 1], [333, 1000, 64], 64),
    (O.FULL, [128, 5, 300], [128, 7, 0], 128),
    (O.SLIDING, [300, 64, 1], [200, 700, 511], 64),
    (O.SLIDING, [700, 130], [100, 1500], 256),
])
def test_prefill_varlen_paged_history(kind, lens, pos0, P):
    _prefill_varlen_case(kind, lens, pos0, P=P)


def test_prefill_varlen_tight_block_table():
    """pos0 = 900 with 64-row pages and a 15-page table: the last history tile [896, 1024) reaches
    rows 960.. that no table entry covers (they are past the history and masked)."""
    _prefill_varlen_case(O.FULL, [1, 30], [900, 100], P=64, tight=True)


def test_prefill_varlen_unfused_q():
    _prefill_varlen_case(O.FULL, [200, 33], [70, 0], fused_q=False)


def test_prefill_varlen_rejects_q8_history():
    cfg = sa.spark_layer_cfg_for_kind(O.FULL)
    kp = torch.zeros(4, 4, 64, 256, dtype=torch.uint8, device="cuda")
    ks = torch.zeros(4, 4, 64, 8, dtype=torch.float16, device="cuda")
    kv = sa.paged_kv(kp, kp, _i32([0, 1, 2, 3]).view(1, 4), ks, ks)
    q = torch.zeros(10, 16, 256, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(10, 4, 256, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(10, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SparkError) as e:
        sa.spark_attn_prefill_varlen(q.clone(), q, k, k, g, _i32([0, 10]), 10, _i32([5]), kv, cfg)
    assert e.value.status == -2


@pytest.mark.parametrize("kind", [O.SLIDING, O.FULL])
def test_varlen_sequence_longer_than_max_seqlen_is_flagged(kind):
    """A ragged sequence longer than max_seqlen is a device-side argument error (SPARK_ERR_DEVICE_ARG)
    in RoPE (4 and 16 heads), the append (bf16 and 8-bit pools) and the prefill: that sequence is left
    as it was (its rows unrotated, no cache row, no output row), the others are processed."""
    cfg = sa.spark_layer_cfg_for_kind(kind)
    lens, pos0, max_seqlen = [5, 40, 7], [3, 0, 900], 20
    cu = np.concatenate([[0], np.cumsum(lens)])
    long_rows = slice(int(cu[1]), int(cu[2]))
    for H in (16, 4):
        bits, parts = _packed(5, 0, synth.ROLE_Q, lens, pos0, H, 256)
        x = to_dev(bits)
        before = x.clone()
        sa.spark_rope_apply_varlen(x, _i32(cu), max_seqlen, _i32(pos0), cfg)
        with pytest.raises(sa.SparkError) as e:
            sa.spark_check()
        assert e.value.status == -5
        assert torch.equal(x[long_rows].view(torch.int16), before[long_rows].view(torch.int16))
        got = dev_to_f64(x)
        for b in (0, 2):
            ref = O.rope(f64(parts[b]), pos0[b] + np.arange(lens[b]), kind)
            assert_close(got[cu[b]:cu[b + 1]], ref, f"rope varlen H={H} b={b} beside a too-long sequence")
    P = 64
    max_pages = 512 // P if kind == O.SLIDING else 1024 // P
    n_pages = 3 * max_pages
    table = torch.arange(n_pages, dtype=torch.int32, device="cuda").view(3, max_pages)
    kb, kparts = _packed(7, 3, synth.ROLE_K, lens, pos0, 4, 256)
    vb, _ = _packed(7, 3, synth.ROLE_V, lens, pos0, 4, 256)
    for q8 in (False, True):
        dt = torch.uint8 if q8 else torch.bfloat16
        kp = torch.zeros(n_pages, 4, P, 256, dtype=dt, device="cuda")
        vp = torch.zeros_like(kp)
        ks = vs = None
        if q8:
            ks = torch.zeros(n_pages, 4, P, 8, dtype=torch.float16, device="cuda")
            vs = torch.zeros_like(ks)
        kv = sa.paged_kv(kp, vp, table, ks, vs)
        sa.spark_kv_append_varlen(kv, to_dev(kb), to_dev(vb), _i32(cu), max_seqlen, _i32(pos0), cfg)
        with pytest.raises(sa.SparkError) as e:
            sa.spark_check()
        assert e.value.status == -5
        assert not kp[max_pages:2 * max_pages].any()          # sequence 1's pages: nothing written
        row = O.cache_slot(pos0[0], kind)                      # sequence 0's first token was written
        if q8:
            codes, _ = O.quantize_q8(f64(kparts[0][0]).astype(np.float32))
            assert np.array_equal(kp[row // P, :, row % P].cpu().numpy(), codes)
        else:
            got = kp[row // P, :, row % P].view(torch.int16).cpu().numpy().view(np.uint16)
            assert np.array_equal(got, kparts[0][0])
    # the prefill (no history): the too-long sequence's output rows are not written
    total = int(cu[-1])
    qb, _ = _packed(9, 0, synth.ROLE_Q, lens, pos0, 16, 256)
    gb, _ = _packed(9, 0, synth.ROLE_GATE, lens, pos0, 16, 1)
    out = torch.full((total, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    k = to_dev(kb)
    sa.spark_rope_apply_varlen(k, _i32(cu), max(lens), _i32(pos0), cfg)
    sa.spark_attn_prefill_varlen(out, to_dev(qb), k, to_dev(vb), to_dev(gb), _i32(cu), max_seqlen, _i32(pos0), None,
                                 cfg)
    with pytest.raises(sa.SparkError) as e:
        sa.spark_check()
    assert e.value.status == -5
    assert torch.isnan(out[long_rows].float()).all()
    assert torch.isfinite(out[:int(cu[1])].float()).all() and torch.isfinite(out[int(cu[2]):].float()).all()
