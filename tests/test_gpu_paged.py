"""GPU parity of the paged KV cache (pools of pages + per-sequence block tables), through the C ABI.

Appends into pages are checked bit for bit against a host model of the page
placement (bf16) or of the oracle's quantisation (8-bit).  Decode over pages
must give exactly the bits of decode over a dense cache with the same
contents and capacity (same split plan, same tiles), and match the oracle,
also when sequences share the pages of a common prefix, when the pool holds
NaN (or garbage codes) everywhere no token was written, and for sliding rings
spread over pages.  A page index outside the pool is a device-side argument
error that ends the call without a hang.
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


def _pos(vals):
    return torch.tensor(list(vals), dtype=torch.int32, device="cuda")


def _pools(n_pages, P, q8, poison=True):
    """Pools full of NaN (bf16) or garbage codes with NaN scales (8-bit): nothing unwritten is usable."""
    if q8:
        k = torch.full((n_pages, 4, P, 256), 255, dtype=torch.uint8, device="cuda")
        v = torch.full_like(k, 1)
        ks = torch.full((n_pages, 4, P, 8), float("nan") if poison else 0.0, dtype=torch.float16, device="cuda")
        vs = ks.clone()
        return k, v, ks, vs
    k = torch.full((n_pages, 4, P, 256), float("nan") if poison else 0.0, dtype=torch.bfloat16, device="cuda")
    return k, k.clone(), None, None


def _table(rows):
    return torch.tensor(rows, dtype=torch.int32, device="cuda")


def _kv(pools, table):
    k, v, ks, vs = pools
    return sa.paged_kv(k, v, table, ks, vs)


def _gather_rows(pool, table_row, P, rows):
    """Host model of page placement: pool rows of logical rows `rows` of one sequence -> [len, 4, ...]."""
    t = table_row.cpu().numpy()
    h = pool.cpu()
    return torch.stack([h[t[r // P], :, r % P] for r in rows]).numpy()


# ------------------------------------------------------------------ append ----

@pytest.mark.parametrize("kind,P,T,pos0_list", [(O.FULL, 128, 300, [0, 600]), (O.FULL, 64, 1, [1023, 5]),
                                                (O.SLIDING, 64, 700, [0, 0]), (O.SLIDING, 256, 100, [450, 450])])
def test_paged_append_bf16_bit_exact(kind, P, T, pos0_list):
    B = len(pos0_list)
    max_pages = 1024 // P if kind == O.FULL else 512 // P
    n_pages = B * max_pages + 3
    rng = np.random.default_rng(1)
    table = _table(rng.permutation(n_pages)[:B * max_pages].reshape(B, max_pages))
    pools = _pools(n_pages, P, False)
    kv = _kv(pools, table)
    pos = np.array([[p + t for t in range(T)] for p in pos0_list])
    kb = synth.token_tensor(3, tid(0, synth.ROLE_K), B, 4, 256, pos)
    vb = synth.token_tensor(3, tid(0, synth.ROLE_V), B, 4, 256, pos)
    cfg = sa.spark_layer_cfg_for_kind(kind)
    sa.spark_kv_append_paged(kv, to_dev(kb), to_dev(vb), _pos(pos0_list), cfg)
    sa.spark_check()
    for b in range(B):
        last = {}                                    # later tokens overwrite (ring)
        for t in range(T):
            last[O.cache_slot(pos[b, t], kind)] = t
        rows = sorted(last)
        ts = [last[r] for r in rows]
        got_k = _gather_rows(pools[0].view(torch.int16), table[b], P, rows).view(np.uint16)
        got_v = _gather_rows(pools[1].view(torch.int16), table[b], P, rows).view(np.uint16)
        np.testing.assert_array_equal(got_k, kb[b, ts])
        np.testing.assert_array_equal(got_v, vb[b, ts])


def test_paged_append_q8_bit_exact():
    B, P, T, kind = 2, 128, 333, O.FULL
    pos0_list = [10, 500]
    max_pages = 8
    n_pages = 17
    table = _table([[3, 0, 5, 7, 9, 11, 13, 15], [1, 2, 4, 6, 8, 10, 12, 14]])
    pools = _pools(n_pages, P, True)
    kv = _kv(pools, table)
    pos = np.array([[p + t for t in range(T)] for p in pos0_list])
    kb = synth.token_tensor(4, tid(3, synth.ROLE_K), B, 4, 256, pos)
    vb = synth.token_tensor(4, tid(3, synth.ROLE_V), B, 4, 256, pos)
    sa.spark_kv_append_paged(kv, to_dev(kb), to_dev(vb), _pos(pos0_list), sa.spark_layer_cfg_for_kind(kind))
    sa.spark_check()
    for b in range(B):
        rows = list(pos[b])
        for pool_c, pool_s, bits in ((pools[0], pools[2], kb), (pools[1], pools[3], vb)):
            codes, scales = O.quantize_q8(f64(bits[b]).astype(np.float32))
            np.testing.assert_array_equal(_gather_rows(pool_c, table[b], P, rows), codes)
            np.testing.assert_array_equal(_gather_rows(pool_s.view(torch.int16), table[b], P, rows).view(np.uint16),
                                          scales.view(np.uint16))


# ------------------------------------------------------------------ decode ----

def _decode_pair(kind, B, p_list, P, q8, seed=41, layer=0):
    """The same history in a dense cache (zeros elsewhere) and in shuffled pages of a NaN pool;
    returns (dense out, paged out, reference)."""
    sliding = kind == O.SLIDING
    max_pages = 512 // P if sliding else -(-(max(p_list) + 1) // P) + 1
    cap = 512 if sliding else max_pages * P
    n_pages = B * max_pages + 5
    rng = np.random.default_rng(7)
    table = _table(rng.permutation(n_pages)[:B * max_pages].reshape(B, max_pages))
    pools = _pools(n_pages, P, q8)
    kv = _kv(pools, table)
    cfg = sa.spark_layer_cfg_for_kind(kind)
    if q8:
        dk = torch.zeros(B, 4, cap, 256, dtype=torch.uint8, device="cuda")
        dks = torch.zeros(B, 4, cap, 8, dtype=torch.float16, device="cuda")
        dense = (dk, dks, dk.clone(), dks.clone())
    else:
        dk = torch.zeros(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
        dense = (dk, dk.clone())
    n_hist = max(p_list)
    hp = np.broadcast_to(np.arange(n_hist), (B, n_hist))
    kh = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, hp)
    vh = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, hp)
    pnew = np.array(p_list)[:, None]
    qb = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pnew)[:, 0]
    kb = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pnew)
    vb = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pnew)
    gb = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pnew)[:, 0]
    pos = _pos(p_list)
    dense_append = sa.spark_kv_append_q8 if q8 else sa.spark_kv_append
    # history 0..n_hist-1 for every sequence (rows past a shorter sequence's new token hold finite
    # history in both caches and are never visible), then the new token at p_b, RoPE fused
    if n_hist > 0:
        sa.spark_kv_append_paged(kv, to_dev(kh), to_dev(vh), _pos([0] * B), cfg)
        dense_append(*dense, to_dev(kh), to_dev(vh), _pos([0] * B), cfg)
    sa.spark_kv_append_paged(kv, to_dev(kb), to_dev(vb), pos, cfg, flags=sa.SPARK_ROPE_FUSED)
    dense_append(*dense, to_dev(kb), to_dev(vb), pos, cfg, flags=sa.SPARK_ROPE_FUSED)
    out_d = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    out_p = torch.empty_like(out_d)
    if q8:
        ws = torch.empty(sa.spark_decode_q8_workspace_bytes(B, cap, cfg), dtype=torch.uint8, device="cuda")
        sa.spark_attn_decode_q8(out_d, to_dev(qb), to_dev(gb), *dense, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
    else:
        ws = torch.empty(sa.spark_decode_workspace_bytes(B, cap, cfg), dtype=torch.uint8, device="cuda")
        sa.spark_attn_decode(out_d, to_dev(qb), to_dev(gb), *dense, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
    wsp = torch.empty(sa.spark_decode_paged_workspace_bytes(B, kv, cfg), dtype=torch.uint8, device="cuda")
    assert wsp.numel() == ws.numel()
    sa.spark_attn_decode_paged(out_p, to_dev(qb), to_dev(gb), kv, pos, cfg, wsp, flags=sa.SPARK_ROPE_FUSED)
    sa.spark_check()
    refs = []
    for b, p in enumerate(p_list):
        hpos = np.arange(max(0, p - 511) if sliding else 0, p)
        keys = np.concatenate([f64(kh[b, hpos]), O.rope(f64(kb[b]), np.array([p]), kind)])
        vals = np.concatenate([f64(vh[b, hpos]), f64(vb[b])])
        if q8:
            keys = O.dequantize_q8(*O.quantize_q8(keys.astype(np.float32)))
            vals = O.dequantize_q8(*O.quantize_q8(vals.astype(np.float32)))
        kpos = np.concatenate([hpos, [p]])
        qr = O.rope(f64(qb[b])[None], np.array([p]), kind)
        refs.append(np.concatenate([O.attention_group(qr[:, 4 * g:4 * g + 4], keys[:, g], vals[:, g],
                                                      f64(gb[b])[None, 4 * g:4 * g + 4], np.array([p]), kpos,
                                                      kind)[0] for g in range(4)]))
    return out_d, out_p, np.stack(refs)


@pytest.mark.parametrize("q8", [False, True])
@pytest.mark.parametrize("kind,P,p_list", [(O.FULL, 64, [5, 64, 65]), (O.FULL, 128, [127, 128, 3000]),
                                           (O.FULL, 512, [700, 1]), (O.SLIDING, 64, [200, 200]),
                                           (O.SLIDING, 128, [4097, 4097]), (O.SLIDING, 512, [511, 511])])
def test_paged_decode_matches_dense_and_oracle(kind, P, p_list, q8):
    out_d, out_p, ref = _decode_pair(kind, len(p_list), p_list, P, q8)
    assert torch.equal(out_d.view(torch.int16), out_p.view(torch.int16)), "paged and dense decode differ"
    assert_close(dev_to_f64(out_p), ref, f"paged decode {KIND_NAME[kind]} page {P} q8={q8} p={p_list}")


@pytest.mark.parametrize("q8", [False, True])
def test_paged_decode_shared_prefix(q8):
    """Sequence 0 owns positions 0..999; sequence 1 reads sequence 0's pages for 0..511 and its own
    for 512..800; sequence 2 shares 0..255 and owns 256..1500.  Shared pages are written once."""
    P, kind, seed, layer = 64, O.FULL, 9, 3
    cfg = sa.spark_layer_cfg_for_kind(kind)
    lens = [1000, 800, 1500]            # new token of sequence b at position lens[b]
    shared = [None, 512, 256]           # prefix length taken from sequence 0
    max_pages = 1501 // P + 2
    pages0 = list(range(0, max_pages))
    nxt = max_pages
    rows = [pages0]
    for b in (1, 2):
        own = list(range(nxt, nxt + max_pages))
        nxt += max_pages
        rows.append(pages0[:shared[b] // P] + own[shared[b] // P:])
    n_pages = nxt
    table = _table(rows)
    pools = _pools(n_pages, P, q8)
    kv_all = _kv(pools, table)
    tok = {}
    for role in (synth.ROLE_K, synth.ROLE_V):
        tok[role] = [synth.token_tensor(seed, tid(layer, role), 3, 4, 256, np.broadcast_to(np.arange(1501), (3, 1501)))[b]
                     for b in range(3)]
    # history: sequence 0 all of 0..999; sequences 1, 2 only past their shared prefix
    for b, lo in ((0, 0), (1, shared[1]), (2, shared[2])):
        hi = lens[b]
        kv_b = _kv(pools, table[b:b + 1])
        sa.spark_kv_append_paged(kv_b, to_dev(tok[synth.ROLE_K][b][None, lo:hi]),
                                 to_dev(tok[synth.ROLE_V][b][None, lo:hi]), _pos([lo]), cfg)
    pnew = np.array(lens)[:, None]
    qb = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), 3, 16, 256, pnew)[:, 0]
    gb = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), 3, 16, 1, pnew)[:, 0]
    kn = np.stack([tok[synth.ROLE_K][b][lens[b]] for b in range(3)])[:, None]
    vn = np.stack([tok[synth.ROLE_V][b][lens[b]] for b in range(3)])[:, None]
    pos = _pos(lens)
    sa.spark_kv_append_paged(kv_all, to_dev(kn), to_dev(vn), pos, cfg, flags=sa.SPARK_ROPE_FUSED)
    out = torch.empty(3, 16, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(sa.spark_decode_paged_workspace_bytes(3, kv_all, cfg), dtype=torch.uint8, device="cuda")
    sa.spark_attn_decode_paged(out, to_dev(qb), to_dev(gb), kv_all, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
    sa.spark_check()
    got = dev_to_f64(out)
    for b in range(3):
        src = [0 if (b > 0 and p < shared[b]) else b for p in range(lens[b])]
        keys = np.stack([f64(tok[synth.ROLE_K][s][p]) for p, s in enumerate(src)] +
                        [O.rope(f64(kn[b]), np.array([lens[b]]), kind)[0]])
        vals = np.stack([f64(tok[synth.ROLE_V][s][p]) for p, s in enumerate(src)] + [f64(vn[b, 0])])
        if q8:
            keys = O.dequantize_q8(*O.quantize_q8(keys.astype(np.float32)))
            vals = O.dequantize_q8(*O.quantize_q8(vals.astype(np.float32)))
        kpos = np.arange(lens[b] + 1)
        qr = O.rope(f64(qb[b])[None], np.array([lens[b]]), kind)
        ref = np.concatenate([O.attention_group(qr[:, 4 * g:4 * g + 4], keys[:, g], vals[:, g],
                                                f64(gb[b])[None, 4 * g:4 * g + 4], np.array([lens[b]]), kpos,
                                                kind)[0] for g in range(4)])
        assert_close(got[b], ref, f"shared-prefix decode q8={q8} sequence {b}")


def test_paged_bad_page_index_is_reported():
    P, kind = 64, O.FULL
    cfg = sa.spark_layer_cfg_for_kind(kind)
    pools = _pools(8, P, False, poison=False)
    table = _table([[0, 1, 2, 99]])            # page 99 is outside an 8-page pool
    kv = _kv(pools, table)
    k = torch.ones(1, 1, 4, 256, dtype=torch.bfloat16, device="cuda")
    sa.spark_kv_append_paged(kv, k, k, _pos([200]), cfg)          # row 200 -> logical page 3
    with pytest.raises(sa.SparkError) as e:
        sa.spark_check()
    assert e.value.status == -5
    q = torch.zeros(1, 16, 256, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(1, 16, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    ws = torch.empty(sa.spark_decode_paged_workspace_bytes(1, kv, cfg), dtype=torch.uint8, device="cuda")
    sa.spark_attn_decode_paged(out, q, g, kv, _pos([200]), cfg, ws)
    with pytest.raises(sa.SparkError) as e:
        sa.spark_check()
    assert e.value.status in (-5, -4)
    sa.spark_attn_decode_paged(out, q, g, kv, _pos([150]), cfg, ws)   # pages 0..2 only: fine
    sa.spark_check()


def test_paged_host_side_checks():
    cfg = sa.spark_layer_cfg_for_kind(O.SLIDING)
    pools = _pools(4, 64, False)
    kv = _kv(pools, _table([[0, 1, 2, 3]]))          # 4 pages of 64 = 256 rows: too few for a ring
    k = torch.ones(1, 1, 4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SparkError) as e:
        sa.spark_kv_append_paged(kv, k, k, _pos([0]), cfg)
    assert e.value.status == -1
    kv.page_size = 96                                 # not a power of two
    with pytest.raises(sa.SparkError):
        sa.spark_kv_append_paged(kv, k, k, _pos([0]), sa.spark_layer_cfg_for_kind(O.FULL))
