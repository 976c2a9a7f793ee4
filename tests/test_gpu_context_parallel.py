"""GPU parity of context-parallel decode through the C ABI, G ranks emulated in one process.

Each emulated rank owns a shard of a full layer's cache (positions key_off .. key_off + rows - 1); the ranks'
calls are independent launches (nothing waits on another rank), their records are stacked in rank order as
an all-gather lays them out, and the merge is compared with the oracle's decode over the whole cache at
|err| <= 2e-2 + 2e-2 |ref|.  The sharded appends are checked bit-exactly against the unsharded append.
"""
import numpy as np
import pytest
import torch

import full_gqa_attention_spark2_b200 as sa
import synth
from full_gqa_attention_spark2_b200.context_parallel import shard_of
from oracle import spark_oracle as O
from tests.helpers import assert_close, dev_to_f64, f64, tid, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import __graft_entry__
    __graft_entry__.build()
    sa._lib()
    yield


def _cp_case(G, p_list, total, seed=17, layer=3):
    """Returns (merged out, oracle reference, sharded caches == unsharded cache after the append)."""
    B = len(p_list)
    cfg = sa.spark_layer_cfg_for_kind(O.FULL)
    n_hist = max(p_list)
    kc = torch.empty(B, 4, total, 256, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    synth.fill_cache(kc, seed, tid(layer, synth.ROLE_K), n_hist, False)
    synth.fill_cache(vc, seed, tid(layer, synth.ROLE_V), n_hist, False)
    pnew = np.array(p_list)[:, None]
    qb = synth.token_tensor(seed, tid(layer, synth.ROLE_Q), B, 16, 256, pnew)[:, 0]
    kb = synth.token_tensor(seed, tid(layer, synth.ROLE_K), B, 4, 256, pnew)[:, 0]
    vb = synth.token_tensor(seed, tid(layer, synth.ROLE_V), B, 4, 256, pnew)[:, 0]
    gb = synth.token_tensor(seed, tid(layer, synth.ROLE_GATE), B, 16, 1, pnew)[:, 0]
    pos = torch.tensor(p_list, dtype=torch.int32, device="cuda")
    q, k, v, g = to_dev(qb), to_dev(kb), to_dev(vb), to_dev(gb)
    shards = []
    for r in range(G):
        lo, n = shard_of(r, G, total)
        shards.append((lo, kc[:, :, lo:lo + n].clone(), vc[:, :, lo:lo + n].clone()))
    # reference append into the whole cache, sharded appends into every rank's shard
    sa.spark_kv_append(kc, vc, k.view(B, 1, 4, 256), v.view(B, 1, 4, 256), pos, cfg, flags=sa.SPARK_ROPE_FUSED)
    for lo, ks, vs in shards:
        sa.spark_kv_append_cp(ks, vs, lo, k, v, pos, cfg, flags=sa.SPARK_ROPE_FUSED)
    same = (torch.equal(torch.cat([s[1] for s in shards], 2).view(torch.int16), kc.view(torch.int16)) and
            torch.equal(torch.cat([s[2] for s in shards], 2).view(torch.int16), vc.view(torch.int16)))
    n_rec = sa.spark_decode_cp_record_bytes(B) // 4
    records = torch.full((G, n_rec), float("nan"), dtype=torch.float32, device="cuda")
    for r, (lo, ks, vs) in enumerate(shards):
        ws = torch.empty(sa.spark_decode_workspace_bytes(B, ks.shape[2], cfg), dtype=torch.uint8, device="cuda")
        sa.spark_attn_decode_cp_partial(records[r], q, ks, vs, lo, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
    out = torch.full((B, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    sa.spark_attn_decode_cp_merge(out, g, records)
    sa.spark_check()
    refs = []
    for b, p in enumerate(p_list):
        hp = np.arange(p)
        hist_k = np.stack([f64(synth.head_slice(seed, tid(layer, synth.ROLE_K), b, j, 4, 256, hp)) for j in range(4)], 1)
        hist_v = np.stack([f64(synth.head_slice(seed, tid(layer, synth.ROLE_V), b, j, 4, 256, hp)) for j in range(4)], 1)
        refs.append(O.layer_decode(f64(qb[b]), f64(kb[b]), f64(vb[b]), f64(gb[b]), p, O.FULL, hist_k, hist_v, hp))
    return dev_to_f64(out), np.stack(refs), same, records


@pytest.mark.parametrize("G,p_list,total", [
    (1, [0, 5, 300], 400),
    (2, [0, 199, 200, 399], 400),           # rank 1 holds nothing of the first two; 200 is its first row
    (3, [133, 134, 266, 1000], 1001),       # shard boundaries and the last position
    (4, [4095, 4096, 5000, 8190], 8191),    # uneven shards, several splits per shard
])
def test_cp_decode_matches_oracle(G, p_list, total):
    got, ref, same, _ = _cp_case(G, p_list, total)
    assert same, "sharded appends differ from the unsharded append"
    assert_close(got, ref, f"cp decode G={G} p={p_list}")


def test_cp_record_of_a_rank_without_keys():
    """pos before the shard: the rank's log-sum-exp is -inf and its output 0, and the merge ignores it."""
    _, _, _, records = _cp_case(2, [10], 400)
    rec = records[1].cpu().numpy()
    lse = rec[16 * 256:]
    assert np.all(np.isneginf(lse)) and np.all(rec[:16 * 256] == 0)
    assert np.all(np.isfinite(records[0].cpu().numpy()))


def test_cp_rejects_sliding_layers_and_bad_shards():
    cfg_s = sa.spark_layer_cfg_for_kind(O.SLIDING)
    cfg_f = sa.spark_layer_cfg_for_kind(O.FULL)
    kc = torch.zeros(1, 4, 64, 256, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 4, 256, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(sa.SparkError) as e:
        sa.spark_kv_append_cp(kc, kc, 0, k, k, pos, cfg_s)
    assert e.value.status == -2
    with pytest.raises(sa.SparkError) as e:
        sa.spark_kv_append_cp(kc, kc, -1, k, k, pos, cfg_f)
    assert e.value.status == -1
    with pytest.raises(sa.SparkError) as e:
        sa.spark_kv_append_cp(kc, kc, (1 << 20) - 10, k, k, pos, cfg_f)
    assert e.value.status == -1
