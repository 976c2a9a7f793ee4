"""spark_attn_decode_static: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: hosts that plan all device
memory up front and forbid allocation later, hosts that only lend their
inputs and outputs, and code recording a CUDA graph (cudaMalloc cannot be
recorded).  This entry point keeps the split-KV partials in a fixed array of
the library's own device memory.  The test checks it, through the C ABI,
against spark_attn_decode with a caller workspace, on two calls in a row, with
the suite's tolerance.  The file is collected last so that a failure here does
not hide the other tests; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import full_gqa_attention_spark2_b200 as sa
import synth
from oracle import spark_oracle as O
from tests.helpers import assert_close, dev_to_f64, f64, tid, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import __graft_entry__
    __graft_entry__.build()
    sa._lib()
    yield


def _case(kind, B, p_list, seed):
    sliding = kind == sa.SPARK_SLIDING
    cap = 512 if sliding else max(p_list) + 3
    n_hist = p_list[0] if sliding else max(p_list)
    kc = torch.empty(B, 4, cap, 256, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    synth.fill_cache(kc, seed, tid(0, synth.ROLE_K), n_hist, sliding)
    synth.fill_cache(vc, seed, tid(0, synth.ROLE_V), n_hist, sliding)
    pnew = np.array(p_list)[:, None]
    q = to_dev(synth.token_tensor(seed, tid(0, synth.ROLE_Q), B, 16, 256, pnew)[:, 0])
    kn = to_dev(synth.token_tensor(seed, tid(0, synth.ROLE_K), B, 4, 256, pnew))
    vn = to_dev(synth.token_tensor(seed, tid(0, synth.ROLE_V), B, 4, 256, pnew))
    g = to_dev(synth.token_tensor(seed, tid(0, synth.ROLE_GATE), B, 16, 1, pnew)[:, 0])
    pos = torch.tensor(p_list, dtype=torch.int32, device="cuda")
    cfg = sa.spark_layer_cfg_for_kind(kind)
    sa.spark_kv_append(kc, vc, kn, vn, pos, cfg, flags=sa.SPARK_ROPE_FUSED)
    return q, g, kc, vc, pos, cfg


def _oracle_rows(kind, B, p_list, seed, check_b):
    """The oracle's output for sequences check_b of _case: cached keys 0..p-1 (taken as rotated, as
    the generator writes them), the new token's k rotated at p."""
    out = {}
    for b in check_b:
        p = p_list[b]
        hist = np.arange(max(0, p - 511) if kind == sa.SPARK_SLIDING else 0, p)
        qb = f64(synth.token_tensor(seed, tid(0, synth.ROLE_Q), B, 16, 256, np.full((B, 1), p))[b, 0])
        gb = f64(synth.token_tensor(seed, tid(0, synth.ROLE_GATE), B, 16, 1, np.full((B, 1), p))[b, 0])
        rows = np.zeros((16, 256))
        for grp in range(4):
            hs = slice(4 * grp, 4 * grp + 4)
            hk = f64(synth.head_slice(seed, tid(0, synth.ROLE_K), b, grp, 4, 256, hist))
            hv = f64(synth.head_slice(seed, tid(0, synth.ROLE_V), b, grp, 4, 256, hist))
            kn = f64(synth.head_slice(seed, tid(0, synth.ROLE_K), b, grp, 4, 256, np.array([p])))
            vn = f64(synth.head_slice(seed, tid(0, synth.ROLE_V), b, grp, 4, 256, np.array([p])))
            keys = np.concatenate([hk, O.rope(kn[:, None, :], np.array([p]), kind)[:, 0, :]])
            vals = np.concatenate([hv, vn])
            q = O.rope(qb[None, hs], np.array([p]), kind)
            rows[hs] = O.attention_group(q, keys, vals, gb[None, hs], np.array([p]), np.concatenate([hist, [p]]),
                                         kind)[0]
        out[b] = rows
    return out


@pytest.mark.parametrize("kind,B,p_list", [(sa.SPARK_FULL, 3, [100, 700, 2000]),
                                           (sa.SPARK_SLIDING, 2, [600, 600]),
                                           (sa.SPARK_FULL, 64, [32768] * 64)])
def test_static_decode_matches_the_workspace_decode_twice(kind, B, p_list):
    q, g, kc, vc, pos, cfg = _case(kind, B, p_list, seed=31)
    ref = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(sa.spark_decode_workspace_bytes(B, kc.shape[2], cfg), dtype=torch.uint8, device="cuda")
    sa.spark_attn_decode(ref, q, g, kc, vc, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
    sa.spark_check()
    ref64 = dev_to_f64(ref)
    check_b = sorted({0, B - 1})
    oracle = _oracle_rows(kind, B, p_list, 31, check_b)
    for call in range(2):
        out = torch.full((B, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
        sa.spark_attn_decode_static(out, q, g, kc, vc, pos, cfg, flags=sa.SPARK_ROPE_FUSED)
        sa.spark_check()
        got = dev_to_f64(out)
        assert_close(got, ref64, f"static-scratch decode, call {call + 1}")
        for b in check_b:
            assert_close(got[b], oracle[b], f"static-scratch decode against the oracle, b={b}, call {call + 1}")


def test_static_decode_with_fewer_splits_than_the_usual_plan():
    """A full layer at B=300 with a 16384-row cache (20 GB of K and V): the usual plan's partials
    would not fit the 16 MiB array, so the call runs fewer, longer splits.  Positions are mixed, so
    some sequences end in the first split and some span all of them."""
    B, cap = 300, 16384
    cfg = sa.spark_layer_cfg_for_kind(sa.SPARK_FULL)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ns, tps, nbytes = sa.spark_decode_static_plan(B, cap, cfg, sms)
    assert 0 < nbytes <= sa.SPARK_STATIC_SCRATCH_BYTES
    assert sa.spark_decode_workspace_bytes(B, cap, cfg) > sa.SPARK_STATIC_SCRATCH_BYTES   # the usual plan
    assert ns >= 2 and (ns - 1) * tps < cap // 64 <= ns * tps
    rng = np.random.default_rng(5)
    p_list = [cap - 2, cap - 2] + rng.integers(0, cap - 1, B - 2).tolist()
    q, g, kc, vc, pos, cfg = _case(sa.SPARK_FULL, B, p_list, seed=37)
    ref = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(sa.spark_decode_workspace_bytes(B, cap, cfg), dtype=torch.uint8, device="cuda")
    sa.spark_attn_decode(ref, q, g, kc, vc, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
    sa.spark_check()
    del ws
    ref64 = dev_to_f64(ref)
    check_b = [0, int(np.argmin(p_list)), B - 1]
    oracle = _oracle_rows(sa.SPARK_FULL, B, p_list, 37, check_b)
    for call in range(2):
        out = torch.full((B, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
        sa.spark_attn_decode_static(out, q, g, kc, vc, pos, cfg, flags=sa.SPARK_ROPE_FUSED)
        sa.spark_check()
        got = dev_to_f64(out)
        assert_close(got, ref64, f"static-scratch decode with fewer splits, call {call + 1}")
        for b in check_b:
            assert_close(got[b], oracle[b], f"fewer splits against the oracle, b={b}, call {call + 1}")
    del kc, vc
    torch.cuda.empty_cache()


def test_static_decode_rejects_batches_beyond_the_scratch():
    cfg = sa.spark_layer_cfg_for_kind(sa.SPARK_FULL)
    B = 1017
    kc = torch.zeros(B, 4, 8, 256, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(B, 16, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    with pytest.raises(sa.SparkError) as e:
        sa.spark_attn_decode_static(out, q, g, kc, kc, pos, cfg)
    assert e.value.status == -1 and "static scratch" in str(e.value)
