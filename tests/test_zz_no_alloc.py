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
from tests.helpers import assert_close, dev_to_f64, tid, to_dev

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
    for call in range(2):
        out = torch.full((B, 16, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
        sa.spark_attn_decode_static(out, q, g, kc, vc, pos, cfg, flags=sa.SPARK_ROPE_FUSED)
        sa.spark_check()
        assert_close(dev_to_f64(out), ref64, f"static-scratch decode, call {call + 1}")


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
