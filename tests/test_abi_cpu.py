"""The C-ABI library loads and exports every symbol the headers declare (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f), encoding="utf-8").read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(spark_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def _no_gpu():
    """The calls below pass placeholder pointers that only host-side checks may see: with a GPU
    present, a call that passes its checks would launch a kernel on them, so those tests skip."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("placeholder pointers: host-side checks are tested only where no GPU is present")


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    import full_gqa_attention_spark2_b200 as sa
    return ctypes.CDLL(sa.lib_path())


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_binding_covers_the_header():
    import full_gqa_attention_spark2_b200 as sa
    assert set(sa.exported_symbols()) <= set(_declared())


def test_host_helpers_without_a_gpu(lib):
    import full_gqa_attention_spark2_b200 as sa
    from oracle import spark_oracle as O
    for layer in range(36):
        c = sa.spark_layer_cfg_for_layer(layer)
        assert c.kind == O.layer_kind(layer)
        p = O.layer_params(c.kind)
        assert c.rot_dim == p["rot"] and c.theta == p["theta"]
        assert c.n_q == 16 and c.n_kv == 4 and c.head_dim == 256 and c.scale == 0.0625
    with pytest.raises(sa.SparkError):
        sa.spark_layer_cfg_for_layer(36)
    for ctx in (1, 511, 512, 4096, 131072, 1 << 20):
        assert sa.spark_stack_kv_bytes(1, ctx) == O.stack_kv_bytes(ctx)
    full = sa.spark_layer_cfg_for_kind(sa.SPARK_FULL)
    assert sa.spark_kv_cache_bytes(full, 1, 1) == O.kv_bytes_per_token_full_layer()
    assert sa.spark_kv_cache_bytes(full, 1, 1 << 20) == 4 * 2 ** 30


def test_calls_fail_loudly_without_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    import full_gqa_attention_spark2_b200 as sa
    cfg = sa.spark_layer_cfg_for_kind(sa.SPARK_SLIDING)
    x = torch.zeros(1, 1, 16, 256, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        sa.spark_rope_apply(x, torch.zeros(1, dtype=torch.int32), cfg)


def test_host_argument_checks_run_before_the_device(lib):
    """Host-side validation of the C entry points returns its status before any device call, so it
    is checked here without a GPU (fake, never dereferenced pointers)."""
    _no_gpu()
    import full_gqa_attention_spark2_b200 as sa
    L = sa._lib()
    full = sa.spark_layer_cfg_for_kind(sa.SPARK_FULL)
    sliding = sa.spark_layer_cfg_for_kind(sa.SPARK_SLIDING)
    fake = ctypes.c_void_p(1 << 20)          # 16-byte aligned, never dereferenced on these paths
    # context parallelism: full layers only; shards inside [0, 2^20)
    assert L.spark_kv_append_cp(fake, fake, 64, 0, fake, fake, 1, fake, ctypes.byref(sliding), 0, None) == -2
    assert L.spark_kv_append_cp(fake, fake, 64, -1, fake, fake, 1, fake, ctypes.byref(full), 0, None) == -1
    assert L.spark_kv_append_cp(fake, fake, 64, (1 << 20) - 10, fake, fake, 1, fake, ctypes.byref(full), 0,
                                None) == -1
    assert L.spark_attn_decode_cp_partial(fake, fake, fake, fake, 64, 0, 1, fake, ctypes.byref(sliding), fake, 1 << 20,
                                          0, None) == -2
    assert L.spark_attn_decode_cp_partial(None, fake, fake, fake, 64, 0, 1, fake, ctypes.byref(full), fake, 1 << 20,
                                          0, None) == -1
    assert L.spark_attn_decode_cp_merge(fake, fake, fake, 0, 1, None) == -1
    assert L.spark_attn_decode_cp_merge(fake, fake, fake, 2, 0, None) == -1
    assert L.spark_attn_decode_cp_merge(None, fake, fake, 2, 1, None) == -1
    assert L.spark_decode_cp_record_bytes(3) == 3 * 16 * 257 * 4
    assert L.spark_decode_cp_record_bytes(0) == 0
    # prefill: SPARK_APPEND_FUSED needs the caches; unknown flags are refused
    args = (fake, fake, fake, fake, fake, None, None, 0, 1, 128, 0, 0, 0, 0, fake, ctypes.byref(full))
    assert L.spark_attn_prefill(*args, sa.SPARK_APPEND_FUSED, None) == -1
    assert L.spark_attn_prefill(*args, 0x80, None) == -1
    assert "SPARK_APPEND_FUSED" in sa.spark_last_error() or "flags" in sa.spark_last_error()
    # prefill over an 8-bit history: workspace size, flags, pointers and cap before the device
    ws_need = 2 * 4 * 1000 * 256 * 2
    assert L.spark_prefill_q8_workspace_bytes(1, 1000, ctypes.byref(full)) == ws_need
    assert L.spark_prefill_q8_workspace_bytes(2, 512, ctypes.byref(sliding)) == 2 * 2 * 4 * 512 * 256 * 2
    assert L.spark_prefill_q8_workspace_bytes(1, 600, ctypes.byref(sliding)) == 0
    assert L.spark_prefill_q8_workspace_bytes(0, 512, ctypes.byref(sliding)) == 0
    q8 = (fake, fake, fake, fake, fake, fake, fake, fake, fake)
    tail = (1, 128, 0, 0, 0, 0, fake, ctypes.byref(full), fake)
    assert L.spark_attn_prefill_q8(*q8, 1000, *tail, ws_need - 16, 0, None) == -1
    assert "workspace" in sa.spark_last_error()
    assert L.spark_attn_prefill_q8(*q8, 1000, *tail, ws_need, 0x80, None) == -1
    assert L.spark_attn_prefill_q8(*q8[:5], None, *q8[6:], 1000, *tail, ws_need, 0, None) == -1
    assert L.spark_attn_prefill_q8(*q8, 600, 1, 128, 0, 0, 0, 0, fake, ctypes.byref(sliding), fake, 1 << 30, 0,
                                   None) == -1


def test_token_strides_are_checked_on_the_host(lib):
    """Element strides of the token tensors: 0, 0 is the dense layout; a view of a fused projection
    output [B, T, 24, 256] is accepted; rows that are not 16-byte multiples, heads that do not fit a
    token, or sequences that overlap are refused before any device call."""
    _no_gpu()
    import full_gqa_attention_spark2_b200 as sa
    L = sa._lib()
    full = ctypes.byref(sa.spark_layer_cfg_for_kind(sa.SPARK_FULL))
    fake = ctypes.c_void_p(1 << 20)
    B, T = 2, 100
    bad_q = [(T * 4096, 4100), (T * 4096, 2048), (99 * 4096, 4096), (T * 4096 + 4, 4096)]
    for sB, sT in bad_q:
        assert L.spark_rope_apply(fake, B, T, 16, sB, sT, fake, full, None) == -1, (sB, sT)
        assert "strides" in sa.spark_last_error()
        assert L.spark_attn_prefill(fake, fake, fake, fake, fake, None, None, 0, B, T, sB, sT, 0, 0, fake, full, 0,
                                    None) == -1, (sB, sT)
    for sB, sT in [(T * 1024, 1028), (T * 1024, 512), (50 * 1024, 1024)]:
        assert L.spark_kv_append(fake, fake, 4096, fake, fake, B, T, sB, sT, fake, full, 0, None) == -1, (sB, sT)
        assert L.spark_attn_prefill(fake, fake, fake, fake, fake, None, None, 0, B, T, 0, 0, sB, sT, fake, full, 0,
                                    None) == -1, (sB, sT)
    # decode: q's sequence stride must hold a token's 16 heads and keep 16-byte rows
    for q_sB in (4000, 4100):
        assert L.spark_attn_decode(fake, fake, q_sB, fake, fake, fake, 64, B, fake, full, fake, 1 << 30, 0,
                                   None) == -1, q_sB
        assert L.spark_attn_decode_fused(fake, fake, q_sB, fake, fake, 0, fake, fake, fake, 64, B, fake, full, fake,
                                         1 << 30, 0, None) == -1, q_sB
    assert L.spark_attn_decode_fused(fake, fake, 0, fake, fake, 1000, fake, fake, fake, 64, B, fake, full, fake,
                                     1 << 30, 0, None) == -1
    # views of one [B, T, 24, 256] projection output pass the host checks (and fail later, at the device)
    sB, sT = T * 24 * 256, 24 * 256
    assert L.spark_rope_apply(fake, B, T, 16, sB, sT, fake, full, None) not in (0, -1)
    assert L.spark_kv_append(fake, fake, 4096, fake, fake, B, T, sB, sT, fake, full, 0, None) not in (0, -1)
    assert L.spark_attn_prefill(fake, fake, fake, fake, fake, None, None, 0, B, T, sB, sT, sB, sT, fake, full, 0,
                                None) not in (0, -1)
    assert L.spark_attn_decode(fake, fake, 24 * 256, fake, fake, fake, 64, B, fake, full, fake, 1 << 30, 0,
                               None) not in (0, -1)
    assert L.spark_attn_decode_fused(fake, fake, 24 * 256, fake, fake, 24 * 256, fake, fake, fake, 64, B, fake, full,
                                     fake, 1 << 30, 0, None) not in (0, -1)


def test_static_decode_plan_fits_and_covers_every_tile(lib):
    """spark_attn_decode_static's plan: partials within the fixed array, splits that cover every
    64-key tile exactly once; fewer splits than the usual plan where that plan would not fit."""
    import full_gqa_attention_spark2_b200 as sa
    for kind in (sa.SPARK_SLIDING, sa.SPARK_FULL):
        cfg = sa.spark_layer_cfg_for_kind(kind)
        for B in (1, 3, 64, 300, 600, 1016):
            for cap in ((512,) if kind == sa.SPARK_SLIDING else (1, 100, 8192, 16384, 131072, 1 << 20)):
                ns, tps, nbytes = sa.spark_decode_static_plan(B, cap, cfg, 148)
                tiles = -(-min(cap, 512 if kind == sa.SPARK_SLIDING else cap) // 64)
                assert 0 < nbytes <= sa.SPARK_STATIC_SCRATCH_BYTES, (kind, B, cap)
                assert nbytes == B * 16 * ns * 258 * 4
                assert (ns - 1) * tps < tiles <= ns * tps, (kind, B, cap, ns, tps)
                if sa.spark_decode_workspace_bytes(B, cap, cfg) <= sa.SPARK_STATIC_SCRATCH_BYTES:
                    assert nbytes == sa.spark_decode_workspace_bytes(B, cap, cfg)      # the usual plan
    full = sa.spark_layer_cfg_for_kind(sa.SPARK_FULL)
    assert sa.spark_decode_workspace_bytes(300, 16384, full) > sa.SPARK_STATIC_SCRATCH_BYTES
    assert sa.spark_decode_static_plan(1017, 512, full, 148)[2] == 0
