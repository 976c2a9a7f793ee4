"""Failure detection without a GPU fault.

Every device-side wait of the library is bounded.  A child process runs the
decode and prefill kernels with the wait limit set to 1 ns
(SPARK_WAIT_TIMEOUT_NS), so waits that are not satisfied at once run out: the
kernels must return (no hang), spark_check() must report SPARK_ERR_TIMEOUT,
and the parent's own calls afterwards must still be correct.  Nothing here
traps, faults or hangs a GPU.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import full_gqa_attention_spark2_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys, torch
sys.path.insert(0, %r)
import bench, synth
import full_gqa_attention_spark2_b200 as sa
dev = torch.device("cuda")
res = {}
layers = bench.decode_layers(torch, sa, synth, dev, 16, 8192, (3,))
L = layers[0]
pos = torch.full((16,), 8192, dtype=torch.int32, device=dev)
ws = torch.empty(sa.spark_decode_workspace_bytes(16, L["cap"], L["cfg"]), dtype=torch.uint8, device=dev)
bench.decode_step(sa, layers, pos, ws)
try:
    sa.spark_check(); res["decode"] = 0
except sa.SparkError as e:
    res["decode"] = e.status
cfg = sa.spark_layer_cfg_for_kind(sa.SPARK_FULL)
q = torch.randn(1, 2048, 16, 256, device=dev).to(torch.bfloat16)
k = torch.randn(1, 2048, 4, 256, device=dev).to(torch.bfloat16)
g = torch.zeros(1, 2048, 16, device=dev).to(torch.bfloat16)
out = torch.empty_like(q)
p0 = torch.zeros(1, dtype=torch.int32, device=dev)
sa.spark_attn_prefill(out, q, k, k, g, None, None, p0, cfg)
try:
    sa.spark_check(); res["prefill"] = 0
except sa.SparkError as e:
    res["prefill"] = e.status
print("RESULT " + json.dumps(res))
"""


@pytest.mark.gpu
def test_a_wait_that_nothing_completes_times_out(cuda_device):
    import time
    sa.spark_check()
    t0 = time.perf_counter()
    sa.spark_selftest_wait_timeout(50_000_000)          # 50 ms
    with pytest.raises(sa.SparkError) as e:
        sa.spark_check()
    assert e.value.status == -4
    assert 0.04 < time.perf_counter() - t0 < 5.0
    sa.spark_check()                                     # the word was cleared; the context is usable
    from tests.test_gpu_kernels import _decode_case
    from tests.helpers import assert_close
    from oracle import spark_oracle as O
    got, ref = _decode_case(O.SLIDING, 2, [700, 700])
    assert_close(got, ref, "decode after a timed-out wait")


@pytest.mark.gpu
def test_expired_waits_report_timeout_and_return(cuda_device):
    env = dict(os.environ, SPARK_WAIT_TIMEOUT_NS="1")
    r = subprocess.run([sys.executable, "-c", CHILD % ROOT], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    assert res["decode"] == -4 and res["prefill"] == -4, res
    # this process (normal limit) is unaffected
    from tests.test_gpu_kernels import _decode_case
    from tests.helpers import assert_close
    from oracle import spark_oracle as O
    got, ref = _decode_case(O.FULL, 2, [300, 1000])
    assert_close(got, ref, "decode after a timed-out child")


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(sa, "_LIB", None)
    monkeypatch.setattr(sa, "lib_path", lambda: str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        sa.spark_version()
