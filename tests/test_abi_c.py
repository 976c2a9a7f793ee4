"""The boundary as a C ABI: a C99 program (tests/c/abi_host.c) compiled with gcc against
include/spark_attn.h and linked to libspark_attn.so calls the host-side entry points without a GPU;
its answers are compared with the oracle's layer schedule and cache arithmetic."""
import os
import shutil
import subprocess

import pytest

from oracle import spark_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    import __graft_entry__
    __graft_entry__.build()
    import full_gqa_attention_spark2_b200 as sa
    lib_dir = os.path.dirname(sa.lib_path())
    exe = str(tmp_path_factory.mktemp("c") / "abi_host")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", lib_dir, "-lspark_attn",
                    f"-Wl,-rpath,{lib_dir}", "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return out.splitlines()


def test_layer_schedule_from_c(program):
    for layer in range(36):
        line = program[layer].split()
        kind, rot, theta, window = int(line[3]), int(line[5]), float(line[7]), int(line[9])
        p = O.layer_params(O.layer_kind(layer))
        assert kind == O.layer_kind(layer)
        assert rot == p["rot"] and theta == p["theta"]
        assert window == (512 if kind == O.SLIDING else 0)
        assert line[11:14] == ["16", "4", "dim"] and line[14] == "256"
    assert program[36] == "layer 36 status -1"


def test_sizes_and_checks_from_c(program):
    facts = dict(line.rsplit(" ", 1) for line in program[37:])
    assert int(facts["kv bytes full 1 token"]) == O.kv_bytes_per_token_full_layer()
    assert int(facts["kv bytes q8 full 1 token"]) == O.kv_bytes_per_token_full_layer() * O.q8_bytes_per_value() / 2
    assert int(facts["stack bytes 1 sequence 131072"]) == O.stack_kv_bytes(131072)
    assert int(facts["prefill q8 workspace sliding B=2"]) == 2 * 2 * 4 * 512 * 256 * 2
    assert int(facts["prefill q8 workspace sliding cap 600"]) == 0
    assert int(facts["prefill unknown flags status"]) == -1
    assert facts["last error set"] == "1"
