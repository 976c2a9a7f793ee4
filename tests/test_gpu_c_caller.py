"""The hot path driven from C with no Python in the process: tests/c/abi_gpu.c, compiled with gcc
against include/spark_attn.h and linked to libspark_attn.so and the CUDA runtime, runs RoPE, the
prefill, the append and a decode step for both layer kinds and checks the closed form that v = 1
and a gate logit of 0 give 0.5 in every output element."""
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_caller_runs_the_hot_path(tmp_path, cuda_device):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    import __graft_entry__
    __graft_entry__.build()
    import full_gqa_attention_spark2_b200 as sa
    lib_dir = os.path.dirname(sa.lib_path())
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = str(tmp_path / "abi_gpu")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "abi_gpu.c"),
                    "-L", lib_dir, "-lspark_attn", "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm",
                    f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", exe], check=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "c caller ok" in run.stdout
    assert run.stdout.count(" 0 off") == 4, run.stdout
