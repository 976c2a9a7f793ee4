"""Build the CUDA shared libraries in-tree with nvcc for sm_100a."""
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _newer(target, sources):
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(s) <= t for s in sources)


def _compile(src, out, deps, force):
    if not force and _newer(out, deps):
        return out
    cmd = [_nvcc(), *NVCC_FLAGS, src, "-o", out]
    subprocess.run(cmd, check=True)
    return out


def build_library(force=False):
    csrc = os.path.join(PKG, "csrc")
    deps = [os.path.join(csrc, f) for f in os.listdir(csrc)] + [os.path.join(ROOT, "include", "spark_attn.h")]
    return _compile(os.path.join(csrc, "spark_attn.cu"), os.path.join(PKG, "libspark_attn.so"), deps, force)


def build_synth(force=False):
    src = os.path.join(ROOT, "synth", "synth.cu")
    return _compile(src, os.path.join(ROOT, "synth", "libspark_synth.so"), [src], force)


def build_all(force=False):
    return build_library(force), build_synth(force)


if __name__ == "__main__":
    print(build_all(force=True))
