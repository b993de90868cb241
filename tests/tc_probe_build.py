"""Build tests/libtc_probe.so (test harness for the sm_100a primitives)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "tc_probe.cu")
LIB = os.path.join(HERE, "libtc_probe.so")
DEPS = [SRC, os.path.join(os.path.dirname(HERE), "loss_closed_form_b200", "csrc", "tc_ptx.cuh"),
        os.path.join(os.path.dirname(HERE), "loss_closed_form_b200", "csrc", "common.cuh")]


def build(force=False):
    if not force and os.path.exists(LIB) and all(
            os.path.getmtime(d) <= os.path.getmtime(LIB) for d in DEPS):
        return LIB
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-lineinfo",
                    "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-o", LIB + ".tmp", SRC],
                   check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
