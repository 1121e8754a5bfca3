"""Build the conversion probe used by tests/test_gpu_conversions.py (nvcc, sm_100a)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
SRC = os.path.join(HERE, "cvt_probe.cu")
LIB = os.path.join(HERE, "libcvtprobe.so")
DEPS = [SRC, os.path.join(ROOT, "fp4_fake_quant_b200", "csrc", "qf_device.cuh")]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and all(os.path.getmtime(d) <= os.path.getmtime(LIB) for d in DEPS)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-fmad=false", "-Xcompiler", "-fPIC", "-shared",
                    "-I", os.path.join(ROOT, "fp4_fake_quant_b200", "csrc"),
                    "-I", os.path.join(ROOT, "include"), "-o", tmp, SRC], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
