"""Build the host and device input generators in-tree (synth/_lib/)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "_lib")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale(out, srcs):
    return not os.path.exists(out) or any(os.path.getmtime(s) > os.path.getmtime(out) for s in srcs)


def build(force: bool = False) -> None:
    os.makedirs(LIB, exist_ok=True)
    cpu_src = os.path.join(HERE, "synth_cpu.c")
    cpu_out = os.path.join(LIB, "libsynth_cpu.so")
    if force or _stale(cpu_out, [cpu_src]):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-o", cpu_out, cpu_src])
    gpu_src = os.path.join(HERE, "synth_gpu.cu")
    gpu_out = os.path.join(LIB, "libsynth_gpu.so")
    if force or _stale(gpu_out, [gpu_src]):
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-std=c++17",
                               "-o", gpu_out, gpu_src])


if __name__ == "__main__":
    build(force=True)
