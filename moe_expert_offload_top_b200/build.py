"""Builds libftmoe.so (the C-ABI library and its sm_100a kernels) in this directory.

    python moe_expert_offload_top_b200/build.py   (by path: importing the package needs the built library)

nvcc compiles each CUDA source for sm_100a only (-gencode arch=compute_100a,
code=sm_100a) with the CUDA runtime linked statically, in parallel, then links
one shared library next to this file.
"""
import concurrent.futures
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libftmoe.so")
BUILD = os.path.join(ROOT, "_build")
SOURCES = ["api.cu", "router.cu", "permute.cu", "expert_decode.cu", "grouped_gemm_sm100.cu", "noalloc.cu",
           "ffn_fused_f32.cu", "ffn_fused_bf16.cu", "ffn_fused_int4.cu", "ffn_fused_nvfp4.cu", "gemv_int4_mma.cu",
           "gemv_nvfp4_mma.cu", "gemv_bf16_mma.cu"]
HEADERS = ["common.cuh", "kernels.hpp", "cache.hpp", "sm100_sync.cuh", "decode_gemv.cuh", "ffn_fused.cuh",
           "gemv_ring.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-I" + os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "ftmoe.h")]
    objs, jobs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + hdrs):
            jobs.append([NVCC, *FLAGS, "-c", s, "-o", o])
    if jobs:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            for cmd, res in zip(jobs, ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs)):
                if res.returncode != 0:
                    raise RuntimeError("nvcc failed: %s\n%s%s" % (" ".join(cmd), res.stdout, res.stderr))
                if verbose:
                    sys.stdout.write(res.stdout + res.stderr)
    if force or jobs or _stale(LIB, objs):
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
               "-Xcompiler", "-fPIC"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("link failed: %s\n%s" % (res.stdout, res.stderr))
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
