"""Build libdg.so (the C ABI of include/dg.h) in-tree with nvcc for sm_100a.

Each .cu file is compiled to an object in parallel, then linked into one shared library with hidden
visibility except for the dg_* entry points.  ``python -m block_discrete_diffusion_b200.build
[--force] [--ptxas-v]``.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdg.so")
SOURCES = ["dg_api.cu", "gemm.cu", "attention.cu", "misc.cu", "sampler.cu", "sampler_noalloc.cu", "dequant.cu",
           "head_sampler.cu", "expert_fp8.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return files + [os.path.abspath(__file__)]


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(f) for f in _inputs())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    os.makedirs(BUILD, exist_ok=True)
    common = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
              "-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        common += ["-Xptxas", "-v"]

    def compile_one(src):
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        r = subprocess.run(common + ["-c", os.path.join(CSRC, src), "-o", obj], capture_output=True, text=True)
        return src, obj, r

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    errors = [(s, r) for s, _, r in results if r.returncode != 0]
    for s, _, r in results:
        if ptxas_verbose or r.returncode != 0:
            sys.stderr.write(f"== {s}\n{r.stdout}{r.stderr}")
    if errors:
        raise RuntimeError("nvcc failed for " + ", ".join(s for s, _ in errors))
    objs = [o for _, o, _ in results]
    # --no-undefined: a symbol one source declares and none defines fails here, not at load time
    subprocess.run([_nvcc(), *ARCH, "-shared", "-o", LIB + ".tmp", *objs, "-lcudart_static", "-ldl", "-lrt",
                    "-lpthread", "-Xlinker", "--no-undefined"], check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--ptxas-v" in sys.argv))
