"""Build tests/c_abi/attend_loop.c (a C program that drives cvq_attend with no Python in the
loop) against libcvq.so and the CUDA runtime; returns the executable's path."""
import os
import shutil
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
PKG = os.path.join(ROOT, "compressed_attention_cvq_b200")


def cuda_home() -> str:
    for cand in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if cand and os.path.exists(os.path.join(cand, "include", "cuda_runtime.h")):
            return cand
    nvcc = shutil.which("nvcc")
    if nvcc:
        return os.path.dirname(os.path.dirname(os.path.realpath(nvcc)))
    raise RuntimeError("CUDA toolkit not found")


def build(out_path: str) -> str:
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        raise RuntimeError("no C compiler")
    cuda = cuda_home()
    src = os.path.join(ROOT, "tests", "c_abi", "attend_loop.c")
    subprocess.run([cc, "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"), src,
                    "-o", out_path, "-L", PKG, "-lcvq", "-L", os.path.join(cuda, "lib64"),
                    "-lcudart", f"-Wl,-rpath,{PKG}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}"],
                   check=True)
    return out_path
