"""Build libsplitkv_attn.so in-tree with nvcc for sm_100a (B200).

The library links the CUDA runtime statically and resolves the driver's
tensor-map encoder at run time, so it loads on a machine without a GPU
(every entry point then reports SK_ERR_CUDA / SK_ERR_UNSUPPORTED).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_NAME = "libsplitkv_attn.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
SOURCES = [os.path.join(HERE, "csrc", "splitkv_attn.cu")]
DEPS = SOURCES + [
    os.path.join(HERE, "csrc", f)
    for f in ("ptx.cuh", "attn_common.cuh", "attn_fwd_persistent.cuh", "qk_norm_rope.cuh", "shard_copy.cuh")
] + [os.path.join(ROOT, "include", "splitkv_attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(d) <= t for d in DEPS)


BINDING_SRC = os.path.join(HERE, "csrc", "binding.cpp")
EXT_DIR = os.path.join(HERE, "_build", "skfast")
EXT_NAME = "skfast"


def build_binding(verbose: bool = False):
    """Compile (or load, when up to date) the compiled argument-marshalling
    module for attn_fwd_split_kv, in-tree under _build/skfast; returns it."""
    from torch.utils.cpp_extension import load

    os.makedirs(EXT_DIR, exist_ok=True)
    return load(name=EXT_NAME, sources=[BINDING_SRC], build_directory=EXT_DIR,
                extra_cflags=["-O2", "-I" + os.path.join(ROOT, "include")], with_cuda=True, verbose=verbose)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp%d" % os.getpid()
    cmd = [nvcc()] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose_ptxas else []) + [
        "-o", tmp] + SOURCES + ["-lrt", "-lpthread", "-ldl"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
    print(build_binding().__file__)
