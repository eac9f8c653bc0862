"""Builds libltxattn.so in-tree with nvcc for sm_100a (no JIT cache, no torch extension)."""
from __future__ import annotations

import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libltxattn.so")
DEBUG_LIB = os.path.join(PKG, "libltxattn_debug.so")  # -DLTXATTN_DEBUG: workspace guard words
SOURCES = ["ltxattn.cu"]
DEPS = ["ltxattn.cu", "attn_fwd.cuh", "attn_fwd_pp.cuh", "attn_fwd_skv.cuh", "attn_fwd_pair.cuh",
        "attn_fwd_a2v.cuh", "qk_prologue.cuh",
        "na3d_fwd.cuh", "combine.cuh", "debug_guard.cuh", "sm100_ptx.cuh"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", "ltxattn.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile csrc/ltxattn.cu (+ headers) into joint_audio_video_flash_b200/libltxattn.so, or,
    with debug=True, the guard-word build libltxattn_debug.so (-DLTXATTN_DEBUG)."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *(["-DLTXATTN_DEBUG"] if debug else []), "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose=True))
