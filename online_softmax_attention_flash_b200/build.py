"""Build libattn_b200.so in-tree with nvcc for sm_100a.

    python -m online_softmax_attention_flash_b200.build [--verbose-ptxas]

The library is one CUDA translation unit (csrc/attn_lib.cu) linked against the
static CUDA runtime; it needs no GPU to build.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libattn_b200.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
_NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
               "-Xcompiler", "-fvisibility=hidden"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh")))


def _strip_comments(text: str) -> str:
    """C / C++ source without its comments and blank lines (string literals kept as they are)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


# The files each kernel's machine code and launch configuration come from (besides the
# shared PTX / tensor-map / status headers and this file's compiler flags).
KERNEL_SOURCES = {
    "encoder_fwd_kernel": ("encoder.cuh", "attn_lib.cu"),   # launch set-up lives in attn_lib.cu
    "encoder_1q_kernel": ("encoder1q.cuh", "attn_lib.cu"),
    "decode_stream_kernel": ("decode.cuh",),
    "decode_stream_mma_kernel": ("decode_mma.cuh", "decode.cuh"),
    "paged_history_kernel": ("paged.cuh",),
    "rope_qk_kernel": ("rope.cuh",),
    "proj_gemm_kernel": ("proj.cuh", "attn_lib.cu"),
}
_COMMON_SOURCES = ("ptx.cuh", "tmap.cuh", "status.cuh")


def source_digest(kernel: str = None) -> str:
    """sha256 over source files with comments removed: it changes exactly when the code
    a build comes from changes. With `kernel` (a key of KERNEL_SOURCES) only the files
    that kernel is built and launched from count, plus the compiler flags; without it,
    every CUDA source and the header."""
    import hashlib
    h = hashlib.sha256()
    if kernel is None:
        paths = sources() + [os.path.join(INCLUDE, "attn.h")]
    else:
        paths = [os.path.join(CSRC, f) for f in KERNEL_SOURCES[kernel] + _COMMON_SOURCES]
        h.update(" ".join(ARCH_FLAGS + _NVCC_FLAGS).encode())
    for path in paths:
        h.update(os.path.basename(path).encode())
        with open(path, encoding="utf-8") as f:
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    deps = sources() + [os.path.join(INCLUDE, "attn.h"), os.path.abspath(__file__)]
    return all(os.path.getmtime(p) <= t for p in deps)


def build(force: bool = False, verbose_ptxas: bool = False, out: str = LIB_PATH,
          extra_flags=None) -> str:
    if not force and out == LIB_PATH and up_to_date():
        return out
    cmd = [nvcc_path(), *ARCH_FLAGS, *_NVCC_FLAGS,
           "-I", INCLUDE, "-I", CSRC,
           "-o", out, os.path.join(CSRC, "attn_lib.cu")]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    if extra_flags:
        cmd[1:1] = list(extra_flags)
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB_PATH)
