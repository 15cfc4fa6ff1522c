"""Build the in-tree shared libraries with nvcc for sm_100a (B200).

  libkv4.so     the INT4 KV cache library (C ABI in include/kv4.h)
  libkv4gen.so  the GPU twin of the seeded input generator (tests and benchmark only)

Run ``python -m int4_kv_cache_append_b200.build`` (or ``__graft_entry__.build()``).  Objects are
rebuilt only when a source or header is newer than the library.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
          "-Xptxas", "-v"]

LIBS = {
    "libkv4.so": ["kv4_api.cu", "kv4_append.cu", "kv4_decode.cu", "kv4_bf16.cu", "kv4_mixed.cu"],
    "libkv4gen.so": ["kv4gen.cu"],
}


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> dict[str, str]:
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "kv4.h")]
    out = {}
    for lib, srcs in LIBS.items():
        target = os.path.join(HERE, lib)
        src_paths = [os.path.join(CSRC, s) for s in srcs]
        if force or _stale(target, src_paths + headers):
            tmp = target + f".tmp{os.getpid()}"
            cmd = [NVCC, *ARCH, *COMMON, "-I", os.path.join(ROOT, "include"), "-o", tmp, *src_paths]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
                raise RuntimeError(f"nvcc failed for {lib}")
            if verbose:
                sys.stderr.write(r.stderr)
            os.replace(tmp, target)
        out[lib] = target
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
