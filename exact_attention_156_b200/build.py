"""Build the sm_100a shared libraries in-tree with nvcc.

  libattn156.so       - the product: the C ABI of include/attn.h
  libattn156_diag.so  - test-only diagnostics of the tcgen05 / TMA building blocks

Run ``python -m exact_attention_156_b200.build`` (or call ``build()``).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
         "-Xcompiler", "-fvisibility=hidden", "-Xptxas", "-v"]

TARGETS = {
    "libattn156.so": ["api.cu"],
    "libattn156_diag.so": ["diag.cu"],
}


def nvcc_path() -> str:
    p = shutil.which("nvcc")
    if p:
        return p
    cand = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(cand):
        return cand
    raise RuntimeError("nvcc not found")


def _needs_build(out: str, srcs) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(ROOT, "include", "attn.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose: bool = False, log_path: str | None = None) -> dict:
    """Compile every library; returns {name: ptxas log}."""
    logs = {}
    for name, srcs in TARGETS.items():
        out = os.path.join(PKG, name)
        if not force and not _needs_build(out, srcs):
            continue
        cmd = [nvcc_path(), *ARCH, *FLAGS, "-I", os.path.join(ROOT, "include"),
               *[os.path.join(CSRC, s) for s in srcs], "-o", out + ".tmp"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {name}:\n{r.stdout}\n{r.stderr}")
        os.replace(out + ".tmp", out)
        logs[name] = r.stderr
        if verbose:
            print(r.stderr, file=sys.stderr)
    if log_path and logs:
        with open(log_path, "w") as f:
            for k, v in logs.items():
                f.write(f"== {k}\n{v}\n")
    return logs


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
