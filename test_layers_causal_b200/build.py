"""Builds libttt_la.so in-tree with nvcc for sm_100a (no JIT cache).

    python -m test_layers_causal_b200.build [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "ttt_la.cu")
OUT = os.path.join(HERE, "libttt_la.so")
DEBUG_OUT = os.path.join(HERE, "libttt_la_debug.so")  # -DTTT_LA_DEBUG: device-side bounds checks
DEPS = [os.path.join(HERE, "csrc", f) for f in sorted(os.listdir(os.path.join(HERE, "csrc")))]
DEPS.append(os.path.join(ROOT, "include", "ttt_la.h"))


def nvcc_cmd(out=OUT, verbose=False, debug=False):
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I" + os.path.join(ROOT, "include"), "-o", out, SRC, "-lcudart"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if debug:
        cmd.insert(1, "-DTTT_LA_DEBUG")
    return cmd


def up_to_date(out=OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force=False, verbose=False, out=OUT, debug=False) -> str:
    if not force and up_to_date(out):
        return out
    cmd = nvcc_cmd(out, verbose, debug)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    return out


def build_all(force=False, verbose=False):
    """The release library and its debug build (device-side bounds checks)."""
    return build(force, verbose), build(force, verbose, out=DEBUG_OUT, debug=True)


if __name__ == "__main__":
    if "--debug" in sys.argv:
        print(build(force=True, verbose="--verbose" in sys.argv, out=DEBUG_OUT, debug=True))
    else:
        print(build(force=True, verbose="--verbose" in sys.argv))
