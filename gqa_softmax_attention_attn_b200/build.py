"""Builds libattn_sink.so in-tree with nvcc for sm_100a (python -m gqa_softmax_attention_attn_b200.build)."""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB_DIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIB_DIR, "libattn_sink.so")
SOURCES = ["attn_sink_api.cu", "simt_kernels.cu", "fwd_tc.cu", "fwd_band.cu", "decode_tc.cu", "bwd_tc.cu", "prologue.cu",
           "host_fwd.cu"]
HEADERS = ["kernels.h", "sm100_ptx.cuh", "selftest.cu"]
SELFTEST_LIB = os.path.join(LIB_DIR, "libattn_sink_selftest.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-DNDEBUG"]


def _digest() -> str:
    h = hashlib.sha256()
    for f in SOURCES + HEADERS:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(ROOT, "include", "attn_sink.h"), "rb") as fh:
        h.update(fh.read())
    h.update(" ".join(FLAGS).encode())
    return h.hexdigest()


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(LIB_DIR, exist_ok=True)
    stamp = LIB + ".sha256"
    dig = _digest()
    if not force and os.path.exists(LIB) and os.path.exists(stamp) and open(stamp).read().strip() == dig:
        return LIB
    objs = []
    obj_dir = os.path.join(LIB_DIR, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    for src in SOURCES:
        obj = os.path.join(obj_dir, src.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, "-I", os.path.join(ROOT, "include"), "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs,
                           "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map")])
    os.replace(tmp, LIB)
    # device self-tests of kernel helpers (test support, not the product ABI)
    tmp = SELFTEST_LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *FLAGS, "-shared", "-o", tmp, os.path.join(CSRC, "selftest.cu")])
    os.replace(tmp, SELFTEST_LIB)
    with open(stamp, "w") as fh:
        fh.write(dig)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
