"""Build and load tests/csrc/umma_selftest.cu (primitive checks for the tensor-core path)."""
from __future__ import annotations

import ctypes
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "umma_selftest.cu")
OUT = os.path.join(HERE, "csrc", "libumma_selftest.so")
DEPS = [SRC, os.path.join(os.path.dirname(HERE), "linear_attention_token_b200", "csrc", "sm100.cuh")]


def build(force=False) -> str:
    if (not force and os.path.exists(OUT)
            and all(os.path.getmtime(OUT) >= os.path.getmtime(d) for d in DEPS)):
        return OUT
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                    SRC, "-o", OUT], check=True)
    return OUT


def load():
    L = ctypes.CDLL(build())
    P = ctypes.c_void_p
    L.selftest_umma.argtypes = [P, P, P, ctypes.c_int, P]
    L.selftest_cluster.argtypes = [P]
    L.selftest_tma.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
    return L
