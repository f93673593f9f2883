"""Build and load the scalar C oracle (``brute.c``) - TEST INFRASTRUCTURE ONLY.

``build()`` compiles ``libbrute.so`` beside this file with gcc; ``load()``
returns a ctypes handle with argument types set.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "brute.c")
LIB = os.path.join(HERE, "libbrute.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
                               SRC, "-o", LIB, "-lm"])
    return LIB


def load() -> ctypes.CDLL:
    lib = ctypes.CDLL(build())
    D, I, L, P = ctypes.c_double, ctypes.c_int, ctypes.c_long, ctypes.c_void_p
    lib.brute_round_bf16.argtypes, lib.brute_round_bf16.restype = [D], D
    lib.brute_gelu.argtypes, lib.brute_gelu.restype = [D], D
    lib.brute_token_a.argtypes = [P, I, I, I, I, I, I, I, P, P, D, I, P]
    lib.brute_token_a.restype = None
    lib.brute_token_y.argtypes = [P, I, I, I, I, I, I, I, P, P, D, P, P, I, P, P, I, I, P, P, P]
    lib.brute_token_y.restype = None
    lib.brute_row_of_token.argtypes, lib.brute_row_of_token.restype = [I, I, I, I, I, I, I], L
    lib.brute_row_of_newline.argtypes, lib.brute_row_of_newline.restype = [I, I, I, I], L
    lib.brute_row_of_separator.argtypes, lib.brute_row_of_separator.restype = [I, I], L
    lib.brute_dense.argtypes = [P, I, P, P, I, I, I, P]
    lib.brute_dense.restype = None
    return lib
