"""Builds the C-ABI shared library ``libattn_b200.so`` in this package directory.

nvcc compiles ``csrc/attn_lib.cu``, which includes every other source under ``csrc/``, as one
translation unit for sm_100a only (``-gencode arch=compute_100a,code=sm_100a``) into one shared
object that exports
the ``extern "C"`` entry points declared in ``include/attn.h``. Run ``python -m
exact_io_aware_41_b200.build`` (``--force`` rebuilds, ``--verbose`` prints ptxas resource usage,
``--emu-variant`` also builds the test variant with FMA-pipe exponentials).
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libattn_b200.so")
UNITY = os.path.join(HERE, "csrc", "attn_lib.cu")  # includes every other .cu under csrc/
SOURCES = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))
HEADERS = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(HERE, "csrc", "*.h")) +
                 glob.glob(os.path.join(ROOT, "include", "*.h")))
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libattn_b200.so")


# A test build of the same sources with the FMA-pipe exponential switched on for part of every
# tile's columns at each head dim (the product build evaluates every exponential on the exp unit).
# The GPU tests check this variant against the oracle, so the emulated branch is exercised.
EMU_LIB_PATH = os.path.join(HERE, "libattn_b200_emu.so")
EMU_DEFINES = ["-DATTN_EMU_COLS_D32=64", "-DATTN_EMU_COLS_D64=64", "-DATTN_EMU_COLS_D128=32",
               "-DATTN_EMU_COLS_D256=32"]


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in SOURCES + HEADERS + [__file__])


def _compile(path: str, defines, verbose: bool) -> str:
    cmd = [_nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared", "-Xcompiler", "-fPIC", *defines,
           "-I", os.path.join(ROOT, "include"), "-o", path + ".tmp", UNITY]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(path + ".tmp", path)
    return path


def build(force: bool = False, verbose: bool = False) -> str:
    """The product library (libattn_b200.so)."""
    if not force and up_to_date(LIB_PATH):
        return LIB_PATH
    return _compile(LIB_PATH, [], verbose)


def build_emu_variant(force: bool = False, verbose: bool = False) -> str:
    """The test variant with FMA-pipe exponentials (libattn_b200_emu.so)."""
    if not force and up_to_date(EMU_LIB_PATH):
        return EMU_LIB_PATH
    return _compile(EMU_LIB_PATH, EMU_DEFINES, verbose)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--emu-variant", action="store_true", help="also build the emulated-exponential test variant")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
    if a.emu_variant:
        print(build_emu_variant(force=a.force, verbose=a.verbose))
