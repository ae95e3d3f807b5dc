"""Build liborbitquant.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m quantized_linear_token_b200.build [--force] [--verbose]

The library goes next to this file, so it travels with the source tree.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "liborbitquant.so")

SOURCES = ["oq_api.cu", "oq_rotate_quantize.cu", "oq_rotate_quantize_tc.cu", "oq_gemm.cu", "oq_gemm_pair.cu", "oq_gemm_skinny.cu", "oq_gemm_w16.cu",
           "oq_levels.cu", "oq_host_io.cu", "oq_int4.cu",
           "oq_noalloc.cu", "oq_diag.cu", "oq_fused.cu", "oq_gemv.cu", "oq_weight_io.cpp", "oq_host.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17"]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build liborbitquant")
    return exe


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "orbitquant.h"))
    return files


STAMP = LIB + ".srchash"


def source_hash() -> str:
    """SHA-256 over every source and header the library is built from, and
    the compiler flags, in a fixed order: the identity of a build."""
    import hashlib
    m = hashlib.sha256()
    m.update(" ".join(ARCH + FLAGS).encode())
    for f in sorted(_deps()):
        m.update(os.path.basename(f).encode() + b"\0")
        with open(f, "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()


def up_to_date() -> bool:
    """The library exists and was built from exactly the sources present now
    (a stamp with their hash is written beside it by every build); file times
    are not trusted, since a copied tree keeps no build order."""
    if not (os.path.exists(LIB) and os.path.exists(STAMP)):
        return False
    with open(STAMP) as f:
        return f.read().strip() == source_hash()


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    return res.stdout + res.stderr


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every source for sm_100a (in parallel) and link the library."""
    if not force and up_to_date():
        return LIB
    stamp = source_hash()
    from concurrent.futures import ThreadPoolExecutor

    objdir = os.path.join(ROOT, "_build")
    os.makedirs(objdir, exist_ok=True)
    common = [nvcc(), *ARCH, *FLAGS, "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        common += ["-Xptxas", "-v"]
    jobs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src + ".o")
        jobs.append((obj, common + ["-c", os.path.join(CSRC, src), "-o", obj]))
    with ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        outs = list(ex.map(lambda j: _run(j[1], verbose), jobs))
    if verbose or ptxas_verbose:
        sys.stdout.write("".join(outs))
    _run([nvcc(), *ARCH, "--shared", "-o", LIB + ".tmp"] + [o for o, _ in jobs], verbose)
    if os.path.exists(STAMP):
        os.remove(STAMP)
    os.replace(LIB + ".tmp", LIB)
    with open(STAMP + ".tmp", "w") as f:
        f.write(stamp + "\n")
    os.replace(STAMP + ".tmp", STAMP)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    args = ap.parse_args()
    print(build(args.force, args.verbose, args.ptxas_verbose))


if __name__ == "__main__":
    main()
