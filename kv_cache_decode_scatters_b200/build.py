"""Build libkvdecode.so in-tree with nvcc for sm_100a (B200).

    python kv_cache_decode_scatters_b200/build.py [--force] [--verbose-ptxas]

(run it as a script: importing the package loads the library it builds)

The library is written next to this file so it travels with the source tree;
it is rebuilt when any source or the public header is newer than it.
"""
import concurrent.futures
import glob
import os
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libkvdecode.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                    "-I", INCLUDE, "--use_fast_math"]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    with tempfile.TemporaryDirectory(dir=HERE, prefix="_build_") as tmp:
        objs = [os.path.join(tmp, os.path.basename(src) + ".o") for src in sources()]
        # the translation units are independent: compile them concurrently
        jobs = max(1, min(len(objs), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(jobs) as pool:
            runs = [pool.submit(subprocess.run, [nvcc(), *flags, "-c", src, "-o", obj], check=True)
                    for src, obj in zip(sources(), objs)]
            for r in runs:
                r.result()  # re-raises a failed compile
        out = os.path.join(tmp, "libkvdecode.so")
        subprocess.run([nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", out, *objs], check=True)
        os.replace(out, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
