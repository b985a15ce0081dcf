"""Build libkda.so in-tree with nvcc for sm_100a.

    python -m gated_delta_rule_127_b200.build [--force]

Each .cu under csrc/ becomes one object (compiled in parallel); they are linked into
gated_delta_rule_127_b200/libkda.so with the CUDA runtime linked statically.  The same objects, with
kda_api.cu compiled again with -DKDA_DEBUG (host-side checks of packed batches before any launch),
make libkda_debug.so, which the binding loads when KDA_DEBUG=1 is set.
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libkda.so")
LIB_DEBUG = os.path.join(PKG, "libkda_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def _compile(src, extra, suffix=""):
    obj = os.path.join(BUILD, os.path.basename(src) + suffix + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link libkda.so; returns its path."""
    newest = max(os.path.getmtime(p) for p in _deps() + [__file__])
    if (not force and all(os.path.exists(p) and os.path.getmtime(p) >= newest for p in (LIB, LIB_DEBUG))):
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    api = os.path.join(CSRC, "kda_api.cu")
    jobs = [(s, extra, "") for s in _sources()] + [(api, ["-DKDA_DEBUG"], ".debug")]
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda j: _compile(*j), jobs))
    if verbose_ptxas:
        for _, log in results:
            sys.stderr.write(log)
    objs = [o for o, _ in results[:-1]]
    debug_objs = [results[-1][0] if o.endswith("kda_api.cu.o") else o for o in objs]
    for lib, lib_objs in ((LIB, objs), (LIB_DEBUG, debug_objs)):
        tmp = lib + ".tmp"
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *lib_objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
