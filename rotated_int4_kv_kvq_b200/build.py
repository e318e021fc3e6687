"""Build libkvq.so in-tree for sm_100a with nvcc.

    python -m rotated_int4_kv_kvq_b200.build [--verbose-ptxas] [--all]

Each translation unit of csrc/ is compiled in parallel, then linked into
``rotated_int4_kv_kvq_b200/libkvq.so`` (CUDA runtime linked statically).
``--all`` also builds the test-only variants (``libkvq_test_<name>.so``).
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libkvq.so")

SOURCES = ["kvq_api.cu", "kvq_d64.cu", "kvq_d128.cu", "kvq_d256.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# Hidden visibility: only the C API (KVQ_API in include/kvq.h) is exported.
# Otherwise the function-local statics of inline and template code are
# exported as process-wide unique symbols and shared by every build of the
# library loaded into one process.
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr", "-I", INCLUDE,
         "-I", CSRC]
# Extra nvcc flags (e.g. -D tuning overrides) and an alternative output
# path, for building variants side by side.
EXTRA = os.environ.get("KVQ_NVCC_EXTRA", "").split()
LIB = os.environ.get("KVQ_LIB_OUT", LIB)
BUILD = os.environ.get("KVQ_BUILD_DIR", BUILD)


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


# Test-only variants of the library, built beside it from the same sources
# with extra defines.  "timeout": bounded waits give up after 1 ms and the
# forward kernel issues no copy for input tile 0, so that the device-status
# time-out path runs (tests/test_zz_device_timeout.py); product builds never
# define these.
TEST_VARIANTS = {
    "timeout": ["-DKVQ_WAIT_LIMIT_NS=1000000ull", "-DKVQ_TEST_SKIP_TILE=0"],
}


def variant_path(name: str) -> str:
    return os.path.join(PKG, f"libkvq_test_{name}.so")


def _compile(src: str, ptxas_verbose: bool, build_dir: str, extra) -> tuple[str, str]:
    obj = os.path.join(build_dir, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, *EXTRA, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    return obj, r.stderr


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "kvq.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def _codelets() -> None:
    """Regenerate kvq_rfft.cuh when the generator is newer than it."""
    gen = os.path.join(CSRC, "gen_rfft.py")
    out = os.path.join(CSRC, "kvq_rfft.cuh")
    if not os.path.exists(out) or os.path.getmtime(gen) > os.path.getmtime(out):
        subprocess.run([sys.executable, gen], check=True, capture_output=True)


def _build_one(lib: str, build_dir: str, extra, force: bool, ptxas_verbose: bool,
               quiet: bool) -> str:
    if not force and not _stale(lib):
        return lib
    os.makedirs(build_dir, exist_ok=True)
    logs = []
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        futs = [ex.submit(_compile, s, ptxas_verbose, build_dir, extra) for s in SOURCES]
        objs = []
        for f in futs:
            obj, log = f.result()
            objs.append(obj)
            logs.append(log)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    if not quiet or ptxas_verbose:
        sys.stderr.write("".join(logs))
    return lib


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True) -> str:
    """Build libkvq.so (the product library)."""
    _codelets()
    return _build_one(LIB, BUILD, [], force, ptxas_verbose, quiet)


def build_test_variant(name: str, force: bool = False) -> str:
    """Build the test-only library variant `name` (see TEST_VARIANTS)."""
    _codelets()
    return _build_one(variant_path(name), os.path.join(BUILD, f"test_{name}"),
                      TEST_VARIANTS[name], force, False, True)


def build_all(force: bool = False) -> list[str]:
    """The product library and every test variant, built concurrently."""
    _codelets()
    jobs = [(LIB, BUILD, [])] + [(variant_path(n), os.path.join(BUILD, f"test_{n}"), e)
                                 for n, e in TEST_VARIANTS.items()]
    with cf.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        futs = [ex.submit(_build_one, lib, bd, e, force, False, True) for lib, bd, e in jobs]
        return [f.result() for f in futs]


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--all", action="store_true", help="also build the test-only variants")
    a = ap.parse_args()
    if a.all:
        print("\n".join(build_all(force=a.force)))
    else:
        print(build(force=True if a.verbose_ptxas else a.force, ptxas_verbose=a.verbose_ptxas))


if __name__ == "__main__":
    main()
