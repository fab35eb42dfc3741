"""Builds libtra.so (the C-ABI library of hand-written sm_100a kernels) in
the package directory, and with --check the checked build libtra_check.so
(TRA_CHECK: kernels test the indices they derive before using them and report
an index outside its extent through the device error word).  Usage:
python -m entropy_adaptive_radius_b200.build [--force] [--verbose-ptxas] [--check]."""
import argparse
import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libtra.so")
BUILD_CHECK = os.path.join(ROOT, "_build_check")
LIB_CHECK = os.path.join(HERE, "libtra_check.so")
SOURCES = ["api.cu", "permute.cu", "radius.cu", "mask.cu", "attention.cu", "mask_noalloc.cu",
           "quant.cu", "selftest.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _flags(verbose_ptxas: bool):
    f = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I" + INCLUDE,
                "-I" + CSRC, "--expt-relaxed-constexpr"]
    if verbose_ptxas:
        f += ["-Xptxas", "-v"]
    return f


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return hs + [os.path.join(INCLUDE, "tra.h")]


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src] + _headers())


def build(force: bool = False, verbose_ptxas: bool = False, quiet: bool = False,
          check: bool = False) -> str:
    """Compiles the library (check=True: the checked build) and returns its path."""
    build_dir, lib = (BUILD_CHECK, LIB_CHECK) if check else (BUILD, LIB)
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()
    flags = _flags(verbose_ptxas) + (["-DTRA_CHECK"] if check else [])
    jobs = []
    objs = []
    for s in SOURCES:
        src = os.path.join(CSRC, s)
        obj = os.path.join(build_dir, s.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, src):
            jobs.append([cc, "-c", src, "-o", obj] + flags)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    failed = False
    with concurrent.futures.ThreadPoolExecutor(max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for cmd, r in ex.map(run, jobs):
            out = (r.stdout + r.stderr).strip()
            if r.returncode != 0:
                failed = True
                sys.stderr.write(f"FAILED: {' '.join(cmd)}\n{out}\n")
            elif out and (verbose_ptxas or not quiet):
                sys.stderr.write(out + "\n")
    if failed:
        raise RuntimeError("nvcc failed")
    if jobs or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        cmd = [cc, "-shared"] + ARCH + ["-o", lib] + objs + ["-lcudart_static", "-ldl", "-lrt", "-lpthread"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + r.stdout + r.stderr)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--check", action="store_true", help="build libtra_check.so (TRA_CHECK)")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, check=a.check))
