"""Build libfrt.so (the CUDA library) in-tree for sm_100a with nvcc, and its
bounds-checked variant libfrt_debug.so (FRT_DEBUG_BOUNDS, relocatable device
code so that every source shares one device-side violation counter).

    python -m memory_bound_non_b200.build        # build both if sources changed
    python -m memory_bound_non_b200.build -f     # force
"""
import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfrt.so")
DEBUG_LIB = os.path.join(PKG, "libfrt_debug.so")
DEBUG_FLAGS = ["-rdc=true", "-DFRT_DEBUG_BOUNDS"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile every source to an object in parallel (one nvcc per file),
    then link the shared library (the bounds-checked one with
    debug_bounds)."""
    lib = DEBUG_LIB if debug_bounds else LIB
    extra = DEBUG_FLAGS if debug_bounds else []
    if not force and not _stale(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    objdir = tempfile.mkdtemp(prefix="frt_build_")
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"] + extra
    jobs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc] + compile_flags + ["-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        jobs.append((cmd, obj))
    try:
        with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as pool:
            results = list(pool.map(lambda j: subprocess.run(j[0], capture_output=True, text=True), jobs))
        failed = False
        for (cmd, _), r in zip(jobs, results):
            if r.stdout or r.stderr:
                sys.stdout.write(r.stdout)
                sys.stderr.write(r.stderr)
            if r.returncode != 0:
                failed = True
                sys.stderr.write("failed: %s\n" % " ".join(cmd))
        if failed:
            raise subprocess.CalledProcessError(1, "nvcc")
        tmp = lib + ".tmp.%d" % os.getpid()
        subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared"] + extra[:1] + ["-o", tmp] +
                       [o for _, o in jobs], check=True)
        os.replace(tmp, lib)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return lib


def build_all(force: bool = False, verbose: bool = False):
    """Both libraries, built side by side (their objects are independent)."""
    with concurrent.futures.ThreadPoolExecutor(max_workers=2) as pool:
        release = pool.submit(build, force, verbose)
        debug = pool.submit(build, force, verbose, True)
        return release.result(), debug.result()


if __name__ == "__main__":
    for path in build_all(force="-f" in sys.argv, verbose="-v" in sys.argv):
        print(path)
