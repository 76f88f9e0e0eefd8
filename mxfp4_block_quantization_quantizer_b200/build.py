"""Build libmxfp4.so (the C-ABI library) in-tree with nvcc for sm_100a.

No fast-math (subnormals are kept) and --fmad=false (no multiply-add is
fused behind the code's back; intended fused operations are written as
explicit intrinsics).
"""
import glob
import os
import shutil
import subprocess
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmxfp4.so")
HEADER = os.path.join(ROOT, "include", "mxfp4.h")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-O3", "-std=c++17", "--fmad=false", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-Wall"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER]
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(out: str, defines=(), verbose: bool = False) -> None:
    """Compile each .cu under csrc/ to an object in parallel, then link them
    into the shared library `out` (written atomically)."""
    nvcc = os.environ.get("NVCC", "nvcc")
    flags = NVCC_FLAGS + ["-D" + d for d in defines] + (["-Xptxas", "-v"] if verbose else [])
    tmpdir = tempfile.mkdtemp(prefix="mxfp4_build_")
    try:
        objs, procs = [], []
        for src in sources():
            obj = os.path.join(tmpdir, os.path.basename(src) + ".o")
            objs.append(obj)
            procs.append((src, subprocess.Popen([nvcc] + flags + ["-c", "-o", obj, src])))
        failed = [src for src, pr in procs if pr.wait() != 0]
        if failed:
            raise RuntimeError("nvcc failed on " + ", ".join(failed))
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.run([nvcc] + NVCC_FLAGS + ["-shared", "-o", tmp] + objs, check=True)
        os.replace(tmp, out)
    finally:
        shutil.rmtree(tmpdir, ignore_errors=True)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ into libmxfp4.so if it is out of date."""
    if not force and not _stale():
        return LIB
    _compile(LIB, verbose=verbose)
    return LIB


def build_variant(out: str, defines) -> str:
    """The same library built with extra preprocessor definitions (e.g.
    MXFP4_ACC_WAIT_POLLS=0, the test build whose accumulator waits give up
    at once) into `out`, outside the package."""
    _compile(out, defines=defines)
    return out


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv))
