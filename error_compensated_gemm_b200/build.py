"""Build libheal.so in-tree: every .cu under csrc/ compiled for sm_100a and linked into
one shared library next to this file (static CUDA runtime, no libcuda link: the driver
is reached through the runtime's entry-point query, so the library also loads on a
machine without a GPU)."""
import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libheal.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-I", os.path.join(ROOT, "include"),
         "--expt-relaxed-constexpr", "-diag-suppress", "20044"]


def nvcc():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _needs(obj, src, deps):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src] + deps)


DEBUG_LIB = os.path.join(HERE, "libheal_debug.so")


def build(verbose=False, jobs=None, debug=False):
    """debug=True builds libheal_debug.so: the same sources with HEAL_DEBUG defined, whose
    kernels check every global store index and TMA coordinate they compute and record a
    violation in the device status word (HEAL_ERR_INVALID_ARGUMENT) instead of faulting."""
    build_dir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = DEBUG_LIB if debug else LIB
    flags = FLAGS + (["-DHEAL_DEBUG=1"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(ROOT, "include", "heal.h"))
    cc = nvcc()
    objs = []
    cmds = []
    for f in srcs:
        src = os.path.join(CSRC, f)
        obj = os.path.join(build_dir, f[:-3] + ".o")
        objs.append(obj)
        if _needs(obj, src, deps):
            cmds.append([cc] + ARCH + flags + ["-c", src, "-o", obj])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
        if verbose:
            sys.stdout.write(r.stdout + r.stderr)

    with concurrent.futures.ThreadPoolExecutor(max_workers=jobs or os.cpu_count() or 4) as ex:
        list(ex.map(run, cmds))
    if cmds or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        run([cc] + ARCH + ["-shared", "-cudart", "static", "-o", lib] + objs)
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, debug="--debug" in sys.argv))
