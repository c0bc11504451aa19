"""Build the SAGA CUDA library in-tree: csrc/*.cu -> _lib/libsaga_b200.so.

sm_100a only. Each translation unit compiles in parallel into _build/, then
one link produces the shared library with the CUDA runtime linked statically
(the library then needs only the driver at run time).

build(check=True) makes the bounds-checked variant _lib/libsaga_b200_check.so
(compiled with -DSAGA_CHECK: explicit index checks in the kernels that set
SAGA_DEVERR_BOUNDS in the device error word and skip the access, instead of
trapping); the binding loads it when SAGA_CHECKED_BUILD=1 is set.
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(ROOT, "_build", "saga")
LIB_DIR = os.path.join(HERE, "_lib")
LIB_PATH = os.path.join(LIB_DIR, "libsaga_b200.so")
CHECK_LIB_PATH = os.path.join(LIB_DIR, "libsaga_b200_check.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
              "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
              "-I", SRC]


def _compile(src, ptxas_verbose, obj_dir=OBJ, extra=()):
    obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
    cmd = ["nvcc", *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    return src, obj, r


def build(verbose=False, ptxas_verbose=False, check=False):
    obj_dir = OBJ + "_check" if check else OBJ
    extra = ("-DSAGA_CHECK",) if check else ()
    lib_path = CHECK_LIB_PATH if check else LIB_PATH
    os.makedirs(obj_dir, exist_ok=True)
    os.makedirs(LIB_DIR, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(SRC, "*.cu")))
    objs = []
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        for src, obj, r in ex.map(lambda s: _compile(s, ptxas_verbose, obj_dir, extra), srcs):
            if verbose or ptxas_verbose or r.returncode != 0:
                sys.stdout.write(r.stdout)
                sys.stderr.write(r.stderr)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
            objs.append(obj)
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart",
           "static", "-o", lib_path, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stderr)
        raise RuntimeError(f"link of {os.path.basename(lib_path)} failed")
    return lib_path


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, ptxas_verbose="--ptxas" in sys.argv,
                check="--check" in sys.argv))
