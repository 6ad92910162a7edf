"""Builds libvsl.so (the C-ABI library) in-tree with nvcc for sm_100a, and the
test library tests/libvsl_test.so (the same objects plus the test-only probes
of tests/csrc/vsl_test_probes.cu; never part of libvsl.so)."""
import os
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "libvsl.so")
TEST_SRC = os.path.join(ROOT, "tests", "csrc", "vsl_test_probes.cu")
TEST_LIB_PATH = os.path.join(ROOT, "tests", "libvsl_test.so")
SOURCES = ["vsl_api.cu", "vsl_gemm.cu", "vsl_sample.cu", "vsl_verify.cu", "vsl_processed.cu", "vsl_tiles.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [*ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build():
    if not os.path.exists(LIB_PATH) or not os.path.exists(TEST_LIB_PATH):
        return True
    t = min(os.path.getmtime(LIB_PATH), os.path.getmtime(TEST_LIB_PATH))
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps += [os.path.join(ROOT, "include", "vsl.h"), TEST_SRC]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def _compile(src, obj, verbose):
    cmd = [_nvcc(), *NVCC_FLAGS, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)


def _link(objs, path):
    tmp = path + ".tmp"
    subprocess.run([_nvcc(), "-shared", *ARCH, "-o", tmp, *objs], check=True)
    os.replace(tmp, path)


def build(force=False, verbose=False):
    """Compile every CUDA source and link libvsl.so next to this file (and the test library)."""
    if not force and not needs_build():
        return LIB_PATH
    objdir = os.path.join(ROOT, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        _compile(os.path.join(CSRC, src), obj, verbose)
        objs.append(obj)
    _link(objs, LIB_PATH)
    probe = os.path.join(objdir, "vsl_test_probes.o")
    _compile(TEST_SRC, probe, verbose)
    _link(objs + [probe], TEST_LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB_PATH)
