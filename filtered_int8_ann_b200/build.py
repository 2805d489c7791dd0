"""Build libst.so (the C-ABI search library) in-tree for sm_100a with nvcc, and
libst_peaks.so (the dp4a peak microbenchmark the benchmark reports against)."""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libst.so")
PEAKS_SRC = os.path.join(HERE, "microbench", "dp4a_peak.cu")
PEAKS_OUT = os.path.join(HERE, "libst_peaks.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def up_to_date(out=OUT):
    if not os.path.exists(out):
        return False
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(HERE, "..", "include", "st.h"), __file__]
    t = os.path.getmtime(out)
    return all(os.path.getmtime(p) <= t for p in deps)


def build_peaks(force=False):
    if force or not os.path.exists(PEAKS_OUT) or os.path.getmtime(PEAKS_SRC) > os.path.getmtime(PEAKS_OUT):
        nvcc = os.environ.get("NVCC", "nvcc")
        subprocess.run([nvcc, *ARCH, *FLAGS, PEAKS_SRC, "-o", PEAKS_OUT], check=True)
    return PEAKS_OUT


def build(force=False, verbose=False, out=OUT):
    build_peaks(force)
    if not force and up_to_date(out):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *ARCH, *FLAGS, *(["-Xptxas", "-v"] if verbose else []), *sources(), "-o", out]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
