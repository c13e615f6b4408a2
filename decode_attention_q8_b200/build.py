"""Builds libkvq.so in-tree with nvcc for sm_100a (B200).

    python decode_attention_q8_b200/build.py            # incremental
    python decode_attention_q8_b200/build.py --force    # rebuild

The library links the CUDA runtime statically, so it loads on a machine
without a GPU (entry points that only compute sizes work there; launches
report KVQ_ERR_CUDA).
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libkvq.so")
OBJDIR = os.path.join(HERE, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "-Xptxas", "-v", "--expt-relaxed-constexpr"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "kvq.h"))
    files.append(os.path.abspath(__file__))
    return files


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False):
    """Compile every .cu under csrc/ and link libkvq.so; returns its path."""
    deps = _deps()
    os.makedirs(OBJDIR, exist_ok=True)
    objs = []
    nvcc = _nvcc()
    procs = []
    for src in sorted(f for f in os.listdir(CSRC) if f.endswith(".cu")):
        obj = os.path.join(OBJDIR, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, deps):
            cmd = [nvcc, *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", os.path.join(CSRC, src), "-o", obj]
            procs.append((src, obj, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                                     text=True)))
    failed = []
    for src, obj, pr in procs:  # translation units compile in parallel
        out, err = pr.communicate()
        if pr.returncode != 0:
            failed.append(f"nvcc failed for {src}:\n{out}\n{err}")
            if os.path.exists(obj):
                os.remove(obj)
        elif verbose:
            sys.stderr.write(err)
    if failed:
        raise RuntimeError("\n".join(failed))
    if force or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)   # atomic: a reader never sees a partly written library
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
