"""Build the sm_100a shared library libmoe_route07.so in-tree with nvcc.

    python -m combine_moe_route_07_b200.build [--force]

Each .cu file compiles to an object in parallel, then one link step.  Flags:
sm_100a only, -O3, -lineinfo, IEEE float (no fast-math: the gate softmax and
FP8 scales rely on correctly rounded division), -Xptxas -v logged to
_build/ptxas.log for register / spill checks.
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe_route07.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE,
          "-I", CSRC, "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, obj, extra):
    cmd = [NVCC] + ARCH + CFLAGS + extra + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    return src, r.returncode, r.stdout + r.stderr


def build(force: bool = False, lib: str = LIB, extra=(), tag: str = "") -> str:
    """Compile every kernel source and link `lib`; returns its path."""
    if not force and not _stale(lib, _deps()):
        return lib
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    objs = [os.path.join(BUILD, os.path.basename(s)[:-3] + tag + ".o") for s in srcs]
    logs = []
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        futs = [ex.submit(_compile, s, o, list(extra)) for s, o in zip(srcs, objs)]
        for f in futs:
            src, rc, out = f.result()
            logs.append(f"== {os.path.basename(src)}\n{out}")
            if rc != 0:
                sys.stderr.write(out)
                raise RuntimeError(f"nvcc failed on {src}")
    with open(os.path.join(BUILD, f"ptxas{tag}.log"), "w") as f:
        f.write("\n".join(logs))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc link failed")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
