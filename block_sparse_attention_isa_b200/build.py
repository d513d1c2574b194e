"""Build ``libisa.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_sparse_attention_isa_b200.build [--verbose]

The library links the CUDA runtime statically and reaches the driver only
through the runtime's entry-point query, so it loads on a machine without a
GPU driver (the C ABI then reports ISA_ERR_CUDA on any call that needs one).
"""
from __future__ import annotations

import glob
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libisa.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps.append(os.path.join(os.path.dirname(PKG), "include", "isa.h"))
    return all(os.path.getmtime(d) <= t for d in deps if os.path.exists(d))


# Kernels that move registers between warpgroups with setmaxnreg. Their split is sized for
# exactly this many registers per thread at launch (a split above the launch budget would make
# setmaxnreg.inc wait for ever), so the build fails if ptxas assigns another count.
REGISTER_SPLIT_KERNELS = {
    "attention_pair_kernel": 168,
    "attention_kernel": 168,
    "attention_mixed_kernel": 168,
    "attention_bwd_kernel": 168,
}


def register_counts(ptxas_log: str) -> dict:
    """{mangled kernel name: registers per thread} from the `-Xptxas -v` report."""
    counts, current = {}, None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current:
            counts[current] = int(m.group(1))
            current = None
    return counts


def check_register_split(ptxas_log: str) -> None:
    """Raise if a register-split kernel was compiled to a count other than its split's budget."""
    counts = register_counts(ptxas_log)
    for kern, want in REGISTER_SPLIT_KERNELS.items():
        # mangled names hold the identifier as <length><name>
        tag = f"{len(kern)}{kern}"
        found = {n: c for n, c in counts.items() if tag in n}
        if not found:
            raise RuntimeError(f"ptxas reported no entry function named {kern}")
        bad = {n: c for n, c in found.items() if c != want}
        if bad:
            raise RuntimeError(f"{kern}: compiled to {sorted(set(bad.values()))} registers per thread, its "
                               f"warpgroup register split needs exactly {want}")


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-cudart", "static", "--expt-relaxed-constexpr",
           "-I", os.path.join(os.path.dirname(PKG), "include"), "-Xptxas", "-v"]
    cmd += sources() + ["-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    try:
        check_register_split(res.stdout + res.stderr)
    except RuntimeError:
        os.remove(tmp)
        raise
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True))
