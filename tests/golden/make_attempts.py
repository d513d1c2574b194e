"""Write tests/golden/attempts.json: the accepted generator attempt of every slice.

For each workload and each (batch, head) slice, draw attempt 0, 1, 2, ... of
the seeded generator and keep the first one whose top-k and routing decisions
both clear a relative margin of 1e-3 in the oracle's float64 stages 1-3. Near
ties are rejected so that the float32 GPU path and the float64 oracle must
agree exactly on the kept context blocks and on the routing. A workload where
some slice finds no such draw within 100 attempts uses a 1e-4 margin for all
its slices instead; the margin used is stored with the attempts.

Calls only ``oracle`` and ``isa_synth``. Run from the repository root:
    python tests/golden/make_attempts.py [workload ...]
"""
import json
import multiprocessing as mp
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import isa_synth  # noqa: E402
from oracle import isa_oracle as O  # noqa: E402

MARGIN = 1e-3
# Fallback for workloads where the 1e-3 rule is too rare to meet: with the
# context tokens scaled down to 0.3 and half of the context kept, the k-th and
# (k+1)-th context scores sit in the densest part of their distribution and
# fewer than 1 draw in 25 clears 1e-3. 1e-4 is still about 100 times the
# relative error of the float32 scores on the GPU.
MARGIN_FALLBACK = 1e-4
SEED = 0
MAX_ATTEMPTS = 100
MAX_ATTEMPTS_FALLBACK = 400


def _slice_job(args):
    """First attempt of one slice that clears each margin, for every workload of a group sharing its draws."""
    names, bi, h = args
    ws = [isa_synth.all_workloads()[n] for n in names]
    w0 = ws[0]
    strict, loose = {}, {}
    for a in range(MAX_ATTEMPTS_FALLBACK):
        need_strict = a < MAX_ATTEMPTS and any(w.name not in strict for w in ws)
        need_loose = any(w.name not in loose for w in ws)
        if not need_strict and not need_loose:
            break
        q, k, _ = isa_synth.make_slice(w0, SEED, bi, h, a)
        for w in ws:
            if w.name in strict and w.name in loose:
                continue
            r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
            m = min(r["topk_margin"], r["route_margin"])
            if a < MAX_ATTEMPTS and w.name not in strict and m >= MARGIN:
                strict[w.name] = a
            if w.name not in loose and m >= MARGIN_FALLBACK:
                loose[w.name] = a
    missing = [w.name for w in ws if w.name not in loose]
    if missing:
        raise RuntimeError(f"no accepted attempt for slice ({bi},{h}) of {missing}")
    return bi, h, strict, loose


def groups(selected):
    """Workloads that share generator draws (same sizes, sigma range and s_ctx) form one group."""
    g = {}
    for w in isa_synth.all_workloads().values():
        if selected and w.name not in selected:
            continue
        key = (w.B, w.H, w.D, w.L_src, w.L_ctx, w.b, w.sigma_lo, w.sigma_hi, w.s_ctx, w.dtype)
        g.setdefault(key, []).append(w.name)
    return list(g.values())


def main(selected):
    path = os.path.join(ROOT, "tests", "golden", "attempts.json")
    table = isa_synth.load_attempts(path)
    ctx = mp.get_context("spawn")
    with ctx.Pool(max(1, min(os.cpu_count() or 1, 16))) as pool:
        for names in groups(selected):
            t0 = time.time()
            w0 = isa_synth.all_workloads()[names[0]]
            jobs = [(names, bi, h) for bi in range(w0.B) for h in range(w0.H)]
            res = pool.map(_slice_job, jobs)
            for n in names:
                att = np.zeros((w0.B, w0.H), np.int64)
                strict_ok = all(n in st for _, _, st, _ in res)
                for bi, h, st, lo in res:
                    att[bi, h] = st[n] if strict_ok else lo[n]
                table[n] = {"seed": SEED, "margin": MARGIN if strict_ok else MARGIN_FALLBACK,
                            "attempts": att.tolist()}
            print(f"{len(names)} workload(s) from {names[0]}: {time.time() - t0:.1f}s", flush=True)
    with open(path, "w") as f:
        json.dump(dict(sorted(table.items())), f, indent=0)
        f.write("\n")


if __name__ == "__main__":
    main(set(sys.argv[1:]))
