"""GPU parity at the full workload sizes, in the launch configuration bench.py times.

For the 8K, 16K and 32K-token workloads and every point of the 51K-token sweep:
* the kept context blocks and the routing of every (batch, head) slice match the
  float64 oracle bit-exactly (stages 1-3 of the oracle are cheap at any size);
* sampled output rows (exact-path and Taylor-path rows of every head) match the
  oracle's rows within max-abs 2e-2 and relative L2 5e-3;
* every output element is finite and lies within its head's per-dimension
  [min, max] of V (each row is a convex combination of V rows).
Inputs are drawn with the accepted per-slice attempts stored in
tests/golden/attempts.json (tie margins of 1e-3, or 1e-4 where recorded).
"""
import multiprocessing as mp
import os

import numpy as np
import pytest

import isa_synth
from parity_util import MAX_ABS, REL_L2

pytestmark = pytest.mark.gpu

ROWS_PER_PATH = 8  # sampled rows per head and path


def _slice_work(args):
    """Worker: draw one slice and run the oracle's stages 1-3 and its sampled rows."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import isa_synth as S
    from oracle import isa_oracle as O
    name, bi, h, attempt = args
    w = S.all_workloads()[name]
    q, k, v = S.make_slice(w, 0, bi, h, attempt)
    sr = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    rng = np.random.default_rng([bi, h, 7])
    rows = []
    for blocks in (sr["exact"], sr["taylor"]):
        if len(blocks):
            blk = rng.choice(blocks, size=ROWS_PER_PATH)
            rows += list(blk * w.b + rng.integers(0, w.b, size=ROWS_PER_PATH))
    rows = np.array(sorted(set(int(r) for r in rows)), np.int64)
    ref_rows = O.isa_rows_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, rows, sr=sr)
    return (bi, h, q, k, v, sr["sel"], np.concatenate([sr["exact"], sr["taylor"]]), rows, ref_rows,
            sr["topk_margin"], sr["route_margin"])


_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = mp.get_context("spawn").Pool(max(2, min(16, (os.cpu_count() or 4) - 1)))
    return _POOL


def teardown_module(module):
    global _POOL
    if _POOL is not None:
        _POOL.terminate()
        _POOL = None


FULL = [isa_synth.WORKLOADS[n] for n in ("bf16_n8192_b64", "bf16_n16384_b64", "bf16_n32768_b128")] + \
    list(isa_synth.SWEEP_51K.values())


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_full_size_parity(w):
    import torch
    import block_sparse_attention_isa_b200 as isa
    table = isa_synth.load_attempts()
    att = isa_synth.attempts_for(w, 0, table)
    if att is None:
        pytest.fail(f"no stored attempts for {w.name}: run tests/golden/make_attempts.py")
    margin = table[w.name]["margin"]
    jobs = [(w.name, bi, h, int(att[bi, h])) for bi in range(w.B) for h in range(w.H)]
    res = _pool().map(_slice_work, jobs)

    dev = torch.device("cuda")
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    shape = (w.B, w.H, w.N, w.D)
    tq, tk, tv = (torch.empty(shape, dtype=dt, device=dev) for _ in range(3))
    for bi, h, q, k, v, *_ in res:
        tq[bi, h].copy_(torch.from_numpy(q))
        tk[bi, h].copy_(torch.from_numpy(k))
        tv[bi, h].copy_(torch.from_numpy(v))
    n_q, kk, _ = isa.plan(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f)
    out = torch.empty_like(tq)
    sel = torch.empty((w.B, w.H, kk), dtype=torch.int32, device=dev)
    route = torch.empty((w.B, w.H, n_q), dtype=torch.int32, device=dev)
    ws = torch.empty(isa.workspace_bytes(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s), dtype=torch.uint8,
                     device=dev)
    isa.forward_into(tq, tk, tv, out, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, sel, route, workspace=ws)
    isa.device_status(ws)

    # properties at full size: finite, inside each head's per-dimension range of V
    assert torch.isfinite(out).all()
    vmin = tv.float().amin(dim=2, keepdim=True)
    vmax = tv.float().amax(dim=2, keepdim=True)
    o = out.float()
    slack = MAX_ABS  # bf16 rounding of outputs near |4| is up to 1.6e-2
    assert bool(((o >= vmin - slack) & (o <= vmax + slack)).all())

    sel_h, route_h, out_h = sel.cpu().numpy(), route.cpu().numpy(), out.float().cpu().numpy()
    diffs, refs = [], []
    for bi, h, q, k, v, sel_ref, route_ref, rows, ref_rows, tm, rm in res:
        assert min(tm, rm) >= margin
        np.testing.assert_array_equal(sel_h[bi, h], sel_ref, err_msg=f"kept blocks, slice {bi},{h}")
        np.testing.assert_array_equal(route_h[bi, h], route_ref, err_msg=f"routing, slice {bi},{h}")
        diffs.append(out_h[bi, h, rows] - ref_rows)
        refs.append(ref_rows)
    d = np.concatenate(diffs)
    r = np.concatenate(refs)
    max_abs = float(np.abs(d).max())
    rel = float(np.linalg.norm(d) / np.linalg.norm(r))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"sampled rows: max-abs {max_abs:.3e}, rel-L2 {rel:.3e}"
