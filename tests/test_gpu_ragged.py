"""GPU parity for lengths that b does not divide: the last source or context block is short.

The CUDA path against the ragged-length oracle (float64), element by element:
kept blocks, routing and (with alpha_ns) the exact key blocks bit-exactly,
outputs within max-abs 2e-2 and relative L2 5e-3. Inputs whose top-k, routing
or exact-block choice lies within a relative 1e-3 of a tie are redrawn. The
cases cover a short block in either part or both, b = 64 and 128, D = 64 and
128, bf16 and fp32, the dense point, the Taylor path with both short blocks
kept, a context shorter than one block, a padded source part reaching past the
end of the sequence, and the alpha_ns path.
"""
import numpy as np
import pytest

import isa_synth
from oracle import isa_oracle_ragged as R
from parity_util import MARGIN, compare_out, to_device

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, D, L_src, L_ctx, b, alpha_s, alpha_f, dtype, alpha_ns
    ("b128_both_short", 1, 2, 128, 1000, 1100, 128, 0.5, 0.5, "bf16", 0.0),
    ("b64_both_short", 1, 2, 128, 657, 453, 64, 0.3, 0.5, "bf16", 0.0),
    ("d64_b64_source_short", 1, 2, 64, 1000, 512, 64, 0.25, 0.5, "bf16", 0.0),
    ("d64_b128_context_short", 1, 2, 64, 1024, 1000, 128, 0.5, 0.5, "bf16", 0.0),
    ("f32_both_short", 1, 2, 64, 600, 450, 64, 0.5, 0.5, "f32", 0.0),
    ("dense_point", 1, 2, 128, 1000, 1100, 128, 1.0, 0.0, "bf16", 0.0),
    ("taylor_both_short_kept", 1, 2, 128, 1000, 1100, 128, 1.0, 1.0, "bf16", 0.0),
    ("context_below_b", 1, 2, 128, 1024, 40, 64, 1.0, 0.5, "bf16", 0.0),
    ("padding_past_end", 1, 2, 128, 65, 10, 64, 1.0, 0.5, "bf16", 0.0),
    ("f32_padding_past_end", 1, 2, 64, 65, 10, 64, 1.0, 0.5, "f32", 0.0),
    ("b2_h2_both_short", 2, 2, 128, 700, 500, 128, 0.5, 0.25, "bf16", 0.0),
    ("ns_b128", 1, 2, 128, 1000, 1100, 128, 0.5, 0.5, "bf16", 0.25),
    ("ns_b64", 1, 2, 128, 657, 453, 64, 0.5, 0.5, "bf16", 0.25),
]


def _inputs(w, a_ns, max_attempts=64):
    att = np.zeros((w.B, w.H), np.int64)
    for bi in range(w.B):
        for h in range(w.H):
            for a in range(max_attempts):
                q, k, _ = isa_synth.make_slice(w, 0, bi, h, a)
                r = R.isa_select_route_ragged(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, a_ns)
                if min(r["topk_margin"], r["route_margin"], r["ns_margin"]) >= MARGIN:
                    att[bi, h] = a
                    break
            else:
                raise RuntimeError(f"no accepted attempt for slice {bi},{h}")
    return isa_synth.make_inputs(w, 0, att)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_ragged_full_parity(case):
    import torch
    import block_sparse_attention_isa_b200 as isa
    name, B, H, D, L_src, L_ctx, b, a_s, a_f, dt, a_ns = case
    w = isa_synth.Workload(name, B, H, D, L_src, L_ctx, b, a_s, a_f, 0.1, 1.0, 0.5, dt)
    q, k, v = _inputs(w, a_ns)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    res = isa.forward(tq, tk, tv, L_src, L_ctx, b, a_s, a_f, debug=True, alpha_ns=a_ns)
    isa.device_status()
    torch.cuda.synchronize()
    out, sel, route = (x.cpu() for x in res[:3])
    out = out.float().numpy()
    ref_out = np.zeros_like(out, dtype=np.float64)
    for bi in range(B):
        for h in range(H):
            r = R.isa_slice_ref_ragged(q[bi, h], k[bi, h], v[bi, h], L_src, L_ctx, b, a_s, a_f, a_ns)
            np.testing.assert_array_equal(sel[bi, h].numpy(), r["sel"], err_msg=f"kept blocks {bi},{h}")
            np.testing.assert_array_equal(route[bi, h].numpy(), r["route"], err_msg=f"routing {bi},{h}")
            if a_ns:
                ns = res[3][bi, h].cpu().numpy()
                np.testing.assert_array_equal(ns[r["taylor"]], r["ns_sel"][r["taylor"]])
            ref_out[bi, h] = r["out"]
    compare_out(out, ref_out)


# ---------------------------------------------------------------- full size

def _ragged_slice_work(args):
    """Worker: the accepted draw of one slice and its whole-slice ragged oracle."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import isa_synth as S
    from oracle import isa_oracle_ragged as RR
    from threadpoolctl import threadpool_limits
    w, bi, h, margin, threads = args
    with threadpool_limits(limits=threads):
        for a in range(64):
            q, k, v = S.make_slice(w, 0, bi, h, a)
            sr = RR.isa_select_route_ragged(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
            if min(sr["topk_margin"], sr["route_margin"]) >= margin:
                break
        else:
            raise RuntimeError(f"no accepted attempt for slice {bi},{h}")
        r = RR.isa_slice_ref_ragged(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, sr=sr)
    return bi, h, q, k, v, r["sel"], r["route"], r["out"]


def test_ragged_full_size_32k():
    """The headline shape with both parts ragged: L_src = 16300 (127 blocks + 44 tokens),
    L_ctx = 16500 (128 blocks + 116 tokens), b = 128, alpha_s = 0.25, alpha_f = 0.6, 4 heads,
    every output row compared."""
    import multiprocessing as mp
    import os
    import torch
    import block_sparse_attention_isa_b200 as isa
    w = isa_synth.Workload("ragged_n32800_b128", 1, 4, 128, 16300, 16500, 128, 0.25, 0.6, 0.1, 1.0, 0.5, "bf16")
    threads = max(1, (os.cpu_count() or 4) // (w.B * w.H))
    pool = mp.get_context("spawn").Pool(w.B * w.H)
    try:
        res = pool.map(_ragged_slice_work, [(w, bi, h, MARGIN, threads) for bi in range(w.B) for h in range(w.H)],
                       chunksize=1)
    finally:
        pool.terminate()
    shape = (w.B, w.H, w.N, w.D)
    q, k, v = (np.zeros(shape, np.float32) for _ in range(3))
    for bi, h, qs, ks, vs, *_ in res:
        q[bi, h], k[bi, h], v[bi, h] = qs, ks, vs
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    out, sel, route = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
    isa.device_status()
    out, sel, route = out.float().cpu().numpy(), sel.cpu().numpy(), route.cpu().numpy()
    ref = np.zeros(shape, np.float64)
    for bi, h, _, _, _, sel_ref, route_ref, out_ref in res:
        np.testing.assert_array_equal(sel[bi, h], sel_ref, err_msg=f"kept blocks {bi},{h}")
        np.testing.assert_array_equal(route[bi, h], route_ref, err_msg=f"routing {bi},{h}")
        ref[bi, h] = out_ref
    compare_out(out, ref)
