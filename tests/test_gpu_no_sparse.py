"""GPU parity of the no-sparsity ratio alpha_ns: exact key blocks inside the Taylor path.

For every Taylor query block the k_ns = ceil(alpha_ns * n_new - 1e-4) blocks of
K_new with the largest coarse scores are computed key by key, the others through
their pooled rows with weight b, in one softmax (papernotes.org, Key designs 2
and 3). Small workloads are compared in full against the float64 oracle: kept
blocks, routing and the per-block exact-block lists bit-exactly (inputs whose
choices lie within 1e-3 of a tie are redrawn), outputs within max-abs 2e-2 and
relative L2 5e-3. The 32K-token workload is checked in every row of its first
two heads (exact blocks, and the Taylor blocks whose exact-block choice clears
the same tie margin) and on sampled rows of such blocks in the other heads.
"""
import multiprocessing as mp
import os

import numpy as np
import pytest

import isa_synth
from oracle import isa_oracle as O
from parity_util import MARGIN, MAX_ABS, REL_L2, compare_out, to_device

pytestmark = pytest.mark.gpu

W = isa_synth.Workload


def _case(name, B, H, D, L_src, L_ctx, b, a_s, a_f, sig=(0.1, 1.0), s_ctx=0.5):
    return W(name, B, H, D, L_src, L_ctx, b, a_s, a_f, sig[0], sig[1], s_ctx, "bf16")


def ns_inputs(w, alpha_ns, seed=0, max_attempts=64):
    """Inputs whose top-k, routing and exact-block choices all clear the tie margin."""
    att = np.zeros((w.B, w.H), np.int64)
    for bi in range(w.B):
        for h in range(w.H):
            for a in range(max_attempts):
                q, k, _ = isa_synth.make_slice(w, seed, bi, h, a)
                r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, alpha_ns)
                if min(r["topk_margin"], r["route_margin"], r["ns_margin"]) >= MARGIN:
                    att[bi, h] = a
                    break
            else:
                raise RuntimeError(f"no accepted attempt for slice {bi},{h}")
    return isa_synth.make_inputs(w, seed, att)


def run_ns(w, alpha_ns, q, k, v):
    import torch
    import block_sparse_attention_isa_b200 as isa
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    out, sel, route, ns = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True,
                                      alpha_ns=alpha_ns)
    isa.device_status()
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), sel.cpu().numpy(), route.cpu().numpy(), ns.cpu().numpy()


CASES = [
    # b = 128: n_new = 40 (one ragged pooled tile), k_ns = 3
    (_case("b128_long", 1, 2, 128, 4096, 4096, 128, 0.25, 0.5), 0.0625),
    # b = 64: n_new = 13, k_ns = 4; odd unions leave half-filled exact tiles; odd n_q
    (_case("b64_ragged", 1, 2, 128, 640, 448, 64, 0.3, 0.5), 0.25),
    # D = 64
    (_case("d64_b64", 1, 2, 64, 1024, 512, 64, 0.25, 0.5), 0.1),
    (_case("d64_b128", 1, 2, 64, 1024, 1024, 128, 0.5, 0.5), 0.3),
    # n_new = 144: two pooled tiles, five bitmask words per query block
    (_case("b64_two_pooled_tiles", 1, 2, 128, 8192, 4096, 64, 0.25, 0.5), 0.0625),
    # every query block on the Taylor path (the exact-item launch has no work)
    (_case("all_taylor", 1, 2, 128, 1024, 1024, 128, 0.25, 1.0), 0.2),
    # nothing kept from the context: K_new is the source part only
    (_case("no_context", 1, 2, 128, 1024, 1024, 64, 0.0, 0.5), 0.125),
    # k_ns = 1
    (_case("one_block", 1, 2, 128, 2048, 1024, 128, 0.5, 0.5), 0.01),
    # alpha_ns = 1: every block exact, all pooled rows masked; Taylor rows become exact attention
    (_case("ns_all", 1, 2, 128, 1024, 1024, 128, 0.5, 0.5), 1.0),
    # several batches and heads
    (_case("b2_h2", 2, 2, 128, 768, 512, 64, 0.5, 0.25), 0.2),
]


@pytest.mark.parametrize("w,a_ns", CASES, ids=[c[0].name for c in CASES])
def test_small_full_parity_ns(w, a_ns):
    q, k, v = ns_inputs(w, a_ns)
    ref = O.isa_forward_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, alpha_ns=a_ns)
    out, sel, route, ns = run_ns(w, a_ns, q, k, v)
    np.testing.assert_array_equal(sel, ref["sel"])
    np.testing.assert_array_equal(route, ref["route"])
    n_new = w.L_src // w.b + sel.shape[-1]
    k_ns = O.no_sparse_block_count(a_ns, n_new)
    assert ns.shape == (w.B, w.H, w.N // w.b, k_ns)
    for bi in range(w.B):
        for h in range(w.H):
            r = O.isa_select_route_ref(q[bi, h], k[bi, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, a_ns)
            # Taylor blocks (margin-checked): bit-exact; exact blocks (unused): a valid ascending set
            np.testing.assert_array_equal(ns[bi, h][r["taylor"]], r["ns_sel"][r["taylor"]])
            for row in ns[bi, h][r["exact"]]:
                assert np.all(np.diff(row) > 0) and row.min() >= 0 and row.max() < n_new
    compare_out(out, ref["out"])


def test_alpha_ns_repeat_runs_bit_identical():
    """The mixed Taylor kernel takes its work items from a per-call counter, so which CTA computes an
    item changes from run to run; every item is computed whole by one CTA, so the outputs may not."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    w = _case("b128_h8", 1, 8, 128, 4096, 4096, 128, 0.25, 0.6)
    q, k, v = ns_inputs(w, 0.0625)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    runs = [isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True, alpha_ns=0.0625)
            for _ in range(3)]
    isa.device_status()
    for other in runs[1:]:
        for x, y in zip(runs[0], other):
            assert torch.equal(x, y)


def test_alpha_ns_zero_equals_plain_entry():
    """isa_forward_ns with alpha_ns = 0 runs exactly the plain pass (bit-identical outputs)."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    w = _case("b128_h3", 1, 3, 128, 1024, 1024, 128, 0.25, 0.6)
    q, k, v = ns_inputs(w, 0.0)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    a = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    b = torch.empty_like(a)
    ws = isa.forward_into(tq, tk, tv, b, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    s = torch.cuda.current_stream().cuda_stream
    rc = isa.lib().isa_forward_ns(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), w.B, w.H, w.L_src, w.L_ctx, w.D,
                                  w.b, w.alpha_s, w.alpha_f, 0.0, isa.ISA_BF16, b.data_ptr(), None, None, None,
                                  ws.data_ptr(), ws.numel(), s)
    assert rc == 0, isa.last_error()
    isa.device_status()
    assert torch.equal(a, b)


def test_alpha_ns_changes_only_taylor_rows():
    """Exact-path rows are the same with and without alpha_ns; Taylor rows move toward exact attention."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    w = _case("b128_long", 1, 2, 128, 4096, 4096, 128, 0.25, 0.5)
    q, k, v = ns_inputs(w, 0.0625)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    plain, _, route = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
    mixed = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, alpha_ns=0.0625)
    isa.device_status()
    n_q, _, n_flat = isa.plan(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f)
    route = route.cpu().numpy()
    for h in range(w.H):
        exact_rows = np.concatenate([np.arange(i * w.b, (i + 1) * w.b) for i in route[0, h, :n_q - n_flat]])
        taylor_rows = np.concatenate([np.arange(i * w.b, (i + 1) * w.b) for i in route[0, h, n_q - n_flat:]])
        assert torch.equal(plain[0, h, exact_rows], mixed[0, h, exact_rows])
        assert not torch.equal(plain[0, h, taylor_rows], mixed[0, h, taylor_rows])


def test_alpha_ns_rejects_f32():
    import torch
    import block_sparse_attention_isa_b200 as isa
    x = torch.zeros((1, 2, 1024, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(isa.IsaError):
        isa.forward(x, x, x, 512, 512, 64, 0.5, 0.5, alpha_ns=0.1)


# ---------------------------------------------------------------- full size

ROWS_PER_BLOCK = 2
BLOCKS_PER_HEAD = 6
ALPHA_NS_FULL = 0.0625
WHOLE_HEADS_NS = 2  # heads compared in every row of the exact blocks and the margin-clear Taylor blocks


def _slice_work_ns(args):
    """Worker: stages 1-3 of the oracle with alpha_ns, then either the whole slice (rows of the
    exact blocks and of every margin-clear Taylor block) or sampled rows of margin-clear Taylor blocks."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import isa_synth as S
    from oracle import isa_oracle as O
    from threadpoolctl import threadpool_limits
    name, bi, h, attempt, a_ns, margin, whole, threads = args
    w = S.all_workloads()[name]
    q, k, v = S.make_slice(w, 0, bi, h, attempt)
    with threadpool_limits(limits=threads):
        sr = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, a_ns)
        clear = np.array([i for i in sr["taylor"] if sr["ns_row_margin"][i] >= margin], np.int64)
        if whole:
            full = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, alpha_ns=a_ns)
            blk = np.sort(np.concatenate([sr["exact"], clear]))
            rows = (blk[:, None] * w.b + np.arange(w.b)[None, :]).ravel()
            ref_rows = full["out"][rows]
        else:
            rng = np.random.default_rng([bi, h, 11])
            blk = rng.choice(clear, size=min(BLOCKS_PER_HEAD, len(clear)), replace=False) if len(clear) else clear
            rows = np.array(sorted(int(i) * w.b + int(o) for i in blk for o in rng.integers(0, w.b, ROWS_PER_BLOCK)),
                            np.int64)
            rows = np.unique(rows)
            ref_rows = O.isa_rows_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, rows, sr=sr,
                                      alpha_ns=a_ns)
    return (bi, h, q, k, v, sr["sel"], np.concatenate([sr["exact"], sr["taylor"]]), clear, sr["ns_sel"], rows,
            ref_rows, len(sr["taylor"]), whole)


def test_full_size_32k_alpha_ns():
    """The 32K-token workload at alpha_ns = 0.0625 (k_ns = 10 of 160 K_new blocks)."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    w = isa_synth.WORKLOADS["bf16_n32768_b128"]
    table = isa_synth.load_attempts()
    att = isa_synth.attempts_for(w, 0, table)
    assert att is not None
    threads_whole = max(1, (os.cpu_count() or 4) // WHOLE_HEADS_NS)
    jobs = [(w.name, bi, h, int(att[bi, h]), ALPHA_NS_FULL, MARGIN, bi * w.H + h < WHOLE_HEADS_NS,
             threads_whole if bi * w.H + h < WHOLE_HEADS_NS else 1) for bi in range(w.B) for h in range(w.H)]
    pool = mp.get_context("spawn").Pool(max(2, min(16, (os.cpu_count() or 4) - 1)))
    try:
        res = pool.map(_slice_work_ns, jobs, chunksize=1)
    finally:
        pool.terminate()
    dev = torch.device("cuda")
    shape = (w.B, w.H, w.N, w.D)
    tq, tk, tv = (torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(3))
    for bi, h, q, k, v, *_ in res:
        tq[bi, h].copy_(torch.from_numpy(q))
        tk[bi, h].copy_(torch.from_numpy(k))
        tv[bi, h].copy_(torch.from_numpy(v))
    out, sel, route, ns = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True,
                                      alpha_ns=ALPHA_NS_FULL)
    isa.device_status()
    assert torch.isfinite(out).all()
    vmin, vmax = tv.float().amin(dim=2, keepdim=True), tv.float().amax(dim=2, keepdim=True)
    o = out.float()
    assert bool(((o >= vmin - MAX_ABS) & (o <= vmax + MAX_ABS)).all())
    sel_h, route_h, ns_h, out_h = sel.cpu().numpy(), route.cpu().numpy(), ns.cpu().numpy(), o.cpu().numpy()
    diffs, refs, n_clear, n_taylor, n_whole = [], [], 0, 0, 0
    for bi, h, q, k, v, sel_ref, route_ref, clear, ns_ref, rows, ref_rows, nt, whole in res:
        np.testing.assert_array_equal(sel_h[bi, h], sel_ref)
        np.testing.assert_array_equal(route_h[bi, h], route_ref)
        np.testing.assert_array_equal(ns_h[bi, h][clear], ns_ref[clear], err_msg=f"exact blocks, slice {bi},{h}")
        n_clear += len(clear)
        n_taylor += nt
        if whole:
            n_whole += 1
            d = out_h[bi, h, rows] - ref_rows
            ma, rl = float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(ref_rows))
            assert ma <= MAX_ABS and rl <= REL_L2, f"whole head {bi},{h}: max-abs {ma:.3e}, rel-L2 {rl:.3e}"
        elif len(rows):
            diffs.append(out_h[bi, h, rows] - ref_rows)
            refs.append(ref_rows)
    assert n_whole == WHOLE_HEADS_NS
    assert n_clear >= n_taylor // 2, (n_clear, n_taylor)
    d, r = np.concatenate(diffs), np.concatenate(refs)
    max_abs, rel = float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(r))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"sampled rows: max-abs {max_abs:.3e}, rel-L2 {rel:.3e}"
