"""Pins for the CPU oracle: closed forms, library routines, brute force, invariants.

Each test ties the oracle to something other than itself, so that a plausible
slip in it (a dropped 1/sqrt(D), a reversed sort, the wrong key set, a
transposed operand) fails at least one of them. ``test_planted_mistakes``
plants such slips in the oracle and checks that they are caught.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import isa_oracle as O
import isa_synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
E = math.e


def _sdpa(q, k, v, mask=None):
    """torch's scaled_dot_product_attention in float64 on the CPU (default scale 1/sqrt(D))."""
    tq = torch.from_numpy(np.asarray(q, np.float64))[None, None]
    tk = torch.from_numpy(np.asarray(k, np.float64))[None, None]
    tv = torch.from_numpy(np.asarray(v, np.float64))[None, None]
    m = None if mask is None else torch.from_numpy(np.array(mask, bool))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m)[0, 0].numpy()


def _small(D=16, b=8, L_src=64, L_ctx=64, a_s=0.5, a_f=0.5, sig=(0.1, 1.0), s_ctx=0.5, dtype="f32"):
    return isa_synth.Workload("t", 1, 1, D, L_src, L_ctx, b, a_s, a_f, sig[0], sig[1], s_ctx, dtype)


def _ctx_mask(w, sel):
    """Key mask that keeps every source key and the keys of the kept context blocks."""
    t = np.arange(w.N)
    keep = t < w.L_src
    for c in sel:
        keep |= (t >= w.L_src + c * w.b) & (t < w.L_src + (c + 1) * w.b)
    return np.broadcast_to(keep, (w.N, w.N))


# ----------------------------------------------------------------------------- worked example

def _worked():
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        return json.load(f)


def test_worked_example_closed_forms():
    ex = _worked()
    q, k, v = (np.array(ex[n], np.float64) for n in ("q", "k", "v"))
    r = O.isa_slice_ref(q, k, v, ex["L_src"], ex["L_ctx"], ex["b"], ex["alpha_s"], ex["alpha_f"])
    np.testing.assert_allclose(r["qc"], [[2, 0, 0, 0], [0, 4, 0, 0], [0, 0, 0, 0], [-2, 0, 0, 0]], atol=0)
    np.testing.assert_allclose(r["kc"], [[1, 0, 0, 0], [0, 1, 0, 0], [1, 1, 0, 0], [0, 0, 0, 0]], atol=0)
    s0 = np.array([E, 1, E, 1]) / (2 * E + 2)
    s1 = np.array([1, E**2, E**2, 1]) / (2 * E**2 + 2)
    np.testing.assert_allclose(r["s_coarse"][0], s0, rtol=1e-14)
    np.testing.assert_allclose(r["s_coarse"][1], s1, rtol=1e-14)
    col = [(E / (2 * E + 2) + E**2 / (2 * E**2 + 2)) / 2, (1 / (2 * E + 2) + 1 / (2 * E**2 + 2)) / 2]
    np.testing.assert_allclose(r["colscore"], col, rtol=1e-14)
    assert r["sel"].tolist() == ex["expected"]["sel"]

    def var3(logits):
        p = np.exp(np.array(logits, float))
        p /= p.sum()
        return ((p - 1 / 3) ** 2).sum() / 3

    m = [var3([1, 0, 1]), var3([0, 2, 2]), 0.0, var3([-1, 0, -1])]
    np.testing.assert_allclose(r["sharp"], m, rtol=1e-13, atol=1e-17)
    assert r["route"].tolist() == ex["expected"]["route"]

    out = r["out"]
    exp_rows = {
        0: np.array([E, 1, E, 0]) / (2 * E + 1),
        1: np.array([1, E**2, E**2, 0]) / (2 * E**2 + 1),
        2: np.array([1, 1, 1, 0]) / 3,
        3: np.array([1 / E, 1, 1 / E, 0]) / (1 + 2 / E),
    }
    for blk, val in exp_rows.items():
        for t in range(2):
            np.testing.assert_allclose(out[blk * 2 + t], val, rtol=1e-13, atol=1e-15)


def test_taylor_vs_exact_closed_form():
    ex = _worked()["taylor_vs_exact"]
    q, kn, vn = (np.array(ex[n], np.float64) for n in ("q", "k_new", "v_new"))
    np.testing.assert_allclose(O.exact_rows(q, kn, vn)[0], np.array([E, 1 / E, 2, 0]) / (E + 1 / E + 2), rtol=1e-14)
    np.testing.assert_allclose(O.taylor_rows(q, kn, vn, 2)[0], [0.25, 0.25, 0.5, 0.0], rtol=1e-14, atol=1e-16)


# ----------------------------------------------------------------------------- reductions to textbook routines

@pytest.mark.parametrize("b,D", [(8, 16), (16, 32)])
def test_dense_point_equals_sdpa(b, D):
    """alpha_s = 1 keeps every context block and alpha_f = 0 routes nothing to Taylor: dense attention."""
    w = _small(D=D, b=b, L_src=96 if b == 8 else 128, L_ctx=64, a_s=1.0, a_f=0.0)
    q, k, v = isa_synth.make_slice(w, 3, 0, 0)
    r = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, 1.0, 0.0)
    assert r["sel"].tolist() == list(range(w.L_ctx // b))
    assert len(r["taylor"]) == 0
    np.testing.assert_allclose(r["out"], _sdpa(q, k, v), rtol=0, atol=1e-12)


def test_exact_path_with_preselection_equals_masked_sdpa():
    """alpha_f = 0: every query attends to the source keys plus the kept context blocks."""
    w = _small(a_s=0.25, a_f=0.0)
    q, k, v = isa_synth.make_slice(w, 5, 0, 1)
    r = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, 0.0)
    assert len(r["sel"]) == 2
    np.testing.assert_allclose(r["out"], _sdpa(q, k, v, _ctx_mask(w, r["sel"])), rtol=0, atol=1e-12)


@pytest.mark.parametrize("a_s", [1.0, 0.25])
def test_taylor_equals_dense_when_keys_constant_in_blocks(a_s):
    """With every key of a block equal to its mean, 0th-order Taylor is exact (alpha_f = 1)."""
    w = _small(a_s=a_s, a_f=1.0)
    q, k, v = isa_synth.make_slice(w, 7, 0, 0, sigma_override=(1.0, 0.0, 1.0))
    r = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, a_s, 1.0)
    assert len(r["exact"]) == 0
    mask = None if a_s == 1.0 else _ctx_mask(w, r["sel"])
    np.testing.assert_allclose(r["out"], _sdpa(q, k, v, mask), rtol=0, atol=1e-12)


def test_block_size_one_taylor_is_dense():
    """b = 1: pooling is the identity, so the Taylor path is dense attention over the kept keys."""
    w = _small(D=8, b=1, L_src=24, L_ctx=16, a_s=0.5, a_f=1.0)
    q, k, v = isa_synth.make_slice(w, 11, 0, 0)
    r = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, 1, 0.5, 1.0)
    np.testing.assert_allclose(r["out"], _sdpa(q, k, v, _ctx_mask(w, r["sel"])), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- brute force on tiny inputs

def test_topk_brute_force():
    """n_ctx = 8, k = 4: the chosen set is the unique 4-subset with the largest total score."""
    w = _small(D=16, b=8, L_src=64, L_ctx=64, a_s=0.5)
    for seed in range(6):
        q, k, v = isa_synth.make_slice(w, seed, 0, 0)
        r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
        sc = r["colscore"]
        best = max(itertools.combinations(range(8), 4), key=lambda s: sum(sc[list(s)]))
        assert r["sel"].tolist() == list(best)
        # every kept block scores at least as high as every dropped block
        dropped = [c for c in range(8) if c not in best]
        assert min(sc[list(best)]) > max(sc[dropped])


def test_routing_brute_force():
    """n_q = 16, n_flat = 8: the Taylor set is the unique 8-subset with the smallest total sharpness."""
    w = _small(D=16, b=8, L_src=64, L_ctx=64, a_s=0.5, a_f=0.5)
    for seed in range(3):
        q, k, v = isa_synth.make_slice(w, seed, 0, 1)
        r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
        m = r["sharp"]
        best = min(itertools.combinations(range(16), 8), key=lambda s: sum(m[list(s)]))
        assert r["taylor"].tolist() == list(best)
        assert sorted(r["exact"].tolist() + r["taylor"].tolist()) == list(range(16))


def test_sharpness_brute_force_loops():
    """Sharpness against a per-block loop over keys written with Python floats."""
    w = _small(D=8, b=4, L_src=16, L_ctx=16, a_s=0.5)
    q, k, v = isa_synth.make_slice(w, 2, 0, 0)
    r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    # pooled keys of K_new, built from the gathered tokens rather than from Kc
    k_new, _ = O.gather_kv(k, v, r["sel"], w.L_src, w.b)
    n_new = k_new.shape[0] // w.b
    for i in range(w.N // w.b):
        qc = [sum(float(q[i * w.b + t, d]) for t in range(w.b)) / w.b for d in range(w.D)]
        logits = []
        for j in range(n_new):
            kc = [sum(float(k_new[j * w.b + t, d]) for t in range(w.b)) / w.b for d in range(w.D)]
            logits.append(sum(a * c for a, c in zip(qc, kc)) / math.sqrt(w.D))
        mx = max(logits)
        ex = [math.exp(z - mx) for z in logits]
        p = [e / sum(ex) for e in ex]
        mean = sum(p) / n_new
        var = sum((x - mean) ** 2 for x in p) / n_new
        assert abs(var - r["sharp"][i]) <= 1e-15 + 1e-12 * var


# ----------------------------------------------------------------------------- invariants

def test_coarse_rows_sum_to_one_and_variance_identity():
    w = _small()
    q, k, v = isa_synth.make_slice(w, 1, 0, 0)
    r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    np.testing.assert_allclose(r["s_coarse"].sum(axis=1), 1.0, rtol=0, atol=1e-14)
    p = O.coarse_scores(r["qc"], r["kc_new"])
    n = p.shape[1]
    np.testing.assert_allclose(r["sharp"], (p**2).sum(1) / n - 1.0 / n**2, rtol=0, atol=1e-15)


def test_permutation_inside_blocks_changes_nothing_pooled():
    w = _small(D=16, b=8)
    q, k, v = isa_synth.make_slice(w, 4, 0, 0)
    r1 = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    rng = np.random.default_rng(0)
    perm = np.concatenate([blk * w.b + rng.permutation(w.b) for blk in range(w.N // w.b)])
    r2 = O.isa_slice_ref(q[perm], k[perm], v[perm], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    np.testing.assert_allclose(r1["qc"], r2["qc"], atol=1e-15)
    np.testing.assert_allclose(r1["kc"], r2["kc"], atol=1e-15)
    assert r1["sel"].tolist() == r2["sel"].tolist()
    assert r1["route"].tolist() == r2["route"].tolist()


def test_context_block_permutation_permutes_selection():
    w = _small(D=16, b=8)
    q, k, v = isa_synth.make_slice(w, 6, 0, 0)
    r1 = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    n_ctx = w.L_ctx // w.b
    pc = np.random.default_rng(1).permutation(n_ctx)  # new block c holds old block pc[c]
    rows = np.arange(w.N)
    for c in range(n_ctx):
        rows[w.L_src + c * w.b:w.L_src + (c + 1) * w.b] = w.L_src + pc[c] * w.b + np.arange(w.b)
    r2 = O.isa_select_route_ref(q[rows], k[rows], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    assert sorted(pc[r2["sel"]].tolist()) == r1["sel"].tolist()


def test_outputs_are_convex_combinations():
    w = _small(a_s=0.25, a_f=0.5)
    q, k, v = isa_synth.make_slice(w, 8, 0, 0)
    r = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    _, v_new = O.gather_kv(k, v, r["sel"], w.L_src, w.b)
    lo, hi = v_new.min(0), v_new.max(0)
    assert (r["out"] >= lo - 1e-12).all() and (r["out"] <= hi + 1e-12).all()


def test_kv_length_after_preselection():
    w = _small(a_s=0.25)
    q, k, v = isa_synth.make_slice(w, 9, 0, 0)
    r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    k_new, v_new = O.gather_kv(k, v, r["sel"], w.L_src, w.b)
    assert k_new.shape[0] == v_new.shape[0] == w.L_src + r["k"] * w.b


# ----------------------------------------------------------------------------- integer counts

@pytest.mark.parametrize("a_s,n_ctx,k", [(0.5, 8, 4), (0.25, 64, 16), (0.25, 128, 32), (0.1, 200, 20),
                                         (0.25, 200, 50), (0.5, 200, 100), (1.0, 200, 200), (0.125, 128, 16),
                                         (0.3, 10, 3), (0.31, 10, 4), (0.0, 10, 0)])
def test_kept_context_blocks(a_s, n_ctx, k):
    assert O.kept_context_blocks(a_s, n_ctx) == k


@pytest.mark.parametrize("a_f,n_q,n", [(0.5, 16, 8), (0.6, 256, 153), (0.5, 128, 64), (0.3, 400, 120),
                                       (0.7, 400, 280), (0.0, 400, 0), (1.0, 400, 400), (0.5, 256, 128)])
def test_taylor_block_count(a_f, n_q, n):
    assert O.taylor_block_count(a_f, n_q) == n


def test_margins_closed_form():
    assert O.topk_margin(np.array([0.5, 0.3, 0.2]), 1) == pytest.approx((0.5 - 0.3) / 0.5)
    assert O.topk_margin(np.array([0.5, 0.3, 0.2]), 3) == math.inf
    assert O.route_margin(np.array([0.4, 0.1, 0.2]), 2) == pytest.approx((0.4 - 0.2) / 0.4)
    assert O.route_margin(np.array([0.4, 0.1, 0.2]), 0) == math.inf


def test_executed_flops_headline_by_hand():
    f = O.executed_flops(1, 40, 16384, 16384, 128, 128, 0.25, 0.6)
    # k = 32 kept blocks, L_new = 16384 + 32*128 = 20480; 153 Taylor and 103 exact query blocks
    assert f["exact"] == 4 * 103 * 128 * 20480 * 128 * 40
    assert f["taylor"] == 4 * 153 * 128 * 160 * 128 * 40
    assert f["dense"] == 4 * 32768 * 32768 * 128 * 40


# ----------------------------------------------------------------------------- planted mistakes

def _pins_pass():
    """Run the pins that do not need parametrisation; True when all pass."""
    try:
        test_worked_example_closed_forms()
        test_taylor_vs_exact_closed_form()
        test_dense_point_equals_sdpa(8, 16)
        test_exact_path_with_preselection_equals_masked_sdpa()
        test_taylor_equals_dense_when_keys_constant_in_blocks(0.25)
        test_routing_brute_force()
        test_sharpness_brute_force_loops()
    except AssertionError:
        return False
    return True


def _mut_no_scale(qc, kc):
    return O._softmax_rows(np.asarray(qc, float) @ np.asarray(kc, float).T)


def _mut_route_reversed(m, n_flat):
    order = sorted(range(len(m)), key=lambda i: (-float(m[i]), i))
    return np.array(sorted(order[n_flat:]), np.int64), np.array(sorted(order[:n_flat]), np.int64)


def _mut_sharp_all_keys(qc, kc_new):
    # wrong key set: pads Kc_new with a zero block as if an extra block were kept
    kc = np.vstack([kc_new, np.zeros((1, kc_new.shape[1]))])
    p = O.coarse_scores(qc, kc)
    n = p.shape[1]
    return ((p - 1.0 / n) ** 2).sum(axis=1) / n


def _mut_exact_transposed(q_rows, k_new, v_new):
    d = q_rows.shape[1]
    s = (np.asarray(q_rows, float) @ np.asarray(k_new, float).T) / math.sqrt(d)
    p = np.exp(s - s.max(0, keepdims=True))
    p = p / p.sum(0, keepdims=True)  # normalised over queries instead of keys
    return p @ np.asarray(v_new, float)


def _mut_taylor_no_pool(q_rows, k_new, v_new, b):
    d = q_rows.shape[1]
    kc = k_new[::b]  # first token instead of the block mean
    vc = O.pool_blocks(v_new, b)
    s = (np.asarray(q_rows, float) @ kc.T) / math.sqrt(d)
    p = np.exp(s - s.max(1, keepdims=True))
    return (p @ vc) / p.sum(1, keepdims=True)


def _mut_select_smallest(score, k):
    order = sorted(range(len(score)), key=lambda c: (float(score[c]), c))
    return np.array(sorted(order[:k]), np.int64)


def _mut_colscore_all_rows(s_coarse, n_src):
    return s_coarse[:, n_src:].mean(axis=0)


@pytest.mark.parametrize("name,fn", [
    ("coarse_scores", _mut_no_scale),
    ("route_blocks", _mut_route_reversed),
    ("sharpness", _mut_sharp_all_keys),
    ("exact_rows", _mut_exact_transposed),
    ("taylor_rows", _mut_taylor_no_pool),
    ("select_context_blocks", _mut_select_smallest),
    ("context_scores", _mut_colscore_all_rows),
])
def test_planted_mistakes(monkeypatch, name, fn):
    assert _pins_pass()
    monkeypatch.setattr(O, name, fn)
    assert not _pins_pass(), f"a planted mistake in {name} went unnoticed"


# ----------------------------------------------------------------------------- no-sparsity ratio alpha_ns

@pytest.mark.parametrize("a_ns,n_new,k", [(0.0, 160, 0), (0.0625, 160, 10), (0.0625, 16, 1), (0.0625, 24, 2),
                                          (1.0, 37, 37), (0.1, 200, 20), (0.5, 5, 3)])
def test_no_sparse_block_count(a_ns, n_new, k):
    assert O.no_sparse_block_count(a_ns, n_new) == k


def test_no_sparse_blocks_brute_force():
    rng = np.random.default_rng(11)
    for _ in range(200):
        n = int(rng.integers(1, 12))
        row = rng.integers(0, 4, size=n).astype(float) / 7.0  # many ties
        for k_ns in range(n + 1):
            ranked = sorted(((-row[j], j) for j in range(n)))
            want = sorted(j for _, j in ranked[:k_ns])
            assert O.no_sparse_blocks(row, k_ns).tolist() == want


def _mixed_by_loops(q_rows, k_new, v_new, b, exact_blocks):
    """The definition's sums written out with scalar loops: exact keys with weight 1, every
    other block's pooled key and value with weight b, then the ratio."""
    d = q_rows.shape[1]
    n_new = k_new.shape[0] // b
    out = np.zeros((q_rows.shape[0], d))
    for r in range(q_rows.shape[0]):
        terms = []  # (score, weight, value vector)
        for j in range(n_new):
            if j in exact_blocks:
                for t in range(j * b, (j + 1) * b):
                    s = sum(float(q_rows[r, x]) * float(k_new[t, x]) for x in range(d)) / math.sqrt(d)
                    terms.append((s, 1.0, [float(v_new[t, x]) for x in range(d)]))
            else:
                kc = [sum(float(k_new[t, x]) for t in range(j * b, (j + 1) * b)) / b for x in range(d)]
                vc = [sum(float(v_new[t, x]) for t in range(j * b, (j + 1) * b)) / b for x in range(d)]
                s = sum(float(q_rows[r, x]) * kc[x] for x in range(d)) / math.sqrt(d)
                terms.append((s, float(b), vc))
        num = [0.0] * d
        den = 0.0
        for s, wgt, vec in terms:
            e = wgt * math.exp(s)
            den += e
            for x in range(d):
                num[x] += e * vec[x]
        out[r] = [n / den for n in num]
    return out


def test_mixed_taylor_brute_force_loops():
    rng = np.random.default_rng(3)
    for b, n_new, D in [(2, 4, 3), (3, 5, 2), (4, 3, 4)]:
        q = rng.standard_normal((5, D))
        k = rng.standard_normal((n_new * b, D))
        v = rng.standard_normal((n_new * b, D))
        for ex in ([], [0], [1, 2], list(range(n_new))):
            np.testing.assert_allclose(O.taylor_mixed_rows(q, k, v, b, ex), _mixed_by_loops(q, k, v, b, ex),
                                       rtol=1e-12, atol=1e-13)


def test_mixed_taylor_limits():
    """No exact block: the plain Taylor path. Every block exact: exact attention over K_new."""
    rng = np.random.default_rng(4)
    b, n_new, D = 8, 6, 16
    q = rng.standard_normal((10, D))
    k = rng.standard_normal((n_new * b, D))
    v = rng.standard_normal((n_new * b, D))
    np.testing.assert_allclose(O.taylor_mixed_rows(q, k, v, b, []), O.taylor_rows(q, k, v, b), rtol=1e-12)
    np.testing.assert_allclose(O.taylor_mixed_rows(q, k, v, b, range(n_new)), _sdpa(q, k, v), rtol=1e-11, atol=1e-13)


def test_mixed_taylor_constant_keys_ignore_selection():
    """Keys constant inside every block: an exact block contributes exp(s_j) * b * Vc_j, the same as
    its pooled stand-in, so any choice of exact blocks gives dense attention."""
    rng = np.random.default_rng(5)
    b, n_new, D = 4, 7, 8
    kc = rng.standard_normal((n_new, D))
    k = np.repeat(kc, b, axis=0)
    v = rng.standard_normal((n_new * b, D))
    q = rng.standard_normal((6, D))
    dense = _sdpa(q, k, v)
    for ex in ([], [3], [0, 6], [1, 2, 4, 5]):
        np.testing.assert_allclose(O.taylor_mixed_rows(q, k, v, b, ex), dense, rtol=1e-11, atol=1e-13)


def test_mixed_taylor_split_and_merge():
    """One softmax over the two key sets equals the merge of the two partial softmaxes
    (running max, sum and unnormalised output), the identity an online softmax relies on."""
    rng = np.random.default_rng(6)
    b, n_new, D = 4, 6, 8
    q = rng.standard_normal((5, D))
    k = rng.standard_normal((n_new * b, D))
    v = rng.standard_normal((n_new * b, D))
    ex = [1, 4]
    rows = np.concatenate([np.arange(j * b, (j + 1) * b) for j in ex])
    pooled = [j for j in range(n_new) if j not in ex]
    kc, vc = O.pool_blocks(k, b)[pooled], O.pool_blocks(v, b)[pooled]
    s1 = q @ k[rows].T / math.sqrt(D)
    s2 = q @ kc.T / math.sqrt(D) + math.log(b)  # weight b as a score bias
    parts = []
    for s, vv in ((s1, v[rows]), (s2, vc)):
        m = s.max(1, keepdims=True)
        p = np.exp(s - m)
        parts.append((m, p.sum(1, keepdims=True), p @ vv))
    m = np.maximum(parts[0][0], parts[1][0])
    l = sum(li * np.exp(mi - m) for mi, li, _ in parts)
    o = sum(oi * np.exp(mi - m) for mi, _, oi in parts)
    np.testing.assert_allclose(o / l, O.taylor_mixed_rows(q, k, v, b, ex), rtol=1e-12)


def test_slice_with_no_sparse_blocks():
    """A whole slice at alpha_ns = 0 is unchanged; at alpha_ns > 0 only the Taylor rows change, each
    flat block using its own top coarse-score key blocks."""
    w = _small(D=16, b=8, L_src=64, L_ctx=64, a_s=0.5, a_f=0.5)
    q, k, v = isa_synth.make_slice(w, 0, 0, 0)
    base = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    same = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, alpha_ns=0.0)
    np.testing.assert_array_equal(base["out"], same["out"])
    ns = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, alpha_ns=0.25)
    n_new = ns["kc_new"].shape[0]
    assert ns["k_ns"] == math.ceil(0.25 * n_new) and ns["ns_sel"].shape == (16, ns["k_ns"])
    p = O.coarse_scores(ns["qc"], ns["kc_new"])
    k_new, v_new = O.gather_kv(k, v, ns["sel"], w.L_src, w.b)
    for i in range(16):
        rr = slice(i * w.b, (i + 1) * w.b)
        if i in set(ns["exact"].tolist()):
            np.testing.assert_array_equal(ns["out"][rr], base["out"][rr])
        else:
            want = set(np.argsort(-p[i], kind="stable")[:ns["k_ns"]].tolist())
            assert set(ns["ns_sel"][i].tolist()) == want
            np.testing.assert_allclose(ns["out"][rr], _mixed_by_loops(q[rr], k_new, v_new, w.b, want), rtol=1e-10)


def _mixed_wrong(q_rows, k_new, v_new, b, exact_blocks):
    """A plausible slip: the pooled blocks lose their weight b."""
    d = q_rows.shape[1]
    n_new = k_new.shape[0] // b
    ex = sorted(set(int(j) for j in exact_blocks))
    pooled = [j for j in range(n_new) if j not in ex]
    kc, vc = O.pool_blocks(k_new, b)[pooled], O.pool_blocks(v_new, b)[pooled]
    rows = np.concatenate([np.arange(j * b, (j + 1) * b) for j in ex]) if ex else np.zeros(0, np.int64)
    s = np.concatenate([q_rows @ k_new[rows].T, q_rows @ kc.T], axis=1) / math.sqrt(d)
    p = np.exp(s - s.max(1, keepdims=True))
    vv = np.concatenate([v_new[rows], vc], axis=0)
    return (p @ vv) / p.sum(1, keepdims=True)


def test_planted_mistake_in_mixed_path(monkeypatch):
    monkeypatch.setattr(O, "taylor_mixed_rows", _mixed_wrong)
    with pytest.raises(AssertionError):
        test_mixed_taylor_brute_force_loops()


# ----------------------------------------------------------------------------- isa_rows_ref and no_sparse_margin
# isa_rows_ref is the oracle behind every sampled full-size GPU comparison. It maps rows to
# paths on its own (row // b in the Taylor set), so it is pinned to the whole-slice oracle,
# which the pins above tie to closed forms, library routines and brute force.

@pytest.mark.parametrize("b,a_s,a_f,a_ns", [(8, 0.5, 0.5, 0.0), (8, 0.25, 0.75, 0.0), (16, 1.0, 0.0, 0.0),
                                            (8, 0.5, 1.0, 0.0), (8, 0.5, 0.5, 0.25), (16, 0.5, 0.625, 0.5)])
def test_rows_ref_equals_slice_ref(b, a_s, a_f, a_ns):
    w = _small(b=b, L_src=64, L_ctx=96, a_s=a_s, a_f=a_f)
    q, k, v = isa_synth.make_slice(w, 11, 0, 0, 0)
    full = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, alpha_ns=a_ns)
    rng = np.random.default_rng(5)
    # every row of two whole blocks, scattered rows, the first and the last row
    rows = np.unique(np.concatenate([np.arange(b, 2 * b), np.arange(w.N - b, w.N),
                                     rng.integers(0, w.N, 40), [0, w.N - 1]]))
    got = O.isa_rows_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, rows, alpha_ns=a_ns)
    np.testing.assert_allclose(got, full["out"][rows], rtol=0, atol=1e-13)
    # the same with the stage 1-3 results passed in, as the GPU tests do
    sr = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, a_ns)
    got2 = O.isa_rows_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, rows, sr=sr, alpha_ns=a_ns)
    np.testing.assert_array_equal(got2, got)
    # all rows at once equal the whole slice
    allr = O.isa_rows_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, np.arange(w.N), alpha_ns=a_ns)
    np.testing.assert_allclose(allr, full["out"], rtol=0, atol=1e-13)


def test_rows_ref_catches_a_row_to_block_slip(monkeypatch):
    """A row mapped to the block of its neighbour takes the wrong path and fails the pin above."""
    w = _small(b=8, L_src=64, L_ctx=96, a_s=0.5, a_f=0.5)
    q, k, v = isa_synth.make_slice(w, 11, 0, 0, 0)
    full = O.isa_slice_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    sr = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    taylor = set(int(t) for t in sr["taylor"])
    # rows whose block and the next block take different paths
    rows = np.array([i * w.b for i in range(w.N // w.b - 1) if (i in taylor) != (i + 1 in taylor)])
    assert len(rows)
    wrong = O.isa_rows_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, rows + w.b, sr=sr)
    assert np.abs(wrong - full["out"][rows]).max() > 1e-3


def test_no_sparse_margin_closed_form():
    p = np.array([[0.5, 0.3, 0.2],
                  [0.1, 0.6, 0.3]])
    # k_ns = 1: row 0 (0.5 - 0.3) / 0.5 = 0.4, row 1 (0.6 - 0.3) / 0.6 = 0.5 -> 0.4
    assert O.no_sparse_margin(p, 1) == pytest.approx(0.4, abs=1e-15)
    # k_ns = 2: row 0 (0.3 - 0.2) / 0.3 = 1/3, row 1 (0.3 - 0.1) / 0.3 = 2/3 -> 1/3
    assert O.no_sparse_margin(p, 2) == pytest.approx(1.0 / 3.0, abs=1e-15)
    # a tie at the boundary is a zero margin; no boundary (k_ns = 0 or all blocks) is infinite
    assert O.no_sparse_margin(np.array([[0.4, 0.4, 0.2]]), 1) == 0.0
    assert O.no_sparse_margin(p, 0) == math.inf
    assert O.no_sparse_margin(p, 3) == math.inf
    assert O.no_sparse_margin(np.zeros((0, 3)), 1) == math.inf
    # the margin is invariant to the row order and to a common positive scale of a row
    assert O.no_sparse_margin(p[::-1] * np.array([[3.0], [0.5]]), 1) == pytest.approx(0.4, abs=1e-15)
