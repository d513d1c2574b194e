"""Pins of the ragged-length oracle (L_src, L_ctx not multiples of b).

Each check compares the oracle with something independent of it: a brute-force
enumeration of the block partition, the whole-block oracle (itself pinned in
test_oracle_pins.py) on lengths that are multiples of b, plain softmax
attention written out where the method reduces to it, and scalar loops for the
selection and routing of a tiny case. A short last block is present in every
ragged case, so that a wrong block length (b instead of the block's own) fails
one of them.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import isa_oracle as O
from oracle import isa_oracle_ragged as R


def _qkv(N, D, seed, spread=1.0):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(N, D)) * spread, rng.normal(size=(N, D)) * spread, rng.normal(size=(N, D)))


def _softmax_attention(q, k, v):
    """Written out: out[i] = sum_t exp(s_it - max_t s_it) v[t] / sum_t exp(s_it - max_t s_it)."""
    s = np.einsum("id,td->it", q, k) / math.sqrt(q.shape[1])
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return np.einsum("it,td->id", e, v) / e.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5])
def test_block_bounds_brute_force(b):
    for L_src, L_ctx in itertools.product(range(1, 14), range(1, 14)):
        bounds = R.block_bounds(L_src, L_ctx, b)
        assert len(bounds) == -(-L_src // b) + -(-L_ctx // b)
        covered = [t for s, e in bounds for t in range(s, e)]
        assert covered == list(range(L_src + L_ctx))               # every token once, in order
        n_src = -(-L_src // b)
        for i, (s, e) in enumerate(bounds):
            assert 0 < e - s <= b
            assert (e <= L_src) if i < n_src else (s >= L_src)       # no block straddles the boundary
            last_of_part = i in (n_src - 1, len(bounds) - 1)
            assert last_of_part or e - s == b                        # only a part's last block is short


@pytest.mark.parametrize("L_src,L_ctx,b,a_s,a_f,a_ns", [
    (512, 512, 64, 0.5, 0.5, 0.0), (768, 512, 128, 0.25, 0.6, 0.0), (640, 448, 64, 0.3, 0.5, 0.25),
    (1024, 512, 64, 1.0, 0.0, 0.0), (512, 1024, 128, 0.5, 1.0, 0.4),
])
def test_whole_blocks_match_the_whole_block_oracle(L_src, L_ctx, b, a_s, a_f, a_ns):
    q, k, v = _qkv(L_src + L_ctx, 32, 7)
    r = R.isa_slice_ref_ragged(q, k, v, L_src, L_ctx, b, a_s, a_f, a_ns)
    p = O.isa_slice_ref(q, k, v, L_src, L_ctx, b, a_s, a_f, alpha_ns=a_ns)
    np.testing.assert_array_equal(r["sel"], p["sel"])
    np.testing.assert_array_equal(r["route"], p["route"])
    if a_ns:
        np.testing.assert_array_equal(r["ns_sel"], p["ns_sel"])
    np.testing.assert_allclose(r["out"], p["out"], rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("L_src,L_ctx,b", [(150, 100, 64), (65, 63, 64), (200, 1, 128), (1, 300, 128)])
def test_dense_point_is_softmax_attention(L_src, L_ctx, b):
    """alpha_s = 1, alpha_f = 0: every context block kept, every query block exact."""
    q, k, v = _qkv(L_src + L_ctx, 16, 3)
    r = R.isa_slice_ref_ragged(q, k, v, L_src, L_ctx, b, 1.0, 0.0)
    assert r["k_new"].shape[0] == L_src + L_ctx
    np.testing.assert_allclose(r["out"], _softmax_attention(q, k, v), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("a_s", [1.0, 0.5])
@pytest.mark.parametrize("L_src,L_ctx,b", [(150, 100, 64), (97, 131, 32)])
def test_block_constant_keys_make_taylor_exact(L_src, L_ctx, b, a_s):
    """alpha_f = 1 with every key of a block equal: a block j then contributes exactly
    len_j * exp(q . kappa_j / sqrt(D)) * mean(V_j), so the Taylor path equals softmax
    attention over K_new, short blocks included (a weight of b would not)."""
    N = L_src + L_ctx
    q, _, v = _qkv(N, 16, 5)
    bounds = R.block_bounds(L_src, L_ctx, b)
    kappa = np.random.default_rng(9).normal(size=(len(bounds), 16))
    k = np.empty((N, 16))
    for i, (s, e) in enumerate(bounds):
        k[s:e] = kappa[i]
    r = R.isa_slice_ref_ragged(q, k, v, L_src, L_ctx, b, a_s, 1.0)
    assert len(r["taylor"]) == len(bounds)
    np.testing.assert_allclose(r["out"], _softmax_attention(q, r["k_new"], r["v_new"]), rtol=1e-10, atol=1e-12)
    if a_s == 1.0:
        np.testing.assert_allclose(r["out"], _softmax_attention(q, k, v), rtol=1e-10, atol=1e-12)


def test_gather_keeps_whole_short_blocks():
    L_src, L_ctx, b = 10, 11, 4          # context blocks [10,14) [14,18) [18,21)
    q, k, v = _qkv(L_src + L_ctx, 3, 1)
    bounds = R.block_bounds(L_src, L_ctx, b)
    k_new, v_new, nb = R.gather_kv_ragged(k, v, np.array([0, 2]), bounds, 3)
    rows = list(range(10)) + [10, 11, 12, 13] + [18, 19, 20]
    np.testing.assert_array_equal(k_new, k[rows])
    np.testing.assert_array_equal(v_new, v[rows])
    assert nb == [(0, 4), (4, 8), (8, 10), (10, 14), (14, 17)]


def _loops_select_route(q, k, L_src, L_ctx, b, a_s, a_f):
    """Stages 1-3 in scalar Python loops, from the token positions up (q, k: lists of rows)."""
    N, D = len(q), len(q[0])
    blk = [t // b if t < L_src else -(-L_src // b) + (t - L_src) // b for t in range(N)]
    n_q = max(blk) + 1
    n_src = -(-L_src // b)
    mean = lambda x, i: [sum(x[t][d] for t in range(N) if blk[t] == i) / blk.count(i) for d in range(D)]
    qc = [mean(q, i) for i in range(n_q)]
    kc = [mean(k, i) for i in range(n_q)]

    def soft(row):
        m = max(row)
        e = [math.exp(x - m) for x in row]
        return [x / sum(e) for x in e]
    dot = lambda a, c: sum(a[d] * c[d] for d in range(D)) / math.sqrt(D)
    S = [soft([dot(qc[i], kc[j]) for j in range(n_q)]) for i in range(n_q)]
    n_ctx = n_q - n_src
    col = [sum(S[i][n_src + c] for i in range(n_src)) / n_src for c in range(n_ctx)]
    kk = max(0, min(n_ctx, math.ceil(float(np.float32(a_s)) * n_ctx - 1e-4)))
    sel = sorted(sorted(range(n_ctx), key=lambda c: (-col[c], c))[:kk])
    new = list(range(n_src)) + [n_src + c for c in sel]
    M = []
    for i in range(n_q):
        p = soft([dot(qc[i], kc[j]) for j in new])
        M.append(sum((x - 1.0 / len(new)) ** 2 for x in p) / len(new))
    n_flat = max(0, min(n_q, math.floor(float(np.float32(a_f)) * n_q + 1e-4)))
    order = sorted(range(n_q), key=lambda i: (M[i], i))
    return sel, sorted(order[n_flat:]) + sorted(order[:n_flat])


@pytest.mark.parametrize("L_src,L_ctx,b,a_s,a_f", [(10, 7, 4, 0.5, 0.5), (9, 13, 4, 0.34, 0.4), (5, 5, 3, 1.0, 0.25)])
def test_selection_and_routing_against_loops(L_src, L_ctx, b, a_s, a_f):
    q, k, _ = _qkv(L_src + L_ctx, 3, 11, spread=2.0)
    sel, route = _loops_select_route(q.tolist(), k.tolist(), L_src, L_ctx, b, a_s, a_f)
    r = R.isa_select_route_ragged(q, k, L_src, L_ctx, b, a_s, a_f)
    assert r["topk_margin"] > 1e-9 and r["route_margin"] > 1e-9
    assert list(r["sel"]) == sel
    assert list(np.concatenate([r["exact"], r["taylor"]])) == route


def test_no_sparsity_limits_on_ragged_blocks():
    """alpha_ns = 1: every K_new block key by key, so Taylor rows are softmax attention over
    K_new; alpha_ns = 0: the plain length-weighted Taylor path."""
    L_src, L_ctx, b = 150, 100, 64
    q, k, v = _qkv(L_src + L_ctx, 16, 13)
    full = R.isa_slice_ref_ragged(q, k, v, L_src, L_ctx, b, 0.5, 1.0, alpha_ns=1.0)
    np.testing.assert_allclose(full["out"], _softmax_attention(q, full["k_new"], full["v_new"]),
                               rtol=1e-10, atol=1e-12)
    none = R.isa_slice_ref_ragged(q, k, v, L_src, L_ctx, b, 0.5, 1.0, alpha_ns=0.0)
    np.testing.assert_allclose(none["out"], R.taylor_rows_ragged(q, none["k_new"], none["v_new"],
                                                                 none["new_bounds"]), rtol=1e-12)
