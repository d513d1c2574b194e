"""Pins of the backward-pass oracle (the gradient of ISA's output, decisions held fixed).

Each check is independent of autograd: the forward it differentiates equals the
numpy oracle; central finite differences of that forward, in float64, match the
gradients along random directions; where the pass reduces to dense softmax
attention (the dense point, and the Taylor path with b = 1) the gradients equal
the textbook closed form written out here; and in a Taylor-only pass every row
of a pooled block receives the same dK and dV, since it enters only through the
block means.
"""
import math

import numpy as np
import pytest
import torch

from oracle import isa_oracle_backward as B
from oracle import isa_oracle_ragged as R


def _qkv(N, D, seed):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(N, D)), rng.normal(size=(N, D)), rng.normal(size=(N, D)), rng.normal(size=(N, D))


def _dense_grads(q, k, v, dout):
    """Softmax attention's gradient, written out: S = Q K^T / sqrt(D), P = softmax(S), O = P V;
    dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dP * P)), dQ = dS K / sqrt(D), dK = dS^T Q / sqrt(D)."""
    c = 1.0 / math.sqrt(q.shape[1])
    S = q @ k.T * c
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    dP = dout @ v.T
    dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
    return P @ v, dS @ k * c, dS.T @ q * c, P.T @ dout


CASES = [
    # L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns
    (64, 48, 16, 0.5, 0.5, 0.0),       # whole blocks
    (70, 45, 16, 0.5, 0.5, 0.0),       # both parts end in a short block
    (64, 48, 16, 0.5, 1.0, 0.0),       # Taylor only
    (70, 45, 16, 0.67, 0.5, 0.34),     # mixed Taylor path on short blocks
]


@pytest.mark.parametrize("case", CASES)
def test_forward_matches_the_numpy_oracle(case):
    L_src, L_ctx, b, a_s, a_f, a_ns = case
    q, k, v, dout = _qkv(L_src + L_ctx, 8, 1)
    g = B.isa_slice_grad_ref(q, k, v, dout, L_src, L_ctx, b, a_s, a_f, a_ns)
    ref = R.isa_slice_ref_ragged(q, k, v, L_src, L_ctx, b, a_s, a_f, a_ns)
    np.testing.assert_allclose(g["out"], ref["out"], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("case", CASES)
def test_gradients_match_finite_differences(case):
    L_src, L_ctx, b, a_s, a_f, a_ns = case
    q, k, v, dout = _qkv(L_src + L_ctx, 8, 2)
    g = B.isa_slice_grad_ref(q, k, v, dout, L_src, L_ctx, b, a_s, a_f, a_ns)
    sr = g["sr"]
    loss = lambda qq, kk, vv: float((B.slice_forward_torch(*(torch.tensor(x) for x in (qq, kk, vv)), sr).numpy()
                                     * dout).sum())
    rng = np.random.default_rng(3)
    eps = 1e-6
    for _ in range(3):
        dq, dk, dv = (rng.normal(size=q.shape) for _ in range(3))
        fd = (loss(q + eps * dq, k + eps * dk, v + eps * dv) - loss(q - eps * dq, k - eps * dk, v - eps * dv)) / (2 * eps)
        an = float((g["dq"] * dq).sum() + (g["dk"] * dk).sum() + (g["dv"] * dv).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (fd, an)


@pytest.mark.parametrize("L_src,L_ctx,b", [(64, 48, 16), (70, 45, 16)])
def test_dense_point_has_the_closed_form_gradient(L_src, L_ctx, b):
    """alpha_s = 1, alpha_f = 0: the pass is softmax attention over all keys."""
    q, k, v, dout = _qkv(L_src + L_ctx, 8, 4)
    g = B.isa_slice_grad_ref(q, k, v, dout, L_src, L_ctx, b, 1.0, 0.0)
    o, dq, dk, dv = _dense_grads(q, k, v, dout)
    for got, want in ((g["out"], o), (g["dq"], dq), (g["dk"], dk), (g["dv"], dv)):
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_taylor_path_with_one_token_blocks_has_the_closed_form_gradient():
    """b = 1: each pooled block is one token with weight 1, so the Taylor path (alpha_f = 1,
    alpha_s = 1) is softmax attention over all keys, gradients included."""
    q, k, v, dout = _qkv(24, 8, 5)
    g = B.isa_slice_grad_ref(q, k, v, dout, 13, 11, 1, 1.0, 1.0)
    assert len(g["sr"]["taylor"]) == 24
    o, dq, dk, dv = _dense_grads(q, k, v, dout)
    for got, want in ((g["out"], o), (g["dq"], dq), (g["dk"], dk), (g["dv"], dv)):
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_taylor_only_gradients_are_constant_inside_blocks():
    """With every query block on the Taylor path, a key or value row enters only through its
    block's mean: all rows of a block get the same dK and dV (and unkept context rows none)."""
    L_src, L_ctx, b = 70, 45, 16
    q, k, v, dout = _qkv(L_src + L_ctx, 8, 6)
    g = B.isa_slice_grad_ref(q, k, v, dout, L_src, L_ctx, b, 0.5, 1.0)
    bounds, n_src = g["sr"]["bounds"], g["sr"]["n_src"]
    kept = set(int(c) for c in g["sr"]["sel"])
    for j, (s, e) in enumerate(bounds):
        for grad in (g["dk"], g["dv"]):
            if j >= n_src and (j - n_src) not in kept:
                assert np.all(grad[s:e] == 0.0)
            else:
                np.testing.assert_allclose(grad[s:e], np.broadcast_to(grad[s], grad[s:e].shape), rtol=1e-12,
                                           atol=1e-15)


# ----------------------------------------------------------------------------- per-row log-sum-exp

def test_lse_at_dense_point_is_torch_logsumexp():
    """alpha_s = 1, alpha_f = 0: every row is exact over all keys, so the saved statistic is the
    log-sum-exp of q K^T / sqrt(D) (a library routine)."""
    import isa_synth
    from oracle import isa_oracle_backward as BW
    w = isa_synth.Workload("t", 1, 1, 16, 48, 40, 8, 1.0, 0.0, 0.1, 1.0, 0.5, "f32")
    q, k, _ = isa_synth.make_slice(w, 2, 0, 0, 0)
    got = BW.isa_slice_lse_ref(q, k, w.L_src, w.L_ctx, w.b, 1.0, 0.0)
    tq, tk = torch.from_numpy(q.astype(np.float64)), torch.from_numpy(k.astype(np.float64))
    want = torch.logsumexp(tq @ tk.T / math.sqrt(16), dim=1).numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("L_src,L_ctx,a_s,a_f", [(64, 64, 0.5, 0.5), (61, 70, 0.5, 0.75), (64, 48, 1.0, 1.0)])
def test_lse_reproduces_the_forward_output(L_src, L_ctx, a_s, a_f):
    """exp(logit - lse) are the normalised weights: with them each row's weighted sum of its
    values is the forward output (exact rows over V_new, Taylor rows over the block means with
    the length weight), also with short last blocks."""
    import isa_synth
    from oracle import isa_oracle_backward as BW
    from oracle import isa_oracle_ragged as RR
    b, D = 8, 16
    w = isa_synth.Workload("t", 1, 1, D, L_src, L_ctx, b, a_s, a_f, 0.1, 1.0, 0.5, "f32")
    q, k, v = isa_synth.make_slice(w, 4, 0, 0, 0)
    sr = RR.isa_select_route_ragged(q, k, L_src, L_ctx, b, a_s, a_f)
    ref = RR.isa_slice_ref_ragged(q, k, v, L_src, L_ctx, b, a_s, a_f, sr=sr)
    lse = BW.isa_slice_lse_ref(q, k, L_src, L_ctx, b, a_s, a_f, sr=sr)
    bounds, new_b = ref["bounds"], ref["new_bounds"]
    k_new, v_new = ref["k_new"], ref["v_new"]
    for i in sr["exact"]:
        s, e = bounds[int(i)]
        p = np.exp(q[s:e].astype(np.float64) @ k_new.T / math.sqrt(D) - lse[s:e, None])
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
        np.testing.assert_allclose(p @ v_new, ref["out"][s:e], atol=1e-12)
    kc = np.stack([k_new[a:z].mean(axis=0) for a, z in new_b])
    vc = np.stack([v_new[a:z].mean(axis=0) for a, z in new_b])
    ln = np.log([z - a for a, z in new_b])
    for i in sr["taylor"]:
        s, e = bounds[int(i)]
        p = np.exp(q[s:e].astype(np.float64) @ kc.T / math.sqrt(D) + ln[None, :] - lse[s:e, None])
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
        np.testing.assert_allclose(p @ vc, ref["out"][s:e], atol=1e-12)


def test_lse_taylor_with_block_size_one_is_dense():
    """b = 1: pooling is the identity and every weight is 1, so a Taylor row's statistic is the
    dense log-sum-exp."""
    import isa_synth
    from oracle import isa_oracle_backward as BW
    w = isa_synth.Workload("t", 1, 1, 8, 20, 12, 1, 1.0, 1.0, 0.1, 1.0, 0.5, "f32")
    q, k, _ = isa_synth.make_slice(w, 6, 0, 0, 0)
    got = BW.isa_slice_lse_ref(q, k, 20, 12, 1, 1.0, 1.0)
    tq, tk = torch.from_numpy(q.astype(np.float64)), torch.from_numpy(k.astype(np.float64))
    np.testing.assert_allclose(got, torch.logsumexp(tq @ tk.T / math.sqrt(8), dim=1).numpy(), atol=1e-12)
