"""GPU parity of the training forward (per-row lse) and the backward pass against the oracle.

The oracle (oracle/isa_oracle_backward.py) restates the forward in torch float64
with the forward's decisions held fixed and takes dQ, dK, dV by autograd; it is
pinned by finite differences and closed forms. Inputs whose top-k or routing
decision lies within a relative 1e-3 of a tie are redrawn, so both sides take
the same decisions.

Tolerances, from the arithmetic of the kernels: inputs are bf16 and exact on
both sides; the kernels round P and dS to bf16 before the accumulating MMAs
(relative 2^-9 each), take delta = rowsum(dO * O) from the bf16 output, and round
the gradients to bf16 (relative 2^-9), with fp32 accumulation throughout. Each
gradient element is a sum of such terms, so its error is a few times 2^-9 of
the magnitudes that enter it: the tests ask max-abs <= 2e-2 * max|ref| and
relative L2 <= 1e-2 per tensor. The saved lse is compared within 1e-2 (an fp32
sum of bf16-rounded p, about 2^-9 relative at worst).
"""
import numpy as np
import pytest

import isa_synth
from oracle import isa_oracle_backward as BW
from oracle import isa_oracle_ragged as R
from parity_util import MARGIN

pytestmark = pytest.mark.gpu

GRAD_MAX_REL = 2e-2
GRAD_REL_L2 = 1e-2
LSE_ABS = 1e-2

CASES = [
    # name, B, H, L_src, L_ctx, b, alpha_s, alpha_f
    ("b128_half", 1, 2, 512, 512, 128, 0.5, 0.5),
    ("b64_odd_exact_tiles", 1, 2, 1024, 1024, 64, 0.25, 0.6),
    ("dense_point", 1, 2, 512, 512, 128, 1.0, 0.0),
    ("all_taylor", 1, 2, 512, 512, 64, 0.5, 1.0),
    ("no_context_kept", 1, 2, 512, 512, 64, 0.0, 0.5),
    ("b2_h2", 2, 2, 768, 512, 128, 0.5, 0.25),
    ("two_pooled_row_tiles", 1, 1, 8192, 8192, 64, 0.25, 0.5),
]


def _draw(w, max_attempts=64):
    att = np.zeros((w.B, w.H), np.int64)
    for bi in range(w.B):
        for h in range(w.H):
            for a in range(max_attempts):
                q, k, _ = isa_synth.make_slice(w, 0, bi, h, a)
                r = R.isa_select_route_ragged(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
                if min(r["topk_margin"], r["route_margin"]) >= MARGIN:
                    att[bi, h] = a
                    break
            else:
                raise RuntimeError(f"no accepted attempt for slice {bi},{h}")
    return isa_synth.make_inputs(w, 0, att)


def _dout(w, seed=17):
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((w.B, w.H, w.N, w.D)).astype(np.float32)
    return isa_synth.bf16_bits_to_f32(isa_synth.round_to_bf16_bits(g))


def _check(name, gpu, ref):
    d = gpu.astype(np.float64) - ref
    scale = float(np.abs(ref).max())
    ma = float(np.abs(d).max())
    rl = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))
    assert np.isfinite(gpu).all(), f"{name}: non-finite"
    assert ma <= GRAD_MAX_REL * max(scale, 1e-30) and rl <= GRAD_REL_L2, \
        f"{name}: max-abs {ma:.3e} (max|ref| {scale:.3e}), rel-L2 {rl:.3e}"


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_parity(case):
    import torch
    import block_sparse_attention_isa_b200 as isa
    name, B, H, L_src, L_ctx, b, a_s, a_f = case
    w = isa_synth.Workload(name, B, H, 128, L_src, L_ctx, b, a_s, a_f, 0.1, 1.0, 0.5, "bf16")
    q, k, v = _draw(w)
    g = _dout(w)
    tq, tk, tv, tg = (torch.from_numpy(x).to("cuda", torch.bfloat16) for x in (q, k, v, g))
    out, lse, ws = isa.forward_train(tq, tk, tv, L_src, L_ctx, b, a_s, a_f)
    dq, dk, dv = isa.backward(tq, tk, tv, out, lse, tg, ws, L_src, L_ctx, b, a_s, a_f)
    isa.device_status(ws)
    # the training forward is the plain forward plus lse
    plain = isa.forward(tq, tk, tv, L_src, L_ctx, b, a_s, a_f)
    isa.device_status()
    assert torch.equal(plain, out)
    lse_h = lse.cpu().numpy()
    got = {n: t.float().cpu().numpy() for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
    refs = {n: np.zeros((B, H, w.N, w.D)) for n in got}
    for bi in range(B):
        for h in range(H):
            sr = R.isa_select_route_ragged(q[bi, h], k[bi, h], L_src, L_ctx, b, a_s, a_f)
            r = BW.isa_slice_grad_ref(q[bi, h], k[bi, h], v[bi, h], g[bi, h], L_src, L_ctx, b, a_s, a_f, sr=sr)
            for n in got:
                refs[n][bi, h] = r[n]
            lse_ref = BW.isa_slice_lse_ref(q[bi, h], k[bi, h], L_src, L_ctx, b, a_s, a_f, sr=sr)
            err = float(np.abs(lse_h[bi, h] - lse_ref).max())
            assert err <= LSE_ABS, f"{name}: lse max-abs {err:.3e}"
    for n in got:
        _check(f"{name} {n}", got[n], refs[n])
    # context rows of blocks that were not kept get no gradient
    if a_s < 1.0:
        for bi in range(B):
            for h in range(H):
                sr = R.isa_select_route_ragged(q[bi, h], k[bi, h], L_src, L_ctx, b, a_s, a_f)
                kept = set(int(c) for c in sr["sel"])
                for c in range(L_ctx // b):
                    if c not in kept:
                        rows = slice(L_src + c * b, L_src + (c + 1) * b)
                        assert not got["dk"][bi, h, rows].any() and not got["dv"][bi, h, rows].any()


def test_backward_is_deterministic():
    """No atomics reach dQ, dK or dV of the exact path; the Taylor path's partial sums go through
    fp32 atomics into the block-mean gradients, so repeat runs agree to within one bf16 step."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    w = isa_synth.Workload("det", 1, 2, 128, 1024, 1024, 128, 0.5, 0.5, 0.1, 1.0, 0.5, "bf16")
    q, k, v = _draw(w)
    g = _dout(w)
    tq, tk, tv, tg = (torch.from_numpy(x).to("cuda", torch.bfloat16) for x in (q, k, v, g))
    out, lse, ws = isa.forward_train(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    a = isa.backward(tq, tk, tv, out, lse, tg, ws, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    c = isa.backward(tq, tk, tv, out, lse, tg, ws, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    isa.device_status(ws)
    assert torch.equal(a[0], c[0])
    for x, y in zip(a[1:], c[1:]):
        assert torch.allclose(x.float(), y.float(), rtol=2 ** -7, atol=1e-6)


def test_backward_rejects_unsupported():
    import torch
    import block_sparse_attention_isa_b200 as isa
    x = torch.zeros((1, 2, 1000, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(isa.IsaError):  # lengths that b does not divide
        out, lse, ws = isa.forward_train(x, x, x, 500, 500, 128, 0.5, 0.5)
        isa.backward(x, x, x, out, lse, x, ws, 500, 500, 128, 0.5, 0.5)
