"""GPU parity of variable-length batches (isa_forward_varlen) against the ragged-length oracle.

Every element of the batch has its own L_src and L_ctx (papernotes.org, Key
design 1 counts context blocks as ceil(L_ctx / b), so short last blocks occur),
and is an independent pass over its heads. The packed batch is compared element
by element with the float64 oracle: kept blocks and routing bit-exactly (inputs
within a relative 1e-3 of a tie are redrawn), outputs within max-abs 2e-2 and
relative L2 5e-3. The cases run the CTA-pair kernel (bf16, D = 128) and the
single-CTA kernel (D = 64).
"""
import numpy as np
import pytest

import isa_synth
from oracle import isa_oracle_ragged as R
from parity_util import MARGIN, compare_out

pytestmark = pytest.mark.gpu

CASES = [
    # name, H, D, b, alpha_s, alpha_f, [(L_src, L_ctx), ...]
    ("pair_b128", 2, 128, 128, 0.5, 0.5, [(1000, 1100), (2048, 2048), (513, 700)]),
    ("pair_b64", 2, 128, 64, 0.25, 0.6, [(4096, 4096), (657, 453)]),
    ("single_d64", 2, 64, 64, 0.5, 0.5, [(600, 450), (1024, 512), (65, 10)]),
]


def _element(H, D, b, a_s, a_f, L_src, L_ctx, index):
    """Draws of one element (generator batch index = element index) whose decisions clear the tie
    margin, with the oracle's per-head results."""
    w = isa_synth.Workload("varlen", 1, H, D, L_src, L_ctx, b, a_s, a_f, 0.1, 1.0, 0.5, "bf16")
    qs, ks, vs, refs = [], [], [], []
    for h in range(H):
        for a in range(64):
            q, k, v = isa_synth.make_slice(w, 0, index, h, a)
            r = R.isa_select_route_ragged(q, k, L_src, L_ctx, b, a_s, a_f)
            if min(r["topk_margin"], r["route_margin"]) >= MARGIN:
                break
        else:
            raise RuntimeError(f"no accepted attempt for element {index}, head {h}")
        qs.append(q), ks.append(k), vs.append(v)
        refs.append(R.isa_slice_ref_ragged(q, k, v, L_src, L_ctx, b, a_s, a_f, sr=r))
    return np.stack(qs), np.stack(ks), np.stack(vs), refs


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_varlen_batch_parity(case):
    import torch
    import block_sparse_attention_isa_b200 as isa
    name, H, D, b, a_s, a_f, lens = case
    parts = [_element(H, D, b, a_s, a_f, ls, lc, i) for i, (ls, lc) in enumerate(lens)]
    # the packed batch as [total rows, D]: the binding takes D from the last dimension
    flat = [np.concatenate([p[j].reshape(-1, D) for p in parts]) for j in range(3)]
    tq, tk, tv = (torch.from_numpy(x).to("cuda", torch.bfloat16) for x in flat)
    Ls, Lc = [ls for ls, _ in lens], [lc for _, lc in lens]
    out, sel, route = isa.forward_varlen(tq, tk, tv, H, Ls, Lc, b, a_s, a_f, debug=True)
    isa.device_status()
    out, sel, route = out.float().cpu().numpy().ravel(), sel.cpu().numpy(), route.cpu().numpy()
    off = off_s = off_r = 0
    for (ls, lc), (_, _, _, refs) in zip(lens, parts):
        N = ls + lc
        o = out[off:off + H * N * D].reshape(H, N, D)
        for h, r in enumerate(refs):
            kk, nq = len(r["sel"]), len(r["route"])
            np.testing.assert_array_equal(sel[off_s:off_s + kk], r["sel"], err_msg=f"{name}: kept blocks")
            np.testing.assert_array_equal(route[off_r:off_r + nq], r["route"], err_msg=f"{name}: routing")
            compare_out(o[h], r["out"])
            off_s += kk
            off_r += nq
        off += H * N * D
    assert off == out.size and off_s == sel.size and off_r == route.size


def test_varlen_equals_separate_calls():
    """The packed batch gives, bit for bit, what one plain call per element gives."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    H, D, b, a_s, a_f = 2, 128, 128, 0.25, 0.5
    lens = [(1000, 1100), (2048, 2048)]
    parts = [_element(H, D, b, a_s, a_f, ls, lc, i) for i, (ls, lc) in enumerate(lens)]
    flat = [np.concatenate([p[j].reshape(-1, D) for p in parts]) for j in range(3)]
    tq, tk, tv = (torch.from_numpy(x).to("cuda", torch.bfloat16) for x in flat)
    out = isa.forward_varlen(tq, tk, tv, H, [l[0] for l in lens], [l[1] for l in lens], b, a_s, a_f)
    isa.device_status()
    off = 0
    for (ls, lc) in lens:
        n = H * (ls + lc)
        shp = (1, H, ls + lc, D)
        one = isa.forward(tq[off:off + n].view(shp), tk[off:off + n].view(shp), tv[off:off + n].view(shp), ls, lc,
                          b, a_s, a_f)
        isa.device_status()
        assert torch.equal(one.view(-1, D), out[off:off + n])
        off += n
