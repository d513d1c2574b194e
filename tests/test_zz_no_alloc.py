"""The allocation-free entry point against the regular one and the oracle, through the C ABI.

isa_select_context_noalloc serves callers that cannot allocate device memory
(operator plugins handed only their inputs and outputs; serving loops that
forbid cudaMalloc because it can synchronise the device). It keeps its scratch
in a fixed array inside the library, so several calls in a row (different sizes,
a ragged shape, fp32 inputs) must each agree with isa_forward_ex, which uses a
caller workspace: the kept context blocks exactly, the context scores within the
tolerance of the stage tests. The kept blocks are also checked against the
float64 oracle on inputs whose top-k clears the tie margin, and the companion
status call must report a clean run after every call. This file is collected
last so that a failure here cannot stop the rest of a -x run.
"""

import numpy as np
import pytest

import isa_synth
from oracle import isa_oracle_ragged as R
from parity_util import MARGIN, to_device

pytestmark = pytest.mark.gpu

CASES = [
    isa_synth.Workload("noalloc_a", 1, 4, 128, 2048, 2048, 128, 0.25, 0.5, 0.1, 1.0, 0.5, "bf16"),
    isa_synth.Workload("noalloc_b", 1, 3, 128, 1536, 1024, 64, 0.5, 0.5, 0.1, 1.0, 0.5, "bf16"),
    # short last blocks in both parts
    isa_synth.Workload("noalloc_ragged", 1, 2, 128, 1000, 1100, 128, 0.5, 0.5, 0.1, 1.0, 0.5, "bf16"),
    # the tiny fp32 workload's shape
    isa_synth.Workload("noalloc_f32", 1, 2, 64, 512, 512, 64, 0.5, 0.5, 0.1, 1.0, 0.5, "f32"),
]


def _inputs(w, max_attempts=64):
    """Draws whose top-k clears the tie margin (oracle stages 1-2), with their oracle selection."""
    att = np.zeros((w.B, w.H), np.int64)
    sel_ref = []
    for bi in range(w.B):
        for h in range(w.H):
            for a in range(max_attempts):
                q, k, _ = isa_synth.make_slice(w, 0, bi, h, a)
                r = R.isa_select_route_ragged(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
                if r["topk_margin"] >= MARGIN:
                    att[bi, h] = a
                    sel_ref.append(r["sel"])
                    break
            else:
                raise RuntimeError(f"no accepted attempt for slice {bi},{h}")
    q, k, v = isa_synth.make_inputs(w, 0, att)
    return q, k, v, np.stack(sel_ref).reshape(w.B, w.H, -1)


def _noalloc(L, tq, tk, tv, w, sel, cs, stream):
    return L.isa_select_context_noalloc(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), w.B, w.H, w.L_src, w.L_ctx, w.D,
                                        w.b, w.alpha_s, 0 if w.dtype == "bf16" else 1, sel.data_ptr(), cs.data_ptr(),
                                        stream)


def test_noalloc_matches_workspace_entry_and_oracle():
    import torch
    import block_sparse_attention_isa_b200 as isa
    from block_sparse_attention_isa_b200 import build
    build.build()
    L = isa.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for w in CASES + CASES[:1]:  # calls in a row with different inputs and sizes, then the first again
        q, k, v, sel_oracle = _inputs(w)
        tq, tk, tv = (to_device(x, w) for x in (q, k, v))
        _, sel_ref, _ = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
        dtype = isa.ISA_BF16 if w.dtype == "bf16" else isa.ISA_F32
        cs_ref = isa.debug_pooled(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, dtype)["colscore"]
        isa.device_status()
        sel = torch.full_like(sel_ref, -1)
        cs = torch.full_like(cs_ref, -1.0)
        rc = _noalloc(L, tq, tk, tv, w, sel, cs, stream)
        assert rc == 0, isa.last_error()
        assert L.isa_select_context_noalloc_status(stream) == 0, isa.last_error()
        torch.cuda.synchronize()
        assert torch.equal(sel, sel_ref), w.name
        np.testing.assert_array_equal(sel.cpu().numpy(), sel_oracle, err_msg=w.name)
        np.testing.assert_allclose(cs.cpu().numpy(), cs_ref.cpu().numpy(), rtol=1e-4, atol=1e-7, err_msg=w.name)


def test_noalloc_rejects_sizes_beyond_the_fixed_array():
    import block_sparse_attention_isa_b200 as isa
    L = isa.lib()
    fake = 0x7F0000000000  # never dereferenced: the size check comes before any GPU work
    # 3 * 64 heads * 2048 blocks * 128 * 4 bytes = 201 MB > 32 MiB
    rc = L.isa_select_context_noalloc(fake, fake, fake, 1, 64, 65536, 65536, 128, 64, 0.25, 0, fake, fake, None)
    assert rc == -3
    assert "scratch" in isa.last_error()
