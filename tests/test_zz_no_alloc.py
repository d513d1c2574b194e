"""The allocation-free entry point against the regular one, through the C ABI.

isa_select_context_noalloc serves callers that cannot allocate device memory
(operator plugins handed only their inputs and outputs; serving loops that
forbid cudaMalloc because it can synchronise the device). It keeps its scratch
in a fixed array inside the library, so two calls in a row must both agree with
isa_forward_ex, which uses a caller workspace: the kept context blocks exactly,
the context scores within the tolerance of the stage tests. This file is
collected last so that a failure here cannot stop the rest of a -x run.
"""

import numpy as np
import pytest

import isa_synth
from parity_util import inputs, to_device

pytestmark = pytest.mark.gpu


def _noalloc(L, tq, tk, tv, w, sel, cs, stream):
    return L.isa_select_context_noalloc(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), w.B, w.H, w.L_src, w.L_ctx, w.D,
                                        w.b, w.alpha_s, 0 if w.dtype == "bf16" else 1, sel.data_ptr(), cs.data_ptr(),
                                        stream)


def test_noalloc_matches_workspace_entry_two_calls():
    import torch
    import block_sparse_attention_isa_b200 as isa
    from block_sparse_attention_isa_b200 import build
    build.build()
    L = isa.lib()
    cases = [isa_synth.Workload("noalloc_a", 1, 4, 128, 2048, 2048, 128, 0.25, 0.5, 0.1, 1.0, 0.5, "bf16"),
             isa_synth.Workload("noalloc_b", 1, 3, 128, 1536, 1024, 64, 0.5, 0.5, 0.1, 1.0, 0.5, "bf16")]
    for w in cases:  # two calls in a row with different inputs and sizes
        q, k, v = inputs(w)
        tq, tk, tv = (to_device(x, w) for x in (q, k, v))
        _, sel_ref, _ = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
        cs_ref = isa.debug_pooled(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s)["colscore"]
        isa.device_status()
        sel = torch.full_like(sel_ref, -1)
        cs = torch.full_like(cs_ref, -1.0)
        stream = torch.cuda.current_stream().cuda_stream
        rc = _noalloc(L, tq, tk, tv, w, sel, cs, stream)
        assert rc == 0, isa.last_error()
        torch.cuda.synchronize()
        assert torch.equal(sel, sel_ref)
        np.testing.assert_allclose(cs.cpu().numpy(), cs_ref.cpu().numpy(), rtol=1e-4, atol=1e-7)


def test_noalloc_rejects_sizes_beyond_the_fixed_array():
    import block_sparse_attention_isa_b200 as isa
    L = isa.lib()
    fake = 0x7F0000000000  # never dereferenced: the size check comes before any GPU work
    # 3 * 64 heads * 2048 blocks * 128 * 4 bytes = 201 MB > 32 MiB
    rc = L.isa_select_context_noalloc(fake, fake, fake, 1, 64, 65536, 65536, 128, 64, 0.25, 0, fake, fake, None)
    assert rc == -3
    assert "scratch" in isa.last_error()
