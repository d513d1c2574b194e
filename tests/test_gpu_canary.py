"""Out-of-bounds writes: every buffer a call writes sits between canary regions, which must survive.

compute-sanitizer is closed on this machine, so this stands in for its memcheck on
writes: each output (out, dbg_sel, dbg_route, dbg_ns, lse, dq, dk, dv) and each
workspace is carved out of a larger device buffer whose head and tail (64 KiB
each, beyond the largest tile any kernel moves) are filled with a byte pattern.
After the call, the pattern must be intact, and the workspace bytes beyond what
isa_workspace_bytes asks for must be untouched too. The cases cover whole and
short last blocks, both attention kernels, the mixed Taylor path, the
variable-length batch entry point and the backward pass.
"""
import numpy as np
import pytest

import isa_synth

pytestmark = pytest.mark.gpu

PAD = 64 * 1024
PATTERN = 0xA5


class Guarded:
    """A device allocation of `nbytes` with PAD canary bytes on both sides (256-byte aligned)."""

    def __init__(self, nbytes, extra=0):
        import torch
        self.nbytes = nbytes
        self.extra = extra  # bytes after the view that the call must not touch either
        self.buf = torch.full((PAD + nbytes + extra + PAD,), PATTERN, dtype=torch.uint8, device="cuda")

    def view(self, dtype, shape):
        import torch
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        assert n <= self.nbytes
        return self.buf[PAD:PAD + n].view(dtype).view(shape)

    def raw(self):
        return self.buf[PAD:PAD + self.nbytes]

    def check(self, name):
        import torch
        head = self.buf[:PAD]
        tail = self.buf[PAD + self.nbytes:]
        assert bool((head == PATTERN).all()), f"{name}: bytes before the buffer were written"
        bad = torch.nonzero(tail != PATTERN)
        assert bad.numel() == 0, f"{name}: {bad.numel()} bytes after the buffer were written (first at +{int(bad[0])})"


def _inputs(w):
    import torch
    q, k, v = isa_synth.make_inputs(w, 0)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return [torch.from_numpy(x).to("cuda", dt) for x in (q, k, v)]


CASES = [
    # B, H, D, L_src, L_ctx, b, alpha_s, alpha_f, dtype, alpha_ns
    (1, 2, 128, 1024, 1024, 128, 0.5, 0.5, "bf16", 0.0),      # CTA-pair kernel
    (1, 2, 128, 1000, 1100, 128, 0.5, 0.5, "bf16", 0.0),      # CTA-pair kernel, short last blocks
    (1, 2, 64, 600, 450, 64, 0.5, 0.5, "f32", 0.0),           # single-CTA kernel, fp32
    (1, 2, 128, 2048, 2048, 128, 0.25, 0.5, "bf16", 0.0625),  # mixed Taylor kernel (split-K)
    (1, 2, 128, 1024, 1024, 64, 0.5, 0.5, "bf16", 0.25),      # mixed Taylor path, b = 64
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[3]}_{c[4]}_b{c[5]}_{c[8]}_ns{c[9]}" for c in CASES])
def test_forward_writes_stay_inside_their_buffers(case):
    import torch
    import block_sparse_attention_isa_b200 as isa
    B, H, D, L_src, L_ctx, b, a_s, a_f, dt, a_ns = case
    w = isa_synth.Workload("canary", B, H, D, L_src, L_ctx, b, a_s, a_f, 0.1, 1.0, 0.5, dt)
    tq, tk, tv = _inputs(w)
    n_q, kk, _, k_ns = isa.plan_ns(B, H, L_src, L_ctx, D, b, a_s, a_f, a_ns)
    dtc = isa.ISA_BF16 if dt == "bf16" else isa.ISA_F32
    ws_bytes = isa.workspace_bytes(B, H, L_src, L_ctx, D, b, a_s, dtc, alpha_ns=a_ns)
    g_out = Guarded(tq.numel() * tq.element_size())
    g_sel = Guarded(4 * B * H * max(kk, 1))
    g_route = Guarded(4 * B * H * n_q)
    g_ns = Guarded(4 * B * H * n_q * max(k_ns, 1))
    g_ws = Guarded(ws_bytes)
    out = g_out.view(tq.dtype, tq.shape)
    sel = g_sel.view(torch.int32, (B, H, kk))
    route = g_route.view(torch.int32, (B, H, n_q))
    ns = g_ns.view(torch.int32, (B, H, n_q, k_ns)) if a_ns else None
    isa.forward_into(tq, tk, tv, out, L_src, L_ctx, b, a_s, a_f, sel, route, workspace=g_ws.raw(), alpha_ns=a_ns,
                     dbg_ns=ns)
    isa.device_status(g_ws.raw())
    torch.cuda.synchronize()
    for g, name in ((g_out, "out"), (g_sel, "dbg_sel"), (g_route, "dbg_route"), (g_ns, "dbg_ns"), (g_ws, "workspace")):
        g.check(name)
    # the inputs are read only
    q2, k2, v2 = _inputs(w)
    assert torch.equal(q2, tq) and torch.equal(k2, tk) and torch.equal(v2, tv)


def test_varlen_writes_stay_inside_their_buffers():
    import torch
    import block_sparse_attention_isa_b200 as isa
    H, D, b = 2, 128, 128
    lens = [(1000, 1100), (513, 700)]
    rows = sum(H * (a + c) for a, c in lens)
    g = torch.Generator().manual_seed(3)
    tq, tk, tv = (torch.randn((rows, D), generator=g).to("cuda", torch.bfloat16) for _ in range(3))
    Ls, Lc = [a for a, _ in lens], [c for _, c in lens]
    ws_bytes = isa.varlen_workspace_bytes(H, Ls, Lc, D, b, 0.5)
    g_out, g_ws = Guarded(rows * D * 2), Guarded(ws_bytes)
    out = g_out.view(torch.bfloat16, (rows, D))
    isa.forward_varlen(tq, tk, tv, H, Ls, Lc, b, 0.5, 0.5, out=out, workspace=g_ws.raw())
    isa.device_status(g_ws.raw())
    torch.cuda.synchronize()
    g_out.check("out")
    g_ws.check("workspace")


def test_backward_writes_stay_inside_their_buffers():
    import torch
    import block_sparse_attention_isa_b200 as isa
    w = isa_synth.Workload("canary_bwd", 1, 2, 128, 1024, 1024, 64, 0.5, 0.5, 0.1, 1.0, 0.5, "bf16")
    tq, tk, tv = _inputs(w)
    shape, nbytes = tq.shape, tq.numel() * 2
    dout = torch.randn(shape, generator=torch.Generator().manual_seed(1)).to("cuda", torch.bfloat16)
    g_out, g_lse = Guarded(nbytes), Guarded(4 * w.B * w.H * w.N)
    g_ws = Guarded(isa.workspace_bytes(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s))
    out = g_out.view(torch.bfloat16, shape)
    lse = g_lse.view(torch.float32, (w.B, w.H, w.N))
    L = isa.lib()
    s = torch.cuda.current_stream().cuda_stream
    rc = L.isa_forward_train(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), w.B, w.H, w.L_src, w.L_ctx, w.D, w.b,
                             w.alpha_s, w.alpha_f, 0, out.data_ptr(), lse.data_ptr(), g_ws.raw().data_ptr(),
                             g_ws.nbytes, s)
    assert rc == 0, isa.last_error()
    g_dq, g_dk, g_dv = Guarded(nbytes), Guarded(nbytes), Guarded(nbytes)
    nb = L.isa_backward_workspace_bytes(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, 0)
    g_bws = Guarded(nb)
    dq, dk, dv = (g.view(torch.bfloat16, shape) for g in (g_dq, g_dk, g_dv))
    rc = L.isa_backward(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), lse.data_ptr(),
                        dout.data_ptr(), w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f, 0,
                        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), g_ws.raw().data_ptr(), g_ws.nbytes,
                        g_bws.raw().data_ptr(), g_bws.nbytes, s)
    assert rc == 0, isa.last_error()
    isa.device_status(g_ws.raw())
    torch.cuda.synchronize()
    for g, name in ((g_out, "out"), (g_lse, "lse"), (g_ws, "forward workspace"), (g_dq, "dq"), (g_dk, "dk"),
                    (g_dv, "dv"), (g_bws, "backward workspace")):
        g.check(name)
