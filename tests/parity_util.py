"""Helpers shared by the GPU parity tests: input drawing with near-tie rejection, GPU runs, comparisons."""

import numpy as np

import isa_synth
from oracle import isa_oracle as O

# Tolerances for bf16 inputs with fp32 accumulation (and the same for fp32 / tf32).
MAX_ABS = 2e-2
REL_L2 = 5e-3
MARGIN = 1e-3


def accepted_attempts(w, seed=0, max_attempts=64):
    """Per-slice attempts whose top-k and routing margins clear MARGIN (oracle stages 1-3)."""
    att = np.zeros((w.B, w.H), np.int64)
    for bi in range(w.B):
        for h in range(w.H):
            for a in range(max_attempts):
                q, k, _ = isa_synth.make_slice(w, seed, bi, h, a)
                r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
                if r["topk_margin"] >= MARGIN and r["route_margin"] >= MARGIN:
                    att[bi, h] = a
                    break
            else:
                raise RuntimeError(f"no accepted attempt for slice {bi},{h}")
    return att


def inputs(w, seed=0):
    att = isa_synth.attempts_for(w, seed)
    if att is None:
        att = accepted_attempts(w, seed)
    return isa_synth.make_inputs(w, seed, att)


def to_device(x, w, device="cuda"):
    import torch
    t = torch.from_numpy(x)
    return t.to(device=device, dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32)


def run_gpu(w, q, k, v):
    import torch
    import block_sparse_attention_isa_b200 as isa
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    out, sel, route = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
    isa.device_status()
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), sel.cpu().numpy(), route.cpu().numpy()


def compare_out(gpu, ref, max_abs=MAX_ABS, rel_l2=REL_L2):
    d = np.abs(gpu.astype(np.float64) - ref)
    ma = float(d.max()) if d.size else 0.0
    rl = float(np.linalg.norm((gpu.astype(np.float64) - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30))
    assert np.isfinite(gpu).all(), "non-finite output"
    assert ma <= max_abs and rl <= rel_l2, f"max-abs {ma:.3e} (<= {max_abs}), rel-L2 {rl:.3e} (<= {rel_l2})"
    return ma, rl
