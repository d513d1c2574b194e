"""CPU oracle for the backward pass of In-context Sparse Attention (trainable ISA).

TEST INFRASTRUCTURE, under the same rule as ``isa_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg of
``bench.py`` may import or call it. It shares no code with the CUDA path.

The pages train with ISA end to end: papernotes.org (overview and "Key design
2") says the forward and backward passes are written as trainable kernels,
and the paperlayer.ai summary (appendix H) says the Triton kernels implement
the forward and backward of block-wise 0th-order Taylor attention. They do not
spell the backward out. The reading taken here:

* The discrete decisions of the forward pass are held fixed: the kept context
  blocks, the routing, and (alpha_ns > 0) each Taylor block's exact key blocks.
  They are taken by ``isa_oracle_ragged.isa_select_route_ragged``, which equals
  ``isa_oracle`` on whole blocks. No gradient flows through the pooling
  probe's scores, the top-k or the sharpness.
* The gradient is that of the output with respect to Q, K and V through
  everything else: K_new and V_new (the gathered rows), the exact path, the
  Taylor path's block means Kc_j and Vc_j with their length weights, and the
  mixed path's exact keys.

The forward is restated with torch float64 operations on CPU, and autograd
gives the gradient. ``tests/test_oracle_backward.py`` pins it against central
finite differences, against the textbook closed form of softmax attention's
gradient where the pass reduces to dense attention, and against the structure
of the block means.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
import torch

from oracle import isa_oracle_ragged as R


def _rows_of(bounds, blocks):
    return [t for j in blocks for t in range(*bounds[int(j)])]


def slice_forward_torch(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, sr: Dict[str, object]) -> torch.Tensor:
    """The forward pass of one [N, D] slice in torch float64, the decisions in ``sr`` held fixed.

    q, k, v may require grad; the result is [N, D], every row at its token position.
    """
    N, D = q.shape
    bounds, n_src = sr["bounds"], int(sr["n_src"])
    L_src = bounds[n_src - 1][1]
    # K_new, V_new: the source rows, then the kept context blocks' rows (ascending)
    new_rows = list(range(L_src)) + _rows_of(bounds, [n_src + int(c) for c in sr["sel"]])
    idx = torch.tensor(new_rows, dtype=torch.long)
    k_new, v_new = k.index_select(0, idx), v.index_select(0, idx)
    # blocks of K_new: the source blocks, then the kept blocks, each with its own length
    new_bounds, start = [], 0
    for j in list(range(n_src)) + [n_src + int(c) for c in sr["sel"]]:
        s, e = bounds[j]
        new_bounds.append((start, start + e - s))
        start += e - s
    scale = 1.0 / math.sqrt(D)
    pieces, pos = [], []
    for i in sr["exact"]:
        s, e = bounds[int(i)]
        p = torch.softmax((q[s:e] @ k_new.T) * scale, dim=1)
        pieces.append(p @ v_new)
        pos += list(range(s, e))
    for i in sr["taylor"]:
        s, e = bounds[int(i)]
        ex = set(int(j) for j in sr["ns_sel"][int(i)]) if int(sr["k_ns"]) else set()
        logits, weights, values = [], [], []
        for j, (a, z) in enumerate(new_bounds):
            if j in ex:  # key by key
                logits.append((q[s:e] @ k_new[a:z].T) * scale)
                weights.append(torch.zeros(z - a, dtype=q.dtype))
                values.append(v_new[a:z])
            else:        # the pooled row, weighing its block's length
                kc = k_new[a:z].mean(dim=0, keepdim=True)
                logits.append((q[s:e] @ kc.T) * scale)
                weights.append(torch.full((1,), math.log(z - a), dtype=q.dtype))
                values.append(v_new[a:z].mean(dim=0, keepdim=True))
        S = torch.cat(logits, dim=1) + torch.cat(weights)[None, :]   # log of the weight added
        pieces.append(torch.softmax(S, dim=1) @ torch.cat(values, dim=0))
        pos += list(range(s, e))
    out = torch.zeros((N, D), dtype=q.dtype)
    return out.index_copy(0, torch.tensor(pos, dtype=torch.long), torch.cat(pieces, dim=0))


def isa_slice_grad_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, dout: np.ndarray, L_src: int, L_ctx: int,
                       b: int, alpha_s: float, alpha_f: float, alpha_ns: float = 0.0,
                       sr: Optional[Dict[str, object]] = None) -> Dict[str, np.ndarray]:
    """Output and the gradients dQ, dK, dV of sum(out * dout) for one slice."""
    if sr is None:
        sr = R.isa_select_route_ragged(q, k, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns)
    qt, kt, vt = (torch.tensor(np.asarray(x, np.float64), requires_grad=True) for x in (q, k, v))
    out = slice_forward_torch(qt, kt, vt, sr)
    out.backward(torch.tensor(np.asarray(dout, np.float64)))
    return dict(out=out.detach().numpy(), dq=qt.grad.numpy(), dk=kt.grad.numpy(), dv=vt.grad.numpy(), sr=sr)


def isa_slice_lse_ref(q: np.ndarray, k: np.ndarray, L_src: int, L_ctx: int, b: int, alpha_s: float,
                      alpha_f: float, sr: Optional[Dict[str, object]] = None) -> np.ndarray:
    """Per-row log-sum-exp of the forward's softmax denominators (float64, [N]), alpha_ns = 0.

    The quantity a trainable kernel saves for its backward pass (papernotes.org, overview and
    "Key design 2": the online softmax keeps a running maximum and sum per row):
    * an exact-path row q: log sum_t exp(q . K_new_t / sqrt(D)) over every key of K_new;
    * a Taylor-path row q: log sum_j L_K(j) exp(q . Kc_j / sqrt(D)) over the blocks j of K_new,
      each weighing its length L_K(j) (b for a whole block), i.e. the log of the literal
      denominator l of "Key design 2".
    """
    if sr is None:
        sr = R.isa_select_route_ragged(q, k, L_src, L_ctx, b, alpha_s, alpha_f)
    N, D = q.shape
    bounds, n_src = sr["bounds"], int(sr["n_src"])
    new_blocks = list(range(n_src)) + [n_src + int(c) for c in sr["sel"]]
    rows = [t for j in new_blocks for t in range(*bounds[j])]
    k_new = np.asarray(k, np.float64)[rows]
    kc = np.stack([np.asarray(k[s:e], np.float64).mean(axis=0) for s, e in (bounds[j] for j in new_blocks)])
    ln_len = np.log(np.array([bounds[j][1] - bounds[j][0] for j in new_blocks], np.float64))
    q64 = np.asarray(q, np.float64)
    out = np.zeros(N, np.float64)

    def lse(z):
        m = z.max(axis=1, keepdims=True)
        return (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0]

    for i in sr["exact"]:
        s, e = bounds[int(i)]
        out[s:e] = lse(q64[s:e] @ k_new.T / math.sqrt(D))
    for i in sr["taylor"]:
        s, e = bounds[int(i)]
        out[s:e] = lse(q64[s:e] @ kc.T / math.sqrt(D) + ln_len[None, :])
    return out
