"""CPU oracle for the In-context Sparse Attention forward pass with ragged lengths.

TEST INFRASTRUCTURE, under the same rule as ``isa_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg of
``bench.py`` may import or call it. It shares no code with the CUDA path.

``isa_oracle`` requires L_src and L_ctx to be multiples of the block size b.
This module restates the same pass for any positive lengths, in numpy
float64. The pages count the context blocks as ceil(L_ctx / b) (papernotes.org,
"Key design 1"), which admits a shorter last block, and say nothing more about
one. The readings taken here:

* Partition: the source tokens [0, L_src) are cut into ceil(L_src / b) blocks
  of b tokens from the start, the last one shorter when b does not divide
  L_src; the context tokens [L_src, N) likewise, starting at L_src. No block
  straddles the source/context boundary. Query blocks and key blocks share
  this partition.
* Pooling probe (paperlayer.ai, section 2 "Pooling Attention"): each block's
  mean is over its own tokens. The coarse map, the context scores (mean over
  the n_src source query blocks, each counted once), the top-k of
  k = ceil(alpha_s * n_ctx) context blocks, the sharpness and the routing are
  as in ``isa_oracle``, on these means.
* Gather (papernotes.org, "Key design 1"): a kept block adds its own tokens to
  K_new and V_new, so L_new = L_src + the lengths of the kept blocks, which
  follow the source part in ascending block order.
* Taylor path (papernotes.org, "Key design 2": l += P^c * L_K and
  O += P^c Vc_j * L_K): L_K is the length of block j, so a short block weighs
  less. With every block whole this is the weight b of ``isa_oracle``.
* No-sparsity ratio alpha_ns: as in ``isa_oracle``, over the n_new blocks of
  K_new; a pooled block keeps its own length as weight.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from oracle.isa_oracle import (F64, context_scores, coarse_scores, kept_context_blocks, no_sparse_block_count,
                               no_sparse_blocks, no_sparse_margin, route_blocks, route_margin,
                               select_context_blocks, sharpness, taylor_block_count, topk_margin)

Bounds = List[Tuple[int, int]]


def block_bounds(L_src: int, L_ctx: int, b: int) -> Bounds:
    """[start, end) of every block: the source part from 0, then the context part from L_src."""
    if L_src <= 0 or L_ctx <= 0 or b <= 0:
        raise ValueError("L_src, L_ctx and b must be positive")
    out = [(s, min(s + b, L_src)) for s in range(0, L_src, b)]
    out += [(s, min(s + b, L_src + L_ctx)) for s in range(L_src, L_src + L_ctx, b)]
    return out


def pool_ragged(x: np.ndarray, bounds: Bounds) -> np.ndarray:
    """Row i is the mean of rows [start_i, end_i) of x."""
    out = np.empty((len(bounds), x.shape[1]), F64)
    for i, (s, e) in enumerate(bounds):
        out[i] = np.asarray(x[s:e], F64).sum(axis=0) / (e - s)
    return out


def gather_kv_ragged(k: np.ndarray, v: np.ndarray, sel: np.ndarray, bounds: Bounds,
                     n_src: int) -> Tuple[np.ndarray, np.ndarray, Bounds]:
    """K_new, V_new (source part, then the kept context blocks in ascending order) and their blocks."""
    L_src = bounds[n_src - 1][1]
    rows = list(range(L_src))
    new_bounds = list(bounds[:n_src])
    for c in sel:
        s, e = bounds[n_src + int(c)]
        new_bounds.append((len(rows), len(rows) + e - s))
        rows += list(range(s, e))
    rows = np.array(rows, np.int64)
    return np.asarray(k, F64)[rows], np.asarray(v, F64)[rows], new_bounds


def exact_rows(q_rows: np.ndarray, k_new: np.ndarray, v_new: np.ndarray) -> np.ndarray:
    """softmax(q K_new^T / sqrt(D)) V_new, the max subtracted first."""
    s = (np.asarray(q_rows, F64) @ np.asarray(k_new, F64).T) / math.sqrt(q_rows.shape[1])
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p @ np.asarray(v_new, F64)) / p.sum(axis=1, keepdims=True)


def taylor_rows_ragged(q_rows: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, new_bounds: Bounds,
                       exact_blocks: Sequence[int] = ()) -> np.ndarray:
    """Block-wise 0th-order Taylor attention, the weight of block j being its own length.

    The blocks in ``exact_blocks`` (alpha_ns > 0) enter key by key instead, in
    the same softmax.
    """
    d = q_rows.shape[1]
    q64 = np.asarray(q_rows, F64)
    ex = set(int(j) for j in exact_blocks)
    terms_s, terms_w, terms_v = [], [], []  # exponent, weight, value row of every term
    for j, (s, e) in enumerate(new_bounds):
        if j in ex:
            for t in range(s, e):
                terms_s.append((q64 @ k_new[t]) / math.sqrt(d))
                terms_w.append(1.0)
                terms_v.append(v_new[t])
        else:
            kc = k_new[s:e].sum(axis=0) / (e - s)
            vc = v_new[s:e].sum(axis=0) / (e - s)
            terms_s.append((q64 @ kc) / math.sqrt(d))
            terms_w.append(float(e - s))
            terms_v.append(vc)
    S = np.stack(terms_s, axis=1)                    # [rows, terms]
    w = np.array(terms_w, F64)[None, :]
    V = np.stack(terms_v, axis=0)                    # [terms, D]
    p = np.exp(S - S.max(axis=1, keepdims=True)) * w
    return (p @ V) / p.sum(axis=1, keepdims=True)


def isa_select_route_ragged(q: np.ndarray, k: np.ndarray, L_src: int, L_ctx: int, b: int, alpha_s: float,
                            alpha_f: float, alpha_ns: float = 0.0) -> Dict[str, object]:
    """Stages 1-3 for one [N, D] slice with any positive L_src, L_ctx."""
    N = q.shape[0]
    if N != L_src + L_ctx:
        raise ValueError("N must equal L_src + L_ctx")
    bounds = block_bounds(L_src, L_ctx, b)
    n_src = -(-L_src // b)
    n_ctx = len(bounds) - n_src
    n_q = len(bounds)
    kk = kept_context_blocks(alpha_s, n_ctx)
    n_flat = taylor_block_count(alpha_f, n_q)
    qc, kc = pool_ragged(q, bounds), pool_ragged(k, bounds)
    s_coarse = coarse_scores(qc, kc)
    colscore = context_scores(s_coarse, n_src)
    sel = select_context_blocks(colscore, kk)
    kc_new = np.concatenate([kc[:n_src], kc[n_src + sel]], axis=0) if kk else kc[:n_src]
    m = sharpness(qc, kc_new)
    exact, taylor = route_blocks(m, n_flat)
    n_new = kc_new.shape[0]
    k_ns = no_sparse_block_count(alpha_ns, n_new)
    p_new = coarse_scores(qc, kc_new)
    ns_sel = (np.stack([no_sparse_blocks(p_new[i], k_ns) for i in range(n_q)]) if k_ns
              else np.zeros((n_q, 0), np.int64))
    return dict(bounds=bounds, n_src=n_src, n_ctx=n_ctx, qc=qc, kc=kc, s_coarse=s_coarse, colscore=colscore,
                sel=sel, kc_new=kc_new, sharp=m, exact=exact, taylor=taylor, k=kk, n_flat=n_flat, k_ns=k_ns,
                ns_sel=ns_sel, topk_margin=topk_margin(colscore, kk), route_margin=route_margin(m, n_flat),
                ns_margin=no_sparse_margin(p_new[taylor], k_ns) if k_ns else float("inf"))


def isa_slice_ref_ragged(q: np.ndarray, k: np.ndarray, v: np.ndarray, L_src: int, L_ctx: int, b: int,
                         alpha_s: float, alpha_f: float, alpha_ns: float = 0.0,
                         sr: Optional[Dict[str, object]] = None) -> Dict[str, object]:
    """The whole forward pass for one slice: every output row at its own token position."""
    r = dict(sr) if sr is not None else isa_select_route_ragged(q, k, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns)
    bounds = r["bounds"]
    k_new, v_new, new_bounds = gather_kv_ragged(k, v, r["sel"], bounds, r["n_src"])
    out = np.zeros(q.shape, F64)
    for i in r["exact"]:
        s, e = bounds[int(i)]
        out[s:e] = exact_rows(q[s:e], k_new, v_new)
    for i in r["taylor"]:
        s, e = bounds[int(i)]
        out[s:e] = taylor_rows_ragged(q[s:e], k_new, v_new, new_bounds,
                                      r["ns_sel"][int(i)] if r["k_ns"] else ())
    r.update(out=out, k_new=k_new, v_new=v_new, new_bounds=new_bounds,
             route=np.concatenate([r["exact"], r["taylor"]]).astype(np.int64))
    return r
