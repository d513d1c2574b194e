"""CPU oracle for the In-context Sparse Attention (ISA) forward pass.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import or call this module.
The product path (the CUDA library and its Python binding) never does, and the
two share no code.

This is a plain, slow restatement in numpy float64 of the method described in
"Lightning Unified Video Editing via In-Context Sparse Attention":

* papernotes.org notes, "Overall framework" and the flowchart: the forward
  pass is a pooling probe, context pre-selection, grouped computation by query
  sharpness, then an exact path and a block-wise 0th-order Taylor path whose
  outputs are written back.
* papernotes.org, "Key design 1, Context Pre-Selection": the coarse map
  S_coarse, the source-query x context-key sub-block, its mean over the query
  axis, Top-k of alpha_s * ceil(L_ctx / b) context blocks, gather + concat into
  K_new, V_new.
* papernotes.org, "Key design 2, Block-wise 0th-order Taylor sparse
  attention": S = Q K^T / sqrt(D) with online softmax for exact blocks, and a
  pooled block standing in as exp(Q Kc^T / sqrt(D)) weighted by the block
  length, paired with Vc.
* papernotes.org, "Key design 3, Grouped computation by query sharpness":
  M_i = Var(softmax(Qc_i Kc^T)), query blocks sorted by M_i and split by the
  flat ratio alpha_f.
* paperlayer.ai summary (arXiv 2605.04569v2), section 2 "Pooling Attention"
  and section 3 "Pre-Selection", "Taylor Sparse Attention", "Grouped
  Computation".

Readings taken where the pages are silent or disagree (each is also listed in
the design notes):

* Blocks are whole: L_src and L_ctx must be multiples of b.
* k = ceil(alpha_s * n_ctx - 1e-4) from the float32 alpha_s, clamped to
  [0, n_ctx]; n_flat = floor(alpha_f * n_q + 1e-4) from the float32 alpha_f.
  The 1e-4 guard keeps float32 ratios such as 0.1 * 200 = 20.0000003 from
  rounding up.
* Every score (coarse map, sharpness, both attention paths) is scaled by
  1/sqrt(D).
* The coarse softmax runs over all n_q key blocks; the context score of
  context block c is the mean of S_coarse[i, n_src + c] over the n_src source
  query blocks.
* Top-k ranks by (score descending, index ascending); the kept blocks enter
  K_new in ascending index order after the whole source part.
* Sharpness uses the pooled blocks of K_new (source blocks then kept context
  blocks), population variance over the n_new blocks.
* alpha_f is the fraction of query blocks with the LOWEST sharpness, sent to
  the Taylor path; ties break by block index. The pages also print the other
  direction (top alpha_f to the exact path); the two agree at alpha_f = 0.5,
  and a caller who wants the other reading passes 1 - alpha_f.
* All n_q query blocks (source and context) are routed and attend to K_new.
* Each query block takes exactly one path, so write-back is a scatter into
  the original token order with no merge.
* The Taylor path is computed literally, with the block-length weight b.
* No-sparsity ratio alpha_ns (papernotes.org, "Key design 2" block mask M_ij;
  "Key design 3": alpha_ns sets the share of key blocks that stay dense inside
  a Taylor query block; paperlayer.ai summary section 2 "Pooling Attention": top-k entries of the
  coarse map give the block mask; section 4 defaults alpha_ns = 0.0625). For
  a Taylor query block i, the k_ns = ceil(alpha_ns * n_new - 1e-4) key blocks
  of K_new with the largest coarse scores softmax_j(Qc_i . Kc_new_j / sqrt(D))
  (ties by lower index) are computed exactly, all of their b keys, and every
  other block of K_new through its pooled row with weight b, in one softmax.
  alpha_ns = 0 is the plain Taylor path. Exact query blocks are unaffected.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "kept_context_blocks",
    "taylor_block_count",
    "pool_blocks",
    "coarse_scores",
    "context_scores",
    "select_context_blocks",
    "gather_kv",
    "sharpness",
    "route_blocks",
    "exact_rows",
    "taylor_rows",
    "isa_slice_ref",
    "isa_forward_ref",
    "isa_select_route_ref",
    "isa_rows_ref",
    "topk_margin",
    "route_margin",
    "executed_flops",
    "no_sparse_block_count",
    "no_sparse_blocks",
    "taylor_mixed_rows",
    "no_sparse_margin",
]

F64 = np.float64


def _f32(x: float) -> float:
    """The ratio as the float32 the library receives, widened back to double."""
    return float(np.float32(x))


def kept_context_blocks(alpha_s: float, n_ctx: int) -> int:
    """Number of kept context blocks k = ceil(alpha_s * ceil(L_ctx / b)).

    papernotes.org, "Key design 1": Top-k keeps alpha_s * ceil(L_ctx/b) blocks.
    Reading: ceil of the product with a 1e-4 guard on the float32 ratio.
    """
    x = _f32(alpha_s) * n_ctx
    k = int(math.ceil(x - 1e-4))
    return max(0, min(n_ctx, k))


def taylor_block_count(alpha_f: float, n_q: int) -> int:
    """Number of query blocks sent to the Taylor path, floor(alpha_f * n_q).

    papernotes.org, "Key design 3": the flat ratio alpha_f splits the sorted
    query blocks. Reading: floor with a 1e-4 guard on the float32 ratio.
    """
    x = _f32(alpha_f) * n_q
    n = int(math.floor(x + 1e-4))
    return max(0, min(n_q, n))


def pool_blocks(x: np.ndarray, b: int) -> np.ndarray:
    """Block means: row i of the result is the mean of rows [i*b, (i+1)*b) of x.

    paperlayer.ai, section 2 "Pooling Attention": Q and K/V are pooled per
    block to compressed block-level representations.
    """
    n, d = x.shape
    assert n % b == 0
    out = np.empty((n // b, d), F64)
    for i in range(n // b):
        out[i] = np.asarray(x[i * b:(i + 1) * b], F64).sum(axis=0) / b
    return out


def _softmax_rows(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, F64)
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


def coarse_scores(qc: np.ndarray, kc: np.ndarray) -> np.ndarray:
    """S_coarse = softmax(Qc Kc^T / sqrt(D)) over all key blocks.

    papernotes.org, "Key design 1": pooling attention gives the coarse map
    S_coarse in R^{N_Q x N_K} per (batch, head).
    """
    d = qc.shape[1]
    return _softmax_rows((np.asarray(qc, F64) @ np.asarray(kc, F64).T) / math.sqrt(d))


def context_scores(s_coarse: np.ndarray, n_src: int) -> np.ndarray:
    """Mean over source query blocks of the source-query x context-key sub-block.

    papernotes.org, "Key design 1": cut out S_coarse[src-Q, ctx-K] and average
    it along the query axis.
    """
    sub = s_coarse[:n_src, n_src:]
    return sub.sum(axis=0) / n_src


def select_context_blocks(score: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest context scores, returned in ascending order.

    papernotes.org, "Key design 1": TopK picks the most salient context blocks.
    Ties rank by lower index first.
    """
    order = sorted(range(len(score)), key=lambda c: (-float(score[c]), c))
    return np.array(sorted(order[:k]), dtype=np.int64)


def gather_kv(k: np.ndarray, v: np.ndarray, sel: np.ndarray, L_src: int, b: int) -> Tuple[np.ndarray, np.ndarray]:
    """K_new = [K_src ; kept context blocks], same for V.

    papernotes.org, "Key design 1": gather + concat rebuild K_new and V_new of
    length L_src + alpha_s * L_ctx.
    """
    kp = [np.asarray(k[:L_src], F64)] + [np.asarray(k[L_src + c * b:L_src + (c + 1) * b], F64) for c in sel]
    vp = [np.asarray(v[:L_src], F64)] + [np.asarray(v[L_src + c * b:L_src + (c + 1) * b], F64) for c in sel]
    return np.concatenate(kp, axis=0), np.concatenate(vp, axis=0)


def sharpness(qc: np.ndarray, kc_new: np.ndarray) -> np.ndarray:
    """M_i = Var_j softmax_j(Qc_i . Kc_new_j / sqrt(D)), population variance.

    papernotes.org, "Key design 3": M_i = Var(softmax(Q^c_i (K^c)^T)), read
    from the pooling scores. The mean of a softmax row is 1/n, so the variance
    is the mean of (p_j - 1/n)^2.
    """
    p = coarse_scores(qc, kc_new)
    n = p.shape[1]
    return ((p - 1.0 / n) ** 2).sum(axis=1) / n


def route_blocks(m: np.ndarray, n_flat: int) -> Tuple[np.ndarray, np.ndarray]:
    """Split query blocks: the n_flat lowest-sharpness blocks go to the Taylor path.

    papernotes.org, "Key design 3": sort by M_i; sharp queries take the exact
    path, the rest the 0th-order Taylor path. Ties break by block index.
    Returns (exact blocks ascending, Taylor blocks ascending).
    """
    order = sorted(range(len(m)), key=lambda i: (float(m[i]), i))
    taylor = np.array(sorted(order[:n_flat]), dtype=np.int64)
    exact = np.array(sorted(order[n_flat:]), dtype=np.int64)
    return exact, taylor


def exact_rows(q_rows: np.ndarray, k_new: np.ndarray, v_new: np.ndarray) -> np.ndarray:
    """softmax(q K_new^T / sqrt(D)) V_new for each query row.

    papernotes.org, "Key design 2" (M_ij = 1 branch): S = Q K^T / sqrt(D),
    P = exp(S), l = rowsum(P), O = P V / l. Online softmax reaches the same
    value; the oracle uses the textbook max-subtracted softmax over all keys.
    """
    d = q_rows.shape[1]
    s = (np.asarray(q_rows, F64) @ np.asarray(k_new, F64).T) / math.sqrt(d)
    return _softmax_rows(s) @ np.asarray(v_new, F64)


def taylor_rows(q_rows: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, b: int) -> np.ndarray:
    """Block-wise 0th-order Taylor attention of each query row against K_new's blocks.

    papernotes.org, "Key design 2" (M_ij = 0 branch): a block j stands in as
    S^c = q Kc_j^T / sqrt(D), P^c = exp(S^c); l += P^c * L_K and
    O += P^c Vc_j * L_K with L_K = b; finally O = O / l. The maximum is
    subtracted before exp (the ratio is unchanged).
    """
    d = q_rows.shape[1]
    kc_new = pool_blocks(k_new, b)
    vc_new = pool_blocks(v_new, b)
    s = (np.asarray(q_rows, F64) @ kc_new.T) / math.sqrt(d)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    num = (p * b) @ vc_new
    den = (p * b).sum(axis=1, keepdims=True)
    return num / den


def no_sparse_block_count(alpha_ns: float, n_new: int) -> int:
    """k_ns = ceil(alpha_ns * n_new - 1e-4) from the float32 ratio, clamped to [0, n_new].

    papernotes.org, "Key design 3": alpha_ns is the share of a Taylor query
    block's key blocks that are not made sparse; the count is rounded up like
    the kept context blocks.
    """
    a = _f32(alpha_ns)
    if a <= 0.0:
        return 0
    return int(min(n_new, max(0, math.ceil(a * n_new - 1e-4))))


def no_sparse_blocks(p_row: np.ndarray, k_ns: int) -> np.ndarray:
    """The k_ns key blocks of K_new with the largest coarse scores in one row, ascending.

    paperlayer.ai summary, section 2: top-k entries of the coarse attention map
    give the block mask. Ranked by (score descending, index ascending).
    """
    order = sorted(range(len(p_row)), key=lambda j: (-float(p_row[j]), j))
    return np.array(sorted(order[:k_ns]), dtype=np.int64)


def taylor_mixed_rows(q_rows: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, b: int,
                      exact_blocks: Sequence[int]) -> np.ndarray:
    """Taylor attention with some key blocks computed exactly, in one softmax.

    papernotes.org, "Key design 2": for M_ij = 1, S_ij = q K_j^T / sqrt(D) and
    P_ij = exp(S_ij) over the block's keys, l += rowsum(P_ij), O += P_ij V_j;
    for M_ij = 0, S^c_ij = q Kc_j^T / sqrt(D), P^c_ij = exp(S^c_ij),
    l += P^c_ij * L_K, O += P^c_ij Vc_j * L_K (L_K = b); finally O = O / l.
    The maximum over all terms is subtracted before exp (the ratio is unchanged).
    """
    d = q_rows.shape[1]
    n_new = k_new.shape[0] // b
    ex = sorted(set(int(j) for j in exact_blocks))
    pooled = [j for j in range(n_new) if j not in set(ex)]
    q64 = np.asarray(q_rows, F64)
    kc_new = pool_blocks(k_new, b)
    vc_new = pool_blocks(v_new, b)
    rows = np.concatenate([np.arange(j * b, (j + 1) * b) for j in ex]) if ex else np.zeros(0, np.int64)
    se = (q64 @ np.asarray(k_new, F64)[rows].T) / math.sqrt(d)      # exact keys
    sc = (q64 @ kc_new[pooled].T) / math.sqrt(d)                     # pooled blocks
    m = np.maximum(se.max(axis=1, initial=-np.inf), sc.max(axis=1, initial=-np.inf))[:, None]
    pe = np.exp(se - m)
    pc = np.exp(sc - m) * b
    num = pe @ np.asarray(v_new, F64)[rows] + pc @ vc_new[pooled]
    den = pe.sum(axis=1, keepdims=True) + pc.sum(axis=1, keepdims=True)
    return num / den


def no_sparse_margin(p_rows: np.ndarray, k_ns: int) -> float:
    """Smallest relative gap, over the given coarse rows, between their k_ns-th and (k_ns+1)-th scores."""
    if k_ns <= 0 or p_rows.shape[1] <= k_ns or p_rows.shape[0] == 0:
        return float("inf")
    srt = -np.sort(-p_rows, axis=1)
    a, c = srt[:, k_ns - 1], srt[:, k_ns]
    return float(np.min((a - c) / np.maximum(np.abs(a), 1e-300)))


def _validate(N: int, L_src: int, L_ctx: int, b: int):
    if L_src + L_ctx != N:
        raise ValueError("N must equal L_src + L_ctx")
    if L_src <= 0 or L_ctx <= 0 or L_src % b or L_ctx % b:
        raise ValueError("L_src and L_ctx must be positive multiples of b")


def isa_select_route_ref(q: np.ndarray, k: np.ndarray, L_src: int, L_ctx: int, b: int,
                         alpha_s: float, alpha_f: float, alpha_ns: float = 0.0) -> Dict[str, np.ndarray]:
    """Stages 1-3 for one [N, D] slice: pooling probe, pre-selection, routing.

    Returns the pooled Qc/Kc, the coarse map's context scores, the kept blocks
    ``sel``, the sharpness M over all query blocks, the routing and the two
    tie margins used to reject near-tie inputs. With alpha_ns > 0 also the
    exactly computed key blocks of every query block (``ns_sel``, [n_q, k_ns])
    and the tie margin of that choice over the Taylor blocks.
    """
    N, D = q.shape
    _validate(N, L_src, L_ctx, b)
    n_q, n_src, n_ctx = N // b, L_src // b, L_ctx // b
    kk = kept_context_blocks(alpha_s, n_ctx)
    n_flat = taylor_block_count(alpha_f, n_q)
    qc = pool_blocks(q, b)
    kc = pool_blocks(k, b)
    s_coarse = coarse_scores(qc, kc)
    colscore = context_scores(s_coarse, n_src)
    sel = select_context_blocks(colscore, kk)
    k_new_pooled = np.concatenate([kc[:n_src], kc[n_src + sel]], axis=0) if kk else kc[:n_src]
    m = sharpness(qc, k_new_pooled)
    exact, taylor = route_blocks(m, n_flat)
    n_new = k_new_pooled.shape[0]
    k_ns = no_sparse_block_count(alpha_ns, n_new)
    p_new = coarse_scores(qc, k_new_pooled) if k_ns else np.zeros((n_q, n_new))
    ns_sel = np.stack([no_sparse_blocks(p_new[i], k_ns) for i in range(n_q)]) if k_ns else np.zeros((n_q, 0), np.int64)
    return dict(qc=qc, kc=kc, s_coarse=s_coarse, colscore=colscore, sel=sel, kc_new=k_new_pooled,
                sharp=m, exact=exact, taylor=taylor, k=kk, n_flat=n_flat, k_ns=k_ns, ns_sel=ns_sel,
                topk_margin=topk_margin(colscore, kk), route_margin=route_margin(m, n_flat),
                ns_margin=no_sparse_margin(p_new[taylor], k_ns) if k_ns else float("inf"),
                ns_row_margin=np.array([no_sparse_margin(p_new[[i]], k_ns) for i in range(n_q)]) if k_ns
                else np.full(n_q, np.inf))


def isa_slice_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, L_src: int, L_ctx: int, b: int,
                  alpha_s: float, alpha_f: float, row_chunk: int = 2048, alpha_ns: float = 0.0) -> Dict[str, np.ndarray]:
    """The whole forward pass for one (batch, head) slice of [N, D] arrays.

    Rows are processed in chunks of ``row_chunk`` to bound memory; every row's
    softmax still runs over all of its keys in one piece.
    """
    N, D = q.shape
    r = isa_select_route_ref(q, k, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns)
    k_new, v_new = gather_kv(k, v, r["sel"], L_src, b)
    out = np.zeros((N, D), F64)
    if r["k_ns"]:  # mixed Taylor path: each flat block with its own exactly computed key blocks
        for i in r["taylor"]:
            rr = np.arange(i * b, (i + 1) * b)
            out[rr] = taylor_mixed_rows(q[rr], k_new, v_new, b, r["ns_sel"][i])
    for blocks, fn in ((r["exact"], "exact"), (r["taylor"], "taylor")):
        if len(blocks) == 0 or (fn == "taylor" and r["k_ns"]):
            continue
        rows = np.concatenate([np.arange(i * b, (i + 1) * b) for i in blocks])
        for s in range(0, len(rows), row_chunk):
            rr = rows[s:s + row_chunk]
            if fn == "exact":
                out[rr] = exact_rows(q[rr], k_new, v_new)
            else:
                out[rr] = taylor_rows(q[rr], k_new, v_new, b)
    r["out"] = out
    r["route"] = np.concatenate([r["exact"], r["taylor"]]).astype(np.int64)
    return r


def isa_rows_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, L_src: int, L_ctx: int, b: int,
                 alpha_s: float, alpha_f: float, rows: Sequence[int],
                 sr: Optional[Dict[str, np.ndarray]] = None, alpha_ns: float = 0.0) -> np.ndarray:
    """Output rows ``rows`` of one slice only (for sampled checks at full size)."""
    if sr is None:
        sr = isa_select_route_ref(q, k, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns)
    k_new, v_new = gather_kv(k, v, sr["sel"], L_src, b)
    taylor = set(int(t) for t in sr["taylor"])
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), q.shape[1]), F64)
    is_t = np.array([int(r) // b in taylor for r in rows], dtype=bool)
    if (~is_t).any():
        out[~is_t] = exact_rows(q[rows[~is_t]], k_new, v_new)
    if is_t.any():
        if sr.get("k_ns", 0):
            for n, r_ in enumerate(rows):
                if is_t[n]:
                    out[n] = taylor_mixed_rows(q[[r_]], k_new, v_new, b, sr["ns_sel"][int(r_) // b])[0]
        else:
            out[is_t] = taylor_rows(q[rows[is_t]], k_new, v_new, b)
    return out


def isa_forward_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, L_src: int, L_ctx: int, b: int,
                    alpha_s: float, alpha_f: float, alpha_ns: float = 0.0) -> Dict[str, np.ndarray]:
    """Whole forward pass for [B, H, N, D] inputs; slices are independent.

    Returns ``out`` [B,H,N,D] (float64), ``sel`` [B,H,k] and ``route``
    [B,H,n_q] (exact blocks ascending, then Taylor blocks ascending).
    """
    B, H, N, D = q.shape
    outs, sels, routes = [], [], []
    for bi in range(B):
        for h in range(H):
            r = isa_slice_ref(q[bi, h], k[bi, h], v[bi, h], L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns=alpha_ns)
            outs.append(r["out"])
            sels.append(r["sel"])
            routes.append(r["route"])
    kk = len(sels[0])
    return dict(out=np.stack(outs).reshape(B, H, N, D),
                sel=np.stack(sels).reshape(B, H, kk) if kk else np.zeros((B, H, 0), np.int64),
                route=np.stack(routes).reshape(B, H, N // b))


def topk_margin(score: np.ndarray, k: int) -> float:
    """Relative gap between the k-th and (k+1)-th largest context scores (inf if no boundary)."""
    n = len(score)
    if k <= 0 or k >= n:
        return math.inf
    s = np.sort(np.asarray(score, F64))[::-1]
    return float((s[k - 1] - s[k]) / s[k - 1])


def route_margin(m: np.ndarray, n_flat: int) -> float:
    """Relative gap between the largest Taylor sharpness and the smallest exact one."""
    n = len(m)
    if n_flat <= 0 or n_flat >= n:
        return math.inf
    s = np.sort(np.asarray(m, F64))
    if s[n_flat] <= 0:
        return 0.0
    return float((s[n_flat] - s[n_flat - 1]) / s[n_flat])


def executed_flops(B: int, H: int, L_src: int, L_ctx: int, D: int, b: int, alpha_s: float, alpha_f: float) -> Dict[str, float]:
    """Multiply-add work of each stage, 2 FLOP per multiply-add, over all slices."""
    N = L_src + L_ctx
    n_q, n_src, n_ctx = N // b, L_src // b, L_ctx // b
    kk = kept_context_blocks(alpha_s, n_ctx)
    n_flat = taylor_block_count(alpha_f, n_q)
    n_new = n_src + kk
    L_new = n_new * b
    bh = B * H
    coarse = 2.0 * n_src * n_q * D * bh
    route = 2.0 * n_q * n_new * D * bh
    exact = 4.0 * (n_q - n_flat) * b * L_new * D * bh
    taylor = 4.0 * n_flat * b * n_new * D * bh
    return dict(coarse=coarse, route=route, exact=exact, taylor=taylor,
                total=coarse + route + exact + taylor, dense=4.0 * N * N * D * bh)
