"""fp64 CPU oracle for the WorldAttention HSA decode step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code, table or helper with the CUDA
library; it receives the exact input values the GPU receives (bf16/fp32 bits,
widened to float64) and computes every step in float64 with numpy.

Each function follows one step of the method as the WorldAttention pages state it
(citations give the page and the section, equation or step):

  S0 prompt_select      -- §3.2 "Stage 1: prompt-level retrieval" (cosine top-1 chunk)
  S1 page_scores /      -- §3.2 "Stage 2: page-level retrieval", the alpha_{m,j} equation
     select_pages          and the top-K_p choice of pages
  S2 gather_pages       -- §3.2 "Active KV construction"; summary step (4): the chosen
                           pages joined into K_active, V_active
  key_block_bounds      -- §3.3 "Inter- and intra-chunk sparse granularity" (history blocks
                           of B_inter tokens, the current chunk's blocks of B_intra)
  S3 block_select       -- §3.3 "Head-level sparsity adaptation" (minimal block set whose
                           cumulative mass reaches tau_h); summary step (5), coarse
                           selection over pooled blocks
  S4 linear_project /   -- §3.3 "Linear branch", the O_lin equation with
     linear_attention      K~ = E_K^T K, V~ = E_V^T V (Linformer projection)
  S5 sparse_attention   -- §3.3 "Sparse branch"; Appendix A.1.3 block-sparse attention
  S6 gate_fuse          -- §3.3 "Gated fusion of two branches" (sigmoid gate)
     gate_fuse2            the same section's two-gate form O_lin (.) G_lin + O_sp (.) G_sp
                           with G = sigmoid of a logit per (token, head)
  cube_order            -- Appendix A.1.3: the token re-indexing under which every group
                           of B consecutive tokens is one (C_t, C_h, C_w) cube

Readings where the pages are silent (each one is listed in the design notes):
  * Q-bar in the page score is per head; the per-head scores are averaged over heads,
    giving one page set per layer (one shared 49,920-token active buffer).
  * The chosen pages are concatenated in ascending candidate position.
  * Ties in any ranking go to the lower index.
  * The mass condition is read as ">= tau_h"; tau_h >= 1 keeps every block, and so
    does a row whose cumulative mass never reaches tau_h.
  * Block pooling is the mean over the valid rows of a block; a block's score is
    q-bar . k-bar / sqrt(d); the mass is the softmax of one (head, query block) row.
  * E_K, E_V are shared by all heads, shape [L][r], unless given per head ([H][L][r],
    the main text's K~^(h) read as one projection per head); no extra scaling.
  * Keys of both branches are the retrieved history; with k_cur/v_cur the sparse
    branch also takes the current chunk's own keys (after the history); no causal mask.
  * Key block sizes (§3.3 "Inter- and intra-chunk sparse granularity"): the history
    is cut into blocks of B_inter tokens (128 in the pages, B by default) that tile the
    concatenated history K_active, so a block may span two adjacent pages; the current
    chunk's own keys and the queries use blocks of B (B_intra = 64).  One softmax runs
    over all key blocks of a row, whatever their size.
  * O = sigmoid(g) * O_sp + (1 - sigmoid(g)) * O_lin, per token and head (or two gates).
  * Cube order (its formula is lost): cubes in raster order of their corners, tokens
    in raster order inside a cube, the last cube along a side cut short when the side
    is not a multiple of the cube side.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np


def f64(x) -> np.ndarray:
    """Widen a torch tensor or array to float64 (exact for bf16/fp32 inputs)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------- token order
def cube_order(T: int, H_l: int, W_l: int, C_t: int, C_h: int, C_w: int) -> list:
    """Appendix A.1.3 (block-sparse attention): the flattened video tokens are
    re-indexed so that each run of C_t*C_h*C_w consecutive tokens is one
    (C_t, C_h, C_w) cube.  Returns perm with perm[n] = raster index (t*H_l + h)*W_l + w
    of the token at position n: walk the cubes in raster order of their corners and,
    inside each, the tokens in raster order (cubes at the far edges cut short)."""
    perm = []
    for t0 in range(0, T, C_t):
        for h0 in range(0, H_l, C_h):
            for w0 in range(0, W_l, C_w):
                for t in range(t0, min(T, t0 + C_t)):
                    for h in range(h0, min(H_l, h0 + C_h)):
                        for w in range(w0, min(W_l, w0 + C_w)):
                            perm.append((t * H_l + h) * W_l + w)
    return perm


# ----------------------------------------------------------------------------- S0
def prompt_select(e_cur, e_chunks) -> int:
    """Index of the history chunk whose prompt embedding has the largest cosine
    similarity with the current prompt embedding (§3.2 Stage 1).  Ties -> lowest index.
    A zero-norm embedding has no cosine similarity and raises ValueError."""
    e = f64(e_cur)
    E = f64(e_chunks)
    ne = math.sqrt(float(np.dot(e, e)))
    nE = np.sqrt(np.einsum("md,md->m", E, E))
    if ne == 0.0 or np.any(nE == 0.0):
        raise ValueError("zero-norm prompt embedding")
    cos = (E @ e) / (nE * ne)
    best = 0
    for m in range(1, len(cos)):
        if cos[m] > cos[best]:
            best = m
    return best


def prompt_margin(e_cur, e_chunks) -> float:
    """Gap between the best and the second-best cosine (inf with one chunk)."""
    e = f64(e_cur)
    E = f64(e_chunks)
    cos = (E @ e) / (np.sqrt(np.einsum("md,md->m", E, E)) * math.sqrt(float(np.dot(e, e))))
    s = np.sort(cos)[::-1]
    return float(s[0] - s[1]) if len(s) > 1 else math.inf


# ----------------------------------------------------------------------------- S1
def page_scores(q, k_pages) -> np.ndarray:
    """alpha_j = (1/H) sum_h  Qbar_h . Kbar_{h,j} / sqrt(d)   (§3.2 Stage 2).

    q: [Nq][H][d] queries of the current chunk; k_pages: [n_c][T_p][H][d] keys of the
    candidate pages.  Qbar_h is the mean query of head h over the chunk, Kbar_{h,j}
    the mean key of page j for head h."""
    Q = f64(q)
    K = f64(k_pages)
    d = Q.shape[2]
    q_bar = Q.mean(axis=0)                 # [H][d]
    k_bar = K.mean(axis=1)                 # [n_c][H][d]
    per_head = np.einsum("hd,jhd->jh", q_bar, k_bar) / math.sqrt(d)
    return per_head.mean(axis=1)


def select_pages(alpha: Sequence[float], K_p: int) -> list:
    """Candidate positions of the top-K_p scores (ties -> lower position), returned in
    ascending position, i.e. the chronological order of the pages in the chunk."""
    n_c = len(alpha)
    if K_p > n_c or K_p < 1:
        raise ValueError("need 1 <= K_p <= n_c")
    order = sorted(range(n_c), key=lambda j: (-float(alpha[j]), j))
    return sorted(order[:K_p])


def page_margin(alpha: Sequence[float], K_p: int) -> float:
    """alpha_(K_p) - alpha_(K_p+1) in descending order (inf when every page is kept)."""
    a = sorted((float(x) for x in alpha), reverse=True)
    return a[K_p - 1] - a[K_p] if K_p < len(a) else math.inf


# ----------------------------------------------------------------------------- S2
def gather_pages(pool, page_ids: Iterable[int]):
    """Concatenate pool pages [P][T_p][...] in the given order -> [K_p*T_p][...].
    Works on any array type (the copy is exact)."""
    ids = list(page_ids)
    if hasattr(pool, "detach"):
        import torch
        return torch.cat([pool[i] for i in ids], dim=0)
    return np.concatenate([np.asarray(pool[i]) for i in ids], axis=0)


# ----------------------------------------------------------------------------- S3
def block_bounds(n: int, B: int, start: int = 0) -> list:
    """[start + b*B, start + min(n, (b+1)*B)) for the ceil(n/B) blocks of n tokens."""
    return [(start + b, start + min(n, b + B)) for b in range(0, n, B)]


def key_block_bounds(L_hist: int, B_inter: int, L_cur: int = 0, B_intra: Optional[int] = None) -> list:
    """Key blocks of the sparse branch (§3.3 "Inter- and intra-chunk sparse
    granularity"): the retrieved history's L_hist tokens in blocks of B_inter, then
    the current chunk's own L_cur tokens in blocks of B_intra."""
    return block_bounds(L_hist, B_inter) + block_bounds(L_cur, B_intra or B_inter, start=L_hist)


def block_means_at(x, bounds) -> np.ndarray:
    """Mean over the rows of each block [s, e) of ``bounds``.  x: [N][H][d] -> [n][H][d]."""
    X = f64(x)
    out = np.empty((len(bounds),) + X.shape[1:], dtype=np.float64)
    for b, (s0, e0) in enumerate(bounds):
        out[b] = X[s0:e0].mean(axis=0)
    return out


def block_means(x, B: int) -> np.ndarray:
    """Mean over the valid rows of each block of B consecutive tokens.
    x: [N][H][d] -> [ceil(N/B)][H][d]; the last block may hold fewer than B rows."""
    return block_means_at(x, block_bounds(f64(x).shape[0], B))


def expand_blocks(kept_row, bounds, B: int) -> list:
    """The B-token blocks (of the key sequence) that the kept blocks of ``bounds`` cover,
    ascending: the same key set at the granularity of B."""
    out = set()
    for j in kept_row:
        s0, e0 = bounds[j]
        out.update(range(s0 // B, (e0 - 1) // B + 1))
    return sorted(out)


def softmax(s: np.ndarray) -> np.ndarray:
    """Softmax of a 1-D score vector, with the maximum subtracted first."""
    z = np.exp(s - np.max(s))
    return z / z.sum()


def select_row(scores: np.ndarray, tau: float) -> tuple:
    """Minimal prefix of the scores sorted in descending order (ties -> lower block)
    whose softmax mass reaches tau (§3.3 head-level sparsity).

    Returns (sorted ascending list of kept blocks, margin).  The margin is the
    smallest of: the score gap at the cut, C_m - tau and tau - C_{m-1}; it is inf
    when every block is kept because tau >= 1."""
    n = len(scores)
    p = softmax(scores)
    order = sorted(range(n), key=lambda j: (-float(scores[j]), j))
    if tau >= 1.0:
        return list(range(n)), math.inf
    c = 0.0
    prev = 0.0
    m = None
    for t, j in enumerate(order):
        prev = c
        c += p[j]
        if c >= tau:
            m = t + 1
            break
    if m is None:
        # the rounded total stayed below tau: every block is kept
        return list(range(n)), tau - c
    kept = sorted(order[:m])
    gap = float(scores[order[m - 1]] - scores[order[m]]) if m < n else math.inf
    margin = min(gap, c - tau, (tau - prev) if m > 1 else math.inf)
    return kept, margin


def block_scores(q, k_act, B: int, key_bounds=None) -> np.ndarray:
    """Pooled block scores s[h][i][j] = qbar_{h,i} . kbar_{h,j} / sqrt(d); query blocks
    of B, key blocks of B or ``key_bounds``."""
    qb = block_means(q, B)                 # [n_qb][H][d]
    kb = block_means(k_act, B) if key_bounds is None else block_means_at(k_act, key_bounds)
    d = qb.shape[2]
    # per head: [n_qb][d] @ [d][n_kb]
    return np.stack([qb[:, h, :] @ kb[:, h, :].T for h in range(qb.shape[1])]) / math.sqrt(d)


def block_select(q, k_act, tau, B: int, scores: Optional[np.ndarray] = None, key_bounds=None):
    """Per (head, query block): the kept key blocks (ascending) and the margin.

    Returns (kept[h][i] -> list, margin[h][i] -> float)."""
    s = block_scores(q, k_act, B, key_bounds) if scores is None else scores
    H, n_qb, _ = s.shape
    tau = f64(tau)
    kept = [[None] * n_qb for _ in range(H)]
    margin = np.empty((H, n_qb))
    for h in range(H):
        for i in range(n_qb):
            kept[h][i], margin[h, i] = select_row(s[h, i], float(tau[h]))
    return kept, margin


# ----------------------------------------------------------------------------- S4
def linear_project(k_act, v_act, e_k, e_v):
    """K~ = E_K^T K, V~ = E_V^T V per head (§3.3 linear branch, K~^(h) = E_K^T K^(h)).
    k_act, v_act: [L][H][d]; e_k, e_v: [L][r] shared by the heads, or [H][L][r] one
    per head -> K~, V~: [r][H][d]."""
    K = f64(k_act)
    V = f64(v_act)
    EK = f64(e_k)
    EV = f64(e_v)
    L, H, d = K.shape
    if EK.ndim == 3:
        # one E per head: K~[:, h, :] = E_K[h]^T K[:, h, :]
        kt = np.stack([EK[h].T @ K[:, h, :] for h in range(H)], axis=1)
        vt = np.stack([EV[h].T @ V[:, h, :] for h in range(H)], axis=1)
        return kt, vt
    # sum over l of E[l][c] * X[l][h][:], as one [r][L] @ [L][H*d] product
    kt = (EK.T @ K.reshape(L, H * d)).reshape(-1, H, d)
    vt = (EV.T @ V.reshape(L, H * d)).reshape(-1, H, d)
    return kt, vt


def linear_attention(q, k_til, v_til, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """O_lin[n,h] = softmax_r(Q[n,h] . K~_h^T / sqrt(d)) V~_h  (§3.3, O_lin equation).
    q: [Nq][H][d]; k_til, v_til: [r][H][d] -> [Nq][H][d] (or only ``rows``)."""
    Q = f64(q)
    if rows is not None:
        Q = Q[rows]
    KT = f64(k_til)
    VT = f64(v_til)
    d = Q.shape[2]
    out = np.empty_like(Q)
    for h in range(Q.shape[1]):
        s = Q[:, h, :] @ KT[:, h, :].T / math.sqrt(d)          # [n][r]
        s = s - s.max(axis=1, keepdims=True)
        w = np.exp(s)
        w /= w.sum(axis=1, keepdims=True)
        out[:, h, :] = w @ VT[:, h, :]
    return out


# ----------------------------------------------------------------------------- S5
def sparse_attention_block(q, k_act, v_act, h: int, i: int, kept_blocks, B: int,
                           key_bounds=None) -> np.ndarray:
    """Exact attention of the rows of query block i, head h, over the keys of the kept
    key blocks only (§3.3 sparse branch; A.1.3: a block is computed whole or skipped).
    Two passes: scores, then softmax-weighted values.  -> [rows][d]."""
    Q = f64(q)
    Nq = Q.shape[0]
    L = k_act.shape[0]
    r0, r1 = i * B, min(Nq, (i + 1) * B)
    kb = block_bounds(L, B) if key_bounds is None else key_bounds
    keys = np.concatenate([np.arange(kb[j][0], kb[j][1]) for j in kept_blocks])
    Kh = f64(k_act[keys, h, :] if not hasattr(k_act, "detach") else k_act[keys, h, :])
    Vh = f64(v_act[keys, h, :] if not hasattr(v_act, "detach") else v_act[keys, h, :])
    d = Q.shape[2]
    s = Q[r0:r1, h, :] @ Kh.T / math.sqrt(d)
    s = s - s.max(axis=1, keepdims=True)
    w = np.exp(s)
    w /= w.sum(axis=1, keepdims=True)
    return w @ Vh


def sparse_attention(q, k_act, v_act, kept, B: int, key_bounds=None) -> np.ndarray:
    """O_sp for every (query block, head): [Nq][H][d]."""
    Q = f64(q)
    Nq, H, d = Q.shape
    out = np.empty((Nq, H, d))
    for h in range(H):
        for i in range(len(kept[h])):
            out[i * B:min(Nq, (i + 1) * B), h, :] = sparse_attention_block(
                Q, k_act, v_act, h, i, kept[h][i], B, key_bounds)
    return out


# ----------------------------------------------------------------------------- S6
def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def gate_fuse(o_sp, o_lin, g) -> np.ndarray:
    """O = sigmoid(g) * O_sp + (1 - sigmoid(g)) * O_lin, g per (token, head)."""
    G = sigmoid(f64(g))[..., None]
    return G * f64(o_sp) + (1.0 - G) * f64(o_lin)


def gate_fuse2(o_sp, o_lin, g_sp, g_lin) -> np.ndarray:
    """O = sigmoid(g_sp) * O_sp + sigmoid(g_lin) * O_lin: one sigmoid gate per branch,
    each per (token, head) (the two-gate form of the gated fusion)."""
    return sigmoid(f64(g_sp))[..., None] * f64(o_sp) + sigmoid(f64(g_lin))[..., None] * f64(o_lin)


# ----------------------------------------------------------------------------- step
def hsa_step(inp: dict, B: int, K_p: int, rows_of_blocks: Optional[Sequence[tuple]] = None,
             B_inter: Optional[int] = None) -> dict:
    """The whole decode step S0..S6 on one input dict (see the workload module).

    ``B_inter`` (default B) is the block size of the retrieved history in the sparse
    branch (main text §3.3, "Inter- and intra-chunk sparse granularity": 128 for the
    history pages, B = 64 for the current chunk); queries always use blocks of B.

    With ``rows_of_blocks`` = [(h, i), ...] only those (head, query block) outputs are
    computed (the selection is still computed for every row); otherwise all of O.

    With ``k_cur``/``v_cur`` in the input (the current chunk's own keys and values,
    [Nq][H][d]), the sparse branch's key sequence is the retrieved history followed by
    the current chunk (main text §3.3, "Inter- and intra-chunk sparse granularity":
    the sparse branch attends to both, in blocks of the same kernel); block selection
    runs over all blocks of that sequence jointly, and the linear branch stays over
    the history, whose positions E indexes."""
    res: dict = {}
    if "e_cur" in inp:
        m = prompt_select(inp["e_cur"], inp["e_chunks"])
        res["chunk"] = m
        cand = [int(x) for x in inp["chunk_pages"][m]]
    else:
        cand = [int(x) for x in inp["cand"]]
    res["cand"] = cand
    k_pool, v_pool = inp["k_pool"], inp["v_pool"]
    k_cand = np.stack([f64(k_pool[p]) for p in cand])
    alpha = page_scores(inp["q"], k_cand)
    del k_cand
    pos = select_pages(alpha, K_p)
    sel = [cand[j] for j in pos]
    res.update(alpha=alpha, sel=sel, page_margin=page_margin(alpha, K_p))
    k_act = gather_pages(k_pool, sel)
    v_act = gather_pages(v_pool, sel)
    res["k_act"], res["v_act"] = k_act, v_act
    k_sp, v_sp = k_act, v_act
    L_hist = k_act.shape[0]
    L_cur = 0
    if inp.get("k_cur") is not None:
        k_sp = np.concatenate([f64(k_act), f64(inp["k_cur"])], axis=0)
        v_sp = np.concatenate([f64(v_act), f64(inp["v_cur"])], axis=0)
        L_cur = k_sp.shape[0] - L_hist
    kbounds = key_block_bounds(L_hist, B_inter or B, L_cur, B)
    kept, margin = block_select(inp["q"], k_sp, inp["tau"], B, key_bounds=kbounds)
    res["kept"], res["block_margin"], res["key_bounds"] = kept, margin, kbounds
    kt, vt = linear_project(k_act, v_act, inp["e_k"], inp["e_v"])
    res["k_til"], res["v_til"] = kt, vt
    Q = f64(inp["q"])
    Nq, H, d = Q.shape
    g = f64(inp["gate"])
    g_lin = f64(inp["gate_lin"]) if inp.get("gate_lin") is not None else None
    if rows_of_blocks is None:
        o_sp = sparse_attention(Q, k_sp, v_sp, kept, B, kbounds)
        o_lin = linear_attention(Q, kt, vt)
        res["o_sp"], res["o_lin"] = o_sp, o_lin
        res["o"] = gate_fuse(o_sp, o_lin, g) if g_lin is None else gate_fuse2(o_sp, o_lin, g, g_lin)
    else:
        outs = {}
        for (h, i) in rows_of_blocks:
            r0, r1 = i * B, min(Nq, (i + 1) * B)
            osp = sparse_attention_block(Q, k_sp, v_sp, h, i, kept[h][i], B, kbounds)
            olin = linear_attention(Q[r0:r1, h:h + 1, :], kt[:, h:h + 1, :], vt[:, h:h + 1, :])[:, 0, :]
            G = sigmoid(g[r0:r1, h])[:, None]
            Gl = (1.0 - G) if g_lin is None else sigmoid(g_lin[r0:r1, h])[:, None]
            outs[(h, i)] = dict(o_sp=osp, o_lin=olin, o=G * osp + Gl * olin)
        res["blocks"] = outs
    return res
