"""Pins for the fp64 oracle: checks that do not reuse its own formulas.

Each test ties one oracle step to something fixed from outside it: the page
arithmetic printed by the WorldAttention pages, closed forms, brute force on tiny
inputs, invariants, and the textbook softmax attention of torch's
``scaled_dot_product_attention`` (fp64 on CPU) where the method reduces to it
(tau = 1 for the sparse branch; E = I or a row-selection E for the linear branch).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import hsa_oracle as O
from linear_attention_paged_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa(q, k, v, mask=None):
    """Textbook attention softmax(q k^T / sqrt(d)) v from torch, fp64, [n,d],[m,d],[m,d]."""
    q = torch.as_tensor(q, dtype=torch.float64)[None, None]
    k = torch.as_tensor(k, dtype=torch.float64)[None, None]
    v = torch.as_tensor(v, dtype=torch.float64)[None, None]
    m = None if mask is None else torch.as_tensor(mask)[None, None]
    return F.scaled_dot_product_attention(q, k, v, attn_mask=m)[0, 0].numpy()


def rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- page arithmetic
def test_page_arithmetic_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "page_arithmetic.json")))
    assert g["K_p"] * g["frames_per_page"] * g["tokens_per_frame"] == g["active_tokens"]
    assert g["fps"] * g["seconds"] == g["frames_60s"]
    assert g["frames_60s"] // g["frames_per_page"] == g["pages_60s"]
    assert g["frames_60s"] * g["tokens_per_frame"] == g["tokens_60s"]
    c1 = W.C1
    assert c1.T_p == g["frames_per_page"] * g["tokens_per_frame"]
    assert c1.L == g["active_tokens"]
    assert c1.B == g["B_intra"]
    assert c1.T_p // c1.B == g["blocks_per_page_B64"] and c1.T_p % c1.B == 0
    assert W.C3.n_pool_pages == g["pages_60s"]


# ----------------------------------------------------------------------------- S0
def test_prompt_select_closed_form_angles():
    # e_cur along axis 0; chunk m at angle theta_m in the (0,1) plane, cos = cos(theta_m)
    D = 16
    thetas = [1.2, 0.4, 2.5, 0.9, 0.41]
    e_cur = np.zeros(D); e_cur[0] = 3.0
    E = np.zeros((len(thetas), D))
    for m, t in enumerate(thetas):
        E[m, 0], E[m, 1] = math.cos(t) * (m + 1), math.sin(t) * (m + 1)
    assert O.prompt_select(e_cur, E) == 1
    assert O.prompt_margin(e_cur, E) == pytest.approx(math.cos(0.4) - math.cos(0.41), rel=1e-9)


def test_prompt_select_scale_invariance_and_ties():
    r = rng(1)
    e = r.normal(size=64); E = r.normal(size=(9, 64))
    m = O.prompt_select(e, E)
    scales = r.uniform(0.1, 10, size=9)
    assert O.prompt_select(e * 7.5, E * scales[:, None]) == m
    # exact copies of the best chunk: the lowest index wins
    E2 = np.concatenate([E[:2], E[m:m + 1], E[m:m + 1]])
    E2[0] = -E[m]
    assert O.prompt_select(e, E2) == 2
    with pytest.raises(ValueError):
        O.prompt_select(np.zeros(64), E)


# ----------------------------------------------------------------------------- S1
def test_page_scores_equal_mean_of_pairwise_dots():
    # bilinearity: Qbar.Kbar = mean over all (query, key) pairs of q.k -- a different
    # computation (pairs, not means) that pins the means, the 1/sqrt(d) and the head average
    r = rng(2)
    Nq, n_c, T_p, H, d = 5, 4, 6, 3, 8
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(n_c, T_p, H, d))
    alpha = O.page_scores(q, k)
    for j in range(n_c):
        acc = 0.0
        for n in range(Nq):
            for t in range(T_p):
                for h in range(H):
                    acc += float(np.dot(q[n, h], k[j, t, h]))
        assert alpha[j] == pytest.approx(acc / (Nq * T_p * H * math.sqrt(d)), rel=1e-12, abs=1e-14)


def test_page_scores_closed_form_constant_pages():
    H, d, T_p = 2, 16, 10
    u = np.linspace(-1, 1, d)
    c = np.array([0.5, -2.0, 3.0, 1.0])
    q = np.tile(u, (7, H, 1))
    k = np.stack([np.tile(cj * u, (T_p, H, 1)) for cj in c])
    alpha = O.page_scores(q, k)
    np.testing.assert_allclose(alpha, c * float(u @ u) / math.sqrt(d), rtol=1e-13)
    assert O.select_pages(alpha, 2) == [2, 3]
    assert O.page_margin(alpha, 2) == pytest.approx((1.0 - 0.5) * float(u @ u) / 4.0)


def test_select_pages_brute_force_and_invariants():
    r = rng(3)
    for trial in range(30):
        n_c = int(r.integers(2, 9)); K_p = int(r.integers(1, n_c + 1))
        alpha = r.normal(size=n_c)
        got = O.select_pages(alpha, K_p)
        best = max(itertools.combinations(range(n_c), K_p), key=lambda s: sum(alpha[list(s)]))
        assert got == sorted(best)
        # positive scaling keeps the set; negation picks the bottom-K_p
        assert O.select_pages(alpha * 3.3, K_p) == got
        worst = min(itertools.combinations(range(n_c), K_p), key=lambda s: sum(alpha[list(s)]))
        assert O.select_pages(-alpha, K_p) == sorted(worst)
    # ties go to the lower position
    assert O.select_pages([1.0, 2.0, 1.0, 1.0], 2) == [0, 1]
    with pytest.raises(ValueError):
        O.select_pages([1.0, 2.0], 3)


def test_page_selection_permutation_invariant():
    r = rng(4)
    Nq, n_c, T_p, H, d = 6, 6, 5, 2, 4
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(n_c, T_p, H, d)) + r.normal(size=(n_c, 1, H, d))
    sel = O.select_pages(O.page_scores(q, k), 3)
    perm = r.permutation(n_c)
    sel_p = O.select_pages(O.page_scores(q, k[perm]), 3)
    assert sorted(perm[sel_p].tolist()) == sel


# ----------------------------------------------------------------------------- S2
def test_gather_is_exact_copy():
    pool = torch.randn(6, 5, 2, 3).to(torch.bfloat16)
    out = O.gather_pages(pool, [4, 1, 5])
    assert out.dtype == torch.bfloat16 and out.shape == (15, 2, 3)
    assert torch.equal(out[0:5], pool[4]) and torch.equal(out[5:10], pool[1]) and torch.equal(out[10:], pool[5])


# ----------------------------------------------------------------------------- S3
def test_block_means_ragged_tail_closed_form():
    N, B = 10, 4
    x = np.arange(N, dtype=np.float64).reshape(N, 1, 1) * np.ones((1, 2, 3))
    m = O.block_means(x, B)
    assert m.shape == (3, 2, 3)
    np.testing.assert_array_equal(m[:, 0, 0], [1.5, 5.5, 8.5])  # last block = rows 8, 9 only


def test_block_scores_equal_mean_pairwise_dots():
    r = rng(5)
    Nq, L, H, d, B = 7, 9, 2, 4, 4
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(L, H, d))
    s = O.block_scores(q, k, B)
    for h in range(H):
        for i in range(2):
            rows = range(i * B, min(Nq, (i + 1) * B))
            for j in range(3):
                keys = range(j * B, min(L, (j + 1) * B))
                acc = sum(float(q[a, h] @ k[b, h]) for a in rows for b in keys)
                assert s[h, i, j] == pytest.approx(acc / (len(rows) * len(keys) * math.sqrt(d)), rel=1e-12, abs=1e-14)


def test_select_row_brute_force_minimal_set():
    r = rng(6)
    for trial in range(200):
        n = int(r.integers(1, 11))
        s = r.normal(size=n) * r.uniform(0.1, 4)
        tau = float(r.uniform(0.05, 0.999))
        kept, margin = O.select_row(s, tau)
        p = np.exp(s - s.max()); p /= p.sum()
        assert abs(p.sum() - 1.0) < 1e-12
        feasible = [c for m in range(1, n + 1) for c in itertools.combinations(range(n), m)
                    if p[list(c)].sum() >= tau]
        best_size = min(len(c) for c in feasible)
        best_mass = max(p[list(c)].sum() for c in feasible if len(c) == best_size)
        if margin > 1e-9:
            assert len(kept) == best_size
            assert p[kept].sum() == pytest.approx(best_mass, abs=1e-12)
        assert kept == sorted(kept)


def test_select_row_limits():
    r = rng(7)
    s = r.normal(size=40)
    assert O.select_row(s, 1e-12)[0] == [int(np.argmax(s))]
    assert O.select_row(s, 1.0)[0] == list(range(40))
    assert O.select_row(s, 1.5)[0] == list(range(40))
    # known weights: p = w exactly up to rounding of log/exp
    w = np.array([0.05, 0.5, 0.15, 0.3])
    s = np.log(w)
    assert O.select_row(s, 0.7)[0] == [1, 3]
    assert O.select_row(s, 0.81)[0] == [1, 2, 3]
    assert O.select_row(s, 0.4)[0] == [1]
    # equal scores: ties go to the lower block index
    assert O.select_row(np.zeros(8), 0.3)[0] == [0, 1, 2]


# ----------------------------------------------------------------------------- S4
def test_linear_branch_identity_projection_is_dense_attention():
    r = rng(8)
    Nq, L, H, d = 9, 12, 2, 8
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    I = np.eye(L)
    kt, vt = O.linear_project(k, v, I, I)
    o = O.linear_attention(q, kt, vt)
    for h in range(H):
        np.testing.assert_allclose(o[:, h], sdpa(q[:, h], k[:, h], v[:, h]), rtol=1e-12, atol=1e-12)


def test_linear_branch_row_selection_pins_orientation():
    # E[l, c] = 1 if l == idx[c]: K~ = K[idx_k], V~ = V[idx_v]  (E_K != E_V)
    r = rng(9)
    Nq, L, H, d, rr = 6, 20, 2, 4, 7
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    ik = r.choice(L, rr, replace=False); iv = r.choice(L, rr, replace=False)
    EK = np.zeros((L, rr)); EK[ik, np.arange(rr)] = 1
    EV = np.zeros((L, rr)); EV[iv, np.arange(rr)] = 1
    kt, vt = O.linear_project(k, v, EK, EV)
    o = O.linear_attention(q, kt, vt)
    for h in range(H):
        np.testing.assert_allclose(o[:, h], sdpa(q[:, h], k[ik, h], v[iv, h]), rtol=1e-12, atol=1e-12)


def test_linear_branch_rank_one_closed_form():
    r = rng(10)
    Nq, L, H, d, rr = 5, 16, 2, 4, 3
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    E = np.ones((L, rr)) / math.sqrt(L)
    kt, vt = O.linear_project(k, v, E, E)
    np.testing.assert_allclose(kt[1], math.sqrt(L) * k.mean(axis=0), rtol=1e-12)
    o = O.linear_attention(q, kt, vt)
    # all K~ rows are equal -> uniform weights -> O_lin = V~ row = sqrt(L) * mean V
    np.testing.assert_allclose(o, np.broadcast_to(math.sqrt(L) * v.mean(axis=0), o.shape), rtol=1e-12)


def test_linear_project_is_linear_in_E():
    r = rng(11)
    L, H, d, rr = 10, 2, 3, 4
    k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    E1, E2 = r.normal(size=(L, rr)), r.normal(size=(L, rr))
    a1, b1 = O.linear_project(k, v, E1, E2)
    a2, b2 = O.linear_project(k, v, E2, E1)
    a3, b3 = O.linear_project(k, v, E1 - 2 * E2, E2 + 0.5 * E1)
    np.testing.assert_allclose(a3, a1 - 2 * a2, atol=1e-12)
    np.testing.assert_allclose(b3, b1 + 0.5 * b2, atol=1e-12)


# ----------------------------------------------------------------------------- S5
def test_sparse_branch_all_blocks_is_dense_attention():
    r = rng(12)
    Nq, L, H, d, B = 11, 14, 2, 8, 4       # ragged query and key tails
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    tau = np.ones(H)
    kept, _ = O.block_select(q, k, tau, B)
    assert all(kept[h][i] == [0, 1, 2, 3] for h in range(H) for i in range(3))
    o = O.sparse_attention(q, k, v, kept, B)
    for h in range(H):
        np.testing.assert_allclose(o[:, h], sdpa(q[:, h], k[:, h], v[:, h]), rtol=1e-12, atol=1e-12)


def test_sparse_branch_matches_masked_dense_attention():
    r = rng(13)
    Nq, L, H, d, B = 10, 22, 3, 4, 4
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    n_qb, n_kb = 3, 6
    kept = [[sorted(r.choice(n_kb, int(r.integers(1, n_kb + 1)), replace=False).tolist())
             for _ in range(n_qb)] for _ in range(H)]
    o = O.sparse_attention(q, k, v, kept, B)
    for h in range(H):
        mask = np.zeros((Nq, L), dtype=bool)
        for i in range(n_qb):
            for j in kept[h][i]:
                mask[i * B:(i + 1) * B, j * B:(j + 1) * B] = True
        np.testing.assert_allclose(o[:, h], sdpa(q[:, h], k[:, h], v[:, h], mask), rtol=1e-12, atol=1e-12)


def test_sparse_branch_single_block_identical_keys():
    r = rng(14)
    B, H, d = 4, 1, 6
    q = r.normal(size=(B, H, d)); k = np.tile(r.normal(size=(1, H, d)), (3 * B, 1, 1))
    v = r.normal(size=(3 * B, H, d))
    o = O.sparse_attention(q, k, v, [[[1]]], B)
    np.testing.assert_allclose(o[:, 0], np.broadcast_to(v[B:2 * B, 0].mean(axis=0), (B, d)), rtol=1e-12)


# ----------------------------------------------------------------------------- S6
def test_gate_limits():
    r = rng(15)
    a = r.normal(size=(4, 2, 3)); b = r.normal(size=(4, 2, 3))
    np.testing.assert_allclose(O.gate_fuse(a, b, np.full((4, 2), 60.0)), a, atol=1e-20)
    np.testing.assert_allclose(O.gate_fuse(a, b, np.full((4, 2), -60.0)), b, atol=1e-20)
    np.testing.assert_allclose(O.gate_fuse(a, b, np.zeros((4, 2))), 0.5 * (a + b), rtol=1e-15)
    g = r.normal(size=(4, 2))
    np.testing.assert_allclose(O.sigmoid(g) + O.sigmoid(-g), 1.0, rtol=1e-15)


def test_two_gate_fusion_pins():
    """Two sigmoid gates, one per branch: limits per gate, the zero point, the one-gate
    form as the special case g_lin = -g_sp, and per-(token, head) independence."""
    r = rng(16)
    a = r.normal(size=(4, 2, 3)); b = r.normal(size=(4, 2, 3))
    big = np.full((4, 2), 60.0)
    np.testing.assert_allclose(O.gate_fuse2(a, b, big, -big), a, atol=1e-20)
    np.testing.assert_allclose(O.gate_fuse2(a, b, -big, big), b, atol=1e-20)
    np.testing.assert_allclose(O.gate_fuse2(a, b, big, big), a + b, rtol=1e-15)
    np.testing.assert_allclose(O.gate_fuse2(a, b, -big, -big), 0.0, atol=1e-20)
    np.testing.assert_allclose(O.gate_fuse2(a, b, np.zeros((4, 2)), np.zeros((4, 2))), 0.5 * (a + b),
                               rtol=1e-15)
    g = r.normal(size=(4, 2))
    np.testing.assert_allclose(O.gate_fuse2(a, b, g, -g), O.gate_fuse(a, b, g), rtol=1e-14)
    # changing one (token, head) gate changes only that (token, head) row
    g2 = r.normal(size=(4, 2)); gl = r.normal(size=(4, 2))
    base = O.gate_fuse2(a, b, g2, gl)
    gl_mod = gl.copy(); gl_mod[1, 0] += 1.0
    mod = O.gate_fuse2(a, b, g2, gl_mod)
    changed = np.any(mod != base, axis=2)
    assert changed[1, 0] and changed.sum() == 1


def _intra_cfg(**kw):
    # ragged query tail (Nq % B = 8): the current chunk's last key block has 8 rows
    return W.C0.with_(T_p=64, Nq=72, intra=True, **kw)


def test_intra_keys_tau_one_is_dense_attention_over_history_and_chunk():
    """tau = 1 keeps every block, so the sparse branch is textbook attention over
    the retrieved history followed by the current chunk's own keys."""
    cfg = _intra_cfg(tau_const=1.0)
    inp = W.make_inputs(cfg)
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    k_all = np.concatenate([O.f64(res["k_act"]), O.f64(inp["k_cur"])])
    v_all = np.concatenate([O.f64(res["v_act"]), O.f64(inp["v_cur"])])
    n_all = -(-k_all.shape[0] // cfg.B)
    assert all(len(row) == n_all for row in res["kept"][0])
    q = O.f64(inp["q"])[:, 0, :]
    np.testing.assert_allclose(res["o_sp"][:, 0, :], sdpa(q, k_all[:, 0, :], v_all[:, 0, :]),
                               rtol=1e-12, atol=1e-13)


def test_intra_keys_hot_chunk_blocks_are_selected_and_linear_branch_ignores_them():
    """Current-chunk keys pushed toward the mean query carry almost all pooled mass:
    a low tau keeps only chunk blocks, including the 8-row tail pooled over its valid
    rows; the linear branch (over the history) does not change."""
    cfg = _intra_cfg(tau_const=0.5)
    inp = W.make_inputs(cfg)
    # a common query direction u for every query block, and chunk keys along u
    u = torch.from_numpy(rng(18).normal(size=(cfg.H, cfg.d))).float()
    u = u / u.norm(dim=-1, keepdim=True)
    inp["q"] = inp["q"] + 3.0 * u[None]
    inp["k_cur"] = inp["k_cur"] + 40.0 * u[None]
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    n_hist = cfg.L // cfg.B
    n_all = n_hist + -(-cfg.Nq // cfg.B)
    for row in res["kept"][0]:
        assert row and all(n_hist <= j < n_all for j in row)
    base = dict(inp); base.pop("k_cur"); base.pop("v_cur")
    res0 = O.hsa_step(base, cfg.B, cfg.K_p)
    np.testing.assert_array_equal(res["o_lin"], res0["o_lin"])
    # the tail block's pooled mean uses its 8 valid rows
    kb = O.block_means(np.concatenate([O.f64(res["k_act"]), O.f64(inp["k_cur"])]), cfg.B)
    tail = O.f64(inp["k_cur"])[64:72].mean(axis=0)
    np.testing.assert_allclose(kb[n_all - 1], tail, rtol=1e-15, atol=1e-15)


def test_step_two_gates_matches_recombined_branches():
    cfg = W.C0.with_(T_p=64, Nq=72)
    inp = W.make_inputs(cfg)
    inp["gate_lin"] = torch.from_numpy(rng(17).normal(size=(cfg.Nq, cfg.H))).float()
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    expect = O.gate_fuse2(res["o_sp"], res["o_lin"], inp["gate"].double().numpy(),
                          inp["gate_lin"].double().numpy())
    np.testing.assert_array_equal(res["o"], expect)
    inp_one = dict(inp); inp_one["gate_lin"] = -inp["gate"]
    res_one = O.hsa_step(inp_one, cfg.B, cfg.K_p)
    np.testing.assert_allclose(res_one["o"], O.gate_fuse(res["o_sp"], res["o_lin"], inp["gate"]),
                               rtol=1e-13, atol=1e-15)


# ----------------------------------------------------------------------------- step
def test_step_composes_pinned_parts_on_tiny_workload():
    cfg = W.C0.with_(T_p=64, Nq=72)
    inp = W.make_inputs(cfg)
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    assert len(res["sel"]) == cfg.K_p and res["sel"] == sorted(res["sel"])
    k_act = torch.cat([inp["k_pool"][p] for p in res["sel"]]).double().numpy()
    v_act = torch.cat([inp["v_pool"][p] for p in res["sel"]]).double().numpy()
    q = inp["q"].double().numpy()
    # sparse branch = masked textbook attention; linear branch = textbook attention over
    # the projected keys; gate by the sigmoid of g
    h = 0
    mask = np.zeros((cfg.Nq, cfg.L), dtype=bool)
    for i, ks in enumerate(res["kept"][h]):
        for j in ks:
            mask[i * cfg.B:(i + 1) * cfg.B, j * cfg.B:(j + 1) * cfg.B] = True
    o_sp = sdpa(q[:, h], k_act[:, h], v_act[:, h], mask)
    EK = inp["e_k"].double().numpy(); EV = inp["e_v"].double().numpy()
    o_lin = sdpa(q[:, h], EK.T @ k_act[:, h], EV.T @ v_act[:, h])
    s = 1.0 / (1.0 + np.exp(-inp["gate"].double().numpy()[:, h:h + 1]))
    np.testing.assert_allclose(res["o"][:, h], s * o_sp + (1 - s) * o_lin, rtol=1e-10, atol=1e-12)


def test_step_sampled_rows_equal_full():
    cfg = W.C0.with_(T_p=64, Nq=100)
    inp = W.make_inputs(cfg)
    full = O.hsa_step(inp, cfg.B, cfg.K_p)
    part = O.hsa_step(inp, cfg.B, cfg.K_p, rows_of_blocks=[(0, 1), (0, 0)])
    for (h, i), blk in part["blocks"].items():
        np.testing.assert_allclose(blk["o"], full["o"][i * cfg.B:(i + 1) * cfg.B, h], rtol=1e-13, atol=1e-14)


def test_prompt_selected_chunk_drives_candidates():
    cfg = W.C0.with_(T_p=64, Nq=64, n_chunks=3, prompt_dim=32)
    inp = W.make_inputs(cfg)
    inp["e_cur"] = inp["e_chunks"][2] * 2.0
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    assert res["chunk"] == 2
    assert set(res["sel"]) <= set(range(2 * cfg.n_c, 3 * cfg.n_c))


# ---------------------------------------------------------------- token order (A.1.3)
def test_cube_order_hand_examples():
    # 2 frames of 2 x 4 tokens (raster ids 0-7 in frame 0, 8-15 in frame 1), cubes of
    # (1, 2, 2): frame 0 left cube {0, 1, 4, 5}, right cube {2, 3, 6, 7}, then frame 1
    assert O.cube_order(2, 2, 4, 1, 2, 2) == [0, 1, 4, 5, 2, 3, 6, 7, 8, 9, 12, 13, 10, 11, 14, 15]
    # one 3 x 3 frame, (1, 2, 2) cubes cut short at the far edges:
    # {0, 1, 3, 4}, {2, 5}, {6, 7}, {8}
    assert O.cube_order(1, 3, 3, 1, 2, 2) == [0, 1, 3, 4, 2, 5, 6, 7, 8]
    # one cube covering everything, a cube per token, and a cube per row are raster order
    for cube in [(2, 3, 5), (1, 1, 1), (1, 1, 5)]:
        assert O.cube_order(2, 3, 5, *cube) == list(range(30))


@pytest.mark.parametrize("grid,cube", [((8, 10, 16), (8, 2, 4)), ((4, 6, 8), (2, 3, 4)),
                                       ((8, 30, 52), (8, 2, 4))])
def test_cube_order_groups_are_cubes(grid, cube):
    T, Hl, Wl = grid
    ct, ch, cw = cube
    perm = O.cube_order(T, Hl, Wl, ct, ch, cw)
    n = T * Hl * Wl
    assert sorted(perm) == list(range(n))          # a permutation
    Bc = ct * ch * cw
    corners = []
    for g in range(n // Bc):
        pts = [divmod(divmod(x, Wl)[0], Hl) + (x % Wl,) for x in perm[g * Bc:(g + 1) * Bc]]
        ts, hs, ws = zip(*pts)
        t0, h0, w0 = min(ts), min(hs), min(ws)
        # the group is exactly the cube with this corner, aligned to the cube grid
        assert (t0 % ct, h0 % ch, w0 % cw) == (0, 0, 0)
        assert set(pts) == {(t, h, w) for t in range(t0, t0 + ct) for h in range(h0, h0 + ch)
                            for w in range(w0, w0 + cw)}
        corners.append((t0, h0, w0))
    assert corners == sorted(corners)              # cubes in raster order of their corners


# --------------------------------------------- mixed key-block granularity (§3.3)
def test_key_block_bounds_hand_example_and_page_shape():
    # 10 history tokens in blocks of 4, then 5 chunk tokens in blocks of 2
    assert O.key_block_bounds(10, 4, 5, 2) == [(0, 4), (4, 8), (8, 10), (10, 12), (12, 14), (14, 15)]
    assert O.key_block_bounds(8, 4) == [(0, 4), (4, 8)]
    # the one-layer shape: 4 pages of 12,480 tokens in 128-token blocks = 390 blocks (no
    # ragged block); block 97 spans pages 0 and 1; then 4680 chunk tokens in 74 blocks of 64
    kb = O.key_block_bounds(4 * 12480, 128, 4680, 64)
    assert len(kb) == 390 + 74
    assert kb[97] == (12416, 12544) and kb[97][0] < 12480 < kb[97][1]
    assert kb[389] == (49792, 49920) and kb[390] == (49920, 49984)
    assert kb[-1] == (49920 + 4672, 49920 + 4680)
    # expansion to 64-token blocks: a 128-block covers two, a chunk block one
    assert O.expand_blocks([97, 390], kb, 64) == [194, 195, 780]
    assert O.expand_blocks([2], O.key_block_bounds(10, 4), 2) == [4]


def test_mixed_block_means_closed_form():
    # x[n] = n in every entry: the mean of rows [s, e) is (s + e - 1) / 2
    n = 200
    x = np.arange(n, dtype=np.float64).reshape(n, 1, 1) * np.ones((1, 2, 3))
    kb = O.key_block_bounds(150, 128, 50, 64)   # blocks (0,128), (128,150), (150,200)
    m = O.block_means_at(x, kb)
    np.testing.assert_array_equal(m[:, 1, 2], [63.5, 138.5, 174.5])
    # a block spanning two 64-token halves has the mean of the two halves' means
    m64 = O.block_means(x[:128], 64)
    np.testing.assert_array_equal(m[0], 0.5 * (m64[0] + m64[1]))


def test_mixed_granularity_tau_one_is_dense_attention():
    """With tau = 1 every block is kept whatever its size: the sparse branch is textbook
    attention over the history followed by the chunk's own keys."""
    cfg = W.C0.with_(T_p=192, Nq=72, intra=True, tau_const=1.0)
    inp = W.make_inputs(cfg)
    res = O.hsa_step(inp, cfg.B, cfg.K_p, B_inter=128)
    kb = res["key_bounds"]
    assert len(kb) == (cfg.L // 128) + 2 and all(e - s == 128 for s, e in kb[:cfg.L // 128])
    k_all = np.concatenate([O.f64(res["k_act"]), O.f64(inp["k_cur"])])
    v_all = np.concatenate([O.f64(res["v_act"]), O.f64(inp["v_cur"])])
    q = O.f64(inp["q"])[:, 0, :]
    np.testing.assert_allclose(res["o_sp"][:, 0, :], sdpa(q, k_all[:, 0, :], v_all[:, 0, :]),
                               rtol=1e-12, atol=1e-13)


def test_mixed_granularity_selection_brute_force():
    """Per row: scores of mixed-size blocks from pairwise dot products (mean over the
    query block's rows and the key block's rows), then the kept set is the smallest set
    of blocks whose softmax mass reaches tau, the largest mass among those."""
    r = rng(31)
    H, d, B = 2, 4, 4
    for trial in range(12):
        L_hist, L_cur, Nq = int(r.integers(9, 24)), int(r.integers(1, 9)), int(r.integers(3, 10))
        q = r.normal(size=(Nq, H, d))
        k = r.normal(size=(L_hist + L_cur, H, d)) * r.uniform(0.3, 3)
        kb = O.key_block_bounds(L_hist, 8, L_cur, B)
        if len(kb) > 10:
            continue
        tau = np.full(H, r.uniform(0.2, 0.95))
        kept, margin = O.block_select(q, k, tau, B, key_bounds=kb)
        for h in range(H):
            for i in range(-(-Nq // B)):
                rows = range(i * B, min(Nq, (i + 1) * B))
                s = np.array([sum(float(q[a, h] @ k[b, h]) for a in rows for b in range(s0, e0))
                              / (len(rows) * (e0 - s0) * math.sqrt(d)) for (s0, e0) in kb])
                p = np.exp(s - s.max()); p /= p.sum()
                feasible = [c for m in range(1, len(kb) + 1) for c in itertools.combinations(range(len(kb)), m)
                            if p[list(c)].sum() >= tau[h]]
                best = min(len(c) for c in feasible)
                best_mass = max(p[list(c)].sum() for c in feasible if len(c) == best)
                if margin[h, i] > 1e-9:
                    assert len(kept[h][i]) == best
                    assert p[kept[h][i]].sum() == pytest.approx(best_mass, abs=1e-12)


def test_mixed_granularity_equal_sizes_is_uniform():
    cfg = _intra_cfg(tau_const=0.7)
    inp = W.make_inputs(cfg)
    a = O.hsa_step(inp, cfg.B, cfg.K_p)
    b = O.hsa_step(inp, cfg.B, cfg.K_p, B_inter=cfg.B)
    assert a["kept"] == b["kept"]
    np.testing.assert_array_equal(a["o"], b["o"])


# ----------------------------------------------- per-head Linformer projections (§3.3)
def test_linear_branch_per_head_row_selection():
    """One E per head (K~^(h) = E_K^(h)T K^(h)): with a different row selection per head
    and per branch, each head's linear branch is textbook attention over its own
    selected rows -- which pins the head each E goes with and its orientation."""
    r = rng(41)
    Nq, L, H, d, rr = 5, 18, 3, 4, 6
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    EK = np.zeros((H, L, rr)); EV = np.zeros((H, L, rr))
    sel_k = [r.choice(L, rr, replace=False) for _ in range(H)]
    sel_v = [r.choice(L, rr, replace=False) for _ in range(H)]
    for h in range(H):
        EK[h, sel_k[h], np.arange(rr)] = 1
        EV[h, sel_v[h], np.arange(rr)] = 1
    kt, vt = O.linear_project(k, v, EK, EV)
    o = O.linear_attention(q, kt, vt)
    for h in range(H):
        np.testing.assert_allclose(o[:, h], sdpa(q[:, h], k[sel_k[h], h], v[sel_v[h], h]),
                                   rtol=1e-12, atol=1e-12)


def test_linear_branch_per_head_identity_is_dense_attention():
    r = rng(42)
    Nq, L, H, d = 4, 9, 2, 3
    q = r.normal(size=(Nq, H, d)); k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    E = np.stack([np.eye(L)] * H)
    kt, vt = O.linear_project(k, v, E, E)
    o = O.linear_attention(q, kt, vt)
    for h in range(H):
        np.testing.assert_allclose(o[:, h], sdpa(q[:, h], k[:, h], v[:, h]), rtol=1e-12, atol=1e-12)


def test_linear_project_per_head_copies_equal_shared():
    """A per-head E whose heads all hold the same matrix is the shared projection."""
    r = rng(43)
    L, H, d, rr = 11, 3, 4, 5
    k = r.normal(size=(L, H, d)); v = r.normal(size=(L, H, d))
    EK = r.normal(size=(L, rr)); EV = r.normal(size=(L, rr))
    kt_s, vt_s = O.linear_project(k, v, EK, EV)
    kt_h, vt_h = O.linear_project(k, v, np.stack([EK] * H), np.stack([EV] * H))
    np.testing.assert_allclose(kt_h, kt_s, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(vt_h, vt_s, rtol=1e-13, atol=1e-13)
