"""GPU parity: every libwa entry point against the float64 oracle on the same seeded
inputs.  Small shapes span several tiles with ragged query (and key) tails; the
one-layer bf16 workload runs at full size in the launch configuration the bench
times (the fused page-table step) and is checked on sampled (head, query block)
outputs plus every page / block selection."""
import math

import numpy as np
import pytest
import torch

from oracle import hsa_oracle as O
from linear_attention_paged_b200 import workloads as W
from tests.helpers import (MARGIN_F64, assert_close, compare_selection, mask_to_sets, kept_fraction,
                           to64)

pytestmark = pytest.mark.gpu

# small multi-tile shapes (ragged query tails; odd n_qb leaves one unpaired block)
SMALL_BF16 = W.HSAConfig("small_bf16", H=2, d=128, T_p=1280, n_c=6, Nq=520, K_p=3, B=64, r=128,
                         dtype="bf16", seed=11, recipe="offset")
SMALL_BF16_D64 = W.HSAConfig("small_bf16_d64", H=4, d=64, T_p=640, n_c=5, Nq=300, K_p=2, B=64,
                             r=256, dtype="bf16", seed=12, recipe="offset")
SMALL_STRESS = W.HSAConfig("small_stress", H=4, d=128, T_p=1280, n_c=4, Nq=640, K_p=2, B=64, r=128,
                           dtype="bf16", seed=13, recipe="stress", hot_beta_scale=12.0)
SMALL_F32 = W.HSAConfig("small_f32", H=2, d=128, T_p=320, n_c=4, Nq=150, K_p=2, B=64, r=48,
                        dtype="f32", seed=14, recipe="offset")


@pytest.fixture(scope="module")
def wa():
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa as _wa
    return _wa


def inputs(cfg, device="cuda"):
    return W.make_inputs(cfg, device=device)


def dkey(cfg):
    return "f32" if cfg.dtype == "f32" else "bf16"


def check_device_ok(wa):
    flags = wa.wa_device_error()
    assert flags == 0, f"device error flags 0x{flags:x}"


# ---------------------------------------------------------------- S0
def test_prompt_select(wa):
    g = torch.Generator().manual_seed(5)
    e = torch.randn(4096, generator=g)
    E = torch.randn(15, 4096, generator=g)
    E[9] = e * 0.5 + E[9] * 0.1
    got = int(wa.wa_prompt_select(e.cuda(), E.cuda()).item())
    assert got == O.prompt_select(e, E) == 9
    for s in range(5):
        E = torch.randn(40, 512, generator=g)
        e = torch.randn(512, generator=g)
        assert int(wa.wa_prompt_select(e.cuda(), E.cuda()).item()) == O.prompt_select(e, E)
    check_device_ok(wa)


def test_prompt_select_zero_norm_flags(wa):
    E = torch.randn(4, 64)
    E[2] = 0
    out = wa.wa_prompt_select(torch.randn(64).cuda(), E.cuda())
    assert int(out.item()) == -1
    assert wa.wa_device_error() & wa.DEVERR_ZERO_NORM


# ---------------------------------------------------------------- S1 + S2
@pytest.mark.parametrize("cfg", [W.C0, SMALL_BF16, SMALL_BF16_D64, SMALL_F32], ids=lambda c: c.name)
def test_page_score_and_gather(wa, cfg):
    inp = inputs(cfg)
    alpha, sel, kbm = wa.wa_page_score(inp["q"], inp["k_pool"], inp["cand"], cfg.K_p, cfg.B,
                                       want_blockmean=True)
    k_cand = np.stack([to64(inp["k_pool"][int(p)]) for p in inp["cand"].cpu()])
    a_ref = O.page_scores(inp["q"], k_cand)
    np.testing.assert_allclose(to64(alpha), a_ref, rtol=1e-10, atol=1e-13)
    margin = O.page_margin(a_ref, cfg.K_p)
    ref_sel = [int(inp["cand"][j]) for j in O.select_pages(a_ref, cfg.K_p)]
    if margin >= MARGIN_F64:
        assert sel.cpu().tolist() == ref_sel
    # block means of every candidate page
    ref_bm = np.stack([O.block_means(k_cand[c], cfg.B) for c in range(cfg.n_c)])
    np.testing.assert_allclose(to64(kbm), ref_bm, rtol=1e-10, atol=1e-13)
    # gather: a bit-exact copy
    k_act, v_act = wa.wa_gather_pages(inp["k_pool"], inp["v_pool"], sel)
    assert torch.equal(k_act, O.gather_pages(inp["k_pool"], sel.cpu().tolist()))
    assert torch.equal(v_act, O.gather_pages(inp["v_pool"], sel.cpu().tolist()))
    check_device_ok(wa)


def test_page_score_bad_page_id_is_flagged(wa):
    cfg = SMALL_BF16
    inp = inputs(cfg)
    cand = inp["cand"].clone()
    cand[1] = cfg.n_pool_pages + 5            # outside the pool: skipped and recorded
    wa.wa_page_score(inp["q"], inp["k_pool"], cand, cfg.K_p, cfg.B)
    assert wa.wa_device_error() & wa.DEVERR_PAGE_ID
    sel = torch.tensor([0, 99], dtype=torch.int32, device="cuda")
    wa.wa_gather_pages(inp["k_pool"], inp["v_pool"], sel)
    assert wa.wa_device_error() & wa.DEVERR_PAGE_ID


# ---------------------------------------------------------------- S3
@pytest.mark.parametrize("cfg", [W.C0, SMALL_BF16, SMALL_BF16_D64, SMALL_STRESS, SMALL_F32],
                         ids=lambda c: c.name)
def test_block_select(wa, cfg):
    inp = inputs(cfg)
    sel = [int(x) for x in inp["cand"][: cfg.K_p].cpu()]
    k_act = O.gather_pages(inp["k_pool"], sel)
    kept, margin = O.block_select(inp["q"], k_act, inp["tau"], cfg.B)
    idx, cnt, mask = wa.wa_block_select(inp["q"], inp["tau"].cuda(), cfg.B, k_act=k_act)
    gpu = mask_to_sets(mask, cfg.n_kb)
    compare_selection(gpu, kept, margin, f"{cfg.name} block masks")
    # index lists and counts agree with the mask
    idx_c, cnt_c = idx.cpu().numpy(), cnt.cpu().numpy()
    for h in range(cfg.H):
        for i in range(cfg.n_qb):
            c = int(cnt_c[h, i])
            assert idx_c[h, i, :c].tolist() == gpu[h][i]
            assert (idx_c[h, i, c:] == -1).all()
    print(f"[info] {cfg.name} kept fraction per head: {np.round(kept_fraction(kept, cfg.n_kb), 3)}")
    # the same from precomputed block means
    kbm = torch.from_numpy(O.block_means(k_act, cfg.B)).cuda()
    _, _, mask2 = wa.wa_block_select(inp["q"], inp["tau"].cuda(), cfg.B, k_blockmean=kbm, L=cfg.L)
    compare_selection(mask_to_sets(mask2, cfg.n_kb), kept, margin, f"{cfg.name} masks from means")
    check_device_ok(wa)


def test_block_select_limits(wa):
    cfg = SMALL_BF16
    inp = inputs(cfg)
    k_act = O.gather_pages(inp["k_pool"], [0, 1, 2])
    for tval, expect in ((1.0, "all"), (1e-9, "one")):
        tau = torch.full((cfg.H,), tval, dtype=torch.float32, device="cuda")
        _, cnt, mask = wa.wa_block_select(inp["q"], tau, cfg.B, k_act=k_act)
        c = cnt.cpu().numpy()
        if expect == "all":
            assert (c == cfg.n_kb).all()
        else:
            assert (c == 1).all()
            s = O.block_scores(inp["q"], k_act, cfg.B)
            gpu = mask_to_sets(mask, cfg.n_kb)
            for h in range(cfg.H):
                for i in range(cfg.n_qb):
                    assert gpu[h][i] == [int(np.argmax(s[h, i]))]


@pytest.mark.parametrize("n_kb", [1, 7, 32, 33, 64, 100, 128, 200, 256, 300, 512, 700, 1024, 1025,
                                  1500])
def test_block_select_key_list_lengths(wa, n_kb):
    """The block choice at every class of key-list length: rows of up to 1024 blocks
    are sorted by one warp (1 to 32 positions per lane), longer ones by a whole CTA.
    Every row of a key block is the same, so a block's mean is exact; repeated blocks
    give bit-identical scores on both sides (exact ties, broken towards the lower
    block) and zero blocks scores of +-0.  Every row must match the oracle exactly."""
    g = torch.Generator().manual_seed(500 + n_kb)
    H, d, B = 2, 64, 64
    Nq = 3 * B - 5
    q = torch.randn(Nq, H, d, generator=g).to(torch.bfloat16)
    rows = torch.randn(n_kb, H, d, generator=g)
    for j in range(n_kb):
        if j % 5 == 4:
            rows[j] = rows[j // 2]
        if j % 7 == 6:
            rows[j] = 0.0
    k_act = rows.to(torch.bfloat16).repeat_interleave(B, dim=0)
    n_qb = -(-Nq // B)
    for tau_vals in ((0.9, 0.3), (0.6, 0.97), (1e-9, 1.0)):
        tau = torch.tensor(tau_vals, dtype=torch.float32)
        kept, _ = O.block_select(q, k_act, tau, B)
        idx, cnt, mask = wa.wa_block_select(q.cuda(), tau.cuda(), B, k_act=k_act.cuda())
        gpu = mask_to_sets(mask, n_kb)
        idx_c, cnt_c = idx.cpu().numpy(), cnt.cpu().numpy()
        for h in range(H):
            for i in range(n_qb):
                assert gpu[h][i] == kept[h][i], (n_kb, tau_vals, h, i)
                c = int(cnt_c[h, i])
                assert c == len(kept[h][i])
                assert idx_c[h, i, :c].tolist() == kept[h][i]
                assert (idx_c[h, i, c:] == -1).all()
    check_device_ok(wa)


# ---------------------------------------------------------------- S4a
@pytest.mark.parametrize("cfg", [W.C0, SMALL_BF16, SMALL_BF16_D64, SMALL_F32], ids=lambda c: c.name)
def test_linear_project(wa, cfg):
    inp = inputs(cfg)
    sel = [int(x) for x in inp["cand"][: cfg.K_p].cpu()]
    k_act = O.gather_pages(inp["k_pool"], sel)
    v_act = O.gather_pages(inp["v_pool"], sel)
    kt, vt = wa.wa_linear_project(k_act, v_act, inp["e_k"], inp["e_v"])
    kr, vr = O.linear_project(k_act, v_act, inp["e_k"], inp["e_v"])
    assert_close(kt, kr, dkey(cfg), f"{cfg.name} K~")
    assert_close(vt, vr, dkey(cfg), f"{cfg.name} V~")
    check_device_ok(wa)


@pytest.mark.parametrize("cfg", [SMALL_BF16, SMALL_BF16_D64, SMALL_F32], ids=lambda c: c.name)
def test_linear_project_per_head(wa, cfg):
    """One projection per head (e_k, e_v [H][L][r]): each head's K~, V~ against the
    oracle; the bf16 path then tiles the columns within one head."""
    cfg = cfg.with_(e_per_head=True)
    inp = inputs(cfg)
    assert inp["e_k"].dim() == 3 and inp["e_k"].shape[0] == cfg.H
    sel = [int(x) for x in inp["cand"][: cfg.K_p].cpu()]
    k_act = O.gather_pages(inp["k_pool"], sel)
    v_act = O.gather_pages(inp["v_pool"], sel)
    kt, vt = wa.wa_linear_project(k_act, v_act, inp["e_k"], inp["e_v"])
    kr, vr = O.linear_project(k_act, v_act, inp["e_k"], inp["e_v"])
    assert_close(kt, kr, dkey(cfg), f"{cfg.name} per-head K~")
    assert_close(vt, vr, dkey(cfg), f"{cfg.name} per-head V~")
    check_device_ok(wa)


# ---------------------------------------------------------------- S4b + S5 + S6
@pytest.mark.parametrize("cfg", [W.C0, SMALL_BF16, SMALL_BF16_D64, SMALL_STRESS, SMALL_F32],
                         ids=lambda c: c.name)
def test_hsa_attention(wa, cfg):
    inp = inputs(cfg)
    sel = [int(x) for x in inp["cand"][: cfg.K_p].cpu()]
    k_act = O.gather_pages(inp["k_pool"], sel)
    v_act = O.gather_pages(inp["v_pool"], sel)
    kept, margin = O.block_select(inp["q"], k_act, inp["tau"], cfg.B)
    _, _, mask = wa.wa_block_select(inp["q"], inp["tau"].cuda(), cfg.B, k_act=k_act)
    compare_selection(mask_to_sets(mask, cfg.n_kb), kept, margin, f"{cfg.name} masks")
    kt, vt = O.linear_project(k_act, v_act, inp["e_k"], inp["e_v"])
    # the branches take the projected keys in the input dtype
    kt_in = torch.from_numpy(kt).to(cfg.torch_dtype).cuda()
    vt_in = torch.from_numpy(vt).to(cfg.torch_dtype).cuda()
    out, o_sp, o_lin = wa.wa_hsa_attention(inp["q"], k_act, v_act, mask, kt_in, vt_in, inp["gate"],
                                           cfg.B, want_branches=True)
    ref_sp = O.sparse_attention(inp["q"], k_act, v_act, kept, cfg.B)
    ref_lin = O.linear_attention(inp["q"], kt_in, vt_in)
    ref = O.gate_fuse(ref_sp, ref_lin, inp["gate"])
    assert_close(o_lin, ref_lin, dkey(cfg), f"{cfg.name} O_lin")
    assert_close(o_sp, ref_sp, dkey(cfg), f"{cfg.name} O_sp")
    assert_close(out, ref, dkey(cfg), f"{cfg.name} O")
    check_device_ok(wa)


def test_hsa_attention_identities(wa):
    """tau = 1 gives dense attention; an empty mask gives O_sp = 0; a ragged key tail."""
    cfg = SMALL_BF16.with_(seed=21)
    inp = inputs(cfg)
    L = 1000                                      # not a multiple of B: masked key tail
    k_act = O.gather_pages(inp["k_pool"], [0])[:L].contiguous()
    v_act = O.gather_pages(inp["v_pool"], [0])[:L].contiguous()
    n_kb = -(-L // cfg.B)
    ones = torch.ones(cfg.H, dtype=torch.float32, device="cuda")
    _, cnt, mask = wa.wa_block_select(inp["q"], ones, cfg.B, k_act=k_act)
    assert (cnt.cpu() == n_kb).all()
    e = torch.randn(L, cfg.r, generator=torch.Generator().manual_seed(3)) / math.sqrt(L)
    e = e.to(torch.bfloat16).cuda()
    kt, vt = wa.wa_linear_project(k_act, v_act, e, e)
    out, o_sp, o_lin = wa.wa_hsa_attention(inp["q"], k_act, v_act, mask, kt, vt, inp["gate"], cfg.B,
                                           want_branches=True)
    dense = O.sparse_attention(inp["q"], k_act, v_act, [[list(range(n_kb))] * cfg.n_qb] * cfg.H, cfg.B)
    assert_close(o_sp, dense, "bf16", "tau=1 sparse branch = dense attention")
    zero = torch.zeros_like(mask)
    out0, o_sp0, o_lin0 = wa.wa_hsa_attention(inp["q"], k_act, v_act, zero, kt, vt, inp["gate"], cfg.B,
                                              want_branches=True)
    assert float(o_sp0.abs().max()) == 0.0
    s = torch.sigmoid(inp["gate"]).unsqueeze(-1)
    assert_close(out0, (1 - s) * o_lin0, "bf16", "empty mask -> (1 - sigmoid(g)) O_lin")
    check_device_ok(wa)


@pytest.mark.parametrize("cfg", [SMALL_BF16, SMALL_BF16_D64, SMALL_F32], ids=lambda c: c.name)
def test_hsa_attention_two_gates(wa, cfg):
    """sigmoid(g_sp) O_sp + sigmoid(g_lin) O_lin against the oracle's two-gate fusion;
    g_lin = -g_sp reproduces the one-gate entry point."""
    inp = inputs(cfg)
    sel = [int(x) for x in inp["cand"][: cfg.K_p].cpu()]
    k_act = O.gather_pages(inp["k_pool"], sel)
    v_act = O.gather_pages(inp["v_pool"], sel)
    kept, margin = O.block_select(inp["q"], k_act, inp["tau"], cfg.B)
    _, _, mask = wa.wa_block_select(inp["q"], inp["tau"].cuda(), cfg.B, k_act=k_act)
    compare_selection(mask_to_sets(mask, cfg.n_kb), kept, margin, f"{cfg.name} masks")
    kt, vt = O.linear_project(k_act, v_act, inp["e_k"], inp["e_v"])
    kt_in = torch.from_numpy(kt).to(cfg.torch_dtype).cuda()
    vt_in = torch.from_numpy(vt).to(cfg.torch_dtype).cuda()
    g_lin = torch.randn(inp["gate"].shape, generator=torch.Generator().manual_seed(cfg.seed + 5)).cuda()
    out, o_sp, o_lin = wa.wa_hsa_attention(inp["q"], k_act, v_act, mask, kt_in, vt_in, inp["gate"],
                                           cfg.B, want_branches=True, gate_lin=g_lin)
    ref_sp = O.sparse_attention(inp["q"], k_act, v_act, kept, cfg.B)
    ref_lin = O.linear_attention(inp["q"], kt_in, vt_in)
    assert_close(o_lin, ref_lin, dkey(cfg), f"{cfg.name} O_lin")
    assert_close(o_sp, ref_sp, dkey(cfg), f"{cfg.name} O_sp")
    assert_close(out, O.gate_fuse2(ref_sp, ref_lin, inp["gate"], g_lin), dkey(cfg), f"{cfg.name} O (two gates)")
    one = wa.wa_hsa_attention(inp["q"], k_act, v_act, mask, kt_in, vt_in, inp["gate"], cfg.B)
    neg = wa.wa_hsa_attention(inp["q"], k_act, v_act, mask, kt_in, vt_in, inp["gate"], cfg.B,
                              gate_lin=-inp["gate"])
    assert torch.equal(neg, one), f"{cfg.name}: g_lin = -g must reproduce the one-gate output exactly"
    check_device_ok(wa)


# ---------------------------------------------------------------- whole step
@pytest.mark.parametrize("cfg", [SMALL_BF16, SMALL_F32], ids=lambda c: c.name)
def test_hsa_step_two_gates(wa, cfg):
    inp = inputs(cfg)
    g_lin = torch.randn(inp["gate"].shape, generator=torch.Generator().manual_seed(cfg.seed + 6)).cuda()
    out, inter = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                                inp["e_v"], inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B,
                                keep_intermediates=True, gate_lin=g_lin)
    inp_o = dict(inp)
    inp_o["gate_lin"] = g_lin.cpu()
    res = O.hsa_step(inp_o, cfg.B, cfg.K_p)
    compare_selection(mask_to_sets(inter["blk_mask"], cfg.n_kb), res["kept"], res["block_margin"],
                      f"{cfg.name} step masks")
    assert_close(out, res["o"], dkey(cfg), f"{cfg.name} step O (two gates)")
    check_device_ok(wa)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "gathered"])
@pytest.mark.parametrize("cfg", [W.C0, SMALL_BF16, SMALL_BF16_D64, SMALL_F32], ids=lambda c: c.name)
def test_hsa_step_small(wa, cfg, fused):
    inp = inputs(cfg)
    out, inter = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                                inp["e_v"], inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B,
                                fused_gather=fused, keep_intermediates=True)
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    if res["page_margin"] >= MARGIN_F64:
        assert inter["sel"].cpu().tolist() == res["sel"]
    compare_selection(mask_to_sets(inter["blk_mask"], cfg.n_kb), res["kept"], res["block_margin"],
                      f"{cfg.name} step masks")
    assert_close(inter["k_til"], res["k_til"], dkey(cfg), f"{cfg.name} step K~")
    assert_close(out, res["o"], dkey(cfg), f"{cfg.name} step O ({'fused' if fused else 'gathered'})")
    check_device_ok(wa)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "gathered"])
@pytest.mark.parametrize("cfg", [SMALL_BF16, SMALL_BF16_D64, SMALL_F32], ids=lambda c: c.name)
def test_hsa_step_per_head_projection(wa, cfg, fused):
    cfg = cfg.with_(e_per_head=True)
    inp = inputs(cfg)
    out, inter = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                                inp["e_v"], inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B,
                                fused_gather=fused, keep_intermediates=True)
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    assert_close(inter["k_til"], res["k_til"], dkey(cfg), f"{cfg.name} step per-head K~")
    assert_close(out, res["o"], dkey(cfg), f"{cfg.name} step O (per-head E, {'fused' if fused else 'gathered'})")
    check_device_ok(wa)


def sparse_blocks(cfg):
    """Key blocks of the sparse branch: the history, plus the chunk's own with intra keys."""
    return -(-(cfg.L + (cfg.Nq if cfg.intra else 0)) // cfg.B)


def expanded_kept(res, B):
    """The oracle's kept blocks at B-token granularity (what the step's mask holds)."""
    kb = res["key_bounds"]
    return [[O.expand_blocks(row, kb, B) for row in kh] for kh in res["kept"]]


def _full_size_step(wa, cfg, samples, gen_device="cuda", B_inter=0):
    inp = W.make_inputs(cfg, device="cuda", gen_device=gen_device)
    e_cur = inp.get("e_cur")
    step = wa.HSAStep(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"], inp["e_v"],
                      inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B, e_cur=e_cur,
                      e_chunks=inp.get("e_chunks"), fused_gather=True, keep_intermediates=True,
                      k_cur=inp.get("k_cur"), v_cur=inp.get("v_cur"), B_inter=B_inter)
    out = step()
    torch.cuda.synchronize()
    res = O.hsa_step(inp, cfg.B, cfg.K_p, rows_of_blocks=samples, B_inter=B_inter or None)
    if "chunk" in res:
        assert int(step.inter["chunk"].item()) == res["chunk"]
    np.testing.assert_allclose(to64(step.inter["alpha"]), res["alpha"], rtol=1e-9, atol=1e-13)
    if res["page_margin"] >= MARGIN_F64:
        assert step.inter["sel"].cpu().tolist() == res["sel"]
    n_kb = sparse_blocks(cfg)
    compare_selection(mask_to_sets(step.inter["blk_mask"], n_kb), expanded_kept(res, cfg.B),
                      res["block_margin"], f"{cfg.name} masks")
    print(f"[info] {cfg.name} kept fraction per head: "
          f"{np.round(kept_fraction(res['kept'], len(res['key_bounds'])), 3)}")
    assert_close(step.inter["k_til"], res["k_til"], "bf16", f"{cfg.name} K~")
    assert_close(step.inter["v_til"], res["v_til"], "bf16", f"{cfg.name} V~")
    for (h, i), blk in res["blocks"].items():
        r0, r1 = i * cfg.B, min(cfg.Nq, (i + 1) * cfg.B)
        assert_close(out[r0:r1, h], blk["o"], "bf16", f"{cfg.name} O[h={h}, block {i}]")
    check_device_ok(wa)


def test_full_size_layer_step(wa):
    cfg = W.C1
    n_qb = cfg.n_qb
    samples = [(0, 0), (11, n_qb - 1), (5, 37), (3, n_qb - 2), (8, 12), (11, 0)]
    _full_size_step(wa, cfg, samples)


def test_full_size_layer_step_intra_keys(wa):
    """C1 with the current chunk's own K/V in the sparse branch (780 + 74 key blocks,
    the last one 8 rows)."""
    cfg = W.C1.with_(name="c1_intra", intra=True)
    samples = [(0, 0), (11, cfg.n_qb - 1), (4, 30), (9, 60)]
    _full_size_step(wa, cfg, samples)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "gathered"])
@pytest.mark.parametrize("cfg", [SMALL_BF16, SMALL_BF16_D64, SMALL_F32], ids=lambda c: c.name)
def test_hsa_step_intra_keys_small(wa, cfg, fused):
    cfg = cfg.with_(intra=True)
    inp = inputs(cfg)
    out, inter = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                                inp["e_v"], inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B,
                                fused_gather=fused, keep_intermediates=True, k_cur=inp["k_cur"],
                                v_cur=inp["v_cur"])
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    n_kb = sparse_blocks(cfg)
    assert inter["blk_mask"].shape[-1] == -(-n_kb // 32)
    compare_selection(mask_to_sets(inter["blk_mask"], n_kb), res["kept"], res["block_margin"],
                      f"{cfg.name} intra masks")
    chunk_kept = sum(1 for h in res["kept"] for row in h for j in row if j >= cfg.L // cfg.B)
    assert chunk_kept > 0, "no chunk block kept: the case would not test the second segment"
    assert_close(out, res["o"], dkey(cfg), f"{cfg.name} step O with intra keys ({'fused' if fused else 'gathered'})")
    check_device_ok(wa)


def test_full_size_narrow_projection_step(wa):
    """Three heads of d=64 (H*d = 192, one 64-column projection tile) and r = 128 at the
    one-layer page shapes: the smallest projection configuration, whose pipeline leaves
    room on an SM for block-selection CTAs running beside it on the other stream."""
    cfg = W.C1.with_(name="c1_narrow_proj", H=3, d=64, r=128, seed=43)
    samples = [(0, 0), (2, cfg.n_qb - 1), (1, 36)]
    _full_size_step(wa, cfg, samples)


def test_full_size_layer_step_inter_intra_granularity(wa):
    """C1 with the chunk's own keys, history blocks of 128 tokens (390 of them, some
    spanning two pages) and chunk blocks of 64 (74, the last one 8 rows)."""
    cfg = W.C1.with_(name="c1_inter128", intra=True)
    samples = [(0, 0), (11, cfg.n_qb - 1), (6, 33)]
    _full_size_step(wa, cfg, samples, B_inter=128)


MIXED_SMALL = [SMALL_BF16.with_(name="mixed_bf16"),
               W.HSAConfig("mixed_f32_odd", H=2, d=64, T_p=192, n_c=4, Nq=150, K_p=3, B=64, r=48,
                           dtype="f32", seed=15, recipe="offset"),
               SMALL_BF16_D64.with_(name="mixed_bf16_d64_odd", T_p=576, K_p=3)]


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "gathered"])
@pytest.mark.parametrize("intra", [True, False], ids=["intra", "history"])
@pytest.mark.parametrize("cfg", MIXED_SMALL, ids=lambda c: c.name)
def test_hsa_step_inter_granularity_small(wa, cfg, intra, fused):
    """History blocks of 2B = 128 tokens (an odd number of 64-token blocks leaves a
    64-token last history block), with or without the chunk's own keys in blocks of 64."""
    cfg = cfg.with_(intra=intra)
    inp = inputs(cfg)
    out, inter = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                                inp["e_v"], inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B,
                                fused_gather=fused, keep_intermediates=True, k_cur=inp.get("k_cur"),
                                v_cur=inp.get("v_cur"), B_inter=128)
    res = O.hsa_step(inp, cfg.B, cfg.K_p, B_inter=128)
    n_kb = sparse_blocks(cfg)
    compare_selection(mask_to_sets(inter["blk_mask"], n_kb), expanded_kept(res, cfg.B),
                      res["block_margin"], f"{cfg.name} masks (B_inter 128)")
    assert_close(out, res["o"], dkey(cfg), f"{cfg.name} step O (B_inter 128, {'intra' if intra else 'history'})")
    check_device_ok(wa)


def test_full_size_layer_step_per_head_projection(wa):
    """C1 with one E_K / E_V pair per head (12 x 49,920 x 256 each)."""
    cfg = W.C1.with_(name="c1_e_per_head", e_per_head=True)
    samples = [(0, 0), (11, cfg.n_qb - 1), (7, 21)]
    _full_size_step(wa, cfg, samples)


def test_full_size_stress_step(wa):
    cfg = W.C2
    samples = [(0, 0), (4, cfg.n_qb - 1), (7, 20), (11, 50)]
    _full_size_step(wa, cfg, samples)


# ---------------------------------------------------------------- page pool
def test_pool_index_and_append(wa):
    cfg = SMALL_BF16
    inp = inputs(cfg)
    P_, T_p = cfg.n_pool_pages, cfg.T_p
    pages = torch.arange(P_, dtype=torch.int32, device="cuda")
    idx = wa.wa_pool_index(inp["k_pool"], pages, cfg.B)
    for p in range(P_):
        ref = O.block_means(inp["k_pool"][p], cfg.B) * cfg.B
        np.testing.assert_allclose(to64(idx[p]), ref, rtol=1e-12, atol=1e-12)
    # append 700 rows across the boundary of pages 2 and 3
    g = torch.Generator(device="cuda").manual_seed(9)
    n, off = 700, 2 * T_p + 900
    k_new = torch.randn((n, cfg.H, cfg.d), generator=g, device="cuda").to(torch.bfloat16)
    v_new = torch.randn((n, cfg.H, cfg.d), generator=g, device="cuda").to(torch.bfloat16)
    k_before = inp["k_pool"].clone()
    wa.wa_pool_append(inp["k_pool"], inp["v_pool"], k_new, v_new, off, page_index=idx, B=cfg.B)
    torch.cuda.synchronize()
    flat_k = inp["k_pool"].view(P_ * T_p, cfg.H, cfg.d)
    flat_v = inp["v_pool"].view(P_ * T_p, cfg.H, cfg.d)
    assert torch.equal(flat_k[off:off + n], k_new) and torch.equal(flat_v[off:off + n], v_new)
    untouched = torch.ones(P_ * T_p, dtype=torch.bool)
    untouched[off:off + n] = False
    assert torch.equal(flat_k[untouched.cuda()], k_before.view(P_ * T_p, cfg.H, cfg.d)[untouched.cuda()])
    for p in (2, 3):
        ref = O.block_means(inp["k_pool"][p], cfg.B) * cfg.B
        np.testing.assert_allclose(to64(idx[p]), ref, rtol=1e-12, atol=1e-12)
    check_device_ok(wa)


@pytest.mark.parametrize("cfg", [SMALL_BF16, SMALL_BF16_D64], ids=lambda c: c.name)
def test_hsa_step_with_page_index(wa, cfg):
    inp = inputs(cfg)
    pages = torch.arange(cfg.n_pool_pages, dtype=torch.int32, device="cuda")
    idx = wa.wa_pool_index(inp["k_pool"], pages, cfg.B)
    out, inter = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                                inp["e_v"], inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B,
                                keep_intermediates=True, page_index=idx)
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    np.testing.assert_allclose(to64(inter["alpha"]), res["alpha"], rtol=1e-9, atol=1e-13)
    if res["page_margin"] >= MARGIN_F64:
        assert inter["sel"].cpu().tolist() == res["sel"]
    compare_selection(mask_to_sets(inter["blk_mask"], cfg.n_kb), res["kept"], res["block_margin"],
                      f"{cfg.name} masks (page index)")
    assert_close(out, res["o"], "bf16", f"{cfg.name} step O (page index)")
    check_device_ok(wa)


def test_full_size_long_history_step(wa):
    """120-page pool (1.5 M tokens, 9.2 GB of K+V); prompt-level retrieval picks the chunk."""
    cfg = W.C3
    samples = [(0, 0), (11, cfg.n_qb - 1), (6, 40)]
    _full_size_step(wa, cfg, samples)


def test_denoise_stack_procedure(wa):
    """The full denoise-stack procedure at one-layer shapes: steps with fresh queries,
    new chunks' KV appended to the pool between chunks with the page index kept
    current, checked against the oracle on the first and last steps."""
    cfg = W.C1.with_(name="c4_layer", n_chunks=2, seed=41)   # 16-page pool: 8 history + 8 for appends
    inp = W.make_inputs(cfg, device="cuda", gen_device="cuda")
    P_ = cfg.n_pool_pages
    hist = inp["chunk_pages"][0:1]                            # the candidate chunk stays the history
    idx = wa.wa_pool_index(inp["k_pool"], torch.arange(P_, dtype=torch.int32, device="cuda"), cfg.B)
    g = torch.Generator(device="cuda").manual_seed(77)
    fill = cfg.n_c * cfg.T_p
    n_chunks, n_steps = 3, 2
    checked = []
    for chunk in range(n_chunks):
        for s in range(n_steps):
            q = (torch.randn((cfg.Nq, cfg.H, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(torch.bfloat16)
            gate = torch.randn((cfg.Nq, cfg.H), generator=g, device="cuda")
            out, inter = wa.wa_hsa_step(q, inp["k_pool"], inp["v_pool"], hist, inp["e_k"], inp["e_v"],
                                        inp["tau"].cuda(), gate, cfg.K_p, cfg.B, keep_intermediates=True,
                                        page_index=idx)
            if (chunk, s) in ((0, 0), (n_chunks - 1, n_steps - 1)):
                checked.append((q.clone(), gate.clone(), out.clone(), inter["sel"].cpu().tolist()))
        # the chunk's own KV (3 frames) goes into the pool after its denoising steps
        k_new = (torch.randn((cfg.Nq, cfg.H, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(torch.bfloat16)
        v_new = (torch.randn((cfg.Nq, cfg.H, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(torch.bfloat16)
        wa.wa_pool_append(inp["k_pool"], inp["v_pool"], k_new, v_new, fill, page_index=idx, B=cfg.B)
        fill += cfg.Nq
    torch.cuda.synchronize()
    # the index of the appended pages matches the keys now in the pool
    for p in (cfg.n_c, cfg.n_c + 1):
        ref = O.block_means(inp["k_pool"][p], cfg.B) * cfg.B
        np.testing.assert_allclose(to64(idx[p]), ref, rtol=1e-12, atol=1e-12)
    for k, (q, gate, out, sel) in enumerate(checked):
        step_inp = dict(inp, q=q, gate=gate, cand=hist[0].cpu())
        step_inp.pop("e_cur", None)
        res = O.hsa_step(step_inp, cfg.B, cfg.K_p, rows_of_blocks=[(0, 0), (7, cfg.n_qb - 1)])
        if res["page_margin"] >= MARGIN_F64:
            assert sel == res["sel"]
        for (h, i), blk in res["blocks"].items():
            r0, r1 = i * cfg.B, min(cfg.Nq, (i + 1) * cfg.B)
            assert_close(out[r0:r1, h], blk["o"], "bf16", f"denoise stack step {k}: O[h={h}, block {i}]")
    check_device_ok(wa)
