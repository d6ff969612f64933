"""The full denoise stack (30 layers x 4 denoising steps x 20 chunks of 3 frames at
the one-layer shapes), run through the library as a serving loop would, with sampled
steps checked against the float64 oracle.

Each layer owns a 16-page pool (the 8-page history chunk and room for the appended
chunks), its E_K / E_V and tau, and a float64 page index that every step reads.  After
each chunk's four denoising steps, that chunk's K/V (4680 new tokens per layer, drawn
per (layer, chunk)) is appended to every layer's pool and the index refreshed.  The
queries and gate logits of every (layer, step, chunk) are drawn afresh from a seed of
their own, so the sampled steps -- layers {0, 29} x steps {0, 3} x chunks {0, 19} --
can be redone by the oracle on the same inputs.  The history chunk stays the
candidate chunk (20 chunks x 3 frames = 60 frames complete no new 8-page chunk), so
each sampled step is checked against the oracle run on the pool as it stands then;
at the end the appended pages must hold exactly the appended K/V, the history pages
must be untouched, and the page index must equal the block sums of the final pool."""
import numpy as np
import pytest
import torch

from linear_attention_paged_b200 import workloads as W
from oracle import hsa_oracle as O
from tests.helpers import MARGIN_F64, assert_close, compare_selection, mask_to_sets, to64

pytestmark = pytest.mark.gpu

N_LAYERS, N_STEPS, N_CHUNKS = 30, 4, 20
SAMPLED = {(l, s, c) for l in (0, N_LAYERS - 1) for s in (0, N_STEPS - 1) for c in (0, N_CHUNKS - 1)}


@pytest.fixture(scope="module")
def wa():
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa as _wa
    return _wa


def _qg(cfg, layer, step, chunk):
    g = torch.Generator(device="cuda").manual_seed(1_000_003 * layer + 10_007 * chunk + 101 * step + 17)
    q = (torch.randn((cfg.Nq, cfg.H, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(torch.bfloat16)
    gate = torch.randn((cfg.Nq, cfg.H), generator=g, device="cuda")
    return q, gate


def _new_kv(cfg, layer, chunk):
    g = torch.Generator(device="cuda").manual_seed(7_000_001 * layer + 31 * chunk + 5)
    k = (torch.randn((cfg.Nq, cfg.H, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(torch.bfloat16)
    v = (torch.randn((cfg.Nq, cfg.H, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(torch.bfloat16)
    return k, v


def test_full_denoise_stack_sampled_against_oracle(wa):
    base = W.C1.with_(name="c4_layer", n_chunks=2)          # 16-page pool per layer
    P_, T_p = base.n_pool_pages, base.T_p
    layers = []
    for l in range(N_LAYERS):
        cfg = base.with_(seed=4000 + l)
        inp = W.make_inputs(cfg, device="cuda", gen_device="cuda")
        hist = inp["chunk_pages"][0:1].contiguous()
        idx = wa.wa_pool_index(inp["k_pool"], torch.arange(P_, dtype=torch.int32, device="cuda"), cfg.B)
        step = wa.HSAStep(inp["q"], inp["k_pool"], inp["v_pool"], hist, inp["e_k"], inp["e_v"],
                          inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B, keep_intermediates=True,
                          page_index=idx)
        keep = None
        if l in (0, N_LAYERS - 1):
            keep = (inp["k_pool"][:cfg.n_c].clone(), inp["v_pool"][:cfg.n_c].clone())
        layers.append(dict(cfg=cfg, inp=inp, idx=idx, step=step, hist=hist, keep=keep))
    import ctypes
    fill = base.n_c * T_p
    seen = {}
    for c in range(N_CHUNKS):
        for s in range(N_STEPS):
            for l, L_ in enumerate(layers):
                q, gate = _qg(L_["cfg"], l, s, c)
                a = L_["step"].args
                a.q = ctypes.c_void_p(q.data_ptr())
                a.gate = ctypes.c_void_p(gate.data_ptr())
                out = L_["step"]()
                if (l, s, c) in SAMPLED:
                    seen[(l, s, c)] = dict(q=q, gate=gate, out=out.clone(),
                                           sel=L_["step"].inter["sel"].clone(),
                                           mask=L_["step"].inter["blk_mask"].clone())
                else:
                    del q, gate
        for l, L_ in enumerate(layers):
            k_new, v_new = _new_kv(L_["cfg"], l, c)
            wa.wa_pool_append(L_["inp"]["k_pool"], L_["inp"]["v_pool"], k_new, v_new, fill,
                              page_index=L_["idx"], B=base.B)
        fill += base.Nq
    torch.cuda.synchronize()
    assert wa.wa_device_error() == 0
    assert len(seen) == len(SAMPLED)

    for l in (0, N_LAYERS - 1):
        L_ = layers[l]
        cfg, inp = L_["cfg"], L_["inp"]
        # the history pages are untouched; the appended region holds exactly the appended K/V
        assert torch.equal(inp["k_pool"][:cfg.n_c], L_["keep"][0])
        assert torch.equal(inp["v_pool"][:cfg.n_c], L_["keep"][1])
        flat_k = inp["k_pool"].view(P_ * T_p, cfg.H, cfg.d)
        flat_v = inp["v_pool"].view(P_ * T_p, cfg.H, cfg.d)
        off = cfg.n_c * T_p
        for c in range(N_CHUNKS):
            k_new, v_new = _new_kv(cfg, l, c)
            assert torch.equal(flat_k[off + c * cfg.Nq: off + (c + 1) * cfg.Nq], k_new)
            assert torch.equal(flat_v[off + c * cfg.Nq: off + (c + 1) * cfg.Nq], v_new)
        # the page index equals the block sums of the final pool (appended pages included)
        for p in (0, cfg.n_c - 1, cfg.n_c, cfg.n_c + 6, cfg.n_c + 7):
            ref = O.block_means(inp["k_pool"][p], cfg.B) * cfg.B
            np.testing.assert_allclose(to64(L_["idx"][p]), ref, rtol=1e-12, atol=1e-12)
        # the sampled steps against the oracle, on the pool as it stood (the candidate
        # pages never change, so it is the pool's history chunk)
        for (ll, s, c), got in sorted(seen.items()):
            if ll != l:
                continue
            step_inp = {k: v for k, v in inp.items() if k not in ("e_cur", "e_chunks")}
            step_inp.update(q=got["q"], gate=got["gate"], cand=L_["hist"][0].cpu())
            n_qb = cfg.n_qb
            res = O.hsa_step(step_inp, cfg.B, cfg.K_p, rows_of_blocks=[(0, 0), (cfg.H - 1, n_qb - 1), (5, 37)])
            if res["page_margin"] >= MARGIN_F64:
                assert got["sel"].cpu().tolist() == res["sel"], f"layer {l} step {s} chunk {c}: pages"
            compare_selection(mask_to_sets(got["mask"], cfg.n_kb), res["kept"], res["block_margin"],
                              f"stack layer {l} step {s} chunk {c} masks")
            for (h, i), blk in res["blocks"].items():
                r0, r1 = i * cfg.B, min(cfg.Nq, (i + 1) * cfg.B)
                assert_close(got["out"][r0:r1, h], blk["o"], "bf16",
                             f"stack layer {l} step {s} chunk {c}: O[h={h}, block {i}]")
