"""The page tier on the GPU: slots always hold the pages the tier says they hold,
dirty pages survive eviction through the host copy, prefetched pages arrive, and a
decode step over the tier's slot pool gives the same bits as over the full pool."""
import random

import pytest
import torch

from linear_attention_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wa():
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa as mod
    return mod


def _pages(n_pages, shape, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((n_pages,) + shape, generator=g).to(torch.bfloat16).pin_memory()
    v = torch.randn((n_pages,) + shape, generator=g).to(torch.bfloat16).pin_memory()
    return k, v


def _check_slots(t, host_k, host_v, slot_k, slot_v, pages, slots):
    torch.cuda.current_stream().synchronize()
    for p, s in zip(pages, slots):
        assert t.slot_of(p) == s
        assert torch.equal(slot_k[s].cpu(), host_k[p]), f"K of page {p} in slot {s}"
        assert torch.equal(slot_v[s].cpu(), host_v[p]), f"V of page {p} in slot {s}"


def test_tier_random_access_prefetch_and_writeback(wa):
    n_pages, n_slots, shape = 12, 4, (128, 2, 64)
    host_k, host_v = _pages(n_pages, shape, 1)
    ref_k, ref_v = host_k.clone(), host_v.clone()          # what each page should hold
    slot_k = torch.empty((n_slots,) + shape, dtype=torch.bfloat16, device="cuda")
    slot_v = torch.empty_like(slot_k)
    t = wa.Tier(host_k, host_v, slot_k, slot_v)
    rnd = random.Random(5)
    for it in range(60):
        req = rnd.sample(range(n_pages), rnd.randint(1, n_slots))
        slots = t.ensure(req)
        torch.cuda.current_stream().synchronize()
        for p, s in zip(req, slots):
            assert torch.equal(slot_k[s].cpu(), ref_k[p]), f"iteration {it}: K of page {p}"
            assert torch.equal(slot_v[s].cpu(), ref_v[p]), f"iteration {it}: V of page {p}"
        if it % 7 == 3:
            # the device writes one page (an appended chunk), then marks it dirty
            p, s = req[0], slots[0]
            slot_k[s] += 1.0
            slot_v[s] -= 1.0
            t.mark_dirty(p)
            torch.cuda.current_stream().synchronize()
            ref_k[p] = slot_k[s].cpu()
            ref_v[p] = slot_v[s].cpu()
        t.release()
        if it % 5 == 1:
            t.prefetch(rnd.sample(range(n_pages), 2))
    t.flush()
    torch.cuda.synchronize()
    for p in range(n_pages):
        assert torch.equal(host_k[p], ref_k[p]) and torch.equal(host_v[p], ref_v[p]), f"host page {p}"
    st = t.stats()
    assert st["misses"] > 0 and st["evictions"] > 0 and st["writebacks"] > 0
    assert st["bytes_h2d"] > 0 and st["bytes_d2h"] > 0
    t.close()


def test_step_over_the_slot_pool_matches_the_full_pool(wa):
    cfg = W.HSAConfig("tier_small", H=2, d=128, T_p=1280, n_c=6, Nq=520, K_p=3, B=64, r=128,
                      dtype="bf16", seed=31, recipe="offset", n_chunks=2)
    inp = W.make_inputs(cfg, device="cuda")
    P_ = cfg.n_pool_pages                                        # 12 pages, two chunks
    host_k = inp["k_pool"].cpu().pin_memory()
    host_v = inp["v_pool"].cpu().pin_memory()
    n_slots = 8
    slot_k = torch.empty((n_slots,) + tuple(inp["k_pool"].shape[1:]), dtype=torch.bfloat16, device="cuda")
    slot_v = torch.empty_like(slot_k)
    t = wa.Tier(host_k, host_v, slot_k, slot_v)
    tau = inp["tau"].cuda()
    for chunk in (1, 0, 1):
        pages = inp["chunk_pages"][chunk].cpu().tolist()
        slots = t.ensure(pages)
        full = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"][chunk:chunk + 1],
                              inp["e_k"], inp["e_v"], tau, inp["gate"], cfg.K_p, cfg.B)
        via = wa.wa_hsa_step(inp["q"], slot_k, slot_v,
                             torch.tensor([slots], dtype=torch.int32, device="cuda"),
                             inp["e_k"], inp["e_v"], tau, inp["gate"], cfg.K_p, cfg.B)
        t.release()
        torch.cuda.synchronize()
        assert torch.equal(full, via), f"chunk {chunk}: step over the slot pool differs"
    assert wa.wa_device_error() == 0
    t.close()


def test_pipeline_over_host_buffers_matches_direct_steps(wa):
    """Steps submitted through the host-buffer pipeline (double-buffered device sets,
    overlapped copies) give the same bits as direct steps on the same inputs."""
    cfg = W.HSAConfig("pipe_small", H=2, d=128, T_p=1280, n_c=6, Nq=520, K_p=3, B=64, r=128,
                      dtype="bf16", seed=33, recipe="offset")
    inp = W.make_inputs(cfg, device="cuda")
    tau = inp["tau"].cuda()
    step = wa.HSAStep(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"], inp["e_v"],
                      tau, inp["gate"], cfg.K_p, cfg.B)
    g = torch.Generator().manual_seed(4)
    n = 5
    qs = [(torch.randn(inp["q"].shape, generator=g) / cfg.d ** 0.5).to(torch.bfloat16).pin_memory()
          for _ in range(n)]
    gs = [torch.randn(inp["gate"].shape, generator=g).pin_memory() for _ in range(n)]
    outs = [torch.empty(inp["q"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(n)]
    pipe = wa.HSAPipeline(step, inp["q"], inp["gate"])
    pipe.begin()
    for k in range(n):
        pipe.submit(qs[k], gs[k], outs[k])
    pipe.end()
    pipe.sync()
    pipe.close()
    for k in range(n):
        ref = wa.wa_hsa_step(qs[k].cuda(), inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                             inp["e_v"], tau, gs[k].cuda(), cfg.K_p, cfg.B)
        assert torch.equal(outs[k], ref.cpu()), f"pipelined step {k} differs"
    assert wa.wa_device_error() == 0
