#!/usr/bin/env python
"""Benchmark of the HSA decode step (one chunk-layer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one call of wa_hsa_step -- page scoring + top-4 pages, page-table
addressing (no gather copy), head-adaptive block selection, the Linformer
projection, the linear and block-sparse attention branches and the sigmoid gate --
on the one-layer bf16 workload: 12 heads, d=128, 8-frame pages of 1560-token
frames, a candidate chunk of 8 pages resident in HBM, a 3-frame query chunk (4680
tokens), top-4 pages -> 49,920 keys, B=64, r=256.  Inputs are seeded synthetic
tensors (see linear_attention_paged_b200/workloads.py) already resident in HBM;
the pool read per step (>600 MB) is larger than the 126 MB L2, so no flush is
needed between steps.

Metric: attention frames/s = frames per chunk (3) / (120 chunk-layers per chunk:
30 layers x 4 denoising steps) / ms per chunk-layer, summed over ranks (each rank
runs its own layer: weak scaling, no data-path collective).

The JSON line also carries: per-stage ms (CUDA events recorded by the library on
the launching stream), the roofline of the dominant kernel (the block-sparse
attention, counting selected-block FLOPs only), the HBM fraction of the page
retrieval stage and of its block-sum pass alone, an end-to-end number through the
public API with pinned host buffers (H2D of the step's q and gate, D2H of its
output, inside the timed region), the clock record, the same step with two gates,
over a 120-page pool (long history) and on the head-adaptive stress inputs, the
page tier's host-to-device rate, and the fp64 oracle timed on the host cores on a
bounded sample of the same workload (rank 0, N=1 only).

--impl reference times that oracle alone (the reference arm: the method is
described only in prose, so there is no upstream implementation to install).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from linear_attention_paged_b200 import replicas  # noqa: E402

METRIC = "HSA ms/chunk-layer & attention frames/s; % of BF16 tensor / HBM roofline"
# DRAM bytes per launch of the sparse-branch attention kernel per head, from one ncu
# capture of the 6-head C1 launch with the work items longest first over all heads
# (330.7 MB read + 22.6 MB written) / 6; set to None when the kernel or its item order
# changes
ATTN_DRAM_BYTES_PER_HEAD = (330707456 + 22639360) / 6
FRAMES_PER_CHUNK = 3
CHUNK_LAYERS_PER_CHUNK = 30 * 4
# stage -> (start event, end event) of the events wa_hsa_step records; the
# projection and the linear branch run on a side stream concurrently with block
# selection and the work list, so their stages overlap those
STAGES = {"page_retrieval": (0, 1), "gather": (1, 2), "block_select": (2, 3),
          "projection": (2, 4), "linear_branch": (4, 5), "work_list_and_join": (3, 6),
          "sparse_branch_gate": (6, 7)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def workload_desc(cfg, b_inter=0):
    intra = (f"; sparse branch also over the chunk's own {cfg.Nq} keys (intra-chunk keys)"
             if cfg.intra else "")
    if b_inter and b_inter != cfg.B:
        intra += f"; history selected in blocks of {b_inter} tokens (inter-chunk granularity)"
    return (f"{cfg.name}: one HSA decode step (chunk-layer), H={cfg.H}, d={cfg.d}, T_p={cfg.T_p} "
            f"(8 frames x 1560 tokens), n_c={cfg.n_c} candidate pages, Nq={cfg.Nq}, K_p={cfg.K_p} "
            f"-> L={cfg.L}, B={cfg.B}, r={cfg.r}, tau_h=0.80+0.15h/11, bf16{intra}")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        sel = []
        try:
            props = torch.cuda.get_device_properties(device_index)
            bus = getattr(props, "pci_bus_id", None)
            dom = getattr(props, "pci_domain_id", None)
            dev = getattr(props, "pci_device_id", None)
            if bus is not None and dom is not None and dev is not None:
                sel = ["-i", f"{dom:08X}:{bus:02X}:{dev:02X}.0"]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "100"] + sel

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle
def oracle_sample(inp, cfg, n_blocks=2, head_frac=1, l_slices=8, seed=0):
    """Time the fp64 oracle on a bounded sample of one step and scale each part to
    the full step: page scores in full, block selection for one head (x H), the
    projection on 1/l_slices of L (x l_slices), both attention branches for
    n_blocks sampled (head, query block) pairs (x H*n_qb).  Returns seconds per
    full step (estimate) and a description."""
    from oracle import hsa_oracle as O
    rng = np.random.default_rng(seed)
    t = {}
    t0 = time.perf_counter()
    cand = [int(x) for x in inp["cand"]]
    # page scores over 1/l_slices of every candidate page's rows: same cost per row
    Ts = cfg.T_p // l_slices
    k_cand = np.stack([O.f64(inp["k_pool"][p][:Ts]) for p in cand])
    alpha = O.page_scores(inp["q"], k_cand)
    sel = [cand[j] for j in O.select_pages(alpha, cfg.K_p)]
    del k_cand
    t["page_retrieval"] = (time.perf_counter() - t0) * l_slices
    t0 = time.perf_counter()
    k_act = O.gather_pages(inp["k_pool"], sel)
    v_act = O.gather_pages(inp["v_pool"], sel)
    t["gather"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    h = int(rng.integers(cfg.H))
    s = O.block_scores(inp["q"][:, h:h + 1], k_act[:, h:h + 1], cfg.B)
    kept, _ = O.block_select(None, None, O.f64(inp["tau"])[h:h + 1], cfg.B, scores=s)
    t["block_select"] = (time.perf_counter() - t0) * cfg.H
    t0 = time.perf_counter()
    Ls = cfg.L // l_slices
    # a partial sum over L/l_slices rows: same cost per row, same output shape
    kt, vt = O.linear_project(k_act[:Ls], v_act[:Ls], inp["e_k"][:Ls], inp["e_v"][:Ls])
    t["projection"] = (time.perf_counter() - t0) * l_slices
    t0 = time.perf_counter()
    for _ in range(n_blocks):
        i = int(rng.integers(cfg.n_qb))
        O.sparse_attention_block(inp["q"], k_act, v_act, h, i, kept[0][i], cfg.B)
        r0, r1 = i * cfg.B, min(cfg.Nq, (i + 1) * cfg.B)
        O.linear_attention(O.f64(inp["q"][r0:r1, h:h + 1]), kt[:, h:h + 1], vt[:, h:h + 1])
    t["attention"] = (time.perf_counter() - t0) / n_blocks * cfg.H * cfg.n_qb
    total = sum(t.values())
    desc = (f"fp64 numpy oracle on a bounded sample of one step: page scores on T_p/{l_slices} rows "
            f"of each candidate page (x{l_slices}), block "
            f"selection for 1 of {cfg.H} heads (x{cfg.H}), projection on L/{l_slices} (x{l_slices}), "
            f"both branches for {n_blocks} of {cfg.H * cfg.n_qb} (head, query block) pairs "
            f"(x{cfg.H * cfg.n_qb // n_blocks}); per-step time extrapolated")
    return total, desc, t


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def frames_per_s(ms_per_chunk_layer, n=1):
    """Whole-job frames/s of n replicas whose slowest takes ms_per_chunk_layer per step."""
    return replicas.job_throughput(FRAMES_PER_CHUNK / CHUNK_LAYERS_PER_CHUNK, n, ms_per_chunk_layer / 1000.0)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    from linear_attention_paged_b200 import workloads as W
    cfg = W.C1
    inp = W.make_inputs(cfg, device="cpu")
    for _ in range(args.warmup):
        oracle_sample(inp, cfg, n_blocks=1, seed=0)
    ts = []
    desc = ""
    for k in range(args.steps):
        tot, desc, _ = oracle_sample(inp, cfg, n_blocks=1, seed=k + 1)
        ts.append(tot)
    sec = float(np.mean(ts))
    ms = sec * 1000.0
    v = frames_per_s(ms)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "frames/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "device": "host cpu"},
            "cpu_baseline": {"value": v, "unit": "frames/s", "cores": cores(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": "frames/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def selected_flops(mask, cfg):
    """4 * b_q(i) * b_k(j) * d summed over kept (head, query block, key block)."""
    m = mask.cpu().numpy().astype(np.uint32)
    H, n_qb, W_ = m.shape
    bq = np.array([min(cfg.Nq, (i + 1) * cfg.B) - i * cfg.B for i in range(n_qb)], dtype=np.float64)
    # key blocks: the history, then (intra-chunk keys) the chunk's own Nq rows
    bk = [min(cfg.L, (j + 1) * cfg.B) - j * cfg.B for j in range(cfg.n_kb)]
    if cfg.intra:
        bk += [min(cfg.Nq, (j + 1) * cfg.B) - j * cfg.B for j in range(-(-cfg.Nq // cfg.B))]
    bk = np.array(bk, dtype=np.float64)
    n_kb = len(bk)
    total = 0.0
    kept = 0
    for h in range(H):
        for i in range(n_qb):
            bits = np.unpackbits(m[h, i].view(np.uint8), bitorder="little")[:n_kb].astype(bool)
            kept += int(bits.sum())
            total += 4.0 * bq[i] * float(bk[bits].sum()) * cfg.d
    return total, kept / float(H * n_qb * n_kb)


def run_ours(args, rank, world, local_rank):
    from linear_attention_paged_b200 import build as wb
    if rank == 0:
        wb.build()
    replicas.barrier(world)
    from linear_attention_paged_b200 import wa, workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    base = W.C1 if args.heads is None else W.C1.with_(name=f"c1_layer_bf16_h{args.heads}", H=args.heads)
    if args.intra:
        base = base.with_(name=base.name + "_intra", intra=True)
    if args.b_inter:
        base = base.with_(name=base.name + f"_inter{args.b_inter}")
    cfg = base.with_(seed=replicas.rank_seed(base.seed, rank))   # each rank: its own layer
    inp = W.make_inputs(cfg, device="cuda", gen_device="cuda")
    tau = inp["tau"].cuda()
    stream = torch.cuda.current_stream()

    step = wa.HSAStep(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"], inp["e_v"],
                      tau, inp["gate"], cfg.K_p, cfg.B, fused_gather=True, keep_intermediates=True,
                      k_cur=inp.get("k_cur"), v_cur=inp.get("v_cur"), B_inter=args.b_inter)
    step()
    torch.cuda.synchronize()
    flags = wa.wa_device_error()
    if flags:
        raise RuntimeError(f"device error flags 0x{flags:x}")
    flops, kept_frac = selected_flops(step.inter["blk_mask"], cfg)
    # per step: the block-sum pass over the queries and candidate pages, page scores
    # and top-k, block scores, block choice, pairing, work items, the sparse attention
    # and (when key lists are split, i.e. the tile pairs fill fewer than two waves of
    # one CTA per SM) the combine; projection, split reduction and linear branch
    n_pairs = cfg.H * ((cfg.n_qb + 1) // 2)
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    launches_per_step = (10 + (1 if n_pairs < 2 * n_sm else 0)
                         + (1 if cfg.intra else 0))   # + block sums of the chunk's keys

    n_ev = 8  # WA_STEP_EVENTS
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for row in ev:                 # torch creates the CUDA event on first record
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    ev_ptrs = [ctypes_void_array(e) for e in ev]
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    clk = ClockSampler(local_rank)
    clk.start()
    replicas.barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        step.args.stage_events = ev_ptrs[k][0]
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    replicas.barrier(world)
    clocks = clk.stop()
    step.args.stage_events = None
    elapsed = t_start.elapsed_time(t_end)
    elapsed_max = replicas.max_over_ranks(elapsed, world, dev)
    ms_step = elapsed_max / args.steps

    stage_ms = {}
    for name, (a0, a1) in STAGES.items():
        stage_ms[name] = float(np.mean([ev[k][a0].elapsed_time(ev[k][a1]) for k in range(args.steps)]))
    attn_ms = stage_ms["sparse_branch_gate"]
    peaks, peak_src = load_peaks()
    # the burst GEMM figure applies to a timed region of well under a few seconds
    # (clocks have not yet settled at the power cap); the sustained one to a
    # region of seconds or more
    timed_s = elapsed_max * 1e-3
    peak_key = "bf16_tflops_sustained" if timed_s >= 2.0 else "bf16_tflops"
    peak_t = float(peaks.get(peak_key, peaks["bf16_tflops"]))
    achieved_t = flops / (attn_ms * 1e-3) / 1e12
    page_bytes = (cfg.Nq * cfg.H * cfg.d + cfg.n_c * cfg.T_p * cfg.H * cfg.d) * 2
    hbm_achieved = page_bytes / (stage_ms["page_retrieval"] * 1e-3) / 1e9

    # end to end through the public API: pinned host q/gate in, output back to the host,
    # through the step pipeline (uploads of step k+1 and downloads of step k-1 overlap
    # step k; every step still moves its own inputs and output across PCIe)
    e2e_steps = 0 if args.no_e2e else max(3, min(args.steps, 50))
    q_host = inp["q"].cpu().pin_memory()
    g_host = inp["gate"].cpu().pin_memory()
    o_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    pipe = wa.HSAPipeline(step, inp["q"], inp["gate"], stream)
    for _ in range(2 if e2e_steps else 0):
        pipe.submit(q_host, g_host, o_host)
    pipe.sync()
    torch.cuda.synchronize()
    replicas.barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.begin()
    for _ in range(e2e_steps):
        pipe.submit(q_host, g_host, o_host)
    pipe.end()
    e1.record(stream)
    torch.cuda.synchronize()
    pipe.close()
    e2e_ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev) / max(e2e_steps, 1)
    h2d = q_host.numel() * q_host.element_size() + g_host.numel() * g_host.element_size()
    d2h = o_host.numel() * o_host.element_size()

    # S2 on its own: the gather of the selected pages that the fused step avoids
    # (non-fused path), K and V read once and written once
    sel = step.inter["sel"]
    ka = torch.empty((cfg.L, cfg.H, cfg.d), dtype=inp["k_pool"].dtype, device=dev)
    va = torch.empty_like(ka)
    for _ in range(3):
        wa.wa_gather_pages(inp["k_pool"], inp["v_pool"], sel, out=(ka, va))
    n_g = 20
    gs, ge = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gs.record(stream)
    for _ in range(n_g):
        wa.wa_gather_pages(inp["k_pool"], inp["v_pool"], sel, out=(ka, va))
    ge.record(stream)
    torch.cuda.synchronize()
    gather_ms = gs.elapsed_time(ge) / n_g
    gather_bytes = 2 * 2 * ka.numel() * ka.element_size()
    gather_gbs = gather_bytes / (gather_ms * 1e-3) / 1e9
    # S1's HBM pass on its own: the float64 block sums of the candidate pages (the same
    # kernel the step runs, here through the page-index entry point), K read once
    cand_pages = inp["chunk_pages"][0].to(torch.int32).contiguous()
    pidx = torch.zeros((inp["k_pool"].shape[0], cfg.T_p // cfg.B, cfg.H, cfg.d), dtype=torch.float64,
                       device=dev)
    for _ in range(3):
        wa.wa_pool_index(inp["k_pool"], cand_pages, cfg.B, page_index=pidx)
    bs_, be_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    bs_.record(stream)
    for _ in range(n_g):
        wa.wa_pool_index(inp["k_pool"], cand_pages, cfg.B, page_index=pidx)
    be_.record(stream)
    torch.cuda.synchronize()
    pass_ms = bs_.elapsed_time(be_) / n_g
    pass_bytes = cand_pages.numel() * cfg.T_p * cfg.H * cfg.d * inp["k_pool"].element_size()
    pass_gbs = pass_bytes / (pass_ms * 1e-3) / 1e9
    del pidx
    # cube-tile token order: the active keys (K_p pages) re-ordered page by page into
    # (8, 2, 4) cubes of an 8-frame 30 x 52 latent page, one row gather over L rows
    perm_ms = perm_gbs = perm_bytes = None
    if cfg.T_p == W.PAGE_FRAMES * 30 * 52:
        pp = wa.wa_cube_order(W.PAGE_FRAMES, 30, 52, 8, 2, 4).long()
        perm = torch.cat([pp + s_ * cfg.T_p for s_ in range(cfg.K_p)]).to(torch.int32).to(dev)
        kc = torch.empty_like(ka)
        for _ in range(3):
            wa.wa_permute_rows(ka, perm, out=kc)
        ps, pe = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ps.record(stream)
        for _ in range(n_g):
            wa.wa_permute_rows(ka, perm, out=kc)
        pe.record(stream)
        torch.cuda.synchronize()
        perm_ms = ps.elapsed_time(pe) / n_g
        perm_bytes = 2 * ka.numel() * ka.element_size() + perm.numel() * 4
        perm_gbs = perm_bytes / (perm_ms * 1e-3) / 1e9
        del kc
    del ka, va

    # two-gate fusion (O = G_lin * O_lin + G_sp * O_sp, gates from independent logits):
    # the same step with a second, seeded gate
    two_gate_ms = None
    if not cfg.intra and not args.b_inter:
        g_lin = torch.randn(inp["gate"].shape, generator=torch.Generator().manual_seed(cfg.seed + 6)).to(dev)
        step2 = wa.HSAStep(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                           inp["e_v"], tau, inp["gate"], cfg.K_p, cfg.B, fused_gather=True, gate_lin=g_lin)
        for _ in range(3):
            step2()
        ts_, te_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts_.record(stream)
        for _ in range(n_g):
            step2()
        te_.record(stream)
        torch.cuda.synchronize()
        two_gate_ms = ts_.elapsed_time(te_) / n_g
        del step2, g_lin

    # L1 <-> L2 page tier: the candidate pages in pinned host memory, K_p device slots;
    # each request brings in K_p pages that are not resident (host -> device copies)
    tier = tier_measure(inp, cfg, dev, stream)

    # long history (config 4 of the workloads): a 120-page pool, the candidate chunk
    # chosen by prompt embeddings, then the same step; its time against C1's shows
    # whether retrieval grows with the history
    c3 = c2 = None
    if not args.no_c3 and args.heads is None and not args.intra and not args.b_inter:
        c3 = config_measure(W.C3, dev, stream, n_g, peak_t)
        c3["workload"] = (f"{W.C3.name}: one-layer shapes over a pool of {W.C3.n_pool_pages} pages "
                          f"({c3['pool_gb']:.1f} GB of K and V); prompt embeddings of {W.C3.prompt_dim} "
                          f"pick the candidate chunk among {W.C3.n_chunks}")
        c2 = config_measure(W.C2, dev, stream, n_g, peak_t)
        c2["workload"] = (f"{W.C2.name}: one-layer shapes, Student-t values, 1-32 planted hot key "
                          f"blocks per head, tau_h ~ U[0.5, 0.99] (kept fractions from about 1 % to 100 %)")

    # the full denoise stack (spec config 5) on the same GPU, after the one-layer
    # figures: every rank runs its own stack
    c4 = None
    if not args.no_c4 and args.heads is None and not args.intra and not args.b_inter:
        c4 = c4_measure(args, rank, world, local_rank)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            inp_cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
            sec, desc, parts = oracle_sample(inp_cpu, cfg, n_blocks=2)
            cpu = {"value": frames_per_s(sec * 1000.0), "unit": "frames/s", "cores": cores(),
                   "kind": "oracle", "sample": desc, "ms_per_step": sec * 1000.0,
                   "parts_s": {k: round(v, 3) for k, v in parts.items()}}
        line = {
            "metric": METRIC, "value": frames_per_s(ms_step, world), "unit": "frames/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "ms_per_chunk_layer": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_desc(cfg, args.b_inter),
                       "l2": "no flush: each step reads >600 MB (candidate keys + selected K/V), "
                             "larger than the 126 MB L2",
                       "parallelism": f"replicas x{world} (one layer per rank, no collective)"},
            "roofline": {"bound": "tensor", "achieved": achieved_t, "peak": peak_t, "unit": "TFLOP/s",
                         "frac": achieved_t / peak_t,
                         "traffic": (ATTN_DRAM_BYTES_PER_HEAD * cfg.H
                                     if ATTN_DRAM_BYTES_PER_HEAD is not None and not cfg.intra else None),
                         "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one "
                                           "6-head launch of this kernel on the same workload, "
                                           "scaled by heads",
                         "kernel": "k_umma_attention (sparse branch + gate)",
                         "flops_per_launch": flops, "kept_fraction": kept_frac,
                         "peak_source": f"{peak_key} (timed region {timed_s:.2f} s), of {peak_src}",
                         "frac_of_sustained": achieved_t / float(peaks.get("bf16_tflops_sustained",
                                                                           peaks["bf16_tflops"]))},
            "hbm_page_scoring": {"achieved": hbm_achieved, "peak": float(peaks["hbm_gbs"]),
                                 "unit": "GB/s", "frac": hbm_achieved / float(peaks["hbm_gbs"]),
                                 "bytes_per_launch": page_bytes},
            "hbm_block_sum_pass": {"kernel": "k_block_sums over the candidate pages (S1's HBM pass, "
                                             "through wa_pool_index)", "achieved": pass_gbs,
                                   "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                                   "frac": pass_gbs / float(peaks["hbm_gbs"]),
                                   "bytes_per_launch": pass_bytes, "ms_per_launch": pass_ms},
            "hbm_gather": {"kernel": "k_gather (non-fused S2)", "achieved": gather_gbs,
                           "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                           "frac": gather_gbs / float(peaks["hbm_gbs"]), "bytes_per_launch": gather_bytes,
                           "ms_per_launch": gather_ms},
            "hbm_cube_permute": ({"kernel": "k_permute_rows (cube-tile token order of the active keys)",
                                  "achieved": perm_gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                                  "frac": perm_gbs / float(peaks["hbm_gbs"]), "bytes_per_launch": perm_bytes,
                                  "ms_per_launch": perm_ms} if perm_ms else None),
            "c3_long_history": c3,
            "c2_head_adaptive_stress": c2,
            "two_gate_step": ({"ms_per_step": two_gate_ms, "frames_per_s": frames_per_s(two_gate_ms),
                               "steps": n_g} if two_gate_ms else None),
            "page_tier": tier,
            "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "e2e": ({"value": frames_per_s(e2e_ms, world), "unit": "frames/s", "ms_per_step": e2e_ms,
                     "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                     "api": "HSAPipeline (wa_pipe_*): pinned host buffers, uploads and downloads "
                            "on their own streams overlapping the previous/next step"}
                    if e2e_steps else None),
            "cpu_baseline": cpu,
            "c4_denoise_stack": ({"value": c4["frames_per_s"], "unit": "frames/s", "ms_total": c4["ms_total"],
                                  "ms_per_step": c4["ms_per_step"], "steps": c4["steps"],
                                  "workload": c4["workload"], "clocks": c4["clocks"],
                                  "gpu_launches": c4["gpu_launches"]} if c4 else None),
            "clocks": clocks,
            "gpu_launches": launches_per_step * args.steps,
            "context": {"pages_end_to_end_fps_h100": 22.0, "pages_e2e_speedup_h100": 2.21,
                        "pages_sparse_kernel_speedup_vs_fa3_hopper": 14.02,
                        "note": "the pages' numbers are end-to-end or relative on H100 with trained "
                                "weights; context only, not this metric"},
        }
        print(json.dumps(line), flush=True)
    return 0


def config_measure(cfg, dev, stream, n_steps, peak_t):
    """The step on another full-size workload (the long-history pool with prompt-level
    chunk selection, or the head-adaptive stress inputs): ms per step, and the sparse
    branch's selected-block FLOP rate from one more step with stage events."""
    from linear_attention_paged_b200 import wa, workloads as W
    inp = W.make_inputs(cfg, device="cuda", gen_device="cuda")
    step = wa.HSAStep(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"], inp["e_v"],
                      inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B, e_cur=inp.get("e_cur"),
                      e_chunks=inp.get("e_chunks"), fused_gather=True, keep_intermediates=True)
    for _ in range(3):
        step()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    for e in ev:
        e.record(stream)
    torch.cuda.synchronize()
    arr, keep = ctypes_void_array(ev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_steps):
        step()
    e1.record(stream)
    step.args.stage_events = arr     # one more step with stage events, outside the timing
    step()
    step.args.stage_events = None
    torch.cuda.synchronize()
    flags = wa.wa_device_error()
    if flags:
        raise RuntimeError(f"device error flags 0x{flags:x}")
    ms = e0.elapsed_time(e1) / n_steps
    flops, kept = selected_flops(step.inter["blk_mask"], cfg)
    attn_ms = ev[6].elapsed_time(ev[7])
    pool_bytes = 2 * inp["k_pool"].numel() * inp["k_pool"].element_size()
    del step, inp, keep
    torch.cuda.empty_cache()
    return {"pool_gb": pool_bytes / 1e9, "ms_per_step": ms, "frames_per_s": frames_per_s(ms),
            "steps": n_steps, "page_retrieval_ms": ev[0].elapsed_time(ev[1]),
            "sparse_branch_gate_ms": attn_ms, "kept_fraction": kept,
            "sparse_tflops": flops / (attn_ms * 1e-3) / 1e12,
            "sparse_frac_of_peak": flops / (attn_ms * 1e-3) / 1e12 / peak_t}


def tier_measure(inp, cfg, dev, stream, rounds=4):
    """Host -> device page traffic of the L1 <-> L2 tier: the n_c candidate pages in
    pinned host memory, K_p device slots, requests alternating between two disjoint
    sets of K_p pages so that every request misses; GB/s of page bytes moved."""
    from linear_attention_paged_b200 import wa
    n_pages = cfg.n_c
    if n_pages < 2 * cfg.K_p:
        return None
    shape = tuple(inp["k_pool"].shape[1:])
    host_k = torch.empty((n_pages,) + shape, dtype=inp["k_pool"].dtype).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    host_k.copy_(inp["k_pool"][:n_pages])
    host_v.copy_(inp["v_pool"][:n_pages])
    slot_k = torch.empty((cfg.K_p,) + shape, dtype=host_k.dtype, device=dev)
    slot_v = torch.empty_like(slot_k)
    t = wa.Tier(host_k, host_v, slot_k, slot_v)
    sets = [list(range(cfg.K_p)), list(range(cfg.K_p, 2 * cfg.K_p))]
    t.ensure(sets[1], stream)
    t.release(stream)
    torch.cuda.synchronize()
    page_bytes = 2 * host_k[0].numel() * host_k.element_size()
    ms = []
    for r in range(rounds):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        t.ensure(sets[r % 2], stream)
        e1.record(stream)
        t.release(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    stats = t.stats()
    t.close()
    moved = cfg.K_p * page_bytes
    return {"what": f"wa_tier_ensure of {cfg.K_p} non-resident pages (K and V) from pinned host memory "
                    f"into device slots, {rounds} requests alternating between two page sets",
            "bytes_per_request": moved, "ms_per_request": sum(ms) / len(ms), "ms_best": min(ms),
            "achieved_gbs": moved / (sum(ms) / len(ms) * 1e-3) / 1e9, "unit": "GB/s",
            "pcie_gen5_x16_nominal_gbs": 64.0, "misses": stats["misses"], "hits": stats["hits"],
            "bytes_h2d": stats["bytes_h2d"]}


def c4_measure(args, rank, world, local_rank):
    """Full denoise stack: `layers` layers x 4 denoising steps per chunk x `chunks`
    chunks of 3 frames.  Each layer owns a 16-page pool (8 history pages = the
    candidate chunk, 8 pages of room for appended chunks), its E_K/E_V and tau, and
    a float64 page index of its pool.  Per chunk: 4 x layers HSA steps (queries and
    gates cycle through a resident set of pre-drawn tensors), then every layer's
    new 4680-token KV is appended to its pool with the index refreshed.  The index
    of the history pages is built before timing (it belongs to the cache state);
    appends and all steps are timed.  Returns the figures of rank 0 (None elsewhere)."""
    from linear_attention_paged_b200 import wa, workloads as W
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    n_layers, n_steps, n_chunks = args.layers, 4, args.chunks
    base = W.C1.with_(name="c4_layer", n_chunks=2)
    layers = []
    for l in range(n_layers):
        cfg = base.with_(seed=replicas.rank_seed(4000 + l, rank))
        inp = W.make_inputs(cfg, device="cuda", gen_device="cuda")
        P_ = cfg.n_pool_pages
        hist = inp["chunk_pages"][0:1].contiguous()
        idx = wa.wa_pool_index(inp["k_pool"], hist[0].contiguous(), cfg.B,
                               page_index=torch.zeros((P_, cfg.T_p // cfg.B, cfg.H, cfg.d),
                                                      dtype=torch.float64, device=dev))
        g = torch.Generator(device="cuda").manual_seed(cfg.seed + 7)
        k_new = (torch.randn((cfg.Nq, cfg.H, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(torch.bfloat16)
        v_new = (torch.randn((cfg.Nq, cfg.H, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(torch.bfloat16)
        step = wa.HSAStep(inp["q"], inp["k_pool"], inp["v_pool"], hist, inp["e_k"], inp["e_v"],
                          inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B, page_index=idx)
        for key in ("q", "gate", "e_cur", "e_chunks"):
            inp.pop(key, None)
        layers.append(dict(cfg=cfg, inp=inp, idx=idx, step=step, k_new=k_new, v_new=v_new))
    n_rot = 8
    gq = torch.Generator(device="cuda").manual_seed(99 + rank)
    qs = [(torch.randn((base.Nq, base.H, base.d), generator=gq, device="cuda") / base.d ** 0.5).to(torch.bfloat16)
          for _ in range(n_rot)]
    gs = [torch.randn((base.Nq, base.H), generator=gq, device="cuda") for _ in range(n_rot)]
    import ctypes
    fill0 = base.n_c * base.T_p

    def run(chunks, fill):
        k = 0
        for _ in range(chunks):
            for _ in range(n_steps):
                for L_ in layers:
                    a = L_["step"].args
                    a.q = ctypes.c_void_p(qs[k % n_rot].data_ptr())
                    a.gate = ctypes.c_void_p(gs[k % n_rot].data_ptr())
                    L_["step"]()
                    k += 1
            for L_ in layers:
                wa.wa_pool_append(L_["inp"]["k_pool"], L_["inp"]["v_pool"], L_["k_new"], L_["v_new"], fill,
                                  page_index=L_["idx"], B=base.B)
            fill += base.Nq
        return fill

    run(1, fill0)                     # warm-up chunk (writes the first append slot)
    torch.cuda.synchronize()
    flags = wa.wa_device_error()
    if flags:
        raise RuntimeError(f"device error flags 0x{flags:x}")
    clk = ClockSampler(local_rank)
    clk.start()
    replicas.barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(n_chunks, fill0)              # rewrites the pool tail from the same offset
    e1.record(stream)
    torch.cuda.synchronize()
    replicas.barrier(world)
    clocks = clk.stop()
    total_ms = replicas.max_over_ranks(e0.elapsed_time(e1), world, dev)
    frames = world * FRAMES_PER_CHUNK * n_chunks
    del layers, qs, gs
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    n_step_calls = n_chunks * n_steps * n_layers
    # per step: block sums of the queries and the page scores from the index, block
    # scores and choice, pairing and work items, sparse attention and combine; on the
    # side stream projection, split reduction and linear branch; per append: two
    # copies and the index refresh
    return {"frames_per_s": frames / (total_ms / 1000.0), "ms_total": total_ms,
            "ms_per_step": total_ms / n_step_calls, "steps": n_step_calls,
            "workload": f"c4 full denoise stack: {n_layers} layers x {n_steps} denoising steps "
                        f"x {n_chunks} chunks of 3 frames, one-layer shapes as C1, pool of "
                        f"16 pages per layer with a float64 page index; each chunk's KV "
                        f"appended to every layer's pool (index refreshed) inside the "
                        f"timed region; queries/gates cycle through {n_rot} resident draws",
            "clocks": clocks, "gpu_launches": n_step_calls * 11 + n_chunks * n_layers * 3}


def run_c4(args, rank, world, local_rank):
    from linear_attention_paged_b200 import build as wb
    if rank == 0:
        wb.build()
    replicas.barrier(world)
    c4 = c4_measure(args, rank, world, local_rank)
    if rank == 0:
        line = {
            "metric": METRIC, "value": c4["frames_per_s"], "unit": "frames/s", "n_gpus": world,
            "steps": c4["steps"], "warmup": c4["steps"] // args.chunks, "ms_per_step": c4["ms_per_step"],
            "ms_total": c4["ms_total"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": c4["workload"],
                       "l2": "no flush: each step reads >300 MB of selected K/V",
                       "parallelism": f"replicas x{world} (independent layer stacks, no collective)"},
            "clocks": c4["clocks"], "gpu_launches": c4["gpu_launches"],
        }
        print(json.dumps(line), flush=True)
    return 0


def ctypes_void_array(events):
    import ctypes
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    return (ctypes.cast(arr, ctypes.c_void_p), arr)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end loop (profiling runs)")
    ap.add_argument("--heads", type=int, default=None,
                    help="override H of the workload (smaller profiling captures)")
    ap.add_argument("--config", choices=["c1", "c4"], default="c1",
                    help="c1: one-layer step (default); c4: the full denoise stack")
    ap.add_argument("--layers", type=int, default=30, help="c4: layers")
    ap.add_argument("--no-c4", action="store_true",
                    help="c1: skip the full denoise stack figure added to the line")
    ap.add_argument("--no-c3", action="store_true",
                    help="c1: skip the long-history (120-page pool) and stress figures added to the line")
    ap.add_argument("--b-inter", type=int, default=0, choices=[0, 64, 128],
                    help="c1: block size of the history in block selection (128: inter-chunk "
                         "granularity; the chunk's own keys keep 64)")
    ap.add_argument("--intra", action="store_true",
                    help="c1: add the chunk's own keys to the sparse branch (intra-chunk keys)")
    ap.add_argument("--chunks", type=int, default=20, help="c4: chunks")
    args = ap.parse_args()
    rank, world, local_rank = replicas.env_ranks()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        torch.cuda.set_device(local_rank)
        replicas.init(world, "nccl", 120.0, device=torch.device("cuda", local_rank))
    try:
        if args.config == "c4":
            return run_c4(args, rank, world, local_rank)
        return run_ours(args, rank, world, local_rank)
    finally:
        replicas.shutdown(world)


if __name__ == "__main__":
    sys.exit(main())
