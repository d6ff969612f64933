"""Seeded synthetic workloads for the HSA decode step.

This module only draws random tensors with the shapes and value distributions of
the workloads below; it holds none of the method's arithmetic (no means, scores,
softmax or attention).  Both the CUDA path and the fp64 oracle take their inputs
from here, so the two never share anything else.

Shapes follow the WorldAttention pages: a frame is 1560 latent tokens (a 30x52
grid in raster order), a KV page is 8 frames (WorldAttention, §3.2 "page-level KV
abstraction"), and 4 retrieved pages give 4*8*1560 = 49,920 active tokens
(§3.2 "Stage 2: page-level retrieval").  No public dataset stands behind these
inputs: the pages' Wan2.1 480p activations are replaced by Gaussian / Student-t
draws with per-page mean offsets so that page retrieval and block selection have
structure to find.

Layouts (all dense, token-major):
  q       [Nq][H][d]          queries of the current chunk
  k_pool  [P][T_p][H][d]      key pages of the HBM page pool
  v_pool  [P][T_p][H][d]      value pages
  cand    [n_c] int32         pool page ids of the candidate history chunk
  e_k,e_v [L][r]              Linformer projections, shared by heads
  gate    [Nq][H] fp32        gate logits g
  tau     [H] fp32            per-head mass thresholds
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

FRAME_TOKENS = 1560          # 30 x 52 latent grid per frame
PAGE_FRAMES = 8              # frames per KV page


@dataclasses.dataclass(frozen=True)
class HSAConfig:
    """One HSA-step workload: sizes, dtype, value recipe and seed."""
    name: str
    H: int
    d: int
    T_p: int                 # tokens per page
    n_c: int                 # pages in the candidate chunk
    Nq: int                  # query tokens of the current chunk
    K_p: int                 # retrieved pages
    B: int                   # block size (query and key)
    r: int                   # projection rank
    dtype: str               # "f32" or "bf16"
    seed: int
    recipe: str = "gauss"    # "gauss" (C0), "offset" (C1/C3/C4), "stress" (C2)
    tau_const: Optional[float] = None
    n_chunks: int = 1        # chunks in the pool (C3: 15); each chunk has n_c pages
    prompt_dim: int = 0      # prompt embedding dimension (C3: 4096)
    # C2: hot-block shift, in units of sigma_k*sqrt(d).  3 ("+3 sigma") left every
    # head's kept fraction between 36 % and 97 %; 7 spreads the per-head means from
    # 0.8 % to 90 %, the intended 1 % -> 100 % range.
    hot_beta_scale: float = 7.0
    # the current chunk's own K and V ([Nq][H][d]) join the sparse branch's keys
    intra: bool = False
    # one Linformer projection per head: e_k, e_v of shape [H][L][r]
    e_per_head: bool = False

    @property
    def L(self) -> int:
        return self.K_p * self.T_p

    @property
    def n_qb(self) -> int:
        return (self.Nq + self.B - 1) // self.B

    @property
    def n_kb(self) -> int:
        return (self.L + self.B - 1) // self.B

    @property
    def n_pool_pages(self) -> int:
        return self.n_chunks * self.n_c

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "HSAConfig":
        return dataclasses.replace(self, **kw)


# Tiny fp32 case: 1 head, d=64, 8 pages x 512 tokens, 256 queries, top-4 -> L=2048,
# B=64, tau=0.9, r=32.
C0 = HSAConfig("c0_tiny_f32", H=1, d=64, T_p=512, n_c=8, Nq=256, K_p=4, B=64, r=32,
               dtype="f32", seed=0, recipe="gauss", tau_const=0.9)
# One layer in bf16: 12 heads, d=128, 1560-token frames, 8-frame pages, a chunk of
# 8 pages, 3-frame query chunk (4680 tokens), top-4 -> L=49,920, B=64, r=256.
C1 = HSAConfig("c1_layer_bf16", H=12, d=128, T_p=PAGE_FRAMES * FRAME_TOKENS, n_c=8,
               Nq=3 * FRAME_TOKENS, K_p=4, B=64, r=256, dtype="bf16", seed=1,
               recipe="offset")
# Head-adaptive stress: C1 shapes, heavy-tailed values, planted hot key blocks.
C2 = C1.with_(name="c2_stress_bf16", seed=2, recipe="stress")
# Long history: 15 chunks x 8 pages = 120 pages (1.5M tokens) in the pool.
C3 = C1.with_(name="c3_long_bf16", seed=3, n_chunks=15, prompt_dim=4096)
CONFIGS = {c.name: c for c in (C0, C1, C2, C3)}


def tau_for(cfg: HSAConfig) -> torch.Tensor:
    """Per-head thresholds: constant (C0), 0.80+0.15*h/(H-1) (C1/C3/C4), U[0.5,0.99] (C2).

    The U[0.5,0.99] draw uses its own CPU generator seeded from ``cfg.seed`` so it
    does not depend on where the tensors are drawn."""
    H = cfg.H
    if cfg.tau_const is not None:
        return torch.full((H,), float(cfg.tau_const), dtype=torch.float32)
    if cfg.recipe == "stress":
        g = torch.Generator().manual_seed(cfg.seed * 7919 + 17)
        u = torch.rand(H, generator=g, dtype=torch.float64)
        return (0.5 + 0.49 * u).to(torch.float32)
    den = max(H - 1, 1)
    return torch.tensor([0.80 + 0.15 * h / den for h in range(H)], dtype=torch.float32)


def _student_t3_unit(shape, gen, device) -> torch.Tensor:
    """Student-t (nu=3) draws scaled to unit variance (var of t3 is 3)."""
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    # chi-square with 3 degrees of freedom = sum of three squared normals
    c = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(3):
        c += torch.randn(shape, generator=gen, device=device, dtype=torch.float32) ** 2
    return z / torch.sqrt(c / 3.0) / math.sqrt(3.0)


def make_inputs(cfg: HSAConfig, device: str = "cpu", gen_device: Optional[str] = None) -> dict:
    """Draw every input of one HSA step for ``cfg`` (seeded; same seed -> same bits).

    ``gen_device`` is where the random numbers are drawn (defaults to ``device``);
    the draws are a function of (seed, gen_device) only.
    """
    gdev = gen_device or device
    gen = torch.Generator(device=gdev)
    gen.manual_seed(cfg.seed)
    H, d, T_p, Nq, r = cfg.H, cfg.d, cfg.T_p, cfg.Nq, cfg.r
    P = cfg.n_pool_pages
    L = cfg.L
    dt = cfg.torch_dtype

    def randn(*shape):
        return torch.randn(shape, generator=gen, device=gdev, dtype=torch.float32)

    out: dict = {}
    inv_sqrt_d = 1.0 / math.sqrt(d)
    if cfg.recipe == "gauss":
        q = randn(Nq, H, d)
        k_pool = randn(P, T_p, H, d)
        v_pool = randn(P, T_p, H, d)
    else:
        if cfg.recipe == "stress":
            q = _student_t3_unit((Nq, H, d), gen, gdev) * inv_sqrt_d
            k_pool = _student_t3_unit((P, T_p, H, d), gen, gdev) * inv_sqrt_d
            v_pool = _student_t3_unit((P, T_p, H, d), gen, gdev) * inv_sqrt_d
        else:
            q = randn(Nq, H, d) * inv_sqrt_d
            k_pool = randn(P, T_p, H, d) * inv_sqrt_d
            v_pool = randn(P, T_p, H, d) * inv_sqrt_d
        # per-(page, head) mean offsets ~ N(0, 0.5) per dimension (variance 0.5),
        # drawn independently for K and V
        sd = math.sqrt(0.5)
        k_pool += (randn(P, 1, H, d) * sd)
        v_pool += (randn(P, 1, H, d) * sd)
        if cfg.recipe == "stress":
            # a per-head query mean mu_h ~ N(0, 0.5) per dimension on every Q row
            mu = randn(H, d) * sd
            q += mu.unsqueeze(0)
            # hot key blocks: per head n_h ~ U{1..32} blocks of the candidate chunk,
            # keys shifted by beta * mu_h/|mu_h| with beta = scale * sigma_k * sqrt(d)
            nblk_page = T_p // cfg.B
            n_cand_blocks = cfg.n_c * nblk_page
            beta = cfg.hot_beta_scale * inv_sqrt_d * math.sqrt(d)
            hot = []
            for h in range(H):
                n_h = int(torch.randint(1, 33, (1,), generator=gen, device=gdev).item())
                perm = torch.randperm(n_cand_blocks, generator=gen, device=gdev)[:n_h]
                unit = mu[h] / mu[h].norm()
                for b in perm.tolist():
                    pg, blk = divmod(b, nblk_page)
                    k_pool[pg, blk * cfg.B:(blk + 1) * cfg.B, h, :] += beta * unit
                hot.append(sorted(perm.tolist()))
            out["hot_blocks"] = hot
            out["hot_beta"] = beta
    e_k = randn(L, r) * (1.0 / math.sqrt(L))
    e_v = randn(L, r) * (1.0 / math.sqrt(L))
    gate = randn(Nq, H)
    tau = tau_for(cfg)

    # the candidate chunk: C3 picks it by prompt similarity, all others have one chunk
    if cfg.n_chunks > 1:
        out["e_cur"] = randn(cfg.prompt_dim).to(device)
        out["e_chunks"] = randn(cfg.n_chunks, cfg.prompt_dim).to(device)
    if cfg.intra:
        # the current chunk's own keys and values, drawn last so that every other
        # input keeps its bits: N(0,1) (gauss) or N(0,1)/sqrt(d), no page offset
        sc = 1.0 if cfg.recipe == "gauss" else inv_sqrt_d
        out["k_cur"] = (randn(Nq, H, d) * sc).to(dt).to(device)
        out["v_cur"] = (randn(Nq, H, d) * sc).to(dt).to(device)
    if cfg.e_per_head:
        # one E pair per head, drawn after every other input so that those keep their bits
        e_k = randn(H, L, r) * (1.0 / math.sqrt(L))
        e_v = randn(H, L, r) * (1.0 / math.sqrt(L))
    out["chunk_pages"] = torch.arange(P, dtype=torch.int32).reshape(cfg.n_chunks, cfg.n_c).to(device)
    out["cand"] = out["chunk_pages"][0].clone()

    out["q"] = q.to(dt).to(device)
    out["k_pool"] = k_pool.to(dt).to(device)
    del k_pool
    out["v_pool"] = v_pool.to(dt).to(device)
    del v_pool
    out["e_k"] = e_k.to(dt).to(device)
    out["e_v"] = e_v.to(dt).to(device)
    out["gate"] = gate.to(device)
    out["tau"] = tau.to(device)
    return out


def append_chunk_kv(k_pool: torch.Tensor, v_pool: torch.Tensor, fill: int, n_tokens: int,
                    gen: torch.Generator, first_free_page: int) -> int:
    """Write ``n_tokens`` new K/V rows (same recipe as C1) at pool token offset
    ``first_free_page*T_p + fill``; returns the new fill.  Used by the full
    denoise-stack workload, where each new chunk's KV is appended to the pool."""
    P, T_p, H, d = k_pool.shape
    flat_k = k_pool.view(P * T_p, H, d)
    flat_v = v_pool.view(P * T_p, H, d)
    s = first_free_page * T_p + fill
    e = s + n_tokens
    assert e <= P * T_p, "pool is full"
    inv = 1.0 / math.sqrt(d)
    flat_k[s:e] = (torch.randn((n_tokens, H, d), generator=gen, device=k_pool.device) * inv).to(k_pool.dtype)
    flat_v[s:e] = (torch.randn((n_tokens, H, d), generator=gen, device=k_pool.device) * inv).to(v_pool.dtype)
    return fill + n_tokens
