"""GPU checks of the cube-tile token order (WorldAttention Appendix A.1.3): the device
row permutation against plain indexing, and an HSA step run on cube-ordered pages and
queries against the oracle fed the same inputs permuted by its own cube order."""
import numpy as np
import pytest
import torch

from oracle import hsa_oracle as O
from linear_attention_paged_b200 import workloads as W
from tests.helpers import MARGIN_F64, assert_close, compare_selection, mask_to_sets

pytestmark = pytest.mark.gpu

# pages of 8 frames x 10 x 16 latents, (8, 2, 4) cubes: 20 cubes = 20 key blocks per
# page; the query chunk is 2 frames x 10 x 26 (cubes cut short along t and w)
CUBE_CFG = W.HSAConfig("small_bf16_cube", H=2, d=128, T_p=1280, n_c=6, Nq=520, K_p=3, B=64, r=128,
                       dtype="bf16", seed=21, recipe="offset")
PAGE_GRID, Q_GRID, CUBE = (8, 10, 16), (2, 10, 26), (8, 2, 4)


@pytest.fixture(scope="module")
def wa():
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa as _wa
    return _wa


def test_permute_rows_gather_scatter(wa):
    g = torch.Generator(device="cpu").manual_seed(5)
    n, cols = 4680, 1536
    x = torch.randn(n, cols, generator=g).to(torch.bfloat16).cuda()
    perm = torch.randperm(n, generator=g).to(torch.int32)
    pd = perm.cuda()
    y = wa.wa_permute_rows(x, pd)
    assert torch.equal(y, x[perm.long().cuda()])
    z = wa.wa_permute_rows(y, pd, inverse=True)
    assert torch.equal(z, x)
    # rows of 48 bytes (three vectors: the tail loop only)
    xs = torch.randn(37, 12, generator=g).cuda()
    ps = torch.randperm(37, generator=g).to(torch.int32)
    assert torch.equal(wa.wa_permute_rows(xs, ps.cuda()), xs[ps.long().cuda()])
    assert wa.wa_device_error() == 0


def test_permute_rows_bad_index_is_flagged(wa):
    x = torch.arange(64 * 8, dtype=torch.float32, device="cuda").reshape(64, 8)
    perm = torch.arange(64, dtype=torch.int32)
    perm[5] = 64                                  # outside [0, 64): skipped and recorded
    out = torch.zeros_like(x)
    wa.wa_permute_rows(x, perm.cuda(), out=out)
    assert wa.wa_device_error() & wa.DEVERR_ROW_ID
    assert torch.equal(out[:5], x[:5]) and torch.equal(out[6:], x[6:]) and not out[5].any()


def test_hsa_step_on_cube_order(wa):
    cfg = CUBE_CFG
    assert np.prod(PAGE_GRID) == cfg.T_p and np.prod(Q_GRID) == cfg.Nq
    inp = W.make_inputs(cfg, device="cuda")
    pp = wa.wa_cube_order(*PAGE_GRID, *CUBE)
    pq = wa.wa_cube_order(*Q_GRID, *CUBE)
    pp_d, pq_d = pp.cuda(), pq.cuda()
    # device side: every pool page and the queries into cube order
    k_pool = torch.stack([wa.wa_permute_rows(inp["k_pool"][p], pp_d) for p in range(cfg.n_pool_pages)])
    v_pool = torch.stack([wa.wa_permute_rows(inp["v_pool"][p], pp_d) for p in range(cfg.n_pool_pages)])
    q = wa.wa_permute_rows(inp["q"], pq_d)
    gate = inp["gate"][pq_d.long()].contiguous()       # [Nq][H] float32 rows are 8 bytes
    out_c, inter = wa.wa_hsa_step(q, k_pool, v_pool, inp["chunk_pages"], inp["e_k"], inp["e_v"],
                                  inp["tau"].cuda(), gate, cfg.K_p, cfg.B, fused_gather=True,
                                  keep_intermediates=True)
    out = wa.wa_permute_rows(out_c, pq_d, inverse=True)
    # oracle side: the same inputs permuted by the oracle's own cube order, on the host
    op = torch.tensor(O.cube_order(*PAGE_GRID, *CUBE))
    oq = torch.tensor(O.cube_order(*Q_GRID, *CUBE))
    ref_in = dict(inp)
    ref_in["k_pool"] = inp["k_pool"].cpu()[:, op]
    ref_in["v_pool"] = inp["v_pool"].cpu()[:, op]
    ref_in["q"] = inp["q"].cpu()[oq]
    ref_in["gate"] = inp["gate"].cpu()[oq]
    res = O.hsa_step(ref_in, cfg.B, cfg.K_p)
    if res["page_margin"] >= MARGIN_F64:
        assert inter["sel"].cpu().tolist() == res["sel"]
    compare_selection(mask_to_sets(inter["blk_mask"], cfg.n_kb), res["kept"], res["block_margin"],
                      "cube-order masks")
    o_raster = np.empty_like(res["o"])
    o_raster[oq.numpy()] = res["o"]
    assert_close(out, o_raster, "bf16", "cube-order step O (back in raster order)")
    assert wa.wa_device_error() == 0
