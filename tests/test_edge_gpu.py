"""GPU parity at the limits of the kernels' internal tables, against the float64
oracle (every row compared):

  * more than 128 query blocks: the attention work list pairs neighbouring query
    blocks instead of searching its distance table;
  * more than 64 pages in the active key sequence: the attention kernel reads the
    page table from global memory instead of staging it in shared memory;
  * the largest key list the library takes, 8192 key blocks (524,288 keys), with pages
    of 2048 blocks: the key-list scan, the block-selection sort of 8192 scores and
    the 256-word masks at their maximum;
  * the smallest steps: one query row over one key block of one page (bf16 and
    fp32), and a query tail of a single row.
"""
import pytest
import torch

from oracle import hsa_oracle as O
from linear_attention_paged_b200 import workloads as W
from tests.helpers import MARGIN_F64, assert_close, compare_selection, mask_to_sets
from tests.test_parity_gpu import check_device_ok, dkey

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wa():
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa as _wa
    return _wa


def _check_step(wa, cfg, fused=True):
    inp = W.make_inputs(cfg, device="cuda")
    out, inter = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                                inp["e_v"], inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B,
                                fused_gather=fused, keep_intermediates=True)
    torch.cuda.synchronize()
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    if res["page_margin"] >= MARGIN_F64:
        assert inter["sel"].cpu().tolist() == res["sel"]
    compare_selection(mask_to_sets(inter["blk_mask"], cfg.n_kb), res["kept"], res["block_margin"],
                      f"{cfg.name} masks")
    assert_close(inter["k_til"], res["k_til"], dkey(cfg), f"{cfg.name} K~")
    assert_close(out, res["o"], dkey(cfg), f"{cfg.name} O ({'fused' if fused else 'gathered'})")
    check_device_ok(wa)
    return res


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "gathered"])
def test_step_many_query_blocks_neighbour_pairing(wa, fused):
    # 130 query blocks (the last 5 rows): more than the 128 the pairing table holds
    cfg = W.HSAConfig("edge_many_qblocks", H=1, d=64, T_p=640, n_c=4, Nq=129 * 64 + 5, K_p=2, B=64,
                      r=128, dtype="bf16", seed=51, recipe="offset")
    assert cfg.n_qb == 130
    _check_step(wa, cfg, fused)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "gathered"])
def test_step_more_pages_than_the_staged_page_table(wa, fused):
    # 70 retrieved pages of one block each: the active sequence spans more pages than
    # the 64 page-table entries the attention kernel stages
    cfg = W.HSAConfig("edge_many_pages", H=2, d=64, T_p=64, n_c=80, Nq=200, K_p=70, B=64, r=128,
                      dtype="bf16", seed=52, recipe="offset")
    assert cfg.L // cfg.T_p == 70
    _check_step(wa, cfg, fused)


def test_step_at_the_largest_key_list(wa):
    # 4 pages of 131,072 keys: 8192 key blocks, the most a step takes
    cfg = W.HSAConfig("edge_max_keys", H=1, d=64, T_p=131072, n_c=4, Nq=128, K_p=4, B=64, r=128,
                      dtype="bf16", seed=53, recipe="offset")
    assert cfg.n_kb == 8192
    res = _check_step(wa, cfg)
    kept = [len(row) for row in res["kept"][0]]
    print(f"[info] {cfg.name}: kept blocks per query block {kept} of {cfg.n_kb}")


SMALLEST = [
    W.HSAConfig("edge_one_query", H=1, d=64, T_p=64, n_c=1, Nq=1, K_p=1, B=64, r=128, dtype="bf16",
                seed=54, recipe="offset"),
    W.HSAConfig("edge_one_row_tail", H=1, d=128, T_p=128, n_c=2, Nq=65, K_p=1, B=64, r=128,
                dtype="bf16", seed=55, recipe="offset"),
    W.HSAConfig("edge_one_query_f32", H=1, d=64, T_p=64, n_c=1, Nq=1, K_p=1, B=64, r=8, dtype="f32",
                seed=56, recipe="gauss", tau_const=0.9),
]


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "gathered"])
@pytest.mark.parametrize("cfg", SMALLEST, ids=lambda c: c.name)
def test_smallest_steps(wa, cfg, fused):
    _check_step(wa, cfg, fused)
