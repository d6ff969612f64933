"""Failure detection on the GPU without a fault: a bounded wait is made to run out.

A dedicated one-CTA kernel waits, through the same bounded mbarrier wait the tcgen05
kernels use, on a barrier that nothing ever arrives at.  With a 1 ms limit it must
give up, record WA_DEVERR_TIMEOUT in the device error word and return; the context
stays usable, which a decode step run right after (checked against the oracle)
confirms.  No product kernel is ever made to abort on the GPU."""
import pytest
import torch

from linear_attention_paged_b200 import workloads as W
from oracle import hsa_oracle as O
from tests.helpers import assert_close, compare_selection, mask_to_sets

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wa():
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa as _wa
    return _wa


def _small_step_ok(wa, seed):
    cfg = W.HSAConfig("fd_small", H=2, d=128, T_p=1280, n_c=6, Nq=520, K_p=3, B=64, r=128,
                      dtype="bf16", seed=seed, recipe="offset")
    inp = W.make_inputs(cfg, device="cuda")
    out, inter = wa.wa_hsa_step(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"],
                                inp["e_v"], inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B,
                                keep_intermediates=True)
    res = O.hsa_step(inp, cfg.B, cfg.K_p)
    compare_selection(mask_to_sets(inter["blk_mask"], cfg.n_kb), res["kept"], res["block_margin"],
                      "step after the timeout")
    assert_close(out, res["o"], "bf16", "step after the timeout")
    assert wa.wa_device_error() == 0


def test_bounded_wait_runs_out_and_reports(wa):
    assert wa.wa_device_error() == 0
    limit = 1_000_000                       # 1 ms
    el = wa.wa_check_bounded_wait(limit)
    flags = wa.wa_device_error()            # synchronises, reads and clears the word
    assert flags & wa.DEVERR_TIMEOUT, f"no timeout recorded (flags 0x{flags:x})"
    elapsed = int(el.item())
    print(f"[failure-detection] wait gave up after {elapsed / 1e6:.3f} ms (limit 1 ms)")
    assert limit <= elapsed < 200 * limit
    # the word was cleared and the context still runs kernels correctly
    assert wa.wa_device_error() == 0
    _small_step_ok(wa, seed=61)


def test_kernels_take_the_configured_wait_limit(wa):
    """A different (longer) bound reaches the tcgen05 kernels without changing results."""
    default = wa.wa_get_wait_limit_ns()
    wa.wa_set_wait_limit_ns(5_000_000_000)
    try:
        _small_step_ok(wa, seed=62)
    finally:
        wa.wa_set_wait_limit_ns(default)
