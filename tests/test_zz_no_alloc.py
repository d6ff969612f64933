"""The projection entry point that allocates nothing (wa_linear_project_noalloc).

It exists for callers that cannot allocate device memory, for example code running
inside a host framework that owns all device memory through its own pool, or a
real-time loop where an allocation is not allowed.  It keeps its split partials
in a fixed array inside libwa instead of a caller workspace.  This test calls it
through the C ABI, twice in a row on different inputs, and checks each result
against the existing workspace-based entry point wa_linear_project, within the
bf16 tolerance the other parity tests use, and against the float64 oracle.  Where
both entry points split L the same way, their results are the same bits.  The file
is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

from linear_attention_paged_b200 import workloads as W
from oracle import hsa_oracle as O
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wa():
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa as _wa
    return _wa


def _inputs(L, H, d, r, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = (torch.randn((L, H, d), generator=g, device="cuda") / d ** 0.5 + 0.3).to(torch.bfloat16)
    v = (torch.randn((L, H, d), generator=g, device="cuda") / d ** 0.5 - 0.2).to(torch.bfloat16)
    ek = (torch.randn((L, r), generator=g, device="cuda") / L ** 0.5).to(torch.bfloat16)
    ev = (torch.randn((L, r), generator=g, device="cuda") / L ** 0.5).to(torch.bfloat16)
    return k, v, ek, ev


def _noalloc(wa, k, v, ek, ev):
    L, H, d = k.shape
    r = ek.shape[1]
    kt = torch.full((r, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vt = torch.full_like(kt, float("nan"))
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = wa.lib.wa_linear_project_noalloc(
        ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(ek.data_ptr()),
        ctypes.c_void_p(ev.data_ptr()), L, H, d, r, wa.WA_BF16, ctypes.c_void_p(kt.data_ptr()),
        ctypes.c_void_p(vt.data_ptr()), st)
    assert rc == wa.WA_OK, wa.last_error()
    return kt, vt


def test_noalloc_projection_matches_workspace_projection_twice(wa):
    # call 1: the one-layer bench shape (L = 49,920, 12 heads x 128, r = 256)
    cfg = W.C1
    k, v, ek, ev = _inputs(cfg.L, cfg.H, cfg.d, cfg.r, seed=101)
    kt_ref, vt_ref = wa.wa_linear_project(k, v, ek, ev)
    kt, vt = _noalloc(wa, k, v, ek, ev)
    torch.cuda.synchronize()
    assert_close(kt, kt_ref, "bf16", "no-alloc K~ (call 1)")
    assert_close(vt, vt_ref, "bf16", "no-alloc V~ (call 1)")
    # against the oracle on two heads (the first and the last), all r rows
    for h in (0, cfg.H - 1):
        kr, vr = O.linear_project(k[:, h:h + 1].cpu(), v[:, h:h + 1].cpu(), ek.cpu(), ev.cpu())
        assert_close(kt[:, h:h + 1], kr, "bf16", f"no-alloc K~ (call 1, head {h}) vs oracle")
        assert_close(vt[:, h:h + 1], vr, "bf16", f"no-alloc V~ (call 1, head {h}) vs oracle")
    # call 2, right after: another shape and other values; the shared scratch
    # still holds call 1's partials and must not leak into this result
    k2, v2, ek2, ev2 = _inputs(3000, 4, 64, 128, seed=202)
    kt2_ref, vt2_ref = wa.wa_linear_project(k2, v2, ek2, ev2)
    kt2, vt2 = _noalloc(wa, k2, v2, ek2, ev2)
    torch.cuda.synchronize()
    assert_close(kt2, kt2_ref, "bf16", "no-alloc K~ (call 2)")
    assert_close(vt2, vt2_ref, "bf16", "no-alloc V~ (call 2)")
    # this shape fits the scratch with the default number of splits of L, so both
    # entry points add the same partials in the same order
    assert torch.equal(kt2, kt2_ref) and torch.equal(vt2, vt2_ref)
    kr2, vr2 = O.linear_project(k2.cpu(), v2.cpu(), ek2.cpu(), ev2.cpu())
    assert_close(kt2, kr2, "bf16", "no-alloc K~ (call 2) vs oracle")
    assert_close(vt2, vr2, "bf16", "no-alloc V~ (call 2) vs oracle")
    assert wa.wa_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(wa):
    # 2 x r x H*d x 4 bytes per split: r = 256, H*d = 16,448 needs ~33.7 MB > 32 MiB.
    # Real device buffers of the claimed sizes, so that the call could not touch
    # memory it does not own even if the size check were missing.
    L, H, d, r = 1024, 257, 64, 256
    k, v, ek, ev = _inputs(L, H, d, r, seed=303)
    kt = torch.empty((r, H, d), dtype=torch.bfloat16, device="cuda")
    vt = torch.empty_like(kt)
    rc = wa.lib.wa_linear_project_noalloc(
        ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(ek.data_ptr()),
        ctypes.c_void_p(ev.data_ptr()), L, H, d, r, wa.WA_BF16, ctypes.c_void_p(kt.data_ptr()),
        ctypes.c_void_p(vt.data_ptr()), None)
    assert rc == wa.WA_ERR_UNSUPPORTED
    assert "scratch" in wa.last_error()
    torch.cuda.synchronize()
    assert wa.wa_device_error() == 0
