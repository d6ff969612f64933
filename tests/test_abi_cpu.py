"""Host-side checks of libwa that need no GPU: the library loads, exports every
function include/wa.h declares, and rejects bad arguments on the host before any
device work (null pointers, K_p > n_c, unsupported shapes, short workspaces)."""
import ctypes
import subprocess

import pytest

from linear_attention_paged_b200 import build as wa_build

wa_build.build()
from linear_attention_paged_b200 import wa  # noqa: E402

FAKE = ctypes.c_void_p(4096)   # a non-null pointer that is never dereferenced on these paths


def test_exports_every_declared_function():
    declared = wa.header_functions()
    assert len(declared) >= 15
    out = subprocess.run(["nm", "-D", "--defined-only", wa.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared if f not in exported]
    assert not missing, f"declared but not exported: {missing}"
    # and nothing else: internal helpers and kernels stay hidden
    extra = sorted(e for e in exported if e not in declared)
    assert not extra, f"exported but not declared in wa.h: {extra[:8]}"
    for f in declared:
        assert hasattr(wa.lib, f)


def test_version_and_error_string():
    assert "sm_100a" in wa.version()
    assert isinstance(wa.last_error(), str)


def test_workspace_sizes_positive_and_reject_bad_sizes():
    assert wa.lib.wa_page_score_workspace_size(4680, 12, 128, 8, 12480, 64) > 0
    assert wa.lib.wa_page_score_workspace_size(0, 12, 128, 8, 12480, 64) == 0
    assert wa.lib.wa_block_select_workspace_size(4680, 12, 128, 49920, 64) > 0
    assert wa.lib.wa_linear_project_workspace_size(49920, 12, 128, 256, wa.WA_BF16) > 0
    assert wa.lib.wa_linear_project_workspace_size(2048, 1, 64, 32, wa.WA_F32) == 0
    assert wa.lib.wa_hsa_attention_workspace_size(4680, 12, 128, 49920, 64, 256, wa.WA_BF16) > 0


def _page_score(**kw):
    a = dict(q=FAKE, Nq=4680, H=12, d=128, k_pool=FAKE, P=8, T_p=12480, cand=FAKE, n_c=8, K_p=4,
             B=64, dt=wa.WA_BF16, alpha=FAKE, sel=FAKE, kbm=None, ws=FAKE, nbytes=1 << 40)
    a.update(kw)
    return wa.lib.wa_page_score(a["q"], a["Nq"], a["H"], a["d"], a["k_pool"], a["P"], a["T_p"],
                                a["cand"], a["n_c"], a["K_p"], a["B"], a["dt"], a["alpha"], a["sel"],
                                a["kbm"], a["ws"], a["nbytes"], None)


def test_page_score_validation():
    assert _page_score(q=None) == wa.WA_ERR_INVALID_ARG
    assert _page_score(K_p=9) == wa.WA_ERR_INVALID_ARG
    assert "K_p" in wa.last_error()
    assert _page_score(K_p=0) == wa.WA_ERR_INVALID_ARG
    assert _page_score(d=96) == wa.WA_ERR_UNSUPPORTED
    assert _page_score(B=128) == wa.WA_ERR_UNSUPPORTED
    assert _page_score(dt=7) == wa.WA_ERR_INVALID_ARG
    assert _page_score(kbm=FAKE, T_p=12481) == wa.WA_ERR_UNSUPPORTED
    assert _page_score(nbytes=16) == wa.WA_ERR_WORKSPACE
    assert _page_score(ws=ctypes.c_void_p(4096 + 8)) == wa.WA_ERR_WORKSPACE


def test_block_select_validation():
    f = wa.lib.wa_block_select
    # both key sources
    assert f(FAKE, 100, 1, 64, FAKE, FAKE, 640, 64, wa.WA_F32, FAKE, None, None, None, FAKE, 1 << 30,
             None) == wa.WA_ERR_INVALID_ARG
    # neither
    assert f(FAKE, 100, 1, 64, None, None, 640, 64, wa.WA_F32, FAKE, None, None, None, FAKE, 1 << 30,
             None) == wa.WA_ERR_INVALID_ARG
    # too many key blocks
    assert f(FAKE, 100, 1, 64, FAKE, None, 64 * 8193, 64, wa.WA_F32, FAKE, None, None, None, FAKE,
             1 << 40, None) == wa.WA_ERR_INVALID_ARG


def test_attention_and_projection_validation():
    f = wa.lib.wa_hsa_attention
    ok = dict(q=FAKE, Nq=256, H=1, d=64, k=FAKE, v=FAKE, L=2048, B=64, m=FAKE, kt=FAKE, vt=FAKE, r=32,
              g=FAKE, dt=wa.WA_F32, out=FAKE)

    def call(**kw):
        a = dict(ok); a.update(kw)
        return f(a["q"], a["Nq"], a["H"], a["d"], a["k"], a["v"], a["L"], a["B"], a["m"], a["kt"],
                 a["vt"], a["r"], a["g"], a["dt"], a["out"], None, None, FAKE, 1 << 40, None)
    assert call(m=None) == wa.WA_ERR_INVALID_ARG
    assert call(r=0) == wa.WA_ERR_INVALID_ARG
    assert call(dt=wa.WA_BF16, r=32) == wa.WA_ERR_UNSUPPORTED     # tensor-core path needs r in {128,256}
    assert call(d=32) == wa.WA_ERR_UNSUPPORTED
    g = wa.lib.wa_linear_project
    assert g(FAKE, FAKE, FAKE, None, 2048, 1, 64, 32, wa.WA_F32, FAKE, FAKE, None, 0, None) == wa.WA_ERR_INVALID_ARG
    f2 = wa.lib.wa_hsa_attention_gated2

    def call2(gl):
        a = ok
        return f2(a["q"], a["Nq"], a["H"], a["d"], a["k"], a["v"], a["L"], a["B"], a["m"], a["kt"],
                  a["vt"], a["r"], a["g"], gl, a["dt"], a["out"], None, None, FAKE, 1 << 40, None)
    assert call2(None) == wa.WA_ERR_INVALID_ARG         # the second gate is required here


def _step_args(**kw):
    a = wa.StepArgs()
    a.chunk_pages = FAKE; a.n_c = 8
    a.q = FAKE; a.Nq = 4680; a.H = 12; a.d = 128
    a.k_pool = FAKE; a.v_pool = FAKE; a.n_pool_pages = 8; a.T_p = 12480
    a.K_p = 4; a.B = 64; a.r = 256
    a.e_k = FAKE; a.e_v = FAKE; a.tau = FAKE; a.gate = FAKE
    a.dtype = wa.WA_BF16; a.fused_gather = 1; a.out = FAKE
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_step_validation_and_workspace():
    a = _step_args()
    n = wa.lib.wa_hsa_step_workspace_size(ctypes.byref(a))
    assert n > 0
    # non-fused needs room for K_active and V_active (2 x 153 MB at this shape)
    b = _step_args(fused_gather=0)
    assert wa.lib.wa_hsa_step_workspace_size(ctypes.byref(b)) > 2 * 49920 * 12 * 128 * 2
    assert wa.lib.wa_hsa_step(ctypes.byref(_step_args(K_p=9)), FAKE, 1 << 40, None) == wa.WA_ERR_INVALID_ARG
    assert wa.lib.wa_hsa_step(ctypes.byref(_step_args(q=None)), FAKE, 1 << 40, None) == wa.WA_ERR_INVALID_ARG
    assert wa.lib.wa_hsa_step(ctypes.byref(_step_args(T_p=12481)), FAKE, 1 << 40, None) == wa.WA_ERR_UNSUPPORTED
    assert wa.lib.wa_hsa_step(ctypes.byref(_step_args(r=200)), FAKE, 1 << 40, None) == wa.WA_ERR_UNSUPPORTED
    assert wa.lib.wa_hsa_step(ctypes.byref(a), FAKE, 64, None) == wa.WA_ERR_WORKSPACE
    assert wa.lib.wa_hsa_step_workspace_size(ctypes.byref(_step_args(K_p=9))) == 0
    # a prompt set needs its embeddings
    assert wa.lib.wa_hsa_step(ctypes.byref(_step_args(e_cur=FAKE, n_chunks=0)), FAKE, 1 << 40,
                              None) == wa.WA_ERR_INVALID_ARG


def test_binding_has_no_fallback():
    # the binding exposes the library's functions only; every entry point named in
    # the header is bound to the shared object
    for name in wa.header_functions():
        assert getattr(wa.lib, name).__name__ == name


def test_cube_order_matches_oracle():
    # the library's closed form against the oracle's walk over the cubes (host only)
    from oracle import hsa_oracle as O
    shapes = [(2, 2, 4, 1, 2, 2), (1, 3, 3, 1, 2, 2), (8, 30, 52, 8, 2, 4), (3, 30, 52, 8, 2, 4),
              (5, 7, 11, 2, 3, 4), (2, 10, 26, 8, 2, 4), (1, 1, 1, 4, 4, 4), (4, 9, 13, 4, 4, 4)]
    for sh in shapes:
        assert wa.wa_cube_order(*sh).tolist() == O.cube_order(*sh), sh


def test_cube_order_and_permute_validation():
    perm = (ctypes.c_int32 * 4)()
    assert wa.lib.wa_cube_order(0, 2, 2, 1, 1, 1, perm) == wa.WA_ERR_INVALID_ARG
    assert wa.lib.wa_cube_order(1, 2, 2, 1, 0, 1, perm) == wa.WA_ERR_INVALID_ARG
    assert wa.lib.wa_cube_order(1, 2, 2, 1, 1, 1, None) == wa.WA_ERR_INVALID_ARG
    assert wa.lib.wa_cube_order(65536, 65536, 2, 1, 1, 1, perm) == wa.WA_ERR_INVALID_ARG
    f = wa.lib.wa_permute_rows
    assert f(None, FAKE, FAKE, 4, 16, 0, None) == wa.WA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 0, 16, 0, None) == wa.WA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 2**31 - 1, 16, 0, None) == wa.WA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 4, 24, 0, None) == wa.WA_ERR_UNSUPPORTED     # rows of 16-byte multiples
    assert f(FAKE, ctypes.c_void_p(4096 + 8), FAKE, 4, 16, 0, None) == wa.WA_ERR_UNSUPPORTED


def test_noalloc_projection_host_rejections():
    """wa_linear_project_noalloc rejects on the host, before any CUDA call: shapes whose
    split partials exceed its fixed scratch, and an H so large that H*d would wrap
    around in 32-bit arithmetic (2^25 + 1 heads of 128 -> 128 columns)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake pointers are used only where no GPU can be reached")
    f = wa.lib.wa_linear_project_noalloc
    assert f(FAKE, FAKE, FAKE, FAKE, 1024, 257, 64, 256, wa.WA_BF16, FAKE, FAKE, None) == \
        wa.WA_ERR_UNSUPPORTED
    assert "scratch" in wa.last_error()
    assert f(FAKE, FAKE, FAKE, FAKE, 1024, (1 << 25) + 1, 128, 128, wa.WA_BF16, FAKE, FAKE, None) == \
        wa.WA_ERR_UNSUPPORTED
    assert "scratch" in wa.last_error()
    assert f(FAKE, FAKE, FAKE, FAKE, 1024, 12, 128, 256, wa.WA_F32, FAKE, FAKE, None) == \
        wa.WA_ERR_UNSUPPORTED
    assert f(None, FAKE, FAKE, FAKE, 1024, 12, 128, 256, wa.WA_BF16, FAKE, FAKE, None) == \
        wa.WA_ERR_INVALID_ARG


def test_wait_limit_setting_and_selftest_validation():
    """The bound of the kernels' mbarrier waits is a process-wide setting with a checked
    range; the bounded-wait self-test rejects limits outside its range on the host."""
    default = wa.wa_get_wait_limit_ns()
    assert default == 2_000_000_000
    for bad in (0, 999, 60_000_000_001):
        assert wa.lib.wa_set_wait_limit_ns(bad) == wa.WA_ERR_INVALID_ARG
    assert wa.wa_get_wait_limit_ns() == default
    wa.wa_set_wait_limit_ns(5_000_000)
    assert wa.wa_get_wait_limit_ns() == 5_000_000
    wa.wa_set_wait_limit_ns(default)
    for bad in (0, 999, 1_000_000_001):
        assert wa.lib.wa_check_bounded_wait(bad, None, None) == wa.WA_ERR_INVALID_ARG
        assert "limit" in wa.last_error()
