"""ctypes binding of libwa (include/wa.h) with the same function names.

Argument marshalling only: every step runs in the CUDA kernels of libwa.so.
Tensors are torch tensors on the current CUDA device (contiguous, token-major,
see include/wa.h); workspaces are carved from a per-device cached torch buffer,
so the library itself never allocates.  Importing this module raises ImportError
when libwa.so has not been built -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwa.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "wa.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m linear_attention_paged_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

WA_OK, WA_ERR_INVALID_ARG, WA_ERR_UNSUPPORTED, WA_ERR_CUDA, WA_ERR_DEVICE, WA_ERR_WORKSPACE = range(6)
WA_F32, WA_BF16 = 0, 1
DEVERR_PAGE_ID, DEVERR_ZERO_NORM, DEVERR_TIMEOUT, DEVERR_ROW_ID = 1, 2, 4, 8

c_void_p, c_int, c_size_t = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
P = c_void_p


class WAError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


class StepArgs(ctypes.Structure):
    """Mirror of ``wa_step_args`` (field order and types must match include/wa.h)."""
    _fields_ = [
        ("e_cur", P), ("e_chunks", P), ("n_chunks", c_int), ("D", c_int),
        ("chunk_pages", P), ("n_c", c_int),
        ("q", P), ("Nq", c_int), ("H", c_int), ("d", c_int),
        ("k_pool", P), ("v_pool", P), ("n_pool_pages", c_int), ("T_p", c_int),
        ("K_p", c_int), ("B", c_int), ("r", c_int),
        ("e_k", P), ("e_v", P), ("tau", P), ("gate", P),
        ("dtype", c_int), ("fused_gather", c_int),
        ("out", P),
        ("chunk_out", P), ("alpha_out", P), ("sel_out", P), ("blk_mask_out", P),
        ("k_til_out", P), ("v_til_out", P),
        ("stage_events", P),
        ("page_index", P),
        ("gate_lin", P),
        ("k_cur", P), ("v_cur", P),
        ("B_inter", c_int),
        ("e_head_stride", ctypes.c_longlong),
    ]


_SIGS = {
    "wa_last_error": (ctypes.c_char_p, []),
    "wa_version": (ctypes.c_char_p, []),
    "wa_device_error": (c_int, [P, P]),
    "wa_prompt_select": (c_int, [P, P, c_int, c_int, P, P]),
    "wa_page_score_workspace_size": (c_size_t, [c_int] * 6),
    "wa_page_score": (c_int, [P, c_int, c_int, c_int, P, c_int, c_int, P, c_int, c_int, c_int,
                              c_int, P, P, P, P, c_size_t, P]),
    "wa_gather_pages": (c_int, [P, P, c_int, c_int, c_int, c_int, P, c_int, c_int, P, P, P]),
    "wa_block_select_workspace_size": (c_size_t, [c_int] * 5),
    "wa_block_select": (c_int, [P, c_int, c_int, c_int, P, P, c_int, c_int, c_int, P, P, P, P,
                                P, c_size_t, P]),
    "wa_linear_project_workspace_size": (c_size_t, [c_int] * 5),
    "wa_linear_project": (c_int, [P, P, P, P, c_int, c_int, c_int, c_int, c_int, P, P, P,
                                  c_size_t, P]),
    "wa_linear_project_noalloc": (c_int, [P, P, P, P, c_int, c_int, c_int, c_int, c_int, P, P, P]),
    "wa_linear_project_heads": (c_int, [P, P, P, P, c_int, c_int, c_int, c_int, c_int, ctypes.c_longlong,
                                        P, P, P, c_size_t, P]),
    "wa_hsa_attention_workspace_size": (c_size_t, [c_int] * 7),
    "wa_hsa_attention": (c_int, [P, c_int, c_int, c_int, P, P, c_int, c_int, P, P, P, c_int, P,
                                 c_int, P, P, P, P, c_size_t, P]),
    "wa_hsa_attention_gated2": (c_int, [P, c_int, c_int, c_int, P, P, c_int, c_int, P, P, P, c_int,
                                        P, P, c_int, P, P, P, P, c_size_t, P]),
    "wa_pool_index": (c_int, [P, c_int, c_int, c_int, c_int, c_int, c_int, P, c_int, P, P]),
    "wa_pool_append": (c_int, [P, P, c_int, c_int, c_int, c_int, c_int, P, P, c_int, ctypes.c_longlong,
                               P, c_int, P]),
    "wa_hsa_step_workspace_size": (c_size_t, [ctypes.POINTER(StepArgs)]),
    "wa_hsa_step": (c_int, [ctypes.POINTER(StepArgs), P, c_size_t, P]),
    "wa_pipe_create": (c_int, [ctypes.POINTER(StepArgs), P, P, P, P, c_size_t, P, P]),
    "wa_pipe_destroy": (c_int, [P]),
    "wa_pipe_begin": (c_int, [P]),
    "wa_pipe_submit": (c_int, [P, P, P, P]),
    "wa_pipe_end": (c_int, [P]),
    "wa_pipe_sync": (c_int, [P]),
    "wa_tier_create": (c_int, [c_int, c_int, c_size_t, P, P, P, P, P]),
    "wa_tier_destroy": (c_int, [P]),
    "wa_tier_ensure": (c_int, [P, P, c_int, P, P]),
    "wa_tier_release": (c_int, [P, P]),
    "wa_tier_prefetch": (c_int, [P, P, c_int, P]),
    "wa_tier_mark_dirty": (c_int, [P, c_int]),
    "wa_tier_flush": (c_int, [P, P]),
    "wa_tier_slot_of": (c_int, [P, c_int, P]),
    "wa_tier_get_stats": (c_int, [P, P]),
    "wa_set_wait_limit_ns": (c_int, [ctypes.c_uint64]),
    "wa_get_wait_limit_ns": (ctypes.c_uint64, []),
    "wa_check_bounded_wait": (c_int, [ctypes.c_uint64, P, P]),
    "wa_cube_order": (c_int, [c_int] * 6 + [P]),
    "wa_permute_rows": (c_int, [P, P, P, c_int, c_size_t, c_int, P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def header_functions() -> list:
    """Names of the functions declared in include/wa.h."""
    txt = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:WA_API\s+)?(?:const\s+)?\w+\*?\s+\**(wa_\w+)\s*\(", txt, re.M)))


def last_error() -> str:
    return lib.wa_last_error().decode()


def version() -> str:
    return lib.wa_version().decode()


def _check(fn: str, status: int) -> None:
    if status != WA_OK:
        raise WAError(fn, status, last_error())


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return WA_F32
    if t.dtype == torch.bfloat16:
        return WA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


_WS: dict = {}

# Canary byte for the buffers this binding hands to the library (outputs and
# workspaces), or None.  Tests set it (0xFF: NaN in every float and float64, -1 in
# every int) so that a kernel which leaves part of an output or a workspace
# unwritten, or reads scratch it did not write first, shows up as a wrong value.
CANARY: Optional[int] = None


def _fill(t: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if t is not None and CANARY is not None:
        t.view(torch.uint8).fill_(CANARY)
    return t


def _empty(shape, dtype, device) -> torch.Tensor:
    return _fill(torch.empty(shape, dtype=dtype, device=device))


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """Cached per-device scratch buffer of at least ``nbytes`` (256-byte aligned)."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    buf = _WS.get(dev)
    if buf is None or buf.numel() < nbytes:
        _WS.pop(dev, None)
        buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
        assert buf.data_ptr() % 256 == 0
        _WS[dev] = buf
    return _fill(buf)


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            assert t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors"


# --------------------------------------------------------------------- S0
def wa_prompt_select(e_cur: torch.Tensor, e_chunks: torch.Tensor, stream=None) -> torch.Tensor:
    _need_cuda(e_cur, e_chunks)
    out = _empty(1, torch.int32, e_cur.device)
    _check("wa_prompt_select", lib.wa_prompt_select(_p(e_cur), _p(e_chunks), e_chunks.shape[0],
                                                    e_chunks.shape[1], _p(out), _stream(stream)))
    return out


# --------------------------------------------------------------------- S1
def wa_page_score(q, k_pool, cand_pages, K_p: int, B: int = 64, want_blockmean: bool = False,
                  stream=None):
    _need_cuda(q, k_pool, cand_pages)
    Nq, H, d = q.shape
    P_, T_p = k_pool.shape[0], k_pool.shape[1]
    n_c = cand_pages.numel()
    alpha = _empty(n_c, torch.float64, q.device)
    sel = _empty(K_p, torch.int32, q.device)
    kbm = _empty((n_c, T_p // B, H, d), torch.float64, q.device) if want_blockmean else None
    nbytes = lib.wa_page_score_workspace_size(Nq, H, d, n_c, T_p, B)
    ws = workspace(nbytes, q.device)
    _check("wa_page_score", lib.wa_page_score(
        _p(q), Nq, H, d, _p(k_pool), P_, T_p, _p(cand_pages), n_c, K_p, B, dtype_code(q),
        _p(alpha), _p(sel), _p(kbm), _p(ws), nbytes, _stream(stream)))
    return alpha, sel, kbm


# --------------------------------------------------------------------- S2
def wa_gather_pages(k_pool, v_pool, sel, stream=None, out=None):
    """K_active, V_active = the selected pool pages, concatenated in `sel` order
    (``out``: optional preallocated (k_act, v_act))."""
    _need_cuda(k_pool, v_pool, sel)
    P_, T_p, H, d = k_pool.shape
    K_p = sel.numel()
    if out is None:
        k_act = _empty((K_p * T_p, H, d), k_pool.dtype, k_pool.device)
        v_act = _empty((K_p * T_p, H, d), k_pool.dtype, k_pool.device)
    else:
        k_act, v_act = out
        _need_cuda(k_act, v_act)
        assert k_act.shape == (K_p * T_p, H, d) and v_act.shape == k_act.shape
        assert k_act.dtype == k_pool.dtype and v_act.dtype == k_pool.dtype
    _check("wa_gather_pages", lib.wa_gather_pages(
        _p(k_pool), _p(v_pool), P_, T_p, H, d, _p(sel), K_p, dtype_code(k_pool), _p(k_act),
        _p(v_act), _stream(stream)))
    return k_act, v_act


# --------------------------------------------------------------------- token order
def wa_cube_order(T: int, H_l: int, W_l: int, C_t: int, C_h: int, C_w: int) -> torch.Tensor:
    """Cube-tile token order (host, int32 CPU tensor): element n is the raster index
    of the token at cube-order position n."""
    perm = torch.empty(T * H_l * W_l, dtype=torch.int32)
    _check("wa_cube_order", lib.wa_cube_order(T, H_l, W_l, C_t, C_h, C_w, _p(perm)))
    return perm


def wa_permute_rows(src, perm, inverse: bool = False, out=None, stream=None):
    """Rows of ``src`` (first dimension) permuted on the device: out[n] = src[perm[n]],
    or out[perm[n]] = src[n] with ``inverse``; ``perm`` a device int32 permutation."""
    _need_cuda(src, perm)
    assert perm.dtype == torch.int32 and perm.numel() == src.shape[0]
    if out is None:
        out = _empty(src.shape, src.dtype, src.device)
    else:
        _need_cuda(out)
        assert out.shape == src.shape and out.dtype == src.dtype
    row_bytes = src[0].numel() * src.element_size()
    _check("wa_permute_rows", lib.wa_permute_rows(
        _p(src), _p(out), _p(perm), src.shape[0], row_bytes, 1 if inverse else 0, _stream(stream)))
    return out


# --------------------------------------------------------------------- pool
def wa_pool_index(k_pool, pages, B: int = 64, page_index=None, stream=None):
    """Float64 block sums [P][T_p/B][H][d] of the given pool pages (others untouched)."""
    _need_cuda(k_pool, pages, page_index)
    P_, T_p, H, d = k_pool.shape
    if page_index is None:
        page_index = torch.zeros((P_, T_p // B, H, d), dtype=torch.float64, device=k_pool.device)
    _check("wa_pool_index", lib.wa_pool_index(_p(k_pool), P_, T_p, H, d, B, dtype_code(k_pool),
                                              _p(pages), pages.numel(), _p(page_index),
                                              _stream(stream)))
    return page_index


def wa_pool_append(k_pool, v_pool, k_new, v_new, token_offset: int, page_index=None, B: int = 64,
                   stream=None):
    """Write new K/V rows into the pool's flat token space (and refresh the index)."""
    _need_cuda(k_pool, v_pool, k_new, v_new, page_index)
    P_, T_p, H, d = k_pool.shape
    _check("wa_pool_append", lib.wa_pool_append(
        _p(k_pool), _p(v_pool), P_, T_p, H, d, dtype_code(k_pool), _p(k_new), _p(v_new),
        k_new.shape[0], int(token_offset), _p(page_index), B, _stream(stream)))


# --------------------------------------------------------------------- S3
def wa_block_select(q, tau, B: int = 64, k_act=None, k_blockmean=None, L: Optional[int] = None,
                    stream=None):
    _need_cuda(q, tau, k_act, k_blockmean)
    Nq, H, d = q.shape
    if L is None:
        L = k_act.shape[0] if k_act is not None else k_blockmean.shape[0] * B
    n_qb, n_kb = -(-Nq // B), -(-L // B)
    W = -(-n_kb // 32)
    idx = _empty((H, n_qb, n_kb), torch.int32, q.device)
    cnt = _empty((H, n_qb), torch.int32, q.device)
    mask = _empty((H, n_qb, W), torch.int32, q.device)
    nbytes = lib.wa_block_select_workspace_size(Nq, H, d, L, B)
    ws = workspace(nbytes, q.device)
    _check("wa_block_select", lib.wa_block_select(
        _p(q), Nq, H, d, _p(k_act), _p(k_blockmean), L, B, dtype_code(q), _p(tau), _p(idx),
        _p(cnt), _p(mask), _p(ws), nbytes, _stream(stream)))
    return idx, cnt, mask


# --------------------------------------------------------------------- S4a
def wa_linear_project(k_act, v_act, e_k, e_v, stream=None):
    """K~ = E_K^T K, V~ = E_V^T V; e_k / e_v [L][r] (shared) or [H][L][r] (one per head)."""
    _need_cuda(k_act, v_act, e_k, e_v)
    L, H, d = k_act.shape
    r = e_k.shape[-1]
    if e_k.dim() == 3:
        k_til = _empty((r, H, d), k_act.dtype, k_act.device)
        v_til = _empty((r, H, d), k_act.dtype, k_act.device)
        dt = dtype_code(k_act)
        nbytes = lib.wa_linear_project_workspace_size(L, H, d, r, dt)
        ws = workspace(nbytes, k_act.device)
        _check("wa_linear_project_heads", lib.wa_linear_project_heads(
            _p(k_act), _p(v_act), _p(e_k), _p(e_v), L, H, d, r, dt, L * r, _p(k_til), _p(v_til),
            _p(ws), nbytes, _stream(stream)))
        return k_til, v_til
    k_til = _empty((r, H, d), k_act.dtype, k_act.device)
    v_til = _empty((r, H, d), k_act.dtype, k_act.device)
    dt = dtype_code(k_act)
    nbytes = lib.wa_linear_project_workspace_size(L, H, d, r, dt)
    ws = workspace(nbytes, k_act.device)
    _check("wa_linear_project", lib.wa_linear_project(
        _p(k_act), _p(v_act), _p(e_k), _p(e_v), L, H, d, r, dt, _p(k_til), _p(v_til), _p(ws),
        nbytes, _stream(stream)))
    return k_til, v_til


def wa_linear_project_noalloc(k_act, v_act, e_k, e_v, stream=None):
    """The projection without a workspace: the library keeps the split partials in
    its own fixed device array (see include/wa.h).  Outputs are new tensors here;
    the C call itself allocates nothing."""
    _need_cuda(k_act, v_act, e_k, e_v)
    L, H, d = k_act.shape
    r = e_k.shape[1]
    k_til = _empty((r, H, d), k_act.dtype, k_act.device)
    v_til = _empty((r, H, d), k_act.dtype, k_act.device)
    _check("wa_linear_project_noalloc", lib.wa_linear_project_noalloc(
        _p(k_act), _p(v_act), _p(e_k), _p(e_v), L, H, d, r, dtype_code(k_act), _p(k_til),
        _p(v_til), _stream(stream)))
    return k_til, v_til


# --------------------------------------------------------------------- S4b+S5+S6
def wa_hsa_attention(q, k_act, v_act, blk_mask, k_til, v_til, gate, B: int = 64,
                     want_branches: bool = False, stream=None, gate_lin=None):
    """out = sigmoid(gate) O_sp + (1 - sigmoid(gate)) O_lin, or with ``gate_lin``
    sigmoid(gate) O_sp + sigmoid(gate_lin) O_lin (wa_hsa_attention_gated2)."""
    _need_cuda(q, k_act, v_act, blk_mask, k_til, v_til, gate, gate_lin)
    Nq, H, d = q.shape
    L = k_act.shape[0]
    r = k_til.shape[0]
    dt = dtype_code(q)
    out = _empty(q.shape, q.dtype, q.device)
    o_sp = _empty(q.shape, torch.float32, q.device) if want_branches else None
    o_lin = _empty(q.shape, torch.float32, q.device) if want_branches else None
    nbytes = lib.wa_hsa_attention_workspace_size(Nq, H, d, L, B, r, dt)
    ws = workspace(nbytes, q.device)
    if gate_lin is None:
        _check("wa_hsa_attention", lib.wa_hsa_attention(
            _p(q), Nq, H, d, _p(k_act), _p(v_act), L, B, _p(blk_mask), _p(k_til), _p(v_til), r,
            _p(gate), dt, _p(out), _p(o_sp), _p(o_lin), _p(ws), nbytes, _stream(stream)))
    else:
        _check("wa_hsa_attention_gated2", lib.wa_hsa_attention_gated2(
            _p(q), Nq, H, d, _p(k_act), _p(v_act), L, B, _p(blk_mask), _p(k_til), _p(v_til), r,
            _p(gate), _p(gate_lin), dt, _p(out), _p(o_sp), _p(o_lin), _p(ws), nbytes,
            _stream(stream)))
    return (out, o_sp, o_lin) if want_branches else out


# --------------------------------------------------------------------- step
class HSAStep:
    """A prepared decode step: the argument block, outputs and workspace are built
    once; ``__call__`` is a single wa_hsa_step launch sequence on the stream."""

    def __init__(self, q, k_pool, v_pool, chunk_pages, e_k, e_v, tau, gate, K_p: int = 4,
                 B: int = 64, e_cur=None, e_chunks=None, fused_gather: bool = True,
                 keep_intermediates: bool = False, out=None, page_index=None, gate_lin=None,
                 k_cur=None, v_cur=None, B_inter: int = 0):
        _need_cuda(q, k_pool, v_pool, chunk_pages, e_k, e_v, tau, gate, e_cur, e_chunks, gate_lin,
                   k_cur, v_cur)
        Nq, H, d = q.shape
        P_, T_p = k_pool.shape[0], k_pool.shape[1]
        if chunk_pages.dim() == 1:
            chunk_pages = chunk_pages.reshape(1, -1)
        n_chunks, n_c = chunk_pages.shape
        r = e_k.shape[-1]
        L = K_p * T_p
        n_qb, n_kb = -(-Nq // B), -(-(L + (Nq if k_cur is not None else 0)) // B)
        W = -(-n_kb // 32)
        dev = q.device
        self.out = out if out is not None else _empty(q.shape, q.dtype, q.device)
        self._keep = [q, k_pool, v_pool, chunk_pages, e_k, e_v, tau, gate, e_cur, e_chunks]
        a = StepArgs()
        a.e_cur, a.e_chunks = _p(e_cur), _p(e_chunks)
        a.n_chunks = n_chunks if e_cur is not None else 0
        a.D = e_cur.numel() if e_cur is not None else 0
        a.chunk_pages, a.n_c = _p(chunk_pages), n_c
        a.q, a.Nq, a.H, a.d = _p(q), Nq, H, d
        a.k_pool, a.v_pool, a.n_pool_pages, a.T_p = _p(k_pool), _p(v_pool), P_, T_p
        a.K_p, a.B, a.r = K_p, B, r
        a.e_k, a.e_v, a.tau, a.gate = _p(e_k), _p(e_v), _p(tau), _p(gate)
        a.dtype, a.fused_gather = dtype_code(q), int(bool(fused_gather))
        a.out = _p(self.out)
        a.page_index = _p(page_index)
        a.gate_lin = _p(gate_lin)
        a.k_cur, a.v_cur = _p(k_cur), _p(v_cur)
        a.B_inter = int(B_inter)
        a.e_head_stride = L * r if e_k.dim() == 3 else 0
        self._keep += [page_index, gate_lin, k_cur, v_cur]
        self.inter = {}
        if keep_intermediates:
            self.inter = dict(
                chunk=_empty(1, torch.int32, dev),
                alpha=_empty(n_c, torch.float64, dev),
                sel=_empty(K_p, torch.int32, dev),
                blk_mask=_empty((H, n_qb, W), torch.int32, dev),
                k_til=_empty((r, H, d), q.dtype, dev),
                v_til=_empty((r, H, d), q.dtype, dev))
            a.chunk_out = _p(self.inter["chunk"])
            a.alpha_out = _p(self.inter["alpha"])
            a.sel_out = _p(self.inter["sel"])
            a.blk_mask_out = _p(self.inter["blk_mask"])
            a.k_til_out = _p(self.inter["k_til"])
            a.v_til_out = _p(self.inter["v_til"])
        self.args = a
        nbytes = lib.wa_hsa_step_workspace_size(ctypes.byref(a))
        if nbytes == 0:
            # a zero size means validation failed: surface the reason
            _check("wa_hsa_step_workspace_size", lib.wa_hsa_step(ctypes.byref(a), None, 0, None))
        self.nbytes = nbytes
        self.ws = _empty(nbytes, torch.uint8, dev)
        assert self.ws.data_ptr() % 256 == 0

    def __call__(self, stream=None):
        _check("wa_hsa_step", lib.wa_hsa_step(ctypes.byref(self.args), _p(self.ws), self.nbytes,
                                              _stream(stream)))
        return self.out


def wa_hsa_step(q, k_pool, v_pool, chunk_pages, e_k, e_v, tau, gate, K_p: int = 4, B: int = 64,
                e_cur=None, e_chunks=None, fused_gather: bool = True, keep_intermediates: bool = False,
                stream=None, page_index=None, gate_lin=None, k_cur=None, v_cur=None, B_inter: int = 0):
    """One HSA decode step; returns ``out`` (and the intermediates when asked)."""
    st = HSAStep(q, k_pool, v_pool, chunk_pages, e_k, e_v, tau, gate, K_p, B, e_cur, e_chunks,
                 fused_gather, keep_intermediates, page_index=page_index, gate_lin=gate_lin,
                 k_cur=k_cur, v_cur=v_cur, B_inter=B_inter)
    out = st(stream)
    return (out, st.inter) if keep_intermediates else out


def wa_set_wait_limit_ns(limit_ns: int) -> None:
    """Bound of every mbarrier wait in the kernels launched from now on (ns)."""
    _check("wa_set_wait_limit_ns", lib.wa_set_wait_limit_ns(int(limit_ns)))


def wa_get_wait_limit_ns() -> int:
    return int(lib.wa_get_wait_limit_ns())


def wa_check_bounded_wait(limit_ns: int, stream=None) -> torch.Tensor:
    """Run the bounded-wait self-test kernel (a wait nobody ends); returns a device
    uint64 tensor (as int64) holding the time the wait took, in ns."""
    el = _empty(1, torch.int64, torch.device("cuda", torch.cuda.current_device()))
    _check("wa_check_bounded_wait", lib.wa_check_bounded_wait(int(limit_ns), _p(el), _stream(stream)))
    return el


def wa_device_error(stream=None) -> int:
    """Synchronise, read and clear the device error word; returns its WA_DEVERR_* bits."""
    flags = ctypes.c_uint32(0)
    lib.wa_device_error(_stream(stream), ctypes.byref(flags))
    return int(flags.value)


# --------------------------------------------------------------------- L1 <-> L2 tiering
class TierStats(ctypes.Structure):
    """Mirror of ``wa_tier_stats``."""
    _fields_ = [(n, ctypes.c_longlong) for n in
                ("hits", "misses", "prefetch_hits", "prefetches", "evictions", "writebacks",
                 "bytes_h2d", "bytes_d2h")]


class Tier:
    """A page tier over a device slot pool and pinned host pages (see wa_tier_* in
    include/wa.h).  ``host_k``/``host_v`` are pinned CPU tensors [n_pages][...] and
    ``slot_k``/``slot_v`` device tensors [n_slots][...] of the same page shape; with
    none of them the tier only keeps the books (``n_pages``, ``n_slots`` given)."""

    def __init__(self, host_k=None, host_v=None, slot_k=None, slot_v=None, n_pages=None,
                 n_slots=None, page_bytes=None):
        bufs = (host_k, host_v, slot_k, slot_v)
        self.books = all(b is None for b in bufs)
        if self.books:
            self._keep = ()
            ptrs = (None,) * 4
        else:
            assert host_k.is_pinned() and host_v.is_pinned()
            _need_cuda(slot_k, slot_v)
            n_pages, n_slots = host_k.shape[0], slot_k.shape[0]
            page_bytes = host_k[0].numel() * host_k.element_size()
            assert slot_k[0].numel() * slot_k.element_size() == page_bytes
            for b in bufs:
                assert b.is_contiguous()
            self._keep = bufs
            ptrs = tuple(_p(b) for b in bufs)
        self.n_pages, self.n_slots = n_pages, n_slots
        h = ctypes.c_void_p()
        _check("wa_tier_create", lib.wa_tier_create(n_pages, n_slots, page_bytes or 1, *ptrs,
                                                    ctypes.byref(h)))
        self.h = h

    def _st(self, stream):
        return None if self.books else _stream(stream)

    def ensure(self, pages, stream=None):
        ids = (ctypes.c_int32 * len(pages))(*[int(p) for p in pages])
        out = (ctypes.c_int32 * len(pages))()
        st = self._st(stream)
        _check("wa_tier_ensure", lib.wa_tier_ensure(self.h, ids, len(pages), out, st))
        return list(out)

    def release(self, stream=None):
        _check("wa_tier_release", lib.wa_tier_release(self.h, self._st(stream)))

    def prefetch(self, pages) -> int:
        ids = (ctypes.c_int32 * len(pages))(*[int(p) for p in pages])
        n = ctypes.c_int(0)
        _check("wa_tier_prefetch", lib.wa_tier_prefetch(self.h, ids, len(pages), ctypes.byref(n)))
        return int(n.value)

    def mark_dirty(self, page: int):
        _check("wa_tier_mark_dirty", lib.wa_tier_mark_dirty(self.h, int(page)))

    def flush(self, stream=None):
        _check("wa_tier_flush", lib.wa_tier_flush(self.h, self._st(stream)))

    def slot_of(self, page: int) -> int:
        s = ctypes.c_int32(0)
        _check("wa_tier_slot_of", lib.wa_tier_slot_of(self.h, int(page), ctypes.byref(s)))
        return int(s.value)

    def stats(self) -> dict:
        st = TierStats()
        _check("wa_tier_get_stats", lib.wa_tier_get_stats(self.h, ctypes.byref(st)))
        return {n: int(getattr(st, n)) for n, _ in TierStats._fields_}

    def close(self):
        if getattr(self, "h", None):
            lib.wa_tier_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# --------------------------------------------------------------------- host-buffer pipeline
class HSAPipeline:
    """Steps over host buffers with uploads and downloads overlapping the compute
    (wa_pipe_* in include/wa.h).  Built on a prepared HSAStep, whose q, gate and out
    are the first device set; the second set is allocated here."""

    def __init__(self, step: "HSAStep", q, gate, stream=None):
        self.step = step
        self.q1, self.g1 = torch.empty_like(q), torch.empty_like(gate)
        self.o1 = torch.empty_like(step.out)
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        h = ctypes.c_void_p()
        _check("wa_pipe_create", lib.wa_pipe_create(ctypes.byref(step.args), _p(self.q1), _p(self.g1),
                                                    _p(self.o1), _p(step.ws), step.nbytes,
                                                    _stream(self.stream), ctypes.byref(h)))
        self.h = h

    def begin(self):
        _check("wa_pipe_begin", lib.wa_pipe_begin(self.h))

    def submit(self, q_host, gate_host, out_host):
        for t in (q_host, gate_host, out_host):
            assert t.device.type == "cpu" and t.is_contiguous()
        _check("wa_pipe_submit", lib.wa_pipe_submit(self.h, ctypes.c_void_p(q_host.data_ptr()),
                                                    ctypes.c_void_p(gate_host.data_ptr()),
                                                    ctypes.c_void_p(out_host.data_ptr())))

    def end(self):
        _check("wa_pipe_end", lib.wa_pipe_end(self.h))

    def sync(self):
        _check("wa_pipe_sync", lib.wa_pipe_sync(self.h))

    def close(self):
        if getattr(self, "h", None):
            lib.wa_pipe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
