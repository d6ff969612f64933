"""Shared helpers of the GPU parity tests: tolerances, mask conversion, logging."""
import math

import numpy as np
import torch

# Tolerances against the float64 oracle: bf16 inputs -> max-abs 2e-2 and relative
# Frobenius 5e-3; fp32 inputs -> 1e-4 for both.
TOL = {"bf16": (2e-2, 5e-3), "f32": (1e-4, 1e-4)}
# Rows whose oracle margin is below MARGIN are near ties: they are counted and
# logged.  The GPU takes every index decision in float64 as the oracle does, from the
# same input bits, so only a margin at the scale of float64 rounding of the sums
# (below MARGIN_F64) may decide a row differently; every other row must match bit
# for bit, near tie or not.
MARGIN = 1e-5
MARGIN_F64 = 1e-12


def to64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def err_stats(got, ref):
    g, r = to64(got), to64(ref)
    d = np.abs(g - r)
    maxabs = float(d.max()) if d.size else 0.0
    nr = float(np.linalg.norm(r))
    relf = float(np.linalg.norm(g - r)) / nr if nr > 0 else float(np.linalg.norm(g - r))
    return maxabs, relf


def assert_close(got, ref, dtype: str, what: str):
    maxabs, relf = err_stats(got, ref)
    ta, tf = TOL[dtype]
    print(f"[parity] {what}: max-abs {maxabs:.3e} (tol {ta:g}), rel-Frobenius {relf:.3e} (tol {tf:g})")
    assert not math.isnan(maxabs), f"{what}: NaN in output"
    assert maxabs <= ta and relf <= tf, f"{what}: max-abs {maxabs:.3e}, rel-F {relf:.3e}"


def mask_to_sets(mask: torch.Tensor, n_kb: int):
    """[H][n_qb][W] int32 bitmask -> nested lists of sorted block lists."""
    m = mask.cpu().numpy().astype(np.uint32)
    H, n_qb, W = m.shape
    out = []
    for h in range(H):
        row = []
        for i in range(n_qb):
            bits = np.unpackbits(m[h, i].view(np.uint8), bitorder="little")[:n_kb]
            row.append(np.nonzero(bits)[0].tolist())
        out.append(row)
    return out


def compare_selection(gpu_sets, kept, margin, what: str):
    """Rows must match exactly unless the oracle margin is below MARGIN_F64; rows with
    a margin below MARGIN (near ties) are counted and logged whether they match or not."""
    H = len(kept)
    n_rows = n_excused = 0
    bad = []
    for h in range(H):
        for i in range(len(kept[h])):
            n_rows += 1
            if gpu_sets[h][i] != kept[h][i]:
                if margin[h][i] < MARGIN_F64:
                    n_excused += 1
                    print(f"[near-tie] {what}: head {h} block {i} margin {margin[h][i]:.2e}")
                else:
                    bad.append((h, i, margin[h][i], len(gpu_sets[h][i]), len(kept[h][i])))
    n_near = int(sum(1 for h in range(H) for i in range(len(kept[h])) if margin[h][i] < MARGIN))
    print(f"[parity] {what}: {n_rows} rows, {len(bad)} mismatches, {n_excused} excused "
          f"(margin < {MARGIN_F64:g}); {n_near} near ties (margin < {MARGIN:g}) checked bit for bit")
    assert not bad, f"{what}: selection mismatches (h, i, margin, |gpu|, |oracle|): {bad[:5]}"
    return n_excused


def kept_fraction(kept, n_kb):
    return [float(np.mean([len(r) for r in kh])) / n_kb for kh in kept]
