"""Comparison helpers for the GPU parity tests (no arithmetic of the method here)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances.  Block indices: bit-exact, except where the oracle's score at the last
# taken slot and the first left-out candidate differ by less than REL_TIE relative
# (the GPU scores in fp32, the oracle in fp64).  Ineligible blocks carry score -inf.  Attention outputs (bf16 inputs, fp32
# accumulation, bf16 output): max-abs 2e-2 and mean-abs 2e-3 against the fp64 oracle.
REL_TIE = 1e-5
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of bf16 bit patterns (same sign)."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordered(a) - ordered(b))


def forced_set(t: int, topk: int, n_init: int, n_local: int, block: int = 64) -> set:
    cur = t // block
    f = set(range(min(n_init, cur + 1)))
    if n_local > 0:
        f |= set(range(max(cur - n_local + 1, 0), cur + 1))
    return f


def check_row_selection(gpu_row, ora_row, scores, t, topk, n_init, n_local):
    """Returns 'exact', 'tie' (differs only through a near-tie) or an error string."""
    g = [int(x) for x in gpu_row]
    o = [int(x) for x in ora_row]
    if g == o:
        return "exact"
    gs = [x for x in g if x >= 0]
    if g[len(gs):] != [-1] * (len(g) - len(gs)) or sorted(set(gs)) != gs:
        return f"malformed row {g}"
    F = forced_set(t, topk, n_init, n_local)
    if not F <= set(gs):
        return f"forced blocks {sorted(F - set(gs))} missing"
    if len(gs) != len([x for x in o if x >= 0]):
        return f"count {len(gs)} != {len([x for x in o if x >= 0])}"
    cand = [(scores[j], j) for j in range(len(scores)) if np.isfinite(scores[j]) and j not in F and j <= t // 64]
    cand.sort(key=lambda sj: (-sj[0], sj[1]))
    m = topk - len(F)
    if m <= 0 or len(cand) <= m:
        return f"sets differ with no threshold: gpu {gs} oracle {o}"
    sigma, nxt = cand[m - 1][0], cand[m][0]
    if not (sigma - nxt <= REL_TIE * max(abs(sigma), 1e-300)):
        return f"sets differ at a clear gap ({sigma:.9g} vs {nxt:.9g}): gpu {gs} oracle {o}"
    chosen = set(gs) - F
    band = REL_TIE * abs(sigma)  # scores may be negative (logit-sum scoring)
    for s, j in cand:
        if s > sigma + band and j not in chosen:
            return f"block {j} (score {s:.9g}) above the tie band is missing"
        if j in chosen and s < sigma - band:
            return f"block {j} (score {s:.9g}) below the tie band was taken"
    return "tie"


def compare_selection(gpu_idx, ora_idx, ora_scores, positions, p, max_tie_frac=0.02):
    """gpu_idx/ora_idx [B, Hkv, R, topk]; positions [B, R] query positions."""
    B, H, R, _ = ora_idx.shape
    n_tie = 0
    for b in range(B):
        for g in range(H):
            for r in range(R):
                res = check_row_selection(gpu_idx[b, g, r], ora_idx[b, g, r], ora_scores[b, g, r],
                                          int(positions[b, r]), p.topk, p.n_init, p.n_local)
                if res == "tie":
                    n_tie += 1
                elif res != "exact":
                    raise AssertionError(f"selection mismatch at b={b} g={g} row={r} t={positions[b, r]}: {res}")
    assert n_tie <= max(2, max_tie_frac * B * H * R), f"{n_tie} near-tie rows"
    rows_equal = np.all(gpu_idx == ora_idx, axis=-1)  # [B, H, R]
    return rows_equal, n_tie


def compare_attention(o_gpu: np.ndarray, o_ora: np.ndarray, lse_gpu=None, lse_ora=None, mask=None):
    """o_* [..., d] float arrays; mask selects the rows to compare (broadcast over d)."""
    diff = np.abs(o_gpu.astype(np.float64) - o_ora)
    if mask is not None:
        diff = diff[mask]
    assert diff.size > 0
    mx, mean = float(diff.max()), float(diff.mean())
    assert mx <= O_MAX_ABS, f"max abs error {mx}"
    assert mean <= O_MEAN_ABS, f"mean abs error {mean}"
    if lse_gpu is not None:
        dl = np.abs(lse_gpu.astype(np.float64) - lse_ora)
        finite = np.isfinite(lse_ora)
        assert np.all(np.isfinite(lse_gpu)[finite])
        assert float(dl[finite].max()) <= LSE_MAX_ABS, f"lse max abs error {float(dl[finite].max())}"
    return mx, mean


# Gradients of the backward pass: every error source is a bf16 rounding (of P and dS as
# MMA operands, of the forward's O inside D = dO.O, and of the bf16 outputs), 2^-8
# relative to the terms it rounds.  The terms' scale differs by orders of magnitude from
# row to row (a query row that attends to 2 keys has a dq ~ 20x that of one attending to
# a thousand; a key attended by every row has a larger dK than one attended by few), so
# errors are measured against the RMS of their own gradient row (128 values: one (token,
# head) of dq, one key of dK / dV), with a floor of 1e-3 x the tensor's RMS for rows whose
# exact gradient is (nearly) zero.  A row's largest element is ~3 RMS, so the roundings
# leave ~2^-8 x 6 RMS = 2.3e-2 RMS at most and ~2^-8 / 2 RMS on average.  Bars: max 5e-2,
# mean 5e-3 (of the row RMS).
GRAD_MAX_ROW_RMS = 5e-2
GRAD_MEAN_ROW_RMS = 5e-3


def compare_grad(g, ref, what=""):
    """g: GPU gradient (torch, any float dtype); ref: fp64 oracle gradient (numpy); the
    last axis is the row of 128 values.  Returns (max, mean) error over the row RMS."""
    g = g.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), what
    rms_all = float(np.sqrt(np.mean(ref * ref)))
    assert rms_all > 0, what
    row_rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    rel = np.abs(g - ref) / np.maximum(row_rms, 1e-3 * rms_all)
    mx, mean = float(rel.max()), float(rel.mean())
    assert mx <= GRAD_MAX_ROW_RMS, f"{what}: max abs error {mx:.3g} x its row's RMS"
    assert mean <= GRAD_MEAN_ROW_RMS, f"{what}: mean abs error {mean:.3g} x its row's RMS"
    return mx, mean
