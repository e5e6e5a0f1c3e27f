"""Comparison of the CUDA path with the float64 oracle.

Tolerances (floating point) -- the contract's, plus a tighter internal one:
  scores: |I_gpu - I_ora| <= 1e-2 * max(|I_ora|, rms(I_ora row))   (relative, with
          the row rms as the floor where signed head weights make I cross 0)
  top-k:  (1) the oracle's selection rerun on the GPU's own fp32 scores equals
              the GPU's indices bit for bit;
          (2) against the oracle's own selection, the symmetric difference holds
              only positions whose oracle score is within 1e-3 * max(|tau|, rms)
              of the oracle's k-th score tau.
  MLA:    on the GPU's own indices, bf16: |d| <= 2e-2 + 1e-2 |ref|, and the
          tighter |d| <= 1e-2 * rms(ref) + 2e-2 |ref|; fp32: |d| <= 1e-4 (1 + |ref|).
"""
from __future__ import annotations

import numpy as np

from oracle import dsa_ref as R

SCORE_RTOL = 1e-2
TIE_BAND = 1e-3


def rms(x):
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def check_scores(gpu_row: np.ndarray, ora_row: np.ndarray, where=""):
    g = np.asarray(gpu_row, dtype=np.float64)
    o = np.asarray(ora_row, dtype=np.float64)
    assert g.shape == o.shape, where
    assert np.isfinite(g).all(), f"non-finite GPU scores {where}"
    tol = SCORE_RTOL * np.maximum(np.abs(o), rms(o))
    bad = np.abs(g - o) > tol
    assert not bad.any(), (f"scores {where}: {bad.sum()} of {g.size} outside tolerance; worst "
                           f"|d|={np.abs(g - o).max():.3e} at {int(np.argmax(np.abs(g - o)))}")


def check_topk(gpu_idx: np.ndarray, gpu_scores_row: np.ndarray, ora_scores_row: np.ndarray,
               k: int, where=""):
    gi = np.asarray(gpu_idx, dtype=np.int64)
    # (1) bit-exact against the oracle's rule applied to the GPU's own scores
    rerun = R.topk_row(np.asarray(gpu_scores_row, dtype=np.float32).astype(np.float64), k)
    assert np.array_equal(gi, rerun), f"top-k {where}: differs from oracle rule on GPU scores"
    # (2) against the oracle's own selection, only tie-band differences
    own = R.topk_row(ora_scores_row, k)
    a, b = set(gi[gi >= 0].tolist()), set(own[own >= 0].tolist())
    diff = a ^ b
    if diff:
        tau = R.kth_score(ora_scores_row, k)
        band = TIE_BAND * max(abs(tau), rms(ora_scores_row))
        far = [s for s in diff if abs(ora_scores_row[s] - tau) > band]
        assert not far, f"top-k {where}: {len(far)} differences outside the tie band"
    return len(diff)


def check_mla(gpu_out: np.ndarray, gpu_lse: np.ndarray, ora_out: np.ndarray, ora_lse: np.ndarray,
              bf16: bool, where=""):
    g = np.asarray(gpu_out, dtype=np.float64)
    o = np.asarray(ora_out, dtype=np.float64)
    d = np.abs(g - o)
    if bf16:
        assert (d <= 2e-2 + 1e-2 * np.abs(o)).all(), f"MLA {where}: contract tolerance, max {d.max():.3e}"
        tight = 1e-2 * rms(o) + 2e-2 * np.abs(o)
        assert (d <= tight).all(), f"MLA {where}: tight tolerance, max {d.max():.3e} rms {rms(o):.3e}"
        lt = 1e-3 * (1 + np.abs(ora_lse))
    else:
        assert (d <= 1e-4 * (1 + np.abs(o))).all(), f"MLA {where}: fp32 tolerance, max {d.max():.3e}"
        lt = 1e-5 * (1 + np.abs(ora_lse))
    gl = np.asarray(gpu_lse, dtype=np.float64)
    fin = np.isfinite(ora_lse)
    assert np.array_equal(np.isfinite(gl), fin), f"lse {where}: finiteness differs"
    assert (np.abs(gl[fin] - ora_lse[fin]) <= lt[fin]).all(), f"lse {where}"


def to_np(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def check_rows(inp: dict, rows, scores, idx, out, lse, check_score=True):
    """Full three-stage parity on the listed rows (host arrays from the GPU)."""
    k = int(inp["topk"])
    bf16 = inp["mla_dtype"] == "bf16"
    ndiff = 0
    for t in rows:
        klen = int(inp["row_klen"][t])
        ora_sc = R.row_scores(inp, t)
        if scores is not None:
            g_sc = scores[t, :klen]
            if check_score:
                check_scores(g_sc, ora_sc, f"row {t}")
            ndiff += check_topk(idx[t], g_sc, ora_sc, k, f"row {t}")
        o, l = R.row_attention(inp, t, idx[t])
        check_mla(out[t], lse[t], o, l, bf16, f"row {t}")
    return ndiff
