"""Comparison rules between the CUDA path and the fp64 oracle.

  top-k   where the oracle's k-th / (k+1)-th logit gap exceeds 1e-5 relative,
          the GPU's selected set must equal the oracle's and its order must
          follow the oracle's logits except among entries within 1e-5 of each
          other; closer calls are valid either way, and the oracle then
          recomputes that token with the GPU's selection
  G1      fp32-output mode: per token max|y - y_oracle| / max|y_oracle| <= 2e-3
  G2      bf16-output mode: bit-equal to round-to-nearest-even of the same
          call's fp32 output
"""
from __future__ import annotations

import numpy as np

TOPK_REL_GAP = 1e-5
G1_TOL = 2e-3


def rel_gap(a: float, b: float) -> float:
    den = max(abs(a), abs(b))
    return abs(a - b) / den if den > 0 else 0.0


def check_topk_row(l: np.ndarray, gpu_idx: np.ndarray, k: int):
    """-> (decisive, problems): decisive = the k/k+1 gap exceeds 1e-5."""
    E = l.size
    order = sorted(range(E), key=lambda e: (-l[e], e))
    problems = []
    decisive = k == E or rel_gap(l[order[k - 1]], l[order[k]]) > TOPK_REL_GAP
    gi = [int(v) for v in gpu_idx]
    if len(set(gi)) != k or min(gi) < 0 or max(gi) >= E:
        problems.append(f"invalid selection {gi}")
        return decisive, problems
    if decisive and set(gi) != set(order[:k]):
        problems.append(f"set differs: gpu {sorted(gi)} oracle {sorted(order[:k])}")
    for a, b in zip(gi, gi[1:]):
        if l[a] < l[b] and rel_gap(l[a], l[b]) > TOPK_REL_GAP:
            problems.append(f"order: {a} ({l[a]}) before {b} ({l[b]})")
        if l[a] == l[b] and a > b:
            problems.append(f"tie order: {a} before {b}")
    # every non-selected expert must not beat the weakest selected one decisively
    weakest = min(l[e] for e in gi)
    sel = set(gi)
    for e in range(E):
        if e not in sel and l[e] > weakest and rel_gap(l[e], weakest) > TOPK_REL_GAP:
            problems.append(f"missed {e} ({l[e]} > {weakest})")
            break
    return decisive, problems


def g1_error(y: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per-token max|y - ref| / max|ref|."""
    y = np.asarray(y, dtype=np.float64)
    den = np.abs(ref).max(axis=-1)
    den = np.where(den > 0, den, 1.0)
    return np.abs(y - ref).max(axis=-1) / den


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
