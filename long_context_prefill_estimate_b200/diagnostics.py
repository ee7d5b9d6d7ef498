"""Block-selection accuracy of the round-robin estimate against exact attention mass.

RRAttention (paperpeel.com/paper/2602.05853) validates its estimate by comparing the
selected blocks with the ones full attention would pick (Sec. 4.3 "Block Selection
Accuracy", details in its Appendix D, which the page does not carry).  Here the reference
is the same estimator run with stride S = 1: every query is sampled and keys are not
pooled, so its block scores are the exact mean causal attention mass of each block.  Both
score sets go through the same Top-tau selection, and for each head we report

    precision = |RR and exact| / |RR|,   recall = |RR and exact| / |exact|,
    F1, and captured mass = sum of exact block mass over the RR-selected blocks / rows,

the last one being the attention mass the sparse prefill keeps (the quantity the paper's
Sec. 2.1 selection objective is about).  All computation runs in the library's kernels;
this module only compares the two CSR masks on the host.

    python -m long_context_prefill_estimate_b200.diagnostics --workload 1 --L 16384
"""
from __future__ import annotations

import argparse
import json
import sys
from typing import Dict

import numpy as np
import torch

from . import estimate, select


def csr_to_mask(row_ptr: np.ndarray, col_idx: np.ndarray, H: int, Nb: int) -> np.ndarray:
    """Boolean [H][Nb][Nb] block mask from per-head CSR block lists."""
    mask = np.zeros((H * Nb, Nb), dtype=bool)
    counts = np.diff(row_ptr)
    rows = np.repeat(np.arange(H * Nb), counts)
    mask[rows, col_idx[: row_ptr[-1]]] = True
    return mask.reshape(H, Nb, Nb)


def mask_metrics(sel: np.ndarray, ref: np.ndarray, ref_mass: np.ndarray) -> Dict[str, np.ndarray]:
    """Per-head precision, recall, F1 of `sel` against `ref`, and the share of `ref_mass`
    (rows summing to 1) that `sel` keeps, averaged over the query blocks."""
    H = sel.shape[0]
    inter = (sel & ref).reshape(H, -1).sum(1).astype(np.float64)
    n_sel = sel.reshape(H, -1).sum(1).astype(np.float64)
    n_ref = ref.reshape(H, -1).sum(1).astype(np.float64)
    precision = np.divide(inter, n_sel, out=np.ones(H), where=n_sel > 0)
    recall = np.divide(inter, n_ref, out=np.ones(H), where=n_ref > 0)
    f1 = np.divide(2 * precision * recall, precision + recall, out=np.zeros(H),
                   where=(precision + recall) > 0)
    captured = (ref_mass * sel).sum(-1).mean(-1)
    return {"precision": precision, "recall": recall, "f1": f1, "captured_mass": captured}


def classify_masks(rows_a, rows_b, diag_b, A_b, A_a, cum_tol: float = 1e-4):
    """Compare two Top-tau selections of the same rows, row by row.

    rows_a, rows_b: per-row lists of selected blocks (ascending) of side a (e.g. the GPU) and
    side b (a reference selecting from its own scores A_b); row r is query block r % Nb of a
    head (the lists start at a head boundary).  diag_b: side b's per-row selection record
    [k*, cum_(k*-1), cum_(k*), tau*T, gap].  A_a, A_b: the two sides' scores of the same
    rows, [rows][Nb].  A mismatching row is
      boundary          if side b's cumulative sum just before or at the cut is within
                        cum_tol of tau*T;
      near tie          if both keep the same number of blocks and every block they disagree
                        on has a side-b score within 2*delta of side b's cut score, delta the
                        row's largest score difference (a score error of delta can swap only
                        such blocks);
      sum within error  if the counts differ and a cumulative sum at the cut is within
                        2*n*delta of tau*T (n causal blocks in the row);
    and unexplained otherwise.  Returns (counts, unexplained [(row, a, b), ...])."""
    Nb = np.shape(A_b)[-1]
    diag_b = np.asarray(diag_b)
    bnd = (np.abs(diag_b[:, 1] - diag_b[:, 3]) < cum_tol) | (np.abs(diag_b[:, 2] - diag_b[:, 3]) < cum_tol)
    out = {"rows": len(rows_b), "boundary_rows": int(bnd.sum()), "mismatch_rows": 0,
           "mismatch_boundary": 0, "near_tie_swaps": 0, "sum_within_error": 0}
    unexplained = []
    for r, (a, b) in enumerate(zip(rows_a, rows_b)):
        a, b = list(a), list(b)
        if a == b:
            continue
        out["mismatch_rows"] += 1
        if bnd[r]:
            out["mismatch_boundary"] += 1
            continue
        n = r % Nb + 1
        sb = np.asarray(A_b[r], np.float64)
        delta = float(np.abs(np.asarray(A_a[r], np.float64)[:n] - sb[:n]).max())
        cut = float(sb[b].min())
        diff = set(a) ^ set(b)
        if len(a) == len(b) and all(abs(sb[J] - cut) <= 2 * delta for J in diff):
            out["near_tie_swaps"] += 1
            continue
        _, cb, ca, thr, _ = diag_b[r]
        if len(a) != len(b) and min(abs(cb - thr), abs(ca - thr)) <= 2 * n * delta:
            out["sum_within_error"] += 1
            continue
        unexplained.append((r, a, b))
    return out, unexplained


def csr_rows(row_ptr, col_idx):
    """Per-row lists of a CSR."""
    rp = np.asarray(row_ptr)
    ci = np.asarray(col_idx)
    return [ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)]


def selection_accuracy(Q: torch.Tensor, K: torch.Tensor, S: int, B: int, tau: float,
                       protect_last: bool = True, strategy: str = "head",
                       layer: int = 0) -> Dict[str, object]:
    """Compare the RR selection (stride S) with the exact-mass selection (stride 1)."""
    H, L, _ = Q.shape
    Nb = L // B
    A_rr = estimate(Q, K, S, B, strategy=strategy, layer=layer)
    A_exact = estimate(Q, K, 1, B)
    rp_rr, ci_rr, _ = select(A_rr, tau, protect_last)
    rp_ex, ci_ex, _ = select(A_exact, tau, protect_last)
    torch.cuda.synchronize()
    sel = csr_to_mask(rp_rr.cpu().numpy(), ci_rr.cpu().numpy(), H, Nb)
    ref = csr_to_mask(rp_ex.cpu().numpy(), ci_ex.cpu().numpy(), H, Nb)
    m = mask_metrics(sel, ref, A_exact.cpu().numpy().astype(np.float64))
    causal = H * Nb * (Nb + 1) / 2
    return {
        "per_head": {k: v.tolist() for k, v in m.items()},
        "mean": {k: float(np.mean(v)) for k, v in m.items()},
        "density_rr": float(sel.sum() / causal),
        "density_exact": float(ref.sum() / causal),
    }


def main(argv=None):
    import workloads

    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--L", type=int, default=16384)
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--strategy", default="head", choices=["head", "none", "layer", "hybrid"])
    ap.add_argument("--S", type=int, default=None)
    a = ap.parse_args(argv)
    w = workloads.get(a.workload, L=a.L)
    t = workloads.generate(w)
    d = {k: v.cuda() for k, v in t.items()}
    res = selection_accuracy(d["Q"], d["K"], a.S or w.S, w.B, a.tau or w.tau, strategy=a.strategy)
    res["config"] = {"workload": w.name, "L": w.L, "S": a.S or w.S, "B": w.B, "tau": a.tau or w.tau,
                     "strategy": a.strategy}
    del res["per_head"]
    print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
