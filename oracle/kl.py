"""Plain CPU float64 oracle of the fused chunked KL distillation loss.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this file: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code, table or helper with the CUDA
library; the only thing both sides see is the seeded input arrays.

What it computes is the plain definition, written out without any of the
kernel's blocking or fusion (the pages call the dense, forward-chunked and
fused variants mathematically equivalent: mind-verse.de article, section
"Zwei systemische Optimierungen für Kosteneffizienz", item 2 "Ein
zusammengeführter, chunked KL-Verlust", the three-variant list):

* the student distribution P_S = softmax(z) with z = hidden @ W^T over the full
  vocabulary (the fused variant folds this output projection into the loss,
  same list, "Fused chunked KL" item);
* the teacher distribution P_T is rebuilt as a dense vocabulary row from the
  cached top-K (index, logit) pairs (same list, "Dense KL" item), with
  P_T = softmax(topk_logit / tau) over the K cached entries and zero elsewhere;
* the objective is KL(P_T || P_S) = sum_v P_T(v) log(P_T(v) / P_S(v))
  (llm-wiki study note, section "표준 KD의 손실 함수");
* the batch reduction divides the summed per-token KL by the number of valid
  tokens (the ``reduction='batchmean'`` idiom in the llm-wiki note, section
  "전통적인 KL 손실의 문제", applied to the flattened, masked tokens);
* the gradient w.r.t. the logits is G = (g / N_valid) (P_S - P_T) on valid rows
  and 0 on masked rows; dHidden = G W and dW = G^T hidden.

Readings where the pages are silent (each also listed in the design notes):
  R1 tau divides the teacher logits only; no tau^2 factor.
  R3 P_T is renormalised over the cached entries; the tail is exactly 0.
  R4 the teacher entropy term is kept, so the value is a true KL.
  R5 loss = sum over valid rows / N_valid; N_valid = 0 gives loss 0 and zero grads.
  R6 masked rows add nothing to loss or grads; their lse is still reported.
  R7 a logit of -inf gives P_T = 0 for that entry.  A row with a NaN or +inf
     logit among its in-range entries, or whose in-range logits are all -inf,
     is flagged NONFINITE and treated as masked.
  R8 entries with an index outside [0, V) are dropped before the softmax and
     flagged IDX_RANGE; a row left with no entry is treated as masked.
     Repeated indices are flagged IDX_DUP and their probabilities add up on
     the shared vocabulary entry.
"""
from __future__ import annotations

import dataclasses

import numpy as np

FLAG_IDX_RANGE = 1
FLAG_IDX_DUP = 2
FLAG_NONFINITE = 4


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


@dataclasses.dataclass
class Teacher:
    """Per-row teacher distribution over the cached entries."""
    P: np.ndarray         # [N, K] float64, 0 for dropped or -inf entries
    keep: np.ndarray      # [N, K] bool, entry has an in-range index
    row_ok: np.ndarray    # [N] bool, row usable (finite, at least one entry)
    flags: int


def teacher_distribution(topk_idx: np.ndarray, topk_logit: np.ndarray, V: int, tau: float) -> Teacher:
    """P_T = softmax(topk_logit / tau) over each row's in-range cached entries (R1, R3, R7, R8)."""
    idx = np.asarray(topk_idx, dtype=np.int64)
    x = np.asarray(topk_logit, dtype=np.float64) / float(tau)
    N, K = idx.shape
    flags = 0
    keep = (idx >= 0) & (idx < V)
    if not keep.all():
        flags |= FLAG_IDX_RANGE
    bad_val = keep & (np.isnan(x) | (x == np.inf))
    xk = np.where(keep, x, -np.inf)
    all_neginf = ~np.isfinite(np.where(keep & ~np.isnan(x), xk, -np.inf)).any(axis=1) & keep.any(axis=1)
    nonfinite_row = bad_val.any(axis=1) | all_neginf
    if nonfinite_row.any():
        flags |= FLAG_NONFINITE
    row_ok = keep.any(axis=1) & ~nonfinite_row
    with np.errstate(invalid="ignore", over="ignore"):
        m = np.where(row_ok, np.where(row_ok[:, None], xk, 0.0).max(axis=1), 0.0)
        e = np.where(row_ok[:, None], np.exp(xk - m[:, None]), 0.0)
    P = e / np.where(row_ok, e.sum(axis=1), 1.0)[:, None]
    # repeated in-range indices within a row (dropped entries get distinct negative keys)
    keyed = np.where(keep, idx, -1 - np.arange(K, dtype=np.int64)[None, :])
    keyed.sort(axis=1)
    if (keyed[:, 1:] == keyed[:, :-1]).any():
        flags |= FLAG_IDX_DUP
    return Teacher(P, keep, row_ok, flags)


def _dense_teacher(idx_rows: np.ndarray, P_rows: np.ndarray, keep_rows: np.ndarray, V: int) -> np.ndarray:
    """Scatter-add the cached probabilities into a dense [rows, V] teacher distribution."""
    R = idx_rows.shape[0]
    dense = np.zeros((R, V), dtype=np.float64)
    rr, kk = np.nonzero(keep_rows)
    np.add.at(dense, (rr, idx_rows[rr, kk]), P_rows[rr, kk])
    return dense


def _logsumexp(z: np.ndarray) -> np.ndarray:
    m = z.max(axis=1, keepdims=True)
    return (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0]


@dataclasses.dataclass
class Result:
    loss: float
    lse: np.ndarray            # [rows] float64 (every requested row, masked ones included)
    kl: np.ndarray             # [rows] float64 (0 on rows that do not count)
    n_valid: int
    flags: int
    rows: np.ndarray           # row indices the per-row arrays refer to
    dH: np.ndarray | None = None   # [rows, d]
    dW: np.ndarray | None = None   # [V, d] (only when every row was processed)
    G: np.ndarray | None = None    # [rows, V] (only when asked for)


def effective_mask(mask: np.ndarray, teacher: Teacher) -> np.ndarray:
    return (np.asarray(mask) != 0) & teacher.row_ok


@dataclasses.dataclass(frozen=True)
class Variant:
    """Loss-design variant (the pages report loss-design ablations without details:
    chatpaper.ai abstract, last sentences).  The default is the plain KL.

    P_S = softmax(z / student_tau).  Per valid row the loss is
        gamma * KL(P_T || P_S) + ce_weight * (-log P_S(label))
    with gamma = kd_weight * (student_tau^2 if kd_scale_tau_sq else 1) (Hinton's
    tau^2 factor) and the hard-label term only on rows whose label lies in [0, V).
    """
    student_tau: float = 1.0
    kd_weight: float = 1.0
    kd_scale_tau_sq: bool = False
    ce_weight: float = 0.0

    @property
    def gamma(self) -> float:
        return self.kd_weight * (self.student_tau ** 2 if self.kd_scale_tau_sq else 1.0)


PLAIN = Variant()


def kl_loss(hidden_bits, W_bits, topk_idx, topk_logit, mask, tau, *, grad_loss: float = 1.0,
            rows: np.ndarray | None = None, row_chunk: int = 64, want_grads: bool = True,
            want_dW: bool = True, want_G: bool = False, W_f64: np.ndarray | None = None,
            H_f64: np.ndarray | None = None, variant: Variant = PLAIN,
            labels: np.ndarray | None = None) -> Result:
    """Loss, per-row lse and (optionally) dHidden / dW by the plain definition.

    ``rows`` restricts the per-row work (lse, kl, dH) to a subset; N_valid and the
    loss normaliser always come from every row.  The loss itself is only
    returned when every row was processed (``rows is None``), else it is NaN.
    ``W_f64`` / ``H_f64`` replace the bf16 inputs by arbitrary float64 values
    (the finite-difference pins perturb them continuously).  ``variant`` and
    ``labels`` select a loss-design variant (see ``Variant``); lse is then the
    log-sum-exp of z / student_tau and ``kl`` holds each row's combined loss.
    """
    idx = np.asarray(topk_idx, dtype=np.int64)
    N, K = idx.shape
    W = bf16_bits_to_f64(W_bits) if W_f64 is None else W_f64
    V, d = W.shape
    teacher = teacher_distribution(idx, topk_logit, V, tau)
    m_eff = effective_mask(mask, teacher)
    n_valid = int(m_eff.sum())
    all_rows = rows is None
    rows = np.arange(N, dtype=np.int64) if all_rows else np.asarray(rows, dtype=np.int64)
    scale = (float(grad_loss) / n_valid) if n_valid > 0 else 0.0

    lse = np.empty(rows.size, dtype=np.float64)
    kl = np.zeros(rows.size, dtype=np.float64)
    dH = np.zeros((rows.size, d), dtype=np.float64) if want_grads else None
    dW = np.zeros((V, d), dtype=np.float64) if (want_grads and want_dW and all_rows) else None
    G_all = np.zeros((rows.size, V), dtype=np.float64) if want_G else None

    ts = float(variant.student_tau)
    gamma = variant.gamma
    beta = float(variant.ce_weight)
    lab = None if labels is None else np.asarray(labels, dtype=np.int64)
    for c0 in range(0, rows.size, row_chunk):
        sel = rows[c0:c0 + row_chunk]
        H = bf16_bits_to_f64(hidden_bits[sel]) if H_f64 is None else np.asarray(H_f64, np.float64)[sel]
        z = (H @ W.T) / ts                            # [R, V] student logits (softened)
        lse_c = _logsumexp(z)
        logP_S = z - lse_c[:, None]
        P_T = _dense_teacher(idx[sel], teacher.P[sel], teacher.keep[sel], V)
        pos = P_T > 0
        safe = np.where(pos, P_T, 1.0)
        kl_c = gamma * np.where(pos, P_T * (np.log(safe) - logP_S), 0.0).sum(axis=1)
        target = gamma * P_T
        if beta != 0.0 and lab is not None:
            ls = lab[sel]
            has = (ls >= 0) & (ls < V)
            rr = np.nonzero(has)[0]
            kl_c = kl_c + beta * np.where(has, -logP_S[np.arange(sel.size), np.clip(ls, 0, V - 1)], 0.0)
            onehot = np.zeros_like(P_T)
            onehot[rr, ls[rr]] = 1.0
            target = target + beta * onehot
        valid = m_eff[sel]
        lse[c0:c0 + sel.size] = lse_c
        kl[c0:c0 + sel.size] = np.where(valid, kl_c, 0.0)
        if want_grads or want_G:
            wsum = target.sum(axis=1, keepdims=True)       # gamma (+ beta where a label counts)
            G = (scale / ts * valid.astype(np.float64))[:, None] * (wsum * np.exp(logP_S) - target)
            if want_G:
                G_all[c0:c0 + sel.size] = G
            if want_grads:
                dH[c0:c0 + sel.size] = G @ W
                if dW is not None:
                    dW += G.T @ H

    loss = float(kl.sum() / n_valid) if (all_rows and n_valid > 0) else (0.0 if all_rows else float("nan"))
    return Result(loss, lse, kl, n_valid, teacher.flags, rows, dH, dW, G_all)


def kl_loss_from_logits(z: np.ndarray, topk_idx, topk_logit, mask, tau, grad_loss: float = 1.0):
    """Same definition when the student logits z[N, V] are given directly.

    Returns (loss, dlogits).  Used by the special-case pins (K = V, K = 1),
    where the logits are chosen freely instead of coming from a projection.
    """
    z = np.asarray(z, dtype=np.float64)
    N, V = z.shape
    idx = np.asarray(topk_idx, dtype=np.int64)
    teacher = teacher_distribution(idx, topk_logit, V, tau)
    m_eff = effective_mask(mask, teacher)
    n_valid = int(m_eff.sum())
    lse = _logsumexp(z)
    logP_S = z - lse[:, None]
    P_T = _dense_teacher(idx, teacher.P, teacher.keep, V)
    pos = P_T > 0
    kl = np.where(pos, P_T * (np.log(np.where(pos, P_T, 1.0)) - logP_S), 0.0).sum(axis=1)
    kl = np.where(m_eff, kl, 0.0)
    loss = float(kl.sum() / n_valid) if n_valid else 0.0
    scale = grad_loss / n_valid if n_valid else 0.0
    G = (scale * m_eff)[:, None] * (np.exp(logP_S) - P_T)
    return loss, G
