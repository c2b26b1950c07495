"""Plain CPU float64 oracle of the teacher top-K cache producer.

TEST INFRASTRUCTURE ONLY (see ``oracle/kl.py``): nothing on the product path
imports it.

The offline cache is built by running the teacher once and keeping, for each
token position, the K most likely vocabulary entries as (index, logit) pairs
(mind-verse.de article, section "Zwei systemische Optimierungen", item 1;
llm-wiki note, section "사전 계산 파이프라인", steps 2-3).  With the teacher's
last hidden state h and output head W_T, the logits are z = h W_T^T and "most
likely" is "largest logit" (softmax is monotone).  The plain definition:

    order every vocabulary entry by (z descending, index ascending) and keep
    the first K; report them in that order.

Reading: the pages do not say how ties are broken or in which order the
entries are stored; ties go to the smaller index and entries are stored by
descending logit (the order the synthetic caches use).
"""
from __future__ import annotations

import numpy as np

from .kl import bf16_bits_to_f64


def teacher_logits(hidden_bits: np.ndarray, W_bits: np.ndarray, rows: np.ndarray | None = None) -> np.ndarray:
    H = bf16_bits_to_f64(hidden_bits if rows is None else hidden_bits[rows])
    return H @ bf16_bits_to_f64(W_bits).T


def topk_from_logits(z: np.ndarray, K: int):
    """(indices [R, K] int64, values [R, K] float64) by (value desc, index asc)."""
    z = np.asarray(z, dtype=np.float64)
    R, V = z.shape
    cols = np.broadcast_to(np.arange(V), (R, V))
    order = np.lexsort((cols, -z), axis=1)[:, :K]   # last key is primary: -z, then index
    return order.astype(np.int64), np.take_along_axis(z, order, axis=1)


def teacher_topk(hidden_bits: np.ndarray, W_bits: np.ndarray, K: int, rows: np.ndarray | None = None,
                 row_chunk: int = 64):
    """Top-K (index, logit) per row of z = hidden W^T, processed in row chunks."""
    n = hidden_bits.shape[0] if rows is None else len(rows)
    all_rows = np.arange(hidden_bits.shape[0]) if rows is None else np.asarray(rows)
    idx = np.empty((n, K), dtype=np.int64)
    val = np.empty((n, K), dtype=np.float64)
    for c0 in range(0, n, row_chunk):
        sel = all_rows[c0:c0 + row_chunk]
        z = teacher_logits(hidden_bits, W_bits, sel)
        idx[c0:c0 + sel.size], val[c0:c0 + sel.size] = topk_from_logits(z, K)
    return idx, val
