"""Seeded synthetic inputs for the fused chunked KL distillation loss.

This module only draws random inputs: it holds none of the loss arithmetic.
Both the CPU oracle (``oracle/``) and the CUDA path's tests and bench feed on
exactly these arrays, so the two sides always see the same bytes.

What the inputs stand for (paper "Efficient Knowledge Distillation for LLMs:
Offline Top-K Logits and a Fused Chunked KL Loss", mind-verse.de article,
section "Zwei systemische Optimierungen", item 1): an offline teacher cache
holds, for every token position, the K most likely vocabulary entries as
(index, logit) pairs.  No teacher model or dataset exists here, so the cache,
the student's last hidden state and the output-head weight are all drawn from
seeded distributions with the workload shapes listed in ``CONFIGS``.

Recipe (one numpy PCG64 generator per input set, seeded ``20260802 + config
number``, plus ``N`` for the long-context sweep points):

* hidden[N, d] ~ N(0, 1) rounded to bf16 (round to nearest even);
* W[V, d] ~ N(0, 0.02^2) rounded to bf16;
* ``uniform`` cache: K distinct vocabulary indices per row drawn uniformly
  without replacement, logits ~ N(0, logit_std^2) sorted descending;
* ``zipf`` cache: ranks drawn with replacement from Zipf(s) over [0, V) by
  inverse CDF, the first K distinct draws kept in draw order, each mapped
  through a per-row affine bijection pi_n(r) = (a_n r + b_n) mod V with
  gcd(a_n, V) = 1 (stand-in for a per-row random vocabulary permutation),
  and the k-th kept rank gets the k-th largest of K logits ~ N(0, std^2);
* mask[N] uint8: exactly round(frac * N) rows set to 0 (packed-sequence
  boundaries), chosen by a seeded permutation; all ones when frac == 0.
"""
from __future__ import annotations

import dataclasses

import numpy as np

BASE_SEED = 20260802


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    number: int          # config number 1..5
    N: int
    d: int
    V: int
    K: int
    tau: float
    cache: str           # "uniform" or "zipf"
    logit_std: float
    mask_frac: float
    zipf_s: float = 1.1


CONFIGS = {
    "tiny": Workload("tiny", 1, 256, 256, 4096, 16, 1.0, "uniform", 2.0, 0.0),
    "small": Workload("small", 2, 4096, 2048, 32768, 100, 1.0, "zipf", 3.0, 0.05),
    "8b": Workload("8b", 3, 32768, 4096, 128256, 100, 1.0, "zipf", 3.0, 0.05),
    "sweep": Workload("sweep", 4, 4096, 4096, 128256, 100, 2.0, "zipf", 3.0, 0.05),
    "large_vocab": Workload("large_vocab", 5, 131072, 2880, 201088, 100, 1.0, "zipf", 3.0, 0.02),
}
SWEEP_N = (4096, 16384, 65536, 131072, 262144)


@dataclasses.dataclass
class Inputs:
    """One seeded input set.  bf16 tensors are kept as raw uint16 bit patterns."""
    hidden_bits: np.ndarray   # [N, d] uint16 (bf16 bits)
    W_bits: np.ndarray        # [V, d] uint16 (bf16 bits)
    topk_idx: np.ndarray      # [N, K] int32
    topk_logit: np.ndarray    # [N, K] float32
    mask: np.ndarray          # [N] uint8
    tau: float

    @property
    def shape(self):
        N, d = self.hidden_bits.shape
        return N, d, self.W_bits.shape[0], self.topk_idx.shape[1]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def seed_for(w: Workload, N: int | None = None) -> int:
    s = BASE_SEED + w.number
    if w.name == "sweep":
        s += int(N if N is not None else w.N)
    return s


def _normal_bf16(rng: np.random.Generator, shape, std: float, block_rows: int = 8192) -> np.ndarray:
    rows, cols = shape
    out = np.empty(shape, dtype=np.uint16)
    for r0 in range(0, rows, block_rows):
        r1 = min(rows, r0 + block_rows)
        x = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[r0:r1] = f32_to_bf16_bits(x)
    return out


def _uniform_cache(rng, N, V, K):
    idx = np.empty((N, K), dtype=np.int32)
    for n in range(N):
        idx[n] = rng.choice(V, size=K, replace=False)
    return idx


def _zipf_cdf(V: int, s: float) -> np.ndarray:
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    return cdf


def _first_k_distinct(draws: np.ndarray, K: int):
    """Per row, the first K distinct values in draw order; rows short of K flagged."""
    order = np.argsort(draws, axis=1, kind="stable")
    sv = np.take_along_axis(draws, order, axis=1)
    first_sorted = np.ones_like(sv, dtype=bool)
    first_sorted[:, 1:] = sv[:, 1:] != sv[:, :-1]
    is_first = np.empty_like(first_sorted)
    np.put_along_axis(is_first, order, first_sorted, axis=1)
    cum = np.cumsum(is_first, axis=1)
    ok = cum[:, -1] >= K
    sel = is_first & (cum <= K)
    return sel, ok


def _affine_params(rng, n_rows: int, V: int):
    a = rng.integers(1, V, size=n_rows, dtype=np.int64)
    bad = np.gcd(a, V) != 1
    while bad.any():
        a[bad] = rng.integers(1, V, size=int(bad.sum()), dtype=np.int64)
        bad = np.gcd(a, V) != 1
    b = rng.integers(0, V, size=n_rows, dtype=np.int64)
    return a, b


def _zipf_cache(rng, N, V, K, s, block_rows=4096):
    cdf = _zipf_cdf(V, s)
    idx = np.empty((N, K), dtype=np.int32)
    M = 2 * K + 16
    for r0 in range(0, N, block_rows):
        r1 = min(N, r0 + block_rows)
        B = r1 - r0
        ranks = np.empty((B, K), dtype=np.int64)
        todo = np.arange(B)
        m = M
        while todo.size:
            u = rng.random((todo.size, m))
            draws = np.minimum(np.searchsorted(cdf, u, side="right"), V - 1).astype(np.int64)
            sel, ok = _first_k_distinct(draws, K)
            good = todo[ok]
            if good.size:
                ranks[good] = draws[ok][sel[ok]].reshape(good.size, K)
            todo = todo[~ok]
            m *= 2
        a, b = _affine_params(rng, B, V)
        idx[r0:r1] = ((a[:, None] * ranks + b[:, None]) % V).astype(np.int32)
    return idx


def make_inputs(w: Workload, N: int | None = None, *, seed: int | None = None) -> Inputs:
    """Draw the seeded input set of workload ``w`` (``N`` overrides its token count)."""
    N = int(w.N if N is None else N)
    rng = np.random.default_rng(seed_for(w, N) if seed is None else seed)
    hidden = _normal_bf16(rng, (N, w.d), 1.0)
    W = _normal_bf16(rng, (w.V, w.d), 0.02)
    if w.cache == "uniform":
        idx = _uniform_cache(rng, N, w.V, w.K)
    elif w.cache == "zipf":
        idx = _zipf_cache(rng, N, w.V, w.K, w.zipf_s)
    else:
        raise ValueError(w.cache)
    logit = rng.standard_normal((N, w.K), dtype=np.float32) * np.float32(w.logit_std)
    logit = -np.sort(-logit, axis=1)
    mask = np.ones(N, dtype=np.uint8)
    n_off = int(round(w.mask_frac * N))
    if n_off:
        mask[rng.permutation(N)[:n_off]] = 0
    return Inputs(hidden, W, idx, np.ascontiguousarray(logit, dtype=np.float32), mask, float(w.tau))


def custom_inputs(N, d, V, K, *, seed, tau=1.0, cache="uniform", logit_std=2.0,
                  mask_frac=0.0, w_std=0.02, h_std=1.0, zipf_s=1.1) -> Inputs:
    """Same recipe at arbitrary sizes (ragged tails, edge cases)."""
    rng = np.random.default_rng(seed)
    hidden = _normal_bf16(rng, (N, d), h_std)
    W = _normal_bf16(rng, (V, d), w_std)
    if cache == "uniform":
        idx = _uniform_cache(rng, N, V, K)
    else:
        idx = _zipf_cache(rng, N, V, K, zipf_s)
    logit = rng.standard_normal((N, K), dtype=np.float32) * np.float32(logit_std)
    logit = -np.sort(-logit, axis=1)
    mask = np.ones(N, dtype=np.uint8)
    n_off = int(round(mask_frac * N))
    if n_off:
        mask[rng.permutation(N)[:n_off]] = 0
    return Inputs(hidden, W, idx.astype(np.int32), np.ascontiguousarray(logit, dtype=np.float32),
                  mask, float(tau))


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """A seeded, sorted subset of row indices (used for sampled parity checks)."""
    rng = np.random.default_rng(seed)
    count = min(count, N)
    return np.sort(rng.choice(N, size=count, replace=False)).astype(np.int64)


def flops_fwd_bwd(N: int, d: int, V: int) -> float:
    """Algorithmic tensor work of one forward+backward: 8 N d V (projection counted twice)."""
    return 8.0 * N * d * V

