"""Comparison of a GPU routing result with the fp64 oracle, by the stated tolerances.

Rules (MoRE, "MoRE: Scaling mixture of experts with hardware-aware low-rank routing";
margin of §3 Definition 1; the kernels carry z as a bf16 pair z_hi + z_lo, finer than the single bf16 of App. F Algorithm 1):
  * tol_n = 1e-2 x rms_n, rms_n the root-mean-square of token n's M oracle logits.
  * logits: every returned logit is within tol_n of the oracle's logit of the same expert.
  * index sets are compared where the oracle's margin l_(k) - l_(k+1) exceeds tol_n;
    the expert at slot j where the gaps on both sides of slot j exceed tol_n.
  * gates: within 2e-3 absolute, per expert id, on tokens whose sets matched.
  * counts: always equal to the bincount of the GPU's own indices and sum to N k;
    bit-exact with the oracle when every token was compared and every set matched.
  * validity (all tokens): indices in [0, M) and distinct per token, logits
    non-increasing, equal logits in increasing index order, gates summing to 1 and
    non-increasing.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import oracle

LOGIT_TOL = 1e-2
GATE_TOL = 2e-3


@dataclass
class ParityReport:
    rows_checked: int
    set_compared: int
    set_matched: int
    slot_compared: int
    max_logit_err_over_rms: float
    max_gate_err: float

    @property
    def set_fraction(self) -> float:
        return self.set_compared / max(1, self.rows_checked)


def check_validity(idx, gate, counts, logits, M, k):
    N = idx.shape[0]
    assert idx.shape == (N, k) and gate.shape == (N, k) and counts.shape == (M,)
    assert idx.min(initial=0) >= 0 and idx.max(initial=0) < M, "expert index out of range"
    if N:
        s = np.sort(idx, axis=1)
        assert np.all(s[:, 1:] != s[:, :-1]) if k > 1 else True, "repeated expert in a token"
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=M), "counts != bincount(idx)")
    assert counts.sum() == N * k
    assert np.all(np.abs(gate.sum(axis=1) - 1.0) <= 1e-5), "gates do not sum to 1"
    assert np.all(gate[:, 1:] <= gate[:, :-1] + 1e-7), "gates not in routing order"
    if logits is not None:
        assert np.all(logits[:, 1:] <= logits[:, :-1]), "logits not in routing order"
        eq = logits[:, 1:] == logits[:, :-1]
        assert np.all(idx[:, 1:][eq] > idx[:, :-1][eq]), "equal logits not in index order"


def compare(X, R1, R2, N, h, r, M, k, idx, gate, counts, logits, rows=None, exact=False,
            logit_tol=LOGIT_TOL, gate_tol=GATE_TOL, min_set_fraction=0.5) -> ParityReport:
    """Check GPU outputs (numpy) against the oracle on ``rows`` (default: every token).

    ``exact`` demands identical indices and counts on every token (for inputs whose
    logits are exact in fp32, e.g. small integers).
    """
    idx = np.asarray(idx)
    gate = np.asarray(gate)
    counts = np.asarray(counts)
    logits = None if logits is None else np.asarray(logits)
    check_validity(idx, gate, counts, logits, M, k)
    all_rows = rows is None
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    o = oracle.route(X, R1, R2, N, h, r, M, k, rows=rows)
    g_idx, g_gate = idx[rows], gate[rows]
    tol = logit_tol * o.rms
    max_logit = 0.0
    if logits is not None and rows.size:
        ref = oracle.logits_at(X, R1, R2, N, h, r, M, np.repeat(rows, k), g_idx.ravel()).reshape(-1, k)
        err = np.abs(logits[rows] - ref)
        bad = err > tol[:, None]
        assert not bad.any(), f"logit error above tolerance at rows {rows[np.where(bad.any(1))[0][:5]]}"
        max_logit = float((err / np.maximum(o.rms, 1e-30)[:, None]).max())
    if exact:
        np.testing.assert_array_equal(g_idx, o.idx)
        np.testing.assert_allclose(g_gate, o.gate, rtol=0, atol=1e-6)
        if all_rows:
            np.testing.assert_array_equal(counts, o.counts)
        return ParityReport(rows.size, rows.size, rows.size, rows.size * k, max_logit,
                            float(np.abs(g_gate - o.gate).max(initial=0.0)))
    set_cmp = o.margin > tol
    matched = np.zeros(rows.size, bool)
    max_gate = 0.0
    for q in np.where(set_cmp)[0]:
        gs, os_ = set(g_idx[q].tolist()), set(o.idx[q].tolist())
        assert gs == os_, f"token {rows[q]}: GPU set {sorted(gs)} != oracle set {sorted(os_)} " \
                          f"(margin {o.margin[q]:.4g}, tol {tol[q]:.4g})"
        matched[q] = True
        gmap = dict(zip(g_idx[q].tolist(), g_gate[q].tolist()))
        d = max(abs(gmap[e] - og) for e, og in zip(o.idx[q].tolist(), o.gate[q].tolist()))
        assert d <= gate_tol, f"token {rows[q]}: gate error {d:.3g}"
        max_gate = max(max_gate, d)
    # slot order: slot j is fixed when the gaps on both of its sides exceed tol
    left = np.concatenate([np.full((rows.size, 1), np.inf), o.gaps[:, :-1]], axis=1)
    slot_ok = (left > tol[:, None]) & (o.gaps > tol[:, None])
    mism = slot_ok & (g_idx != o.idx)
    assert not mism.any(), f"slot order differs at rows {rows[np.where(mism.any(1))[0][:5]]}"
    if all_rows and matched.all():
        np.testing.assert_array_equal(counts, o.counts)
    frac = set_cmp.mean() if rows.size else 1.0
    if rows.size >= 64:
        assert frac >= min_set_fraction, f"only {frac:.2%} of tokens had a comparable margin"
    return ParityReport(rows.size, int(set_cmp.sum()), int(matched.sum()), int(slot_ok.sum()), max_logit,
                        max_gate)


def sample_rows(N: int, n_sample: int, seed: int = 0) -> np.ndarray:
    """Token rows for sampled comparison: the first and last tile, the ragged tail, random rows."""
    if N <= n_sample:
        return np.arange(N)
    rng = np.random.default_rng(seed)
    fixed = np.unique(np.concatenate([np.arange(min(N, 64)), np.arange(max(0, N - 200), N)]))
    rest = rng.choice(N, size=max(0, n_sample - fixed.size), replace=False)
    return np.unique(np.concatenate([fixed, rest]))
