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
  * tolerance-valid top-k (every compared token, whatever its margin): each returned
    expert's oracle logit is at least l_(k) - tol_n, and each expert whose oracle logit
    exceeds l_(k) + tol_n is returned (l_(k): the oracle's k-th largest logit).  So a
    near-tie token may swap experts only among those within tol_n of the cut.
  * fine comparison: the same set and slot rules at tol_fine = 1e-4 x rms_n.  The kernels
    carry z as z_hi + z_lo, which is within 2^-18 |z_i| of z per component, so their
    logits err by about 1e-5 x rms_n; 1e-4 x rms_n leaves a margin of ten, and the index
    comparison then covers almost every token instead of those with a clear 1e-2 margin.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import oracle

LOGIT_TOL = 1e-2
GATE_TOL = 2e-3
FINE_TOL = 1e-4


@dataclass
class ParityReport:
    rows_checked: int
    set_compared: int
    set_matched: int
    slot_compared: int
    max_logit_err_over_rms: float
    max_gate_err: float
    fine_set_compared: int = 0

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
    """Check GPU outputs (numpy) of the low-rank router against the oracle on ``rows``
    (default: every token).

    ``exact`` demands identical indices and counts on every token (for inputs whose
    logits are exact in fp32, e.g. small integers).
    """
    rows_ = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    o = oracle.route(X, R1, R2, N, h, r, M, k, rows=rows_)
    ref_at = lambda rr, ee: oracle.logits_at(X, R1, R2, N, h, r, M, rr, ee)
    return _compare(o, ref_at, rows, rows_, M, k, idx, gate, counts, logits, exact, logit_tol, gate_tol,
                    min_set_fraction)


def compare_fullrank(X, W, N, h, M, k, idx, gate, counts, logits, rows=None, exact=False,
                     logit_tol=LOGIT_TOL, gate_tol=GATE_TOL, min_set_fraction=0.5) -> ParityReport:
    """:func:`compare` for the standard full-rank router x . W (App. H.3), by the same rules."""
    rows_ = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    o = oracle.route_fullrank(X, W, N, h, M, k, rows=rows_)
    ref_at = lambda rr, ee: oracle.logits_at_fullrank(X, W, N, h, M, rr, ee)
    return _compare(o, ref_at, rows, rows_, M, k, idx, gate, counts, logits, exact, logit_tol, gate_tol,
                    min_set_fraction)


def _compare(o, ref_at, rows_arg, rows, M, k, idx, gate, counts, logits, exact, logit_tol, gate_tol,
             min_set_fraction) -> ParityReport:
    """The rules of this module, given the oracle's result ``o`` on ``rows`` and ``ref_at``,
    the oracle's logits of (row, expert) pairs."""
    idx = np.asarray(idx)
    gate = np.asarray(gate)
    counts = np.asarray(counts)
    logits = None if logits is None else np.asarray(logits)
    check_validity(idx, gate, counts, logits, M, k)
    all_rows = rows_arg is None
    g_idx, g_gate = idx[rows], gate[rows]
    tol = logit_tol * o.rms
    max_logit = 0.0
    if rows.size:
        # oracle logits of the experts the GPU returned
        ref = ref_at(np.repeat(rows, k), g_idx.ravel()).reshape(-1, k)
        if logits is not None:
            err = np.abs(logits[rows] - ref)
            bad = err > tol[:, None]
            assert not bad.any(), f"logit error above tolerance at rows {rows[np.where(bad.any(1))[0][:5]]}"
            max_logit = float((err / np.maximum(o.rms, 1e-30)[:, None]).max())
        # tolerance-valid top-k on every token: nothing returned from below the cut, nothing
        # clearly above it left out
        lk = o.logit[:, k - 1]
        low = ref < (lk - tol)[:, None]
        assert not low.any(), (f"returned expert more than tol below the k-th oracle logit at rows "
                               f"{rows[np.where(low.any(1))[0][:5]]}")
        present = (o.idx[:, :, None] == g_idx[:, None, :]).any(axis=2)
        missing = (o.logit > (lk + tol)[:, None]) & ~present
        assert not missing.any(), (f"expert clearly above the k-th oracle logit not returned at rows "
                                   f"{rows[np.where(missing.any(1))[0][:5]]}")
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
    # fine comparison: sets and slots wherever the margins exceed FINE_TOL x rms
    ftol = FINE_TOL * o.rms
    fine_set = o.margin > ftol
    if fine_set.any():
        gs = np.sort(g_idx[fine_set], axis=1)
        os_ = np.sort(o.idx[fine_set], axis=1)
        diff = np.any(gs != os_, axis=1)
        assert not diff.any(), (f"set differs at the fine tolerance at rows {rows[fine_set][diff][:5]} "
                                f"(margins {o.margin[fine_set][diff][:5] / o.rms[fine_set][diff][:5]} x rms)")
    fleft = np.concatenate([np.full((rows.size, 1), np.inf), o.gaps[:, :-1]], axis=1)
    fslot = (fleft > ftol[:, None]) & (o.gaps > ftol[:, None])
    fmism = fslot & (g_idx != o.idx)
    assert not fmism.any(), f"slot order differs at the fine tolerance at rows {rows[np.where(fmism.any(1))[0][:5]]}"
    return ParityReport(rows.size, int(set_cmp.sum()), int(matched.sum()), int(slot_ok.sum()), max_logit,
                        max_gate, int(fine_set.sum()))


def sample_rows(N: int, n_sample: int, seed: int = 0, tiles=(), extra=()) -> np.ndarray:
    """Token rows for sampled comparison: the first 64 rows and the last 200 (the ragged
    tail), the whole 128-token tiles listed in ``tiles``, the rows in ``extra``, and random
    rows up to ``n_sample`` in total."""
    if N <= n_sample:
        return np.arange(N)
    rng = np.random.default_rng(seed)
    parts = [np.arange(min(N, 64)), np.arange(max(0, N - 200), N), np.asarray(extra, dtype=np.int64)]
    for t in tiles:
        parts.append(np.arange(128 * t, min(N, 128 * (t + 1))))
    fixed = np.unique(np.concatenate(parts))
    rest = rng.choice(N, size=max(0, n_sample - fixed.size), replace=False)
    return np.unique(np.concatenate([fixed, rest]))


def near_tie_rows(X, R1, R2, N, h, r, M, k, count, scan=None) -> np.ndarray:
    """The ``count`` rows with the smallest oracle margin l_(k) - l_(k+1) relative to their
    rms, among ``scan`` rows (default: all N) -- the tokens on which a selection kernel's
    tie handling and exact re-check decide the result."""
    scan = np.arange(N) if scan is None else np.asarray(scan, dtype=np.int64)
    o = oracle.route(X, R1, R2, N, h, r, M, k, rows=scan)
    rel = o.margin / np.maximum(o.rms, 1e-30)
    return np.sort(scan[np.argsort(rel, kind="stable")[:count]])


def near_tie_rows_fullrank(X, W, N, h, M, k, count, scan=None) -> np.ndarray:
    """:func:`near_tie_rows` for the full-rank router x . W."""
    scan = np.arange(N) if scan is None else np.asarray(scan, dtype=np.int64)
    o = oracle.route_fullrank(X, W, N, h, M, k, rows=scan)
    rel = o.margin / np.maximum(o.rms, 1e-30)
    return np.sort(scan[np.argsort(rel, kind="stable")[:count]])
