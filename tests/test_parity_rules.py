"""The GPU-vs-oracle comparison rules of tests/parity.py, checked on the CPU.

Outputs built from the oracle itself must pass every rule; outputs with a planted wrong
selection must fail, including on tokens whose margin is below the 1e-2 x rms tolerance
(where the set comparison alone would not look).  This pins the rules that the GPU parity
tests rely on, without a GPU.
"""
import numpy as np
import pytest

import oracle
import synthetic as syn
from tests import parity

N, h, r, M, k = 512, 128, 32, 192, 4


@pytest.fixture(scope="module")
def case():
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=11)
    o = oracle.route(X, R1, R2, N, h, r, M, k)
    full = oracle.logits(X, R1, R2, N, h, r, M)
    return X, R1, R2, o, full


def outputs_from_oracle(o):
    idx = o.idx.copy()
    logits = o.logit.astype(np.float32)
    ex = np.exp(o.logit - o.logit[:, :1])
    gate = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    counts = np.bincount(idx.ravel(), minlength=M).astype(np.int32)
    return idx, gate, counts, logits


def replace_expert(full, idx, logits, n, slot, e):
    """Put expert e into token n's slot with its correct logit, then restore routing order."""
    idx = idx.copy()
    logits = logits.copy()
    idx[n, slot] = e
    logits[n, slot] = full[n, e]
    order = np.lexsort((idx[n], -logits[n].astype(np.float64)))
    idx[n], logits[n] = idx[n][order], logits[n][order]
    return idx, logits


def gates_of(logits):
    ex = np.exp(logits.astype(np.float64) - logits[:, :1])
    return (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)


def test_oracle_outputs_pass_every_rule(case):
    X, R1, R2, o, _ = case
    idx, gate, counts, logits = outputs_from_oracle(o)
    rep = parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, counts, logits)
    assert rep.set_matched == rep.set_compared
    assert rep.fine_set_compared >= rep.set_compared


def test_far_replacement_on_a_near_tie_token_is_caught(case):
    """A token whose margin is below tol: swapping its k-th expert for one ranked far below
    (with that expert's correct logit) passes the set rule, which skips the token, but not
    the tolerance-valid top-k rule."""
    X, R1, R2, o, full = case
    tol = parity.LOGIT_TOL * o.rms
    near = np.where(o.margin < tol)[0]
    assert near.size > 0, "the seeded case has near-tie tokens"
    n = int(near[0])
    far = int(np.argsort(-full[n], kind="stable")[30])   # the 31st-ranked expert
    idx, gate, counts, logits = outputs_from_oracle(o)
    idx, logits = replace_expert(full, idx, logits, n, k - 1, far)
    gate = gates_of(logits)
    counts = np.bincount(idx.ravel(), minlength=M).astype(np.int32)
    with pytest.raises(AssertionError, match="below the k-th oracle logit"):
        parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, counts, logits)


def test_missing_clear_winner_is_caught(case):
    """Dropping an expert far above the cut in favour of the (k+1)-th is caught even when
    the token's own margin is tiny."""
    X, R1, R2, o, full = case
    tol = parity.LOGIT_TOL * o.rms
    cand = np.where((o.margin < tol) & (o.logit[:, 0] > o.logit[:, k - 1] + 2 * tol))[0]
    assert cand.size > 0
    n = int(cand[0])
    next_best = int(np.argsort(-full[n], kind="stable")[k])
    idx, gate, counts, logits = outputs_from_oracle(o)
    idx, logits = replace_expert(full, idx, logits, n, 0, next_best)
    gate = gates_of(logits)
    counts = np.bincount(idx.ravel(), minlength=M).astype(np.int32)
    with pytest.raises(AssertionError):
        parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, counts, logits)


def test_fine_rule_catches_a_swap_inside_the_coarse_tolerance(case):
    """A token whose margin lies between 1e-4 and 1e-2 x rms: swapping its k-th and (k+1)-th
    experts passes the coarse rules but fails the fine set comparison."""
    X, R1, R2, o, full = case
    rel = o.margin / o.rms
    mid = np.where((rel > 10 * parity.FINE_TOL) & (rel < parity.LOGIT_TOL))[0]
    assert mid.size > 0
    n = int(mid[0])
    nxt = int(np.argsort(-full[n], kind="stable")[k])
    idx, gate, counts, logits = outputs_from_oracle(o)
    idx, logits = replace_expert(full, idx, logits, n, k - 1, nxt)
    gate = gates_of(logits)
    counts = np.bincount(idx.ravel(), minlength=M).astype(np.int32)
    with pytest.raises(AssertionError, match="fine tolerance"):
        parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, counts, logits)


def test_near_tie_rows_are_the_smallest_margins(case):
    X, R1, R2, o, _ = case
    rows = parity.near_tie_rows(X, R1, R2, N, h, r, M, k, 10)
    rel = o.margin / o.rms
    assert set(rows.tolist()) == set(np.argsort(rel, kind="stable")[:10].tolist())


def test_sample_rows_include_whole_tiles_and_extras():
    rows = parity.sample_rows(100_000, 2000, seed=1, tiles=(3, 500), extra=(77_777,))
    for t in (3, 500):
        assert set(range(128 * t, 128 * t + 128)) <= set(rows.tolist())
    assert 77_777 in rows and 0 in rows and 99_999 in rows
