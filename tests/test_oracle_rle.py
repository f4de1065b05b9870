"""Pins for the run-level (adjacent folding) oracle, no GPU.

Section 3.3 of "ROSA-Tuning" (arXiv 2602.02499) folds consecutive equal
symbols into runs, moves the automaton and the matching state only at run
boundaries, and maps a hit back to the start of the next key run.  The
oracle's two forms (the definition over runs, and suffix automata over the
key runs with a run-start array) are pinned to: hand-worked cases
(tests/golden/rle_hand_cases.txt), the plain operator on streams without
adjacent repeats (where every run is one symbol), an independent checker of
the run-level properties (tests/invariants.py), their agreement with each
other, and mutants of plausible slips that the checker must reject.
"""
import numpy as np
import pytest

import oracle
from tests.conftest import read_golden
from tests.invariants import check_rle_stream
from suffix_automaton_retrieval_b200 import workloads


def _ints(s):
    return np.array([int(x) for x in s.split()], dtype=np.int64)


@pytest.mark.parametrize("form", ["brute", "sam"])
def test_rle_golden_hand_cases(form):
    cases = read_golden("rle_hand_cases.txt")
    assert len(cases) >= 5
    fn = oracle.match_rle_brute if form == "brute" else oracle.match_rle_sam
    for c in cases:
        q = _ints(c["q"]).astype(np.uint8)
        k = q if c["k"] == "same" else _ints(c["k"]).astype(np.uint8)
        v = k if c["v"] == "same" else _ints(c["v"]).astype(np.uint8)
        end, ln, sym = fn(q, k, v, g=int(c["g"]))
        assert end[0].tolist() == _ints(c["end"]).tolist(), c["case"]
        assert ln[0].tolist() == _ints(c["len"]).tolist(), c["case"]
        assert sym[0].tolist() == _ints(c["sym"]).tolist(), c["case"]


def _no_repeats(rng, S, T, K):
    x = np.empty((S, T), np.uint8)
    x[:, 0] = rng.integers(0, K, S)
    for t in range(1, T):
        step = rng.integers(1, K, S)            # never 0: the symbol always changes
        x[:, t] = (x[:, t - 1] + step) % K
    return x


def test_rle_without_adjacent_repeats_is_the_plain_operator():
    """Every run one symbol long: run indices are time indices, so the
    run-level operator must equal the plain one (a different matcher)."""
    rng = np.random.default_rng(11)
    for _ in range(200):
        S, T = 4, int(rng.integers(1, 150))
        K = int(rng.choice([2, 3, 5, 16, 256]))
        g = int(rng.integers(1, 4))
        q = _no_repeats(rng, S, T, K)
        k = q if rng.random() < 0.3 else _no_repeats(rng, S, T, K)
        v = rng.integers(0, 256, (S, T)).astype(np.uint8)
        plain = oracle.match_brute(q, k, v, g=g)
        for fn in (oracle.match_rle_brute, oracle.match_rle_sam):
            got = fn(q, k, v, g=g)
            for a, b in zip(got, plain):
                assert np.array_equal(a, b), (fn.__name__, T, K, g)


def test_rle_brute_vs_sam_random():
    """4 000 random streams with many runs and repeats (small alphabets)."""
    rng = np.random.default_rng(21)
    for _ in range(400):
        S, T = 10, int(rng.integers(1, 120))
        K = int(rng.choice([1, 2, 3, 4]))
        g = int(rng.integers(1, 5))
        q = rng.integers(0, K, (S, T)).astype(np.uint8)
        k = q if rng.random() < 0.3 else rng.integers(0, K, (S, T)).astype(np.uint8)
        v = None if rng.random() < 0.5 else rng.integers(0, 256, (S, T)).astype(np.uint8)
        a = oracle.match_rle_brute(q, k, v, g=g)
        b = oracle.match_rle_sam(q, k, v, g=g, threads=1)
        for x, y in zip(a, b):
            assert np.array_equal(x, y), (T, K, g)


def test_rle_brute_vs_sam_workload_recipes():
    cases = [workloads.binary_iid(T=3000), workloads.planted_copies(B=1, R=2, T=3000),
             workloads.zipf_planted(S=2, T=3000), workloads.markov(B=1, R=3, T=3000)]
    for w in cases:
        a = oracle.match_rle_brute(w.q, w.k, g=w.g)
        b = oracle.match_rle_sam(w.q, w.k, g=w.g)
        for x, y in zip(a, b):
            assert np.array_equal(x, y), w.name


def test_rle_invariants_full_small():
    rng = np.random.default_rng(31)
    for _ in range(80):
        T = int(rng.integers(1, 100))
        K = int(rng.choice([2, 3, 4]))
        g = int(rng.integers(1, 4))
        q = rng.integers(0, K, T).astype(np.uint8)
        k = q if rng.random() < 0.4 else rng.integers(0, K, T).astype(np.uint8)
        end, ln, sym = oracle.match_rle_sam(q, k, g=g)
        check_rle_stream(q, k, k, g, end[0], ln[0], sym[0], full=True)


def test_rle_invariants_sampled_markov():
    w = workloads.markov(B=1, R=1, T=6000)
    end, ln, sym = oracle.match_rle_sam(w.q, w.k, g=w.g)
    check_rle_stream(w.q[0], w.k[0], w.k[0], w.g, end[0], ln[0], sym[0], full=False, sample=80)
    assert (ln > 0).mean() > 0.5


def _rle_mutants(q, k, g):
    """Plausible slips, made on the CPU from the oracle's own output or by
    running an oracle with a wrong parameter."""
    end, ln, sym = (x[0].copy() for x in oracle.match_rle_brute(q, k, g=g))
    out = {}
    out["lag-1"] = tuple(x[0] for x in oracle.match_rle_brute(q, k, g=g - 1))
    out["lag+1"] = tuple(x[0] for x in oracle.match_rle_brute(q, k, g=g + 1))
    out["unfolded"] = tuple(x[0] for x in oracle.match_brute(q, k, g=g))
    # tau at the matched run's own start instead of the next run's
    T = len(k)
    kstart = np.flatnonzero(np.r_[True, k[1:] != k[:-1]])
    e2 = end.copy()
    for t in range(T):
        if end[t] >= 0:
            e2[t] = kstart[np.searchsorted(kstart, end[t], side="right") - 1] - 1
    out["own-run"] = (e2, ln, np.where(e2 >= 0, k[np.maximum(e2 + 1, 0)], -1))
    out["sym-at-end"] = (end, ln, np.where(end >= 0, k[np.maximum(end, 0)], -1))
    out["len-in-steps"] = (end, np.where(ln > 0, ln + 1, 0), sym)
    return out


def test_rle_pins_catch_mutants():
    rng = np.random.default_rng(41)
    q = rng.integers(0, 3, 400).astype(np.uint8)
    k = rng.integers(0, 3, 400).astype(np.uint8)
    g = 2
    for name, (e, l, s) in _rle_mutants(q, k, g).items():
        with pytest.raises(AssertionError):
            check_rle_stream(q, k, k, g, e, l, s, full=True)
            raise RuntimeError(f"mutant {name} passed the run-level checker")


def _binary_rle_closed_form(q, k, v, g):
    """Run-level retrieval on a binary alphabet written out from the fact the
    GPU's binary path rests on: folded binary streams alternate, so query run m
    shares min(m, l) + 1 runs with key run l when their symbols agree and none
    otherwise; the answer is the last admissible key run with query run m's
    symbol.  Independent of the oracle's code (numpy on one stream)."""
    T = len(q)
    def runs(a):
        starts = [0] + [t for t in range(1, T) if a[t] != a[t - 1]]
        run_of = np.zeros(T, np.int64)
        for i, s in enumerate(starts):
            run_of[s:] = i
        return np.array(starts), run_of
    ks, krun = runs(k)
    qs, qrun = runs(q)
    end = np.full(T, -1, np.int64); ln = np.zeros(T, np.int64); sym = np.full(T, -1, np.int64)
    for t in range(T):
        m = qrun[t]
        p = qs[m] - g + 1                 # the next key run must start by here
        if p < 0:
            continue
        X = krun[p] - 1                   # last admissible key run
        if X < 0:
            continue
        l = X if k[ks[X]] == q[qs[m]] else X - 1
        if l < 0:
            continue
        end[t] = ks[l + 1] - 1
        ln[t] = min(l, m) + 1
        sym[t] = v[ks[l + 1]]
    return end, ln, sym


def test_rle_binary_closed_form_matches_the_definition():
    rng = np.random.default_rng(2024)
    for trial in range(300):
        T = int(rng.integers(1, 160))
        r = int(rng.choice([1, 2, 4]))
        q = np.repeat(rng.integers(0, 2, T), rng.integers(1, r + 1, T))[:T].astype(np.uint8)
        k = q if rng.random() < 0.3 else np.repeat(rng.integers(0, 2, T), rng.integers(1, r + 1, T))[:T].astype(np.uint8)
        v = k if rng.random() < 0.5 else rng.integers(0, 256, T).astype(np.uint8)
        g = int(rng.integers(1, 4))
        want = oracle.match_rle_brute(q[None], k[None], v[None], g=g)
        got = _binary_rle_closed_form(q, k, v, g)
        for name, a, b in zip(("end", "len", "sym"), got, want):
            assert np.array_equal(a, b[0]), (trial, name, T, g, q.tolist(), k.tolist())
