"""Pins for the CPU oracle (no GPU).

The oracle is pinned to things other than itself: hand-worked cases under
tests/golden/, closed forms for constant and periodic streams, an
independent invariant checker (maximality and recency by direct search), and
cross-agreement of the two matchers (definition vs suffix automaton), which
share no code.  A mutation test shows each pin is sharp enough to catch a
plausible slip.
"""
import numpy as np
import pytest

import oracle
from tests.conftest import read_golden
from tests.invariants import check_stream
from suffix_automaton_retrieval_b200 import workloads


def _ints(s):
    return np.array([int(x) for x in s.split()], dtype=np.int64)


# ---------------------------------------------------------------- golden

@pytest.mark.parametrize("matcher", ["brute", "sam"])
def test_golden_hand_cases(matcher):
    cases = read_golden("match_hand_cases.txt")
    assert len(cases) >= 6
    fn = oracle.match_brute if matcher == "brute" else oracle.match_sam
    for c in cases:
        q = _ints(c["q"]).astype(np.uint8)
        k = q if c["k"] == "same" else _ints(c["k"]).astype(np.uint8)
        v = k if c["v"] == "same" else _ints(c["v"]).astype(np.uint8)
        end, ln, sym = fn(q, k, v, g=int(c["g"]))
        assert end[0].tolist() == _ints(c["end"]).tolist(), c["case"]
        assert ln[0].tolist() == _ints(c["len"]).tolist(), c["case"]
        assert sym[0].tolist() == _ints(c["sym"]).tolist(), c["case"]


def test_golden_discretize():
    (c,) = read_golden("discretize_hand_case.txt")
    B, T, C, M = (int(c[x]) for x in ("B", "T", "C", "M"))
    x = np.array([int(h, 16) for h in c["x"].split()], np.uint16).reshape(B, T, C)
    sym = oracle.discretize(x, M)
    assert sym.reshape(-1).tolist() == _ints(c["sym"]).tolist()


def test_golden_gather():
    (c,) = read_golden("gather_hand_case.txt")
    B, T, Cv, R, d, rho = (int(c[x]) for x in ("B", "T", "Cv", "R", "d", "rho"))
    V = np.array([[[100 * t + col for col in range(Cv)] for t in range(T)]], np.uint16)
    assert V.shape == (B, T, Cv)
    end = _ints(c["end_idx"]).astype(np.int32).reshape(B * R, T)
    out = oracle.gather(V, end, R, d, rho)
    assert out.reshape(-1).tolist() == _ints(c["out"]).tolist()


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("g", [1, 2, 3, 5])
@pytest.mark.parametrize("matcher", ["brute", "sam"])
def test_constant_stream_closed_form(g, matcher):
    T = 300
    q = np.full(T, 7, np.uint8)
    fn = oracle.match_brute if matcher == "brute" else oracle.match_sam
    end, ln, sym = fn(q, q, g=g)
    t = np.arange(T)
    L = np.maximum(t - g + 1, 0)
    assert (ln[0] == L).all()
    assert (end[0] == np.where(L > 0, t - g, -1)).all()
    assert (sym[0] == np.where(L > 0, 7, -1)).all()


@pytest.mark.parametrize("p,g", [(3, 1), (3, 2), (5, 3), (7, 7), (16, 2)])
@pytest.mark.parametrize("matcher", ["brute", "sam"])
def test_periodic_stream_closed_form(p, g, matcher):
    """Period p with distinct symbols in the period and g <= p: a match must
    keep the phase, so the latest admissible end is t - p and the whole
    prefix k[0..t-p] matches: L_t = t - p + 1, i = t - p (none for t < p)."""
    T = 257
    q = (np.arange(T) % p).astype(np.uint8)
    fn = oracle.match_brute if matcher == "brute" else oracle.match_sam
    end, ln, _ = fn(q, q, g=g)
    t = np.arange(T)
    assert (ln[0] == np.where(t >= p, t - p + 1, 0)).all()
    assert (end[0] == np.where(t >= p, t - p, -1)).all()


def test_single_symbol_alphabet_and_tiny_T():
    for T in (1, 2, 3):
        q = np.zeros(T, np.uint8)
        for g in (1, 2):
            a = oracle.match_brute(q, q, g=g)
            b = oracle.match_sam(q, q, g=g)
            for x, y in zip(a, b):
                assert (x == y).all()
    end, ln, sym = oracle.match_sam(np.zeros(1, np.uint8), np.zeros(1, np.uint8), g=1)
    assert end.tolist() == [[-1]] and ln.tolist() == [[0]] and sym.tolist() == [[-1]]


def test_empty_batch():
    q = np.zeros((0, 5), np.uint8)
    end, ln, sym = oracle.match_sam(q, q, g=2)
    assert end.shape == (0, 5)


# ---------------------------------------------------------------- cross-agreement

def test_brute_vs_sam_random():
    """7 000 random streams (T < 130, K up to 256, g = 1..4), ten per call."""
    rng = np.random.default_rng(1234)
    for _ in range(700):
        S = 10
        T = int(rng.integers(1, 130))
        K = int(rng.choice([1, 2, 3, 4, 16, 256]))
        g = int(rng.integers(1, 5))
        q = rng.integers(0, K, (S, T)).astype(np.uint8)
        mode = rng.integers(0, 3)
        k = q if mode == 0 else rng.integers(0, K, (S, T)).astype(np.uint8)
        v = None if rng.random() < 0.5 else rng.integers(0, 256, (S, T)).astype(np.uint8)
        a = oracle.match_brute(q, k, v, g=g)
        b = oracle.match_sam(q, k, v, g=g, threads=1)
        for x, y in zip(a, b):
            assert (x == y).all(), (T, K, g)


def test_brute_vs_sam_workload_recipes():
    """The five input recipes at oracle-friendly sizes; brute force is exact."""
    cases = [
        workloads.binary_iid(T=4096),
        workloads.planted_copies(B=1, R=2, T=3000),
        workloads.zipf_planted(S=2, T=3000),
        workloads.markov(B=1, R=3, T=2048),
    ]
    for w in cases:
        a = oracle.match_brute(w.q, w.k, g=w.g)
        b = oracle.match_sam(w.q, w.k, g=w.g)
        for x, y in zip(a, b):
            assert (x == y).all(), w.name


# ---------------------------------------------------------------- invariants

def test_invariants_full_small():
    rng = np.random.default_rng(7)
    for _ in range(60):
        T = int(rng.integers(1, 90))
        K = int(rng.choice([2, 3, 4]))
        g = int(rng.integers(1, 4))
        q = rng.integers(0, K, T).astype(np.uint8)
        k = q if rng.random() < 0.5 else rng.integers(0, K, T).astype(np.uint8)
        end, ln, sym = oracle.match_sam(q, k, g=g)
        check_stream(q, k, k, g, end[0], ln[0], sym[0], full=True)


def test_invariants_sampled_recipes():
    w = workloads.zipf_planted(S=1, T=6000)
    end, ln, sym = oracle.match_sam(w.q, w.k, g=w.g)
    check_stream(w.q[0], w.k[0], w.k[0], w.g, end[0], ln[0], sym[0], full=False, sample=60)
    assert ln.max() >= 16  # the planted repeats are found


# ---------------------------------------------------------------- pins catch slips

def _mutants(q, k, g):
    """Outputs of plausible slips, made on the CPU from the oracle's own
    (correct) output or by running it with a wrong parameter."""
    end, ln, sym = (x[0].copy() for x in oracle.match_brute(q, k, g=g))
    out = {}
    e2, l2, s2 = (x[0] for x in oracle.match_brute(q, k, g=g - 1))      # lag off by one
    out["lag-1"] = (e2, l2, s2)
    # earliest instead of most recent end: rerun the definition by hand
    T = len(q)
    ee = end.copy()
    for t in range(T):
        L = ln[t]
        if L > 0:
            for j in range(L - 1, t - g + 1):
                if np.array_equal(k[j - L + 1:j + 1], q[t - L + 1:t + 1]):
                    ee[t] = j
                    break
    out["earliest"] = (ee, ln, np.where(ee >= 0, k[np.minimum(ee + 1, T - 1)], -1))
    out["sym-at-i"] = (end, ln, np.where(end >= 0, k[np.maximum(end, 0)], -1))
    out["len-minus-1"] = (end, np.maximum(ln - 1, 0), sym)
    return out


def test_pins_catch_mutants():
    rng = np.random.default_rng(99)
    q = rng.integers(0, 2, 200).astype(np.uint8)
    k = rng.integers(0, 2, 200).astype(np.uint8)
    g = 2
    for name, (e, l, s) in _mutants(q, k, g).items():
        with pytest.raises(AssertionError):
            check_stream(q, k, k, g, e, l, s, full=True)
            raise RuntimeError(f"mutant {name} passed the invariant checker")


def test_discretize_bit_order_and_threshold():
    """Symbols built from known bits come back exactly, for every M."""
    rng = np.random.default_rng(5)
    pos, neg, zero = 0x3F80, 0xBF80, 0x0000   # +1, -1, +0 in bf16
    for M in range(1, 9):
        B, T, R = 2, 5, 3
        want = rng.integers(0, 2 ** M, size=(B, R, T))
        x = np.empty((B, T, R * M), np.uint16)
        for b in range(B):
            for t in range(T):
                for r in range(R):
                    for j in range(M):
                        bit = (int(want[b, r, t]) >> j) & 1
                        x[b, t, r * M + j] = pos if bit else (neg if (j + t) % 2 else zero)
        assert (oracle.discretize(x, M) == want).all()
