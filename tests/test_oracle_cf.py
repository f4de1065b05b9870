"""Pins for the counterfactual part of the CPU oracle (no GPU).

"ROSA-Tuning" section 3.5 treats each query bit as a decision switch: the
branches "force the bit to 0" and "force it to 1" each take one retrieval
step from the same historical state.  The oracle gives, for every position
t, bit j and value beta, the branch's most recent admissible end and match
length (``oracle.match_cf_brute`` from the definition, ``match_cf_sam`` with
the suffix automaton).  They are pinned to hand-worked cases, to the
ordinary (already pinned) matcher run on the stream with q[t] replaced by
the branch symbol, to the ordinary result on the branch that keeps the
actual bit, and to each other.
"""
import numpy as np
import pytest

import oracle
from tests.conftest import read_golden
from suffix_automaton_retrieval_b200 import workloads


def _ints(s):
    return [int(x) for x in s.split()]


@pytest.mark.parametrize("matcher", ["brute", "sam"])
def test_cf_golden_hand_cases(matcher):
    cases = read_golden("cf_hand_cases.txt")
    assert len(cases) >= 3
    fn = oracle.match_cf_brute if matcher == "brute" else oracle.match_cf_sam
    for c in cases:
        q = np.array(_ints(c["q"]), np.uint8)
        k = q if c["k"] == "same" else np.array(_ints(c["k"]), np.uint8)
        end, ln = fn(q, k, int(c["M"]), g=int(c["g"]))
        assert end[0].ravel().tolist() == _ints(c["end"]), c["case"]
        assert ln[0].ravel().tolist() == _ints(c["len"]), c["case"]


def test_cf_is_the_ordinary_step_on_the_substituted_stream():
    """Branch (t, j, beta) = the ordinary matcher at t on q with q[t] set to
    the branch symbol (keys unchanged: at step t only keys before t count)."""
    rng = np.random.default_rng(11)
    for _ in range(60):
        T = int(rng.integers(1, 24))
        M = int(rng.integers(1, 4))
        g = int(rng.integers(1, 4))
        q = rng.integers(0, 1 << M, T).astype(np.uint8)
        k = q.copy() if rng.random() < 0.4 else rng.integers(0, 1 << M, T).astype(np.uint8)
        end, ln = oracle.match_cf_brute(q, k, M, g=g)
        for t in range(T):
            for j in range(M):
                for beta in range(2):
                    qb = q.copy()
                    qb[t] = (int(q[t]) & ~(1 << j)) | (beta << j)
                    e2, l2, _ = oracle.match_brute(qb, k.copy(), g=g)
                    assert end[0, t, j, beta] == e2[0, t] and ln[0, t, j, beta] == l2[0, t], (T, M, g, t, j, beta)


def test_cf_branch_keeping_the_bit_is_the_ordinary_result():
    rng = np.random.default_rng(12)
    for _ in range(40):
        S, T, M, g = 4, int(rng.integers(1, 200)), int(rng.integers(1, 9)), int(rng.integers(1, 4))
        q = rng.integers(0, 1 << M, (S, T)).astype(np.uint8)
        k = q if rng.random() < 0.5 else rng.integers(0, 1 << M, (S, T)).astype(np.uint8)
        end, ln = oracle.match_cf_sam(q, k, M, g=g, threads=2)
        e0, l0, _ = oracle.match_sam(q, k, g=g, threads=2)
        bits = (q[:, :, None] >> np.arange(M)[None, None, :]) & 1
        kept_end = np.take_along_axis(end, bits[..., None].astype(np.int64), axis=3)[..., 0]
        kept_len = np.take_along_axis(ln, bits[..., None].astype(np.int64), axis=3)[..., 0]
        assert (kept_end == e0[:, :, None]).all() and (kept_len == l0[:, :, None]).all()


def test_cf_brute_vs_sam_random():
    """Definition and automaton agree on 3 000 random streams (T < 100, M = 1..8, g = 1..4)."""
    rng = np.random.default_rng(13)
    for _ in range(300):
        S, T = 10, int(rng.integers(1, 100))
        M, g = int(rng.integers(1, 9)), int(rng.integers(1, 5))
        K = int(rng.choice([1, 2, 3, 1 << M])) if M > 1 else int(rng.choice([1, 2]))
        K = min(K, 1 << M)
        q = rng.integers(0, K, (S, T)).astype(np.uint8)
        k = q if rng.random() < 0.4 else rng.integers(0, K, (S, T)).astype(np.uint8)
        a = oracle.match_cf_brute(q, k, M, g=g)
        b = oracle.match_cf_sam(q, k, M, g=g, threads=1)
        assert (a[0] == b[0]).all() and (a[1] == b[1]).all(), (T, M, g)


def test_cf_brute_vs_sam_recipes():
    """The markov-4 (M = 2) and binary (M = 1) recipes at reduced sizes, planted repeats in zipf (M = 8)."""
    cases = [(workloads.markov(B=1, R=4, T=600), 2), (workloads.binary_iid(T=800), 1),
             (workloads.zipf_planted(S=2, T=1200), 8)]
    for w, M in cases:
        a = oracle.match_cf_brute(w.q, w.k, M, g=w.g)
        b = oracle.match_cf_sam(w.q, w.k, M, g=w.g)
        assert (a[0] == b[0]).all() and (a[1] == b[1]).all(), w.name


def test_cf_rejects_symbols_wider_than_M():
    q = np.array([[0, 4, 1]], np.uint8)
    with pytest.raises(ValueError):
        oracle.match_cf_sam(q, q, 2)
