"""The seeded input recipes draw what they state: shapes, alphabets, seeds,
the q = k convention, planted-repeat coverage, the Zipf and Markov laws, and
the value/projection tensors' sizes and scales (no GPU; reduced sizes where
a full-size draw would take long)."""
import numpy as np
import pytest

from suffix_automaton_retrieval_b200 import workloads as W


def test_registry_names_and_shapes():
    names = [v["name"] for v in W.WORKLOADS.values()]
    assert names == ["binary-4k", "planted-16", "qwen-proj-64", "zipf-256-131k", "markov-4-train"]
    assert W.spec("qwen-proj-64")["channels"] == 64 and W.spec("markov-4-train")["d"] == 64
    with pytest.raises(KeyError):
        W.spec("no-such-workload")


def test_draws_are_seeded():
    a, b = W.zipf_planted(S=2, T=4096), W.zipf_planted(S=2, T=4096)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k, b.k)
    c = W.zipf_planted(S=2, T=4096, seed_q=99)
    assert not np.array_equal(a.q, c.q)


def test_binary_iid():
    w = W.binary_iid()
    assert (w.S, w.T, w.K, w.g) == (1, 4096, 2, 2) and w.same_qk
    assert set(np.unique(w.q)) <= {0, 1}
    assert abs(w.q.mean() - 0.5) < 0.05


def _covered_by_copies(x, lmin):
    """Positions of x inside a segment of length >= lmin that also occurs
    earlier in x (an exact repeat), found by hashing windows of length lmin."""
    T = len(x)
    seen, covered = {}, np.zeros(T, bool)
    for s in range(T - lmin + 1):
        key = x[s:s + lmin].tobytes()
        if key in seen and seen[key] + lmin <= s:
            covered[s:s + lmin] = True
        seen.setdefault(key, s)
    return covered


def test_planted_copies_cover_about_five_percent():
    """Destinations (disjoint) are planted until they cover 5 % of the stream;
    a later destination may overwrite an earlier copy's source, so the exact
    repeats that remain cover a little less."""
    w = W.planted_copies(B=1, R=4, T=16384)
    assert w.K == 16 and w.same_qk and int(w.q.max()) < 16
    for s in range(w.S):
        assert _covered_by_copies(w.q[s], 32).mean() >= 0.04


def test_zipf_law_and_planted_repeats():
    w = W.zipf_planted(S=2, T=32768)
    assert w.K == 256 and not w.same_qk
    # rank-frequency follows p_r ~ r^-1.1 (symbol = rank - 1): the head's share
    p = np.bincount(w.k[0], minlength=256) / w.T
    want = W._zipf_p(256, 1.1)
    assert abs(p[0] - want[0]) < 0.02 and abs(p[1] - want[1]) < 0.02
    # >= 2 % of query positions lie in repeats of length >= 16 that occur in the key stream earlier
    for s in range(w.S):
        q, k = w.q[s], w.k[s]
        keyset = {}
        for a in range(w.T - 16 + 1):
            keyset.setdefault(k[a:a + 16].tobytes(), a)
        cov = np.zeros(w.T, bool)
        for b in range(w.T - 16 + 1):
            a = keyset.get(q[b:b + 16].tobytes())
            if a is not None and a + 16 + w.g <= b + 16:
                cov[b:b + 16] = True
        assert cov.mean() >= 0.02


def test_markov_chain_law():
    w = W.markov(B=1, R=8, T=8192)
    assert (w.K, w.T, w.S) == (4, 8192, 8) and not w.same_qk
    x = w.q.astype(np.int64)
    stay = (x[:, 1:] == x[:, :-1]).mean()
    assert abs(stay - 0.7) < 0.02
    moved = x[:, 1:][x[:, 1:] != x[:, :-1]] - x[:, :-1][x[:, 1:] != x[:, :-1]]
    counts = np.bincount(moved % 4, minlength=4)[1:]   # steps +1, +2, +3 (mod 4): the other symbols
    assert abs(counts / counts.sum() - 1 / 3).max() < 0.03


def test_projection_and_value_tensors():
    H, Wq, Wk = W.qwen_projection_inputs(T=64, width=256, channels=8)
    assert H.shape == (1, 64, 256) and Wq.shape == (256, 8) and Wk.shape == (256, 8)
    assert str(H.dtype) == "torch.bfloat16"
    assert abs(float(Wq.float().std()) - 256 ** -0.5) < 0.01
    V = W.value_rows(2, 16, 64, seed=33)
    assert V.shape == (2, 16, 64) and abs(float(V.float().std()) - 1.0) < 0.1
