"""Pins for the dense parts of the CPU oracle (no GPU): the read-out
embedding and injection of appendix C.3 and the layer norm + projection of
section 3.2 that precede the threshold.

Pins that do not re-run the oracle's own formula: hand-worked cases under
tests/golden/; the identity W_out, which reduces the injection to the
embedding y itself (so the selection of e0 / e1 / mask per recalled bit is
checked on its own); a one-column W_out; closed forms of the layer norm
(constant rows, two-valued rows); its invariance to shifting and scaling a
row; and the threshold-and-pack step against the already pinned
discretisation of the same values.  Mutants of plausible slips must fail.
"""
import numpy as np
import pytest

import oracle
from tests.conftest import read_golden


def _bf(x):
    """float -> bf16 bits (round toward zero; the tests use exactly representable values)."""
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _floats(s):
    return np.array([float(x) for x in s.split()])


# ---------------------------------------------------------------- injection

def test_inject_golden_hand_case():
    (c,) = read_golden("inject_hand_case.txt")
    B, R, M, T = (int(c[k]) for k in ("B", "R", "M", "T"))
    C = R * M
    e0, e1 = _bf(_floats(c["e0"])), _bf(_floats(c["e1"]))
    W = _bf(_floats(c["W"]).reshape(-1, C))
    sym = _floats(c["sym"]).astype(np.int32).reshape(B * R, T)
    got = oracle.inject(sym, e0, e1, W, B, R, M)
    assert got.reshape(-1).tolist() == _floats(c["inj"]).tolist()


def _embedding_by_hand(sym, e0, e1, B, R, M):
    """y[b, t, c] built route by route, bit by bit (the selection alone)."""
    T = sym.shape[1]
    y = np.zeros((B, T, R * M))
    for b in range(B):
        for r in range(R):
            for t in range(T):
                a = int(sym[b * R + r, t])
                for j in range(M):
                    if a >= 0:
                        y[b, t, r * M + j] = _f(e1)[r * M + j] if (a >> j) & 1 else _f(e0)[r * M + j]
    return y


@pytest.mark.parametrize("B,R,M,T", [(1, 3, 1, 7), (2, 4, 2, 5), (1, 2, 8, 9)])
def test_inject_identity_is_the_embedding(B, R, M, T):
    rng = np.random.default_rng(B * 100 + R * 10 + M)
    C = R * M
    e0 = _bf(rng.standard_normal(C))
    e1 = _bf(rng.standard_normal(C))
    sym = rng.integers(-1, 1 << M, (B * R, T)).astype(np.int32)
    W = _bf(np.eye(C))
    got = oracle.inject(sym, e0, e1, W, B, R, M)
    assert np.array_equal(got, _embedding_by_hand(sym, e0, e1, B, R, M))


def test_inject_one_column_and_masks():
    rng = np.random.default_rng(3)
    B, R, M, T, D = 1, 3, 2, 11, 5
    C = R * M
    e0, e1 = _bf(rng.standard_normal(C)), _bf(rng.standard_normal(C))
    sym = rng.integers(-1, 4, (B * R, T)).astype(np.int32)
    for c in range(C):
        Wf = np.zeros((D, C), np.float32)
        Wf[:, c] = rng.standard_normal(D)
        W = _bf(Wf)
        got = oracle.inject(sym, e0, e1, W, B, R, M)
        y = _embedding_by_hand(sym, e0, e1, B, R, M)[..., c]
        assert np.array_equal(got, y[..., None] * _f(W)[:, c][None, None, :])
    # every route masked: nothing is injected
    none = np.full((B * R, T), -1, np.int32)
    assert not oracle.inject(none, e0, e1, _bf(rng.standard_normal((D, C))), B, R, M).any()


def test_inject_pins_catch_mutants():
    rng = np.random.default_rng(9)
    B, R, M, T = 1, 2, 3, 6
    C = R * M
    e0, e1 = _bf(rng.standard_normal(C)), _bf(rng.standard_normal(C))
    sym = rng.integers(-1, 8, (B * R, T)).astype(np.int32)
    want = _embedding_by_hand(sym, e0, e1, B, R, M)
    I = _bf(np.eye(C))
    mutants = {
        "e0/e1 swapped": oracle.inject(sym, e1, e0, I, B, R, M),
        "bits msb-first": oracle.inject(np.where(sym >= 0, np.array([int(f"{a:03b}"[::-1], 2) if a >= 0 else -1
                                                                     for a in sym.ravel()]).reshape(sym.shape),
                                                 -1).astype(np.int32), e0, e1, I, B, R, M),
        "mask ignored": oracle.inject(np.where(sym < 0, 0, sym).astype(np.int32), e0, e1, I, B, R, M),
        "routes swapped": oracle.inject(sym[::-1].copy(), e0, e1, I, B, R, M),
    }
    for name, got in mutants.items():
        assert not np.array_equal(got, want), name


# ---------------------------------------------------------------- layer norm and projection

def test_ln_project_golden_hand_case():
    (c,) = read_golden("ln_project_hand_case.txt")
    D, N = int(c["D"]), int(c["N"])
    H = _bf(_floats(c["h"])).reshape(1, D)
    W = _bf(_floats(c["W"]).reshape(D, N))
    P, A = oracle.ln_project(H, W, _floats(c["gamma"]), _floats(c["beta"]), eps=float(c["eps"]))
    assert np.allclose(P.ravel(), _floats(c["P"]), rtol=0, atol=1e-12)
    assert (A > 0).all()


def test_ln_project_constant_row_gives_beta_projection():
    rng = np.random.default_rng(4)
    D, N = 16, 3
    W = _bf(rng.standard_normal((D, N)))
    beta = rng.standard_normal(D).astype(np.float32)
    H = _bf(np.full((2, D), 1.5))
    P, _ = oracle.ln_project(H, W, rng.standard_normal(D).astype(np.float32), beta, eps=1e-5)
    want = beta.astype(np.float64) @ _f(W)
    assert np.allclose(P, want[None, :], rtol=0, atol=1e-9)


def test_ln_project_two_valued_row_closed_form():
    """h alternates +a / -a: mu = 0, var = a^2, u = gamma * sign * a / sqrt(a^2 + eps)."""
    D, N, a, eps = 8, 2, 2.0, 0.25
    sgn = np.array([1, -1] * (D // 2), np.float64)
    H = _bf(sgn * a)[None]
    W = _bf(np.eye(D)[:, :N] + np.eye(D)[:, 1:N + 1])     # column n sums u_n + u_{n+1}
    P, _ = oracle.ln_project(H, W, None, None, eps=eps)
    u = sgn * a / np.sqrt(a * a + eps)
    assert np.allclose(P[0], [u[0] + u[1], u[1] + u[2]], rtol=0, atol=1e-12)


def test_ln_project_shift_and_scale_invariance():
    rng = np.random.default_rng(5)
    D, N = 32, 4
    base = rng.integers(-8, 9, D).astype(np.float64)          # small integers: exact under shift and scale
    W = _bf(rng.standard_normal((D, N)))
    g = rng.standard_normal(D).astype(np.float32)
    b = rng.standard_normal(D).astype(np.float32)
    P0, _ = oracle.ln_project(_bf(base)[None], W, g, b, eps=0.0)
    P1, _ = oracle.ln_project(_bf(base + 16)[None], W, g, b, eps=0.0)
    P2, _ = oracle.ln_project(_bf(base * 4)[None], W, g, b, eps=0.0)
    assert np.allclose(P0, P1, rtol=0, atol=1e-9) and np.allclose(P0, P2, rtol=0, atol=1e-9)


def test_pack_bits_agrees_with_the_pinned_discretisation():
    """Values exact in bf16: thresholding and packing them must give what the
    discretisation (pinned by its own tests) gives on their bit patterns."""
    rng = np.random.default_rng(6)
    for M in (1, 2, 4, 8):
        B, T, C = 2, 9, 8 * M
        x = _bf(rng.standard_normal((B, T, C)))
        x[0, 0, :4] = [0x0000, 0x8000, 0x7FC0, 0x0001]        # +0, -0, NaN, tiny positive
        P = np.nan_to_num(_f(x).reshape(B * T, C), nan=0.0)
        assert np.array_equal(oracle.pack_bits(P, B, T, M), oracle.discretize(x, M))
