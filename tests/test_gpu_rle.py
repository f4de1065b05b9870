"""Parity of the run-level (adjacent folding) retrieval on the GPU with the
CPU oracle: section 3.3 of "ROSA-Tuning" (arXiv 2602.02499), both streams
folded into runs, each query run answered at its start, the hit mapped to
the start of the next key run.  Bit-exact on every output, through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.conftest import read_golden
from tests.invariants import check_rle_stream
from suffix_automaton_retrieval_b200 import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def rosa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from suffix_automaton_retrieval_b200 import build
    build.build()
    import suffix_automaton_retrieval_b200.binding as b
    return b


def _gpu_rle(rosa, q, k, v, K, g, status=True):
    qd = torch.from_numpy(np.ascontiguousarray(q)).to(DEV)
    same = k is q
    kd = qd if same else torch.from_numpy(np.ascontiguousarray(k)).to(DEV)
    vd = None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(DEV)
    S, T = qd.shape
    ws = torch.empty(rosa.match_rle_workspace_size(S, T, K), dtype=torch.uint8, device=DEV)
    e, l, s = rosa.match_rle(qd, None if same else kd, vd, K=K, g=g, workspace=ws)
    torch.cuda.synchronize()
    if status:
        assert rosa.match_device_status(ws) == 0
    return e.cpu().numpy(), l.cpu().numpy(), s.cpu().numpy()


def _assert_same(got, want, tag=""):
    for name, a, b in zip(("end_idx", "len", "sym"), got, want):
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            s, t = bad[0]
            raise AssertionError(f"{tag} {name} differs at {len(bad)} places; first (s={s}, t={t}): "
                                 f"gpu={a[s, t]} oracle={b[s, t]}")


def _ints(s):
    return np.array([int(x) for x in s.split()], dtype=np.int64)


def test_rle_golden_hand_cases(rosa):
    for c in read_golden("rle_hand_cases.txt"):
        q = _ints(c["q"]).astype(np.uint8)[None]
        k = q if c["k"] == "same" else _ints(c["k"]).astype(np.uint8)[None]
        v = None if c["v"] == "same" else _ints(c["v"]).astype(np.uint8)[None]
        K = int(max(q.max(), k.max())) + 1
        got = _gpu_rle(rosa, q, k, v, K, int(c["g"]))
        assert got[0][0].tolist() == _ints(c["end"]).tolist(), c["case"]
        assert got[1][0].tolist() == _ints(c["len"]).tolist(), c["case"]
        assert got[2][0].tolist() == _ints(c["sym"]).tolist(), c["case"]


def _runny(rng, S, T, K, r):
    """[S, T] symbols drawn as runs: each drawn symbol repeated 1..r times."""
    out = np.empty((S, T), np.uint8)
    for i in range(S):
        base = rng.integers(0, K, T).astype(np.uint8)
        out[i] = np.repeat(base, rng.integers(1, r + 1, T))[:T]
    return out


def test_rle_random_small(rosa):
    rng = np.random.default_rng(77)
    for _ in range(200):
        S = int(rng.integers(1, 5))
        T = int(rng.integers(1, 300))
        K = int(rng.choice([1, 2, 3, 4, 16, 256]))
        g = int(rng.integers(1, 4))
        r = int(rng.choice([1, 2, 4]))
        q = _runny(rng, S, T, K, r)
        k = q if rng.random() < 0.35 else _runny(rng, S, T, K, r)
        v = rng.integers(0, 256, (S, T)).astype(np.uint8) if rng.random() < 0.3 else None
        got = _gpu_rle(rosa, q, k, v, K, g)
        want = oracle.match_rle_brute(q, k, v, g=g)
        _assert_same(got, want, f"S={S} T={T} K={K} g={g} r={r}")


@pytest.mark.parametrize("T", [2047, 2048, 2049, 4097, 6144])
def test_rle_tile_edges(rosa, T):
    """Runs that span the 2048-position tiles of the folding kernels."""
    rng = np.random.default_rng(T)
    q = _runny(rng, 3, T, 4, 8)
    k = _runny(rng, 3, T, 4, 8)
    for qq, kk in ((q, k), (q, q)):
        got = _gpu_rle(rosa, qq, kk, None, 4, 2)
        _assert_same(got, oracle.match_rle_sam(qq, kk, g=2), f"T={T}")


def test_rle_degenerate_streams(rosa):
    T = 1500
    const = np.full((2, T), 3, np.uint8)
    alt = np.tile(np.array([0, 1], np.uint8), (2, T // 2))
    blocks = np.repeat(np.arange(T // 50, dtype=np.uint8) % 7, 50)[None].repeat(2, 0)
    for name, q, K in (("constant", const, 4), ("alternating", alt, 2), ("blocks", blocks, 7)):
        for g in (1, 2, 3):
            got = _gpu_rle(rosa, q, q, None, K, g)
            _assert_same(got, oracle.match_rle_brute(q, q, g=g), f"{name} g={g}")
    # one symbol alphabet, q != k: nothing is ever admissible
    got = _gpu_rle(rosa, const, const.copy(), None, 4, 2)
    assert (got[0] == -1).all() and (got[1] == 0).all()


def test_rle_errors_and_empty(rosa):
    q = torch.zeros((2, 100), dtype=torch.uint8, device=DEV)
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(rosa.RosaError):
        rosa.match_rle(q, K=4, workspace=small)
    with pytest.raises(rosa.RosaError):
        rosa.match_rle(q, K=4, g=0)
    e, l, s = rosa.match_rle(torch.zeros((0, 9), dtype=torch.uint8, device=DEV), K=4)
    assert e.shape == (0, 9)
    assert rosa.match_rle_launch_count(2, 100, 4, True) > rosa.match_launch_count(2, 100, 4, True)


# ---------------------------------------------------------------- full-size workloads, every stream

def _full(rosa, w, tag):
    got = _gpu_rle(rosa, w.q, w.q if w.same_qk else w.k, None, w.K, w.g)
    want = oracle.match_rle_sam(w.q, w.q if w.same_qk else w.k, g=w.g)
    _assert_same(got, want, tag)
    check_rle_stream(w.q[0], w.k[0], w.k[0], w.g, got[0][0], got[1][0], got[2][0], full=False, sample=40)
    return got


def test_rle_full_binary_4k(rosa):
    w = workloads.binary_iid()
    got = _gpu_rle(rosa, w.q, w.q, None, w.K, w.g)
    _assert_same(got, oracle.match_rle_brute(w.q, w.q, g=w.g), "binary-4k")   # the definition


def test_rle_full_planted_16(rosa):
    _full(rosa, workloads.planted_copies(), "planted-16")


def test_rle_full_zipf_256_131k(rosa):
    _full(rosa, workloads.zipf_planted(), "zipf-256-131k")


def test_rle_full_markov_4_train(rosa):
    got = _full(rosa, workloads.markov(), "markov-4-train")
    assert (got[1] > 0).mean() > 0.5


def test_rle_full_qwen_proj_64(rosa):
    c = workloads.spec("qwen-proj-64")
    T, width, ch, M = c["T"], c["width"], c["channels"], c["M"]
    H, Wq, Wk = workloads.qwen_projection_inputs(T=T, width=width, channels=ch, device=DEV)
    qv, kv = (H @ Wq).contiguous(), (H @ Wk).contiguous()
    del H
    R = ch // M
    sq, sk = rosa.discretize_pair(qv, kv, M)
    qh, kh = sq.view(R, T).cpu().numpy(), sk.view(R, T).cpu().numpy()
    got = _gpu_rle(rosa, qh, kh, None, 2 ** M, 2)
    _assert_same(got, oracle.match_rle_sam(qh, kh, g=2), "qwen-proj-64")
