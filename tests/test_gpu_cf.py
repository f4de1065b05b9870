"""Parity of the per-bit counterfactual destinations on the GPU with the CPU
oracle: section 3.5 of "ROSA-Tuning" (arXiv 2602.02499), every query bit
forced to 0 and to 1, one retrieval step each from the same history
(appendix C.5 uses tau^(0), tau^(1)).  Bit-exact on every output, through
the C ABI; the recalled symbol of a branch is v[end + 1] by the operator's
definition.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.conftest import read_golden
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


def _gpu_cf(rosa, q, k, v, M, g):
    qd = torch.from_numpy(np.ascontiguousarray(q)).to(DEV)
    same = k is q
    kd = qd if same else torch.from_numpy(np.ascontiguousarray(k)).to(DEV)
    vd = None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(DEV)
    S, T = qd.shape
    ws = torch.empty(rosa.match_cf_workspace_size(S, T, M), dtype=torch.uint8, device=DEV)
    out = rosa.match_cf(qd, None if same else kd, vd, M=M, g=g, workspace=ws)
    torch.cuda.synchronize()
    assert rosa.match_device_status(ws) == 0
    return out


def _want_sym(end, v):
    """sym of a branch: v[end + 1] where a match exists, else -1."""
    S = v.shape[0]
    e = end.reshape(S, -1)
    y = np.where(e >= 0, np.take_along_axis(v.astype(np.int32), np.maximum(e + 1, 0), axis=1), -1)
    return y.reshape(end.shape)


def _check(out, q, k, v, M, g, tag, brute=False, streams=None):
    """All six outputs against the oracle (optionally for a subset of streams)."""
    sl = slice(None) if streams is None else streams
    qs, ks = q[sl], k[sl]
    vs = ks if v is None else v[sl]
    cf = (oracle.match_cf_brute if brute else oracle.match_cf_sam)(qs, ks, M, g=g)
    plain = (oracle.match_brute if brute else oracle.match_sam)(qs, ks, vs, g=g)
    want = list(plain) + [cf[0], cf[1], _want_sym(cf[0], vs)]
    names = ("end_idx", "len", "sym", "end_cf", "len_cf", "sym_cf")
    for name, a, b in zip(names, out, want):
        a = a[sl].cpu().numpy()
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            raise AssertionError(f"{tag}: {name} differs at {len(bad)} places; first {tuple(bad[0])}: "
                                 f"gpu={a[tuple(bad[0])]} oracle={b[tuple(bad[0])]}")


def _ints(s):
    return [int(x) for x in s.split()]


def test_cf_golden_hand_cases(rosa):
    for c in read_golden("cf_hand_cases.txt"):
        q = np.array(_ints(c["q"]), np.uint8)[None]
        k = q if c["k"] == "same" else np.array(_ints(c["k"]), np.uint8)[None]
        M = int(c["M"])
        out = _gpu_cf(rosa, q, k, None, M, int(c["g"]))
        assert out[3][0].cpu().numpy().ravel().tolist() == _ints(c["end"]), c["case"]
        assert out[4][0].cpu().numpy().ravel().tolist() == _ints(c["len"]), c["case"]


def test_cf_random_small(rosa):
    rng = np.random.default_rng(505)
    for _ in range(150):
        S = int(rng.integers(1, 4))
        T = int(rng.integers(1, 200))
        M = int(rng.choice([1, 2, 3, 4, 8]))
        g = int(rng.integers(1, 4))
        K = 1 << M
        hi = int(rng.choice([K, min(K, 3)]))    # low-entropy symbols too
        q = rng.integers(0, hi, (S, T)).astype(np.uint8)
        k = q if rng.random() < 0.35 else rng.integers(0, hi, (S, T)).astype(np.uint8)
        v = rng.integers(0, 256, (S, T)).astype(np.uint8) if rng.random() < 0.3 else None
        out = _gpu_cf(rosa, q, k, v, M, g)
        _check(out, q, k, v, M, g, f"S={S} T={T} M={M} g={g}", brute=True)


@pytest.mark.parametrize("T", [2047, 2048, 2049, 4097])
def test_cf_tile_edges(rosa, T):
    rng = np.random.default_rng(T + 1)
    for M in (1, 2):
        q = rng.integers(0, 1 << M, (3, T)).astype(np.uint8)
        k = rng.integers(0, 1 << M, (3, T)).astype(np.uint8)
        for kk in (k, q):
            _check(_gpu_cf(rosa, q, kk, None, M, 2), q, kk, None, M, 2, f"T={T} M={M}")


def test_cf_degenerate_streams(rosa):
    T = 3000
    const = np.zeros((2, T), np.uint8)
    alt = np.tile(np.array([0, 1], np.uint8), (2, T // 2))
    per = (np.arange(T) % 3).astype(np.uint8)[None].repeat(2, 0)
    for name, q, M in (("constant", const, 1), ("alternating", alt, 1), ("period-3", per, 2)):
        for g in (1, 2):
            _check(_gpu_cf(rosa, q, q, None, M, g), q, q, None, M, g, f"{name} g={g}")
            k = q.copy()
            _check(_gpu_cf(rosa, q, k, None, M, g), q, k, None, M, g, f"{name} q!=k g={g}")


def test_cf_errors(rosa):
    q = torch.zeros((2, 50), dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        rosa.match_cf_workspace_size(2, 50, 0)
    with pytest.raises(ValueError):
        rosa.match_cf_workspace_size(2, 50, 9)
    with pytest.raises(rosa.RosaError):
        rosa.match_cf(q, M=2, g=0)
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(rosa.RosaError):
        rosa.match_cf(q, M=2, workspace=small)
    assert rosa.match_cf_launch_count(2, 50, 2, False) > rosa.match_launch_count(2, 50, 4, False)


# ---------------------------------------------------------------- full-size workloads

def test_cf_full_binary_4k(rosa):
    w = workloads.binary_iid()
    _check(_gpu_cf(rosa, w.q, w.q, None, 1, w.g), w.q, w.q, None, 1, w.g, "binary-4k", brute=True)


def test_cf_full_markov_4_train(rosa):
    w = workloads.markov()
    _check(_gpu_cf(rosa, w.q, w.k, None, 2, w.g), w.q, w.k, None, 2, w.g, "markov-4-train")


def test_cf_full_planted_16(rosa):
    w = workloads.planted_copies()
    _check(_gpu_cf(rosa, w.q, w.q, None, 4, w.g), w.q, w.q, None, 4, w.g, "planted-16")


def test_cf_full_qwen_proj_64(rosa):
    c = workloads.spec("qwen-proj-64")
    T, width, ch, M = c["T"], c["width"], c["channels"], c["M"]
    H, Wq, Wk = workloads.qwen_projection_inputs(T=T, width=width, channels=ch, device=DEV)
    qv, kv = (H @ Wq).contiguous(), (H @ Wk).contiguous()
    del H
    sq, sk = rosa.discretize_pair(qv, kv, M)
    R = ch // M
    qh, kh = sq.view(R, T).cpu().numpy(), sk.view(R, T).cpu().numpy()
    _check(_gpu_cf(rosa, qh, kh, None, M, 2), qh, kh, None, M, 2, "qwen-proj-64")


def test_cf_full_zipf_256_131k(rosa):
    """All 128 streams in one call (M = 8: sixteen branches per position);
    compared with the oracle 32 streams at a time to bound host memory."""
    w = workloads.zipf_planted()
    out = _gpu_cf(rosa, w.q, w.k, None, 8, w.g)
    for s0 in range(0, w.S, 32):
        _check(out, w.q, w.k, None, 8, w.g, f"zipf-256-131k streams {s0}..", streams=slice(s0, s0 + 32))
