"""Parity at the full sizes of the five workloads, in the launch
configuration the benchmark times (one rosa_match over all streams, one
workspace, preallocated outputs).

Every stream of every workload is compared bit for bit with the CPU
oracle's online suffix automaton (linear in T, all host cores), the
gathered rows are compared bitwise over the whole output (one batch element
at a time), and the independent invariant checker covers sampled positions
of a few streams on top.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.invariants import check_stream
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


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _run_match(rosa, q, k, K, g, same):
    S, T = q.shape
    ws = rosa.alloc_workspace(S, T, K, DEV)
    outs = tuple(torch.empty((S, T), dtype=torch.int32, device=DEV) for _ in range(3))
    rosa.match(q, None if same else k, K=K, g=g, out=outs, workspace=ws)
    torch.cuda.synchronize()
    assert rosa.match_device_status(ws) == 0
    return [o.cpu().numpy() for o in outs]


def _check_all_streams(got, qh, kh, g, tag, invariant_streams=(0,), sample_pos=40):
    """Whole outputs against the oracle; first mismatch reported by place."""
    want = oracle.match_sam(qh, kh, g=g)
    for name, a, b in zip(("end_idx", "len", "sym"), got, want):
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            s, t = bad[0]
            raise AssertionError(f"{tag}: {name} differs at {len(bad)} places; first stream {s} t={t}: "
                                 f"gpu={a[s, t]} oracle={b[s, t]}")
    for s0 in invariant_streams:
        check_stream(qh[s0], kh[s0], kh[s0], g, got[0][s0], got[1][s0], got[2][s0], full=False,
                     sample=sample_pos)
    return want


def _check_gather_all(rosa_out, V, want_end, R, d, rho, tag):
    """Bitwise comparison of the whole gathered output, one batch element at a time."""
    B = V.shape[0]
    for b in range(B):
        want = oracle.gather(_bits(V[b:b + 1]), want_end[b * R:(b + 1) * R], R, d, rho)
        got = _bits(rosa_out[b:b + 1])
        if not np.array_equal(got, want):
            bad = np.argwhere(got != want)
            raise AssertionError(f"{tag}: gather differs at {len(bad)} places; first {tuple(bad[0])}")


def _symbol_case(rosa, w):
    q = torch.from_numpy(w.q).to(DEV)
    k = q if w.same_qk else torch.from_numpy(w.k).to(DEV)
    got = _run_match(rosa, q, k, w.K, w.g, w.same_qk)
    want = _check_all_streams(got, w.q, w.k, w.g, w.name, invariant_streams=(0, w.S - 1))
    return got, want


def test_full_binary_4k(rosa):
    w = workloads.binary_iid()
    q = torch.from_numpy(w.q).to(DEV)
    got = _run_match(rosa, q, q, w.K, w.g, True)
    want = oracle.match_brute(w.q, w.q, g=w.g)      # the definition, exhaustively
    for a, b in zip(got, want):
        assert np.array_equal(a, b)
    w64 = workloads.binary_iid(T=64)
    q = torch.from_numpy(w64.q).to(DEV)
    got = _run_match(rosa, q, q, w64.K, w64.g, True)
    for a, b in zip(got, oracle.match_brute(w64.q, w64.q, g=w64.g)):
        assert np.array_equal(a, b)


def test_full_planted_16(rosa):
    got, _ = _symbol_case(rosa, workloads.planted_copies())
    assert got[1].max() >= 32          # the planted copies are found


def test_full_zipf_256_131k(rosa):
    got, _ = _symbol_case(rosa, workloads.zipf_planted())
    assert got[1].max() >= 16          # the planted repeats are found


def test_full_markov_4_train_with_gather(rosa):
    c = workloads.spec("markov-4-train")
    w = workloads.markov()
    got, want = _symbol_case(rosa, w)
    V = workloads.value_rows(w.B, w.T, w.R * c["rho"], seed=c["seed_v"], device=DEV)
    end = torch.from_numpy(got[0]).to(DEV)
    out = rosa.gather(V, end, w.R, c["d"], c["rho"])
    torch.cuda.synchronize()
    _check_gather_all(out, V, want[0], w.R, c["d"], c["rho"], w.name)


def test_full_qwen_proj_64_path(rosa):
    c = workloads.spec("qwen-proj-64")
    T, width, ch, M, d, rho = c["T"], c["width"], c["channels"], c["M"], c["d"], c["rho"]
    H, Wq, Wk = workloads.qwen_projection_inputs(T=T, width=width, channels=ch, device=DEV)
    qv, kv = (H @ Wq).contiguous(), (H @ Wk).contiguous()
    del H
    R = ch // M
    V = workloads.value_rows(1, T, R * rho, seed=c["seed_v"], device=DEV)
    sq, sk = rosa.discretize(qv, M), rosa.discretize(kv, M)
    got = _run_match(rosa, sq.view(R, T), sk.view(R, T), 2 ** M, 2, False)
    end = torch.from_numpy(got[0]).to(DEV)
    out = rosa.gather(V, end, R, d, rho)
    torch.cuda.synchronize()
    oq, ok = oracle.discretize(_bits(qv), M), oracle.discretize(_bits(kv), M)
    assert np.array_equal(sq.cpu().numpy(), oq) and np.array_equal(sk.cpu().numpy(), ok)
    qh, kh = oq.reshape(R, T), ok.reshape(R, T)
    want = _check_all_streams(got, qh, kh, 2, "qwen-proj-64", invariant_streams=(0, R - 1))
    _check_gather_all(out, V, want[0], R, d, rho, "qwen-proj-64")
