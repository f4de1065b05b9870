"""rosa_match_noalloc: the matcher for callers that cannot allocate device
memory (hosts that own every device allocation, serving loops that must not
call cudaMalloc/cudaFree because those can synchronise the device).

It takes its scratch space from a fixed array inside the library instead of
a caller workspace.  This file runs last so that a failure here comes after
every other test has run.  Its output must equal the regular entry point's,
bit for bit, on two calls in a row (the array keeps the previous call's
contents, which must not leak into the next result).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from suffix_automaton_retrieval_b200 import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SCRATCH_BYTES = 64 << 20


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from suffix_automaton_retrieval_b200 import build
    build.build()
    import suffix_automaton_retrieval_b200.binding as b
    f = b.lib.rosa_match_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp, vp]
    f.restype = i
    return b


def _noalloc_rc(b, q, k, v, K, g):
    S, T = q.shape
    outs = [torch.full((S, T), 12345, dtype=torch.int32, device=DEV) for _ in range(3)]
    vp = ctypes.c_void_p
    rc = b.lib.rosa_match_noalloc(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()) if v is not None else None,
                                  S, T, K, g, vp(outs[0].data_ptr()), vp(outs[1].data_ptr()),
                                  vp(outs[2].data_ptr()), vp(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, outs


def _noalloc(b, q, k, v, K, g):
    rc, outs = _noalloc_rc(b, q, k, v, K, g)
    assert rc == 0, b.status_string(rc)
    return [o.cpu().numpy() for o in outs]


def _noalloc_status(b):
    st = ctypes.c_uint32(0xdead)
    f = b.lib.rosa_match_noalloc_device_status
    f.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]
    f.restype = ctypes.c_int
    rc = f(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(st))
    assert rc == 0, b.status_string(rc)
    return st.value


def _regular(b, q, k, v, K, g):
    e, l, s = b.match(q, None if k is q else k, v, K=K, g=g)
    torch.cuda.synchronize()
    return [e.cpu().numpy(), l.cpu().numpy(), s.cpu().numpy()]


def test_no_alloc_matches_regular_entry_point(lib):
    cases = [workloads.zipf_planted(S=4, T=8192, seed_q=7, seed_k=8, seed_plant=9),
             workloads.markov(B=1, R=8, T=4096, seed_q=3, seed_k=4),
             workloads.planted_copies(B=1, R=4, T=8192, seed=5)]
    for w in cases:
        q = torch.from_numpy(w.q).to(DEV)
        k = q if w.same_qk else torch.from_numpy(w.k).to(DEV)
        assert lib.match_workspace_size(w.S, w.T, w.K) <= SCRATCH_BYTES
        want = _regular(lib, q, k, None, w.K, w.g)
        for _ in range(2):                      # two calls in a row share the array
            got = _noalloc(lib, q, k, None, w.K, w.g)
            for a, b_ in zip(got, want):
                assert np.array_equal(a, b_), w.name
    # a different problem right after: nothing of the previous call leaks in
    rng = np.random.default_rng(1)
    qh = rng.integers(0, 2, (3, 1000)).astype(np.uint8)
    vh = rng.integers(0, 256, (3, 1000)).astype(np.uint8)
    q = torch.from_numpy(qh).to(DEV)
    v = torch.from_numpy(vh).to(DEV)
    got = _noalloc(lib, q, q, v, 2, 1)
    want = oracle.match_sam(qh, qh, vh, g=1)
    for a, b_ in zip(got, want):
        assert np.array_equal(a, b_)


def test_no_alloc_rejects_sizes_beyond_the_array(lib):
    S, T, K = 64, 16384, 256
    assert lib.match_workspace_size(S, T, K) > SCRATCH_BYTES
    vp = ctypes.c_void_p
    fake = vp(0x10000)   # never dereferenced: the size check comes first
    rc = lib.lib.rosa_match_noalloc(fake, vp(0x20000), None, S, T, K, 2, fake, fake, fake, None)
    assert rc == 2      # ROSA_ERR_WORKSPACE


def test_no_alloc_near_the_limit(lib):
    """The array almost full: the largest q != k problem of 16384-symbol
    streams over 256 symbols that fits, then a self-retrieval problem as
    large as the array admits, both bit-exact against rosa_match."""
    T, K = 16384, 256
    S = 1
    while lib.match_workspace_size(S + 1, T, K) <= SCRATCH_BYTES:
        S += 1
    assert lib.match_workspace_size(S, T, K) > 0.9 * SCRATCH_BYTES
    w = workloads.zipf_planted(S=S, T=T, K=K, seed_q=11, seed_k=12, seed_plant=13, lmax=512)
    q, k = torch.from_numpy(w.q).to(DEV), torch.from_numpy(w.k).to(DEV)
    want = _regular(lib, q, k, None, K, w.g)
    got = _noalloc(lib, q, k, None, K, w.g)
    for a, b_ in zip(got, want):
        assert np.array_equal(a, b_)
    assert _noalloc_status(lib) == 0
    # self-retrieval needs about half the scratch per position: grow S until rejected
    wq = workloads.planted_copies(B=1, R=3 * S, T=T, K=16, seed=21)
    Sq = 3 * S
    while True:
        qq = torch.from_numpy(np.ascontiguousarray(wq.q[:Sq])).to(DEV)
        rc, _ = _noalloc_rc(lib, qq, qq, None, 16, wq.g)
        if rc == 0:
            break
        assert rc == 2          # ROSA_ERR_WORKSPACE, nothing launched
        Sq -= 1
    assert Sq < 3 * S           # the limit was reached, not the start size
    assert Sq > S               # the self-retrieval form admits more streams
    want = _regular(lib, qq, qq, None, 16, wq.g)
    got = _noalloc(lib, qq, qq, None, 16, wq.g)
    for a, b_ in zip(got, want):
        assert np.array_equal(a, b_)


def test_no_alloc_reports_out_of_range_symbols(lib):
    rng = np.random.default_rng(3)
    qh = rng.integers(0, 4, (2, 700)).astype(np.uint8)
    qh[1, 350] = 9                            # >= K = 4: masked and flagged
    q = torch.from_numpy(qh).to(DEV)
    _noalloc(lib, q, q, None, 4, 2)
    assert _noalloc_status(lib) & lib.DEV_SYMBOL_RANGE
    qh[1, 350] = 1
    q = torch.from_numpy(qh).to(DEV)
    _noalloc(lib, q, q, None, 4, 2)
    assert _noalloc_status(lib) == 0          # cleared by the next call
