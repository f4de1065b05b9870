"""Parity of the CUDA path with the CPU oracle (needs a CUDA device).

Integer outputs (end index, length, recalled symbol) and the uint8 symbols
must be bit-exact; gathered bf16 rows must be bitwise equal (a pure copy).
Every call goes through the C ABI via the thin binding.
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


def _gpu_match(rosa, q, k, v, K, g):
    qd = torch.from_numpy(np.ascontiguousarray(q)).to(DEV)
    kd = qd if k is q else torch.from_numpy(np.ascontiguousarray(k)).to(DEV)
    vd = None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(DEV)
    e, l, s = rosa.match(qd, None if k is q else kd, vd, K=K, g=g)
    torch.cuda.synchronize()
    return e.cpu().numpy(), l.cpu().numpy(), s.cpu().numpy()


def _assert_same(got, want, tag=""):
    for name, a, b in zip(("end_idx", "len", "sym"), got, want):
        if not np.array_equal(a, b):
            bad = np.argwhere(a != b)
            s, t = bad[0]
            raise AssertionError(f"{tag} {name} differs at {len(bad)} places; first (s={s}, t={t}): "
                                 f"gpu={a[s, t]} oracle={b[s, t]}")


# ---------------------------------------------------------------- match, small

def test_match_random_small(rosa):
    rng = np.random.default_rng(2024)
    for it in range(300):
        S = int(rng.integers(1, 5))
        T = int(rng.integers(1, 300))
        K = int(rng.choice([1, 2, 3, 4, 16, 256]))
        g = int(rng.integers(1, 4))
        q = rng.integers(0, K, (S, T)).astype(np.uint8)
        mode = int(rng.integers(0, 3))
        k = q if mode == 0 else (q.copy() if mode == 1 else rng.integers(0, K, (S, T)).astype(np.uint8))
        v = rng.integers(0, 256, (S, T)).astype(np.uint8) if rng.random() < 0.3 else None
        want = oracle.match_brute(q, k, v, g=g)
        got = _gpu_match(rosa, q, k, v, K, g)
        _assert_same(got, want, f"it={it} S={S} T={T} K={K} g={g} mode={mode}")


@pytest.mark.parametrize("T", [1, 2, 3, 57, 58, 59, 60, 2047, 2048, 2049, 4096])
def test_match_tile_boundaries(rosa, T):
    rng = np.random.default_rng(T)
    for K in (2, 256):
        q = rng.integers(0, K, (3, T)).astype(np.uint8)
        k = rng.integers(0, K, (3, T)).astype(np.uint8)
        for g in (1, 2):
            _assert_same(_gpu_match(rosa, q, k, None, K, g), oracle.match_sam(q, k, g=g), f"T={T} K={K} g={g}")
            _assert_same(_gpu_match(rosa, q, q, None, K, g), oracle.match_sam(q, q, g=g), f"T={T} K={K} self")


def test_match_degenerate_streams(rosa):
    """Constant and periodic streams: deep ties, long doubling chains, big groups."""
    T = 4096
    cases = []
    cases.append((np.zeros((1, T), np.uint8), None, 1))                       # one group of ~T items
    c = np.full((2, T), 3, np.uint8)
    cases.append((c, c.copy(), 4))                                             # q != k, group > 4096
    p = (np.arange(T) % 5).astype(np.uint8)[None]
    cases.append((p, None, 5))
    ab = np.tile(np.array([0, 1], np.uint8), T // 2)[None]
    cases.append((ab, None, 2))
    for q, k, K in cases:
        k = q if k is None else k
        for g in (1, 2, 3):
            _assert_same(_gpu_match(rosa, q, k, None, K, g), oracle.match_sam(q, k, g=g), f"K={K} g={g}")


@pytest.mark.parametrize("T", [20, 32, 33, 64, 65, 128, 129, 256, 257, 1024, 1025])
def test_match_wide_intervals_near_powers_of_two(rosa, T):
    """Low-entropy streams, where many matches share a short suffix with hundreds of ranks, so
    their most recent admissible end comes from the wavelet matrix; T around powers of two moves
    the number of wavelet levels (none up to T = 32, the last five bits are always a leaf scan)."""
    rng = np.random.default_rng(300 + T)
    S = 6
    streams = [
        (np.zeros((S, T), np.uint8), 1),
        ((rng.random((S, T)) < 0.1).astype(np.uint8), 2),
        (((np.arange(T)[None, :] + rng.integers(0, 3, (S, 1))) % 3).astype(np.uint8), 3),
    ]
    for q, K in streams:
        k_ind = (rng.random((S, T)) < 0.1).astype(np.uint8) if K > 1 else np.zeros((S, T), np.uint8)
        for k in (q, q.copy(), k_ind):
            for g in (1, 2):
                want = oracle.match_brute(q, k, g=g)
                _assert_same(_gpu_match(rosa, q, k, None, K, g), want, f"T={T} K={K} g={g} k_is_q={k is q}")


def test_match_many_short_streams(rosa):
    """Many streams of a few positions: grids sized by the stream count (over 65535 streams too)."""
    rng = np.random.default_rng(77)
    for S, T, K in [(70000, 2, 256), (20000, 3, 2), (5000, 17, 4), (3000, 40, 256)]:
        q = rng.integers(0, K, (S, T)).astype(np.uint8)
        k = rng.integers(0, K, (S, T)).astype(np.uint8)
        for kk in (q, k):
            for g in (1, 2):
                _assert_same(_gpu_match(rosa, q, kk, None, K, g), oracle.match_brute(q, kk, g=g),
                             f"S={S} T={T} K={K} g={g}")


def test_match_recipes_reduced(rosa):
    """The five input recipes at sizes the oracle finishes in seconds."""
    ws = [
        workloads.binary_iid(T=4096),
        workloads.binary_iid(T=64),
        workloads.planted_copies(B=2, R=4, T=16384),
        workloads.zipf_planted(S=4, T=32768),
        workloads.markov(B=2, R=16, T=8192),
    ]
    for w in ws:
        want = oracle.match_sam(w.q, w.k, g=w.g)
        _assert_same(_gpu_match(rosa, w.q, w.k, None, w.K, w.g), want, w.name)
    # the 4096 and 64 binary streams also against the definition itself
    for w in ws[:2]:
        _assert_same(_gpu_match(rosa, w.q, w.k, None, w.K, w.g), oracle.match_brute(w.q, w.k, g=w.g), w.name)


def test_match_symbol_range_flag(rosa):
    q = torch.tensor([[0, 1, 2, 1, 0]], dtype=torch.uint8, device=DEV)
    ws = rosa.alloc_workspace(1, 5, 2, DEV)
    rosa.match(q, K=2, g=1, workspace=ws)
    assert rosa.match_device_status(ws) & rosa.DEV_SYMBOL_RANGE
    q2 = torch.tensor([[0, 1, 1, 1, 0]], dtype=torch.uint8, device=DEV)
    rosa.match(q2, K=2, g=1, workspace=ws)
    assert rosa.match_device_status(ws) == 0


def test_match_errors(rosa):
    q = torch.zeros((2, 16), dtype=torch.uint8, device=DEV)
    small = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(rosa.RosaError) as e:
        rosa.match(q, K=2, g=2, workspace=small)
    assert e.value.code == 2
    with pytest.raises(rosa.RosaError):
        rosa.match(q, K=2, g=0)


def test_match_empty(rosa):
    q = torch.zeros((0, 7), dtype=torch.uint8, device=DEV)
    e, l, s = rosa.match(q, K=4)
    assert e.shape == (0, 7)
    q = torch.zeros((3, 0), dtype=torch.uint8, device=DEV)
    e, l, s = rosa.match(q, K=4)
    assert e.shape == (3, 0)


# ---------------------------------------------------------------- discretize

def _bf16_bits_special(rng, shape):
    x = rng.standard_normal(shape).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    special = np.array([0x0000, 0x8000, 0x7FC0, 0xFFC0, 0x7F80, 0xFF80, 0x0001, 0x8001, 0x7F7F, 0xFF7F],
                       np.uint16)
    mask = rng.random(shape) < 0.1
    bits[mask] = rng.choice(special, size=int(mask.sum()))
    return bits


@pytest.mark.parametrize("B,T,C,M", [(1, 1, 8, 4), (2, 33, 64, 1), (1, 100, 16, 2), (3, 65, 24, 3),
                                     (1, 64, 2048, 4), (2, 31, 40, 8), (1, 1000, 64, 1), (1, 7, 520, 5)])
def test_discretize_parity(rosa, B, T, C, M):
    rng = np.random.default_rng(B * 1000 + T + C + M)
    bits = _bf16_bits_special(rng, (B, T, C))
    want = oracle.discretize(bits, M)
    xd = torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)
    got = rosa.discretize(xd, M)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), want)


@pytest.mark.parametrize("B,T,C,M,misalign", [(1, 65, 64, 1, False), (2, 40, 24, 3, False), (1, 33, 48, 2, True)])
def test_discretize_pair_parity(rosa, B, T, C, M, misalign):
    """Query and key in one launch: each equals the oracle's discretisation;
    with one operand at an odd element offset both take the scalar path."""
    rng = np.random.default_rng(7 * B + T + C + M)
    bq, bk = _bf16_bits_special(rng, (B, T, C)), _bf16_bits_special(rng, (B, T, C))
    xq = torch.from_numpy(bq.view(np.int16)).to(DEV).view(torch.bfloat16)
    xk = torch.from_numpy(bk.view(np.int16)).to(DEV).view(torch.bfloat16)
    if misalign:
        buf = torch.empty(xk.numel() + 1, dtype=torch.bfloat16, device=DEV)
        view = buf[1:].view(xk.shape)
        view.copy_(xk)
        xk = view
    sq, sk = rosa.discretize_pair(xq, xk, M)
    torch.cuda.synchronize()
    assert np.array_equal(sq.cpu().numpy(), oracle.discretize(bq, M))
    assert np.array_equal(sk.cpu().numpy(), oracle.discretize(bk, M))


def test_discretize_unaligned_view(rosa):
    rng = np.random.default_rng(3)
    bits = _bf16_bits_special(rng, (1, 50, 65))
    xd = torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)[:, :, 1:].contiguous()
    # a contiguous tensor at an odd element offset inside a larger buffer
    buf = torch.empty(xd.numel() + 1, dtype=torch.bfloat16, device=DEV)
    view = buf[1:].view(xd.shape)
    view.copy_(xd)
    got = rosa.discretize(view, 4)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), oracle.discretize(bits[:, :, 1:], 4))


# ---------------------------------------------------------------- gather

@pytest.mark.parametrize("B,R,T,d,rho,extra", [(1, 2, 50, 8, 8, 0), (2, 3, 40, 16, 16, 0), (1, 4, 33, 8, 0, 0),
                                               (1, 2, 20, 5, 5, 0), (2, 64, 17, 128, 128, 0),
                                               (1, 3, 30, 8, 8, 8), (1, 600, 9, 8, 8, 0)])
def test_gather_parity(rosa, B, R, T, d, rho, extra):
    rng = np.random.default_rng(B + R + T + d)
    W = (R - 1) * rho + d + extra
    Vb = rng.integers(0, 65536, (B, T, W)).astype(np.uint16)
    end = rng.integers(-1, T - 1, (B * R, T)).astype(np.int32)
    end[:, 0] = -1
    want = oracle.gather(Vb, end, R, d, rho)
    Vd = torch.from_numpy(Vb.view(np.int16)).to(DEV).view(torch.bfloat16)
    ed = torch.from_numpy(end).to(DEV)
    got = rosa.gather(Vd, ed, R, d, rho)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().view(torch.int16).numpy().view(np.uint16), want)


def test_gather_ignores_out_of_range_indices(rosa):
    T = 10
    Vd = torch.ones((1, T, 8), dtype=torch.bfloat16, device=DEV)
    end = torch.tensor([[-5, -1, 0, 8, 9, 100, 3, 2, 1, 0]], dtype=torch.int32, device=DEV)
    got = rosa.gather(Vd, end, 1, 8).float().cpu()
    ok = torch.tensor([0, 0, 1, 1, 0, 0, 1, 1, 1, 1], dtype=torch.float32)
    assert torch.equal(got[0, :, 0], ok)


# ---------------------------------------------------------------- full path on hidden states

def test_full_path_hidden_states_reduced(rosa):
    """Discretise projected hidden states, match, gather: the qwen-proj recipe
    at T=4096.  The oracle consumes the same projected bf16 tensors."""
    H, Wq, Wk = workloads.qwen_projection_inputs(T=4096, width=512, channels=16, device=DEV)
    qv = (H @ Wq).contiguous()
    kv = (H @ Wk).contiguous()
    V = workloads.value_rows(1, 4096, 16 * 32, seed=33, device=DEV)
    sq = rosa.discretize(qv, 1)
    sk = rosa.discretize(kv, 1)
    S, T = 16, 4096
    e, l, s = rosa.match(sq.view(S, T), sk.view(S, T), K=2, g=2)
    out = rosa.gather(V, e, 16, 32)
    torch.cuda.synchronize()
    qb = qv.cpu().view(torch.int16).numpy().view(np.uint16)
    kb = kv.cpu().view(torch.int16).numpy().view(np.uint16)
    oq, ok = oracle.discretize(qb, 1), oracle.discretize(kb, 1)
    assert np.array_equal(sq.cpu().numpy(), oq) and np.array_equal(sk.cpu().numpy(), ok)
    want = oracle.match_sam(oq.reshape(S, T), ok.reshape(S, T), g=2)
    _assert_same((e.cpu().numpy(), l.cpu().numpy(), s.cpu().numpy()), want, "hidden")
    Vb = V.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16),
                          oracle.gather(Vb, want[0], 16, 32, 32))
