"""Parity of the fused layer norm + projection + discretisation (section 3.2
of "ROSA-Tuning", arXiv 2602.02499: U = LN(H), Q = U W_q, K = U W_k, the
strict threshold and packing) with the double-precision oracle.

The kernel folds the layer norm into the contraction and multiplies the raw
rows by gamma o W held as a bf16 high + low pair, accumulating in fp32.  Its
projection therefore differs from the exact one by at most
  rstd * (2^-16 + 2 D 2^-24) * sum_k |h_k| |gamma_k W_kn|
  + D 2^-24 * (|mu| rstd sum_k |gamma_k W_kn| + sum_k |beta_k W_kn|)
plus a few fp32 roundings of the epilogue (covered by 2^-20 |P|).  Where
the exact projection is farther from zero than that, the symbol bit must
match; the few channels inside the band may take either bit.  Inputs whose
arithmetic is exact (small integers, power-of-two width, no affine) must
match everywhere.
"""
import numpy as np
import pytest
import torch

import oracle
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
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _check(rosa, H, Wq, Wk, M, gamma=None, beta=None, eps=1e-5, exact=False, tag=""):
    B, T, D = H.shape
    C = Wq.shape[1]
    sq, sk = rosa.ln_project_discretize(H.to(DEV), Wq.to(DEV), Wk.to(DEV), M,
                                        None if gamma is None else gamma.to(DEV),
                                        None if beta is None else beta.to(DEV), eps=eps)
    torch.cuda.synchronize()
    hb = _bits(H).reshape(B * T, D)
    W = np.concatenate([_bits(Wq), _bits(Wk)], axis=1)                  # [D, 2C]
    g = None if gamma is None else gamma.numpy()
    b = None if beta is None else beta.numpy()
    P, A = oracle.ln_project(hb, W, g, b, eps=eps)
    got_q, got_k = sq.cpu().numpy(), sk.cpu().numpy()
    if exact:
        # integer rows and weights: the exact projection is rstd * (an integer / D), so it is
        # either 0 (bit 0 under the strict threshold) or at least rstd / D away from it; the
        # double-precision evaluation of a zero lands within 1e-9 A of it
        Pz = np.where(np.abs(P) <= 1e-9 * A, 0.0, P)
        assert np.array_equal(got_q, oracle.pack_bits(Pz[:, :C], B, T, M)), tag
        assert np.array_equal(got_k, oracle.pack_bits(Pz[:, C:], B, T, M)), tag
        return 0.0
    # the rounding band of the kernel's arithmetic, per (row, channel)
    h = _f(hb)
    mu = h.mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(((h - mu) ** 2).mean(axis=1, keepdims=True) + eps)
    gw = np.abs((np.ones(D) if g is None else g.astype(np.float64))[:, None] * _f(W))
    bw = np.abs((np.zeros(D) if b is None else b.astype(np.float64))[:, None] * _f(W)).sum(axis=0)
    band = (rstd * (2.0 ** -16 + 2 * D * 2.0 ** -24) * (np.abs(h) @ gw)
            + D * 2.0 ** -24 * (np.abs(mu) * rstd * gw.sum(axis=0) + bw) + 2.0 ** -20 * np.abs(P))
    sure = np.abs(P) > band                                                # [B*T, 2C]
    # expand the symbols back to bits and compare where the decision is sure
    def unpack(sym):
        # [B, C//M, T] -> [B*T, C] bits
        bits = ((sym[..., None] >> np.arange(M)) & 1).transpose(0, 2, 1, 3).reshape(B * T, -1)
        return bits
    got = np.concatenate([unpack(got_q), unpack(got_k)], axis=1)
    want = (P > 0).astype(np.uint8)
    bad = (got != want) & sure
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{tag}: {bad.sum()} sure bits differ; first {i}: P={P[i]} band={band[i]}")
    return float((~sure).mean())


@pytest.mark.parametrize("B,T,D,C,M,affine", [(1, 300, 256, 16, 1, False), (2, 130, 512, 32, 2, True),
                                              (1, 257, 2048, 64, 1, True), (1, 100, 128, 24, 3, False),
                                              (1, 129, 64, 40, 5, True), (2, 65, 192, 8, 8, False),
                                              (1, 140, 1024, 96, 4, True)])
def test_ln_project_parity(rosa, B, T, D, C, M, affine):
    g = torch.Generator().manual_seed(B + T + D + C + M)
    H = torch.randn(B, T, D, generator=g).to(torch.bfloat16)
    Wq = (torch.randn(D, C, generator=g) * D ** -0.5).to(torch.bfloat16)
    Wk = (torch.randn(D, C, generator=g) * D ** -0.5).to(torch.bfloat16)
    gamma = (1 + 0.3 * torch.randn(D, generator=g)).float() if affine else None
    beta = (0.1 * torch.randn(D, generator=g)).float() if affine else None
    frac = _check(rosa, H, Wq, Wk, M, gamma, beta, tag=f"B={B} T={T} D={D} C={C} M={M}")
    assert frac < 0.05                     # the undecided band stays narrow


def test_ln_project_exact_integers(rosa):
    """Small integers, D a power of two, no affine: every sum in the kernel is
    exact in fp32, so every bit must match (exact zeros give bit 0)."""
    g = torch.Generator().manual_seed(8)
    B, T, D, C, M = 1, 333, 256, 32, 2
    H = torch.randint(-8, 9, (B, T, D), generator=g).to(torch.bfloat16)
    Wq = torch.randint(-2, 3, (D, C), generator=g).to(torch.bfloat16)
    Wk = torch.randint(-2, 3, (D, C), generator=g).to(torch.bfloat16)
    _check(rosa, H, Wq, Wk, M, eps=0.0, exact=True, tag="integers")


def test_ln_project_qwen_proj_64_workload(rosa):
    """The Qwen3-1.7B-shaped workload: 32768 positions of width 2048 onto 64
    query and 64 key channels (M = 1), with a seeded layer norm."""
    c = workloads.spec("qwen-proj-64")
    H, Wq, Wk = workloads.qwen_projection_inputs(T=c["T"], width=c["width"], channels=c["channels"])
    g = torch.Generator().manual_seed(35)
    gamma = (1 + 0.2 * torch.randn(c["width"], generator=g)).float()
    beta = (0.05 * torch.randn(c["width"], generator=g)).float()
    frac = _check(rosa, H, Wq, Wk, c["M"], gamma, beta, tag="qwen-proj-64")
    assert frac < 0.02
