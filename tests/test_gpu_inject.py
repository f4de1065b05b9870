"""Parity of the tensor-core read-out embedding and injection with the oracle
(appendix C.3 of "ROSA-Tuning", arXiv 2602.02499: y = m((1 - b)e0 + b e1),
inj = W_out y).

The kernel accumulates in fp32 and rounds the result to bf16, so it is
compared with the oracle's double-precision result within the bound that
arithmetic implies: half an ulp of bf16 (2^-9 relative) for the final
rounding plus at most K * 2^-24 * sum_c |W_out[d, c] y_c| for the fp32
accumulation of K = R*M products (each product of two bf16 values is exact
in fp32).  The test uses |err| <= 2^-8 |ref| + K * 2^-23 * A, twice both
terms, with A from the oracle run on |W_out|, |e0|, |e1|.
"""
import numpy as np
import pytest
import torch

import oracle

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


def _inputs(B, R, M, T, D, seed, none_frac=0.2):
    g = torch.Generator().manual_seed(seed)
    C = R * M
    sym = torch.randint(0, 1 << M, (B * R, T), generator=g, dtype=torch.int32)
    sym[torch.rand((B * R, T), generator=g) < none_frac] = -1
    e0 = torch.randn(C, generator=g).to(torch.bfloat16)
    e1 = torch.randn(C, generator=g).to(torch.bfloat16)
    W = (torch.randn(D, C, generator=g) * C ** -0.5).to(torch.bfloat16)
    return sym, e0, e1, W


def _check(got, sym, e0, e1, W, B, R, M, tag):
    s, b0, b1, bw = sym.cpu().numpy(), _bits(e0), _bits(e1), _bits(W)
    ref = oracle.inject(s, b0, b1, bw, B, R, M)
    mag = oracle.inject(s, b0 & 0x7FFF, b1 & 0x7FFF, bw & 0x7FFF, B, R, M)   # sum |W| |y|
    K = R * M
    g = _f(_bits(got)).reshape(ref.shape)
    tol = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -23 * mag + 1e-30
    bad = np.abs(g - ref) > tol
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{tag}: {bad.sum()} entries outside the bound; first {i}: gpu={g[i]} ref={ref[i]} "
                             f"tol={tol[i]}")
    # masked rows inject exactly zero
    return ref


@pytest.mark.parametrize("B,R,M,T,D", [(1, 64, 1, 300, 2048), (2, 16, 2, 200, 512), (1, 5, 3, 77, 40),
                                       (1, 256, 2, 130, 512), (1, 4, 8, 129, 300), (3, 7, 1, 33, 16),
                                       (1, 96, 2, 257, 264), (1, 160, 4, 100, 136), (2, 32, 2, 40000, 200)])
def test_inject_parity(rosa, B, R, M, T, D):
    sym, e0, e1, W = _inputs(B, R, M, T, D, seed=B * 1000 + R * 10 + M + T + D)
    got = rosa.inject(sym.to(DEV), e0.to(DEV), e1.to(DEV), W.to(DEV), B, R, M)
    torch.cuda.synchronize()
    _check(got, sym, e0, e1, W, B, R, M, f"B={B} R={R} M={M} T={T} D={D}")


def test_inject_all_masked_is_zero(rosa):
    B, R, M, T, D = 1, 8, 2, 150, 64
    sym, e0, e1, W = _inputs(B, R, M, T, D, seed=3, none_frac=1.0)
    got = rosa.inject(sym.to(DEV), e0.to(DEV), e1.to(DEV), W.to(DEV), B, R, M)
    torch.cuda.synchronize()
    assert not _bits(got).any()


def test_inject_exact_on_small_integers(rosa):
    """Integer-valued e0, e1 and W_out with small sums are exact in fp32 and
    in bf16, so the kernel must equal the oracle exactly."""
    B, R, M, T, D = 1, 16, 2, 140, 48
    g = torch.Generator().manual_seed(11)
    sym = torch.randint(-1, 4, (B * R, T), generator=g, dtype=torch.int32)
    e0 = torch.randint(-3, 4, (R * M,), generator=g).to(torch.bfloat16)
    e1 = torch.randint(-3, 4, (R * M,), generator=g).to(torch.bfloat16)
    W = torch.randint(-2, 3, (D, R * M), generator=g).to(torch.bfloat16)
    got = rosa.inject(sym.to(DEV), e0.to(DEV), e1.to(DEV), W.to(DEV), B, R, M)
    torch.cuda.synchronize()
    ref = oracle.inject(sym.numpy(), _bits(e0), _bits(e1), _bits(W), B, R, M)
    assert np.array_equal(_f(_bits(got)).reshape(ref.shape), ref)


def test_inject_full_qwen_proj_64_shape(rosa):
    """Qwen3-1.7B-shaped: 32768 positions, 64 binary routes, width 2048."""
    B, R, M, T, D = 1, 64, 1, 32768, 2048
    sym, e0, e1, W = _inputs(B, R, M, T, D, seed=64)
    got = rosa.inject(sym.to(DEV), e0.to(DEV), e1.to(DEV), W.to(DEV), B, R, M)
    torch.cuda.synchronize()
    _check(got, sym, e0, e1, W, B, R, M, "qwen-proj-64 shape")


def test_inject_full_markov_4_train_shape(rosa):
    """markov-4-train-shaped: 8 x 8192 positions, 256 routes of 2 bits (512
    channels, eight K blocks), width 512; several row tiles per CTA.  Sampled
    positions of every batch element are compared with the oracle."""
    B, R, M, T, D = 8, 256, 2, 8192, 512
    sym, e0, e1, W = _inputs(B, R, M, T, D, seed=256)
    got = rosa.inject(sym.to(DEV), e0.to(DEV), e1.to(DEV), W.to(DEV), B, R, M)
    torch.cuda.synchronize()
    sel = np.unique(np.concatenate([np.arange(0, 300), np.arange(T - 300, T),
                                    np.random.default_rng(5).choice(T, 400, replace=False)]))
    sub = sym.reshape(B, R, T)[:, :, sel].reshape(B * R, len(sel)).contiguous()
    got_sub = got.reshape(B, T, D)[:, sel, :].contiguous()
    _check(got_sub, sub, e0, e1, W, B, R, M, "markov-4-train shape (sampled)")
