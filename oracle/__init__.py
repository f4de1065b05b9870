"""CPU oracle for the ROSA retrieval step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
(``suffix_automaton_retrieval_b200``) and never imports it.

The arithmetic lives in ``rosa_oracle.c`` (plain C, compiled here with gcc);
this module only marshals numpy arrays.  Citations are to "ROSA-Tuning:
Enhancing Windowed Attention with Global Recall" (arXiv 2602.02499):

* ``discretize`` -- section 3.2, Eqs. (10)-(15); section 4.1 (R = C / M).
* ``match_brute`` -- the definition of the retrieval destination, section 3.3
  Eq. (16) and appendix B.3, written out as an O(T^2) longest-common-suffix
  recurrence.
* ``match_sam`` -- the online suffix automaton of section 2.2 run in lockstep
  with the query stream (appendix B.3: tau = endpos + 1).
* ``gather`` -- appendix C.4 read-out at tau with the Eq. (17) mask.
* ``match_rle_brute`` / ``match_rle_sam`` -- run-level retrieval with
  adjacent folding (section 3.3, the run-length encoding paragraph): both
  streams folded into runs, the answer taken per query run at its start
  time and mapped back to the start of the next key run (definition and
  automaton forms).
* ``inject`` -- appendix C.3, Eqs. (21)-(22): the recalled bits embedded as
  y = m((1 - b)e0 + b e1) and injected as W_out y (double precision).
* ``ln_project`` / ``ln_project_discretize`` -- section 3.2: U = LN(H),
  the query and key projections, then the strict threshold and packing.
* ``match_cf_brute`` / ``match_cf_sam`` -- the per-bit counterfactual
  destinations of section 3.5: every query bit forced to 0 and to 1, one
  retrieval step each from the same historical state (definition and
  automaton forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rosa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``rosa_oracle.c`` into ``liboracle.so`` (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i32p = ctypes.POINTER(ctypes.c_int32)
        c_int = ctypes.c_int
        lib.oracle_discretize.argtypes = [u16p, c_int, c_int, c_int, c_int, u8p]
        lib.oracle_match_brute.argtypes = [u8p, u8p, u8p, c_int, c_int, c_int, i32p, i32p, i32p]
        lib.oracle_match_sam.argtypes = [u8p, u8p, u8p, c_int, c_int, c_int, i32p, i32p, i32p, c_int]
        lib.oracle_gather.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, i32p,
                                      c_int, c_int, c_int, c_int, u16p]
        f64p = ctypes.POINTER(ctypes.c_double)
        f32p = ctypes.POINTER(ctypes.c_float)
        lib.oracle_inject.argtypes = [i32p, u16p, u16p, u16p, c_int, c_int, c_int, c_int, c_int, f64p]
        lib.oracle_ln_project.argtypes = [u16p, f32p, f32p, u16p, c_int, c_int, c_int, ctypes.c_double, f64p, f64p]
        lib.oracle_match_rle_brute.argtypes = [u8p, u8p, u8p, c_int, c_int, c_int, i32p, i32p, i32p]
        lib.oracle_match_rle_sam.argtypes = [u8p, u8p, u8p, c_int, c_int, c_int, i32p, i32p, i32p, c_int]
        lib.oracle_match_cf_brute.argtypes = [u8p, u8p, c_int, c_int, c_int, c_int, i32p, i32p]
        lib.oracle_match_cf_sam.argtypes = [u8p, u8p, c_int, c_int, c_int, c_int, i32p, i32p, c_int]
        for f in (lib.oracle_discretize, lib.oracle_match_brute, lib.oracle_match_sam, lib.oracle_gather,
                  lib.oracle_match_cf_brute, lib.oracle_match_cf_sam, lib.oracle_match_rle_brute,
                  lib.oracle_match_rle_sam, lib.oracle_inject, lib.oracle_ln_project):
            f.restype = c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def discretize(x_bits: np.ndarray, M: int) -> np.ndarray:
    """bf16 bit patterns ``[B, T, C]`` (uint16) -> uint8 symbols ``[B, C//M, T]``."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    B, T, C = x_bits.shape
    if M < 1 or M > 8 or C % M:
        raise ValueError("need 1 <= M <= 8 and C % M == 0")
    out = np.empty((B, C // M, T), dtype=np.uint8)
    _check(_load().oracle_discretize(_ptr(x_bits, ctypes.c_uint16), B, T, C, M,
                                     _ptr(out, ctypes.c_uint8)), "discretize")
    return out


def _match(fn: str, q, k, v, g, threads=None):
    q = np.ascontiguousarray(q, dtype=np.uint8)
    k = np.ascontiguousarray(k, dtype=np.uint8)
    if q.ndim == 1:
        q, k = q[None], k[None]
        if v is not None:
            v = np.asarray(v)[None]
    S, T = q.shape
    if k.shape != (S, T):
        raise ValueError("q and k must have the same shape [S, T]")
    v = k if v is None else np.ascontiguousarray(v, dtype=np.uint8)
    if v.shape != (S, T):
        raise ValueError("v must have shape [S, T]")
    end = np.empty((S, T), np.int32)
    ln = np.empty((S, T), np.int32)
    sym = np.empty((S, T), np.int32)
    lib = _load()
    args = [_ptr(q, ctypes.c_uint8), _ptr(k, ctypes.c_uint8), _ptr(v, ctypes.c_uint8), S, T, g,
            _ptr(end, ctypes.c_int32), _ptr(ln, ctypes.c_int32), _ptr(sym, ctypes.c_int32)]
    if fn in ("sam", "rle_sam"):
        args.append(threads if threads else (os.cpu_count() or 1))
    _check(getattr(lib, "oracle_match_" + fn)(*args), "match_" + fn)
    return end, ln, sym


def match_brute(q, k, v=None, g: int = 2):
    """Definition-level matcher, O(T^2) per stream.  Returns (end_idx, len, sym)."""
    return _match("brute", q, k, v, g)


def match_sam(q, k, v=None, g: int = 2, threads: int | None = None):
    """Online suffix-automaton matcher over host threads.  Returns (end_idx, len, sym)."""
    return _match("sam", q, k, v, g, threads)


def match_rle_brute(q, k, v=None, g: int = 2):
    """Run-level retrieval by the definition over runs, O(runs^2) per stream.
    Returns per-time-step (end_idx, len, sym); tau = end_idx + 1 is the start
    of the key run after the matched one, len counts runs."""
    return _match("rle_brute", q, k, v, g)


def match_rle_sam(q, k, v=None, g: int = 2, threads: int | None = None):
    """Run-level retrieval with suffix automata over the key runs, host threads."""
    return _match("rle_sam", q, k, v, g, threads)


def _match_cf(fn: str, q, k, M, g, threads=None):
    q = np.ascontiguousarray(q, dtype=np.uint8)
    k = np.ascontiguousarray(k, dtype=np.uint8)
    if q.ndim == 1:
        q, k = q[None], k[None]
    S, T = q.shape
    if k.shape != (S, T):
        raise ValueError("q and k must have the same shape [S, T]")
    if M < 1 or M > 8 or (q.size and int(q.max()) >= (1 << M)):
        raise ValueError("need 1 <= M <= 8 and query symbols below 2^M")
    end = np.empty((S, T, M, 2), np.int32)
    ln = np.empty((S, T, M, 2), np.int32)
    lib = _load()
    args = [_ptr(q, ctypes.c_uint8), _ptr(k, ctypes.c_uint8), S, T, M, g,
            _ptr(end, ctypes.c_int32), _ptr(ln, ctypes.c_int32)]
    if fn == "sam":
        args.append(threads if threads else (os.cpu_count() or 1))
        _check(lib.oracle_match_cf_sam(*args), "match_cf_sam")
    else:
        _check(lib.oracle_match_cf_brute(*args), "match_cf_brute")
    return end, ln


def match_cf_brute(q, k, M: int, g: int = 2):
    """Counterfactual destinations by the definition.  Returns (end_idx, len),
    each ``[S, T, M, 2]``: position t with query bit j forced to beta."""
    return _match_cf("brute", q, k, M, g)


def match_cf_sam(q, k, M: int, g: int = 2, threads: int | None = None):
    """Counterfactual destinations with the suffix automaton (same layout)."""
    return _match_cf("sam", q, k, M, g, threads)


def gather(V_bits: np.ndarray, end_idx: np.ndarray, R: int, d: int, rho: int) -> np.ndarray:
    """Row read-out at tau = end_idx + 1.

    ``V_bits``: ``[B, T, Cv]`` uint16 (bf16 bits); route r reads columns
    ``r*rho .. r*rho + d``.  ``end_idx``: ``[B*R, T]`` int32.
    Returns ``[B, T, R*d]`` uint16, zero rows where end_idx = -1.
    """
    V_bits = np.ascontiguousarray(V_bits, dtype=np.uint16)
    end_idx = np.ascontiguousarray(end_idx, dtype=np.int32)
    B, T, Cv = V_bits.shape
    if end_idx.shape != (B * R, T):
        raise ValueError("end_idx must be [B*R, T]")
    if (R - 1) * rho + d > Cv:
        raise ValueError("route slice exceeds the V row")
    out = np.empty((B, T, R * d), np.uint16)
    _check(_load().oracle_gather(_ptr(V_bits, ctypes.c_uint16), Cv, rho, _ptr(end_idx, ctypes.c_int32),
                                 B, R, T, d, _ptr(out, ctypes.c_uint16)), "gather")
    return out


def inject(sym: np.ndarray, e0_bits: np.ndarray, e1_bits: np.ndarray, W_bits: np.ndarray, B: int, R: int,
           M: int) -> np.ndarray:
    """Read-out embedding and injection (appendix C.3).  ``sym``: int32
    ``[B*R, T]`` recalled value symbols (-1: no match); ``e0_bits``,
    ``e1_bits``: uint16 ``[C]`` (C = R*M, bf16 bits); ``W_bits``: uint16
    ``[D, C]``.  Returns float64 ``[B, T, D]``."""
    sym = np.ascontiguousarray(sym, dtype=np.int32)
    e0 = np.ascontiguousarray(e0_bits, dtype=np.uint16)
    e1 = np.ascontiguousarray(e1_bits, dtype=np.uint16)
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    if sym.ndim != 2 or sym.shape[0] != B * R:
        raise ValueError("sym must be [B*R, T]")
    T = sym.shape[1]
    C = R * M
    if e0.shape != (C,) or e1.shape != (C,) or W.ndim != 2 or W.shape[1] != C:
        raise ValueError("e0, e1 must be [C] and W [D, C] with C = R*M")
    D = W.shape[0]
    out = np.empty((B, T, D), np.float64)
    _check(_load().oracle_inject(_ptr(sym, ctypes.c_int32), _ptr(e0, ctypes.c_uint16), _ptr(e1, ctypes.c_uint16),
                                 _ptr(W, ctypes.c_uint16), B, R, M, T, D, _ptr(out, ctypes.c_double)), "inject")
    return out


def ln_project(H_bits: np.ndarray, W_bits: np.ndarray, gamma=None, beta=None, eps: float = 1e-5):
    """U = LN(H) then U W (section 3.2), double precision.  ``H_bits``: uint16
    ``[rows, D]``; ``W_bits``: uint16 ``[D, N]``; ``gamma``, ``beta``: float32
    ``[D]`` or None.  Returns (P ``[rows, N]``, A ``[rows, N]``) with
    A = sum_k |u_k W[k, n]| (the scale of rounding errors in P)."""
    H = np.ascontiguousarray(H_bits, dtype=np.uint16)
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, D = H.shape
    if W.shape[0] != D:
        raise ValueError("W must be [D, N]")
    N = W.shape[1]
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float32)
    b = None if beta is None else np.ascontiguousarray(beta, dtype=np.float32)
    out = np.empty((rows, N), np.float64)
    mag = np.empty((rows, N), np.float64)
    f32 = ctypes.POINTER(ctypes.c_float)
    _check(_load().oracle_ln_project(_ptr(H, ctypes.c_uint16), _ptr(g, ctypes.c_float) if g is not None
                                     else ctypes.cast(None, f32), _ptr(b, ctypes.c_float) if b is not None
                                     else ctypes.cast(None, f32), _ptr(W, ctypes.c_uint16), rows, D, N, float(eps),
                                     _ptr(out, ctypes.c_double), _ptr(mag, ctypes.c_double)), "ln_project")
    return out, mag


def pack_bits(P: np.ndarray, B: int, T: int, M: int) -> np.ndarray:
    """Strict threshold and multi-route packing of section 3.2 (Eqs. 10-15)
    on real values ``P`` ``[B*T, C]``: symbols ``[B, C//M, T]``."""
    C = P.shape[1]
    bits = (P > 0).astype(np.uint8).reshape(B, T, C // M, M)
    sym = np.zeros((B, T, C // M), np.uint8)
    for j in range(M):
        sym += bits[..., j] << j
    return np.ascontiguousarray(sym.transpose(0, 2, 1))
