"""ctypes binding of ``librosa_b200.so`` (C ABI in ``include/rosa.h``).

Argument marshalling only: every step of the retrieval runs in the CUDA
library.  Tensors must be CUDA tensors; there is no CPU fallback, and
importing this module fails loudly when the library has not been built.
torch is used for device memory and the current CUDA stream.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librosa_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"CUDA library {LIB_PATH} is missing: build it with "
        "`python -m suffix_automaton_retrieval_b200.build` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
lib.rosa_status_string.argtypes = [_i]
lib.rosa_status_string.restype = ctypes.c_char_p
lib.rosa_discretize.argtypes = [_vp, _i, _i, _i, _i, _vp, _vp]
lib.rosa_discretize.restype = _i
lib.rosa_discretize_pair.argtypes = [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]
lib.rosa_discretize_pair.restype = _i
lib.rosa_match_workspace_size.argtypes = [_i, _i, _i]
lib.rosa_match_workspace_size.restype = ctypes.c_size_t
lib.rosa_match.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.rosa_match.restype = _i
lib.rosa_match_cf_workspace_size.argtypes = [_i, _i, _i]
lib.rosa_match_cf_workspace_size.restype = ctypes.c_size_t
lib.rosa_match_cf.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.rosa_match_cf.restype = _i
lib.rosa_match_cf_launch_count.argtypes = [_i, _i, _i, _i]
lib.rosa_match_cf_launch_count.restype = _i
lib.rosa_match_rle_workspace_size.argtypes = [_i, _i, _i]
lib.rosa_match_rle_workspace_size.restype = ctypes.c_size_t
lib.rosa_match_rle.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.rosa_match_rle.restype = _i
lib.rosa_match_rle_launch_count.argtypes = [_i, _i, _i, _i]
lib.rosa_match_rle_launch_count.restype = _i
lib.rosa_match_launch_count.argtypes = [_i, _i, _i, _i]
lib.rosa_match_launch_count.restype = _i
lib.rosa_match_device_status.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
lib.rosa_match_device_status.restype = _i
lib.rosa_ln_project_workspace_size.argtypes = [_i, _i, _i]
lib.rosa_ln_project_workspace_size.restype = ctypes.c_size_t
lib.rosa_ln_project_discretize.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp,
                                           _vp, ctypes.c_size_t, _vp, _vp]
lib.rosa_ln_project_discretize.restype = _i
lib.rosa_inject.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp]
lib.rosa_inject.restype = _i
lib.rosa_gather.argtypes = [_vp, _i64, _i64, _vp, _i, _i, _i, _i, _vp, _vp]
lib.rosa_gather.restype = _i

EXPORTED = ("rosa_status_string", "rosa_discretize", "rosa_discretize_pair", "rosa_match_workspace_size", "rosa_match",
            "rosa_match_launch_count", "rosa_match_device_status", "rosa_gather", "rosa_match_rle",
            "rosa_match_rle_workspace_size", "rosa_match_rle_launch_count", "rosa_match_cf",
            "rosa_match_cf_workspace_size", "rosa_match_cf_launch_count", "rosa_inject",
            "rosa_ln_project_discretize", "rosa_ln_project_workspace_size")

DEV_SYMBOL_RANGE = 1


class RosaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


def status_string(code: int) -> str:
    return lib.rosa_status_string(code).decode()


def _check(code: int, what: str):
    if code != 0:
        raise RosaError(code, what)


def _stream(device) -> _vp:
    return _vp(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("the ROSA retrieval step runs on CUDA tensors only")


def _ptr(t):
    return _vp(t.data_ptr()) if t is not None and t.numel() > 0 else _vp(None)


def discretize(x: torch.Tensor, M: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 ``[B, T, C]`` -> uint8 symbols ``[B, C // M, T]`` (Eqs. 10-15)."""
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 3:
        raise ValueError("x must be a bf16 tensor [B, T, C]")
    x = x.contiguous()
    B, T, C = x.shape
    if M < 1 or M > 8 or C % M:
        raise ValueError("need 1 <= M <= 8 and C % M == 0")
    if out is None:
        out = torch.empty((B, C // M, T), dtype=torch.uint8, device=x.device)
    _check(lib.rosa_discretize(_ptr(x), B, T, C, M, _ptr(out), _stream(x.device)), "rosa_discretize")
    return out


def discretize_pair(xq: torch.Tensor, xk: torch.Tensor, M: int, out=None):
    """The query and key projections, both bf16 ``[B, T, C]``, discretised in
    one launch -> ``(sym_q, sym_k)``, each uint8 ``[B, C // M, T]``."""
    _need_cuda(xq, xk)
    for x in (xq, xk):
        if x.dtype != torch.bfloat16 or x.dim() != 3:
            raise ValueError("xq and xk must be bf16 tensors [B, T, C]")
    if xq.shape != xk.shape:
        raise ValueError("xq and xk must have the same shape")
    xq, xk = xq.contiguous(), xk.contiguous()
    B, T, C = xq.shape
    if M < 1 or M > 8 or C % M:
        raise ValueError("need 1 <= M <= 8 and C % M == 0")
    if out is None:
        out = tuple(torch.empty((B, C // M, T), dtype=torch.uint8, device=xq.device) for _ in range(2))
    sq, sk = out
    _check(lib.rosa_discretize_pair(_ptr(xq), _ptr(xk), B, T, C, M, _ptr(sq), _ptr(sk), _stream(xq.device)),
           "rosa_discretize_pair")
    return sq, sk


def match_workspace_size(S: int, T: int, K: int) -> int:
    n = lib.rosa_match_workspace_size(S, T, K)
    if n == 0:
        raise ValueError(f"invalid match sizes S={S} T={T} K={K}")
    return n


def alloc_workspace(S: int, T: int, K: int, device) -> torch.Tensor:
    return torch.empty(match_workspace_size(S, T, K), dtype=torch.uint8, device=device)


def match(q: torch.Tensor, k: torch.Tensor | None = None, v: torch.Tensor | None = None, *, K: int = 256,
          g: int = 2, out=None, workspace: torch.Tensor | None = None):
    """Suffix retrieval over S streams (section 3.3, Eq. 16; appendix B.3).

    ``q``, ``k``, ``v``: uint8 ``[S, T]`` CUDA tensors; ``k=None`` (or the
    same tensor as ``q``) selects self-retrieval, ``v=None`` reads values
    from ``k``.  Returns int32 ``(end_idx, len, sym)``, each ``[S, T]``.
    """
    _need_cuda(q, k, v, workspace)
    same = k is None or k is q
    if q.dtype != torch.uint8 or q.dim() != 2:
        raise ValueError("q must be uint8 [S, T]")
    q = q.contiguous()
    k = q if same else k.contiguous()
    S, T = q.shape
    if k.shape != q.shape or k.dtype != torch.uint8:
        raise ValueError("k must be uint8 with the shape of q")
    if v is not None:
        v = v.contiguous()
        if v.shape != q.shape or v.dtype != torch.uint8:
            raise ValueError("v must be uint8 with the shape of q")
    if out is None:
        out = tuple(torch.empty((S, T), dtype=torch.int32, device=q.device) for _ in range(3))
    end_idx, ln, sym = out
    if workspace is None:
        workspace = alloc_workspace(S, T, K, q.device)
    _check(lib.rosa_match(_ptr(q), _ptr(k), _ptr(v), S, T, K, g, _ptr(end_idx), _ptr(ln), _ptr(sym),
                          _vp(workspace.data_ptr()), workspace.numel(), _stream(q.device)), "rosa_match")
    return end_idx, ln, sym


def _match_args(q, k, v):
    same = k is None or k is q
    if q.dtype != torch.uint8 or q.dim() != 2:
        raise ValueError("q must be uint8 [S, T]")
    q = q.contiguous()
    k = q if same else k.contiguous()
    if k.shape != q.shape or k.dtype != torch.uint8:
        raise ValueError("k must be uint8 with the shape of q")
    if v is not None:
        v = v.contiguous()
        if v.shape != q.shape or v.dtype != torch.uint8:
            raise ValueError("v must be uint8 with the shape of q")
    return q, k, v


def match_cf_workspace_size(S: int, T: int, M: int) -> int:
    n = lib.rosa_match_cf_workspace_size(S, T, M)
    if n == 0:
        raise ValueError(f"invalid counterfactual sizes S={S} T={T} M={M}")
    return n


def match_cf(q: torch.Tensor, k: torch.Tensor | None = None, v: torch.Tensor | None = None, *, M: int,
             g: int = 2, out=None, workspace: torch.Tensor | None = None):
    """Ordinary retrieval plus the per-bit counterfactual destinations
    (section 3.5, appendix C.5): for every position and query bit j < M the
    branches with bit j forced to 0 and to 1.  Returns
    ``(end_idx, len, sym, end_cf, len_cf, sym_cf)``: int32 ``[S, T]`` and
    int32 ``[S, T, M, 2]`` (forced bit value last)."""
    _need_cuda(q, k, v, workspace)
    q, k, v = _match_args(q, k, v)
    S, T = q.shape
    if out is None:
        out = tuple(torch.empty((S, T), dtype=torch.int32, device=q.device) for _ in range(3)) + \
            tuple(torch.empty((S, T, M, 2), dtype=torch.int32, device=q.device) for _ in range(3))
    if workspace is None:
        workspace = torch.empty(match_cf_workspace_size(S, T, M), dtype=torch.uint8, device=q.device)
    _check(lib.rosa_match_cf(_ptr(q), _ptr(k), _ptr(v), S, T, M, g, *(_ptr(o) for o in out),
                             _vp(workspace.data_ptr()), workspace.numel(), _stream(q.device)), "rosa_match_cf")
    return out


def match_cf_launch_count(S: int, T: int, M: int, same: bool) -> int:
    n = lib.rosa_match_cf_launch_count(S, T, M, 1 if same else 0)
    if n < 0:
        raise ValueError("invalid counterfactual sizes")
    return n


def match_rle_workspace_size(S: int, T: int, K: int) -> int:
    n = lib.rosa_match_rle_workspace_size(S, T, K)
    if n == 0:
        raise ValueError(f"invalid match sizes S={S} T={T} K={K}")
    return n


def match_rle(q: torch.Tensor, k: torch.Tensor | None = None, v: torch.Tensor | None = None, *, K: int = 256,
              g: int = 2, out=None, workspace: torch.Tensor | None = None):
    """Run-level retrieval with adjacent folding (section 3.3): both streams
    fold into runs of equal symbols, each query run is answered at its start
    and the hit maps to the start of the next key run.  Same arguments and
    outputs as ``match``; ``len`` counts runs."""
    _need_cuda(q, k, v, workspace)
    q, k, v = _match_args(q, k, v)
    S, T = q.shape
    if out is None:
        out = tuple(torch.empty((S, T), dtype=torch.int32, device=q.device) for _ in range(3))
    end_idx, ln, sym = out
    if workspace is None:
        workspace = torch.empty(match_rle_workspace_size(S, T, K), dtype=torch.uint8, device=q.device)
    _check(lib.rosa_match_rle(_ptr(q), _ptr(k), _ptr(v), S, T, K, g, _ptr(end_idx), _ptr(ln), _ptr(sym),
                              _vp(workspace.data_ptr()), workspace.numel(), _stream(q.device)), "rosa_match_rle")
    return end_idx, ln, sym


def match_rle_launch_count(S: int, T: int, K: int, same: bool) -> int:
    n = lib.rosa_match_rle_launch_count(S, T, K, 1 if same else 0)
    if n < 0:
        raise ValueError("invalid match sizes")
    return n


def match_launch_count(S: int, T: int, K: int, same: bool) -> int:
    """Kernel launches one ``match`` call enqueues (reported by the library)."""
    n = lib.rosa_match_launch_count(S, T, K, 1 if same else 0)
    if n < 0:
        raise ValueError("invalid match sizes")
    return n


def match_device_status(workspace: torch.Tensor) -> int:
    st = ctypes.c_uint32(0)
    _check(lib.rosa_match_device_status(_vp(workspace.data_ptr()), _stream(workspace.device),
                                        ctypes.byref(st)), "rosa_match_device_status")
    return st.value


def gather(V: torch.Tensor, end_idx: torch.Tensor, R: int, d: int, rho: int | None = None,
           out: torch.Tensor | None = None) -> torch.Tensor:
    """Rows of ``V`` ``[B, T, W]`` at tau = end_idx + 1 -> ``[B, T, R*d]``
    (appendix C.4, Eq. 17 mask).  Route r reads columns ``r*rho .. r*rho+d``
    (``rho`` defaults to d; 0 shares one row)."""
    _need_cuda(V, end_idx)
    if V.dtype != torch.bfloat16 or V.dim() != 3 or V.stride(2) != 1:
        raise ValueError("V must be bf16 [B, T, W] with unit inner stride")
    if end_idx.dtype != torch.int32:
        raise ValueError("end_idx must be int32")
    B, T, _ = V.shape
    rho = d if rho is None else rho
    end_idx = end_idx.contiguous()
    if end_idx.shape != (B * R, T):
        raise ValueError("end_idx must be [B*R, T]")
    if V.stride(0) != T * V.stride(1):
        V = V.contiguous()
    if out is None:
        out = torch.empty((B, T, R * d), dtype=torch.bfloat16, device=V.device)
    _check(lib.rosa_gather(_ptr(V), V.stride(1), rho, _ptr(end_idx), B, R, T, d, _ptr(out),
                           _stream(V.device)), "rosa_gather")
    return out


def inject(sym: torch.Tensor, e0: torch.Tensor, e1: torch.Tensor, W_out: torch.Tensor, B: int, R: int, M: int,
           out: torch.Tensor | None = None, status: torch.Tensor | None = None) -> torch.Tensor:
    """Read-out embedding and injection (appendix C.3) on the tensor cores:
    ``sym`` int32 ``[B*R, T]`` recalled value symbols (-1: none), ``e0``,
    ``e1`` bf16 ``[R*M]``, ``W_out`` bf16 ``[D, R*M]`` -> bf16 ``[B, T, D]``."""
    _need_cuda(sym, e0, e1, W_out, out, status)
    if sym.dtype != torch.int32 or sym.dim() != 2 or sym.shape[0] != B * R:
        raise ValueError("sym must be int32 [B*R, T]")
    for t_ in (e0, e1, W_out):
        if t_.dtype != torch.bfloat16:
            raise ValueError("e0, e1 and W_out must be bf16")
    C = R * M
    if e0.numel() != C or e1.numel() != C or W_out.dim() != 2 or W_out.shape[1] != C:
        raise ValueError("e0, e1 must have R*M entries and W_out must be [D, R*M]")
    sym, e0, e1, W_out = sym.contiguous(), e0.contiguous(), e1.contiguous(), W_out.contiguous()
    T, D = sym.shape[1], W_out.shape[0]
    if out is None:
        out = torch.empty((B, T, D), dtype=torch.bfloat16, device=sym.device)
    _check(lib.rosa_inject(_ptr(sym), _ptr(e0), _ptr(e1), _ptr(W_out), B, R, M, T, D, _ptr(out),
                           _ptr(status), _stream(sym.device)), "rosa_inject")
    return out


def ln_project_workspace_size(D: int, C: int, M: int) -> int:
    n = lib.rosa_ln_project_workspace_size(D, C, M)
    if n == 0:
        raise ValueError(f"invalid sizes D={D} C={C} M={M}")
    return n


def ln_project_discretize(H: torch.Tensor, Wq: torch.Tensor, Wk: torch.Tensor, M: int,
                          gamma: torch.Tensor | None = None, beta: torch.Tensor | None = None, eps: float = 1e-5,
                          out=None, workspace: torch.Tensor | None = None, status: torch.Tensor | None = None):
    """U = LN(H), the query and key projections, threshold and packing in one
    pass (section 3.2): ``H`` bf16 ``[B, T, D]``, ``Wq``, ``Wk`` bf16
    ``[D, C]``, ``gamma``, ``beta`` float32 ``[D]`` or None ->
    ``(sym_q, sym_k)``, uint8 ``[B, C // M, T]`` each."""
    _need_cuda(H, Wq, Wk, gamma, beta, workspace, status)
    if H.dtype != torch.bfloat16 or H.dim() != 3:
        raise ValueError("H must be bf16 [B, T, D]")
    for w in (Wq, Wk):
        if w.dtype != torch.bfloat16 or w.dim() != 2:
            raise ValueError("Wq and Wk must be bf16 [D, C]")
    for v in (gamma, beta):
        if v is not None and v.dtype != torch.float32:
            raise ValueError("gamma and beta must be float32 [D]")
    H, Wq, Wk = H.contiguous(), Wq.contiguous(), Wk.contiguous()
    gamma = None if gamma is None else gamma.contiguous()
    beta = None if beta is None else beta.contiguous()
    B, T, D = H.shape
    C = Wq.shape[1]
    if Wq.shape != (D, C) or Wk.shape != (D, C):
        raise ValueError("Wq and Wk must both be [D, C]")
    if out is None:
        out = tuple(torch.empty((B, C // M, T), dtype=torch.uint8, device=H.device) for _ in range(2))
    if workspace is None:
        workspace = torch.empty(ln_project_workspace_size(D, C, M), dtype=torch.uint8, device=H.device)
    _check(lib.rosa_ln_project_discretize(_ptr(H), _ptr(gamma), _ptr(beta), _ptr(Wq), _ptr(Wk), B, T, D, C, M,
                                          float(eps), _ptr(out[0]), _ptr(out[1]), _vp(workspace.data_ptr()),
                                          workspace.numel(), _ptr(status), _stream(H.device)),
           "rosa_ln_project_discretize")
    return out
