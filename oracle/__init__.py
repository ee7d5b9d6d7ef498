"""CPU oracle for the RRAttention prefill path -- TEST INFRASTRUCTURE ONLY.

Plain double-precision C (``rr_oracle.c``) behind ctypes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg import this package;
the product library never does, and the two share no code.

Each function follows the RRAttention paper (paperpeel.com/paper/2602.05853); the
per-step citations and the readings of the passages the extracted pages lost are in
the header of ``rr_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rr_oracle.c")
_LIB = os.path.join(_HERE, "librro.so")

HEAD_RR, NO_RR, LAYER_RR, HYBRID_RR = 0, 1, 2, 3

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with plain -O2 (no fast-math: IEEE double semantics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    # RRO_LIB_OVERRIDE: the mutation tests load deliberately broken copies of the oracle.
    lib = ctypes.CDLL(os.environ.get("RRO_LIB_OVERRIDE") or build())
    P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_double
    lib.rro_threads.restype = I
    lib.rro_offset.argtypes = [I, I, I, I]
    lib.rro_offset.restype = I
    lib.rro_sample_position.argtypes = [L, I, I, I, I]
    lib.rro_sample_position.restype = L
    lib.rro_pool_keys.argtypes = [P, I, I, I, I, P]
    lib.rro_pool_keys.restype = None
    lib.rro_estimate.argtypes = [P, P, I, I, I, I, I, I, I, I, I, I, P]
    lib.rro_estimate.restype = I
    lib.rro_xattn_estimate.argtypes = [P, P, I, I, I, I, I, I, I, I, P]
    lib.rro_xattn_estimate.restype = I
    lib.rro_select.argtypes = [P, I, I, D, I, P, P, ctypes.c_int64, P]
    lib.rro_select.restype = I
    lib.rro_prefill_rows.argtypes = [P, P, P, I, I, I, I, I, P, P, D, P, ctypes.c_int64, P]
    lib.rro_prefill_rows.restype = I
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _u16(x) -> np.ndarray:
    """bf16 torch tensor or uint16 array -> contiguous uint16 numpy array."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        x = x.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16
    return a


def threads() -> int:
    return _load().rro_threads()


def offset(h: int, S: int, mode: int = HEAD_RR, layer: int = 0) -> int:
    """Offset of the sampled query within each stride for head h."""
    return _load().rro_offset(h, S, mode, layer)


def sample_position(i: int, h: int, S: int, mode: int = HEAD_RR, layer: int = 0) -> int:
    """P(i, h): the position sampled from stride i for head h."""
    return _load().rro_sample_position(i, h, S, mode, layer)


def pool_keys(K, S: int) -> np.ndarray:
    """Kbar[g][j] = sum of the S keys of stride j; returns float64 [Hkv][L/S][d]."""
    k = _u16(K)
    Hkv, L, d = k.shape
    out = np.empty((Hkv, L // S, d), np.float64)
    _load().rro_pool_keys(_ptr(k), Hkv, L, d, S, _ptr(out))
    return out


def estimate(Q, K, S: int, B: int, mode: int = HEAD_RR, layer: int = 0,
             heads: Optional[Tuple[int, int]] = None) -> np.ndarray:
    """Block importance A[H][Nb][Nb] (float64); rows of heads outside ``heads`` are zero."""
    q, k = _u16(Q), _u16(K)
    H, L, d = q.shape
    Hkv = k.shape[0]
    Nb = L // B
    A = np.zeros((H, Nb, Nb), np.float64)
    h0, h1 = heads if heads is not None else (0, H)
    rc = _load().rro_estimate(_ptr(q), _ptr(k), H, Hkv, L, d, S, B, mode, layer, h0, h1, _ptr(A))
    if rc:
        raise ValueError(f"oracle estimate rejected the arguments (code {rc})")
    return A


def xattn_estimate(Q, K, S: int, B: int, heads: Optional[Tuple[int, int]] = None) -> np.ndarray:
    """XAttention's antidiagonal block importance A[H][Nb][Nb] (float64), the comparison
    estimator; rows of heads outside ``heads`` are zero."""
    q, k = _u16(Q), _u16(K)
    H, L, d = q.shape
    Hkv = k.shape[0]
    Nb = L // B
    A = np.zeros((H, Nb, Nb), np.float64)
    h0, h1 = heads if heads is not None else (0, H)
    rc = _load().rro_xattn_estimate(_ptr(q), _ptr(k), H, Hkv, L, d, S, B, h0, h1, _ptr(A))
    if rc:
        raise ValueError(f"oracle xattn_estimate rejected the arguments (code {rc})")
    return A


def select(A: np.ndarray, tau: float, protect_last: bool = True, diag: bool = False):
    """Top-tau CSR: returns (row_ptr int32 [H*Nb+1], col_idx int32 [nnz][, diag [H*Nb][5]])."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    H, Nb, _ = A.shape
    cap = H * Nb * (Nb + 1) // 2
    row_ptr = np.zeros(H * Nb + 1, np.int32)
    col_idx = np.zeros(max(cap, 1), np.int32)
    dg = np.zeros((H * Nb, 5), np.float64) if diag else None
    rc = _load().rro_select(_ptr(A), H, Nb, float(tau), int(bool(protect_last)), _ptr(row_ptr),
                            _ptr(col_idx), cap, _ptr(dg) if diag else None)
    if rc:
        raise ValueError(f"oracle select failed (code {rc})")
    col_idx = col_idx[: row_ptr[-1]].copy()
    return (row_ptr, col_idx, dg) if diag else (row_ptr, col_idx)


def prefill_rows(Q, K, V, B: int, row_ptr: np.ndarray, col_idx: np.ndarray, rows,
                 scale: float = 0.0) -> np.ndarray:
    """Attention output (float64 [n][d]) for the query rows ``rows`` = [(h, q), ...]."""
    q, k, v = _u16(Q), _u16(K), _u16(V)
    H, L, d = q.shape
    Hkv = k.shape[0]
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    if ci.size == 0:
        ci = np.zeros(1, np.int32)
    rw = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    out = np.zeros((rw.shape[0], d), np.float64)
    rc = _load().rro_prefill_rows(_ptr(q), _ptr(k), _ptr(v), H, Hkv, L, d, B, _ptr(rp), _ptr(ci),
                                  float(scale), _ptr(rw), rw.shape[0], _ptr(out))
    if rc:
        raise ValueError(f"oracle prefill rejected the arguments (code {rc})")
    return out


def full_csr(H: int, Nb: int) -> Tuple[np.ndarray, np.ndarray]:
    """CSR that keeps every causal block (J <= I) of every row."""
    counts = np.tile(np.arange(1, Nb + 1, dtype=np.int64), H)
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    col_idx = np.concatenate([np.arange(I + 1) for _ in range(H) for I in range(Nb)]
                             ).astype(np.int32) if H * Nb else np.zeros(0, np.int32)
    return row_ptr, col_idx
