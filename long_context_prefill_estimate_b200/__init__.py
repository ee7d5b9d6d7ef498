"""RRAttention sparse prefill on NVIDIA B200 -- Python binding of librrattn.so.

Argument marshalling only: every step of the path runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream.  There is no CPU fallback: if
the library is missing, or a tensor is not on a CUDA device, calls raise.

    estimate(Q, K, S, B)              -> block_scores [H][L/B][L/B] float32
    select(block_scores, tau)         -> (row_ptr int32 [H*Nb+1], col_idx int32, nnz)
    sparse_prefill(Q, K, V, row_ptr, col_idx, B) -> O [H][L][d] bf16
    prefill(Q, K, V, S, B, tau)       -> O (the three stages back to back)

Shapes: Q [H][L][d], K and V [Hkv][L][d], contiguous bf16 on one CUDA device.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

__all__ = ["RRAttnError", "lib", "library_path", "estimate", "xattn_estimate", "select", "sparse_prefill",
           "prefill", "validate_csr", "estimate_workspace_bytes", "select_workspace_bytes",
           "Workspace", "STRATEGIES", "EXPORTED_SYMBOLS", "device_errors", "default_chunks",
           "head_shard", "host_slices", "selftest_wait"]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "librrattn.so")

STRATEGIES = {"head": 0, "none": 1, "layer": 2, "hybrid": 3}

EXPORTED_SYMBOLS = ("rr_estimate", "rr_estimate_strategy", "rr_estimate_heads",
                    "rr_estimate_workspace_bytes", "rr_xattn_estimate",
                    "rr_select", "rr_select_workspace_bytes", "rr_select_noalloc",
                    "rr_sparse_prefill",
                    "rr_validate_csr", "rr_device_errors", "rr_selftest_wait", "rr_status_string",
                    "rr_last_error",
                    "rr_version")


class RRAttnError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {_STATUS.get(code, code)}: {msg}")
        self.code = code


_STATUS = {0: "RR_OK", 1: "RR_ERR_INVALID_ARG", 2: "RR_ERR_UNSUPPORTED", 3: "RR_ERR_CUDA",
           4: "RR_ERR_WORKSPACE"}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded librrattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RRAttnError("load", -1, f"{library_path} is missing: build it with "
                          "`python -m long_context_prefill_estimate_b200.build`")
    L = ctypes.CDLL(library_path)
    P, I, Z, F, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_double
    I64 = ctypes.c_int64
    L.rr_estimate_workspace_bytes.argtypes = [I, I, I, I, I, I]
    L.rr_estimate_workspace_bytes.restype = Z
    L.rr_estimate.argtypes = [P, P, I, I, I, I, I, I, P, P, Z, P]
    L.rr_estimate.restype = I
    L.rr_estimate_strategy.argtypes = [P, P, I, I, I, I, I, I, I, I, P, P, Z, P]
    L.rr_estimate_strategy.restype = I
    L.rr_estimate_heads.argtypes = [P, P, I, I, I, I, I, I, I, I, I, P, P, Z, P]
    L.rr_estimate_heads.restype = I
    L.rr_xattn_estimate.argtypes = [P, P, I, I, I, I, I, I, P, P]
    L.rr_xattn_estimate.restype = I
    L.rr_select_workspace_bytes.argtypes = [I, I]
    L.rr_select_workspace_bytes.restype = Z
    L.rr_select.argtypes = [P, I, I, D, I, P, P, I64, P, P, Z, P]
    L.rr_select.restype = I
    L.rr_select_noalloc.argtypes = [P, I, I, D, I, P, P, I64, P, P]
    L.rr_select_noalloc.restype = I
    L.rr_sparse_prefill.argtypes = [P, P, P, I, I, I, I, I, P, P, F, P, P]
    L.rr_sparse_prefill.restype = I
    L.rr_validate_csr.argtypes = [P, P, I, I, I64, P, P]
    L.rr_validate_csr.restype = I
    L.rr_device_errors.argtypes = [P, I]
    L.rr_device_errors.restype = I
    L.rr_selftest_wait.argtypes = [ctypes.c_uint32, P]
    L.rr_selftest_wait.restype = I
    L.rr_status_string.argtypes = [I]
    L.rr_status_string.restype = ctypes.c_char_p
    L.rr_last_error.argtypes = []
    L.rr_last_error.restype = ctypes.c_char_p
    L.rr_version.restype = I
    _lib = L
    return L


def _check(fn: str, code: int):
    if code != 0:
        raise RRAttnError(fn, code, lib().rr_last_error().decode(errors="replace"))


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need_cuda(name: str, t: torch.Tensor, dtype: torch.dtype):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise RRAttnError(name, 1, "tensors must live on a CUDA device (no CPU path exists)")
    if t.dtype != dtype:
        raise RRAttnError(name, 1, f"expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise RRAttnError(name, 1, "tensors must be contiguous")


def estimate_workspace_bytes(H: int, Hkv: int, L: int, d: int, S: int, B: int) -> int:
    return int(lib().rr_estimate_workspace_bytes(H, Hkv, L, d, S, B))


def select_workspace_bytes(H: int, Nb: int) -> int:
    return int(lib().rr_select_workspace_bytes(H, Nb))


class Workspace:
    """Reusable device buffers for one layer shape (avoids per-call allocation)."""

    def __init__(self, H: int, Hkv: int, L: int, d: int, S: int, B: int, device="cuda"):
        self.shape = (H, Hkv, L, d, S, B)
        Nb = L // B
        dev = torch.device(device)
        self.est = torch.empty(max(estimate_workspace_bytes(H, Hkv, L, d, S, B), 16),
                               dtype=torch.uint8, device=dev)
        self.sel = torch.empty(max(select_workspace_bytes(H, Nb), 16), dtype=torch.uint8, device=dev)
        self.block_scores = torch.empty((H, Nb, Nb), dtype=torch.float32, device=dev)
        self.row_ptr = torch.empty(H * Nb + 1, dtype=torch.int32, device=dev)
        self.col_idx = torch.empty(max(H * Nb * (Nb + 1) // 2, 1), dtype=torch.int32, device=dev)
        self.nnz = torch.zeros(1, dtype=torch.int64, device=dev)


def estimate(Q: torch.Tensor, K: torch.Tensor, S: int, B: int, strategy: str = "head",
             layer: int = 0, out: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None, head_base: int = 0) -> torch.Tensor:
    """Block importance [H][L/B][L/B] (float32) from round-robin sampled queries.

    Q and K may be a slice of whole KV groups of a larger layer; head_base is then the
    layer-wide index of Q's first head (it sets the round-robin offsets)."""
    _need_cuda("rr_estimate", Q, torch.bfloat16)
    _need_cuda("rr_estimate", K, torch.bfloat16)
    H, L, d = Q.shape
    Hkv = K.shape[0]
    if K.shape != (Hkv, L, d):
        raise RRAttnError("rr_estimate", 1, f"K shape {tuple(K.shape)} does not match Q {tuple(Q.shape)}")
    Nb = L // B if B > 0 else 0
    if out is None:
        out = torch.empty((H, Nb, Nb), dtype=torch.float32, device=Q.device)
    need = estimate_workspace_bytes(H, Hkv, L, d, S, B)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=Q.device)
    _check("rr_estimate", lib().rr_estimate_heads(
        _ptr(Q), _ptr(K), H, Hkv, L, d, S, B, STRATEGIES[strategy], layer, head_base, _ptr(out),
        _ptr(workspace), workspace.numel(), _stream(Q.device)))
    return out



def xattn_estimate(Q: torch.Tensor, K: torch.Tensor, S: int, B: int,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """XAttention's antidiagonal block importance [H][L/B][L/B] (float32): the comparison
    estimator of the pattern-discovery timing, selected with select() like estimate()'s."""
    _need_cuda("rr_xattn_estimate", Q, torch.bfloat16)
    _need_cuda("rr_xattn_estimate", K, torch.bfloat16)
    H, L, d = Q.shape
    Hkv = K.shape[0]
    if K.shape != (Hkv, L, d):
        raise RRAttnError("rr_xattn_estimate", 1, f"K shape {tuple(K.shape)} does not match Q {tuple(Q.shape)}")
    Nb = L // B if B > 0 else 0
    if out is None:
        out = torch.empty((H, Nb, Nb), dtype=torch.float32, device=Q.device)
    _check("rr_xattn_estimate", lib().rr_xattn_estimate(_ptr(Q), _ptr(K), H, Hkv, L, d, S, B, _ptr(out),
                                                        _stream(Q.device)))
    return out


def select(block_scores: torch.Tensor, tau: float, protect_last: bool = True,
           row_ptr: Optional[torch.Tensor] = None, col_idx: Optional[torch.Tensor] = None,
           nnz: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None
           ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Top-tau CSR block lists.  col_idx has worst-case capacity; nnz (device int64) and
    row_ptr[-1] give the used length."""
    _need_cuda("rr_select", block_scores, torch.float32)
    H, Nb, Nb2 = block_scores.shape
    if Nb != Nb2:
        raise RRAttnError("rr_select", 1, "block_scores must be [H][Nb][Nb]")
    dev = block_scores.device
    cap = max(H * Nb * (Nb + 1) // 2, 1)
    if row_ptr is None:
        row_ptr = torch.empty(H * Nb + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(cap, dtype=torch.int32, device=dev)
    if nnz is None:
        nnz = torch.zeros(1, dtype=torch.int64, device=dev)
    if workspace is None:
        workspace = torch.empty(max(select_workspace_bytes(H, Nb), 16), dtype=torch.uint8, device=dev)
    _check("rr_select", lib().rr_select(
        _ptr(block_scores), H, Nb, float(tau), int(bool(protect_last)), _ptr(row_ptr),
        _ptr(col_idx), col_idx.numel(), _ptr(nnz), _ptr(workspace), workspace.numel(),
        _stream(dev)))
    return row_ptr, col_idx, nnz


def sparse_prefill(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, row_ptr: torch.Tensor,
                   col_idx: torch.Tensor, B: int, scale: Optional[float] = None,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Causal block-sparse attention over the CSR-selected blocks -> O [H][L][d] bf16."""
    for n, t in (("Q", Q), ("K", K), ("V", V)):
        _need_cuda("rr_sparse_prefill", t, torch.bfloat16)
    _need_cuda("rr_sparse_prefill", row_ptr, torch.int32)
    _need_cuda("rr_sparse_prefill", col_idx, torch.int32)
    H, L, d = Q.shape
    Hkv = K.shape[0]
    if K.shape != (Hkv, L, d) or V.shape != K.shape:
        raise RRAttnError("rr_sparse_prefill", 1, "K/V shapes do not match Q")
    if out is None:
        out = torch.empty_like(Q)
    _check("rr_sparse_prefill", lib().rr_sparse_prefill(
        _ptr(Q), _ptr(K), _ptr(V), H, Hkv, L, d, B, _ptr(row_ptr), _ptr(col_idx),
        float(scale) if scale else 0.0, _ptr(out), _stream(Q.device)))
    return out


def prefill(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, S: int, B: int, tau: float,
            protect_last: bool = True, strategy: str = "head", layer: int = 0,
            scale: Optional[float] = None, ws: Optional[Workspace] = None,
            out: Optional[torch.Tensor] = None, return_intermediates: bool = False,
            chunks: Optional[int] = None, head_base: int = 0):
    """One attention layer's sparse prefill: estimate -> select -> sparse attention.

    Host (CPU) tensors are accepted: the layer is then processed in `chunks` slices of whole
    KV groups (default: the largest divisor of Hkv that is at most 8), each slice's inputs
    copied in on one stream while the previous slice computes and the one before is copied
    back on a third, and the call returns once O is on the host.  Pinned host memory makes
    the copies asynchronous.  The result is identical to the one-pass device call: every
    stage is independent per query head, and each slice is estimated with its layer-wide
    head index.  The host path allocates its own slice-sized workspace (`ws` applies to the
    device path); with return_intermediates it runs as one slice.

    Q, K, V may themselves be a shard of whole KV groups of a larger layer (see head_shard);
    head_base is then the layer-wide index of Q's first head."""
    host = not Q.is_cuda
    if host and not return_intermediates:
        return _prefill_host_pipelined(Q, K, V, S, B, tau, protect_last, strategy, layer, scale,
                                       out, chunks, head_base)
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        Q, K, V = (t.to(dev, non_blocking=True) for t in (Q, K, V))
    H, L, d = Q.shape
    Hkv = K.shape[0]
    if ws is None:
        ws = Workspace(H, Hkv, L, d, S, B, device=Q.device)
    estimate(Q, K, S, B, strategy=strategy, layer=layer, out=ws.block_scores, workspace=ws.est,
             head_base=head_base)
    select(ws.block_scores, tau, protect_last, row_ptr=ws.row_ptr, col_idx=ws.col_idx,
           nnz=ws.nnz, workspace=ws.sel)
    O = sparse_prefill(Q, K, V, ws.row_ptr, ws.col_idx, B, scale=scale,
                       out=None if host else out)
    if host:
        dst = out if out is not None else torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        dst.copy_(O, non_blocking=True)
        torch.cuda.current_stream(O.device).synchronize()
        O = dst
    if return_intermediates:
        return O, ws
    return O


def head_shard(rank: int, world: int, H: int, Hkv: int) -> Tuple[int, int, int, int]:
    """Rank `rank`'s share of a layer split across `world` GPUs by whole KV groups:
    (h0, h1, g0, g1) = its query heads [h0, h1) and KV heads [g0, g1), contiguous, with the
    groups spread as evenly as they divide.  Every stage is independent per query head, so
    the shards need no exchange; pass h0 as head_base to keep the round-robin offsets."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    if Hkv <= 0 or H % Hkv:
        raise ValueError(f"H={H} is not a multiple of Hkv={Hkv}")
    if world > Hkv:
        raise ValueError(f"{world} ranks cannot share {Hkv} KV groups")
    G = H // Hkv
    g0, g1 = rank * Hkv // world, (rank + 1) * Hkv // world
    return g0 * G, g1 * G, g0, g1


def default_chunks(Hkv: int) -> int:
    """Slices of the host pipeline: the largest divisor of Hkv that is at most 8."""
    return max(c for c in range(1, min(Hkv, 8) + 1) if Hkv % c == 0)


def host_slices(H: int, Hkv: int, chunks: int, peel: bool = True):
    """Slices (h0, h1) of the host pipeline: `chunks` ranges of whole KV groups; with `peel`
    (and more than one query head per group) the layer's first and last query heads become
    slices of their own, so the first copy-in and the last copy-out are short.  Every slice
    is whole KV groups or heads of a single group."""
    G = H // Hkv
    gc = Hkv // chunks
    units = [(c * gc * G, (c + 1) * gc * G) for c in range(chunks)]
    if not peel or G == 1:
        return units
    out = []
    for i, (h0, h1) in enumerate(units):
        parts = [(h0, h1)]
        if i == 0:  # head h0 | the rest of its group | the remaining whole groups
            parts = [(h0, h0 + 1), (h0 + 1, h0 + G)] + ([(h0 + G, h1)] if h1 > h0 + G else [])
        if i == len(units) - 1:  # ... | the last group but its last head | the last head
            a, b = parts.pop()
            if b - a > G:
                parts.append((a, b - G))
                a = b - G
            if b - 1 > a:
                parts.append((a, b - 1))
            parts.append((b - 1, b))
        out += parts
    return out


def _prefill_host_pipelined(Q, K, V, S, B, tau, protect_last, strategy, layer, scale, out, chunks,
                            head_base=0):
    for n, t in (("Q", Q), ("K", K), ("V", V)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise RRAttnError("prefill", 1, f"{n}: host path needs contiguous bf16 CPU tensors")
    H, L, d = Q.shape
    Hkv = K.shape[0]
    if Hkv <= 0 or H % Hkv or K.shape != (Hkv, L, d) or V.shape != K.shape:
        raise RRAttnError("prefill", 1, f"shapes Q {tuple(Q.shape)} K {tuple(K.shape)} V {tuple(V.shape)}")
    n = default_chunks(Hkv) if chunks is None else int(chunks)
    if n <= 0 or Hkv % n:
        raise RRAttnError("prefill", 1, f"chunks={n} must divide Hkv={Hkv}")
    dst = out if out is not None else torch.empty(Q.shape, dtype=Q.dtype, pin_memory=True)
    if dst.shape != Q.shape or dst.dtype != Q.dtype or dst.is_cuda or not dst.is_contiguous():
        raise RRAttnError("prefill", 1, "out must be a contiguous bf16 host tensor shaped like Q")
    dev = torch.device("cuda", torch.cuda.current_device())
    G, Nb = H // Hkv, (L // B if B > 0 else 0)
    # heads of one group may form a slice only where the estimator's per-row arithmetic does
    # not depend on how many heads share a CTA (B/S <= 32); there the bytes match one pass
    slices = host_slices(H, Hkv, n, peel=B > 0 and S > 0 and (B // S) in (4, 8, 16, 32))
    spans = [(h0, h1, h0 // G, (h1 - 1) // G + 1) for h0, h1 in slices]
    mh = max(h1 - h0 for h0, h1, _, _ in spans)
    mg = max(g1 - g0 for _, _, g0, g1 in spans)
    compute = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    Qd, Kd, Vd = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (Q, K, V))
    Od = torch.empty(Q.shape, dtype=Q.dtype, device=dev)
    ws = Workspace(mh, mg, L, d, S, B, device=dev)
    # the fresh buffers may reuse memory last used on the compute stream
    s_in.wait_stream(compute)
    s_out.wait_stream(compute)
    loaded, kv_done = [], 0
    with torch.cuda.stream(s_in):
        for h0, h1, g0, g1 in spans:
            Qd[h0:h1].copy_(Q[h0:h1], non_blocking=True)
            if g1 > kv_done:  # each group's K/V travels with the first slice that needs it
                Kd[kv_done:g1].copy_(K[kv_done:g1], non_blocking=True)
                Vd[kv_done:g1].copy_(V[kv_done:g1], non_blocking=True)
                kv_done = g1
            ev = torch.cuda.Event()
            ev.record(s_in)
            loaded.append(ev)
    for (h0, h1, g0, g1), ev in zip(spans, loaded):
        nh = h1 - h0
        A, rp = ws.block_scores[:nh], ws.row_ptr[:nh * Nb + 1]
        compute.wait_event(ev)
        estimate(Qd[h0:h1], Kd[g0:g1], S, B, strategy=strategy, layer=layer, out=A,
                 workspace=ws.est, head_base=head_base + h0)
        select(A, tau, protect_last, row_ptr=rp, col_idx=ws.col_idx, nnz=ws.nnz, workspace=ws.sel)
        sparse_prefill(Qd[h0:h1], Kd[g0:g1], Vd[g0:g1], rp, ws.col_idx, B, scale=scale, out=Od[h0:h1])
        done = torch.cuda.Event()
        done.record(compute)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            dst[h0:h1].copy_(Od[h0:h1], non_blocking=True)
    s_out.synchronize()
    # every copy and kernel above has completed; later work on the compute stream may
    # reuse the buffers
    compute.wait_stream(s_in)
    compute.wait_stream(s_out)
    return dst


def validate_csr(row_ptr: torch.Tensor, col_idx: torch.Tensor, H: int, Nb: int) -> int:
    """Number of malformed CSR rows (checked on the device; synchronises to read it)."""
    bad = torch.zeros(1, dtype=torch.int32, device=row_ptr.device)
    _check("rr_validate_csr", lib().rr_validate_csr(
        _ptr(row_ptr), _ptr(col_idx), H, Nb, col_idx.numel(), _ptr(bad), _stream(row_ptr.device)))
    return int(bad.item())


def selftest_wait(timeout_us: int = 20000) -> Tuple[bool, bool, int]:
    """Runs the bounded-wait self-test: (gave_up, saw_completed_phase, microseconds)."""
    r = (ctypes.c_uint32 * 3)()
    _check("rr_selftest_wait", lib().rr_selftest_wait(int(timeout_us), r))
    return bool(r[0]), bool(r[1]), int(r[2])


def device_errors(reset: bool = True) -> int:
    """Error bits recorded by the kernels on the current device (0 = none); synchronises."""
    v = ctypes.c_uint32(0)
    _check("rr_device_errors", lib().rr_device_errors(ctypes.byref(v), int(reset)))
    return int(v.value)
