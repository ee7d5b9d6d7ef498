"""rr_select_noalloc: Top-tau selection for callers that cannot allocate device memory.

Such callers (a plugin whose host application owns all device memory, or a path that must
never call cudaMalloc/cudaFree) get their scratch from a fixed array inside the library.
This file is collected last so that a failure here leaves every other test already run.
It checks the allocation-free call through the C ABI against rr_select on three calls in a
row with different shapes, so leftovers of an earlier call in the shared array cannot hide;
the third has rows longer than 1024 blocks, which take the sorting kernel.  It also checks
that sizes beyond the array are refused before any launch, and that a successful call leaves
no stale error text behind.
"""
import ctypes

import numpy as np
import pytest
import torch

import long_context_prefill_estimate_b200 as rr

pytestmark = pytest.mark.gpu


def _scores(H, Nb, seed, ties=False):
    rng = np.random.default_rng(seed)
    A = np.tril(rng.gamma(0.3, size=(H, Nb, Nb))).astype(np.float32)
    if ties:
        A[0, Nb // 2, : Nb // 2 + 1] = 1.0
    A /= A.sum(-1, keepdims=True)
    return torch.from_numpy(np.tril(A).astype(np.float32)).cuda()


def _noalloc(A, tau, protect):
    H, Nb, _ = A.shape
    cap = H * Nb * (Nb + 1) // 2
    rp = torch.full((H * Nb + 1,), -7, dtype=torch.int32, device=A.device)
    ci = torch.full((cap,), -7, dtype=torch.int32, device=A.device)
    nnz = torch.full((1,), -7, dtype=torch.int64, device=A.device)
    code = rr.lib().rr_select_noalloc(A.data_ptr(), H, Nb, float(tau), int(protect), rp.data_ptr(),
                                      ci.data_ptr(), cap, nnz.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert code == 0, rr.lib().rr_last_error()
    return rp, ci, nnz


CALLS = [(32, 256, 0.9, True), (8, 700, 0.8, False), (2, 1100, 0.9, False)]


def test_noalloc_matches_select_on_consecutive_calls(cuda_device):
    for i, (H, Nb, tau, protect) in enumerate(CALLS):
        A = _scores(H, Nb, seed=i, ties=(i == 1))
        rp_ref, ci_ref, nnz_ref = rr.select(A, tau, protect)
        rp, ci, nnz = _noalloc(A, tau, protect)
        torch.cuda.synchronize()
        n = int(nnz_ref.item())
        assert int(nnz.item()) == n
        assert torch.equal(rp, rp_ref)
        assert torch.equal(ci[:n], ci_ref[:n])
        assert rr.validate_csr(rp, ci, H, Nb) == 0


def test_noalloc_refuses_sizes_beyond_the_array(cuda_device):
    H, Nb = 64, 2048   # needs ~34 MB of scratch, the built-in array holds 8 MiB
    code = rr.lib().rr_select_noalloc(1 << 20, H, Nb, 0.9, 1, 1 << 20, 1 << 20,
                                      H * Nb * (Nb + 1) // 2, None, None)
    assert code == 2
    assert b"built-in array" in rr.lib().rr_last_error()


def test_noalloc_success_clears_the_last_error(cuda_device):
    code = rr.lib().rr_select_noalloc(None, 2, 8, 0.9, 1, None, None, 72, None, None)
    assert code == 1 and rr.lib().rr_last_error() != b""
    _noalloc(_scores(2, 8, seed=5), 0.9, True)
    assert rr.lib().rr_last_error() == b""
