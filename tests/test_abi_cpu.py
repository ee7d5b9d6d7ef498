"""C-ABI library: loads, exports every symbol the header declares, validates on the host.

No compute call is made here: every call below is rejected by host-side validation before
any CUDA API is touched, so this runs on a machine without a GPU.
"""
import ctypes
import os
import re

import pytest

import long_context_prefill_estimate_b200 as rr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rr_attn.h")

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 4


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rr_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from long_context_prefill_estimate_b200 import build

    build.build()
    return rr.lib()


def test_exports_every_declared_symbol(L):
    names = _declared_functions()
    assert set(names) >= {"rr_estimate", "rr_select", "rr_sparse_prefill"}
    for n in names:
        assert hasattr(L, n), f"{n} declared in rr_attn.h but not exported"
    assert set(rr.EXPORTED_SYMBOLS) == set(names)


def test_version_and_status_strings(L):
    assert L.rr_version() >= 100
    assert L.rr_status_string(0) == b"RR_OK"
    assert L.rr_status_string(4) == b"RR_ERR_WORKSPACE"
    assert L.rr_status_string(99) == b"RR_ERR_UNKNOWN"


def test_workspace_sizes(L):
    assert rr.estimate_workspace_bytes(32, 8, 131072, 128, 16, 128) == 8 * 8192 * 128 * 4
    assert rr.estimate_workspace_bytes(32, 8, 0, 128, 16, 128) == 0
    assert rr.select_workspace_bytes(32, 1024) >= 32 * 1024 * 4 + 32 * 1024 * 32 * 4


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced (validation fails first)


def _est(L, H=4, Hkv=2, Len=256, d=64, S=8, B=64, strategy=0, layer=0, q=FAKE, k=FAKE, out=FAKE,
         ws=FAKE, wsb=1 << 30):
    return L.rr_estimate_strategy(q, k, H, Hkv, Len, d, S, B, strategy, layer, out, ws, wsb, None)


def test_estimate_rejections(L):
    assert _est(L, H=3, Hkv=2) == INVALID
    assert _est(L, d=96) == UNSUPPORTED
    assert _est(L, B=32) == UNSUPPORTED
    assert _est(L, Len=200) == UNSUPPORTED
    assert _est(L, S=3) == INVALID
    assert _est(L, S=32) == UNSUPPORTED        # B/S = 2 is neither 4 nor a multiple of 8
    assert _est(L, Len=64, S=16) == UNSUPPORTED  # L/S = 4 strides, not a multiple of 8
    assert _est(L, strategy=7) == INVALID
    assert _est(L, q=0) == INVALID
    assert _est(L, k=FAKE + 4) == INVALID      # misaligned
    assert _est(L, ws=0) == WORKSPACE
    assert _est(L, wsb=16) == WORKSPACE
    assert b"workspace" in L.rr_last_error()
    assert _est(L, Len=0, q=0, k=0, out=0, ws=0) == 0   # empty problem: accepted, no launch


def test_xattn_estimate_rejections(L):
    def x(H=4, Hkv=2, Len=256, d=64, S=8, B=64, q=FAKE, k=FAKE, out=FAKE):
        return L.rr_xattn_estimate(q, k, H, Hkv, Len, d, S, B, out, None)

    assert x(H=3) == INVALID
    assert x(d=96) == UNSUPPORTED
    assert x(S=3) == INVALID
    assert x(S=32) == UNSUPPORTED          # B/S = 2
    assert x(S=1) == UNSUPPORTED           # B/S = 64: no kernel for XAttention
    assert x(Len=64, S=16) == UNSUPPORTED  # L/S = 4
    assert x(q=0) == INVALID
    assert x(out=FAKE + 8) == INVALID
    assert b"rr_xattn_estimate" in L.rr_last_error()
    assert x(Len=0, q=0, k=0, out=0) == 0


def test_estimate_heads_rejections(L):
    f = L.rr_estimate_heads
    ok = (FAKE, FAKE, 4, 2, 256, 64, 8, 64, 0, 0)
    assert f(*ok, -1, FAKE, FAKE, 1 << 30, None) == INVALID
    assert f(*ok, (1 << 20) + 1, FAKE, FAKE, 1 << 30, None) == INVALID
    assert b"head_base" in L.rr_last_error()
    assert f(FAKE, FAKE, 4, 2, 0, 64, 8, 64, 0, 0, 4, 0, 0, 0, None) == 0   # empty: no launch


def test_host_path_argument_checks(L):
    import torch

    Q = torch.zeros(4, 128, 64, dtype=torch.bfloat16)
    K = torch.zeros(2, 128, 64, dtype=torch.bfloat16)
    assert rr.default_chunks(8) == 8 and rr.default_chunks(28) == 7 and rr.default_chunks(1) == 1
    with pytest.raises(rr.RRAttnError, match="chunks=3"):
        rr.prefill(Q, K, K, 8, 64, 0.9, chunks=3)
    with pytest.raises(rr.RRAttnError, match="shapes"):
        rr.prefill(Q, K[:, :64].contiguous(), K, 8, 64, 0.9)
    with pytest.raises(rr.RRAttnError, match="contiguous bf16"):
        rr.prefill(Q.float(), K, K, 8, 64, 0.9)


def test_selftest_wait_rejections(L):
    buf = (ctypes.c_uint32 * 3)()
    assert L.rr_selftest_wait(0, buf) == INVALID
    assert L.rr_selftest_wait(3000000, buf) == INVALID
    assert L.rr_selftest_wait(1000, None) == INVALID
    assert b"timeout_us" in L.rr_last_error() or b"result" in L.rr_last_error()


def test_host_pipeline_slices():
    # contiguous, covering, each slice whole KV groups or heads of one group; the first and
    # last query heads stand alone when a group has several heads
    for H, Hkv in [(32, 8), (28, 4), (4, 1), (2, 2), (16, 4), (8, 8), (14, 2)]:
        G = H // Hkv
        for chunks in [c for c in range(1, Hkv + 1) if Hkv % c == 0]:
            for peel in (True, False):
                sl = rr.host_slices(H, Hkv, chunks, peel)
                assert sl[0][0] == 0 and sl[-1][1] == H
                assert all(a[1] == b[0] for a, b in zip(sl, sl[1:]))
                for h0, h1 in sl:
                    assert h1 > h0
                    assert (h1 - 1) // G == h0 // G or (h0 % G == 0 and h1 % G == 0)
                if peel and G > 1:
                    assert sl[0] == (0, 1) and sl[-1] == (H - 1, H)
                if not peel:
                    assert len(sl) == chunks


def test_select_rejections(L):
    P = FAKE
    ok_cap = 2 * 4 * 5 // 2
    assert L.rr_select(P, 2, 4, 0.0, 1, P, P, ok_cap, None, P, 1 << 20, None) == INVALID
    assert L.rr_select(P, 2, 4, 1.5, 1, P, P, ok_cap, None, P, 1 << 20, None) == INVALID
    assert L.rr_select(P, 2, 4, float("nan"), 1, P, P, ok_cap, None, P, 1 << 20, None) == INVALID
    assert L.rr_select(P, 2, 4, 0.9, 1, P, P, ok_cap - 1, None, P, 1 << 20, None) == INVALID
    assert b"col_capacity" in L.rr_last_error()
    assert L.rr_select(P, 2, 4, 0.9, 1, P, P, ok_cap, None, P, 8, None) == WORKSPACE
    assert L.rr_select(P, 2, 4, 0.9, 1, P, P, ok_cap, P + 4, P, 1 << 20, None) == INVALID
    assert L.rr_select(0, 2, 0, 0.9, 1, 0, 0, 0, None, 0, 0, None) == 0  # empty


def test_prefill_rejections(L):
    P = FAKE
    f = L.rr_sparse_prefill
    assert f(P, P, P, 4, 3, 256, 64, 64, P, P, 0.0, P, None) == INVALID
    assert f(P, P, P, 4, 2, 256, 80, 64, P, P, 0.0, P, None) == UNSUPPORTED
    assert f(P, P, P, 4, 2, 250, 64, 64, P, P, 0.0, P, None) == UNSUPPORTED
    assert f(P, P, P, 4, 2, 256, 64, 64, 0, P, 0.0, P, None) == INVALID
    assert f(P, P, P, 4, 2, 256, 64, 64, P, P, float("inf"), P, None) == INVALID
    assert f(0, 0, 0, 4, 2, 0, 64, 64, 0, 0, 0.0, 0, None) == 0


def test_binding_refuses_cpu_tensors(L):
    import torch

    Q = torch.zeros(2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(rr.RRAttnError, match="CUDA device"):
        rr.estimate(Q, Q, 8, 64)
    with pytest.raises(rr.RRAttnError, match="CUDA device"):
        rr.sparse_prefill(Q, Q, Q, torch.zeros(3, dtype=torch.int32), torch.zeros(3, dtype=torch.int32), 64)
