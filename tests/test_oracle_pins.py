"""Pins of the CPU oracle against facts fixed by the paper and by mathematics.

Each pin compares the oracle (plain C, double) with something other than itself:
hand-worked examples (tests/golden/), closed forms that reduce to textbook attention
computed by torch's library routines in float64, brute-force enumeration and
invariants.  No GPU is used.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(shape, seed, std=0.5):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)


def _dense_causal_probs(q64, k64, scale):
    """Textbook causal softmax attention probabilities, [L][L] (torch library routines)."""
    L = q64.shape[0]
    s = (q64 @ k64.T) * scale
    mask = torch.ones(L, k64.shape[0], dtype=torch.bool).tril()
    s = s.masked_fill(~mask, float("-inf"))
    return torch.softmax(s, dim=-1)


# ---------------------------------------------------------------- round-robin sampling
def _golden_positions():
    out = []
    with open(os.path.join(GOLDEN, "rr_positions_head_rr.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            left, right = line.split("|")
            H, S, L = map(int, left.split())
            h, pos = right.split(":")
            out.append((H, S, L, int(h), [int(x) for x in pos.split()]))
    return out


@pytest.mark.parametrize("H,S,L,h,expected", _golden_positions())
def test_rr_positions_hand_worked(H, S, L, h, expected):
    got = [oracle.sample_position(i, h, S) for i in range(L // S)]
    assert got == expected


def test_rr_coverage_when_heads_cover_stride():
    # Sec. 3.2 (every position contributes) with H >= S: all offsets of a stride are used.
    for H, S in [(32, 16), (32, 8), (28, 16), (16, 16)]:
        offs = {oracle.offset(h, S) for h in range(H)}
        assert offs == set(range(S))


def test_rr_unsampled_positions_when_stride_exceeds_heads():
    # Sec. 7 Limitations: with S > H some positions are never sampled.
    H, S = 2, 8
    offs = {oracle.offset(h, S) for h in range(H)}
    assert offs == {0, 1}
    assert set(range(S)) - offs == {2, 3, 4, 5, 6, 7}


def test_rr_strategy_variants_hand_worked():
    # Sec. 4.3 Table 6 strategies; readings: none -> S-1, layer -> l mod S, hybrid -> (h+l) mod S
    S = 8
    assert [oracle.offset(h, S, oracle.NO_RR) for h in range(4)] == [7, 7, 7, 7]
    assert [oracle.offset(h, S, oracle.LAYER_RR, layer=11) for h in range(4)] == [3, 3, 3, 3]
    assert [oracle.offset(h, S, oracle.HYBRID_RR, layer=11) for h in range(4)] == [3, 4, 5, 6]
    assert [oracle.offset(h, S, oracle.HYBRID_RR, layer=6) for h in range(3)] == [6, 7, 0]


# ---------------------------------------------------------------- key pooling
def test_pool_keys_one_hot():
    Hkv, L, d, S = 2, 32, 8, 4
    K = torch.zeros(Hkv, L, d, dtype=torch.bfloat16)
    K[1, 13, 5] = 3.0   # stride 13 // 4 = 3
    K[1, 14, 5] = -1.0  # same stride
    K[0, 0, 0] = 2.0    # stride 0
    Kb = oracle.pool_keys(K, S)
    expect = np.zeros((Hkv, L // S, d))
    expect[1, 3, 5] = 2.0
    expect[0, 0, 0] = 2.0
    np.testing.assert_array_equal(Kb, expect)


def test_pool_keys_sum_of_stride():
    K = _bf16((3, 64, 16), 1)
    Kb = oracle.pool_keys(K, 8)
    ref = K.double().reshape(3, 8, 8, 16).sum(2).numpy()
    np.testing.assert_allclose(Kb, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- estimator closed forms
@pytest.mark.parametrize("H,Hkv,L,d,B", [(2, 2, 128, 16, 16), (4, 2, 192, 8, 32), (3, 1, 64, 32, 8)])
def test_estimate_S1_is_exact_block_attention_mass(H, Hkv, L, d, B):
    """S = 1: every query is sampled and pooled keys are the keys, so A[h][I][J] is the
    mean over the queries of block I of their causal attention mass on key block J."""
    Q, K = _bf16((H, L, d), 2), _bf16((Hkv, L, d), 3)
    A = oracle.estimate(Q, K, S=1, B=B)
    Nb, G = L // B, H // Hkv
    for h in range(H):
        P = _dense_causal_probs(Q[h].double(), K[h // G].double(), 1 / math.sqrt(d))
        mass = P.reshape(Nb, B, Nb, B).sum(dim=(1, 3)) / B
        np.testing.assert_allclose(A[h], mass.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode,layer", [(oracle.HEAD_RR, 0), (oracle.NO_RR, 0),
                                        (oracle.HYBRID_RR, 5)])
@pytest.mark.parametrize("H,Hkv,L,d,S,B", [(4, 2, 256, 16, 4, 16), (2, 2, 256, 8, 8, 32),
                                           (6, 3, 96, 16, 2, 8)])
def test_estimate_duplicated_keys_closed_form(H, Hkv, L, d, S, B, mode, layer):
    """Keys identical within each stride: Kbar_j = S*k_j and the 1/(S sqrt d) scale leaves
    plain attention of the sampled queries over the de-duplicated keys; its block mass over
    (B/S)-stride blocks is the estimate.  Sampled offsets come from the hand-worked rule."""
    Q = _bf16((H, L, d), 4)
    Ns = L // S
    kd = _bf16((Hkv, Ns, d), 5)
    K = kd.repeat_interleave(S, dim=1).contiguous()
    A = oracle.estimate(Q, K, S=S, B=B, mode=mode, layer=layer)
    r, Nb, G = B // S, L // B, H // Hkv
    off_rule = {oracle.HEAD_RR: lambda h: h % S, oracle.NO_RR: lambda h: S - 1,
                oracle.HYBRID_RR: lambda h: (h + layer) % S}[mode]
    for h in range(H):
        qs = Q[h].double()[torch.arange(Ns) * S + off_rule(h)]
        P = _dense_causal_probs(qs, kd[h // G].double(), 1 / math.sqrt(d))
        mass = P.reshape(Nb, r, Nb, r).sum(dim=(1, 3)) / r
        np.testing.assert_allclose(A[h], mass.numpy(), rtol=0, atol=1e-12)


def test_estimate_invariants():
    w = workloads.get(0, L=512)
    t = workloads.generate(w)
    A = oracle.estimate(t["Q"], t["K"], w.S, w.B)
    Nb = w.Nb
    assert (A >= 0).all()
    np.testing.assert_allclose(A.sum(-1), 1.0, rtol=0, atol=1e-12)
    iu = np.triu_indices(Nb, k=1)
    assert (A[:, iu[0], iu[1]] == 0).all()


def test_estimate_depends_on_keys_only_through_stride_sums():
    H, Hkv, L, d, S, B = 2, 1, 128, 16, 8, 32
    Q = _bf16((H, L, d), 6)
    g = torch.Generator().manual_seed(7)
    K = (torch.randint(-6, 7, (Hkv, L, d), generator=g) * 0.25).to(torch.bfloat16)  # exact sums
    A = oracle.estimate(Q, K, S, B)
    perm = torch.cat([torch.randperm(S, generator=torch.Generator().manual_seed(j)) + j * S
                      for j in range(L // S)])
    A2 = oracle.estimate(Q, K[:, perm].contiguous(), S, B)
    np.testing.assert_allclose(A, A2, rtol=0, atol=1e-13)
    K3 = K.clone()
    K3[0, 17] += 0.25   # rows 17 and 18 are both in stride 2: its sum is unchanged
    K3[0, 18] -= 0.25
    np.testing.assert_allclose(A, oracle.estimate(Q, K3, S, B), rtol=0, atol=1e-13)
    K4 = K.clone()
    K4[0, 17] += 0.5
    assert np.abs(oracle.estimate(Q, K4, S, B) - A).max() > 1e-6


def test_estimate_reads_only_sampled_queries():
    H, Hkv, L, d, S, B = 2, 2, 128, 16, 8, 32
    Q, K = _bf16((H, L, d), 8), _bf16((Hkv, L, d), 9)
    A = oracle.estimate(Q, K, S, B)
    Q2 = Q.clone()
    Q2[0, 3::S] = 7.0   # offset 3 is never sampled when H = 2 < S = 8
    Q2[1, 5::S] = -7.0
    np.testing.assert_array_equal(oracle.estimate(Q2, K, S, B), A)
    Q3 = Q.clone()
    Q3[1, 1 + 9 * S] += 1.0  # head 1 samples offset 1 (stride 9, query block 2)
    d1 = np.abs(oracle.estimate(Q3, K, S, B) - A)
    assert d1[1].max() > 1e-6 and d1[0].max() == 0.0


# ---------------------------------------------------------------- XAttention estimate
def _golden_xattn():
    out = []
    with open(os.path.join(GOLDEN, "xattn_worked_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            q, k, a = line.split(";")
            out.append(([float(v) for v in q.split()], [float(v) for v in k.split()],
                        [float(v) for v in a.split()]))
    return out


@pytest.mark.parametrize("qv,kv,expected", _golden_xattn())
def test_xattn_hand_worked(qv, kv, expected):
    L = len(qv)
    B = 2 if len(expected) == 4 else 4
    Q = torch.tensor(qv, dtype=torch.bfloat16).reshape(1, L, 1)
    K = torch.tensor(kv, dtype=torch.bfloat16).reshape(1, L, 1)
    A = oracle.xattn_estimate(Q, K, S=2, B=B)
    np.testing.assert_allclose(A.reshape(-1), expected, rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,Hkv,L,d,B", [(2, 2, 128, 16, 16), (4, 2, 96, 8, 32)])
def test_xattn_S1_is_exact_block_attention_mass(H, Hkv, L, d, B):
    """S = 1: the antidiagonal of a 1 x 1 sub-block is the logit itself."""
    Q, K = _bf16((H, L, d), 21), _bf16((Hkv, L, d), 22)
    A = oracle.xattn_estimate(Q, K, S=1, B=B)
    Nb, G = L // B, H // Hkv
    for h in range(H):
        P = _dense_causal_probs(Q[h].double(), K[h // G].double(), 1 / math.sqrt(d))
        mass = P.reshape(Nb, B, Nb, B).sum(dim=(1, 3)) / B
        np.testing.assert_allclose(A[h], mass.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("H,Hkv,L,d,S,B", [(2, 1, 64, 8, 4, 16), (3, 3, 48, 4, 2, 8), (2, 2, 64, 4, 8, 32)])
def test_xattn_bruteforce_antidiagonals(H, Hkv, L, d, S, B):
    """The full logits matrix (torch float64), the antidiagonal of every S x S sub-block taken
    by flipping it left-right, the stride softmax and block sums written out directly."""
    Q, K = _bf16((H, L, d), 23), _bf16((Hkv, L, d), 24)
    A = oracle.xattn_estimate(Q, K, S=S, B=B)
    Ns, Nb, G, r = L // S, L // B, H // Hkv, B // S
    for h in range(H):
        logits = (Q[h].double() @ K[h // G].double().T / math.sqrt(d)).numpy()
        ref = np.zeros((Nb, Nb))
        for i in range(Ns):
            z = np.array([np.fliplr(logits[i * S:(i + 1) * S, j * S:(j + 1) * S]).trace() / S
                          for j in range(i + 1)])
            p = np.exp(z - z.max())
            p /= p.sum()
            for j in range(i + 1):
                ref[i // r, j // r] += p[j] * S / B
        np.testing.assert_allclose(A[h], ref, rtol=0, atol=1e-12)


def test_xattn_equals_pooled_scores_for_constant_query_strides():
    """Queries identical within each stride: every antidiagonal sum is q . (sum of the stride's
    keys), the round-robin estimate's logit for that query."""
    H, Hkv, L, d, S, B = 2, 1, 128, 16, 8, 32
    qd = _bf16((H, L // S, d), 25)
    Q = qd.repeat_interleave(S, dim=1).contiguous()
    K = _bf16((Hkv, L, d), 26)
    A = oracle.xattn_estimate(Q, K, S=S, B=B)
    Kbar = K.double().reshape(Hkv, L // S, S, d).sum(2)
    Ns, Nb, r = L // S, L // B, B // S
    for h in range(H):
        P = _dense_causal_probs(qd[h].double(), Kbar[0], 1 / (S * math.sqrt(d)))
        mass = P.reshape(Nb, r, Nb, r).sum(dim=(1, 3)) / r
        np.testing.assert_allclose(A[h], mass.numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- selection
def _golden_select():
    out = []
    with open(os.path.join(GOLDEN, "select_worked_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            sc, tau, exp = line.split(";")
            out.append(([float(x) for x in sc.split()], float(tau), [int(x) for x in exp.split()]))
    return out


@pytest.mark.parametrize("scores,tau,expected", _golden_select())
def test_select_hand_worked(scores, tau, expected):
    n = len(scores)
    A = np.zeros((1, n, n))
    A[0, n - 1, :] = scores
    rp, ci = oracle.select(A, tau, protect_last=False)
    assert ci[rp[n - 1]:rp[n]].tolist() == expected


def _golden_select_diag():
    out = []
    with open(os.path.join(GOLDEN, "select_diag_worked_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            sc, tau, exp = line.split(";")
            out.append(([float(x) for x in sc.split()], float(tau), [float(x) for x in exp.split()]))
    return out


@pytest.mark.parametrize("scores,tau,expected", _golden_select_diag())
def test_select_diag_hand_worked(scores, tau, expected):
    # the per-row diagnostics the GPU parity tests classify mismatching rows with: k*, the
    # cumulative sums on both sides of the cut, tau*T and the score gap across the cut
    n = len(scores)
    A = np.zeros((1, n, n))
    A[0, n - 1, :] = scores
    rp, ci, dg = oracle.select(A, tau, protect_last=False, diag=True)
    got = dg[n - 1]
    assert int(got[0]) == int(expected[0]) == rp[n] - rp[n - 1]
    np.testing.assert_allclose(got[1:4], expected[1:4], rtol=0, atol=1e-12)
    if math.isinf(expected[4]):
        assert math.isinf(got[4]) and got[4] > 0
    else:
        assert got[4] == pytest.approx(expected[4], abs=1e-12)


def test_select_diag_bruteforce():
    # the diagnostics against their definitions, recomputed from a brute-force sort
    rng = np.random.default_rng(3)
    for trial in range(40):
        n = int(rng.integers(1, 40))
        a = rng.gamma(0.3, size=n)
        if trial % 4 == 0:
            a = np.round(a * 4) / 4
        tau = float(rng.choice([0.5, 0.8, 0.9, 0.95]))
        A = np.zeros((1, n, n))
        A[0, n - 1] = a
        _, _, dg = oracle.select(A, tau, protect_last=False, diag=True)
        order = sorted(range(n), key=lambda j: (-a[j], j))
        s = a[order]
        cum = np.cumsum(s)   # sequential sums in the sorted order
        T = cum[-1]
        k = int(np.argmax(cum >= tau * T)) + 1
        assert int(dg[n - 1, 0]) == k
        assert dg[n - 1, 1] == pytest.approx(cum[k - 2] if k > 1 else 0.0, abs=1e-12)
        assert dg[n - 1, 2] == pytest.approx(cum[k - 1], abs=1e-12)
        assert dg[n - 1, 3] == pytest.approx(tau * T, abs=1e-12)
        gap = s[k - 1] - s[k] if k < n else math.inf
        assert dg[n - 1, 4] == pytest.approx(gap, abs=1e-12)


def test_select_bruteforce_minimal():
    rng = np.random.default_rng(0)
    for trial in range(60):
        n = int(rng.integers(1, 12))
        a = rng.dirichlet(np.full(n, rng.choice([0.2, 1.0, 5.0])))
        if trial % 5 == 0:
            a = np.round(a * 8) / 8  # exact ties
        tau = float(rng.choice([0.5, 0.8, 0.9, 0.95, 0.99]))
        A = np.zeros((1, n, n))
        A[0, n - 1] = a
        rp, ci = oracle.select(A, tau, protect_last=False)
        chosen = ci[rp[n - 1]:rp[n]].tolist()
        T = a.sum()
        best = None
        for k in range(1, n + 1):
            if any(sum(a[list(c)]) >= tau * T for c in itertools.combinations(range(n), k)):
                best = k
                break
        assert len(chosen) == best
        assert a[chosen].sum() >= tau * T * (1 - 1e-15)
        assert chosen == sorted(chosen)
        order = sorted(range(n), key=lambda j: (-a[j], j))
        assert sorted(order[:best]) == chosen


def test_select_nested_in_tau_and_protection():
    w = workloads.get(0, L=1024)
    t = workloads.generate(w)
    A = oracle.estimate(t["Q"], t["K"], w.S, w.B)
    H, Nb = A.shape[0], A.shape[1]
    sets = {}
    for tau in (0.5, 0.8, 0.9, 0.95, 1.0):
        rp, ci = oracle.select(A, tau, protect_last=True)
        sets[tau] = [set(ci[rp[r]:rp[r + 1]].tolist()) for r in range(H * Nb)]
        for r in range(H * Nb):
            I = r % Nb
            lst = ci[rp[r]:rp[r + 1]].tolist()
            assert lst == sorted(set(lst)) and all(0 <= J <= I for J in lst) and len(lst) >= 1
            if I == Nb - 1 or tau >= 1.0:
                assert lst == list(range(I + 1))
    taus = sorted(sets)
    for a, b in zip(taus, taus[1:]):
        assert all(x <= y for x, y in zip(sets[a], sets[b]))
    rp, ci = oracle.select(A, 0.5, protect_last=False)
    last = [set(ci[rp[h * Nb + Nb - 1]:rp[h * Nb + Nb]].tolist()) for h in range(H)]
    assert any(len(s) < Nb for s in last)


# ---------------------------------------------------------------- sparse attention
@pytest.mark.parametrize("H,Hkv,L,d,B", [(2, 2, 128, 16, 32), (4, 2, 96, 8, 16)])
def test_prefill_full_mask_is_dense_causal_attention(H, Hkv, L, d, B):
    Q, K, V = _bf16((H, L, d), 10), _bf16((Hkv, L, d), 11), _bf16((Hkv, L, d), 12)
    rp, ci = oracle.full_csr(H, L // B)
    rows = [(h, q) for h in range(H) for q in range(L)]
    O = oracle.prefill_rows(Q, K, V, B, rp, ci, rows).reshape(H, L, d)
    G = H // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.double(), K.double().repeat_interleave(G, 0), V.double().repeat_interleave(G, 0),
        is_causal=True)
    np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)


def test_prefill_block_mask_matches_masked_softmax():
    H, Hkv, L, d, B = 4, 2, 128, 16, 16
    Q, K, V = _bf16((H, L, d), 13), _bf16((Hkv, L, d), 14), _bf16((Hkv, L, d), 15)
    Nb, G = L // B, H // Hkv
    rng = np.random.default_rng(1)
    A = np.tril(rng.random((H, Nb, Nb)))
    A /= A.sum(-1, keepdims=True)
    rp, ci = oracle.select(A, 0.6, protect_last=False)
    scale = 0.37
    rows = [(h, q) for h in range(H) for q in range(L)]
    O = oracle.prefill_rows(Q, K, V, B, rp, ci, rows, scale=scale).reshape(H, L, d)
    for h in range(H):
        blk = torch.zeros(Nb, Nb, dtype=torch.bool)
        for I in range(Nb):
            blk[I, torch.as_tensor(ci[rp[h * Nb + I]:rp[h * Nb + I + 1]], dtype=torch.long)] = True
        mask = blk.repeat_interleave(B, 0).repeat_interleave(B, 1) & torch.ones(L, L, dtype=torch.bool).tril()
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q[h].double()[None], K[h // G].double()[None], V[h // G].double()[None],
            attn_mask=mask[None], scale=scale)[0]
        np.testing.assert_allclose(O[h], ref.numpy(), rtol=0, atol=1e-12)


def test_oracle_rejects_bad_shapes():
    Q, K = _bf16((3, 64, 8), 0), _bf16((2, 64, 8), 1)
    with pytest.raises(ValueError):
        oracle.estimate(Q, K, 4, 16)   # H % Hkv != 0
    Q, K = _bf16((2, 64, 8), 0), _bf16((2, 64, 8), 1)
    with pytest.raises(ValueError):
        oracle.estimate(Q, K, 3, 16)   # B % S != 0
