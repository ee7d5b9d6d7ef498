"""Seeded generators: deterministic, right shapes, planted structure present."""
import math

import torch

import workloads


def test_deterministic_and_shapes():
    for idx in range(5):
        w = workloads.get(idx)
        small = w.with_(L=max(w.B * 4, w.frame_len * 2 if w.recipe == "video" else 0))
        a, b = workloads.generate(small, seed=0), workloads.generate(small, seed=0)
        for k in "QKV":
            assert torch.equal(a[k].view(torch.int16), b[k].view(torch.int16))
            assert a[k].dtype == torch.bfloat16 and a[k].is_contiguous()
        assert a["Q"].shape == (w.H, small.L, w.d)
        assert a["K"].shape == (w.Hkv, small.L, w.d) == a["V"].shape
        c = workloads.generate(small, seed=1)
        assert not torch.equal(a["Q"].view(torch.int16), c["Q"].view(torch.int16))


def test_sinks_and_ar_correlation():
    w = workloads.get(0)
    t = workloads.generate(w)
    K = t["K"].float()
    # sink keys (positions 0..3) carry the large shared direction: norm about sqrt(1 + 9) x background
    n_sink = K[:, :4].norm(dim=-1).mean()
    n_bg = K[:, 100:].norm(dim=-1).mean()
    assert n_sink > 2.5 * n_bg
    # AR(1) with coefficient 0.8 along t
    x = K[:, 100:-1].flatten()
    y = K[:, 101:].flatten()
    rho = torch.corrcoef(torch.stack([x, y]))[0, 1].item()
    assert abs(rho - 0.8) < 0.02
    assert abs(n_bg.item() / (0.5 * math.sqrt(w.d)) - 1.0) < 0.05


def test_video_frames_correlated():
    w = workloads.get(4, L=4096)
    K = workloads.generate(w)["K"].float()
    same = torch.nn.functional.cosine_similarity(K[0, 10], K[0, 900], dim=0)
    assert same > 0.6


def test_bench_flop_accounting():
    # with every causal block selected, the selected-block FLOPs (4*B*B*d per off-diagonal
    # block, 4*d*B*(B+1)/2 per diagonal block) equal the dense causal FLOPs 4*d*H*L*(L+1)/2
    import os
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import oracle

    for w in (workloads.get(0), workloads.get(1, H=3, Hkv=1, L=1024), workloads.get(4, L=2048)):
        rp, ci = oracle.full_csr(w.H, w.Nb)
        flops, n_diag, n_off = bench.selected_flops(rp, ci, w.H, w.Nb, w.B, w.d)
        assert n_diag == w.H * w.Nb and n_off == w.H * w.Nb * (w.Nb - 1) // 2
        assert flops == bench.dense_causal_flops(w)


def test_bench_traffic_comes_from_the_matching_capture(tmp_path, monkeypatch):
    # the roofline's DRAM traffic is a committed ncu record at 32K scaled by L, for the
    # captured shape only, and only while every source the record names hashes as recorded
    import hashlib
    import json
    import os
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench

    w32, w128 = workloads.get(1), workloads.get(2)
    fake = tmp_path / "repo"
    (fake / "profiles").mkdir(parents=True)
    src = fake / "kernel.cu"
    src.write_text("// kernel source\n")
    rec = {"shape": {"H": w32.H, "Hkv": w32.Hkv, "L": w32.L, "d": w32.d, "B": w32.B},
           "dram_bytes_read": 3.0e8, "dram_bytes_write": 1.0e8,
           "sources": {"kernel.cu": hashlib.sha256(src.read_bytes()).hexdigest()[:16]}}
    name = bench.PREFILL_RECORDS[w32.B]
    (fake / "profiles" / (name + ".json")).write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(fake))
    assert bench.prefill_traffic_per_launch(w32) == 4.0e8
    assert bench.prefill_traffic_per_launch(w128) == 4 * 4.0e8
    assert bench.prefill_traffic_per_launch(workloads.get(0)) is None      # other shape
    src.write_text("// kernel source\n// edited\n")                       # changed kernel
    assert bench.prefill_traffic_per_launch(w32) is None


def test_committed_counter_records_name_existing_sources():
    import glob
    import json
    import os

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    recs = [r for r in glob.glob(os.path.join(root, "profiles", "*.json")) if "mask_parity" not in r]
    assert recs
    for r in recs:
        rec = json.load(open(r))
        assert rec["sources"] and "command" in rec and "shape" in rec, r
        for path, digest in rec["sources"].items():
            assert os.path.exists(os.path.join(root, path)) and len(digest) == 16, (r, path)
