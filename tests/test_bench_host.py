"""bench.py's host-side measurement arithmetic, on CPU: the roofline of the
dominant kernel (algorithmic flops or bytes per profiled launch over the
measured time, against the peak), the measured-traffic lookup that must go
stale when the kernel's code changes (but not when only its comments do), and
the algorithmic step floor."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synth  # noqa: E402

DIMS = synth.CONFIGS["qwen3_8b_b16"]["model"]
PK = {"hbm": 6500.0, "tc": 1600.0, "tc_sus": 1400.0, "src": "test"}


def _profile(M, us_per_launch):
    """One profiled step: each projection kind launched its per-step count of times."""
    return {k: (cnt * us_per_launch / 1e3, cnt) for k, (cnt, m, n, kk) in bench.gemm_shapes(DIMS, M).items()}


def test_roofline_tensor_bound_at_256_rows():
    M = 256
    r, _, _ = bench.roofline(_profile(M, 50.0), DIMS, M, PK, "no-such-workload")
    shapes = bench.gemm_shapes(DIMS, M)
    flops = sum(cnt * 2.0 * m * n * k for cnt, m, n, k in shapes.values())
    launches = sum(cnt for cnt, *_ in shapes.values())
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == PK["tc_sus"]
    assert r["launches_profiled"] == launches
    assert r["achieved"] == pytest.approx(flops / (launches * 50e-6) / 1e12, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / PK["tc_sus"], rel=1e-3)
    assert r["traffic"] is None  # no capture for this workload


def test_roofline_hbm_bound_at_16_rows():
    M = 16
    r, _, _ = bench.roofline(_profile(M, 20.0), DIMS, M, PK, "no-such-workload")
    shapes = bench.gemm_shapes(DIMS, M)
    byt = sum(cnt * (2.0 * n * k + 2.0 * m * k + 4.0 * m * n) for cnt, m, n, k in shapes.values())
    launches = sum(cnt for cnt, *_ in shapes.values())
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == PK["hbm"]
    assert r["achieved"] == pytest.approx(byt / (launches * 20e-6) / 1e9, rel=1e-3)


def _fake_tree(tmp_path, code):
    csrc = tmp_path / "streaming_decoding_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(code)
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_lookup_follows_code_not_comments(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path, "// header\n__global__ void k() { int a = 1; }  // tail\n/* block */\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path / "profiles"))
    h = bench.src_hash("k.cu")
    (tmp_path / "profiles" / "k.json").write_text(json.dumps(
        {"workload": "w", "sources": ["k.cu"], "source_hash": h, "dram_bytes_per_launch": 123}))
    assert bench.measured_traffic("k", "w") == 123
    assert bench.measured_traffic("k", "other") is None            # another workload
    (csrc / "k.cu").write_text("// a new comment\n__global__ void k() { int a = 1; }\n")
    assert bench.measured_traffic("k", "w") == 123                 # comments only: still valid
    (csrc / "k.cu").write_text("__global__ void k() { int a = 2; }\n")
    assert bench.measured_traffic("k", "w") is None                # code changed: stale


def test_committed_gemm_traffic_profile_is_well_formed():
    with open(os.path.join(ROOT, "profiles", "gemm_tc.json")) as f:
        p = json.load(f)
    assert p["workload"] == "qwen3_8b_b16" and p["sources"] == ["gemm_tc.cu", "gemm_tc.cuh"]
    per, cnt = p["per_projection_dram_bytes"], p["launches_per_step"]
    avg = sum(per[k] * cnt[k] for k in per) / sum(cnt.values())
    assert p["dram_bytes_per_launch"] == pytest.approx(avg, rel=1e-6)
    # every projection reads at least its weights once
    for k, (c, m, n, kk) in bench.gemm_shapes(DIMS, 256).items():
        assert per[k] >= 2 * n * kk


def test_step_floor_counts_weights_kv_and_logits():
    B, W, S = 16, 16, 600.0
    byt, fl = bench.step_bytes_flops(DIMS, B, W, S)
    d, hq, hkv, hd, F, V, L = (DIMS[k] for k in ("d", "hq", "hkv", "hd", "F", "V", "L"))
    params = L * ((hq + 2 * hkv) * hd * d + d * hq * hd + 3 * F * d) + V * d
    assert byt == pytest.approx(2.0 * params + B * S * L * 2 * hkv * hd * 2 + B * W * V * 4)
    assert 15.0e9 < 2.0 * params < 15.3e9  # the 15.1 GB of bf16 weights per step
    assert fl > 2.0 * B * W * params
