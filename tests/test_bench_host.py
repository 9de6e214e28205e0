"""Host-side arithmetic of bench.py (CPU only): roofline fields, traffic table, shared config."""

import os
import types

import pytest

import bench


def test_traffic_table_rows():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.md")) as fh:
        rows = [ln for ln in fh if ln.startswith("| bwd_dkdv ")]
    assert len(rows) == 1
    want = int(rows[0].split("|")[3])
    assert bench.load_traffic("bwd_dkdv") == want
    assert bench.load_traffic("no_such_pass") is None


def test_roofline_tensor_pass():
    step = types.SimpleNamespace(flops_fwd=8.0e9, bytes_dec=2.0e8)
    peaks = {"bf16_tflops": 1600.0, "hbm_gbs": 6500.0}
    comps = {"bwd_dkdv": 0.1, "decode_attention": 0.05}  # milliseconds
    r = bench.roofline_for("bwd_dkdv", comps, step, peaks, "measured")
    # the dK/dV pass does S, dP, dV, dK: twice the forward's FLOPs
    assert r["algorithmic_flops_per_launch"] == pytest.approx(16.0e9)
    assert r["achieved"] == pytest.approx(16.0e9 / 1e-4 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1600.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["kernel"] == "sep_attn_bwd_dkv_kernel"


def test_roofline_decode_pass():
    step = types.SimpleNamespace(flops_fwd=8.0e9, bytes_dec=2.0e8)
    peaks = {"bf16_tflops": 1600.0, "hbm_gbs": 6500.0}
    r = bench.roofline_for("decode_attention", {"decode_attention": 0.05}, step, peaks, "measured")
    assert r["achieved"] == pytest.approx(2.0e8 / 5e-5 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6500.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"


def test_both_arms_share_the_step_configuration():
    a = bench.step_config(2, "flushed", "graph")
    b = bench.step_config(2, "host", "sample")
    for key in ("workload", "train", "decode", "global_batch", "seq_len", "parallelism"):
        assert a[key] == b[key]
    assert a["global_batch"] == 16 and a["parallelism"] == "dp2"
