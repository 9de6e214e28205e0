"""Host-side arithmetic of bench.py (CPU only): roofline fields, traffic table, shared config."""

import os
import types

import pytest

import bench


def test_traffic_table_follows_the_kernel_source(tmp_path, monkeypatch):
    """A capture's DRAM bytes are reported only while the kernel source it was taken from is
    unchanged (the table stores the source file's digest)."""
    import json
    good = bench.source_digest("k_attn_bwd.cu")
    table = {"passes": {"bwd_dkdv": {"source": "k_attn_bwd.cu", "source_sha256": good,
                                     "bytes_per_launch": 123456},
                        "fwd_kernel": {"source": "k_attn_fwd.cu", "source_sha256": "0" * 16,
                                       "bytes_per_launch": 654321}}}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(table))
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(p))
    assert bench.load_traffic("bwd_dkdv") == 123456
    assert bench.load_traffic("fwd_kernel") is None   # source changed since the capture
    assert bench.load_traffic("no_such_pass") is None


def test_committed_traffic_table_is_well_formed():
    import json
    if not os.path.exists(bench.TRAFFIC_JSON):
        pytest.skip("no capture table committed")
    with open(bench.TRAFFIC_JSON) as fh:
        table = json.load(fh)
    for name, e in table["passes"].items():
        assert name in ("fwd_kernel", "bwd_dq", "bwd_dkdv", "decode_attention")
        assert os.path.exists(os.path.join(bench.CSRC, e["source"]))
        assert int(e["bytes_per_launch"]) > 0 and len(e["source_sha256"]) == 16


def test_algorithmic_bytes_of_the_passes():
    # Pythia-160m shape: Q, dO, K, V read, dK, dV written, LSE and Delta (fp32) read
    B, L, H, d = 8, 2048, 12, 64
    t = B * L * H * d * 2
    st = B * H * L * 4
    assert bench.attn_pass_bytes(B, L, H, H, d, "bwd_dkdv") == 6 * t + 2 * st
    assert bench.attn_pass_bytes(B, L, H, H, d, "fwd_kernel") == 4 * t + st
    assert bench.attn_pass_bytes(B, L, H, H, d, "bwd_dq") == 5 * t + 2 * st


def test_pair_slots_counts_whole_tiles():
    import numpy as np
    # L = 512 (4 tiles), n = 64: window tiles t-1..t (t >= 1), tile 0 alone; 200 anchors left
    # of the window of tile 3 make two anchor chunks there
    ge = np.array([[0, 0, 5, 200]])
    slots = bench.pair_slots(ge, 512, 64)
    assert slots == (1 + 2 + (2 + 1) + (2 + 2)) * 128 * 128
    # n >= L: every query tile runs tiles 0..t
    assert bench.pair_slots(np.zeros((1, 4), dtype=int), 512, 512) == (1 + 2 + 3 + 4) * 128 * 128


def test_pair_slots_forward_half_window():
    import numpy as np
    # L = 512, n = 64: query tiles 1..3 have half windows (lower half of tile t-1 outside the
    # band). Anchors: 10 in the lower half of tile 0, 3 in the lower half of tile 1, 7 in the
    # lower half of tile 2 (words 4lo and 4lo + 1 of each tile).
    bits = np.zeros((1, 16), dtype=np.int64)
    bits[0, 0] = (1 << 10) - 1
    bits[0, 4] = 0b111
    bits[0, 9] = (1 << 7) - 1
    # gather_end (anchors left of tile lo): t = 2 sees the 10 of tile 0 plus more in its upper
    # half (say 40 in all), t = 3 sees 170
    ge = np.array([[0, 0, 40, 170]])
    slots = bench.pair_slots(ge, 512, 64, bits)
    # t=0: 1 tile; t=1: G = 0 + 10 <= 64 -> 2 window tiles, no chunk; t=2: G = 43 -> 2;
    # t=3: G = 177 -> 2 + ceil(113 / 128) = 3
    assert slots == (1 + 2 + 2 + 3) * 128 * 128
    # without the bits (dQ, dK/dV): whole chunks of gather_end
    assert bench.pair_slots(ge, 512, 64) == (1 + 2 + 3 + 4) * 128 * 128
    # n = 128: no half windows (the band reaches the lower half), same as without bits
    assert bench.pair_slots(ge, 512, 128, bits) == bench.pair_slots(ge, 512, 128)


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


def test_combined_roofline_takes_the_slower_bound():
    import workloads
    cfg = workloads.PYTHIA160M
    step = types.SimpleNamespace(flops_fwd=8.15e9, bytes_dec=2.0e8, cfg=cfg)
    peaks = {"bf16_tflops": 1638.7, "hbm_gbs": 6555.2}
    r = bench.roofline_for("bwd_dkdv", {"bwd_dkdv": 0.1266}, step, peaks, "measured")
    byts = bench.attn_pass_bytes(cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.d, "bwd_dkdv")
    assert byts == pytest.approx(152.6e6, rel=2e-3)
    t_min = max(2 * 8.15e9 / 1638.7e12, byts / 6555.2e9)
    assert r["combined_frac"] == pytest.approx(t_min / 0.1266e-3)
    assert r["combined_bound"] == "hbm"


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
