"""The seeded input generators: deterministic per seed, and the flag patterns they promise."""

import numpy as np
import torch

import workloads


def test_seed_determinism():
    a = workloads.small_attn_inputs(7, 1, 64, 2, 1, 64)
    b = workloads.small_attn_inputs(7, 1, 64, 2, 1, 64)
    for k in ("sep", "q", "k", "v", "do"):
        assert torch.equal(a[k], b[k])
    c = workloads.small_attn_inputs(8, 1, 64, 2, 1, 64)
    assert not torch.equal(a["q"], c["q"])


def test_bernoulli_density_and_forced_first_position():
    g = torch.Generator().manual_seed(0)
    sep = workloads.separator_flags(g, 4, 20000, "bernoulli", 0.08, force0=True).numpy()
    assert abs(sep.mean() - 0.08) < 0.005
    assert (sep[:, 0] == 0).all()


def test_geometric_segments_end_in_separators():
    g = torch.Generator().manual_seed(1)
    sep = workloads.separator_flags(g, 3, 50000, "geometric", 0.1).numpy()
    for row in sep:
        ends = np.nonzero(row)[0]
        lens = np.diff(np.concatenate([[-1], ends]))  # segment lengths up to each separator
        assert (lens >= 1).all()
        assert abs(lens.mean() - 10.0) < 0.5           # Geometric(p = 0.1): mean 1/p


def test_decode_chunks_regenerate_identically():
    cfg = workloads.SEPCACHE_DECODE
    a = workloads.decode_chunk(cfg, 250, 12, S=3)
    b = workloads.decode_chunk(cfg, 256, 6, S=3)    # a sub-range, drawn alone
    for k in ("sep", "q", "k", "v"):
        assert torch.equal(a[k][6:], b[k])
