"""GPU parity of the backward at sequence lengths where its dK/dV pass changes path.

Every element of dQ, dK and dV (and of O, LSE) is compared with the full fp64 oracle
(`attn_bwd`, the materialised mask) on shapes chosen to force each path of the key-major
dK/dV pass:
  * anchor chunks gathered by more than 16 query tiles: such an anchor item is split into
    segments of 16 query tiles whose fp32 partial sums several CTAs add up;
  * windows wider than 16 key tiles (n > 1920 with more than 16 query tiles): window items are
    split into segments too, and every key row accumulates into position-indexed fp32 sums;
  * all-keep (n = L, dense causal) through the same segmented path;
  * ragged lengths, so that the last query and key tiles are partly outside the sequence.
Tolerances as everywhere: forward max-abs 2e-2 / mean-abs 2e-3, gradients relative L2 1e-2.
The mask is that of the SepLLM summary (atlas.scime.ai, "Approach"); training uses the same
mask (beiduofen.top, "The Mechanics of Compression: Why Separators Work").
"""

import pytest

from gpu_common import check_grad, check_lse, check_out, f64
from oracle import sepattn_ref as R

pytestmark = pytest.mark.gpu

LONG = [
    # B, L, Hq, Hkv, d, a, n, p
    (1, 4096, 4, 2, 128, 4, 64, 0.1),     # anchor chunk 0 gathered by ~30 query tiles
    (1, 4000, 2, 1, 64, 4, 64, 0.1),      # the same, ragged, d = 64
    (1, 2560, 2, 1, 64, 4, 64, 0.1),      # 20 query tiles: two segments per early anchor chunk
    (1, 2560, 2, 1, 64, 4, 2200, 0.1),    # windows of 19 key tiles: segmented window items
    (1, 4096, 2, 1, 64, 4, 2200, 0.1),    # the same over 32 query tiles
    (1, 4000, 2, 1, 128, 0, 4000, 0.0),   # all-keep (dense causal), ragged, d = 128
    (2, 2300, 4, 1, 64, 2, 2300, 0.05),   # all-keep, two sequences, G = 4
]


@pytest.fixture(scope="module")
def S():
    import torch
    assert torch.cuda.is_available()
    from kv_cache_compression_sep_b200 import sepattn
    return sepattn


@pytest.mark.parametrize("B,L,Hq,Hkv,d,a,n,p", LONG)
def test_bwd_long_every_element(S, B, L, Hq, Hkv, d, a, n, p):
    import torch
    import workloads
    inp = workloads.small_attn_inputs(L + 7 * n + d, B, L, Hq, Hkv, d, p=p)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    mask = S.sep_mask_build(dev["sep"], a, n)
    o, lse = S.sep_attn_fwd(dev["q"], dev["k"], dev["v"], mask)
    dq, dk, dv = S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    args = (f64(inp["q"]), f64(inp["k"]), f64(inp["v"]))
    sep = inp["sep"].numpy()
    Or, LSEr = R.attn_fwd(*args, sep, a, n, d ** -0.5)
    check_out(f64(o), Or, "O")
    check_lse(f64(lse), LSEr, "LSE")
    dqr, dkr, dvr = R.attn_bwd(*args, f64(inp["do"]), sep, a, n, d ** -0.5)
    check_grad(f64(dq), dqr, "dQ")
    check_grad(f64(dk), dkr, "dK")
    check_grad(f64(dv), dvr, "dV")
    # the rows the segmented paths write are compared one by one as well: the anchors of the
    # first 128 compacted positions (gathered by the most query tiles) and the first keys
    f = R.anchor_flags(sep[0], a)
    early = [int(j) for j in range(L) if f[j]][:128] + list(range(min(L, 256)))
    for name, got, ref in (("dK", dk, dkr), ("dV", dv, dvr)):
        check_grad(f64(got)[0, early], ref[0, early], f"{name} early rows")


def test_bwd_long_repeatable_within_tolerance(S):
    """Two backward calls on the same inputs: the fp32 atomic sums of multi-segment anchor rows
    may differ in their last bits between runs (addition order), but never beyond rounding."""
    import numpy as np
    import torch
    import workloads
    B, L, Hq, Hkv, d, a, n, p = 1, 4096, 4, 2, 128, 4, 64, 0.1
    inp = workloads.small_attn_inputs(99, B, L, Hq, Hkv, d, p=p)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    mask = S.sep_mask_build(dev["sep"], a, n)
    o, lse = S.sep_attn_fwd(dev["q"], dev["k"], dev["v"], mask)
    g1 = S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask)
    g2 = S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    assert torch.equal(g1[0], g2[0]), "dQ is formed without atomics and must be bit-identical"
    for x, y in zip(g1[1:], g2[1:]):
        a64, b64 = f64(x), f64(y)
        scale = np.abs(a64).max()
        assert np.abs(a64 - b64).max() <= 2 ** -7 * scale
