"""GPU parity of sep_attn_fwd / sep_attn_bwd against the fp64 oracle.

Small and ragged shapes are compared element by element on every output; the configured
workloads are compared in full where the oracle finishes in seconds (tiny GQA, Pythia-160m
training shape) and on sampled rows through the gathered form of the oracle otherwise
(Llama-3-8B prefill, 131072-token stress case). Tolerances: forward max-abs 2e-2 and mean-abs
2e-3, gradients relative L2 1e-2.
"""

import numpy as np
import pytest

from gpu_common import check_grad, check_lse, check_out, f64
from oracle import sepattn_ref as R

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import torch
    assert torch.cuda.is_available()
    from kv_cache_compression_sep_b200 import sepattn
    return sepattn


def _inputs(seed, B, L, Hq, Hkv, d, p, kind="bernoulli", flags=None):
    import workloads
    inp = workloads.small_attn_inputs(seed, B, L, Hq, Hkv, d, p=p, kind=kind)
    if flags is not None:
        inp["sep"] = flags
    return inp


def _to_dev(inp):
    return {k: (v.cuda() if v is not None else None) for k, v in inp.items()}


def _fwd(S, dev, a, n):
    import torch
    mask = S.sep_mask_build(dev["sep"], a, n)
    o, lse = S.sep_attn_fwd(dev["q"], dev["k"], dev["v"], mask)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    return mask, o, lse


SMALL = [
    # B, L, Hq, Hkv, d, a, n, p
    (1, 128, 1, 1, 64, 0, 1, 0.0),
    (1, 200, 2, 1, 64, 4, 64, 0.1),
    (2, 300, 4, 2, 128, 1, 127, 0.1),
    (1, 385, 4, 4, 64, 4, 128, 0.1),
    (1, 512, 8, 1, 128, 4, 256, 0.08),
    (2, 640, 2, 2, 64, 0, 64, 1.0),
    (1, 700, 4, 1, 128, 3, 1000, 0.1),
    (1, 1030, 2, 1, 64, 4, 64, 0.3),
    (1, 333, 8, 8, 128, 0, 5, 0.0),
    (1, 520, 4, 2, 64, 2, 65, 0.15),    # the widest band with half-window pairs at d = 64
    (1, 300, 2, 1, 64, 1, 5, 0.2),      # a narrow band: half-window pairs, few kept per row
]


@pytest.mark.parametrize("B,L,Hq,Hkv,d,a,n,p", SMALL)
def test_fwd_small(S, B, L, Hq, Hkv, d, a, n, p):
    inp = _inputs(L + n, B, L, Hq, Hkv, d, p)
    _, o, lse = _fwd(S, _to_dev(inp), a, n)
    Or, LSEr = R.attn_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), inp["sep"].numpy(), a, n,
                          d ** -0.5)
    check_out(f64(o), Or, "O")
    check_lse(f64(lse), LSEr, "LSE")


@pytest.mark.parametrize("B,L,Hq,Hkv,d,a,n,p", SMALL)
def test_bwd_small(S, B, L, Hq, Hkv, d, a, n, p):
    import torch
    inp = _inputs(L + n + 1, B, L, Hq, Hkv, d, p)
    dev = _to_dev(inp)
    mask, o, lse = _fwd(S, dev, a, n)
    dq, dk, dv = S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    dqr, dkr, dvr = R.attn_bwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["do"]),
                               inp["sep"].numpy(), a, n, d ** -0.5)
    check_grad(f64(dq), dqr, "dQ")
    check_grad(f64(dk), dkr, "dK")
    check_grad(f64(dv), dvr, "dV")


def test_fixed_interval_anchors(S):
    """FixLLM-style anchors (every 16th token) through forward and backward."""
    import torch
    L = 600
    flags = torch.zeros(1, L, dtype=torch.uint8)
    flags[0, 15::16] = 1
    inp = _inputs(3, 1, L, 4, 2, 64, 0.0, flags=flags)
    dev = _to_dev(inp)
    mask, o, lse = _fwd(S, dev, 2, 32)
    dq, dk, dv = S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask)
    torch.cuda.synchronize()
    args = (f64(inp["q"]), f64(inp["k"]), f64(inp["v"]))
    Or, _ = R.attn_fwd(*args, flags.numpy(), 2, 32, 0.125)
    check_out(f64(o), Or)
    dqr, dkr, dvr = R.attn_bwd(*args, f64(inp["do"]), flags.numpy(), 2, 32, 0.125)
    check_grad(f64(dq), dqr)
    check_grad(f64(dk), dkr)
    check_grad(f64(dv), dvr)


def test_varlen_right_padded(S):
    """Variable lengths through right padding: rows below each sequence's length equal the
    unpadded sequence's attention (causal: real rows never read padded keys), and with dO zero
    on padded rows the gradients of the real rows and keys equal the unpadded ones."""
    import torch
    lens, L, Hq, Hkv, d, a, n = (300, 517), 517, 4, 2, 64, 4, 64
    inp = _inputs(77, len(lens), L, Hq, Hkv, d, 0.15)
    for b, lb in enumerate(lens):
        inp["do"][b, lb:] = 0
    dev = _to_dev(inp)
    mask, o, lse = _fwd(S, dev, a, n)
    dq, dk, dv = S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    for b, lb in enumerate(lens):
        sl = lambda t: f64(t[b:b + 1, :lb])  # noqa: E731
        sep = inp["sep"][b:b + 1, :lb].numpy()
        Or, LSEr = R.attn_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sep, a, n, d ** -0.5)
        check_out(f64(o[b:b + 1, :lb]), Or, f"O seq {b}")
        check_lse(f64(lse[b:b + 1, :, :lb]), LSEr, f"LSE seq {b}")
        dqr, dkr, dvr = R.attn_bwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["do"]), sep, a,
                                   n, d ** -0.5)
        check_grad(f64(dq[b:b + 1, :lb]), dqr, f"dQ seq {b}")
        check_grad(f64(dk[b:b + 1, :lb]), dkr, f"dK seq {b}")
        check_grad(f64(dv[b:b + 1, :lb]), dvr, f"dV seq {b}")


def _cfg_inputs(name):
    import workloads
    cfg = workloads.ATTN_CONFIGS[name]
    return cfg, workloads.attn_inputs(cfg)


def test_tiny_config_full(S):
    cfg, inp = _cfg_inputs("tiny-gqa-L512-d64")
    _, o, lse = _fwd(S, _to_dev(inp), cfg.a, cfg.n)
    Or, LSEr = R.attn_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), inp["sep"].numpy(), cfg.a,
                          cfg.n, cfg.scale)
    check_out(f64(o), Or, "O")
    check_lse(f64(lse), LSEr, "LSE")


def test_pythia_config_full(S):
    import torch
    cfg, inp = _cfg_inputs("pythia160m-train-B8-H12-L2048-d64")
    dev = _to_dev(inp)
    mask, o, lse = _fwd(S, dev, cfg.a, cfg.n)
    dq, dk, dv = S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    args = (f64(inp["q"]), f64(inp["k"]), f64(inp["v"]))
    sep = inp["sep"].numpy()
    Or, LSEr = R.attn_fwd(*args, sep, cfg.a, cfg.n, cfg.scale)
    check_out(f64(o), Or, "O")
    check_lse(f64(lse), LSEr, "LSE")
    dqr, dkr, dvr = R.attn_bwd(*args, f64(inp["do"]), sep, cfg.a, cfg.n, cfg.scale)
    check_grad(f64(dq), dqr, "dQ")
    check_grad(f64(dk), dkr, "dK")
    check_grad(f64(dv), dvr, "dV")


def _sample_rows(L, rng, blocks=3, extra=24):
    rows = list(range(0, 128)) + list(range(L - 128, L)) + list(range(L // 2, L // 2 + 64))
    rows += [int(x) for x in rng.integers(0, L, extra)]
    return sorted(set(rows))


def test_llama_prefill_sampled(S):
    cfg, inp = _cfg_inputs("llama3-8b-prefill-H32-8-L8192-d128")
    _, o, lse = _fwd(S, _to_dev(inp), cfg.a, cfg.n)
    rows = _sample_rows(cfg.L, np.random.default_rng(1))
    Or, LSEr = R.attn_fwd_rows(inp["q"].float().numpy(), inp["k"].float().numpy(),
                               inp["v"].float().numpy(), inp["sep"].numpy(), cfg.a, cfg.n,
                               cfg.scale, 0, rows)
    check_out(f64(o)[0, rows], Or, "O")
    check_lse(f64(lse)[0][:, rows].T, LSEr, "LSE")


@pytest.mark.parametrize("all_keep", [False, True])
def test_long_context_sampled(S, all_keep):
    """L = 131072 forward + backward; all_keep runs n = L (dense causal) through the same kernels."""
    import torch
    cfg, inp = _cfg_inputs("long-context-H32-8-L131072-d128")
    n = cfg.L if all_keep else cfg.n
    dev = _to_dev(inp)
    mask, o, lse = _fwd(S, dev, cfg.a, n)
    dq, dk, dv = S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    qf, kf, vf, dof = (inp[x].float().numpy() for x in ("q", "k", "v", "do"))
    sep = inp["sep"].numpy()
    rng = np.random.default_rng(2)
    rows = [0, 1, 127, 128, 4095, 65536, cfg.L - 129, cfg.L - 1] + [int(x) for x in rng.integers(0, cfg.L, 4)]
    Or, LSEr = R.attn_fwd_rows(qf, kf, vf, sep, cfg.a, n, cfg.scale, 0, rows)
    check_out(f64(o)[0, rows], Or, "O")
    check_lse(f64(lse)[0][:, rows].T, LSEr, "LSE")
    # gradients: dQ on sampled rows; dK/dV on keys whose keeping queries are few (non-anchor
    # keys anywhere, anchors near the end)
    f = R.anchor_flags(sep[0], cfg.a)
    if all_keep:
        keys = [cfg.L - 1, cfg.L - 2]
    else:
        non_anchor = np.nonzero(~f)[0]
        late_anchor = np.nonzero(f[cfg.L - 300:])[0] + cfg.L - 300
        keys = [int(non_anchor[5]), int(non_anchor[-3])] + [int(x) for x in late_anchor[:2]]
    qrows = [0, 4095, cfg.L - 1]
    dqr, dkr, dvr = R.attn_bwd_sampled(qf, kf, vf, dof, sep, cfg.a, n, cfg.scale, 0, qrows, keys)
    check_grad(f64(dq)[0, qrows], dqr, "dQ")
    check_grad(f64(dk)[0, keys], dkr, "dK")
    check_grad(f64(dv)[0, keys], dvr, "dV")
