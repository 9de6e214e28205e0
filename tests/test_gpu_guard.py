"""Out-of-bounds write checks on the GPU (a stand-in for a memory sanitizer).

Every output and workspace buffer of the library is carved out of a larger allocation whose
margins on both sides (and the alignment padding right after the buffer) are filled with a
sentinel byte. After mask build, forward, backward, cache prefill, update, decode and export on
small ragged shapes, every margin must still hold the sentinel: no kernel writes a byte past
the buffers it is given. The outputs themselves are also checked against the fp64 oracle, so
that a kernel that wrote nothing would not pass.
"""

import numpy as np
import pytest

from gpu_common import check_grad, check_out, f64
from oracle import sepattn_ref as R
from oracle import sepcache_ref as C

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5
MARGIN = 4096


@pytest.fixture(scope="module")
def S():
    import torch
    assert torch.cuda.is_available()
    from kv_cache_compression_sep_b200 import sepattn
    return sepattn


class Guarded:
    """Tensors carved out of sentinel-filled allocations, and the check of their margins."""

    def __init__(self):
        self.bufs = []

    def tensor(self, shape, dtype, name, fill=None):
        import torch
        esz = torch.tensor([], dtype=dtype).element_size()
        n = int(np.prod(shape)) * esz
        total = MARGIN + (n + 255) // 256 * 256 + MARGIN
        buf = torch.full((total,), SENTINEL, dtype=torch.uint8, device="cuda")
        t = buf[MARGIN:MARGIN + n].view(dtype).view(*shape)
        if fill is not None:
            t.fill_(fill)
        self.bufs.append((name, buf, MARGIN, MARGIN + n))
        return t

    def check(self):
        import torch
        torch.cuda.synchronize()
        for name, buf, lo, hi in self.bufs:
            b = buf.cpu().numpy()
            bad_lo = np.nonzero(b[:lo] != SENTINEL)[0]
            bad_hi = np.nonzero(b[hi:] != SENTINEL)[0]
            assert bad_lo.size == 0, f"{name}: {bad_lo.size} bytes written before the buffer"
            assert bad_hi.size == 0, f"{name}: {bad_hi.size} bytes written after the buffer"


ATTN = [
    # B, L, Hq, Hkv, d, a, n, p
    (1, 1, 4, 2, 64, 4, 64, 0.2),
    (1, 129, 4, 2, 64, 4, 64, 0.2),
    (2, 300, 4, 2, 128, 4, 64, 0.2),
    (1, 1030, 4, 2, 64, 2, 200, 0.2),
    (1, 1030, 2, 1, 128, 4, 1030, 0.1),   # all-keep
    (2, 517, 4, 2, 64, 4, 64, 0.15),      # the right-padded varlen shape
]


@pytest.mark.parametrize("B,L,Hq,Hkv,d,a,n,p", ATTN)
def test_attention_writes_stay_inside_buffers(S, B, L, Hq, Hkv, d, a, n, p):
    import torch
    import workloads
    inp = workloads.small_attn_inputs(L * 3 + d + n, B, L, Hq, Hkv, d, p=p)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    g = Guarded()
    T, W = -(-L // 128), -(-L // 32)
    mask = S.SepMask(sep=dev["sep"],
                     anchor_idx=g.tensor((B, L), torch.int32, "anchor_idx"),
                     anchor_cnt=g.tensor((B,), torch.int32, "anchor_cnt"),
                     anchor_bits=g.tensor((B, W), torch.int32, "anchor_bits"),
                     gather_end=g.tensor((B, T), torch.int32, "gather_end"),
                     tile_map=g.tensor((B, T, T), torch.int8, "tile_map"),
                     kept=g.tensor((B,), torch.int64, "kept"), a=a, n=n)
    S.sep_mask_build(dev["sep"], a, n, out=mask)
    o = g.tensor((B, L, Hq, d), torch.bfloat16, "o")
    lse = g.tensor((B, Hq, L), torch.float32, "lse")
    ws_f = g.tensor((S.sep_attn_fwd_workspace_size(B, L, Hkv, d),), torch.uint8, "fwd workspace")
    S.sep_attn_fwd(dev["q"], dev["k"], dev["v"], mask, out=o, lse=lse, workspace=ws_f)
    grads = (g.tensor((B, L, Hq, d), torch.bfloat16, "dq"),
             g.tensor((B, L, Hkv, d), torch.bfloat16, "dk"),
             g.tensor((B, L, Hkv, d), torch.bfloat16, "dv"))
    ws_b = g.tensor((S.sep_attn_bwd_workspace_size(B, L, Hq, Hkv, d),), torch.uint8,
                    "bwd workspace")
    S.sep_attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], mask, workspace=ws_b,
                   grads=grads)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    g.check()
    args = (f64(inp["q"]), f64(inp["k"]), f64(inp["v"]))
    Or, _ = R.attn_fwd(*args, inp["sep"].numpy(), a, n, d ** -0.5)
    check_out(f64(o), Or, "O")
    dqr, dkr, dvr = R.attn_bwd(*args, f64(inp["do"]), inp["sep"].numpy(), a, n, d ** -0.5)
    for got, ref, name in zip(grads, (dqr, dkr, dvr), ("dQ", "dK", "dV")):
        check_grad(f64(got), ref, name)


def _guarded_cache(S, g, Sq, Hq, Hkv, d, a, s, w, c, orig=False):
    """A SepCache whose state tensors live in guarded allocations."""
    import ctypes
    import torch
    cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0, c=c, original_positions=orig)
    n = cache.n
    cache.k_slots = g.tensor((Sq, Hkv, n, d), torch.bfloat16, "k_slots", fill=0)
    cache.v_slots = g.tensor((Sq, Hkv, n, d), torch.bfloat16, "v_slots", fill=0)
    cache.slot_pos = g.tensor((Sq, n), torch.int32, "slot_pos")
    cache.slot_sep = g.tensor((Sq, n), torch.uint8, "slot_sep")
    cache.meta = g.tensor((Sq, S.META), torch.int32, "meta")
    cache.rope_freq = g.tensor((d // 2,), torch.float64, "rope_freq")
    cache._st = S._SepCacheState(Sq, Hq, Hkv, d, a, s, w, c, int(orig), 500000.0,
                                 cache.k_slots.data_ptr(), cache.v_slots.data_ptr(),
                                 cache.slot_pos.data_ptr(), cache.slot_sep.data_ptr(),
                                 cache.meta.data_ptr(), cache.rope_freq.data_ptr())
    S._check(S._lib.sepcache_state_init(ctypes.byref(cache._st), S._stream()), "init")
    return cache


@pytest.mark.parametrize("Sq,Hq,Hkv,d,a,s,w,c,L,steps,orig", [
    (2, 8, 2, 128, 4, 6, 20, 0, 37, 60, False),
    (3, 6, 2, 64, 2, 5, 11, 30, 53, 80, False),    # Past Window, G = 3
    (2, 8, 1, 128, 0, 3, 9, 0, 1, 40, True),       # no shifting, one-token prompt
])
def test_cache_writes_stay_inside_buffers(S, Sq, Hq, Hkv, d, a, s, w, c, L, steps, orig):
    import torch
    g = Guarded()
    cache = _guarded_cache(S, g, Sq, Hq, Hkv, d, a, s, w, c, orig)
    gen = torch.Generator().manual_seed(Sq * 100 + L)
    k = torch.randn(Sq, L, Hkv, d, generator=gen).to(torch.bfloat16)
    v = torch.randn(Sq, L, Hkv, d, generator=gen).to(torch.bfloat16)
    sep = (torch.rand(Sq, L, generator=gen) < 0.3).to(torch.uint8)
    cache.sepcache_prefill(k.cuda(), v.cuda(), sep.cuda())
    sims = [C.SepCacheSim(a, s, w, c if c > 0 else None) for _ in range(Sq)]
    K = [f64(k[:, t]) for t in range(L)]
    V = [f64(v[:, t]) for t in range(L)]
    for sq in range(Sq):
        for t in range(L):
            sims[sq].append(bool(sep[sq, t]))
    o = g.tensor((Sq, Hq, d), torch.bfloat16, "decode o")
    lse = g.tensor((Sq, Hq), torch.float32, "decode lse")
    for t in range(L, L + steps):
        kn = torch.randn(Sq, Hkv, d, generator=gen).to(torch.bfloat16)
        vn = torch.randn(Sq, Hkv, d, generator=gen).to(torch.bfloat16)
        qn = torch.randn(Sq, Hq, d, generator=gen).to(torch.bfloat16)
        sn = (torch.rand(Sq, generator=gen) < 0.3).to(torch.uint8)
        K.append(f64(kn))
        V.append(f64(vn))
        cache.sepcache_update(kn.cuda(), vn.cuda(), sn.cuda())
        cache.sepcache_decode(qn.cuda(), out=o, lse=lse)
        for sq in range(Sq):
            sims[sq].append(bool(sn[sq]))
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    g.check()
    # the last step's outputs against the oracle
    theta = 500000.0
    for sq in range(Sq):
        order = sims[sq].order()
        kr = np.stack([K[j][sq] for j in order])
        vr = np.stack([V[j][sq] for j in order])
        if orig:
            ks = C.stored_rotated_key(kr, np.array(order)[:, None], theta)
            ro, _ = C.decode_attention_original_positions(f64(qn[sq]), ks, vr, t, theta,
                                                          d ** -0.5)
        else:
            ro, _ = C.decode_attention(f64(qn[sq]), kr, vr, theta, d ** -0.5)
        check_out(f64(o[sq]), ro, f"seq {sq}")
    pos = g.tensor((Sq, cache.n), torch.int32, "export pos")
    cnt = g.tensor((Sq,), torch.int32, "export count")
    import ctypes
    S._check(S._lib.sepcache_export_order(ctypes.byref(cache._st), S._ptr(pos), S._ptr(cnt),
                                          S._stream()), "export")
    g.check()
    for sq in range(Sq):
        assert pos[sq, : int(cnt[sq])].tolist() == sims[sq].order()
