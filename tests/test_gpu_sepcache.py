"""GPU parity of sepcache_update / sepcache_decode against the SepCache oracle.

The retained-position trajectory (logical order of original positions) is compared bit-exactly;
decode outputs are compared with the fp64 oracle at the forward tolerances.
"""

import numpy as np
import pytest

from gpu_common import DECODE_LSE_ABS, check_out, f64
from oracle import sepcache_ref as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import torch
    assert torch.cuda.is_available()
    from kv_cache_compression_sep_b200 import sepattn
    return sepattn


@pytest.mark.parametrize("Sq,Hq,Hkv,d,a,s,w,steps,p,c", [
    (3, 8, 2, 128, 4, 6, 20, 120, 0.2, 0),
    (2, 4, 4, 64, 0, 3, 7, 60, 0.5, 0),
    (2, 8, 1, 128, 2, 0, 9, 50, 0.3, 0),     # s = 0: StreamingLLM with shifting
    (1, 16, 2, 64, 1, 2, 1, 30, 0.6, 0),     # window of one slot
    (2, 32, 8, 128, 4, 64, 300, 500, 0.1, 0),
    # Past Window Cache, compressed when the usage reaches c
    (3, 8, 2, 128, 4, 6, 20, 200, 0.2, 45),
    (2, 4, 4, 64, 0, 3, 7, 120, 0.5, 14),
    (2, 8, 1, 128, 2, 0, 9, 80, 0.3, 20),    # s = 0: compression drops the past window
    (1, 16, 2, 64, 1, 2, 1, 60, 0.6, 7),     # window of one slot
    (2, 32, 8, 128, 4, 64, 256, 900, 0.1, 800),
    # query heads per KV head that are not a power of two (padded with zero queries)
    (2, 6, 2, 128, 4, 6, 20, 120, 0.2, 0),
    (2, 12, 4, 64, 2, 5, 11, 90, 0.3, 30),
    (1, 40, 8, 128, 4, 8, 30, 80, 0.2, 0),
    (2, 16, 2, 64, 1, 4, 9, 70, 0.3, 0),     # G = 8 at d = 64
])
def test_small_every_step(S, Sq, Hq, Hkv, d, a, s, w, steps, p, c):
    import torch
    theta = 500000.0
    g = torch.Generator().manual_seed(Sq * 1000 + w + c)
    cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, theta, c=c)
    sims = [C.SepCacheSim(a, s, w, c if c > 0 else None) for _ in range(Sq)]
    K, V = [], []
    for t in range(steps):
        kn = torch.randn(Sq, Hkv, d, generator=g).to(torch.bfloat16)
        vn = torch.randn(Sq, Hkv, d, generator=g).to(torch.bfloat16)
        qn = torch.randn(Sq, Hq, d, generator=g).to(torch.bfloat16)
        sn = (torch.rand(Sq, generator=g) < p).to(torch.uint8)
        K.append(f64(kn))
        V.append(f64(vn))
        cache.sepcache_update(kn.cuda(), vn.cuda(), sn.cuda())
        lse = torch.empty(Sq, Hq, dtype=torch.float32, device="cuda")
        o = cache.sepcache_decode(qn.cuda(), lse=lse)
        pos, cnt = cache.sepcache_export_order()
        pos, cnt = pos.cpu().numpy(), cnt.cpu().numpy()
        for sq in range(Sq):
            sims[sq].append(bool(sn[sq]))
            order = sims[sq].order()
            assert int(cnt[sq]) == len(order)
            assert pos[sq, : len(order)].tolist() == order, (t, sq)
            assert (pos[sq, len(order):] == -1).all()
            kr = np.stack([K[j][sq] for j in order])
            vr = np.stack([V[j][sq] for j in order])
            ro, rl = C.decode_attention(f64(qn[sq]), kr, vr, theta, d ** -0.5)
            check_out(f64(o[sq]), ro, f"step {t} seq {sq}")
            assert np.abs(f64(lse[sq]) - rl).max() < DECODE_LSE_ABS
    assert S.sep_last_device_error() == 0


def test_sepcache_decode_config_full(S):
    """64 sequences x 65536 steps, c = 800 = 4 + 64 + 732, theta = 5e5.

    Trajectory: all 64 sequences at steps 0..2047 and every 256th step after, bit-exact.
    Outputs: 4 sequences at steps 0..1023 and every 64th step to 2047; every 8th sequence at
    every 1024th step (the retained tokens' K/V regenerated from their chunk seeds).
    """
    import torch
    import workloads
    cfg = workloads.SEPCACHE_DECODE
    dev = "cuda"
    CH = 256
    cache = S.SepCache(cfg.S, cfg.Hq, cfg.Hkv, cfg.d, cfg.a, cfg.s, cfg.w, cfg.theta)
    sims = [C.SepCacheSim(cfg.a, cfg.s, cfg.w) for _ in range(cfg.S)]
    track = [0, 17, 40, 63]
    early_k, early_v = [], []   # host K/V of every sequence, steps < 2048

    def gather(pairs):
        """K/V (fp64) of (sequence, original position) pairs, regenerated chunk by chunk."""
        out = {}
        by_chunk = {}
        for sq, j in pairs:
            by_chunk.setdefault(j // CH, []).append((sq, j))
        for ci, lst in by_chunk.items():
            chk = workloads.decode_chunk(cfg, ci * CH, CH, device=dev)
            st = torch.tensor([j % CH for _, j in lst], device=dev)
            sq = torch.tensor([q for q, _ in lst], device=dev)
            kk = f64(chk["k"][st, sq])
            vv = f64(chk["v"][st, sq])
            for z, key in enumerate(lst):
                out[key] = (kk[z], vv[z])
        return out

    def check(t, o, q, seqs, kv):
        for sq in seqs:
            order = sims[sq].order()
            kr = np.stack([kv[(sq, j)][0] for j in order])
            vr = np.stack([kv[(sq, j)][1] for j in order])
            ro, _ = C.decode_attention(q[sq], kr, vr, cfg.theta, cfg.scale)
            check_out(f64(o[sq]), ro, f"step {t} seq {sq}")

    for t in range(cfg.steps):
        if t % CH == 0:
            chunk = workloads.decode_chunk(cfg, t, CH, device=dev)
            sep_host = chunk["sep"].cpu().numpy()
        lt = t % CH
        kn, vn, qn = chunk["k"][lt], chunk["v"][lt], chunk["q"][lt]
        cache.sepcache_update(kn, vn, chunk["sep"][lt])
        o = cache.sepcache_decode(qn)
        for sq in range(cfg.S):
            sims[sq].append(bool(sep_host[lt, sq]))
        if t < 2048:
            early_k.append(f64(kn))
            early_v.append(f64(vn))
        if t < 2048 or t % 256 == 0:
            pos, cnt = cache.sepcache_export_order()
            pos, cnt = pos.cpu().numpy(), cnt.cpu().numpy()
            for sq in range(cfg.S):
                assert pos[sq, : int(cnt[sq])].tolist() == sims[sq].order(), (t, sq)
        if t < 1024 or (t < 2048 and t % 64 == 0):
            kv = {(sq, j): (early_k[j][sq], early_v[j][sq])
                  for sq in track for j in sims[sq].order()}
            check(t, o, f64(qn), track, kv)
        if t % 1024 == 1023:
            seqs = list(range(0, cfg.S, 8))
            kv = gather([(sq, j) for sq in seqs for j in sims[sq].order()])
            check(t, o, f64(qn), seqs, kv)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0


def test_checkpoint_resume_bit_identical(S):
    """state_dict() after 300 steps, restored into a fresh cache, replays the next 100 steps
    with bit-identical decode outputs and trajectory."""
    import torch
    Sq, Hq, Hkv, d, a, s, w = 3, 8, 2, 128, 4, 16, 40
    g = torch.Generator().manual_seed(77)
    steps = [(torch.randn(Sq, Hkv, d, generator=g).to(torch.bfloat16),
              torch.randn(Sq, Hkv, d, generator=g).to(torch.bfloat16),
              torch.randn(Sq, Hq, d, generator=g).to(torch.bfloat16),
              (torch.rand(Sq, generator=g) < 0.2).to(torch.uint8)) for _ in range(400)]
    a_cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0)
    for kn, vn, qn, sn in steps[:300]:
        a_cache.sepcache_update(kn.cuda(), vn.cuda(), sn.cuda())
    ckpt = a_cache.state_dict()

    def run(cache):
        outs = []
        for kn, vn, qn, sn in steps[300:]:
            cache.sepcache_update(kn.cuda(), vn.cuda(), sn.cuda())
            lse = torch.empty(Sq, Hq, dtype=torch.float32, device="cuda")
            o = cache.sepcache_decode(qn.cuda(), lse=lse)
            outs.append((o.cpu(), lse.cpu()))
        return outs, cache.sepcache_export_order()

    ref_outs, ref_order = run(a_cache)
    b_cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0)
    b_cache.load_state_dict(ckpt)
    got_outs, got_order = run(b_cache)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    for (o1, l1), (o2, l2) in zip(ref_outs, got_outs):
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for x, y in zip(ref_order, got_order):
        assert torch.equal(x.cpu(), y.cpu())


@pytest.mark.parametrize("Sq,Hq,Hkv,d,a,s,w,L,p", [
    (2, 8, 2, 128, 4, 6, 20, 3, 0.3),        # prompt shorter than the initial block
    (2, 8, 2, 128, 4, 6, 20, 15, 0.3),       # window not yet full
    (3, 8, 2, 128, 4, 6, 20, 200, 0.3),      # window wrapped, separator FIFO overflowed
    (2, 4, 4, 64, 0, 3, 7, 100, 0.5),        # no initial block
    (2, 8, 1, 128, 2, 0, 9, 60, 0.3),        # s = 0: separators dropped
    (1, 16, 2, 64, 1, 2, 1, 40, 0.6),        # window of one slot
    (2, 32, 8, 128, 4, 64, 732, 3000, 0.1),  # the decode configuration's capacities
])
def test_prefill_equals_sequential_updates(S, Sq, Hq, Hkv, d, a, s, w, L, p):
    """sepcache_prefill leaves the state L sepcache_update calls leave (bit-identical), whose
    trajectory is the oracle's; a decode step after either gives identical outputs."""
    import torch
    g = torch.Generator().manual_seed(L * 7 + w)
    k = torch.randn(Sq, L, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(Sq, L, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    sep = (torch.rand(Sq, L, generator=g) < p).to(torch.uint8).cuda()
    seq_cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0)
    for t in range(L):
        seq_cache.sepcache_update(k[:, t].contiguous(), v[:, t].contiguous(), sep[:, t].contiguous())
    pre_cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0)
    pre_cache.sepcache_prefill(k, v, sep)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    for name in ("meta", "slot_pos", "slot_sep", "k_slots", "v_slots"):
        assert torch.equal(getattr(seq_cache, name), getattr(pre_cache, name)), name
    pos, cnt = pre_cache.sepcache_export_order()
    pos, cnt = pos.cpu().numpy(), cnt.cpu().numpy()
    flags = sep.cpu().numpy()
    for sq in range(Sq):
        sim = C.SepCacheSim(a, s, w)
        for t in range(L):
            sim.append(bool(flags[sq, t]))
        order = sim.order()
        assert int(cnt[sq]) == len(order)
        assert pos[sq, : len(order)].tolist() == list(order)
    q = torch.randn(Sq, Hq, d, generator=g).to(torch.bfloat16).cuda()
    kn = torch.randn(Sq, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    sn = torch.zeros(Sq, dtype=torch.uint8, device="cuda")
    outs = []
    for cache in (seq_cache, pre_cache):
        cache.sepcache_update(kn, kn, sn)
        outs.append(cache.sepcache_decode(q))
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("Sq,Hq,Hkv,d,a,s,w,steps,p", [
    (2, 8, 2, 128, 4, 300, 32, 300, 0.2),    # every separator retained, w = n
    (3, 4, 4, 64, 1, 4, 9, 150, 0.4),        # separator FIFO overflows
    (2, 32, 8, 128, 4, 64, 200, 400, 0.1),
])
def test_original_positions_every_step(S, Sq, Hq, Hkv, d, a, s, w, steps, p):
    """Without positional shifting: trajectory bit-exact and decode within the forward
    tolerances of the oracle (keys stored rotated at original positions in bf16)."""
    import torch
    theta = 500000.0
    g = torch.Generator().manual_seed(steps + s)
    cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, theta, original_positions=True)
    sims = [C.SepCacheSim(a, s, w) for _ in range(Sq)]
    Kst, V = [], []
    for t in range(steps):
        kn = torch.randn(Sq, Hkv, d, generator=g).to(torch.bfloat16)
        vn = torch.randn(Sq, Hkv, d, generator=g).to(torch.bfloat16)
        qn = torch.randn(Sq, Hq, d, generator=g).to(torch.bfloat16)
        sn = (torch.rand(Sq, generator=g) < p).to(torch.uint8)
        Kst.append(C.stored_rotated_key(f64(kn), t, theta))
        V.append(f64(vn))
        cache.sepcache_update(kn.cuda(), vn.cuda(), sn.cuda())
        lse = torch.empty(Sq, Hq, dtype=torch.float32, device="cuda")
        o = cache.sepcache_decode(qn.cuda(), lse=lse)
        if t % 7 and t < steps - 1:
            for sq in range(Sq):
                sims[sq].append(bool(sn[sq]))
            continue
        pos, cnt = cache.sepcache_export_order()
        pos, cnt = pos.cpu().numpy(), cnt.cpu().numpy()
        for sq in range(Sq):
            sims[sq].append(bool(sn[sq]))
            order = sims[sq].order()
            assert pos[sq, : int(cnt[sq])].tolist() == order, (t, sq)
            kr = np.stack([Kst[j][sq] for j in order])
            vr = np.stack([V[j][sq] for j in order])
            ro, rl = C.decode_attention_original_positions(f64(qn[sq]), kr, vr, t, theta, d ** -0.5)
            check_out(f64(o[sq]), ro, f"step {t} seq {sq}")
            assert np.abs(f64(lse[sq]) - rl).max() < 2e-3
    assert S.sep_last_device_error() == 0


def test_original_positions_prefill_equals_updates(S):
    import torch
    Sq, Hq, Hkv, d, a, s, w, L = 2, 8, 2, 128, 4, 64, 40, 500
    g = torch.Generator().manual_seed(9)
    k = torch.randn(Sq, L, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(Sq, L, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    sep = (torch.rand(Sq, L, generator=g) < 0.15).to(torch.uint8).cuda()
    seq_cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0, original_positions=True)
    for t in range(L):
        seq_cache.sepcache_update(k[:, t].contiguous(), v[:, t].contiguous(), sep[:, t].contiguous())
    pre_cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0, original_positions=True)
    pre_cache.sepcache_prefill(k, v, sep)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    for name in ("meta", "slot_pos", "slot_sep", "k_slots", "v_slots"):
        assert torch.equal(getattr(seq_cache, name), getattr(pre_cache, name)), name


@pytest.mark.parametrize("Sq,Hq,Hkv,d,a,s,w,c,L,p", [
    (2, 8, 2, 128, 4, 6, 20, 45, 15, 0.3),       # window not yet full
    (2, 8, 2, 128, 4, 6, 20, 45, 40, 0.3),       # past window filling, no compression yet
    (3, 8, 2, 128, 4, 6, 20, 45, 400, 0.3),      # many compressions, FIFO overflowed
    (2, 4, 4, 64, 0, 3, 7, 14, 150, 0.5),        # no initial block
    (2, 8, 1, 128, 2, 0, 9, 20, 120, 0.3),       # s = 0: every compression drops the past
    (1, 16, 2, 64, 1, 2, 1, 7, 60, 0.6),         # window of one slot
    (2, 32, 8, 128, 4, 64, 256, 800, 3000, 0.1), # the Past Window configuration of the bench
])
def test_prefill_past_window_equals_sequential_updates(S, Sq, Hq, Hkv, d, a, s, w, c, L, p):
    """With a Past Window (c > 0), sepcache_prefill leaves the metadata, slot maps and occupied
    K/V rows that L sepcache_update calls leave (bit-identical), its trajectory is the oracle's,
    and the next update + decode step gives identical outputs. (Slots emptied by a compression
    keep stale rows after single-token updates, so only occupied rows are compared.)"""
    import torch
    g = torch.Generator().manual_seed(L * 11 + w + c)
    k = torch.randn(Sq, L, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(Sq, L, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    sep = (torch.rand(Sq, L, generator=g) < p).to(torch.uint8).cuda()
    seq_cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0, c=c)
    for t in range(L):
        seq_cache.sepcache_update(k[:, t].contiguous(), v[:, t].contiguous(), sep[:, t].contiguous())
    pre_cache = S.SepCache(Sq, Hq, Hkv, d, a, s, w, 500000.0, c=c)
    pre_cache.sepcache_prefill(k, v, sep)
    torch.cuda.synchronize()
    assert S.sep_last_device_error() == 0
    for name in ("meta", "slot_pos", "slot_sep"):
        assert torch.equal(getattr(seq_cache, name), getattr(pre_cache, name)), name
    occupied = (pre_cache.slot_pos >= 0).cpu()
    for name in ("k_slots", "v_slots"):
        x, y = getattr(seq_cache, name).cpu(), getattr(pre_cache, name).cpu()
        for sq in range(Sq):
            rows = occupied[sq].nonzero()[:, 0]
            assert torch.equal(x[sq][:, rows], y[sq][:, rows]), (name, sq)
    pos, cnt = pre_cache.sepcache_export_order()
    pos, cnt = pos.cpu().numpy(), cnt.cpu().numpy()
    flags = sep.cpu().numpy()
    for sq in range(Sq):
        sim = C.SepCacheSim(a, s, w, c)
        for t in range(L):
            sim.append(bool(flags[sq, t]))
        order = sim.order()
        assert int(cnt[sq]) == len(order)
        assert pos[sq, : len(order)].tolist() == list(order)
    q = torch.randn(Sq, Hq, d, generator=g).to(torch.bfloat16).cuda()
    kn = torch.randn(Sq, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    sn = torch.ones(Sq, dtype=torch.uint8, device="cuda")
    outs = []
    for cache in (seq_cache, pre_cache):
        cache.sepcache_update(kn, kn, sn)
        outs.append(cache.sepcache_decode(q))
    assert torch.equal(outs[0], outs[1])
