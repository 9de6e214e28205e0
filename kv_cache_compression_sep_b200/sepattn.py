"""Thin ctypes binding of libsepattn.so: same names as the C ABI, argument marshalling only.

Every computation runs in the library's CUDA kernels; this module allocates outputs and scratch
with torch (device memory), passes raw pointers and the current CUDA stream, and turns status
codes into exceptions. There is no CPU path: importing this module without the built library
raises.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsepattn.so")

SEP_OK = 0
TILE = 128
META = 8


class SepError(RuntimeError):
    pass


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python -m kv_cache_compression_sep_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "sep_mask_build": (I, [P, I, I, I, I, I, I, P, P, P, P, P, P, P]),
        "sep_attn_fwd_workspace_size": (Z, [I, I, I, I]),
        "sep_attn_fwd": (I, [P, P, P, I, I, I, I, I, F, I, I, P, P, P, P, Z, P]),
        "sep_attn_fwd_stage": (I, [I, P, P, P, I, I, I, I, I, F, I, I, P, P, P, P, Z, P]),
        "sep_attn_fwd_noalloc": (I, [P, P, P, I, I, I, I, I, F, I, I, P, P, P, P]),
        "sep_attn_bwd_workspace_size": (Z, [I, I, I, I, I]),
        "sep_attn_bwd_stage": (I, [I, P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, P, P, P, P, Z, P]),
        "sep_attn_bwd": (I, [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, P, P, P, P, Z, P]),
        "sepcache_state_init": (I, [P, P]),
        "sepcache_update": (I, [P, P, P, P, P]),
        "sepcache_decode": (I, [P, P, P, P, F, P]),
        "sepcache_prefill": (I, [P, P, P, P, I, P]),
        "sepcache_export_order": (I, [P, P, P, P]),
        "sep_last_device_error": (I, []),
        "sep_set_wait_limit_ns": (I, [ctypes.c_ulonglong]),
        "sep_status_string": (ctypes.c_char_p, [I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


class _SepMask(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("L", ctypes.c_int), ("a", ctypes.c_int), ("n", ctypes.c_int),
                ("sep", ctypes.c_void_p), ("anchor_idx", ctypes.c_void_p),
                ("anchor_cnt", ctypes.c_void_p), ("anchor_bits", ctypes.c_void_p),
                ("gather_end", ctypes.c_void_p),
                ("tile_map", ctypes.c_void_p)]


class _SepCacheState(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("a", ctypes.c_int32), ("s", ctypes.c_int32),
                ("w", ctypes.c_int32), ("c", ctypes.c_int32),
                ("original_positions", ctypes.c_int32), ("rope_theta", ctypes.c_float),
                ("k_slots", ctypes.c_void_p), ("v_slots", ctypes.c_void_p),
                ("slot_pos", ctypes.c_void_p), ("slot_sep", ctypes.c_void_p),
                ("meta", ctypes.c_void_p), ("rope_freq", ctypes.c_void_p)]


def _check(status: int, what: str):
    if status != SEP_OK:
        raise SepError(f"{what}: {_lib.sep_status_string(status).decode()} ({status})")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _cuda(t, dtype, name, shape=None):
    """t must be a contiguous CUDA tensor of this dtype and, if given, this shape. The checks
    run before any launch: a buffer of the wrong size would be read or written out of bounds
    by the kernels, which trust the sizes passed to the library."""
    if not isinstance(t, torch.Tensor):
        raise SepError(f"{name} must be a torch.Tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise SepError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise SepError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise SepError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise SepError(f"{name} must be on a CUDA device (there is no CPU path)")


def _current_device_index():
    return torch.cuda.current_device()


def _same_device(dev, *named):
    """Every tensor of a call on one device, and that device the current one: the library
    launches on the current device and builds its copy descriptors over these pointers, so a
    tensor of another GPU would be read as if it were local."""
    for name, t in named:
        if t is not None and t.device != dev:
            raise SepError(f"{name} is on {t.device}, the call's other tensors on {dev}")
    cur = _current_device_index()
    if dev.index is not None and dev.index != cur:
        raise SepError(f"the call's tensors are on {dev} but the current CUDA device is "
                       f"cuda:{cur}; make {dev} current (torch.cuda.device) for this call")


def _mask_tensors(mask):
    return [("mask." + f, getattr(mask, f)) for f in
            ("sep", "anchor_idx", "anchor_cnt", "anchor_bits", "gather_end", "tile_map")]


def _dims(t, ndim, name):
    if not isinstance(t, torch.Tensor) or t.dim() != ndim:
        raise SepError(f"{name} must be a {ndim}-D tensor")
    return tuple(t.shape)


def sep_last_device_error() -> int:
    return int(_lib.sep_last_device_error())


def sep_set_wait_limit_ns(ns: int) -> None:
    """Test hook: limit of each pipeline wait of later forward launches (0 = default 1.5 s)."""
    _check(_lib.sep_set_wait_limit_ns(int(ns)), "sep_set_wait_limit_ns")


@dataclasses.dataclass
class SepMask:
    """Outputs of sep_mask_build (device tensors) plus the flags and parameters used."""
    sep: torch.Tensor
    anchor_idx: torch.Tensor
    anchor_cnt: torch.Tensor
    anchor_bits: torch.Tensor
    gather_end: torch.Tensor
    tile_map: torch.Tensor
    kept: torch.Tensor
    a: int
    n: int

    def _c(self):
        B, L = self.sep.shape
        return _SepMask(B, L, self.a, self.n, self.sep.data_ptr(), self.anchor_idx.data_ptr(),
                        self.anchor_cnt.data_ptr(), self.anchor_bits.data_ptr(),
                        self.gather_end.data_ptr(), self.tile_map.data_ptr())


def sep_mask_build(sep: torch.Tensor, a: int, n: int, bm: int = TILE, bn: int = TILE,
                   out: SepMask | None = None) -> SepMask:
    """Mask artefacts of `sep` [B, L] uint8; `out` reuses the buffers of an earlier result."""
    B, L = _dims(sep, 2, "sep")
    _cuda(sep, torch.uint8, "sep")
    T, U = -(-L // max(bm, 1)), -(-L // max(bn, 1))
    dev = sep.device
    if out is not None:
        for name, dtype, shape in (("anchor_idx", torch.int32, (B, L)),
                                   ("anchor_cnt", torch.int32, (B,)),
                                   ("anchor_bits", torch.int32, (B, -(-L // 32))),
                                   ("gather_end", torch.int32, (B, T)),
                                   ("tile_map", torch.int8, (B, T, U)),
                                   ("kept", torch.int64, (B,))):
            _cuda(getattr(out, name), dtype, f"out.{name}", shape)
        out.sep, out.a, out.n = sep, a, n
    else:
        out = SepMask(sep=sep,
                      anchor_idx=torch.empty(B, L, dtype=torch.int32, device=dev),
                      anchor_cnt=torch.empty(B, dtype=torch.int32, device=dev),
                      anchor_bits=torch.empty(B, -(-L // 32), dtype=torch.int32, device=dev),
                      gather_end=torch.empty(B, T, dtype=torch.int32, device=dev),
                      tile_map=torch.empty(B, T, U, dtype=torch.int8, device=dev),
                      kept=torch.empty(B, dtype=torch.int64, device=dev), a=a, n=n)
    _same_device(dev, *_mask_tensors(out), ("out.kept", out.kept))
    _check(_lib.sep_mask_build(_ptr(sep), B, L, a, n, bm, bn, _ptr(out.anchor_idx),
                               _ptr(out.anchor_cnt), _ptr(out.anchor_bits), _ptr(out.gather_end),
                               _ptr(out.tile_map), _ptr(out.kept), _stream()), "sep_mask_build")
    return out


def sep_attn_fwd_workspace_size(B, L, Hkv, d) -> int:
    return int(_lib.sep_attn_fwd_workspace_size(B, L, Hkv, d))


def sep_attn_bwd_workspace_size(B, L, Hq, Hkv, d) -> int:
    return int(_lib.sep_attn_bwd_workspace_size(B, L, Hq, Hkv, d))


def _attn_inputs(q, k, v, mask):
    """Shapes of q [B, L, Hq, d] and k, v [B, L, Hkv, d], checked against each other and the
    mask's flags [B, L]."""
    B, L, Hq, d = _dims(q, 4, "q")
    Hkv = _dims(k, 4, "k")[2]
    if tuple(mask.sep.shape) != (B, L):
        raise SepError(f"mask was built for flags of shape {tuple(mask.sep.shape)}, "
                       f"q needs {(B, L)}")
    if Hkv < 1 or Hq % Hkv != 0:
        raise SepError(f"Hq = {Hq} is not a multiple of Hkv = {Hkv}")
    _cuda(k, torch.bfloat16, "k", (B, L, Hkv, d))
    _cuda(v, torch.bfloat16, "v", (B, L, Hkv, d))
    _cuda(q, torch.bfloat16, "q")
    return B, L, Hq, Hkv, d


def _workspace(nbytes, device, ws):
    if ws is not None:
        _cuda(ws, torch.uint8, "workspace")
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    return ws


def sep_attn_fwd(q, k, v, mask: SepMask, scale=None, out=None, lse=None, workspace=None,
                 stage=None):
    """O, LSE of separator-sparse attention. q [B,L,Hq,d], k/v [B,L,Hkv,d] bf16 CUDA.

    stage=None runs the whole call; stage=0/1 runs sep_attn_fwd_stage (timing one pass).
    """
    B, L, Hq, Hkv, d = _attn_inputs(q, k, v, mask)
    scale = d ** -0.5 if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=q.device) if lse is None else lse
    _cuda(o, torch.bfloat16, "out", (B, L, Hq, d))
    _cuda(lse, torch.float32, "lse", (B, Hq, L))
    nbytes = sep_attn_fwd_workspace_size(B, L, Hkv, d)
    ws = _workspace(nbytes, q.device, workspace)
    _same_device(q.device, ("k", k), ("v", v), ("out", o), ("lse", lse), ("workspace", ws),
                 *_mask_tensors(mask))
    mc = mask._c()
    args = (_ptr(q), _ptr(k), _ptr(v), B, L, Hq, Hkv, d, float(scale), mask.a, mask.n,
            ctypes.byref(mc), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream())
    if stage is None:
        _check(_lib.sep_attn_fwd(*args), "sep_attn_fwd")
    else:
        _check(_lib.sep_attn_fwd_stage(int(stage), *args), "sep_attn_fwd_stage")
    return o, lse


def sep_attn_fwd_noalloc(q, k, v, mask: SepMask, scale=None, out=None, lse=None):
    """sep_attn_fwd through the library's fixed device scratch instead of a workspace.

    The library allocates nothing for this call; the outputs are allocated here unless given.
    Problems whose compacted anchors exceed SEP_NOALLOC_SCRATCH_BYTES raise SepError
    (SEP_ERR_SCRATCH_LIMIT). Calls that may overlap in time share the scratch and race.
    """
    B, L, Hq, Hkv, d = _attn_inputs(q, k, v, mask)
    scale = d ** -0.5 if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=q.device) if lse is None else lse
    _cuda(o, torch.bfloat16, "out", (B, L, Hq, d))
    _cuda(lse, torch.float32, "lse", (B, Hq, L))
    _same_device(q.device, ("k", k), ("v", v), ("out", o), ("lse", lse), *_mask_tensors(mask))
    mc = mask._c()
    _check(_lib.sep_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), B, L, Hq, Hkv, d, float(scale),
                                     mask.a, mask.n, ctypes.byref(mc), _ptr(o), _ptr(lse),
                                     _stream()), "sep_attn_fwd_noalloc")
    return o, lse


def sep_attn_bwd(q, k, v, o, lse, dout, mask: SepMask, scale=None, workspace=None, grads=None,
                 stage=None):
    """dQ, dK, dV of sum(O * dout) for sep_attn_fwd.

    stage=None runs the whole call; stage=0/1/2 runs sep_attn_bwd_stage (timing one pass).
    """
    B, L, Hq, Hkv, d = _attn_inputs(q, k, v, mask)
    _cuda(o, torch.bfloat16, "o", (B, L, Hq, d))
    _cuda(dout, torch.bfloat16, "dout", (B, L, Hq, d))
    _cuda(lse, torch.float32, "lse", (B, Hq, L))
    scale = d ** -0.5 if scale is None else scale
    if grads is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    else:
        dq, dk, dv = grads
    _cuda(dq, torch.bfloat16, "dq", (B, L, Hq, d))
    _cuda(dk, torch.bfloat16, "dk", (B, L, Hkv, d))
    _cuda(dv, torch.bfloat16, "dv", (B, L, Hkv, d))
    nbytes = sep_attn_bwd_workspace_size(B, L, Hq, Hkv, d)
    ws = _workspace(nbytes, q.device, workspace)
    _same_device(q.device, ("k", k), ("v", v), ("o", o), ("lse", lse), ("dout", dout),
                 ("dq", dq), ("dk", dk), ("dv", dv), ("workspace", ws), *_mask_tensors(mask))
    mc = mask._c()
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), B, L, Hq, Hkv, d,
            float(scale), mask.a, mask.n, ctypes.byref(mc), _ptr(dq), _ptr(dk), _ptr(dv),
            _ptr(ws), ws.numel(), _stream())
    if stage is None:
        _check(_lib.sep_attn_bwd(*args), "sep_attn_bwd")
    else:
        _check(_lib.sep_attn_bwd_stage(int(stage), *args), "sep_attn_bwd_stage")
    return dq, dk, dv


class SepCache:
    """SepCache state for S sequences, held in torch-allocated device memory.

    Capacities: a initial slots, s separator slots, w window slots; c = 0 compresses one token
    at a time, c > a + s + w adds a Past Window that is compressed when the usage reaches c.
    Slots per sequence: n = a + s + w, plus c - a - w past-window slots when c > 0.
    original_positions=True: no positional shifting (keys stored rotated at their original
    positions, the query rotated at its own position).
    Methods map one-to-one to sepcache_update / sepcache_decode / sepcache_export_order.
    """

    def __init__(self, S, Hq, Hkv, d, a, s, w, rope_theta, device="cuda", c=0,
                 original_positions=False):
        self.S, self.Hq, self.Hkv, self.d, self.a, self.s, self.w = S, Hq, Hkv, d, a, s, w
        self.c = int(c)
        self.past = c - a - w if c > 0 else 0
        self.n = a + s + self.past + w
        self.rope_theta = float(rope_theta)
        dev = torch.device(device)
        if dev.type != "cuda":
            raise SepError(f"SepCache state must live on a CUDA device, not {dev} "
                           "(there is no CPU path)")
        self.k_slots = torch.zeros(S, Hkv, self.n, d, dtype=torch.bfloat16, device=dev)
        self.v_slots = torch.zeros(S, Hkv, self.n, d, dtype=torch.bfloat16, device=dev)
        self.slot_pos = torch.empty(S, self.n, dtype=torch.int32, device=dev)
        self.slot_sep = torch.empty(S, self.n, dtype=torch.uint8, device=dev)
        self.meta = torch.empty(S, META, dtype=torch.int32, device=dev)
        self.rope_freq = torch.empty(d // 2, dtype=torch.float64, device=dev)
        self.original_positions = bool(original_positions)
        self._st = _SepCacheState(S, Hq, Hkv, d, a, s, w, self.c, int(self.original_positions),
                                  self.rope_theta,
                                  self.k_slots.data_ptr(), self.v_slots.data_ptr(),
                                  self.slot_pos.data_ptr(), self.slot_sep.data_ptr(),
                                  self.meta.data_ptr(), self.rope_freq.data_ptr())
        self._on_device()
        _check(_lib.sepcache_state_init(ctypes.byref(self._st), _stream()), "sepcache_state_init")

    def _on_device(self, *named):
        _same_device(self.k_slots.device, ("v_slots", self.v_slots), ("slot_pos", self.slot_pos),
                     ("slot_sep", self.slot_sep), ("meta", self.meta),
                     ("rope_freq", self.rope_freq), *named)

    def sepcache_prefill(self, k, v, sep):
        """Seeds every sequence with a prompt: k, v [S, L, Hkv, d] bf16, sep [S, L] uint8."""
        L = _dims(k, 4, "k")[1]
        _cuda(k, torch.bfloat16, "k", (self.S, L, self.Hkv, self.d))
        _cuda(v, torch.bfloat16, "v", (self.S, L, self.Hkv, self.d))
        _cuda(sep, torch.uint8, "sep", (self.S, L))
        self._on_device(("k", k), ("v", v), ("sep", sep))
        _check(_lib.sepcache_prefill(ctypes.byref(self._st), _ptr(k), _ptr(v), _ptr(sep), L,
                                     _stream()), "sepcache_prefill")

    # checkpoint / resume: the whole state lives in these tensors (the RoPE frequency table is a
    # pure function of d and theta and is rebuilt by the constructor)
    _STATE = ("k_slots", "v_slots", "slot_pos", "slot_sep", "meta")

    def state_dict(self):
        """Host copies of every state tensor (stream-ordered after earlier calls)."""
        return {k: getattr(self, k).to("cpu", copy=True) for k in self._STATE}

    def load_state_dict(self, sd):
        """Restores a state_dict() taken from a cache of the same shape."""
        for k in self._STATE:
            dst = getattr(self, k)
            if tuple(sd[k].shape) != tuple(dst.shape) or sd[k].dtype != dst.dtype:
                raise SepError(f"load_state_dict: {k} has shape {tuple(sd[k].shape)}, "
                               f"expected {tuple(dst.shape)}")
            dst.copy_(sd[k])

    def sepcache_update(self, k_new, v_new, sep_new):
        _cuda(k_new, torch.bfloat16, "k_new", (self.S, self.Hkv, self.d))
        _cuda(v_new, torch.bfloat16, "v_new", (self.S, self.Hkv, self.d))
        _cuda(sep_new, torch.uint8, "sep_new", (self.S,))
        self._on_device(("k_new", k_new), ("v_new", v_new), ("sep_new", sep_new))
        _check(_lib.sepcache_update(ctypes.byref(self._st), _ptr(k_new), _ptr(v_new),
                                    _ptr(sep_new), _stream()), "sepcache_update")

    def sepcache_decode(self, q, scale=None, out=None, lse=None):
        _cuda(q, torch.bfloat16, "q", (self.S, self.Hq, self.d))
        scale = self.d ** -0.5 if scale is None else scale
        o = torch.empty_like(q) if out is None else out
        _cuda(o, torch.bfloat16, "out", (self.S, self.Hq, self.d))
        if lse is not None:
            _cuda(lse, torch.float32, "lse", (self.S, self.Hq))
        self._on_device(("q", q), ("out", o), ("lse", lse))
        _check(_lib.sepcache_decode(ctypes.byref(self._st), _ptr(q), _ptr(o), _ptr(lse),
                                    float(scale), _stream()), "sepcache_decode")
        return o

    def sepcache_export_order(self):
        pos = torch.empty(self.S, self.n, dtype=torch.int32, device=self.k_slots.device)
        cnt = torch.empty(self.S, dtype=torch.int32, device=self.k_slots.device)
        self._on_device()
        _check(_lib.sepcache_export_order(ctypes.byref(self._st), _ptr(pos), _ptr(cnt),
                                          _stream()), "sepcache_export_order")
        return pos, cnt
