"""H2O chunked sparse attention for B200 (sm_100a).

A thin Python layer over libh2o.so (see include/h2o.h).  PyTorch supplies device
memory and streams; every step of the chunk -- attention with summed weights,
score accumulation, selection and scatter -- runs in the library's kernels.

    cache = H2OCache(M=2048, R=256, Hq=32, Hkv=8, d=128, dtype=torch.bfloat16)
    out = cache.prefill(q, k, v)          # q [B,Hq,P,d], k/v [B,Hkv,P,d]
    out = cache.step(q, k, v)             # one chunk of S tokens
    slots, scores, positions = cache.read_state()
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (H2O_BF16, H2O_F32, H2O_OK, STATUS_NAMES, lib)

__all__ = ["H2OCache", "H2OError", "select", "attend_noalloc", "step_layers", "lib"]

_DTYPES = {torch.float32: H2O_F32, torch.bfloat16: H2O_BF16}
# eviction policies: heavy hitters (h2o) or recency only (lr); see include/h2o.h
_POLICIES = {"h2o": _lib.H2O_POLICY_H2O, "lr": _lib.H2O_POLICY_LR}


class H2OError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _check(rc: int, handle=None):
    if rc != H2O_OK:
        raise H2OError(rc, lib.h2o_last_error(handle).decode())
    return rc


def _stream_ptr(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


class H2OCache:
    """One layer's H2O caches for B sequences (batch fixed at prefill)."""

    def __init__(self, M: int, R: int, Hq: int, Hkv: int, d: int, dtype=torch.bfloat16,
                 device=None, policy: str = "h2o"):
        if dtype not in _DTYPES:
            raise ValueError("dtype must be torch.float32 or torch.bfloat16")
        if policy not in _POLICIES:
            raise ValueError(f"policy must be one of {sorted(_POLICIES)}")
        self.M, self.R, self.Hq, self.Hkv, self.d, self.dtype = M, R, Hq, Hkv, d, dtype
        self.policy = policy
        self.device = torch.device(device if device is not None else "cuda", )
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        h = ctypes.c_void_p()
        _check(lib.h2o_create_policy(M, R, Hq, Hkv, d, _DTYPES[dtype], _POLICIES[policy],
                                     ctypes.byref(h)))
        self._h = h
        self.B = None
        self.last_S = None

    # -- helpers -------------------------------------------------------------
    def _chk(self, rc):
        return _check(rc, self._h)

    def _args(self, q, k, v, S):
        for name, t, H in (("q", q, self.Hq), ("k", k, self.Hkv), ("v", v, self.Hkv)):
            if t.dtype != self.dtype or not t.is_contiguous() or t.dim() != 4:
                raise ValueError(f"{name} must be a contiguous 4-d {self.dtype} tensor")
            if t.shape[1] != H or t.shape[3] != self.d or t.shape[2] != S:
                raise ValueError(f"{name} has shape {tuple(t.shape)}")
        if k.shape != v.shape or k.shape[0] != q.shape[0]:
            raise ValueError("q, k, v batch / shape mismatch")

    def _out(self, q, out):
        if out is None:
            out = torch.empty_like(q)
        elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
            raise ValueError("out must be contiguous, same shape and dtype as q")
        return out

    # -- API -----------------------------------------------------------------
    def prefill(self, q, k, v, out=None, stream=None, want_out=True):
        B, P = q.shape[0], q.shape[2]
        self._args(q, k, v, P)
        out = self._out(q, out) if want_out else None
        with torch.cuda.device(self.device):
            self._chk(lib.h2o_prefill(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, P,
                                      _stream_ptr(stream, self.device)))
        self.B, self.last_S = B, P
        return out

    def step(self, q, k, v, out=None, stream=None):
        S = q.shape[2]
        self._args(q, k, v, S)
        out = self._out(q, out)
        with torch.cuda.device(self.device):
            self._chk(lib.h2o_step(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), S,
                                   _stream_ptr(stream, self.device)))
        self.last_S = S
        return out

    def read_state(self, stream=None):
        """(slots [B,Hkv,S_last] int32, scores [B,Hkv,M] f32, positions [B,Hkv,M] int32)."""
        dev = self.device
        slots = torch.empty(self.B, self.Hkv, self.last_S, dtype=torch.int32, device=dev)
        scores = torch.empty(self.B, self.Hkv, self.M, dtype=torch.float32, device=dev)
        pos = torch.empty(self.B, self.Hkv, self.M, dtype=torch.int32, device=dev)
        with torch.cuda.device(dev):
            self._chk(lib.h2o_read_state(self._h, _ptr(slots), _ptr(scores), _ptr(pos),
                                         _stream_ptr(stream, dev)))
        return slots, scores, pos

    def read_delta(self, stream=None):
        """The last step's buffer delta: (slots [B,Hkv,S_last] int32, the slots filled in
        chunk order; evicted_positions [B,Hkv,S_last] int32, what each held before, -1 if
        it was empty).  Chunk token i's K/V went to slots[..., i]."""
        dev = self.device
        slots = torch.empty(self.B, self.Hkv, self.last_S, dtype=torch.int32, device=dev)
        evicted = torch.empty(self.B, self.Hkv, self.last_S, dtype=torch.int32, device=dev)
        with torch.cuda.device(dev):
            self._chk(lib.h2o_read_delta(self._h, _ptr(slots), _ptr(evicted), _stream_ptr(stream, dev)))
        return slots, evicted

    def read_kv(self, stream=None):
        shape = (self.B, self.Hkv, self.M, self.d)
        kc = torch.empty(shape, dtype=self.dtype, device=self.device)
        vc = torch.empty(shape, dtype=self.dtype, device=self.device)
        with torch.cuda.device(self.device):
            self._chk(lib.h2o_read_kv(self._h, _ptr(kc), _ptr(vc), _stream_ptr(stream, self.device)))
        return kc, vc

    def info(self):
        arr = (ctypes.c_int64 * 5)()
        self._chk(lib.h2o_info(self._h, arr))
        return {"B": arr[0], "t0": arr[1], "n_valid": arr[2], "last_S": arr[3], "launches": arr[4]}

    def set_profiling(self, on: bool, restart: bool = True):
        """Per-kernel CUDA events on (restarting or continuing the count of
        profiled steps) or off."""
        self._chk(lib.h2o_set_profiling(self._h, (1 if restart else 2) if on else 0))

    def last_timings(self, age: int = 0):
        """ms of [attention, tail (score accumulate + select + scatter)] of the
        profiled step `age` steps before the last (0 = the last; up to 63)."""
        arr = (ctypes.c_float * 2)()
        n = lib.h2o_step_timings(self._h, age, arr, 2)
        if n < 0:
            self._chk(n)
        return list(arr)[:n]

    def close(self):
        if getattr(self, "_h", None):
            lib.h2o_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def step_layers(caches, qs, ks, vs, outs=None, stream=None):
    """One chunk through several layers' caches (h2o_step_layers): the same result
    as caches[l].step(qs[l], ks[l], vs[l], outs[l]) for every l, with one
    attention launch and one tail launch for all layers when they share their
    sizes.  Returns the list of outputs."""
    n = len(caches)
    if n < 1 or not (len(qs) == len(ks) == len(vs) == n):
        raise ValueError("need one (q, k, v) per cache")
    S = qs[0].shape[2]
    if outs is None:
        outs = [None] * n
    outs = list(outs)
    for l, c in enumerate(caches):
        c._args(qs[l], ks[l], vs[l], S)
        outs[l] = c._out(qs[l], outs[l])
    dev = caches[0].device
    if any(c.device != dev for c in caches):
        raise ValueError("all caches must be on one device")
    arr = lambda xs: (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])   # noqa: E731
    hs = (ctypes.c_void_p * n)(*[c._h.value for c in caches])
    with torch.cuda.device(dev):
        _check(lib.h2o_step_layers(hs, n, arr(qs), arr(ks), arr(vs), arr(outs), S,
                                   _stream_ptr(stream, dev)), caches[0]._h)
    for c in caches:
        c.last_S = S
    return outs


def select(scores, positions, t0: int, R: int, need: int, stream=None):
    """Standalone selection: scores [n, M] f32, positions [n, M] int32 (device) ->
    evicted [n, need] int32, ascending slots of the `need` smallest (score, pos)
    among slots with 0 <= pos < t0 - R."""
    n, M = scores.shape
    if scores.dtype != torch.float32 or positions.dtype != torch.int32:
        raise ValueError("scores must be float32 and positions int32")
    if not scores.is_cuda or not positions.is_cuda:
        raise ValueError("scores and positions must be CUDA tensors")
    sc, ps = scores.contiguous(), positions.contiguous()     # kept alive across the call
    ev = torch.empty(n, need, dtype=torch.int32, device=scores.device)
    with torch.cuda.device(scores.device):
        _check(lib.h2o_select(_ptr(sc), _ptr(ps), n, M, t0, R, need, _ptr(ev),
                              _stream_ptr(stream, scores.device)))
    return ev


def attend_noalloc(q, k, v, k_cache, v_cache, n_valid: int, M: int, out=None, colsum=None,
                   stream=None):
    """Attention with summed weights through h2o_attend_noalloc, which allocates
    no device memory itself (for callers that cannot call cudaMalloc).  Every
    buffer comes from the caller: q [B,Hq,S,d], k/v [B,Hkv,S,d], k_cache/v_cache
    [B,Hkv,M,d] (None when n_valid == 0), out [B,Hq,S,d], colsum [B,Hkv,M+S] f32.
    Returns (out, colsum).

    The library reads and writes these buffers through raw pointers and cannot
    check their sizes, so every shape, dtype, layout and device is checked here
    first (ValueError), before any pointer crosses the C ABI."""
    if not isinstance(q, torch.Tensor) or q.dtype not in _DTYPES:
        raise ValueError("q must be a float32 or bfloat16 tensor")
    if q.dim() != 4:
        raise ValueError(f"q must be 4-d [B, Hq, S, d], got shape {tuple(q.shape)}")
    B, Hq, S, d = q.shape
    dev = q.device

    def _need(name, t, shape, dtype):
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{name} must be a tensor")
        if t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
        if t.device != dev:
            raise ValueError(f"{name} must be on {dev}, got {t.device}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")

    _need("q", q, (B, Hq, S, d), q.dtype)
    if k.dim() != 4:
        raise ValueError(f"k must be 4-d [B, Hkv, S, d], got shape {tuple(k.shape)}")
    Hkv = k.shape[1]
    if Hkv < 1 or Hq % Hkv != 0:
        raise ValueError(f"Hq={Hq} must be a multiple of Hkv={Hkv}")
    _need("k", k, (B, Hkv, S, d), q.dtype)
    _need("v", v, (B, Hkv, S, d), q.dtype)
    n_valid, M = int(n_valid), int(M)
    if M < 1 or not 0 <= n_valid <= M:
        raise ValueError(f"need M >= 1 and 0 <= n_valid <= M (n_valid={n_valid}, M={M})")
    if n_valid > 0:
        if k_cache is None or v_cache is None:
            raise ValueError("k_cache and v_cache are required when n_valid > 0")
        _need("k_cache", k_cache, (B, Hkv, M, d), q.dtype)
        _need("v_cache", v_cache, (B, Hkv, M, d), q.dtype)
    else:
        for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
            if t is not None:
                _need(name, t, (B, Hkv, M, d), q.dtype)
    if out is None:
        out = torch.empty_like(q)
    else:
        _need("out", out, (B, Hq, S, d), q.dtype)
    if colsum is None:
        colsum = torch.empty(B, Hkv, M + S, dtype=torch.float32, device=dev)
    else:
        _need("colsum", colsum, (B, Hkv, M + S), torch.float32)
    if not q.is_cuda:
        raise ValueError("every buffer must be a CUDA tensor")
    with torch.cuda.device(dev):
        _check(lib.h2o_attend_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                      B, Hq, Hkv, d, _DTYPES[q.dtype], M, n_valid, S, _ptr(out),
                                      _ptr(colsum), _stream_ptr(stream, dev)))
    return out, colsum
