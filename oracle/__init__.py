"""fp64 CPU oracle for the RAT+ sequence mixer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it and
shares no code with it.

The arithmetic lives in ``ratp_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only compiles it with gcc and marshals numpy arrays through
ctypes.  Each function cites the page passage it follows in the C source:

* ``scan``        -- the forget-gate recurrence of the zhichai.net write-up
                    "RAT+ 深度拆解", section 2.1 (sequential loop); with L,
                    the chunk-local variant of the original RAT.
* ``scan_window`` -- the fixed look-back recurrence of the same section
                    (window of the last L positions), O(T * L) loop.
* ``key_set``     -- dilated key set of the RAT+ abstract / section 1 of the
                    write-up, united with the optional local window.
* ``attention``   -- softmax attention over the enumerated key sets.
* ``attention_mask`` -- brute force over an explicit T x T mask.
* ``attention_per_sample`` -- one dilation per sample (the batch composition
                    of the write-up's section 2.2), sample by sample.
* ``cache_row`` / ``ring_row`` / ``cache_pack`` / ``decode_step`` -- the
                    D-compressed cache and one literal decode step.

All functions are pinned by CPU tests against closed forms, brute force and
a library routine (see ``tests/test_oracle.py``).  No function is marked
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ratp_oracle.c")
_LIB = os.path.join(_HERE, "libratp_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_L = ctypes.POINTER(ctypes.c_long)
_U8 = ctypes.POINTER(ctypes.c_ubyte)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP) into ``libratp_oracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.orc_scan.argtypes = [_D, _D, _D, ctypes.c_long, ctypes.c_long, ctypes.c_long]
        lib.orc_scan_reset.argtypes = [_D, _D, _D] + [ctypes.c_long] * 4
        lib.orc_scan_window.argtypes = [_D, _D, _D] + [ctypes.c_long] * 4
        lib.orc_scan_step.argtypes = [_D, _D, _D, ctypes.c_long]
        lib.orc_key_set.argtypes = [ctypes.c_long, ctypes.c_long, ctypes.c_long, _L]
        lib.orc_key_set.restype = ctypes.c_long
        lib.orc_attention.argtypes = [_D, _D, _D, _D] + [ctypes.c_long] * 6 + [_U8, _L, ctypes.c_long]
        lib.orc_attention_mask.argtypes = [_D, _D, _D, _D] + [ctypes.c_long] * 6 + [_U8]
        lib.orc_cache_row.argtypes = [ctypes.c_long] * 6 + [_U8]
        lib.orc_cache_row.restype = ctypes.c_long
        lib.orc_cache_rows_total.argtypes = [ctypes.c_long] * 4 + [_U8]
        lib.orc_cache_rows_total.restype = ctypes.c_long
        lib.orc_ring_row.argtypes = [ctypes.c_long] * 5
        lib.orc_ring_row.restype = ctypes.c_long
        lib.orc_cache_pack.argtypes = [_D, _D] + [ctypes.c_long] * 7 + [_U8, _D, _D, _D, _D, _L]
        lib.orc_decode_step.argtypes = [_D] * 9 + [_L, _D] + [ctypes.c_long] * 6 + [_U8, ctypes.c_long]
        lib.orc_decode_step.restype = ctypes.c_int
        lib.orc_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray, typ=_D):
    return a.ctypes.data_as(typ)


def _mask(dense_mask, H):
    if dense_mask is None:
        return None, None
    m = np.ascontiguousarray(np.asarray(dense_mask, dtype=np.uint8).reshape(-1))
    assert m.size == H
    return m, _p(m, _U8)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def scan(x, g, L: int = 0) -> np.ndarray:
    """h_t = g_t h_{t-1} + (1 - g_t) x_t along axis 1 of [B, T, ...] arrays.

    L > 0: chunk-local recurrence, the state restarts at every t with
    t mod L == 0 (the original RAT's blocks); L == 0: the full sequence.
    """
    x = _f64(x)
    g = _f64(g)
    assert x.shape == g.shape and x.ndim >= 2 and L >= 0
    B, T = x.shape[0], x.shape[1]
    C = int(np.prod(x.shape[2:])) if x.ndim > 2 else 1
    h = np.empty_like(x)
    if L == 0:
        _load().orc_scan(_p(x), _p(g), _p(h), B, T, C)
    else:
        _load().orc_scan_reset(_p(x), _p(g), _p(h), B, T, C, L)
    return h


def scan_window(x, g, L: int) -> np.ndarray:
    """Fixed look-back recurrence: h_t runs h = g h + (1 - g) x from zero over
    positions max(0, t - L + 1) .. t, along axis 1 of [B, T, ...] arrays."""
    x = _f64(x)
    g = _f64(g)
    assert x.shape == g.shape and x.ndim >= 2 and L >= 1
    B, T = x.shape[0], x.shape[1]
    C = int(np.prod(x.shape[2:])) if x.ndim > 2 else 1
    h = np.empty_like(x)
    _load().orc_scan_window(_p(x), _p(g), _p(h), B, T, C, L)
    return h


def key_set(t: int, D: int, W: int) -> list:
    """Sorted key positions of query t (dilation D, window W)."""
    out = np.zeros(t // max(D, 1) + W + 2, dtype=np.int64)
    n = _load().orc_key_set(t, D, W, _p(out, _L))
    return [int(v) for v in out[:n]]


def attention(q, hk, hv, D: int, W: int, dense_mask=None, rows=None) -> np.ndarray:
    """Dilated/windowed attention; q, hk, hv: [B, T, H, Dh].

    rows: optional int array [n, 3] of (b, t, h); then returns [n, Dh].
    """
    q, hk, hv = _f64(q), _f64(hk), _f64(hv)
    B, T, H, Dh = q.shape
    m, mp = _mask(dense_mask, H)
    if rows is None:
        o = np.empty_like(q)
        _load().orc_attention(_p(q), _p(hk), _p(hv), _p(o), B, T, H, Dh, D, W, mp, None, 0)
        return o
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    o = np.empty((r.shape[0], Dh), dtype=np.float64)
    _load().orc_attention(_p(q), _p(hk), _p(hv), _p(o), B, T, H, Dh, D, W, mp,
                          _p(r, _L), r.shape[0])
    return o


def attention_per_sample(q, hk, hv, D_per_sample, W: int, dense_mask=None, rows=None) -> np.ndarray:
    """Attention with one dilation per sample (the batch composition of the
    write-up's section 2.2: part of the batch dense, D = 1, part dilated):
    sample b is ``attention`` of that sample alone with D = D_per_sample[b].

    rows: optional int array [n, 3] of (b, t, h); then returns [n, Dh].
    """
    q, hk, hv = _f64(q), _f64(hk), _f64(hv)
    B = q.shape[0]
    ds = [int(d) for d in D_per_sample]
    assert len(ds) == B and min(ds, default=1) >= 1
    if rows is None:
        return np.concatenate([attention(q[b:b + 1], hk[b:b + 1], hv[b:b + 1], ds[b], W, dense_mask)
                               for b in range(B)], axis=0) if B else np.empty_like(q)
    r = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    o = np.empty((r.shape[0], q.shape[3]), dtype=np.float64)
    for b in sorted(set(r[:, 0].tolist())):
        sel = np.nonzero(r[:, 0] == b)[0]
        rb = r[sel].copy()
        rb[:, 0] = 0
        o[sel] = attention(q[b:b + 1], hk[b:b + 1], hv[b:b + 1], ds[b], W, dense_mask, rows=rb)
    return o


def attention_mask(q, hk, hv, D: int, W: int, dense_mask=None) -> np.ndarray:
    """Brute force over an explicit T x T mask (tiny T only)."""
    q, hk, hv = _f64(q), _f64(hk), _f64(hv)
    B, T, H, Dh = q.shape
    m, mp = _mask(dense_mask, H)
    o = np.empty_like(q)
    _load().orc_attention_mask(_p(q), _p(hk), _p(hv), _p(o), B, T, H, Dh, D, W, mp)
    return o


def cache_row(b, h, s, H, T_max, D, dense_mask=None) -> int:
    m, mp = _mask(dense_mask, H)
    return int(_load().orc_cache_row(b, h, s, H, T_max, D, mp))


def cache_rows_total(B, H, T_max, D, dense_mask=None) -> int:
    m, mp = _mask(dense_mask, H)
    return int(_load().orc_cache_rows_total(B, H, T_max, D, mp))


def ring_row(b, h, p, H, W) -> int:
    return int(_load().orc_ring_row(b, h, p, H, W))


class Cache:
    """fp64 mirror of the D-compressed cache plus the fp64 recurrent state."""

    def __init__(self, B, H, Dh, T_max, D, W, dense_mask=None, L=0):
        """L > 0: chunk-local recurrence (state zeroed at every t mod L == 0)."""
        assert L >= 0
        self.B, self.H, self.Dh, self.T_max, self.D, self.W = B, H, Dh, T_max, D, W
        self.L = L
        self.mask, self._mp = _mask(dense_mask, H)
        rows = cache_rows_total(B, H, T_max, D, dense_mask)
        self.Kc = np.zeros((rows, Dh))
        self.Vc = np.zeros((rows, Dh))
        wr = max(B * H * W, 1)
        self.Kw = np.zeros((wr, Dh))
        self.Vw = np.zeros((wr, Dh))
        self.len = np.zeros(B, dtype=np.int64)
        self.state = np.zeros((2, B, H, Dh))

    def pack(self, hk, hv, state=None):
        """Fill from prefill histories [B, T, H, Dh]; state = [2, B, H, Dh]."""
        hk, hv = _f64(hk), _f64(hv)
        B, T, H, Dh = hk.shape
        _load().orc_cache_pack(_p(hk), _p(hv), B, T, H, Dh, self.T_max, self.D, self.W,
                               self._mp, _p(self.Kc), _p(self.Vc), _p(self.Kw),
                               _p(self.Vw), _p(self.len, _L))
        if state is not None:
            self.state[...] = state

    def decode_step(self, q, xk, xv, g) -> np.ndarray:
        q, xk, xv, g = _f64(q), _f64(xk), _f64(xv), _f64(g)
        o = np.empty_like(q)
        rc = _load().orc_decode_step(_p(q), _p(xk), _p(xv), _p(g), _p(self.state),
                                     _p(self.Kc), _p(self.Vc), _p(self.Kw), _p(self.Vw),
                                     _p(self.len, _L), _p(o), self.B, self.H, self.Dh,
                                     self.T_max, self.D, self.W, self._mp, self.L)
        if rc != 0:
            raise RuntimeError("oracle decode: cache capacity exceeded")
        return o
