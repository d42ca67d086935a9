"""ctypes binding of ``libratp.so`` (the C ABI declared in ``include/ratp.h``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory and the current
stream.  There is no CPU fallback -- if the library is missing the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# RATP_LIBRARY may name another build of the same C ABI (the guarded debug
# build, libratp_guarded.so, for bounds-checked test runs)
LIB_PATH = os.environ.get("RATP_LIBRARY") or os.path.join(_PKG, "libratp.so")
MAX_HEADS = 256

RATP_F32, RATP_BF16 = 0, 1
_DTYPE = {torch.float32: RATP_F32, torch.bfloat16: RATP_BF16}

STATUS = {0: "OK", 1: "ERR_ARG", 2: "ERR_SHAPE", 3: "ERR_ALIGN", 4: "ERR_CAPACITY",
          5: "ERR_TIMEOUT", 6: "ERR_CUDA", 7: "ERR_UNSUPPORTED", 8: "ERR_BOUNDS"}


class RatpError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (fn, STATUS.get(code, "?"), code))


class CacheStruct(ctypes.Structure):
    """Mirror of ``struct ratp_cache``."""
    _fields_ = [
        ("Kc", ctypes.c_void_p), ("Vc", ctypes.c_void_p),
        ("Kw", ctypes.c_void_p), ("Vw", ctypes.c_void_p),
        ("len", ctypes.c_void_p), ("partial", ctypes.c_void_p), ("counters", ctypes.c_void_p),
        ("in_ring", ctypes.c_void_p),
        ("rows_per_b", ctypes.c_int64),
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("Dh", ctypes.c_int32),
        ("T_max", ctypes.c_int32), ("D", ctypes.c_int32), ("W", ctypes.c_int32),
        ("split_keys", ctypes.c_int32), ("max_splits", ctypes.c_int32),
        ("reset_L", ctypes.c_int32), ("window_L", ctypes.c_int32),
        ("dense", ctypes.c_uint8 * MAX_HEADS),
    ]


class DecodeLayerStruct(ctypes.Structure):
    """Mirror of ``struct ratp_decode_layer``."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("xk", ctypes.c_void_p), ("xv", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("state", ctypes.c_void_p),
        ("cache", ctypes.POINTER(CacheStruct)), ("o", ctypes.c_void_p),
    ]


_lib = None
_lock = threading.Lock()

_P, _I, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "ratp_status_string": ([_I], ctypes.c_char_p),
    "ratp_last_error": ([_P], _I),
    "ratp_device_sm_count": ([ctypes.POINTER(_I)], _I),
    "ratp_debug_fault": ([_I, ctypes.c_longlong], _I),
    "ratp_guard_line": ([ctypes.POINTER(_I)], _I),
    "ratp_debug_guard_probe": ([_P], _I),
    "ratp_scan_workspace_bytes": ([_I, _I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "ratp_scan_prefill": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _SZ, _P], _I),
    "ratp_scan_prefill_kv": ([_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _SZ, _P], _I),
    "ratp_scan_prefill_chunk_local": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _SZ, _P], _I),
    "ratp_scan_prefill_kv_chunk_local": ([_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _SZ, _P], _I),
    "ratp_scan_prefill_kv_window": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P], _I),
    "ratp_scan_prefill_kv_noalloc": ([_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P], _I),
    "ratp_dilated_attn_prefill": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P], _I),
    "ratp_dilated_attn_prefill_simt": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P], _I),
    "ratp_dilated_attn_prefill_per_sample": ([_P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _I, _P], _I),
    "ratp_dilated_attn_prefill_ws": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P, _P], _I),
    "ratp_dilated_attn_prefill_per_sample_ws": ([_P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _I, _P, _P], _I),
    "ratp_prefill_fused_workspace_bytes": ([_I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "ratp_prefill_fused": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P, _SZ, _P], _I),
    "ratp_cache_bytes": ([_I, _I, _I, _I, _I, _I, _P, ctypes.POINTER(_SZ)], _I),
    "ratp_cache_init": ([ctypes.POINTER(CacheStruct), _P, _SZ, _I, _I, _I, _I, _I, _I, _P, _P], _I),
    "ratp_cache_pack": ([ctypes.POINTER(CacheStruct), _P, _P, _I, _P], _I),
    "ratp_cache_set_chunk_local": ([ctypes.POINTER(CacheStruct), _I], _I),
    "ratp_cache_window_bytes": ([_I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "ratp_cache_set_window": ([ctypes.POINTER(CacheStruct), _P, _SZ, _I], _I),
    "ratp_cache_pack_inputs": ([ctypes.POINTER(CacheStruct), _P, _P, _P, _I, _P], _I),
    "ratp_decode_step": ([_P, _P, _P, _P, _P, ctypes.POINTER(CacheStruct), _P, _I, _I, _P, _P], _I),
    "ratp_decode_step_layers": ([ctypes.POINTER(DecodeLayerStruct), _I, _P], _I),
}


def load_library(path: str = LIB_PATH):
    """Load ``libratp.so``; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    "CUDA library %s is missing; build it with "
                    "`python -m recurrence_augmented_dilated_chunked_b200.build`" % path)
            lib = ctypes.CDLL(path)
            for name, (args, res) in _SIGS.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def exported_symbols():
    return sorted(_SIGS)


def _check(fn, code):
    if code != 0:
        raise RatpError(fn, code)


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))


def _mask_buf(head_mask, H):
    if head_mask is None:
        return None, None
    m = bytes(1 if v else 0 for v in list(head_mask))
    if len(m) != H:
        raise ValueError("head_mask must have H = %d entries" % H)
    buf = (ctypes.c_uint8 * H).from_buffer_copy(m)
    return buf, ctypes.cast(buf, ctypes.c_void_p)


_ws_cache = {}


def scan_workspace(B, T, H, Dh, dtype, device, stream=None) -> torch.Tensor:
    """Device scratch for one scan call of this shape on ``stream`` (default:
    the device's current stream).

    A workspace may only be shared by calls ordered on one stream, so the
    cache holds one per (device, stream, size): scans of the same shape on two
    unordered streams get different workspaces."""
    lib = load_library()
    n = ctypes.c_size_t()
    _check("ratp_scan_workspace_bytes",
           lib.ratp_scan_workspace_bytes(B, T, H, Dh, _DTYPE[dtype], ctypes.byref(n)))
    device = torch.device(device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    key = (str(device), stream.cuda_stream, n.value)
    with _lock:
        ws = _ws_cache.get(key)
        if ws is None:
            ws = torch.zeros(max(n.value, 256), dtype=torch.uint8, device=device)   # zero before first use
            if stream.cuda_stream != torch.cuda.current_stream(device).cuda_stream:
                torch.cuda.current_stream(device).synchronize()   # the zero fill precedes its first use
            _ws_cache[key] = ws
    return ws


def scan_prefill(x, g, out=None, final_state=None, workspace=None, L=0):
    """h = forget-gate scan of x with gates g over axis 1 of [B, T, H, Dh].

    L >= 1: chunk-local recurrence (the state restarts at t mod L == 0)."""
    lib = load_library()
    _need(x, "x")
    _need(g, "g", x.dtype)
    B, T, H, Dh = x.shape
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", x.dtype)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32)
    ws = workspace if workspace is not None else scan_workspace(B, T, H, Dh, x.dtype, x.device)
    if L:
        _check("ratp_scan_prefill_chunk_local", lib.ratp_scan_prefill_chunk_local(
            _ptr(x), _ptr(g), _ptr(out), _ptr(final_state), B, T, H, Dh, _DTYPE[x.dtype], int(L),
            _ptr(ws), ws.numel(), _stream(x)))
    else:
        _check("ratp_scan_prefill", lib.ratp_scan_prefill(
            _ptr(x), _ptr(g), _ptr(out), _ptr(final_state), B, T, H, Dh, _DTYPE[x.dtype],
            _ptr(ws), ws.numel(), _stream(x)))
    return out


def scan_prefill_kv(xk, xv, g, hk=None, hv=None, final_state=None, workspace=None, L=0):
    """(hk, hv) = scans of xk and xv sharing the gate tensor g (one pass).

    L >= 1: chunk-local recurrence (the state restarts at t mod L == 0)."""
    lib = load_library()
    _need(xk, "xk")
    _need(xv, "xv", xk.dtype)
    _need(g, "g", xk.dtype)
    B, T, H, Dh = xk.shape
    hk = torch.empty_like(xk) if hk is None else hk
    hv = torch.empty_like(xv) if hv is None else hv
    _need(hk, "hk", xk.dtype)
    _need(hv, "hv", xk.dtype)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32)
    ws = workspace if workspace is not None else scan_workspace(B, T, H, Dh, xk.dtype, xk.device)
    if L:
        _check("ratp_scan_prefill_kv_chunk_local", lib.ratp_scan_prefill_kv_chunk_local(
            _ptr(xk), _ptr(xv), _ptr(g), _ptr(hk), _ptr(hv), _ptr(final_state),
            B, T, H, Dh, _DTYPE[xk.dtype], int(L), _ptr(ws), ws.numel(), _stream(xk)))
    else:
        _check("ratp_scan_prefill_kv", lib.ratp_scan_prefill_kv(
            _ptr(xk), _ptr(xv), _ptr(g), _ptr(hk), _ptr(hv), _ptr(final_state),
            B, T, H, Dh, _DTYPE[xk.dtype], _ptr(ws), ws.numel(), _stream(xk)))
    return hk, hv


def scan_prefill_kv_window(xk, xv, g, L, hk=None, hv=None):
    """(hk, hv) with the fixed look-back recurrence: h_t runs from zero over the
    last L positions up to t (L = 16, 32 or 64)."""
    lib = load_library()
    _need(xk, "xk")
    _need(xv, "xv", xk.dtype)
    _need(g, "g", xk.dtype)
    B, T, H, Dh = xk.shape
    hk = torch.empty_like(xk) if hk is None else hk
    hv = torch.empty_like(xv) if hv is None else hv
    _need(hk, "hk", xk.dtype)
    _need(hv, "hv", xk.dtype)
    _check("ratp_scan_prefill_kv_window", lib.ratp_scan_prefill_kv_window(
        _ptr(xk), _ptr(xv), _ptr(g), _ptr(hk), _ptr(hv), B, T, H, Dh, _DTYPE[xk.dtype], int(L),
        _stream(xk)))
    return hk, hv


def scan_prefill_kv_noalloc(xk, xv, g, hk, hv, final_state=None):
    """(hk, hv) like ``scan_prefill_kv``, but the library supplies the scratch
    from its fixed device array, so nothing is allocated for the call (the
    outputs hk and hv must be passed in)."""
    lib = load_library()
    _need(xk, "xk")
    _need(xv, "xv", xk.dtype)
    _need(g, "g", xk.dtype)
    _need(hk, "hk", xk.dtype)
    _need(hv, "hv", xk.dtype)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32)
    B, T, H, Dh = xk.shape
    _check("ratp_scan_prefill_kv_noalloc", lib.ratp_scan_prefill_kv_noalloc(
        _ptr(xk), _ptr(xv), _ptr(g), _ptr(hk), _ptr(hv), _ptr(final_state),
        B, T, H, Dh, _DTYPE[xk.dtype], _stream(xk)))
    return hk, hv


ATTN_WORKSPACE_BYTES = 256
_attn_ws_cache = {}


def attn_workspace(device, stream=None) -> torch.Tensor:
    """The attention's small device workspace for ``stream`` (default: the
    device's current stream), cached per (device, stream): calls sharing one
    must be ordered on one stream.  It needs no initialisation."""
    device = torch.device(device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    key = (str(device), stream.cuda_stream)
    with _lock:
        ws = _attn_ws_cache.get(key)
        if ws is None:
            ws = torch.empty(ATTN_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
            _attn_ws_cache[key] = ws
    return ws


def _attn(fn_name, q, hk, hv, D, W, head_mask, out, workspace=False):
    lib = load_library()
    _need(q, "q")
    _need(hk, "hk", q.dtype)
    _need(hv, "hv", q.dtype)
    B, T, H, Dh = q.shape
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype)
    _buf, mp = _mask_buf(head_mask, H)
    args = [_ptr(q), _ptr(hk), _ptr(hv), _ptr(out), B, T, H, Dh, int(D), int(W), mp, _DTYPE[q.dtype]]
    if workspace is not False:
        args.append(_ptr(workspace) if workspace is not None else None)
    _check(fn_name, getattr(lib, fn_name)(*args, _stream(q)))
    return out


def dilated_attn_prefill(q, hk, hv, D, W=0, head_mask=None, out=None, workspace=None):
    """Dilated (+ windowed) causal attention of q over recurrent hk, hv.
    ``workspace``: an ``attn_workspace`` (default: the cached one of q's
    device and current stream), with which launches that mix dense and
    dilated items deal them dynamically."""
    if workspace is None and q.is_cuda:
        workspace = attn_workspace(q.device)
    return _attn("ratp_dilated_attn_prefill_ws", q, hk, hv, D, W, head_mask, out, workspace)


def dilated_attn_prefill_simt(q, hk, hv, D, W=0, head_mask=None, out=None):
    """Same operation on the CUDA-core kernel (fp32/bf16, Dh 64/128)."""
    return _attn("ratp_dilated_attn_prefill_simt", q, hk, hv, D, W, head_mask, out)


def dilated_attn_prefill_per_sample(q, hk, hv, D_per_sample, W=0, head_mask=None, out=None, workspace=None):
    """Dilated attention with one dilation per sample (``D_per_sample``: B
    ints >= 1; 1 = the sample runs dense) in one launch; bf16, Dh = 128.
    ``workspace`` as for ``dilated_attn_prefill``."""
    lib = load_library()
    _need(q, "q")
    _need(hk, "hk", q.dtype)
    _need(hv, "hv", q.dtype)
    B, T, H, Dh = q.shape
    if hk.shape != q.shape or hv.shape != q.shape:
        raise ValueError("q, hk, hv must have one shape")
    ds = [int(d) for d in D_per_sample]
    if len(ds) != B:
        raise ValueError("D_per_sample must have B = %d entries" % B)
    dbuf = (ctypes.c_int32 * max(B, 1))(*ds)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype)
    mbuf, mp = _mask_buf(head_mask, H)
    if q.dtype not in _DTYPE:
        raise ValueError("unsupported dtype %s" % q.dtype)
    if workspace is None and q.is_cuda:
        workspace = attn_workspace(q.device)
    _check("ratp_dilated_attn_prefill_per_sample_ws", lib.ratp_dilated_attn_prefill_per_sample_ws(
        _ptr(q), _ptr(hk), _ptr(hv), _ptr(out), B, T, H, Dh, ctypes.cast(dbuf, ctypes.c_void_p),
        int(W), mp, _DTYPE[q.dtype], _ptr(workspace) if workspace is not None else None, _stream(q)))
    return out


_fused_ws_cache = {}


def prefill_fused_workspace(B, T, H, Dh, device, stream=None) -> torch.Tensor:
    """Device scratch for one fused prefill of this shape on ``stream`` (default:
    the device's current stream), cached per (device, stream, size) like the
    scan workspace."""
    lib = load_library()
    n = ctypes.c_size_t()
    _check("ratp_prefill_fused_workspace_bytes",
           lib.ratp_prefill_fused_workspace_bytes(B, T, H, Dh, ctypes.byref(n)))
    device = torch.device(device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    key = (str(device), stream.cuda_stream, n.value)
    with _lock:
        ws = _fused_ws_cache.get(key)
        if ws is None:
            ws = torch.zeros(max(n.value, 256), dtype=torch.uint8, device=device)   # zero before first use
            if stream.cuda_stream != torch.cuda.current_stream(device).cuda_stream:
                torch.cuda.current_stream(device).synchronize()
            _fused_ws_cache[key] = ws
    return ws


def prefill_fused(q, xk, xv, g, D, W=0, head_mask=None, hk=None, hv=None, out=None, final_state=None,
                  workspace=None):
    """(o, hk, hv): the key/value recurrence and the dilated (+ windowed)
    attention over it in one launch; bf16, head dim 128."""
    lib = load_library()
    _need(q, "q")
    for t, nm in ((xk, "xk"), (xv, "xv"), (g, "g")):
        _need(t, nm, q.dtype)
    B, T, H, Dh = q.shape
    if xk.shape != q.shape or xv.shape != q.shape or g.shape != q.shape:
        raise ValueError("q, xk, xv, g must have one shape")
    hk = torch.empty_like(xk) if hk is None else hk
    hv = torch.empty_like(xv) if hv is None else hv
    out = torch.empty_like(q) if out is None else out
    for t, nm in ((hk, "hk"), (hv, "hv"), (out, "out")):
        _need(t, nm, q.dtype)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32)
    if q.dtype not in _DTYPE:
        raise ValueError("unsupported dtype %s" % q.dtype)
    ws = workspace if workspace is not None else prefill_fused_workspace(B, T, H, Dh, q.device)
    _buf, mp = _mask_buf(head_mask, H)
    _check("ratp_prefill_fused", lib.ratp_prefill_fused(
        _ptr(q), _ptr(xk), _ptr(xv), _ptr(g), _ptr(hk), _ptr(hv), _ptr(out), _ptr(final_state),
        B, T, H, Dh, int(D), int(W), mp, _DTYPE[q.dtype], _ptr(ws), ws.numel(), _stream(q)))
    return out, hk, hv


def last_error(device=None):
    """Synchronise and raise if any kernel recorded a device-side error."""
    lib = load_library()
    dev = torch.device("cuda" if device is None else device)
    s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    _check("ratp_last_error", lib.ratp_last_error(s))


FAULT_NONE, FAULT_SPIN_LIMIT, FAULT_SCAN_DROP, FAULT_ATTN_DROP_K, FAULT_FUSED_DROP_CHUNK = 0, 1, 2, 3, 4


def debug_fault(kind: int, arg: int = 0):
    """Plant a failure for tests of the error paths (see ``ratp_debug_fault``)."""
    _check("ratp_debug_fault", load_library().ratp_debug_fault(int(kind), int(arg)))


def sm_count() -> int:
    n = ctypes.c_int()
    _check("ratp_device_sm_count", load_library().ratp_device_sm_count(ctypes.byref(n)))
    return n.value


class KVCache:
    """D-compressed KV cache for decode (one device buffer, see ``ratp.h``)."""

    def __init__(self, B, H, Dh, T_max, D, W=0, head_mask=None, device="cuda", L=0):
        """L >= 1: decode continues a chunk-local recurrence of block L."""
        lib = load_library()
        self.B, self.H, self.Dh, self.T_max, self.D, self.W = B, H, Dh, T_max, D, W
        self.head_mask = [1 if v else 0 for v in head_mask] if head_mask is not None else None
        self._mask_buf, mp = _mask_buf(self.head_mask, H)
        n = ctypes.c_size_t()
        _check("ratp_cache_bytes", lib.ratp_cache_bytes(B, H, Dh, T_max, D, W, mp, ctypes.byref(n)))
        self.buffer = torch.empty(n.value, dtype=torch.uint8, device=device)
        self.c = CacheStruct()
        _check("ratp_cache_init", lib.ratp_cache_init(
            ctypes.byref(self.c), _ptr(self.buffer), n.value, B, H, Dh, T_max, D, W, mp,
            _stream(self.buffer)))
        self.L = int(L)
        _check("ratp_cache_set_chunk_local", lib.ratp_cache_set_chunk_local(ctypes.byref(self.c), self.L))

    def _view(self, addr, numel, dtype):
        off = addr - self.buffer.data_ptr()
        esz = torch.empty((), dtype=dtype).element_size()
        return self.buffer[off: off + numel * esz].view(dtype)

    def dil_rows(self, which="k"):
        """Kc or Vc as [B, rows_per_b, Dh] bf16 (a view of the buffer)."""
        addr = self.c.Kc if which == "k" else self.c.Vc
        rows = self.B * self.c.rows_per_b
        return self._view(addr, rows * self.Dh, torch.bfloat16).view(self.B, self.c.rows_per_b, self.Dh)

    def ring(self, which="k"):
        """Kw or Vw as [B, H, W, Dh] bf16 (None when W == 0)."""
        if self.W == 0:
            return None
        addr = self.c.Kw if which == "k" else self.c.Vw
        n = self.B * self.H * self.W * self.Dh
        return self._view(addr, n, torch.bfloat16).view(self.B, self.H, self.W, self.Dh)

    def lengths(self):
        return self._view(self.c.len, self.B, torch.int32)

    def head_rows(self, h):
        """(offset, capacity) of head h inside one batch item's dilated rows."""
        off = 0
        for k in range(self.H):
            cap = self.T_max if (self.head_mask and self.head_mask[k]) else self.T_max // self.D
            if k == h:
                return off, cap
            off += cap
        raise IndexError(h)

    def pack(self, hk, hv, T=None):
        _need(hk, "hk", torch.bfloat16)
        _need(hv, "hv", torch.bfloat16)
        T = hk.shape[1] if T is None else T
        _check("ratp_cache_pack", load_library().ratp_cache_pack(
            ctypes.byref(self.c), _ptr(hk), _ptr(hv), int(T), _stream(hk)))

    def attach_window(self, L):
        """Continue a fixed look-back recurrence of window L at decode: keeps a
        ring of the last L inputs (x_k, x_v, g) beside the cache."""
        lib = load_library()
        n = ctypes.c_size_t()
        _check("ratp_cache_window_bytes",
               lib.ratp_cache_window_bytes(self.B, self.H, self.Dh, int(L), ctypes.byref(n)))
        self.in_ring = torch.empty(n.value, dtype=torch.uint8, device=self.buffer.device)
        _check("ratp_cache_set_window", lib.ratp_cache_set_window(
            ctypes.byref(self.c), _ptr(self.in_ring), n.value, int(L)))

    def pack_inputs(self, xk, xv, g, T=None):
        """Prefill -> decode hand-off of the look-back inputs (last L positions)."""
        for t, nm in ((xk, "xk"), (xv, "xv"), (g, "g")):
            _need(t, nm, torch.bfloat16)
        T = xk.shape[1] if T is None else T
        _check("ratp_cache_pack_inputs", load_library().ratp_cache_pack_inputs(
            ctypes.byref(self.c), _ptr(xk), _ptr(xv), _ptr(g), int(T), _stream(xk)))

    def decode_step(self, q, xk, xv, g, state, out=None):
        """One token per sequence; state: fp32 [2, B, H, Dh] updated in place."""
        for t, n in ((q, "q"), (xk, "xk"), (xv, "xv"), (g, "g")):
            _need(t, n, torch.bfloat16)
        _need(state, "state", torch.float32)
        if out is None:
            out = torch.empty_like(q)
        _need(out, "out", torch.bfloat16)
        _check("ratp_decode_step", load_library().ratp_decode_step(
            _ptr(q), _ptr(xk), _ptr(xv), _ptr(g), _ptr(state), ctypes.byref(self.c), _ptr(out),
            self.D, self.W, ctypes.cast(self._mask_buf, ctypes.c_void_p) if self._mask_buf is not None else None,
            _stream(q)))
        return out


def decode_step_layers(layers):
    """One decode token through a stack of layers in one call.

    layers: sequence of (cache, q, xk, xv, g, state, out) with ``cache`` a
    ``KVCache`` (its own D, W, head mask and recurrence), q/xk/xv/g/out bf16
    [B, H, Dh] and state fp32 [2, B, H, Dh] (updated in place).  The layers
    run in order on the current stream of the first q.
    """
    n = len(layers)
    arr = (DecodeLayerStruct * max(n, 1))()
    for i, (cache, q, xk, xv, g, state, out) in enumerate(layers):
        for t, nm in ((q, "q"), (xk, "xk"), (xv, "xv"), (g, "g"), (out, "out")):
            _need(t, nm, torch.bfloat16)
        _need(state, "state", torch.float32)
        arr[i] = DecodeLayerStruct(q.data_ptr(), xk.data_ptr(), xv.data_ptr(), g.data_ptr(),
                                   state.data_ptr(), ctypes.pointer(cache.c), out.data_ptr())
    stream = _stream(layers[0][1]) if n else None
    _check("ratp_decode_step_layers", load_library().ratp_decode_step_layers(arr, n, stream))


def guard_line():
    """(guarded build?, source line of the first refused access or 0); the
    call clears the recorded line."""
    n = ctypes.c_int()
    rc = load_library().ratp_guard_line(ctypes.byref(n))
    if rc == 7:
        return False, 0
    _check("ratp_guard_line", rc)
    return True, n.value
