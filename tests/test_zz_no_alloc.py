"""The allocation-free scan entry point, ratp_scan_prefill_kv_noalloc.

Some callers cannot allocate device memory themselves (a plug-in inside an
application whose pool owns all device memory, or a latency-critical path
that may not pay cudaMalloc's implicit synchronisation), so they cannot pass
the scratch workspace that ratp_scan_prefill_kv takes.  This variant uses a
fixed array inside the library instead.  The test calls it through the C ABI
and compares it with the workspace-taking entry point on two calls in a row
(different shapes, so a stale array from the first call would show): both run
the same kernel, so the outputs must be bit-identical.  It also pins the
capacity limit exactly: the largest shape that fits (6,553 chunks) is
accepted and bit-identical, one chunk more is refused.  It lives in a file of
its own, collected last.
"""
import ctypes

import pytest
import torch

import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import prefill_inputs
from parity import bits_equal

pytestmark = pytest.mark.gpu
DEV = "cuda"
CAPACITY = 4          # RATP_ERR_CAPACITY
MAX_CHUNKS = 6553     # 16 MiB of scratch at 2,560 bytes per chunk (+ a 256-byte header)


def _noalloc(lib, xk, xv, g, hk, hv, fs):
    B, T, H, Dh = xk.shape
    dt = 1 if xk.dtype == torch.bfloat16 else 0
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.ratp_scan_prefill_kv_noalloc(
        p(xk), p(xv), p(g), p(hk), p(hv), p(fs), B, T, H, Dh, dt,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _compare(lib, xk, xv, g, what):
    B, T, H, Dh = xk.shape
    fs_ref = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    hk_ref, hv_ref = ratp.scan_prefill_kv(xk, xv, g, final_state=fs_ref)
    hk, hv = torch.full_like(xk, float("nan")), torch.full_like(xv, float("nan"))
    fs = torch.full_like(fs_ref, float("nan"))
    assert _noalloc(lib, xk, xv, g, hk, hv, fs) == 0
    ratp.last_error()
    assert bits_equal(hk, hk_ref), "hk " + what
    assert bits_equal(hv, hv_ref), "hv " + what
    assert bits_equal(fs, fs_ref), "final state " + what


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_scan_matches_workspace_scan_on_two_calls(dtype):
    lib = ratp.load_library()
    for call, (B, T, H, Dh) in enumerate([(2, 3000, 4, 128), (1, 4099, 2, 64)]):
        _, xk, xv, g = prefill_inputs(B, T, H, Dh, dtype, gate_mean=2.0, gate_std=1.5, seed=call)
        _compare(lib, xk.to(DEV), xv.to(DEV), g.to(DEV), "call %d" % call)


@pytest.mark.parametrize("dtype,chunk", [("bf16", 256), ("f32", 128)])
def test_noalloc_capacity_boundary(dtype, chunk):
    """6,553 chunks of one 64-channel slab fit the fixed scratch and match the
    workspace path bit for bit; 6,554 chunks are refused before any launch."""
    lib = ratp.load_library()
    T = MAX_CHUNKS * chunk
    _, xk, xv, g = prefill_inputs(1, T, 1, 64, dtype, gate_mean=2.0, gate_std=1.5, seed=5)
    _compare(lib, xk.to(DEV), xv.to(DEV), g.to(DEV), "at %d chunks" % MAX_CHUNKS)
    x = torch.zeros(16, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device=DEV)
    f = torch.zeros(16, dtype=torch.float32, device=DEV)
    assert _noalloc_raw(lib, x, f, 1, T + 1, 1, 64, dtype) == CAPACITY


def test_noalloc_scan_rejects_oversized_shapes():
    lib = ratp.load_library()
    x = torch.zeros(16, dtype=torch.bfloat16, device=DEV)
    f = torch.zeros(16, dtype=torch.float32, device=DEV)
    # 8 x 65536 tokens x 4096 channels needs far more than the fixed scratch
    assert _noalloc_raw(lib, x, f, 8, 65536, 32, 128, "bf16") == CAPACITY


def _noalloc_raw(lib, x, f, B, T, H, Dh, dtype):
    p = ctypes.c_void_p(x.data_ptr())
    return lib.ratp_scan_prefill_kv_noalloc(p, p, p, p, p, ctypes.c_void_p(f.data_ptr()),
                                            B, T, H, Dh, 1 if dtype == "bf16" else 0,
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
