"""CPU checks of the C ABI: the library builds, loads, exports every function
that ``include/ratp.h`` declares, and rejects bad arguments on the host before
touching the GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import _binding, build

HEADER = os.path.join(ROOT, "include", "ratp.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(ratp_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return ratp.load_library()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(_binding.exported_symbols())


def _struct_fields(body):
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = []
    for decl in body.split(";"):
        parts = [x.strip() for x in decl.strip().split(",") if x.strip()]
        if not parts:
            continue
        names.append(parts[0].split()[-1].lstrip("*"))
        names.extend(x.lstrip("*") for x in parts[1:])
    return [re.sub(r"\[.*\]", "", n) for n in names]


def test_cache_struct_matches_header():
    src = open(HEADER).read()
    body = re.search(r"typedef struct ratp_cache \{(.*?)\} ratp_cache;", src, re.S).group(1)
    assert _struct_fields(body) == [f[0] for f in _binding.CacheStruct._fields_]


def test_debug_fault_rejects_unknown_kind_on_host(lib):
    assert lib.ratp_debug_fault(99, 0) == 1
    assert lib.ratp_debug_fault(-1, 0) == 1


def test_status_strings(lib):
    assert lib.ratp_status_string(0) == b"ok"
    assert b"aligned" in lib.ratp_status_string(3)
    assert b"guarded" in lib.ratp_status_string(8)


def test_normal_build_is_not_guarded(lib):
    line = ctypes.c_int(-1)
    assert lib.ratp_guard_line(ctypes.byref(line)) == 7 and line.value == 0
    assert lib.ratp_debug_guard_probe(None) == 7
    assert lib.ratp_guard_line(None) == 1


def test_guarded_build_exports_the_same_abi():
    from recurrence_augmented_dilated_chunked_b200 import build as B
    path = B.build_library(guarded=True)
    g = ctypes.CDLL(path)
    for name in _binding.exported_symbols():
        assert hasattr(g, name), name


def test_scan_workspace_query(lib):
    n = ctypes.c_size_t()
    assert lib.ratp_scan_workspace_bytes(8, 4096, 16, 128, 1, ctypes.byref(n)) == 0
    # bf16 chunks of 256 tokens x 64 channels; per chunk 32 lanes x 64-bit
    # words: 2 x (1 + 2) aggregate words and 2 x 2 inclusive words
    chunks = 8 * (2048 // 64) * (4096 // 256)
    assert n.value >= chunks * 32 * 8 * (2 * 3 + 2 * 2)
    assert lib.ratp_scan_workspace_bytes(1, 10, 1, 32, 1, ctypes.byref(n)) == 2   # H*Dh % 64
    assert lib.ratp_scan_workspace_bytes(-1, 10, 1, 64, 1, ctypes.byref(n)) == 1
    assert lib.ratp_scan_workspace_bytes(1, 10, 1, 64, 7, ctypes.byref(n)) == 1


def test_fused_prefill_workspace_query(lib):
    n = ctypes.c_size_t()
    assert lib.ratp_prefill_fused_workspace_bytes(2, 16384, 16, 128, ctypes.byref(n)) == 0
    # 256-token x 64-channel chunks: a 4-byte done flag each, plus the chunk
    # scan's descriptor words for two streams (as ratp_scan_workspace_bytes)
    chunks = 2 * (2048 // 64) * (16384 // 256)
    s = ctypes.c_size_t()
    assert lib.ratp_scan_workspace_bytes(2, 16384, 16, 128, 1, ctypes.byref(s)) == 0
    assert n.value >= s.value + 4 * chunks
    # a ragged T rounds the chunks up
    m = ctypes.c_size_t()
    assert lib.ratp_prefill_fused_workspace_bytes(1, 257, 2, 128, ctypes.byref(m)) == 0
    assert m.value >= 4 * (1 * 4 * 2)
    assert lib.ratp_prefill_fused_workspace_bytes(1, 256, 2, 64, ctypes.byref(m)) == 7    # Dh != 128
    assert lib.ratp_prefill_fused_workspace_bytes(-1, 256, 2, 128, ctypes.byref(m)) == 1


def test_fused_prefill_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)
    ws = ctypes.c_void_p(4096)
    # null pointers, misalignment, fp32, too small a workspace, bad D / W
    assert lib.ratp_prefill_fused(p, p, p, p, p, p, p, None, 1, 8, 1, 128, 4, 0, None, 1, None, 0, None) == 1
    assert lib.ratp_prefill_fused(p, p, p, ctypes.c_void_p(18), p, p, p, None, 1, 8, 1, 128, 4, 0, None, 1,
                                  ws, 1 << 20, None) == 3
    assert lib.ratp_prefill_fused(p, p, p, p, p, p, p, None, 1, 8, 1, 128, 4, 0, None, 0, ws, 1 << 20, None) == 7
    assert lib.ratp_prefill_fused(p, p, p, p, p, p, p, None, 1, 8, 1, 128, 4, 0, None, 1, ws, 16, None) == 4
    assert lib.ratp_prefill_fused(p, p, p, p, p, p, p, None, 1, 8, 1, 128, 0, 0, None, 1, ws, 1 << 20, None) == 1
    assert lib.ratp_prefill_fused(p, p, p, p, p, p, p, None, 1, 8, 1, 128, 4, -1, None, 1, ws, 1 << 20, None) == 1


def test_attention_workspace_entry_points_check_arguments_on_host(lib):
    p = ctypes.c_void_p(16)
    # a misaligned workspace, then the checks of the plain calls (D < 1, W < 0)
    assert lib.ratp_dilated_attn_prefill_ws(p, p, p, p, 1, 8, 1, 128, 4, 0, None, 1,
                                            ctypes.c_void_p(18), None) == 3
    assert lib.ratp_dilated_attn_prefill_ws(p, p, p, p, 1, 8, 1, 128, 0, 0, None, 1, p, None) == 1
    assert lib.ratp_dilated_attn_prefill_ws(p, p, p, p, 1, 8, 1, 128, 4, -1, None, 1, p, None) == 1
    ds = (ctypes.c_int32 * 2)(1, 0)
    assert lib.ratp_dilated_attn_prefill_per_sample_ws(p, p, p, p, 2, 8, 1, 128, ctypes.cast(ds, ctypes.c_void_p),
                                                       0, None, 1, p, None) == 1
    assert lib.ratp_dilated_attn_prefill_per_sample_ws(p, p, p, p, 2, 8, 1, 128, ctypes.cast(ds, ctypes.c_void_p),
                                                       0, None, 1, ctypes.c_void_p(18), None) == 3
    assert _binding.ATTN_WORKSPACE_BYTES == 256


def test_cache_bytes_query(lib):
    n = ctypes.c_size_t()
    assert lib.ratp_cache_bytes(64, 16, 128, 33024, 64, 128, None, ctypes.byref(n)) == 0
    rows = 64 * 16 * (33024 // 64)
    ring = 64 * 16 * 128
    assert n.value >= 2 * (rows + ring) * 256
    mask = (ctypes.c_uint8 * 4)(1, 0, 0, 0)
    m = ctypes.c_size_t()
    assert lib.ratp_cache_bytes(1, 4, 128, 64, 4, 0, ctypes.cast(mask, ctypes.c_void_p), ctypes.byref(m)) == 0
    assert m.value >= 2 * (64 + 3 * 16) * 256
    assert lib.ratp_cache_bytes(1, 4, 96, 64, 4, 0, None, ctypes.byref(m)) == 2
    assert lib.ratp_cache_bytes(1, 4, 128, 64, 0, 0, None, ctypes.byref(m)) == 1


def test_attention_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)
    # D < 1, W < 0, Dh unsupported, null pointers, misaligned pointers
    assert lib.ratp_dilated_attn_prefill(p, p, p, p, 1, 8, 1, 128, 0, 0, None, 1, None) == 1
    assert lib.ratp_dilated_attn_prefill(p, p, p, p, 1, 8, 1, 128, 2, -1, None, 1, None) == 1
    assert lib.ratp_dilated_attn_prefill(p, p, p, p, 1, 8, 1, 96, 2, 0, None, 1, None) == 2
    assert lib.ratp_dilated_attn_prefill(None, p, p, p, 1, 8, 1, 128, 2, 0, None, 1, None) == 1
    q = ctypes.c_void_p(24)
    assert lib.ratp_dilated_attn_prefill(q, p, p, p, 1, 8, 1, 128, 2, 0, None, 1, None) == 3
    assert lib.ratp_dilated_attn_prefill_simt(p, p, p, p, 1, 8, 300, 64, 2, 0, None, 0, None) == 2
    # empty problem: nothing to do, no launch
    assert lib.ratp_dilated_attn_prefill(None, None, None, None, 0, 8, 1, 128, 2, 0, None, 1, None) == 0


def test_scan_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)
    assert lib.ratp_scan_prefill(None, p, p, None, 1, 8, 1, 64, 1, p, 1 << 20, None) == 1
    assert lib.ratp_scan_prefill(ctypes.c_void_p(8), p, p, None, 1, 8, 1, 64, 1, p, 1 << 20, None) == 3
    # workspace too small
    assert lib.ratp_scan_prefill(p, p, p, None, 1, 8, 1, 64, 1, p, 16, None) == 4
    assert lib.ratp_scan_prefill_kv(p, p, p, p, p, None, 1, 8, 1, 64, 1, None, 1 << 20, None) == 1
    # T == 0 is a no-op
    assert lib.ratp_scan_prefill(None, None, None, None, 1, 0, 1, 64, 1, None, 0, None) == 0


def test_window_scan_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)
    assert lib.ratp_scan_prefill_kv_window(p, p, p, p, p, 1, 8, 1, 64, 1, 0, None) == 1
    assert lib.ratp_scan_prefill_kv_window(p, p, p, p, p, 1, 8, 1, 64, 1, 48, None) == 7
    assert lib.ratp_scan_prefill_kv_window(p, p, p, p, p, 1, 8, 1, 32, 1, 64, None) == 2
    assert lib.ratp_scan_prefill_kv_window(None, p, p, p, p, 1, 8, 1, 64, 1, 64, None) == 1
    assert lib.ratp_scan_prefill_kv_window(ctypes.c_void_p(8), p, p, p, p, 1, 8, 1, 64, 1, 64, None) == 3
    assert lib.ratp_scan_prefill_kv_window(None, None, None, None, None, 1, 0, 1, 64, 1, 64, None) == 0


def test_chunk_local_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)
    # a negative block length is refused before anything else is looked at
    assert lib.ratp_scan_prefill_kv_chunk_local(p, p, p, p, p, None, 1, 8, 1, 64, 1, -1,
                                                p, 1 << 20, None) == 1
    assert lib.ratp_scan_prefill_chunk_local(p, p, p, None, 1, 8, 1, 64, 1, -5, p, 1 << 20, None) == 1
    assert lib.ratp_scan_prefill_chunk_local(None, p, p, None, 1, 8, 1, 64, 1, 4, p, 1 << 20, None) == 1
    assert lib.ratp_scan_prefill_kv_chunk_local(None, None, None, None, None, None, 1, 0, 1, 64, 1, 4,
                                                None, 0, None) == 0
    c = _binding.CacheStruct()
    assert lib.ratp_cache_set_chunk_local(ctypes.byref(c), -1) == 1
    assert lib.ratp_cache_set_chunk_local(None, 4) == 1
    assert lib.ratp_cache_set_chunk_local(ctypes.byref(c), 16) == 0 and c.reset_L == 16
    assert lib.ratp_cache_set_chunk_local(ctypes.byref(c), 0) == 0 and c.reset_L == 0


def test_decode_rejects_mismatched_cache_on_host(lib):
    c = _binding.CacheStruct()
    c.D, c.W, c.H = 4, 0, 2
    p = ctypes.c_void_p(16)
    assert lib.ratp_decode_step(p, p, p, p, p, ctypes.byref(c), p, 8, 0, None, None) == 1
    assert lib.ratp_decode_step(p, p, p, p, p, ctypes.byref(c), p, 4, 3, None, None) == 1
    mask = (ctypes.c_uint8 * 2)(1, 0)
    assert lib.ratp_decode_step(p, p, p, p, p, ctypes.byref(c), p, 4, 0,
                                ctypes.cast(mask, ctypes.c_void_p), None) == 1


def test_per_sample_attention_rejects_bad_arguments_on_host(lib):
    p = ctypes.c_void_p(16)
    ds = (ctypes.c_int32 * 4)(1, 64, 0, 1)
    dp = ctypes.cast(ds, ctypes.c_void_p)
    assert lib.ratp_dilated_attn_prefill_per_sample(p, p, p, p, 2, 8, 1, 128, None, 0, None, 1, None) == 1
    assert lib.ratp_dilated_attn_prefill_per_sample(p, p, p, p, 4, 8, 1, 128, dp, 0, None, 1, None) == 1
    ds[2] = 4
    assert lib.ratp_dilated_attn_prefill_per_sample(p, p, p, p, 4, 8, 1, 128, dp, 0, None, 0, None) == 7
    assert lib.ratp_dilated_attn_prefill_per_sample(p, p, p, p, 4, 8, 1, 64, dp, 0, None, 1, None) == 7
    big = (ctypes.c_int32 * 2000)(*([1] * 2000))
    assert lib.ratp_dilated_attn_prefill_per_sample(p, p, p, p, 2000, 8, 1, 128,
                                                    ctypes.cast(big, ctypes.c_void_p), 0, None, 1, None) == 2
    # empty problem: nothing to do, no launch
    assert lib.ratp_dilated_attn_prefill_per_sample(None, None, None, None, 4, 0, 1, 128, dp, 0, None, 1,
                                                    None) == 0


def test_cache_window_api_on_host(lib):
    n = ctypes.c_size_t()
    assert lib.ratp_cache_window_bytes(2, 3, 128, 64, ctypes.byref(n)) == 0
    assert n.value == 3 * 2 * 3 * 64 * 128 * 2
    assert lib.ratp_cache_window_bytes(2, 3, 128, 0, ctypes.byref(n)) == 1
    assert lib.ratp_cache_window_bytes(2, 3, 96, 8, ctypes.byref(n)) == 2
    c = _binding.CacheStruct()
    c.B, c.H, c.Dh, c.T_max = 2, 3, 128, 100
    p = ctypes.c_void_p(16)
    assert lib.ratp_cache_set_window(ctypes.byref(c), p, 16, 64) == 4       # ring too small
    assert lib.ratp_cache_set_window(ctypes.byref(c), ctypes.c_void_p(8), 1 << 30, 64) == 3
    assert lib.ratp_cache_set_window(ctypes.byref(c), p, 1 << 30, 64) == 0 and c.window_L == 64
    assert lib.ratp_cache_set_chunk_local(ctypes.byref(c), 4) == 1         # exclusive
    assert lib.ratp_cache_set_window(ctypes.byref(c), None, 0, 0) == 0 and c.window_L == 0
    assert lib.ratp_cache_set_chunk_local(ctypes.byref(c), 4) == 0
    assert lib.ratp_cache_set_window(ctypes.byref(c), p, 1 << 30, 64) == 1  # exclusive
    assert lib.ratp_cache_pack_inputs(ctypes.byref(c), p, p, p, 10, None) == 1  # no window


def test_decode_layers_rejects_bad_arguments_on_host(lib):
    assert lib.ratp_decode_step_layers(None, 0, None) == 0
    assert lib.ratp_decode_step_layers(None, 2, None) == 1
    arr = (_binding.DecodeLayerStruct * 2)()
    assert lib.ratp_decode_step_layers(arr, -1, None) == 1
    # a layer with a NULL field stops the call before any launch
    assert lib.ratp_decode_step_layers(arr, 2, None) == 1


def test_decode_layer_struct_matches_header():
    src = open(HEADER).read()
    body = re.search(r"typedef struct ratp_decode_layer \{(.*?)\} ratp_decode_layer;", src, re.S).group(1)
    assert _struct_fields(body) == [f[0] for f in _binding.DecodeLayerStruct._fields_]


def test_missing_library_fails_loudly(tmp_path):
    saved = _binding._lib
    _binding._lib = None
    try:
        with pytest.raises(RuntimeError, match="missing"):
            _binding.load_library(str(tmp_path / "nope.so"))
    finally:
        _binding._lib = saved


def test_cpu_tensors_are_refused_not_computed():
    """There is no CPU path: host tensors are refused before any call."""
    import torch
    import recurrence_augmented_dilated_chunked_b200 as ratp
    x = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16)
    calls = [
        lambda: ratp.scan_prefill(x, x),
        lambda: ratp.scan_prefill_kv(x, x, x),
        lambda: ratp.scan_prefill_kv(x, x, x, L=4),
        lambda: ratp.scan_prefill_kv_window(x, x, x, 16),
        lambda: ratp.scan_prefill_kv_noalloc(x, x, x, x, x),
        lambda: ratp.dilated_attn_prefill(x, x, x, 4),
        lambda: ratp.dilated_attn_prefill_simt(x, x, x, 4),
        lambda: ratp.dilated_attn_prefill_per_sample(x, x, x, [4]),
    ]
    for call in calls:
        with pytest.raises(ValueError):
            call()
