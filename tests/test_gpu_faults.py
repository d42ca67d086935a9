"""Failure detection on the GPU without a GPU fault.

Each test plants a missing publication (a flag that nothing sets) through
``ratp_debug_fault``, with the device wait bound lowered to 50 ms: the waiting
kernel gives up, records RATP_ERR_TIMEOUT in the device error word, and ends
normally.  The host reads the status, and the same call made afterwards on
the same context computes the right answer.
"""
import time

import pytest

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import _binding, prefill_inputs
from recurrence_augmented_dilated_chunked_b200._binding import RatpError
from parity import assert_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
LIMIT_NS = 50_000_000


@pytest.fixture(autouse=True)
def _reset_faults():
    yield
    ratp.debug_fault(_binding.FAULT_NONE)


def test_scan_missing_chunk_times_out_then_recovers():
    B, T, H, Dh = 2, 4096, 4, 128          # 2 x 8 x 32 = 512 chunks
    _, xk, xv, g = prefill_inputs(B, T, H, Dh, "bf16", seed=21)
    xk, xv, g = xk.to(DEV), xv.to(DEV), g.to(DEV)
    ratp.last_error()
    ratp.debug_fault(_binding.FAULT_SPIN_LIMIT, LIMIT_NS)
    ratp.debug_fault(_binding.FAULT_SCAN_DROP, 200)
    t0 = time.time()
    ratp.scan_prefill_kv(xk, xv, g)
    with pytest.raises(RatpError, match="TIMEOUT"):
        ratp.last_error()
    assert time.time() - t0 < 30
    ratp.debug_fault(_binding.FAULT_NONE)
    hk, hv = ratp.scan_prefill_kv(xk, xv, g)
    ratp.last_error()
    sl = (slice(None), slice(None), slice(0, 1))
    assert_close(hk[sl], oracle.scan(to64(xk[sl].cpu()), to64(g[sl].cpu())), "bf16", "hk after recovery")


def test_attention_missing_tile_times_out_then_recovers():
    B, T, H, D = 1, 1000, 2, 4
    q, k, v, _ = prefill_inputs(B, T, H, 128, "bf16", seed=22)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    ratp.last_error()
    ratp.debug_fault(_binding.FAULT_SPIN_LIMIT, LIMIT_NS)
    ratp.debug_fault(_binding.FAULT_ATTN_DROP_K, 1)
    t0 = time.time()
    ratp.dilated_attn_prefill(q, k, v, D, 0)
    with pytest.raises(RatpError, match="TIMEOUT"):
        ratp.last_error()
    assert time.time() - t0 < 30
    ratp.debug_fault(_binding.FAULT_NONE)
    o = ratp.dilated_attn_prefill(q, k, v, D, 0)
    ratp.last_error()
    ref = oracle.attention(to64(q.cpu()), to64(k.cpu()), to64(v.cpu()), D, 0)
    assert_close(o, ref, "bf16", "attention after recovery")
