"""GPU parity of dilated attention with one dilation per sample in one launch
(the batch composition of active recurrence learning: part of the batch
dense, part dilated) against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, prefill_inputs
from recurrence_augmented_dilated_chunked_b200._binding import RatpError
from parity import assert_close, bits_equal, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, T, H, seed):
    q, xk, xv, g = prefill_inputs(B, T, H, 128, "bf16", seed=seed)
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV))
    return q.to(DEV), hk, hv


@pytest.mark.parametrize("B,T,H,Ds,W,mask", [
    (4, 1000, 2, [1, 64, 1, 64], 0, None),             # half dense, half D = 64
    (4, 1000, 2, [64, 1, 64, 1], 128, None),
    (6, 777, 3, [3, 1, 64, 5, 3, 1000], 16, [1, 0, 0]),  # D > T: self (+ window) only
    (3, 300, 2, [2, 2, 2], 0, [0, 1]),                 # one class: the per-head path's shape
    (5, 129, 2, [1, 1, 1, 1, 1], 0, None),             # every sample dense
    (4, 520, 2, [2, 7, 16, 64], 8, None),              # four dilation classes
])
def test_per_sample_matches_oracle(B, T, H, Ds, W, mask):
    q, hk, hv = _inputs(B, T, H, seed=T + B)
    o = ratp.dilated_attn_prefill_per_sample(q, hk, hv, Ds, W, head_mask=mask)
    ratp.last_error()
    ref = oracle.attention_per_sample(to64(q.cpu()), to64(hk.cpu()), to64(hv.cpu()), Ds, W, dense_mask=mask)
    assert_close(o, ref, "bf16", "per-sample o, D=%s" % Ds)


@pytest.mark.parametrize("Ds,W,mask", [([1, 64, 4, 1, 64], 0, None), ([16, 1, 3, 3, 16], 32, [0, 1])])
def test_per_sample_equals_single_sample_launches_bit_exact(Ds, W, mask):
    """Sample b of the one launch is bit-identical to a launch of sample b
    alone with D = Ds[b] (same tiles, same order)."""
    B, T, H = len(Ds), 640, 2
    q, hk, hv = _inputs(B, T, H, seed=21)
    o = ratp.dilated_attn_prefill_per_sample(q, hk, hv, Ds, W, head_mask=mask)
    for b, d in enumerate(Ds):
        ob = ratp.dilated_attn_prefill(q[b:b + 1].contiguous(), hk[b:b + 1].contiguous(),
                                       hv[b:b + 1].contiguous(), d, W, head_mask=mask)
        assert bits_equal(o[b:b + 1], ob), "sample %d (D=%d)" % (b, d)
    ratp.last_error()


def test_per_sample_errors():
    q, hk, hv = _inputs(6, 64, 1, seed=3)
    with pytest.raises(RatpError) as e:        # five distinct dilations > 1
        ratp.dilated_attn_prefill_per_sample(q, hk, hv, [2, 3, 4, 5, 6, 1])
    assert e.value.code == 7
    with pytest.raises(RatpError) as e:
        ratp.dilated_attn_prefill_per_sample(q, hk, hv, [2, 0, 4, 5, 1, 1])
    assert e.value.code == 1
    qf = q.float()
    with pytest.raises(RatpError) as e:
        ratp.dilated_attn_prefill_per_sample(qf, hk.float(), hv.float(), [1] * 6)
    assert e.value.code == 7
    with pytest.raises(ValueError):
        ratp.dilated_attn_prefill_per_sample(q, hk, hv, [1, 2])
    empty = torch.empty(2, 0, 1, 128, dtype=torch.bfloat16, device=DEV)
    ratp.dilated_attn_prefill_per_sample(empty, empty, empty, [1, 64])
    ratp.last_error()


def test_per_sample_full_size_sampled_rows():
    """The batch composition on the 1.5B-like T = 4096 layer: samples 0-3
    dense, 4-7 at D = 64; sampled query rows of every sample."""
    w = WORKLOADS["bf16_1p5b_T4096_D16"]
    Ds = [1] * (w.B // 2) + [64] * (w.B - w.B // 2)
    q, xk, xv, g = prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV))
    o = ratp.dilated_attn_prefill_per_sample(q.to(DEV), hk, hv, Ds, 0)
    ratp.last_error()
    rng = np.random.default_rng(4)
    hk_c, hv_c = hk.cpu(), hv.cpu()
    for b in range(w.B):
        ts = np.concatenate([[0, 63, 64, 127, w.T - 1], rng.integers(0, w.T, 6)])
        hs = rng.integers(0, w.H, ts.size)
        rows = np.stack([np.zeros_like(ts), ts, hs], 1)
        # one sample at a time keeps the fp64 copies small
        ref = oracle.attention_per_sample(to64(q[b:b + 1]), to64(hk_c[b:b + 1]), to64(hv_c[b:b + 1]),
                                          [Ds[b]], 0, rows=rows)
        got = o[b, torch.as_tensor(ts, device=DEV), torch.as_tensor(hs, device=DEV)]
        assert_close(got, ref, "bf16", "sampled rows of sample %d (D=%d)" % (b, Ds[b]))


def test_per_sample_largest_batch():
    """1024 samples (the most one launch takes), every sample its own mix of
    the dilations {1, 2, 3, 64}; 1025 samples are refused."""
    B, T, H = 1024, 70, 1
    q, hk, hv = _inputs(B, T, H, seed=99)
    Ds = [(1, 2, 3, 64)[(b * 7) % 4] for b in range(B)]
    o = ratp.dilated_attn_prefill_per_sample(q, hk, hv, Ds, 4)
    ratp.last_error()
    ref = oracle.attention_per_sample(to64(q.cpu()), to64(hk.cpu()), to64(hv.cpu()), Ds, 4)
    assert_close(o, ref, "bf16", "1024 samples")
    q2, hk2, hv2 = _inputs(B + 1, 8, 1, seed=98)
    with pytest.raises(RatpError) as e:
        ratp.dilated_attn_prefill_per_sample(q2, hk2, hv2, [1] * (B + 1))
    assert e.value.code == 2


def test_per_sample_dynamic_and_static_dealing_agree_bitwise():
    """With the binding's workspace the mixed batch is dealt dynamically;
    without one (the plain C entry point), in fixed rounds: same bits."""
    import ctypes
    from recurrence_augmented_dilated_chunked_b200 import _binding
    Ds = [1, 64, 1, 64, 4, 1]
    B, T, H = len(Ds), 900, 3
    q, hk, hv = _inputs(B, T, H, seed=44)
    o_dyn = ratp.dilated_attn_prefill_per_sample(q, hk, hv, Ds, 16, head_mask=[0, 1, 0])
    o_static = torch.empty_like(q)
    lib = _binding.load_library()
    dbuf = (ctypes.c_int32 * B)(*Ds)
    mbuf, mp = _binding._mask_buf([0, 1, 0], H)
    rc = lib.ratp_dilated_attn_prefill_per_sample(
        _binding._ptr(q), _binding._ptr(hk), _binding._ptr(hv), _binding._ptr(o_static), B, T, H, 128,
        ctypes.cast(dbuf, ctypes.c_void_p), 16, mp, 1, _binding._stream(q))
    assert rc == 0
    ratp.last_error()
    assert bits_equal(o_dyn, o_static)
