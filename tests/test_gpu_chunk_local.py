"""GPU parity of the chunk-local recurrence (the original RAT: the state
restarts at every block of L tokens) against the oracle, at prefill and at
decode.

Block lengths cover L = 1, L below, equal to and above the scan's chunk
(256 tokens for bf16, 128 for fp32), L that does not divide the chunk (so
blocks straddle CTAs and the look-back must stop at the last restart), and
L >= T (the full-sequence recurrence, bit for bit).
"""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, prefill_inputs
from recurrence_augmented_dilated_chunked_b200._binding import RatpError
from parity import assert_close, bits_equal, to64
from cache_layout import LayoutShadow

pytestmark = pytest.mark.gpu
DEV = "cuda"

LS = [1, 7, 64, 100, 128, 256, 300, 1000, 2048]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", LS)
@pytest.mark.parametrize("B,T,H,Dh", [(2, 1000, 2, 64), (1, 4099, 1, 128)])
def test_chunk_local_scan_kv_matches_oracle(dtype, L, B, T, H, Dh):
    _, xk, xv, g = prefill_inputs(B, T, H, Dh, dtype, gate_mean=2.0, gate_std=1.5, seed=T + L)
    fs = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV), final_state=fs, L=L)
    ratp.last_error()
    rk = oracle.scan(to64(xk), to64(g), L=L)
    rv = oracle.scan(to64(xv), to64(g), L=L)
    assert_close(hk, rk, dtype, "hk")
    assert_close(hv, rv, dtype, "hv")
    assert_close(fs[0], rk[:, -1], "f32", "final k state")
    assert_close(fs[1], rv[:, -1], "f32", "final v state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [16, 333])
def test_chunk_local_single_stream_matches_oracle(dtype, L):
    B, T, H, Dh = 2, 777, 3, 64
    _, x, _, g = prefill_inputs(B, T, H, Dh, dtype, gate_mean=1.0, gate_std=2.0, seed=L)
    fs = torch.zeros(B, H, Dh, dtype=torch.float32, device=DEV)
    h = ratp.scan_prefill(x.to(DEV), g.to(DEV), final_state=fs, L=L)
    ratp.last_error()
    r = oracle.scan(to64(x), to64(g), L=L)
    assert_close(h, r, dtype, "h")
    assert_close(fs, r[:, -1], "f32", "final state")


@pytest.mark.parametrize("L", [3, 128, 200])
def test_chunk_local_constant_gate_closed_form(L):
    B, T, H, Dh, c = 1, 1500, 1, 64, 0.9
    x = torch.ones(B, T, H, Dh, dtype=torch.float32, device=DEV)
    h = ratp.scan_prefill(x, torch.full_like(x, c), L=L)
    ratp.last_error()
    ref = 1.0 - c ** (np.arange(T) % L + 1.0)
    assert_close(h[0, :, 0, :], np.repeat(ref[:, None], Dh, axis=1), "f32", "1 - c^(t mod L + 1)")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_chunk_local_block_covering_sequence_is_full_scan_bit_exact(dtype):
    B, T, H, Dh = 2, 600, 2, 64
    _, xk, xv, g = prefill_inputs(B, T, H, Dh, dtype, seed=11)
    xk, xv, g = xk.to(DEV), xv.to(DEV), g.to(DEV)
    full = ratp.scan_prefill_kv(xk, xv, g)
    for L in (T, T + 1, 1 << 30):
        loc = ratp.scan_prefill_kv(xk, xv, g, L=L)
        assert bits_equal(loc[0], full[0]) and bits_equal(loc[1], full[1])
    ratp.last_error()


def test_chunk_local_negative_block_is_an_argument_error():
    x = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(RatpError) as e:
        ratp.scan_prefill_kv(x, x, x, L=-1)
    assert e.value.code == 1
    with pytest.raises(RatpError):
        ratp.KVCache(1, 1, 128, 16, 4, 0, L=-2)


@pytest.mark.parametrize("name,L", [("bf16_1p5b_T4096_D16", 16), ("bf16_long_T16384_D64_W128", 64),
                                    ("bf16_long_T16384_D64_W128", 1000)])
def test_chunk_local_full_size_sampled_channels(name, L):
    """The original RAT's block L = D on the full-size workloads, and a block
    that does not divide the scan chunk."""
    w = WORKLOADS[name]
    _, xk, xv, g = prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)
    fs = torch.zeros(2, w.B, w.H, w.Dh, dtype=torch.float32, device=DEV)
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV), final_state=fs, L=L)
    ratp.last_error()
    rng = np.random.default_rng(L)
    C = w.H * w.Dh
    cols = np.sort(rng.choice(C, 24, replace=False))
    xk2, xv2, g2 = (t.reshape(w.B, w.T, C)[:, :, cols] for t in (xk, xv, g))
    rk = oracle.scan(to64(xk2), to64(g2), L=L)
    rv = oracle.scan(to64(xv2), to64(g2), L=L)
    assert_close(hk.reshape(w.B, w.T, C)[:, :, cols], rk, w.dtype, "hk sampled")
    assert_close(hv.reshape(w.B, w.T, C)[:, :, cols], rv, w.dtype, "hv sampled")
    assert_close(fs[0].reshape(w.B, C)[:, cols], rk[:, -1], "f32", "final state sampled")


@pytest.mark.parametrize("B,T,n,H,D,W,L", [
    (2, 200, 70, 4, 4, 0, 16),      # blocks of 16 across the prefill boundary
    (2, 131, 40, 2, 16, 16, 16),    # L = D, the original RAT
    (1, 5, 30, 2, 3, 8, 7),
    (2, 256, 20, 2, 64, 128, 256),  # prefill ends on a block boundary
])
def test_chunk_local_prefill_pack_decode_matches_oracle(B, T, n, H, D, W, L):
    Dh = 128
    N = T + n
    q, xk, xv, g = prefill_inputs(B, N, H, Dh, "bf16", gate_mean=1.0, gate_std=2.0, seed=N + L)
    state = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    hk, hv = ratp.scan_prefill_kv(xk[:, :T].contiguous().to(DEV), xv[:, :T].contiguous().to(DEV),
                                  g[:, :T].contiguous().to(DEV), final_state=state, L=L)
    cache = ratp.KVCache(B, H, Dh, N, D, W, L=L)
    shadow = LayoutShadow(cache, N)
    cache.pack(hk, hv)
    ratp.last_error()
    shadow.prefill(hk, hv)
    shadow.check("after pack")

    rk = oracle.scan(to64(xk[:, :T]), to64(g[:, :T]), L=L)
    rv = oracle.scan(to64(xv[:, :T]), to64(g[:, :T]), L=L)
    oc = oracle.Cache(B, H, Dh, N, D, W, L=L)
    oc.pack(rk, rv, state=np.stack([rk[:, -1], rv[:, -1]]))
    for i in range(n):
        t = T + i
        args = [x[:, t].contiguous() for x in (q, xk, xv, g)]
        o = cache.decode_step(*[a.to(DEV) for a in args], state)
        ref = oc.decode_step(*[to64(a) for a in args])
        assert_close(o, ref, "bf16", "decode step %d (t=%d)" % (i, t))
        shadow.append(state)
        shadow.check("after decode step %d" % i)
    ratp.last_error()
    assert_close(state[0], oc.state[0], "f32", "final k state")
    assert_close(state[1], oc.state[1], "f32", "final v state")


def test_chunk_local_decode_consistent_with_gpu_prefill():
    """Decode outputs equal the GPU prefill attention over the chunk-local
    recurrence of the longer sequence."""
    B, T, n, H, Dh, D, W, L = 2, 250, 40, 4, 128, 4, 32, 16
    mask = [1, 0, 0, 0]
    N = T + n
    q, xk, xv, g = prefill_inputs(B, N, H, Dh, "bf16", seed=78)
    hk_all, hv_all = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV), L=L)
    o_all = ratp.dilated_attn_prefill(q.to(DEV), hk_all, hv_all, D, W, head_mask=mask)
    state = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    hk, hv = ratp.scan_prefill_kv(xk[:, :T].contiguous().to(DEV), xv[:, :T].contiguous().to(DEV),
                                  g[:, :T].contiguous().to(DEV), final_state=state, L=L)
    cache = ratp.KVCache(B, H, Dh, N, D, W, head_mask=mask, L=L)
    cache.pack(hk, hv)
    outs = []
    for i in range(n):
        t = T + i
        outs.append(cache.decode_step(*[x[:, t].contiguous().to(DEV) for x in (q, xk, xv, g)], state))
    ratp.last_error()
    got = torch.stack(outs, dim=1)
    err = (got.float() - o_all[:, T:].float()).abs()
    assert err.max().item() <= 3e-2 and err.mean().item() <= 3e-3
