"""GPU parity of the fixed look-back recurrence (each token's state covers
the last L tokens up to itself) against the oracle's O(T * L) loop."""
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

# T spans sequences shorter than one block, block and chunk (256) edges and
# ragged tails; channels span one to 128 32-channel slabs.
SHAPES = [(1, 1, 1, 64), (2, 5, 1, 64), (1, 63, 1, 64), (1, 65, 2, 64), (2, 255, 1, 128),
          (1, 256, 1, 64), (1, 257, 2, 64), (3, 1000, 2, 64), (1, 4099, 1, 128), (1, 300, 32, 128)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [16, 32, 64])
@pytest.mark.parametrize("B,T,H,Dh", SHAPES)
def test_window_scan_matches_oracle(dtype, L, B, T, H, Dh):
    _, xk, xv, g = prefill_inputs(B, T, H, Dh, dtype, gate_mean=2.0, gate_std=1.5, seed=T + L)
    hk, hv = ratp.scan_prefill_kv_window(xk.to(DEV), xv.to(DEV), g.to(DEV), L)
    ratp.last_error()
    assert_close(hk, oracle.scan_window(to64(xk), to64(g), L), dtype, "hk")
    assert_close(hv, oracle.scan_window(to64(xv), to64(g), L), dtype, "hv")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_window_covering_sequence_matches_full_scan(dtype):
    """L >= T: every window reaches back to the first token, so the result is
    the full-sequence recurrence (compared with the chunked scan kernel)."""
    B, T, H, Dh = 2, 60, 2, 64
    _, xk, xv, g = prefill_inputs(B, T, H, Dh, dtype, seed=4)
    xk, xv, g = xk.to(DEV), xv.to(DEV), g.to(DEV)
    wk, wv = ratp.scan_prefill_kv_window(xk, xv, g, 64)
    fk, fv = ratp.scan_prefill_kv(xk, xv, g)
    ratp.last_error()
    assert_close(wk, to64(fk.cpu()), dtype, "hk vs full scan")
    assert_close(wv, to64(fv.cpu()), dtype, "hv vs full scan")


def test_window_constant_gate_closed_form():
    B, T, H, Dh, c, L = 1, 700, 1, 64, 0.9, 64
    x = torch.ones(B, T, H, Dh, dtype=torch.float32, device=DEV)
    hk, _ = ratp.scan_prefill_kv_window(x, x, torch.full_like(x, c), L)
    ratp.last_error()
    ref = 1.0 - c ** np.minimum(np.arange(T) + 1.0, L)
    assert_close(hk[0, :, 0, :], np.repeat(ref[:, None], Dh, axis=1), "f32", "1 - c^min(t+1, L)")


def test_window_gate_zero_is_identity_bit_exact():
    _, x, _, _ = prefill_inputs(2, 517, 2, 64, "bf16", seed=9)
    xd = x.to(DEV)
    hk, hv = ratp.scan_prefill_kv_window(xd, xd, torch.zeros_like(xd), 32)
    ratp.last_error()
    assert bits_equal(hk, xd) and bits_equal(hv, xd)


def test_window_errors_and_empty():
    x = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16, device=DEV)
    for L, code in ((8, 7), (128, 7), (0, 1), (-3, 1)):
        with pytest.raises(RatpError) as e:
            ratp.scan_prefill_kv_window(x, x, x, L)
        assert e.value.code == code
    empty = torch.empty(2, 0, 1, 64, dtype=torch.bfloat16, device=DEV)
    ratp.scan_prefill_kv_window(empty, empty, empty, 64)
    ratp.last_error()


def test_window_full_size_sampled_channels():
    """L* = 64 on the long-context T = 16K layer, sampled channels."""
    w = WORKLOADS["bf16_long_T16384_D64_W128"]
    _, xk, xv, g = prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)
    hk, hv = ratp.scan_prefill_kv_window(xk.to(DEV), xv.to(DEV), g.to(DEV), 64)
    ratp.last_error()
    rng = np.random.default_rng(64)
    C = w.H * w.Dh
    cols = np.sort(rng.choice(C, 16, replace=False))
    xk2, xv2, g2 = (t.reshape(w.B, w.T, C)[:, :, cols] for t in (xk, xv, g))
    assert_close(hk.reshape(w.B, w.T, C)[:, :, cols], oracle.scan_window(to64(xk2), to64(g2), 64),
                 w.dtype, "hk sampled")
    assert_close(hv.reshape(w.B, w.T, C)[:, :, cols], oracle.scan_window(to64(xv2), to64(g2), 64),
                 w.dtype, "hv sampled")


@pytest.mark.parametrize("B,T,n,H,D,W,L,dense", [
    (2, 200, 40, 2, 4, 0, 64, ()),        # the window crosses from prefill into decode
    (2, 40, 30, 2, 16, 16, 64, (0,)),     # prefill shorter than the window
    (1, 300, 20, 4, 64, 128, 16, (1,)),
    (2, 96, 70, 2, 3, 8, 32, ()),         # decode runs past a full window
])
def test_window_prefill_pack_decode_matches_oracle(B, T, n, H, D, W, L, dense):
    """Look-back prefill of T tokens, hand-off of the cache and of the last L
    inputs, then n decode steps: every step equals the oracle's prefill
    attention over the look-back recurrence of all T + n tokens."""
    Dh = 128
    N = T + n
    mask = [1 if h in dense else 0 for h in range(H)]
    q, xk, xv, g = prefill_inputs(B, N, H, Dh, "bf16", gate_mean=1.0, gate_std=2.0, seed=N + L)
    pre = [x[:, :T].contiguous().to(DEV) for x in (xk, xv, g)]
    hk, hv = ratp.scan_prefill_kv_window(*pre, L)
    cache = ratp.KVCache(B, H, Dh, N, D, W, head_mask=mask)
    shadow = LayoutShadow(cache, N, mask)
    cache.attach_window(L)
    cache.pack(hk, hv)
    cache.pack_inputs(*pre)
    shadow.prefill(hk, hv)
    shadow.check("after pack")
    state = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    outs = []
    for i in range(n):
        outs.append(cache.decode_step(*[x[:, T + i].contiguous().to(DEV) for x in (q, xk, xv, g)],
                                      state))
        shadow.append(state)
        shadow.check("after decode step %d" % i)
    ratp.last_error()
    rk = oracle.scan_window(to64(xk), to64(g), L)
    rv = oracle.scan_window(to64(xv), to64(g), L)
    ref = oracle.attention(to64(q), rk, rv, D, W, dense_mask=mask)
    for i in range(n):
        assert_close(outs[i], ref[:, T + i], "bf16", "decode step %d" % i)
    # the state holds the last recurrent key/value
    assert_close(state[0], rk[:, N - 1], "f32", "final k state")
    assert cache.lengths().cpu().tolist() == [N] * B


def test_window_decode_argument_errors():
    cache = ratp.KVCache(1, 1, 128, 16, 4, 0)
    with pytest.raises(RatpError):
        cache.attach_window(300)
    cache.attach_window(8)
    with pytest.raises(RatpError):                 # chunk-local and look-back exclude each other
        ratp._binding._check("set", ratp.load_library().ratp_cache_set_chunk_local(
            ratp._binding.ctypes.byref(cache.c), 4))
    x = torch.zeros(1, 17, 1, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(RatpError) as e:            # T > T_max
        cache.pack_inputs(x, x, x)
    assert e.value.code == 4
