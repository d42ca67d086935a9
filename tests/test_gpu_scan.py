"""GPU parity of the prefill scan (forget-gate recurrence) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, prefill_inputs
from parity import assert_close, bits_equal, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"

# T spans several chunks (256 tokens for bf16, 128 for fp32) and ragged tails;
# the largest case has 4096 channels per token (64 slabs of 64).
SHAPES = [(1, 1, 1, 64), (2, 5, 1, 64), (1, 63, 2, 64), (1, 64, 1, 64), (2, 127, 1, 128),
          (1, 128, 1, 64), (1, 129, 2, 64), (1, 255, 1, 64), (1, 256, 2, 64), (2, 257, 1, 128),
          (3, 1000, 2, 64), (1, 4099, 4, 128), (2, 8191, 1, 64), (1, 300, 32, 128)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,H,Dh", SHAPES)
def test_scan_kv_matches_oracle(dtype, B, T, H, Dh):
    _, xk, xv, g = prefill_inputs(B, T, H, Dh, dtype, gate_mean=2.0, gate_std=1.5, seed=T)
    fs = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV), final_state=fs)
    ratp.last_error()
    rk = oracle.scan(to64(xk), to64(g))
    rv = oracle.scan(to64(xv), to64(g))
    assert_close(hk, rk, dtype, "hk")
    assert_close(hv, rv, dtype, "hv")
    # the fp32 final state is compared at fp32 tolerance in both dtypes
    assert_close(fs[0], rk[:, -1], "f32", "final k state")
    assert_close(fs[1], rv[:, -1], "f32", "final v state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_scan_single_stream_matches_oracle(dtype):
    B, T, H, Dh = 2, 777, 3, 64
    _, x, _, g = prefill_inputs(B, T, H, Dh, dtype, gate_mean=1.0, gate_std=2.0, seed=5)
    fs = torch.zeros(B, H, Dh, dtype=torch.float32, device=DEV)
    h = ratp.scan_prefill(x.to(DEV), g.to(DEV), final_state=fs)
    ratp.last_error()
    r = oracle.scan(to64(x), to64(g))
    assert_close(h, r, dtype, "h")
    assert_close(fs, r[:, -1], "f32", "final state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_scan_gate_zero_is_identity_bit_exact(dtype):
    _, x, _, _ = prefill_inputs(2, 517, 2, 64, dtype, seed=9)
    xd = x.to(DEV)
    h = ratp.scan_prefill(xd, torch.zeros_like(xd))
    ratp.last_error()
    assert bits_equal(h, xd)


def test_scan_constant_gate_closed_form():
    B, T, H, Dh, c = 1, 2000, 1, 64, 0.9
    x = torch.ones(B, T, H, Dh, dtype=torch.float32, device=DEV)
    h = ratp.scan_prefill(x, torch.full_like(x, c))
    ratp.last_error()
    ref = 1.0 - c ** (np.arange(T) + 1.0)
    assert_close(h[0, :, 0, :], np.repeat(ref[:, None], Dh, axis=1), "f32", "1 - c^(t+1)")


def test_scan_repeated_calls_reuse_workspace():
    B, T, H, Dh = 2, 3000, 2, 128
    _, xk, xv, g = prefill_inputs(B, T, H, Dh, "bf16", seed=3)
    xk, xv, g = xk.to(DEV), xv.to(DEV), g.to(DEV)
    first = ratp.scan_prefill_kv(xk, xv, g)
    for _ in range(3):
        again = ratp.scan_prefill_kv(xk, xv, g)
        assert bits_equal(again[0], first[0]) and bits_equal(again[1], first[1])
    ratp.last_error()


@pytest.mark.parametrize("name", ["bf16_1p5b_T4096_D16", "bf16_long_T16384_D64_W128",
                                  "bf16_hybrid_7p6b_T8192_D4"])
def test_scan_full_size_sampled_channels(name):
    w = WORKLOADS[name]
    _, xk, xv, g = prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)
    fs = torch.zeros(2, w.B, w.H, w.Dh, dtype=torch.float32, device=DEV)
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV), final_state=fs)
    ratp.last_error()
    rng = np.random.default_rng(0)
    C = w.H * w.Dh
    cols = np.sort(rng.choice(C, 24, replace=False))
    xk2, xv2, g2 = (t.reshape(w.B, w.T, C)[:, :, cols] for t in (xk, xv, g))
    rk = oracle.scan(to64(xk2), to64(g2))
    rv = oracle.scan(to64(xv2), to64(g2))
    assert_close(hk.reshape(w.B, w.T, C)[:, :, cols], rk, w.dtype, "hk sampled")
    assert_close(hv.reshape(w.B, w.T, C)[:, :, cols], rv, w.dtype, "hv sampled")
    assert_close(fs[0].reshape(w.B, C)[:, cols], rk[:, -1], "f32", "final state sampled")


@pytest.mark.parametrize("B,T", [(1, 0), (0, 32)])
def test_scan_empty_sequence_is_a_no_op(B, T):
    x = torch.empty(B, T, 2, 64, dtype=torch.bfloat16, device=DEV)
    hk, hv = ratp.scan_prefill_kv(x, x, x)
    ratp.last_error()
    assert hk.shape == x.shape and hv.shape == x.shape


def test_scan_graph_replays_with_new_inputs():
    """A scan captured once in a CUDA graph and replayed with new inputs in
    its static buffers matches the oracle on every replay: each replay's
    chunk descriptors carry a fresh tag, so no look-back accepts a
    predecessor's state from the previous replay."""
    B, T, H, Dh = 2, 6000, 4, 128
    x_in = [prefill_inputs(B, T, H, Dh, "bf16", gate_mean=1.0, gate_std=2.0, seed=40 + i)[1:]
            for i in range(3)]
    xk, xv, g = (t.to(DEV) for t in x_in[0])
    hk, hv = torch.empty_like(xk), torch.empty_like(xv)
    fs = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    ws = torch.zeros(ratp.scan_workspace(B, T, H, Dh, xk.dtype, DEV).numel(), dtype=torch.uint8,
                     device=DEV)
    ratp.scan_prefill_kv(xk, xv, g, hk=hk, hv=hv, final_state=fs, workspace=ws)   # warm-up
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ratp.scan_prefill_kv(xk, xv, g, hk=hk, hv=hv, final_state=fs, workspace=ws)
    for i in (1, 2, 0, 1):
        for dst, src in zip((xk, xv, g), x_in[i]):
            dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        ratp.last_error()
        ref_k, ref_v = ratp.scan_prefill_kv(xk, xv, g)
        assert bits_equal(hk, ref_k) and bits_equal(hv, ref_v), "replay with inputs %d" % i
        rk = oracle.scan(to64(x_in[i][0]), to64(x_in[i][2]))
        assert_close(hk, rk, "bf16", "replay with inputs %d" % i)
        assert_close(fs[0], rk[:, -1], "f32", "final k state, replay with inputs %d" % i)
    del graph


def test_scan_on_two_unordered_streams():
    """Scans of one shape issued on two streams with no order between them
    use separate workspaces (the binding keeps one per stream) and both match
    the oracle."""
    B, T, H, Dh = 2, 8000, 8, 128
    ins = [[t.to(DEV) for t in prefill_inputs(B, T, H, Dh, "bf16", seed=60 + i)[1:]] for i in range(2)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for _ in range(3):
        for s, (xk, xv, g) in zip(streams, ins):
            with torch.cuda.stream(s):
                outs.append(ratp.scan_prefill_kv(xk, xv, g))
    torch.cuda.synchronize()
    ratp.last_error()
    for i, (xk, xv, g) in enumerate(ins):
        rk = oracle.scan(to64(xk), to64(g))
        rv = oracle.scan(to64(xv), to64(g))
        for hk, hv in outs[i::2]:
            assert_close(hk, rk, "bf16", "stream %d hk" % i)
            assert_close(hv, rv, "bf16", "stream %d hv" % i)
