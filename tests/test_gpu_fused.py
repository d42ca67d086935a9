"""GPU parity of the fused prefill (recurrence of both streams + dilated,
windowed, head-wise hybrid attention in one launch) against the oracle.

The oracle runs the plain definitions in fp64: the sequential recurrence of
each stream (oracle.scan) and softmax attention over the enumerated key sets
(oracle.attention), on the same seeded inputs.  hk, hv, the final state and o
are compared element by element on shapes that span several 256-token scan
chunks and 128-query tiles, ragged tails, D = 1, D >= T, windows shorter and
longer than a key tile and dense heads; at the full workload sizes on sampled
rows and channels.
"""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, _binding, prefill_inputs
from recurrence_augmented_dilated_chunked_b200._binding import RatpError
from parity import assert_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (B, T, H, D, W, dense heads, gate mean, gate std)
CASES = [
    (1, 1, 1, 4, 0, (), 2.0, 1.5),
    (1, 200, 2, 4, 0, (), 2.0, 1.5),
    (2, 256, 1, 16, 0, (), 2.0, 1.5),
    (1, 257, 2, 3, 3, (), 1.0, 2.0),
    (1, 700, 2, 64, 128, (), 2.0, 1.5),
    (2, 1000, 3, 4, 0, (0,), 1.0, 2.0),
    (1, 513, 2, 1, 0, (), 2.0, 1.5),
    (1, 600, 1, 700, 0, (), 2.0, 1.5),
    (1, 1030, 2, 5, 300, (1,), 1.0, 2.0),
    (1, 2100, 2, 16, 0, (), 2.0, 1.5),
    (3, 640, 4, 4, 64, (0, 3), 1.0, 2.0),
]


def _run(q, xk, xv, g, D, W, mask):
    B, T, H, Dh = q.shape
    fs = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    # h_k/h_v start as NaN: a key or value row read before its recurrence
    # unit is scanned (even one whose softmax weight is 0) would show in o
    hk = torch.full((B, T, H, Dh), float("nan"), dtype=q.dtype, device=DEV)
    hv = torch.full_like(hk, float("nan"))
    o, hk, hv = ratp.prefill_fused(q.to(DEV), xk.to(DEV), xv.to(DEV), g.to(DEV), D, W, head_mask=mask,
                                   hk=hk, hv=hv, final_state=fs)
    ratp.last_error()
    return o, hk, hv, fs


@pytest.mark.parametrize("B,T,H,D,W,dense,gm,gs", CASES)
def test_fused_prefill_matches_oracle(B, T, H, D, W, dense, gm, gs):
    mask = [1 if h in dense else 0 for h in range(H)]
    q, xk, xv, g = prefill_inputs(B, T, H, 128, "bf16", gm, gs, seed=T + D)
    o, hk, hv, fs = _run(q, xk, xv, g, D, W, mask)
    rk = oracle.scan(to64(xk), to64(g))
    rv = oracle.scan(to64(xv), to64(g))
    assert_close(hk, rk, "bf16", "hk")
    assert_close(hv, rv, "bf16", "hv")
    assert_close(fs[0], rk[:, -1], "f32", "final k state")
    assert_close(fs[1], rv[:, -1], "f32", "final v state")
    ref = oracle.attention(to64(q), rk, rv, D, W, dense_mask=mask)
    assert_close(o, ref, "bf16", "o")


def test_fused_prefill_agrees_with_the_two_kernel_path():
    """Same layer through ratp_scan_prefill_kv + ratp_dilated_attn_prefill:
    equal to rounding (the recurrence is associated differently)."""
    B, T, H, D, W = 2, 1500, 4, 16, 32
    mask = [1, 0, 0, 0]
    q, xk, xv, g = (t.to(DEV) for t in prefill_inputs(B, T, H, 128, "bf16", seed=11))
    o, hk, hv, _ = _run(q, xk, xv, g, D, W, mask)
    hk2, hv2 = ratp.scan_prefill_kv(xk, xv, g)
    o2 = ratp.dilated_attn_prefill(q, hk2, hv2, D, W, head_mask=mask)
    ratp.last_error()
    assert_close(hk, to64(hk2), "bf16", "hk")
    assert_close(o, to64(o2), "bf16", "o")


@pytest.mark.parametrize("name", ["bf16_1p5b_T4096_D16", "bf16_long_T16384_D64_W128",
                                  "bf16_hybrid_7p6b_T8192_D4"])
def test_fused_full_size_sampled(name):
    """The full workload in the launch configuration the benchmark times; the
    oracle recomputes sampled heads and output rows from the raw inputs."""
    w = WORKLOADS[name]
    q, xk, xv, g = prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)
    mask = w.dense_mask
    o, hk, hv, fs = _run(q, xk, xv, g, w.D, w.W, mask)
    rng = np.random.default_rng(3)
    heads = sorted(set(list(w.dense_heads) + [int(h) for h in rng.choice(w.H, 2, replace=False)]))
    sub = lambda t: t[:, :, heads, :]
    rk = oracle.scan(to64(sub(xk)), to64(sub(g)))
    rv = oracle.scan(to64(sub(xv)), to64(sub(g)))
    assert_close(hk.cpu()[:, :, heads], rk, "bf16", "hk sampled heads")
    assert_close(fs[1].cpu()[:, heads], rv[:, -1], "f32", "final v state sampled heads")
    rows = [(int(rng.integers(w.B)), t, int(rng.integers(len(heads)))) for t in (0, 1, 255, 256, w.T - 1)]
    while len(rows) < 160:
        rows.append((int(rng.integers(w.B)), int(rng.integers(w.T)), int(rng.integers(len(heads)))))
    rows = np.array(rows, dtype=np.int64)
    ref = oracle.attention(to64(sub(q)), rk, rv, w.D, w.W, dense_mask=[mask[h] for h in heads], rows=rows)
    o_cpu = o.cpu()
    got = torch.stack([o_cpu[b, t, heads[hi]] for b, t, hi in rows])
    assert_close(got, ref, "bf16", name)


def test_fused_graph_replays_with_new_inputs():
    """Captured once, replayed with new inputs: every replay's descriptors
    and flags carry a fresh tag kept in the workspace."""
    B, T, H, D, W = 1, 3000, 2, 16, 16
    ins = [prefill_inputs(B, T, H, 128, "bf16", 1.0, 2.0, seed=70 + i) for i in range(2)]
    q, xk, xv, g = (t.to(DEV) for t in ins[0])
    hk, hv, o = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.zeros(ratp.prefill_fused_workspace(B, T, H, 128, DEV).numel(), dtype=torch.uint8, device=DEV)
    call = lambda: ratp.prefill_fused(q, xk, xv, g, D, W, hk=hk, hv=hv, out=o, workspace=ws)
    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for i in (1, 0, 1):
        for dst, src in zip((q, xk, xv, g), ins[i]):
            dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        ratp.last_error()
        rk = oracle.scan(to64(ins[i][1]), to64(ins[i][3]))
        rv = oracle.scan(to64(ins[i][2]), to64(ins[i][3]))
        assert_close(o, oracle.attention(to64(ins[i][0]), rk, rv, D, W), "bf16", "replay %d" % i)
    del graph


def test_fused_argument_errors():
    x = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(RatpError) as e:
        ratp.prefill_fused(x, x, x, x, 0)
    assert e.value.code == 1
    x64 = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(RatpError) as e:
        ratp.prefill_fused(x64, x64, x64, x64, 4)
    assert e.value.code == 7
    small = torch.zeros(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(RatpError) as e:
        ratp.prefill_fused(x, x, x, x, 4, workspace=small)
    assert e.value.code == 4
    empty = torch.empty(2, 0, 1, 128, dtype=torch.bfloat16, device=DEV)
    ratp.prefill_fused(empty, empty, empty, empty, 4)
    ratp.last_error()


def test_fused_missing_chunk_flag_times_out_then_recovers():
    B, T, H, D = 1, 1000, 2, 4
    q, xk, xv, g = (t.to(DEV) for t in prefill_inputs(B, T, H, 128, "bf16", seed=23))
    ratp.last_error()
    ratp.debug_fault(_binding.FAULT_SPIN_LIMIT, 20_000_000)
    ratp.debug_fault(_binding.FAULT_FUSED_DROP_CHUNK, 1)    # b 0, channels 0..63, positions 256..511
    try:
        ratp.prefill_fused(q, xk, xv, g, D, 0)
        with pytest.raises(RatpError, match="TIMEOUT"):
            ratp.last_error()
    finally:
        ratp.debug_fault(_binding.FAULT_NONE)
    o, hk, hv = ratp.prefill_fused(q, xk, xv, g, D, 0)
    ratp.last_error()
    rk, rv = oracle.scan(to64(xk.cpu()), to64(g.cpu())), oracle.scan(to64(xv.cpu()), to64(g.cpu()))
    assert_close(o, oracle.attention(to64(q.cpu()), rk, rv, D, 0), "bf16", "after recovery")
