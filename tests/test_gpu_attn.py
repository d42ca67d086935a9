"""GPU parity of dilated (+ windowed, + head-wise hybrid) prefill attention.

The tensor-core kernel (bf16, Dh 128) and the CUDA-core kernel (fp32/bf16,
Dh 64/128) are both compared with the fp64 oracle on the same seeded inputs.
Attention is tested as a call of its own (q, hk, hv drawn directly), and end
to end (scan + attention from q, x_k, x_v, g) at the full workload sizes on
sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import WORKLOADS, _binding, prefill_inputs
from parity import assert_close, bits_equal, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _qkv(B, T, H, Dh, dtype, seed, qscale=1.0):
    q, k, v, _ = prefill_inputs(B, T, H, Dh, dtype, seed=seed)
    if qscale != 1.0:
        q = (q.float() * qscale).to(q.dtype)
    return q, k, v


# (B, T, H, D, W, dense heads, q scale): several query tiles (128 rows), ragged
# tails, D = 1 (dense), D >= T (self only), windows shorter and longer than a
# tile, hybrid masks, and sharp softmaxes (q scale 4) that force O rescaling.
TC_CASES = [
    (1, 1, 1, 1, 0, (), 1.0),
    (1, 5, 2, 2, 0, (), 1.0),
    (1, 127, 1, 4, 0, (), 1.0),
    (1, 128, 1, 16, 0, (), 1.0),
    (2, 129, 2, 3, 3, (), 1.0),
    (1, 300, 2, 64, 128, (), 1.0),
    (1, 513, 1, 1, 0, (), 1.0),
    (1, 600, 1, 5, 7, (), 4.0),
    (1, 260, 1, 300, 0, (), 1.0),
    (1, 200, 1, 64, 1, (), 1.0),
    (1, 1000, 2, 16, 0, (0,), 1.0),
    (2, 700, 4, 4, 0, (0, 1), 4.0),
    (1, 1100, 2, 64, 128, (1,), 3.0),
    (1, 2049, 1, 16, 200, (), 2.0),
    # the most heads a launch takes, every seventh one dense
    (1, 130, 256, 2, 3, tuple(range(0, 256, 7)), 1.0),
]


@pytest.mark.parametrize("B,T,H,D,W,dense,qs", TC_CASES)
def test_tensor_core_attention_matches_oracle(B, T, H, D, W, dense, qs):
    q, k, v = _qkv(B, T, H, 128, "bf16", seed=T + D, qscale=qs)
    mask = [1 if h in dense else 0 for h in range(H)]
    o = ratp.dilated_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), D, W, head_mask=mask)
    ratp.last_error()
    ref = oracle.attention(to64(q), to64(k), to64(v), D, W, dense_mask=mask)
    assert_close(o, ref, "bf16", "tc attention")


def test_tensor_core_attention_output_only_16_byte_aligned():
    """An output view that starts 16 bytes into its buffer takes the 16-byte
    store path of the epilogue and gives the same values."""
    B, T, H, D, W = 1, 300, 2, 8, 16
    q, k, v = _qkv(B, T, H, 128, "bf16", seed=5)
    buf = torch.empty(B * T * H * 128 + 8, dtype=torch.bfloat16, device=DEV)
    o = buf[8:].view(B, T, H, 128)
    assert o.data_ptr() % 32 == 16
    ratp.dilated_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), D, W, out=o)
    ratp.last_error()
    ref = oracle.attention(to64(q), to64(k), to64(v), D, W)
    assert_close(o, ref, "bf16", "tc attention, 16-byte aligned output")
    o2 = ratp.dilated_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), D, W)
    assert bits_equal(o2, o)


SIMT_CASES = [
    ("f32", 64, 1, 256, 2, 4, 0, ()),        # the fp32 parity workload, full size
    ("f32", 64, 2, 300, 3, 3, 5, (1,)),
    ("f32", 128, 1, 150, 2, 1, 0, ()),
    ("bf16", 64, 2, 333, 2, 8, 16, (0,)),
    ("bf16", 128, 1, 257, 2, 16, 0, ()),
]


@pytest.mark.parametrize("dtype,Dh,B,T,H,D,W,dense", SIMT_CASES)
def test_cuda_core_attention_matches_oracle(dtype, Dh, B, T, H, D, W, dense):
    q, k, v = _qkv(B, T, H, Dh, dtype, seed=11)
    mask = [1 if h in dense else 0 for h in range(H)]
    o = ratp.dilated_attn_prefill_simt(q.to(DEV), k.to(DEV), v.to(DEV), D, W, head_mask=mask)
    ratp.last_error()
    ref = oracle.attention(to64(q), to64(k), to64(v), D, W, dense_mask=mask)
    assert_close(o, ref, dtype, "simt attention")


def test_dispatch_fp32_runs_cuda_core_kernel():
    q, k, v = _qkv(1, 100, 2, 64, "f32", seed=2)
    a = ratp.dilated_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), 4, 0)
    b = ratp.dilated_attn_prefill_simt(q.to(DEV), k.to(DEV), v.to(DEV), 4, 0)
    assert bits_equal(a, b)


@pytest.mark.parametrize("kernel", ["tc", "simt"])
def test_dilation_beyond_sequence_is_self_bit_exact(kernel):
    q, k, v = _qkv(2, 300, 2, 128, "bf16", seed=4)
    fn = ratp.dilated_attn_prefill if kernel == "tc" else ratp.dilated_attn_prefill_simt
    o = fn(q.to(DEV), k.to(DEV), v.to(DEV), 300, 0)
    ratp.last_error()
    assert bits_equal(o, v)


def test_f32_small_workload_end_to_end():
    """The fp32 single-layer workload: scan + attention from the raw inputs."""
    w = WORKLOADS["f32_small_T256_D4"]
    q, xk, xv, g = prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV))
    o = ratp.dilated_attn_prefill(q.to(DEV), hk, hv, w.D, w.W)
    ratp.last_error()
    rk, rv = oracle.scan(to64(xk), to64(g)), oracle.scan(to64(xv), to64(g))
    assert_close(hk, rk, "f32", "hk")
    ref = oracle.attention(to64(q), rk, rv, w.D, w.W)
    assert_close(o, ref, "f32", "o")


def _sample_rows(rng, B, T, heads, n):
    rows = []
    # always include the first/last query tile edges and random rows
    for t in (0, 1, 127, 128, T - 1):
        rows.append((int(rng.integers(B)), t, int(rng.integers(len(heads)))))
    while len(rows) < n:
        rows.append((int(rng.integers(B)), int(rng.integers(T)), int(rng.integers(len(heads)))))
    return np.array(rows, dtype=np.int64)


@pytest.mark.parametrize("name", ["bf16_1p5b_T4096_D16", "bf16_long_T16384_D64_W128",
                                  "bf16_hybrid_7p6b_T8192_D4"])
def test_full_size_end_to_end_sampled_rows(name):
    """Full workload in the launch configuration the benchmark times; the
    oracle recomputes sampled output rows from the raw inputs in fp64."""
    w = WORKLOADS[name]
    q, xk, xv, g = prefill_inputs(w.B, w.T, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)
    mask = w.dense_mask
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV))
    o = ratp.dilated_attn_prefill(q.to(DEV), hk, hv, w.D, w.W, head_mask=mask)
    ratp.last_error()
    rng = np.random.default_rng(1)
    heads = sorted(set(list(w.dense_heads) + [int(h) for h in rng.choice(w.H, 2, replace=False)]))
    sub = lambda t: t[:, :, heads, :]
    rk = oracle.scan(to64(sub(xk)), to64(sub(g)))
    rv = oracle.scan(to64(sub(xv)), to64(sub(g)))
    rows = _sample_rows(rng, w.B, w.T, heads, 160)
    ref = oracle.attention(to64(sub(q)), rk, rv, w.D, w.W,
                           dense_mask=[mask[h] for h in heads], rows=rows)
    o_cpu = o.cpu()
    got = torch.stack([o_cpu[b, t, heads[hi]] for b, t, hi in rows])
    assert_close(got, ref, "bf16", name)


@pytest.mark.parametrize("B,T,H", [(1, 0, 2), (0, 16, 2), (2, 16, 0)])
def test_empty_problem_launches_nothing(B, T, H):
    """An empty batch, sequence or head set is a no-op that succeeds."""
    q = torch.empty(B, T, H, 128, dtype=torch.bfloat16, device=DEV)
    o = ratp.dilated_attn_prefill(q, q, q, 4, 8)
    ratp.last_error()
    assert o.shape == q.shape


@pytest.mark.parametrize("Dh,dtype", [(128, "bf16"), (64, "bf16"), (64, "f32")])
@pytest.mark.parametrize("D", [1, 2, 3, 4, 16, 64, "T", "T+5"])
def test_small_shape_sweep(Dh, dtype, D):
    """Every combination of T in {1, 2, D-1, D, D+1, 257} and W in {0, 1, 3,
    D, 128} for one dilation (D = T and D = T + 5 taken per T): the bounds of
    the key-set split, the window and the ragged query tile."""
    n = 0
    for T in sorted({1, 2, 257} | ({D - 1, D, D + 1} if isinstance(D, int) else set()) - {0}):
        d = T if D == "T" else T + 5 if D == "T+5" else D
        for W in sorted({0, 1, 3, d, 128}):
            q, k, v = _qkv(1, T, 2, Dh, dtype, seed=1000 * T + 10 * W + d)
            o = ratp.dilated_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), d, W)
            ref = oracle.attention(to64(q), to64(k), to64(v), d, W)
            assert_close(o, ref, dtype, "T=%d D=%d W=%d Dh=%d" % (T, d, W, Dh))
            n += 1
    ratp.last_error()
    assert n >= 10


@pytest.mark.parametrize("B,T,H,D,W,dense", [(2, 700, 4, 4, 0, (0, 1)), (1, 1100, 2, 64, 128, (1,)),
                                             (1, 130, 256, 2, 3, tuple(range(0, 256, 7))),
                                             (4, 1024, 40, 4, 0, (0, 1))])
def test_mixed_launch_dynamic_and_static_dealing_agree_bitwise(B, T, H, D, W, dense):
    """A launch that mixes dense and dilated items deals them dynamically when
    given a workspace (the binding's default) and in fixed rounds without one
    (ratp_dilated_attn_prefill); every item is computed the same way whichever
    CTA takes it, so the outputs are bit-identical, and the static one matches
    the oracle.  The last case has more than 32 dilated (b, h), so its tail is
    interleaved."""
    q, k, v = (t.to(DEV) for t in _qkv(B, T, H, 128, "bf16", seed=5 * T + D, qscale=2.0))
    mask = [1 if h in dense else 0 for h in range(H)]
    o_dyn = ratp.dilated_attn_prefill(q, k, v, D, W, head_mask=mask)
    o_static = _binding._attn("ratp_dilated_attn_prefill", q, k, v, D, W, mask, None)
    ratp.last_error()
    assert torch.equal(o_dyn, o_static)
    if B * T * H <= 2 * 700 * 4:
        ref = oracle.attention(to64(q.cpu()), to64(k.cpu()), to64(v.cpu()), D, W, dense_mask=mask)
        assert_close(o_static, ref, "bf16", "static dealing")
