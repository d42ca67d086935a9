"""A layer with more than 2^31 elements per tensor (B=5, T=65536, H=64, Dh=128:
2.7e9 elements, 5.4 GB each in bf16): every offset of the scan and of the
attention must be computed in 64 bits.  Inputs are drawn on the GPU (seeded);
sampled channels and query rows are checked against the oracle, which reads
the same values copied to the host.
"""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from parity import assert_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
B, T, H, DH = 5, 65536, 64, 128
D, W = 64, 128


@pytest.fixture(scope="module")
def layer():
    assert B * T * H * DH > 2 ** 31
    gen = torch.Generator(DEV).manual_seed(7)
    shape = (B, T, H, DH)
    q = torch.randn(shape, generator=gen, device=DEV, dtype=torch.float32).to(torch.bfloat16)
    xk = torch.randn(shape, generator=gen, device=DEV, dtype=torch.float32).to(torch.bfloat16)
    xv = torch.randn(shape, generator=gen, device=DEV, dtype=torch.float32).to(torch.bfloat16)
    z = torch.randn(shape, generator=gen, device=DEV, dtype=torch.float32)
    g = torch.sigmoid(z * 1.5 + 2.0).to(torch.bfloat16)
    del z
    hk, hv = ratp.scan_prefill_kv(xk, xv, g)
    o = ratp.dilated_attn_prefill(q, hk, hv, D, W)
    ratp.last_error()
    yield q, xk, xv, g, hk, hv, o
    del q, xk, xv, g, hk, hv, o
    torch.cuda.empty_cache()


def test_scan_beyond_2_pow_31_elements(layer):
    _, xk, xv, g, hk, hv, _ = layer
    # every element of sequence 4 lies past element 2^31 (byte 2^32)
    for b, h, c in [(0, 0, 0), (4, 63, 127), (4, 40, 5), (2, 63, 64)]:
        for x, hx in ((xk, hk), (xv, hv)):
            xs = x[b, :, h, c].reshape(1, T, 1).cpu()
            gs = g[b, :, h, c].reshape(1, T, 1).cpu()
            ref = oracle.scan(to64(xs), to64(gs))
            assert_close(hx[b, :, h, c].reshape(1, T, 1), ref, "bf16", "h at b=%d h=%d c=%d" % (b, h, c))


def test_attention_beyond_2_pow_31_elements(layer):
    q, _, _, _, hk, hv, o = layer
    rng = np.random.default_rng(3)
    for b, h in [(4, 63), (0, 0), (4, 31)]:
        ts = np.concatenate([[0, 63, 64, 127, 128, T - 1], rng.integers(0, T, 26)])
        qs, ks, vs = (x[b, :, h].reshape(1, T, 1, DH).cpu() for x in (q, hk, hv))
        rows = np.stack([np.zeros_like(ts), ts, np.zeros_like(ts)], 1)
        ref = oracle.attention(to64(qs), to64(ks), to64(vs), D, W, rows=rows)
        got = o[b, torch.as_tensor(ts, device=DEV), h]
        assert_close(got, ref, "bf16", "o rows at b=%d h=%d" % (b, h))
