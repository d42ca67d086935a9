"""GPU parity of the multi-layer decode token step (layer-wise hybrid: each
layer has its own cache, so its own D, window, head mask and recurrence)
against the oracle, with the whole token step captured in one CUDA graph.
"""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import prefill_inputs
from parity import assert_close, bits_equal, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"

B, H, DH, T, N_STEPS = 2, 4, 128, 100, 24
# (D, W, head_mask, chunk-local L): a dense input layer, a windowed head-wise
# hybrid, a chunk-local dilated layer (the original RAT, L = D), a dense
# middle layer and a long-stride windowed layer
LAYERS = [(1, 0, None, 0), (4, 8, [1, 0, 0, 0], 0), (16, 0, None, 16), (1, 0, None, 0),
          (64, 16, None, 0)]


def _build(seed0):
    """Per layer: GPU cache + state after a T-token prefill, the oracle's
    twin, and the layer's decode inputs for N_STEPS tokens."""
    N = T + N_STEPS
    out = []
    for li, (D, W, mask, L) in enumerate(LAYERS):
        q, xk, xv, g = prefill_inputs(B, N, H, DH, "bf16", gate_mean=1.0, gate_std=2.0, seed=seed0 + li)
        state = torch.zeros(2, B, H, DH, dtype=torch.float32, device=DEV)
        hk, hv = ratp.scan_prefill_kv(xk[:, :T].contiguous().to(DEV), xv[:, :T].contiguous().to(DEV),
                                      g[:, :T].contiguous().to(DEV), final_state=state, L=L)
        cache = ratp.KVCache(B, H, DH, N, D, W, head_mask=mask, L=L)
        cache.pack(hk, hv)
        rk = oracle.scan(to64(xk[:, :T]), to64(g[:, :T]), L=L)
        rv = oracle.scan(to64(xv[:, :T]), to64(g[:, :T]), L=L)
        oc = oracle.Cache(B, H, DH, N, D, W, dense_mask=mask, L=L)
        oc.pack(rk, rv, state=np.stack([rk[:, -1], rv[:, -1]]))
        steps = [x[:, T:].contiguous() for x in (q, xk, xv, g)]   # [B, N_STEPS, H, DH]
        out.append((cache, state, oc, steps))
    return out


def test_layer_stack_decode_graph_matches_oracle():
    layers = _build(seed0=500)
    # static per-layer step buffers, read by the captured token step
    bufs = [[torch.empty(B, H, DH, dtype=torch.bfloat16, device=DEV) for _ in range(5)]
            for _ in LAYERS]

    def token_step():
        ratp.decode_step_layers([(c, b[0], b[1], b[2], b[3], st, b[4])
                                 for (c, st, _, _), b in zip(layers, bufs)])

    def load(i):
        for (_, _, _, steps), b in zip(layers, bufs):
            for k in range(4):
                b[k].copy_(steps[k][:, i].to(DEV))

    # step 0 eagerly (also warms the kernels), the rest by graph replay
    load(0)
    token_step()
    torch.cuda.synchronize()
    outs = [[b[4].clone()] for b in bufs]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):     # records the launches; runs nothing
        token_step()
    for i in range(1, N_STEPS):
        load(i)
        graph.replay()
        for li, b in enumerate(bufs):
            outs[li].append(b[4].clone())
    torch.cuda.synchronize()
    ratp.last_error()
    for li, ((cache, state, oc, steps), (D, W, mask, L)) in enumerate(zip(layers, LAYERS)):
        for i in range(N_STEPS):
            ref = oc.decode_step(*[to64(x[:, i]) for x in steps])
            assert_close(outs[li][i], ref, "bf16", "layer %d (D=%d W=%d L=%d) step %d" % (li, D, W, L, i))
        assert cache.lengths().cpu().tolist() == [T + N_STEPS] * B
        assert_close(state[0], oc.state[0], "f32", "layer %d final k state" % li)
    del graph


def test_layer_stack_equals_per_layer_calls_bit_exact():
    a = _build(seed0=900)
    b = _build(seed0=900)
    for i in range(6):
        ins = [[x[:, i].contiguous().to(DEV) for x in steps] for (_, _, _, steps) in a]
        oa = [torch.empty(B, H, DH, dtype=torch.bfloat16, device=DEV) for _ in LAYERS]
        ob = [torch.empty_like(t) for t in oa]
        ratp.decode_step_layers([(c, *x, st, o) for (c, st, _, _), x, o in zip(a, ins, oa)])
        for (c, st, _, _), x, o in zip(b, ins, ob):
            c.decode_step(*x, st, out=o)
        for li in range(len(LAYERS)):
            assert bits_equal(oa[li], ob[li]), "layer %d step %d" % (li, i)
    ratp.last_error()
    for (ca, sa, _, _), (cb, sb, _, _) in zip(a, b):
        assert bits_equal(sa, sb)
        assert bits_equal(ca.lengths(), cb.lengths())
