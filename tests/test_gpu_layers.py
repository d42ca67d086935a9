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


def test_layer_stack_full_size_sampled():
    """The 24-layer layer-wise hybrid at full size (dense layers 0 and 12, the
    others D = 64 with W = 128; B = 16, H = 16, 32K-token contexts): two
    token steps through one CUDA graph, checked on sampled sequences of a
    dense and a dilated layer against the oracle, which reads the same cache
    contents."""
    n_layers, dense_layers, Bf, Hf, ctx, steps = 24, (0, 12), 16, 16, 32768, 2
    gen = torch.Generator(DEV).manual_seed(11)
    q, xk, xv, g = (x.to(DEV) for x in
                    ratp.decode_inputs(steps, Bf, Hf, DH, "bf16", 2.0, 1.5, seed=12))
    layers = []
    for li in range(n_layers):
        D, W = (1, 0) if li in dense_layers else (64, 128)
        cache = ratp.KVCache(Bf, Hf, DH, ctx + steps, D, W)
        for which in ("k", "v"):
            rows = cache.dil_rows(which)
            rows.copy_(torch.randn(rows.shape, generator=gen, device=DEV))
            if W:
                ring = cache.ring(which)
                ring.copy_(torch.randn(ring.shape, generator=gen, device=DEV))
        if W:
            # a dilated position inside the last W holds one value in both
            # places, as after a prefill (the ring row repeats the slot)
            for h in range(Hf):
                off, _ = cache.head_rows(h)
                for pos in range(ctx - W, ctx):
                    if pos % D == D - 1:
                        for which in ("k", "v"):
                            cache.ring(which)[:, h, pos % W] = cache.dil_rows(which)[:, off + pos // D]
        cache.lengths().fill_(ctx)
        state = torch.randn(2, Bf, Hf, DH, generator=gen, device=DEV)
        layers.append((cache, state, state.clone(), torch.empty(steps, Bf, Hf, DH, dtype=torch.bfloat16,
                                                                device=DEV), D, W))
    # host copies of what the oracle reads (sampled sequences), taken before any step runs
    bs = torch.tensor([0, 13], device=DEV)
    snap = {li: (layers[li][0].dil_rows("k")[bs].cpu(), layers[li][0].dil_rows("v")[bs].cpu(),
                 None if layers[li][5] == 0 else layers[li][0].ring("k")[bs].cpu(),
                 None if layers[li][5] == 0 else layers[li][0].ring("v")[bs].cpu(),
                 layers[li][2][:, bs].cpu()) for li in (0, 1, 12, 23)}
    buf = [torch.empty(Bf, Hf, DH, dtype=torch.bfloat16, device=DEV) for _ in range(4)]

    def token_step(i):
        ratp.decode_step_layers([(c, buf[0], buf[1], buf[2], buf[3], st, o[i]) for c, st, _, o, _, _ in layers])

    for k, x in enumerate((q, xk, xv, g)):
        buf[k].copy_(x[0])
    token_step(0)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        token_step(1)
    for k, x in enumerate((q, xk, xv, g)):
        buf[k].copy_(x[1])
    graph.replay()
    torch.cuda.synchronize()
    ratp.last_error()
    del graph
    for li, (kc, vc, kw, vw, st0) in snap.items():
        cache, _, _, outs, D, W = layers[li]
        assert cache.lengths().cpu().tolist() == [ctx + steps] * Bf
        for j, b in enumerate((0, 13)):
            oc = oracle.Cache(1, Hf, DH, ctx + steps, D, W)
            oc.Kc[:] = to64(kc[j])
            oc.Vc[:] = to64(vc[j])
            if W:
                oc.Kw[:] = to64(kw[j]).reshape(-1, DH)
                oc.Vw[:] = to64(vw[j]).reshape(-1, DH)
            oc.len[:] = ctx
            oc.state[:] = to64(st0[:, j:j + 1])
            for i in range(steps):
                ref = oc.decode_step(*[to64(x[i, b:b + 1].cpu()) for x in (q, xk, xv, g)])
                assert_close(outs[i, b:b + 1], ref, "bf16", "layer %d (D=%d) b=%d step %d" % (li, D, b, i))
