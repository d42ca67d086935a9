"""GPU parity of the D-compressed cache and the fused decode step.

* layout: after the prefill hand-off and after every decode step, the whole
  dilated and ring regions of the GPU cache equal, bit for bit, the oracle's
  pack of the GPU's own recurrent keys/values (the oracle's index map and
  position rule; ``tests/cache_layout.py``);
* numerics: decode outputs match the oracle's literal decode step (itself
  pinned to prefill attention) on the same seeded inputs;
* the decode-from-32K-context and hybrid 7.6B-like workloads at full size,
  compared on sampled sequences.
"""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_chunked_b200 as ratp
from recurrence_augmented_dilated_chunked_b200 import (WORKLOADS, decode_context, decode_inputs,
                                                       prefill_inputs)
from recurrence_augmented_dilated_chunked_b200._binding import RatpError
from parity import assert_close, to64
from cache_layout import LayoutShadow

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("B,T,n,H,D,W,dense,Dh", [
    (2, 200, 70, 4, 4, 0, (0,), 128),
    (2, 131, 40, 2, 16, 16, (), 128),
    (1, 5, 30, 2, 3, 8, (1,), 128),
    (3, 300, 20, 2, 64, 128, (), 128),
    (1, 1, 10, 1, 1, 0, (), 128),
    (2, 100, 25, 3, 4, 8, (1,), 64),
])
def test_prefill_pack_decode_matches_oracle(B, T, n, H, D, W, dense, Dh):
    mask = [1 if h in dense else 0 for h in range(H)]
    N = T + n
    q, xk, xv, g = prefill_inputs(B, N, H, Dh, "bf16", gate_mean=1.0, gate_std=2.0, seed=N)
    # GPU: scan the first T tokens, pack, then n decode steps
    state = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    hk, hv = ratp.scan_prefill_kv(xk[:, :T].contiguous().to(DEV), xv[:, :T].contiguous().to(DEV),
                                  g[:, :T].contiguous().to(DEV), final_state=state)
    cache = ratp.KVCache(B, H, Dh, N, D, W, head_mask=mask)
    shadow = LayoutShadow(cache, N, mask)
    cache.pack(hk, hv)
    ratp.last_error()
    # layout after pack: the oracle's pack of the GPU's own hk/hv, bit for bit
    shadow.prefill(hk, hv)
    shadow.check("after pack")

    # oracle: fp64 scan of the same T tokens, pack, literal decode steps
    rk = oracle.scan(to64(xk[:, :T]), to64(g[:, :T]))
    rv = oracle.scan(to64(xv[:, :T]), to64(g[:, :T]))
    oc = oracle.Cache(B, H, Dh, N, D, W, dense_mask=mask)
    oc.pack(rk, rv, state=np.stack([rk[:, -1], rv[:, -1]]))

    for i in range(n):
        t = T + i
        args = [x[:, t].contiguous() for x in (q, xk, xv, g)]
        o = cache.decode_step(*[a.to(DEV) for a in args], state)
        ref = oc.decode_step(*[to64(a) for a in args])
        assert_close(o, ref, "bf16", "decode step %d" % i)
        # appended rows are the bf16-rounded new state, where the oracle puts them
        shadow.append(state)
        shadow.check("after decode step %d" % i)
    ratp.last_error()
    assert cache.lengths().cpu().tolist() == [N] * B
    assert_close(state[0], oc.state[0], "f32", "final k state")


def test_decode_consistent_with_gpu_prefill():
    """Decode outputs equal the GPU prefill attention of the longer sequence."""
    B, T, n, H, Dh, D, W = 2, 256, 64, 4, 128, 4, 32
    mask = [1, 0, 0, 0]
    N = T + n
    q, xk, xv, g = prefill_inputs(B, N, H, Dh, "bf16", seed=77)
    hk_all, hv_all = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV))
    o_all = ratp.dilated_attn_prefill(q.to(DEV), hk_all, hv_all, D, W, head_mask=mask)
    state = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    hk, hv = ratp.scan_prefill_kv(xk[:, :T].contiguous().to(DEV), xv[:, :T].contiguous().to(DEV),
                                  g[:, :T].contiguous().to(DEV), final_state=state)
    cache = ratp.KVCache(B, H, Dh, N, D, W, head_mask=mask)
    cache.pack(hk, hv)
    outs = []
    for i in range(n):
        t = T + i
        outs.append(cache.decode_step(*[x[:, t].contiguous().to(DEV) for x in (q, xk, xv, g)], state))
    ratp.last_error()
    got = torch.stack(outs, dim=1)
    err = (got.float() - o_all[:, T:].float()).abs()
    assert err.max().item() <= 3e-2 and err.mean().item() <= 3e-3


def test_decode_capacity_is_reported():
    B, T, H, Dh, D = 1, 16, 1, 128, 4
    q, xk, xv, g = prefill_inputs(B, T, H, Dh, "bf16", seed=1)
    hk, hv = ratp.scan_prefill_kv(xk.to(DEV), xv.to(DEV), g.to(DEV))
    cache = ratp.KVCache(B, H, Dh, T, D, 0)
    cache.pack(hk, hv)
    state = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    cache.decode_step(*[x[:, 0].contiguous().to(DEV) for x in (q, xk, xv, g)], state)
    with pytest.raises(RatpError, match="CAPACITY"):
        ratp.last_error()
    assert cache.lengths().cpu().tolist() == [T]
    ratp.last_error()   # the error word was cleared by the previous read


def _fill_decode_context(cache, w, kd, vd, kw, vw):
    kc, vc = cache.dil_rows("k"), cache.dil_rows("v")
    for h in range(w.H):
        off, _ = cache.head_rows(h)
        n = kd[h].shape[1]
        kc[:, off:off + n] = kd[h].to(DEV)
        vc[:, off:off + n] = vd[h].to(DEV)
    ctx = w.decode_ctx
    # ring row r holds the position p with p mod W == r among the last W
    kring, vring = cache.ring("k"), cache.ring("v")
    kring.copy_(kw.to(DEV))
    vring.copy_(vw.to(DEV))
    cache.lengths().fill_(ctx)


def test_decode_from_32k_context_full_size_sampled():
    w = WORKLOADS["bf16_decode_ctx32768_D64_W128"]
    steps = w.decode_steps
    T_max = w.decode_ctx + steps
    kd, vd, kw, vw, st0 = decode_context(w.B, w.H, w.Dh, w.decode_ctx, w.D, w.W)
    q, xk, xv, g = decode_inputs(steps, w.B, w.H, w.Dh, "bf16", w.gate_mean, w.gate_std)
    cache = ratp.KVCache(w.B, w.H, w.Dh, T_max, w.D, w.W)
    _fill_decode_context(cache, w, kd, vd, kw, vw)
    state = st0.to(DEV).contiguous()
    qd, xkd, xvd, gd = (x.to(DEV) for x in (q, xk, xv, g))
    outs = torch.empty(steps, w.B, w.H, w.Dh, dtype=torch.bfloat16, device=DEV)
    for i in range(steps):
        cache.decode_step(qd[i], xkd[i], xvd[i], gd[i], state, out=outs[i])
    ratp.last_error()
    assert cache.lengths().cpu().tolist() == [T_max] * w.B
    # oracle on two sampled sequences (sequences are independent)
    for b in (0, 37):
        oc = oracle.Cache(1, w.H, w.Dh, T_max, w.D, w.W)
        for h in range(w.H):
            for s in range(kd[h].shape[1]):
                row = oracle.cache_row(0, h, s, w.H, T_max, w.D)
                oc.Kc[row] = to64(kd[h][b, s])
                oc.Vc[row] = to64(vd[h][b, s])
        oc.Kw[:] = to64(kw[b]).reshape(-1, w.Dh)
        oc.Vw[:] = to64(vw[b]).reshape(-1, w.Dh)
        oc.len[:] = w.decode_ctx
        oc.state[:] = to64(st0[:, b:b + 1])
        for i in range(steps):
            ref = oc.decode_step(*[to64(x[i, b:b + 1]) for x in (q, xk, xv, g)])
            assert_close(outs[i, b:b + 1], ref, "bf16", "b=%d step %d" % (b, i))


def test_hybrid_prefill_then_decode_full_size_sampled():
    w = WORKLOADS["bf16_hybrid_7p6b_T8192_D4"]
    steps = w.decode_steps
    N = w.T + steps
    q, xk, xv, g = prefill_inputs(w.B, N, w.H, w.Dh, w.dtype, w.gate_mean, w.gate_std, seed=0)
    mask = w.dense_mask
    state = torch.zeros(2, w.B, w.H, w.Dh, dtype=torch.float32, device=DEV)
    T = w.T
    hk, hv = ratp.scan_prefill_kv(xk[:, :T].contiguous().to(DEV), xv[:, :T].contiguous().to(DEV),
                                  g[:, :T].contiguous().to(DEV), final_state=state)
    cache = ratp.KVCache(w.B, w.H, w.Dh, N, w.D, w.W, head_mask=mask)
    cache.pack(hk, hv)
    outs = []
    for i in range(steps):
        t = T + i
        outs.append(cache.decode_step(*[x[:, t].contiguous().to(DEV) for x in (q, xk, xv, g)], state))
    ratp.last_error()
    got = torch.stack(outs).cpu()
    b = 2
    sl = lambda x: x[b:b + 1]
    rk = oracle.scan(to64(sl(xk)[:, :T]), to64(sl(g)[:, :T]))
    rv = oracle.scan(to64(sl(xv)[:, :T]), to64(sl(g)[:, :T]))
    oc = oracle.Cache(1, w.H, w.Dh, N, w.D, w.W, dense_mask=mask)
    oc.pack(rk, rv, state=np.stack([rk[:, -1], rv[:, -1]]))
    for i in range(steps):
        t = T + i
        ref = oc.decode_step(*[to64(sl(x)[:, t]) for x in (q, xk, xv, g)])
        assert_close(got[i, b:b + 1], ref, "bf16", "hybrid decode step %d" % i)


@pytest.mark.parametrize("D,W,dense", [(4, 8, ()), (16, 0, (1,)), (3, 5, (0,))])
def test_decode_ragged_lengths(D, W, dense):
    """Sequences at different positions in one decode launch (len[b] differs):
    each sequence's prefill is packed on its own and copied into its block of
    the shared cache; every decode output equals the oracle's prefill
    attention over that sequence's own tokens."""
    B, H, Dh, n = 3, 2, 128, 12
    lens = [250, 131, 7]
    T_max = max(lens) + n
    mask = [1 if h in dense else 0 for h in range(H)]
    cache = ratp.KVCache(B, H, Dh, T_max, D, W, head_mask=mask)
    state = torch.zeros(2, B, H, Dh, dtype=torch.float32, device=DEV)
    seqs = []
    for b, Tb in enumerate(lens):
        q, xk, xv, g = prefill_inputs(1, Tb + n, H, Dh, "bf16", gate_mean=1.0, gate_std=2.0, seed=70 + b)
        seqs.append((q, xk, xv, g))
        fs = torch.zeros(2, 1, H, Dh, dtype=torch.float32, device=DEV)
        hk, hv = ratp.scan_prefill_kv(xk[:, :Tb].contiguous().to(DEV), xv[:, :Tb].contiguous().to(DEV),
                                      g[:, :Tb].contiguous().to(DEV), final_state=fs)
        one = ratp.KVCache(1, H, Dh, T_max, D, W, head_mask=mask)
        one.pack(hk, hv)
        for which in ("k", "v"):
            cache.dil_rows(which)[b].copy_(one.dil_rows(which)[0])
            if W:
                cache.ring(which)[b].copy_(one.ring(which)[0])
        state[:, b] = fs[:, 0]
    cache.lengths().copy_(torch.tensor(lens, dtype=torch.int32, device=DEV))
    outs = []
    for i in range(n):
        step = [torch.cat([s[k][:, lens[b] + i] for b, s in enumerate(seqs)]).contiguous().to(DEV)
                for k in range(4)]
        outs.append(cache.decode_step(*step, state))
    ratp.last_error()
    assert cache.lengths().cpu().tolist() == [Tb + n for Tb in lens]
    for b, (q, xk, xv, g) in enumerate(seqs):
        rk, rv = oracle.scan(to64(xk), to64(g)), oracle.scan(to64(xv), to64(g))
        ref = oracle.attention(to64(q), rk, rv, D, W, dense_mask=mask)
        for i in range(n):
            assert_close(outs[i][b:b + 1], ref[:, lens[b] + i], "bf16", "b=%d step %d" % (b, i))
