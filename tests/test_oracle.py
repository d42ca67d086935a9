"""Pins for the fp64 oracle: each check ties it to something other than itself.

* recurrence: hand-worked fixture, g = 0 identity, constant-gate closed form
  (geometric sum), and the associative affine-map composition;
* chunk-local recurrence: L = 1 closed form, the constant-gate closed form
  restarted per block, L >= T equal to the full recurrence, blocks equal to
  independent recurrences, and insensitivity to earlier blocks' inputs;
* fixed look-back recurrence: L = 1 closed form, L >= T equal to the full
  recurrence, the constant-gate closed form (a truncated geometric sum), and
  the block decomposition from explicit sums;
* key sets: hand-worked fixture, an independent membership predicate, and a
  closed-form count;
* attention: hand-worked fixture, dense causal attention from
  ``torch.nn.functional.scaled_dot_product_attention`` (fp64) when D = 1 or
  W >= T, the self-only identity when D >= T, and an explicit-mask brute force;
  per-sample dilation: dense samples equal SDPA, samples with D > T are
  self-only;
* cache: hand-worked layout fixture, bijectivity, and prefill/decode
  consistency of the literal decode step.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- recurrence
def test_scan_hand_fixture():
    rows = np.array(read_golden("scan_hand.txt"), dtype=np.float64)
    g, x, h = rows[:, 0], rows[:, 1], rows[:, 2]
    out = oracle.scan(x.reshape(1, -1, 1), g.reshape(1, -1, 1)).ravel()
    assert np.array_equal(out, h)


def test_scan_gate_zero_is_identity():
    x = RNG.standard_normal((2, 37, 3, 5))
    h = oracle.scan(x, np.zeros_like(x))
    assert np.array_equal(h, x)


@pytest.mark.parametrize("c", [0.0, 0.3, 0.9, 0.999])
def test_scan_constant_gate_geometric_sum(c):
    T = 50
    x = RNG.standard_normal((1, T, 4))
    h = oracle.scan(x, np.full_like(x, c))
    for t in range(T):
        w = np.array([(1 - c) * c ** (t - i) for i in range(t + 1)])
        ref = (w[:, None] * x[0, : t + 1]).sum(axis=0)
        np.testing.assert_allclose(h[0, t], ref, rtol=1e-12, atol=1e-12)


def test_scan_constant_gate_unit_input():
    c, T = 0.75, 64
    h = oracle.scan(np.ones((1, T, 1)), np.full((1, T, 1), c)).ravel()
    np.testing.assert_allclose(h, 1 - c ** (np.arange(T) + 1), rtol=0, atol=1e-14)


def test_scan_associative_composition():
    """Each step is the affine map h -> g h + (1-g) x; composing the maps of
    random blocks (a parallel-scan formulation) must give the same states."""
    B, T, C = 2, 97, 6
    x = RNG.standard_normal((B, T, C))
    g = RNG.uniform(0, 1, (B, T, C))
    h = oracle.scan(x, g)
    cuts = sorted(set([0, T] + list(RNG.integers(1, T, 8))))
    carry = np.zeros((B, C))
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        A = np.ones((B, C))
        Bv = np.zeros((B, C))
        for t in range(lo, hi):          # block aggregate of the affine maps
            A, Bv = g[:, t] * A, g[:, t] * Bv + (1 - g[:, t]) * x[:, t]
        end = A * carry + Bv
        np.testing.assert_allclose(h[:, hi - 1], end, rtol=1e-12, atol=1e-12)
        carry = end


# ---------------------------------------------------- chunk-local recurrence
def test_scan_reset_every_token_is_input_weighting():
    x = RNG.standard_normal((2, 23, 7))
    g = RNG.uniform(0, 1, x.shape)
    h = oracle.scan(x, g, L=1)
    np.testing.assert_allclose(h, (1 - g) * x, rtol=0, atol=1e-15)


@pytest.mark.parametrize("L", [3, 16, 64])
def test_scan_reset_constant_gate_unit_input(L):
    c, T = 0.8, 150
    h = oracle.scan(np.ones((1, T, 1)), np.full((1, T, 1), c), L=L).ravel()
    np.testing.assert_allclose(h, 1 - c ** (np.arange(T) % L + 1), rtol=0, atol=1e-14)


@pytest.mark.parametrize("L", [41, 97, 1000])
def test_scan_reset_longer_than_sequence_is_full(L):
    x = RNG.standard_normal((2, 41, 5))
    g = RNG.uniform(0, 1, x.shape)
    assert np.array_equal(oracle.scan(x, g, L=L), oracle.scan(x, g))


@pytest.mark.parametrize("L", [2, 7, 16])
def test_scan_reset_blocks_are_independent(L):
    B, T, C = 2, 53, 4
    x = RNG.standard_normal((B, T, C))
    g = RNG.uniform(0, 1, (B, T, C))
    h = oracle.scan(x, g, L=L)
    for lo in range(0, T, L):
        hi = min(lo + L, T)
        np.testing.assert_allclose(h[:, lo:hi], oracle.scan(x[:, lo:hi], g[:, lo:hi]),
                                   rtol=0, atol=1e-15)
    # inputs of earlier blocks never reach a later block
    x2 = x.copy()
    x2[:, : 2 * L] += 10.0
    h2 = oracle.scan(x2, g, L=L)
    assert np.array_equal(h2[:, 2 * L:], h[:, 2 * L:])
    assert not np.array_equal(h2[:, :L], h[:, :L])


# ------------------------------------------------- fixed look-back recurrence
def test_scan_window_one_token_is_input_weighting():
    x = RNG.standard_normal((2, 19, 3))
    g = RNG.uniform(0, 1, x.shape)
    np.testing.assert_allclose(oracle.scan_window(x, g, 1), (1 - g) * x, rtol=0, atol=1e-15)


@pytest.mark.parametrize("L", [19, 20, 500])
def test_scan_window_covering_sequence_is_full(L):
    x = RNG.standard_normal((2, 19, 4))
    g = RNG.uniform(0, 1, x.shape)
    assert np.array_equal(oracle.scan_window(x, g, L), oracle.scan(x, g))


@pytest.mark.parametrize("L,c", [(4, 0.7), (16, 0.95), (64, 0.9)])
def test_scan_window_constant_gate_closed_form(L, c):
    T = 150
    x = RNG.standard_normal((1, T, 2))
    h = oracle.scan_window(x, np.full_like(x, c), L)
    for t in range(T):
        k = np.arange(min(t + 1, L))
        ref = ((1 - c) * c ** k[:, None] * x[0, t - k]).sum(axis=0)
        np.testing.assert_allclose(h[0, t], ref, rtol=1e-12, atol=1e-12)
    ones = oracle.scan_window(np.ones((1, T, 1)), np.full((1, T, 1), c), L).ravel()
    np.testing.assert_allclose(ones, 1 - c ** np.minimum(np.arange(T) + 1, L), rtol=0, atol=1e-13)


@pytest.mark.parametrize("L", [4, 16])
def test_scan_window_matches_blocks_and_suffix_form(L):
    """At the last position of every block of L the window is the block, so
    the value equals the chunk-local recurrence there; everywhere it equals
    the block decomposition loc_t + A_t * S(t - L), built here from explicit
    sums (A: gate product since the block start, S: the previous block's
    recurrence over positions t-L+1 .. block end)."""
    B, T, C = 2, 61, 3
    x = RNG.standard_normal((B, T, C))
    g = RNG.uniform(0, 1, (B, T, C))
    h = oracle.scan_window(x, g, L)
    loc = oracle.scan(x, g, L=L)
    ends = [t for t in range(T) if t % L == L - 1]
    assert np.allclose(h[:, ends], loc[:, ends], rtol=1e-12, atol=1e-12)
    for t in range(T):
        c0 = (t // L) * L
        A = np.prod(g[:, c0:t + 1], axis=1)
        S = np.zeros((B, C))
        for j in range(max(0, t - L + 1), c0):
            S += np.prod(g[:, j + 1:c0], axis=1) * (1 - g[:, j]) * x[:, j]
        np.testing.assert_allclose(h[:, t], loc[:, t] + A * S, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- key sets
def test_key_set_hand_fixture():
    for row in read_golden("key_sets_hand.txt"):
        t, D, W = int(row[0]), int(row[1]), int(row[2])
        assert oracle.key_set(t, D, W) == [int(v) for v in row[3:]], row


def _member(t, j, D, W):
    return j <= t and (j % D == D - 1 or j == t or (W > 0 and t - j < W))


def test_key_set_matches_predicate():
    for t in range(0, 40):
        for D in range(1, 44):
            for W in (0, 1, 2, 3, 5, 8, 40):
                ref = [j for j in range(t + 1) if _member(t, j, D, W)]
                assert oracle.key_set(t, D, W) == ref, (t, D, W)


def test_key_set_count_closed_form():
    for t in range(0, 300, 7):
        for D in (1, 2, 4, 16, 64):
            for W in (0, 1, 5, 128):
                n = len(oracle.key_set(t, D, W))
                if W == 0:
                    ref = t // D + 1
                else:
                    lo = max(0, t - W + 1)
                    dup = sum(1 for j in range(lo, t) if j % D == D - 1)
                    ref = t // D + min(W, t + 1) - dup
                assert n == ref, (t, D, W)


# ---------------------------------------------------------------- attention
def _rand_qkv(B, T, H, Dh):
    return (RNG.standard_normal((B, T, H, Dh)), RNG.standard_normal((B, T, H, Dh)),
            RNG.standard_normal((B, T, H, Dh)))


def _sdpa_causal(q, k, v):
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    return o.permute(0, 2, 1, 3).numpy()


def test_attention_hand_fixture():
    q = np.array([0.7, 0.0, 1.0]).reshape(1, 3, 1, 1)
    hk = np.array([0.3, math.log(3.0), 0.0]).reshape(1, 3, 1, 1)
    hv = np.array([2.0, 4.0, 8.0]).reshape(1, 3, 1, 1)
    for row in read_golden("attention_hand.txt"):
        D, W = int(row[0]), int(row[1])
        ref = np.array([float(v) for v in row[2:]])
        out = oracle.attention(q, hk, hv, D, W).ravel()
        np.testing.assert_allclose(out, ref, rtol=1e-14, atol=1e-14)


def test_attention_dense_equals_sdpa():
    q, k, v = _rand_qkv(2, 33, 3, 16)
    np.testing.assert_allclose(oracle.attention(q, k, v, 1, 0), _sdpa_causal(q, k, v),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("D", [2, 5, 64])
def test_attention_window_covering_sequence_is_dense(D):
    q, k, v = _rand_qkv(1, 29, 2, 8)
    for W in (29, 40):
        np.testing.assert_allclose(oracle.attention(q, k, v, D, W), _sdpa_causal(q, k, v),
                                   rtol=1e-12, atol=1e-12)


def test_attention_dense_heads_are_dense():
    q, k, v = _rand_qkv(1, 21, 3, 8)
    out = oracle.attention(q, k, v, 4, 0, dense_mask=[1, 0, 1])
    ref = _sdpa_causal(q, k, v)
    np.testing.assert_allclose(out[:, :, 0], ref[:, :, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[:, :, 2], ref[:, :, 2], rtol=1e-12, atol=1e-12)
    assert not np.allclose(out[:, :, 1], ref[:, :, 1])


def test_attention_per_sample_dense_and_self_only_samples():
    """Samples with D = 1 are dense causal attention (SDPA); samples whose D
    exceeds the sequence attend only to themselves (o = hv); the others equal
    the single-dilation attention of their D."""
    q, k, v = _rand_qkv(4, 23, 2, 8)
    ds = [1, 30, 4, 1]
    out = oracle.attention_per_sample(q, k, v, ds, 0)
    ref = _sdpa_causal(q, k, v)
    for b in (0, 3):
        np.testing.assert_allclose(out[b], ref[b], rtol=1e-12, atol=1e-12)
    assert np.array_equal(out[1], v[1])
    assert np.array_equal(out[2], oracle.attention(q, k, v, 4, 0)[2])
    rows = np.array([[2, 22, 1], [0, 5, 0], [1, 7, 1], [2, 3, 0]])
    got = oracle.attention_per_sample(q, k, v, ds, 0, rows=rows)
    for i, (b, t, h) in enumerate(rows):
        assert np.array_equal(got[i], out[b, t, h])


def test_attention_dilation_beyond_sequence_is_self():
    q, k, v = _rand_qkv(2, 17, 2, 8)
    for D in (17, 18, 100):
        assert np.array_equal(oracle.attention(q, k, v, D, 0), v)


@pytest.mark.parametrize("T,D,W", [(1, 1, 0), (5, 2, 0), (16, 4, 0), (16, 4, 3),
                                   (23, 3, 5), (20, 7, 1), (31, 8, 16), (12, 1, 4)])
def test_attention_enumeration_equals_mask(T, D, W):
    q, k, v = _rand_qkv(2, T, 3, 4)
    mask = [0, 1, 0]
    np.testing.assert_allclose(oracle.attention(q, k, v, D, W, dense_mask=mask),
                               oracle.attention_mask(q, k, v, D, W, dense_mask=mask),
                               rtol=1e-12, atol=1e-12)


def test_attention_row_subset_matches_full():
    q, k, v = _rand_qkv(2, 40, 3, 8)
    full = oracle.attention(q, k, v, 4, 3, dense_mask=[0, 0, 1])
    rows = np.array([[0, 0, 0], [1, 39, 2], [0, 17, 1], [1, 3, 0]])
    sub = oracle.attention(q, k, v, 4, 3, dense_mask=[0, 0, 1], rows=rows)
    for i, (b, t, h) in enumerate(rows):
        assert np.array_equal(sub[i], full[b, t, h])


# ---------------------------------------------------------------- cache / decode
def test_cache_layout_hand_fixture():
    mask = [0, 1, 0]
    for kind, b, h, s, ref in read_golden("cache_layout_hand.txt"):
        b, h, s, ref = int(b), int(h), int(s), int(ref)
        if kind == "dil":
            assert oracle.cache_row(b, h, s, 3, 8, 4, mask) == ref
        else:
            assert oracle.ring_row(b, h, s, 3, 4) == ref
    assert oracle.cache_rows_total(2, 3, 8, 4, mask) == 24


def test_cache_layout_is_a_bijection():
    B, H, T_max, D = 3, 5, 37, 4
    mask = [1, 0, 0, 1, 0]
    seen = set()
    for b in range(B):
        for h in range(H):
            Dd = 1 if mask[h] else D
            for s in range(T_max // Dd):
                seen.add(oracle.cache_row(b, h, s, H, T_max, D, mask))
    assert seen == set(range(oracle.cache_rows_total(B, H, T_max, D, mask)))


@pytest.mark.parametrize("D,W,mask", [(1, 0, None), (3, 0, None), (4, 2, None),
                                      (4, 5, [1, 0]), (2, 1, [0, 1]), (8, 3, [1, 1])])
def test_decode_continues_prefill(D, W, mask):
    """pack(T) + n literal decode steps == prefill attention of T + n tokens."""
    B, T, n, H, Dh = 2, 13, 9, 2, 8
    N = T + n
    q = RNG.standard_normal((B, N, H, Dh))
    xk = RNG.standard_normal((B, N, H, Dh))
    xv = RNG.standard_normal((B, N, H, Dh))
    g = RNG.uniform(0, 1, (B, N, H, Dh))
    hk, hv = oracle.scan(xk, g), oracle.scan(xv, g)
    ref = oracle.attention(q, hk, hv, D, W, dense_mask=mask)
    cache = oracle.Cache(B, H, Dh, N, D, W, dense_mask=mask)
    cache.pack(hk[:, :T], hv[:, :T], state=np.stack([hk[:, T - 1], hv[:, T - 1]]))
    for i in range(n):
        t = T + i
        o = cache.decode_step(q[:, t], xk[:, t], xv[:, t], g[:, t])
        np.testing.assert_allclose(o, ref[:, t], rtol=1e-11, atol=1e-11)
    assert list(cache.len) == [N] * B
    # every cached dilated row holds the recurrent key of its position
    for b in range(B):
        for h in range(H):
            Dd = 1 if (mask and mask[h]) else D
            for s in range(N // Dd):
                row = oracle.cache_row(b, h, s, H, N, D, mask)
                np.testing.assert_allclose(cache.Kc[row], hk[b, s * Dd + Dd - 1, h], rtol=1e-12)
                np.testing.assert_allclose(cache.Vc[row], hv[b, s * Dd + Dd - 1, h], rtol=1e-12)


@pytest.mark.parametrize("L,T", [(4, 12), (5, 13), (1, 7), (16, 10)])
def test_decode_chunk_local_continues_prefill(L, T):
    """With chunk-local recurrence the decode step restarts the state at the
    same positions as the prefill scan (blocks cross the prefill boundary)."""
    B, n, H, Dh, D, W = 2, 11, 2, 8, 3, 2
    N = T + n
    q = RNG.standard_normal((B, N, H, Dh))
    xk = RNG.standard_normal((B, N, H, Dh))
    xv = RNG.standard_normal((B, N, H, Dh))
    g = RNG.uniform(0, 1, (B, N, H, Dh))
    hk, hv = oracle.scan(xk, g, L=L), oracle.scan(xv, g, L=L)
    ref = oracle.attention(q, hk, hv, D, W)
    cache = oracle.Cache(B, H, Dh, N, D, W, L=L)
    cache.pack(hk[:, :T], hv[:, :T], state=np.stack([hk[:, T - 1], hv[:, T - 1]]))
    for i in range(n):
        t = T + i
        o = cache.decode_step(q[:, t], xk[:, t], xv[:, t], g[:, t])
        np.testing.assert_allclose(o, ref[:, t], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(cache.state, np.stack([hk[:, N - 1], hv[:, N - 1]]),
                               rtol=1e-12, atol=1e-12)


def test_decode_capacity_error():
    cache = oracle.Cache(1, 1, 4, 3, 1, 0)
    hk = RNG.standard_normal((1, 3, 1, 4))
    cache.pack(hk, hk)
    z = np.zeros((1, 1, 4))
    with pytest.raises(RuntimeError):
        cache.decode_step(z, z, z, z)
