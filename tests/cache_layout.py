"""Exact check of the GPU decode cache against the oracle's layout rule.

The expected cache is built by the oracle alone.  Its pack (``orc_cache_pack``)
places the recurrent key/value of position p = s*D_h + D_h - 1 in dilated
slot s at row ``orc_cache_row(b, h, s)``.  It places each of the last W
positions at ring row ``orc_ring_row(b, h, p)``.  Here it is applied to the
recurrent keys/values that the GPU itself produced: the prefill rows, then
after each decode step the new key/value (the step's fp32 state, rounded to
bf16 as the cache stores it).  The GPU cache buffer is zero-filled before the
hand-off.  Every row of its dilated and ring regions must then equal the
oracle's, bit for bit: rows that should still be empty stay zero.  No index
arithmetic of the test or of the binding takes part.
"""
import numpy as np
import torch

import oracle


class LayoutShadow:
    def __init__(self, cache, n_max, dense_mask=None):
        self.cache = cache
        self.mask = dense_mask
        self.hist = np.zeros((2, cache.B, n_max, cache.H, cache.Dh))
        self.n = 0
        cache.buffer.zero_()          # unwritten rows must read as zero

    def prefill(self, hk, hv):
        """Recurrent keys/values [B, T, H, Dh] of the prefill (GPU tensors)."""
        T = hk.shape[1]
        self.hist[0, :, :T] = hk.detach().to("cpu", torch.float64).numpy()
        self.hist[1, :, :T] = hv.detach().to("cpu", torch.float64).numpy()
        self.n = T

    def append(self, state):
        """The fp32 state [2, B, H, Dh] right after a decode step."""
        self.hist[:, :, self.n] = state.detach().cpu().to(torch.bfloat16).to(torch.float64).numpy()
        self.n += 1

    def check(self, what=""):
        c = self.cache
        oc = oracle.Cache(c.B, c.H, c.Dh, c.T_max, c.D, c.W, dense_mask=self.mask)
        oc.pack(self.hist[0, :, :self.n], self.hist[1, :, :self.n])
        regions = [("Kc", c.dil_rows("k"), oc.Kc), ("Vc", c.dil_rows("v"), oc.Vc)]
        if c.W > 0:
            regions += [("Kw", c.ring("k"), oc.Kw), ("Vw", c.ring("v"), oc.Vw)]
        for name, gpu, ref in regions:
            got = gpu.reshape(-1, c.Dh).to("cpu", torch.float64).numpy()
            assert got.shape == ref.shape, (what, name, got.shape, ref.shape)
            bad = np.flatnonzero(np.any(got != ref, axis=1))
            assert bad.size == 0, "%s: %s rows %s differ from the oracle's layout" % (
                what, name, bad[:8].tolist())
        assert c.lengths().cpu().tolist() == [self.n] * c.B, what
