"""Drive the CUDA cache and the float64 oracle with the same seeded inputs.

Inputs come from ``synth`` on the host (float64 draws cast to the cache's K/V
type); the very same values are copied to the GPU and, as float64, to the
oracle.  Nothing here computes the method: the CUDA side runs through the
library's C ABI (via the binding), the reference side through ``oracle``.
"""

from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import HeadFactor, dense_decode


def rel_err(a, b) -> float:
    """max |a - b| / max |b| (the comparison metric of every parity test)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.abs(b).max()
    return float(np.abs(a - b).max() / (den if den > 0 else 1.0))


class Pair:
    """A CUDA cache and the oracle's per-head factors, fed identically."""

    def __init__(self, cfg, workload: str, seed: int = 0, heads=None, device="cuda", specs=None):
        import online_rank_kv_b200 as ik
        self.ik = ik
        self.cfg = cfg
        self.cache = ik.Cache(cfg)
        self.device = device
        self.L, self.B, self.H = cfg.layers, cfg.batch, cfg.kv_heads
        self.g = cfg.q_heads // cfg.kv_heads
        n = self.L * self.B * self.H
        kdt = cfg.kv_torch_dtype
        sk, sv = specs if specs is not None else (synth.spec_for(workload, "K"),
                                                  synth.spec_for(workload, "V"))
        self.ks = synth.KVStream(sk, n, seed=2 * seed + 1, dtype=kdt)
        self.vs = synth.KVStream(sv, n, seed=2 * seed + 2, dtype=kdt)
        self.heads = heads if heads is not None else [
            (l, b, h) for l in range(self.L) for b in range(self.B) for h in range(self.H)]
        rnd = "bf16" if cfg.coef_dtype == ik.BF16 else "f32"
        P = getattr(cfg, "protect", 0)
        self.P = P
        self.ok = {x: HeadFactor(cfg.head_dim, cfg.rank_k, cfg.window, coef_round=rnd,
                                 sync=bool(cfg.sync), protect=P) for x in self.heads}
        self.ov = {x: HeadFactor(cfg.head_dim, cfg.rank_v, cfg.window, coef_round=rnd,
                                 sync=bool(cfg.sync), protect=P) for x in self.heads}
        self.qseed = 1000 + seed

    # -- inputs ------------------------------------------------------------
    def append(self, t: int):
        """Append t tokens to every layer; returns ready blocks per layer."""
        c = self.cfg
        k = self.ks.next(t).view(self.L, self.B, self.H, t, c.head_dim)
        v = self.vs.next(t).view(self.L, self.B, self.H, t, c.head_dim)
        ready = []
        for l in range(self.L):
            kl = k[l].contiguous().to(self.device)
            vl = v[l].contiguous().to(self.device)
            ready.append(self.cache.append(l, kl, vl))
        for (l, b, h) in self.heads:
            self.ok[(l, b, h)].append(k[l, b, h].double().numpy())
            self.ov[(l, b, h)].append(v[l, b, h].double().numpy())
        return ready

    def fold(self, layer: int, defer: bool = False):
        self.cache.compress_block(layer, defer=defer)
        for (l, b, h) in self.heads:
            if l == layer:
                self.ok[(l, b, h)].fold(defer=defer)
                self.ov[(l, b, h)].fold(defer=defer)

    def sync(self, layer: int):
        self.cache.sync(layer)
        for (l, b, h) in self.heads:
            if l == layer:
                self.ok[(l, b, h)].sync()
                self.ov[(l, b, h)].sync()

    def fold_ready(self, defer_every: int = 0):
        """Fold every ready block of every layer; with defer_every > 0 the
        rewrites are postponed and applied every defer_every folds."""
        for l in range(self.L):
            cnt = 0
            while True:
                T, n_c = self.cache.counts(l)
                if (max(0, T - self.P) - n_c - self.cfg.window) // 64 < 1:
                    break
                self.fold(l, defer=defer_every > 0)
                cnt += 1
                if defer_every > 0 and cnt % defer_every == 0:
                    self.sync(l)
            if defer_every > 0:
                self.sync(l)

    def ring_free(self) -> int:
        """Rows the exact-window ring can still take before a fold."""
        c = self.cfg
        cap = c.window + 64 + (c.ring_extra or 64)
        T, n_c = self.cache.counts(0)
        return cap - (max(0, T - self.P) - n_c)

    def prefill(self, tokens: int, chunk: int = 64, defer_every: int = 0):
        done = 0
        while done < tokens:
            n = min(chunk, tokens - done, self.ring_free())
            self.append(n)
            done += n
            self.fold_ready(defer_every)

    def query(self, scale: float = 1.0):
        c = self.cfg
        q = synth.query_batch(c.batch * c.q_heads, c.head_dim, seed=self.qseed,
                              dtype=c.kv_torch_dtype, scale=scale)
        self.qseed += 1
        return q.view(c.batch, c.q_heads, c.head_dim)

    # -- comparisons -------------------------------------------------------
    def check_counts(self):
        for l in range(self.L):
            T, n_c = self.cache.counts(l)
            for (ll, b, h) in self.heads:
                if ll == l:
                    f = self.ok[(ll, b, h)]
                    assert (T, n_c) == (f.T, f.n_c), (l, T, n_c, f.T, f.n_c)

    def recon_errors(self, layer: int):
        ik = self.ik
        out = {}
        for which, of in ((ik.WHICH_K, self.ok), (ik.WHICH_V, self.ov)):
            got = self.cache.reconstruct(layer, which).cpu().numpy()
            for (l, b, h) in self.heads:
                if l == layer and of[(l, b, h)].n_c > 0 and got.shape[2] > 0:
                    out[(which, b, h)] = rel_err(got[b, h], of[(l, b, h)].reconstruct())
        return out

    def decode(self, layer: int, q):
        out = self.cache.decode_attention(layer, q.to(self.device)).cpu().numpy()
        errs = {}
        c = self.cfg
        qn = q.double().numpy()
        for (l, b, h) in self.heads:
            if l != layer:
                continue
            K = self.ok[(l, b, h)].full()
            V = self.ov[(l, b, h)].full()
            want = dense_decode(qn[b, h * self.g:(h + 1) * self.g], K, V, c.rope_theta,
                                use_rope=bool(c.use_rope))
            errs[(b, h)] = rel_err(out[b, h * self.g:(h + 1) * self.g], want)
        return errs, out
