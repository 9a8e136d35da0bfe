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


class SampledCache:
    """A CUDA cache for every head plus oracle factors for a few of them.

    The oracle factors emulate the cache's bf16 coefficient storage.  With
    ``shadow=True`` a second set of oracle factors keeps float64 coefficients
    (no storage rounding) for the same heads, so that the format drift -- what
    bf16 storage alone costs -- can be reported beside the kernel error."""

    def __init__(self, cfg, workload, sample, seed, sync=True, shadow=False):
        import online_rank_kv_b200 as ik
        self.ik = ik
        self.cfg = cfg
        self.cache = ik.Cache(cfg)
        self.L, self.B, self.H = cfg.layers, cfg.batch, cfg.kv_heads
        self.g = cfg.q_heads // cfg.kv_heads
        nh = self.L * self.B * self.H
        self.ks = synth.KVStream(synth.spec_for(workload, "K"), nh, seed=2 * seed + 1, device="cuda",
                                 dtype=torch.bfloat16)
        self.vs = synth.KVStream(synth.spec_for(workload, "V"), nh, seed=2 * seed + 2, device="cuda",
                                 dtype=torch.bfloat16)
        self.sample = list(sample)
        self.ok = {x: HeadFactor(128, cfg.rank_k, cfg.window, coef_round="bf16", sync=sync)
                   for x in self.sample}
        self.ov = {x: HeadFactor(128, cfg.rank_v, cfg.window, coef_round="bf16", sync=sync)
                   for x in self.sample}
        self.shadow = shadow
        if shadow:
            self.sk = {x: HeadFactor(128, cfg.rank_k, cfg.window, coef_round=None, sync=sync)
                       for x in self.sample}
            self.sv = {x: HeadFactor(128, cfg.rank_v, cfg.window, coef_round=None, sync=sync)
                       for x in self.sample}
        self.folds = 0
        self.qseed = 5000 + seed

    def _oracles(self):
        out = [self.ok, self.ov]
        if self.shadow:
            out += [self.sk, self.sv]
        return out

    def append(self, t):
        k = self.ks.next(t).view(self.L, self.B, self.H, t, 128)
        v = self.vs.next(t).view(self.L, self.B, self.H, t, 128)
        for l in range(self.L):
            self.cache.append(l, k[l].contiguous(), v[l].contiguous())
        for (l, b, h) in self.sample:
            kx = k[l, b, h].double().cpu().numpy()
            vx = v[l, b, h].double().cpu().numpy()
            for i, of in enumerate(self._oracles()):
                of[(l, b, h)].append(kx if i % 2 == 0 else vx)

    def fold_all(self, defer):
        self.cache.compress_block(self.ik.ALL_LAYERS, defer=defer)
        for x in self.sample:
            for of in self._oracles():
                of[x].fold(defer=defer)

    def sync_all(self):
        self.cache.sync(self.ik.ALL_LAYERS)
        for x in self.sample:
            for of in self._oracles():
                of[x].sync()

    def format_drift(self):
        """Worst max |C B^T (bf16 storage) - C B^T (float64 storage)| / max |.|
        over the sampled heads, K and V, both on the oracle (needs shadow)."""
        worst = 0.0
        for x in self.sample:
            for of, sf in ((self.ok, self.sk), (self.ov, self.sv)):
                if of[x].n_c > 0:
                    worst = max(worst, rel_err(of[x].reconstruct(), sf[x].reconstruct()))
        return worst

    def ready(self):
        T, n_c = self.cache.counts(0)
        return (T - n_c - self.cfg.window) // 64

    def prefill(self, tokens, chunk=512, defer_every=64):
        """Append in chunks; fold every ready block with postponed rewrites,
        one rewrite per defer_every folds, as the bench prefills."""
        done = 0
        while done < tokens:
            n = min(chunk, tokens - done)
            self.append(n)
            done += n
            while self.ready() >= 1:
                self.fold_all(defer=defer_every > 0)
                self.folds += 1
                if defer_every > 0 and self.folds % defer_every == 0:
                    self.sync_all()
        if defer_every > 0:
            self.sync_all()

    def check(self, tol=2e-2):
        """Counters exact; reconstructions of the sampled heads within tol.
        Returns the worst error."""
        ik = self.ik
        worst = 0.0
        for l in sorted({x[0] for x in self.sample}):
            T, n_c = self.cache.counts(l)
            for x in self.sample:
                if x[0] == l:
                    assert (T, n_c) == (self.ok[x].T, self.ok[x].n_c)
            for which, of in ((ik.WHICH_K, self.ok), (ik.WHICH_V, self.ov)):
                got = self.cache.reconstruct(l, which)
                for x in self.sample:
                    if x[0] == l and of[x].n_c > 0:
                        e = rel_err(got[x[1], x[2]].cpu().numpy(), of[x].reconstruct())
                        assert e < tol, (l, which, x, e)
                        worst = max(worst, e)
                del got
        return worst

    def decode_check(self, q=None, tol=2e-2):
        """Decode every sampled layer with q (B x Hq x d); compare the sampled
        heads' outputs with dense attention over the oracle's cache."""
        c = self.cfg
        if q is None:
            q = synth.query_batch(c.batch * c.q_heads, 128, seed=self.qseed,
                                  dtype=torch.bfloat16).view(c.batch, c.q_heads, 128)
            self.qseed += 1
        worst = 0.0
        for l in sorted({x[0] for x in self.sample}):
            out = self.cache.decode_attention(l, q.cuda()).cpu().numpy()
            qn = q.double().numpy()
            for x in self.sample:
                if x[0] != l:
                    continue
                b, h = x[1], x[2]
                want = dense_decode(qn[b, h * self.g:(h + 1) * self.g], self.ok[x].full(),
                                    self.ov[x].full(), c.rope_theta, use_rope=True)
                e = rel_err(out[b, h * self.g:(h + 1) * self.g], want)
                worst = max(worst, e)
        assert worst < tol, worst
        return worst
