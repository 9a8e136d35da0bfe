"""Seeded synthetic K/V/query streams shaped like long chain-of-thought caches.

Shared input generator for the CUDA library's tests and bench and for the
float64 oracle's tests.  It holds none of the compression method's
arithmetic: it only draws data.  Everything is plain PyTorch so the same
recipe runs on the host (float64, small cases) or on a GPU (float32, the large
workloads whose sampled heads are copied back for checking).

Recipe for one stream of H head-instances (each a (sequence, layer, KV head)
for K, or the same for V):
  * G_h: ``rank`` x d orthonormal rows (QR of a Gaussian d x rank matrix);
  * token t: x_t = (z_t * lam) @ G_h(t) + noise * n_t, z_t, n_t iid N(0, 1);
  * lam_l = decay**l (decay = 1 gives the flat latent of the tiny case);
  * every ``drift_every`` tokens G_h turns by one Givens rotation by +-angle in
    a randomly chosen coordinate plane (i, j) of R^d (a slowly rotating
    subspace);
  * keys: ``outliers`` seeded channels per head are multiplied by
    ``outlier_scale`` after the draw;
  * the stream is cast to ``dtype`` (the cache's K/V input type).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

__all__ = ["StreamSpec", "KVStream", "spec_for", "query_batch", "recall_query", "recall_queries"]


@dataclass(frozen=True)
class StreamSpec:
    d: int = 128
    rank: int = 48
    decay: float = 1.0
    noise: float = 0.05
    outliers: int = 0
    outlier_scale: float = 10.0
    drift_every: int = 0          # 0: no drift
    drift_angle: float = 0.05


def spec_for(workload: str, kind: str) -> StreamSpec:
    """Stream recipes of the named workloads ("tiny", "qwen3" for the
    Qwen3-8B-shaped caches, "cot" for the long chain-of-thought growth run).

    Keys decay faster than values: keys are the more compressible of the two.
    """
    if kind not in ("K", "V"):
        raise ValueError(kind)
    if workload == "tiny":
        return StreamSpec(d=128, rank=8, decay=1.0, noise=1e-3)
    if workload in ("qwen3", "cot"):
        drift = 512 if workload == "qwen3" else 2048
        if kind == "K":
            return StreamSpec(d=128, rank=48, decay=0.90, noise=0.05, outliers=4,
                              outlier_scale=10.0, drift_every=drift)
        return StreamSpec(d=128, rank=48, decay=0.95, noise=0.05, drift_every=drift)
    raise ValueError(workload)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


class KVStream:
    """H independent seeded streams advanced together, token by token."""

    def __init__(self, spec: StreamSpec, n_heads: int, seed: int = 0,
                 device="cpu", dtype=torch.float32):
        self.spec = spec
        self.H = int(n_heads)
        self.device = torch.device(device)
        self.dtype = dtype
        # float64 on the host (small cases), float32 on a GPU (large cases)
        self.work = torch.float64 if self.device.type == "cpu" else torch.float32
        self.gen = _gen(seed, self.device)
        d, k = spec.d, spec.rank
        a = torch.randn(self.H, d, k, generator=self.gen, device=self.device, dtype=self.work)
        q, _ = torch.linalg.qr(a)
        self.G = q.transpose(1, 2).contiguous()            # H x rank x d
        self.lam = torch.pow(torch.tensor(spec.decay, dtype=self.work, device=self.device),
                             torch.arange(k, device=self.device, dtype=self.work))
        if spec.outliers > 0:
            scores = torch.rand(self.H, d, generator=self.gen, device=self.device)
            self.outlier_idx = torch.topk(scores, spec.outliers, dim=1).indices
        else:
            self.outlier_idx = None
        self.t = 0
        self._last_drift = -1

    def _drift(self):
        d = self.spec.d
        idx = torch.randint(0, d, (self.H, 2), generator=self.gen, device=self.device)
        # make the two coordinates distinct
        same = idx[:, 0] == idx[:, 1]
        idx[:, 1] = torch.where(same, (idx[:, 1] + 1) % d, idx[:, 1])
        sign = torch.randint(0, 2, (self.H,), generator=self.gen, device=self.device) * 2 - 1
        phi = sign.to(self.work) * self.spec.drift_angle
        c, s = torch.cos(phi), torch.sin(phi)
        ar = torch.arange(self.H, device=self.device)
        gi = self.G[ar, :, idx[:, 0]].clone()               # H x rank
        gj = self.G[ar, :, idx[:, 1]].clone()
        self.G[ar, :, idx[:, 0]] = c[:, None] * gi - s[:, None] * gj
        self.G[ar, :, idx[:, 1]] = s[:, None] * gi + c[:, None] * gj

    def next(self, n: int) -> torch.Tensor:
        """The next n tokens of every stream: H x n x d in ``dtype``."""
        sp = self.spec
        out = torch.empty(self.H, n, sp.d, device=self.device, dtype=self.work)
        done = 0
        while done < n:
            span = n - done
            if sp.drift_every > 0:
                if self.t > 0 and self.t % sp.drift_every == 0 and self._last_drift != self.t:
                    self._drift()
                    self._last_drift = self.t
                span = min(span, sp.drift_every - (self.t % sp.drift_every))
            z = torch.randn(self.H, span, sp.rank, generator=self.gen, device=self.device,
                            dtype=self.work) * self.lam
            x = torch.bmm(z, self.G)
            x += sp.noise * torch.randn(self.H, span, sp.d, generator=self.gen,
                                        device=self.device, dtype=self.work)
            out[:, done:done + span] = x
            done += span
            self.t += span
        if self.outlier_idx is not None:
            ar = torch.arange(self.H, device=self.device)[:, None]
            out[ar, :, self.outlier_idx] *= sp.outlier_scale
        return out.to(self.dtype)


def query_batch(n_heads: int, d: int, seed: int, device="cpu", dtype=torch.float32,
                scale: float = 1.0) -> torch.Tensor:
    """``n_heads`` iid N(0, scale^2) query vectors (taken as already rotated)."""
    g = _gen(seed, torch.device(device))
    work = torch.float64 if torch.device(device).type == "cpu" else torch.float32
    q = torch.randn(n_heads, d, generator=g, device=device, dtype=work) * scale
    return q.to(dtype)


def recall_query(k_pre: torch.Tensor, pos: int, theta: float, beta: float) -> torch.Tensor:
    """A query aimed at an old position: beta * RoPE(k_pre, pos) / |k_pre|.

    Used by the long chain-of-thought workload so that some steps put their
    top attention mass on a compressed token.  The rotation is the rotate-half
    form at absolute position ``pos`` (the data side needs its own copy: this
    module shares nothing with the library or the oracle).
    """
    k = k_pre.to(torch.float64)
    d = k.shape[-1]
    h = d // 2
    inv = torch.pow(torch.tensor(float(theta), dtype=torch.float64),
                    -2.0 * torch.arange(h, dtype=torch.float64) / d).to(k.device)
    ang = float(pos) * inv
    c, s = torch.cos(ang), torch.sin(ang)
    x1, x2 = k[..., :h], k[..., h:]
    rot = torch.cat([x1 * c - x2 * s, x1 * s + x2 * c], dim=-1)
    return beta * rot / torch.linalg.vector_norm(k, dim=-1, keepdim=True).clamp_min(1e-30)


def recall_queries(k_pre: torch.Tensor, pos: torch.Tensor, theta: float,
                   beta: float) -> torch.Tensor:
    """Many recall queries at once: row i is beta * RoPE(k_pre[i], pos[i]) /
    |k_pre[i]| (the same construction as ``recall_query``), computed in
    float64 on the rows' device."""
    k = k_pre.to(torch.float64)
    d = k.shape[-1]
    h = d // 2
    inv = torch.pow(torch.tensor(float(theta), dtype=torch.float64, device=k.device),
                    -2.0 * torch.arange(h, dtype=torch.float64, device=k.device) / d)
    ang = pos.to(torch.float64).reshape(-1, 1) * inv.reshape(1, -1)
    c, s = torch.cos(ang), torch.sin(ang)
    x1, x2 = k[..., :h], k[..., h:]
    rot = torch.cat([x1 * c - x2 * s, x1 * s + x2 * c], dim=-1)
    return beta * rot / torch.linalg.vector_norm(k, dim=-1, keepdim=True).clamp_min(1e-30)
