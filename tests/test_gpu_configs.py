"""The benchmark configurations at their full sizes, checked on sampled heads.

All K/V are drawn on the GPU (the same seeded generator as the bench); the
rows of the sampled (layer, sequence, KV head) instances are copied back and
fed to the float64 oracle, which emulates the bf16 coefficient storage and the
same postponed rewrites.  Tolerance 2e-2 (bf16-stored coefficients), counters
exact.

  * the 36-layer, batch-8, 32K-context Qwen3-8B-shaped cache (the bench
    workload): sampled heads (seq 0, layers {0, 35}, KV heads {0, 7});
  * the long chain-of-thought growth run: batch 1, 36 layers, r_K 64, r_V 96,
    W 2048, subspace drift every 2K tokens, grown to 128K tokens, with
    queries aimed at tokens older than 8K (recall of compressed history);
  * the one-layer sweep, every point: ranks {16, 32, 64, 128} x contexts
    {4K, 16K, 64K, 256K} x batches {1, 8, 32} (the three batch sizes of a
    point run in lockstep and share one sampled head's rows), and the
    no-synchronization ablation's reconstruction drift against the
    synchronized path.
"""

import numpy as np
import pytest
import torch

import synth
from iskv_testlib import SampledCache, rel_err
from oracle import HeadFactor, dense_decode

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(autouse=True, scope="module")
def _one_blas_thread():
    # the oracle's many small QR/SVD calls run faster on one BLAS thread
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        yield


def _cfg(**kw):
    import online_rank_kv_b200 as ik
    c = ik.Config(kv_dtype=ik.BF16, coef_dtype=ik.BF16, use_rope=1, rope_theta=1e6,
                  max_deferred=64, ring_extra=512)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_qwen3_36_layers_batch8_32k_sampled_heads():
    cfg = _cfg(batch=8, layers=36, kv_heads=8, q_heads=32, rank_k=32, rank_v=64, window=1024,
               max_tokens=32768 + 1024)
    s = SampledCache(cfg, "qwen3", [(0, 0, 0), (0, 0, 7), (35, 0, 0), (35, 0, 7)], seed=70)
    s.prefill(32768)
    s.check()
    s.decode_check()
    # decode steps, then one block fold with an immediate rewrite (the bench's step)
    for _ in range(3):
        s.append(1)
        s.decode_check()
    while s.ready() < 1:
        s.append(16)
    s.fold_all(defer=False)
    s.check()
    s.decode_check()
    assert s.cache.status() == 0


def test_long_cot_growth_to_128k_with_recall():
    cfg = _cfg(batch=1, layers=36, kv_heads=8, q_heads=32, rank_k=64, rank_v=96, window=2048,
               max_tokens=131072 + 1024)
    sample = [(0, 0, 0), (35, 0, 7)]
    s = SampledCache(cfg, "cot", sample, seed=71)
    s.prefill(8192)
    s.check()
    s.decode_check()
    s.prefill(131072 - 8192)
    T, n_c = s.cache.counts(0)
    assert T == 131072 and n_c == ((T - 2048) // 64) * 64
    s.check()
    s.decode_check()
    # queries whose top attention mass sits on a folded token older than 8K
    g = cfg.q_heads // cfg.kv_heads
    rng = np.random.default_rng(3)
    q = synth.query_batch(cfg.q_heads, 128, seed=77, dtype=torch.float64).view(1, cfg.q_heads, 128)
    for (l, b, h) in sample:
        rec = s.ok[(l, b, h)].reconstruct()
        for j in range(g):
            pos = int(rng.integers(0, T - 8192 - 2048))
            kp = torch.from_numpy(rec[pos])
            beta = 25.0 * np.sqrt(128) / float(torch.linalg.vector_norm(kp))
            q[b, h * g + j] = synth.recall_query(kp, pos, cfg.rope_theta, beta)
    s.decode_check(q.to(torch.bfloat16))
    assert s.cache.status() == 0


class LockstepSweep:
    """Caches of batch 1, 8 and 32 at one (rank, context) point of the sweep,
    fed in lockstep.  Each cache's own rows come from its seeded generator,
    except that the last sequence's KV head 7 receives the same rows in all
    three caches (a one-head stream), so one pair of oracle factors checks all
    three batch sizes -- and a different sequence slot in each."""

    BATCHES = (1, 8, 32)

    def __init__(self, r, T, seed):
        import online_rank_kv_b200 as ik
        self.ik = ik
        self.r, self.T = r, T
        self.caches, self.ks, self.vs = {}, {}, {}
        for B in self.BATCHES:
            cfg = _cfg(batch=B, layers=1, kv_heads=8, q_heads=32, rank_k=r, rank_v=r,
                       window=1024, max_tokens=T + 1024)
            self.caches[B] = ik.Cache(cfg)
            self.ks[B] = synth.KVStream(synth.spec_for("qwen3", "K"), B * 8, seed=seed + 2 * B,
                                        device="cuda", dtype=torch.bfloat16)
            self.vs[B] = synth.KVStream(synth.spec_for("qwen3", "V"), B * 8, seed=seed + 2 * B + 1,
                                        device="cuda", dtype=torch.bfloat16)
        self.cfg = cfg
        self.sk = synth.KVStream(synth.spec_for("qwen3", "K"), 1, seed=seed + 100, device="cuda",
                                 dtype=torch.bfloat16)
        self.sv = synth.KVStream(synth.spec_for("qwen3", "V"), 1, seed=seed + 101, device="cuda",
                                 dtype=torch.bfloat16)
        self.ok = HeadFactor(128, r, 1024, coef_round="bf16")
        self.ov = HeadFactor(128, r, 1024, coef_round="bf16")
        self.folds = 0

    def append(self, n):
        rk, rv = self.sk.next(n)[0], self.sv.next(n)[0]
        for B in self.BATCHES:
            k = self.ks[B].next(n).view(B, 8, n, 128)
            v = self.vs[B].next(n).view(B, 8, n, 128)
            k[B - 1, 7] = rk
            v[B - 1, 7] = rv
            self.caches[B].append(0, k, v)
        self.ok.append(rk.double().cpu().numpy())
        self.ov.append(rv.double().cpu().numpy())

    def prefill(self, chunk=512, defer_every=64):
        done = 0
        while done < self.T:
            n = min(chunk, self.T - done)
            self.append(n)
            done += n
            while self.ok.ready() >= 1:
                for c in self.caches.values():
                    c.compress_block(0, defer=True)
                self.ok.fold(defer=True)
                self.ov.fold(defer=True)
                self.folds += 1
                if self.folds % defer_every == 0:
                    self.sync()
        self.sync()

    def sync(self):
        for c in self.caches.values():
            c.sync(0)
        self.ok.sync()
        self.ov.sync()

    def check(self):
        ik = self.ik
        worst = 0.0
        q = synth.query_batch(4, 128, seed=self.r + self.T, dtype=torch.bfloat16)
        want = dense_decode(q.double().numpy(), self.ok.full(), self.ov.full(), 1e6)
        for B, c in self.caches.items():
            assert c.counts(0) == (self.ok.T, self.ok.n_c)
            for which, of in ((ik.WHICH_K, self.ok), (ik.WHICH_V, self.ov)):
                got = c.reconstruct(0, which)
                e = rel_err(got[B - 1, 7].cpu().numpy(), of.reconstruct())
                del got
                assert e < TOL, (B, which, e)
                worst = max(worst, e)
            qb = synth.query_batch(B * 32, 128, seed=B, dtype=torch.bfloat16).view(B, 32, 128)
            qb[B - 1, 28:32] = q
            out = c.decode_attention(0, qb.cuda())[B - 1, 28:32].cpu().numpy()
            e = rel_err(out, want)
            assert e < TOL, (B, "decode", e)
            worst = max(worst, e)
            assert c.status() == 0
        return worst

    def close(self):
        for c in self.caches.values():
            c.close()
        self.caches = {}
        torch.cuda.empty_cache()


@pytest.mark.parametrize("T", [4096, 16384, 65536, 262144])
@pytest.mark.parametrize("r", [16, 32, 64, 128])
def test_sweep_grid(r, T):
    """Every point of the one-layer sweep: ranks {16, 32, 64, 128} x contexts
    {4K, 16K, 64K, 256K} x batches {1, 8, 32}, r_K = r_V = r, W 1024, bf16
    coefficients; postponed rewrites while prefilling, as the bench does."""
    s = LockstepSweep(r, T, seed=1000 + r + T // 1024)
    s.prefill()
    s.check()
    s.close()


def test_sweep_no_sync_drift():
    """Reconstruction drift ||C B^T - K||_F / ||K||_F over the folded rows
    (pre-RoPE keys), synchronized against the ablation that leaves old
    coefficients in their old basis; the device caches and the oracle agree
    on the synchronized value."""
    import online_rank_kv_b200 as ik
    drift = {}
    for sync in (1, 0):
        cfg = _cfg(batch=1, layers=1, kv_heads=8, q_heads=32, rank_k=32, rank_v=64, window=1024,
                   max_tokens=16384 + 1024, sync=sync)
        s = SampledCache(cfg, "qwen3", [(0, 0, 3)], seed=95, sync=bool(sync))
        s.prefill(16384)
        T, n_c = s.cache.counts(0)
        rec = s.cache.reconstruct(0, ik.WHICH_K)[0, 3].cpu().double().numpy()
        K = s.ok[(0, 0, 3)].rows[:n_c]
        drift[sync] = float(np.linalg.norm(rec - K) / np.linalg.norm(K))
        if sync:
            want = s.ok[(0, 0, 3)].reconstruct()
            want_drift = float(np.linalg.norm(want - K) / np.linalg.norm(K))
            assert abs(drift[1] - want_drift) < 0.1 * want_drift + 1e-4
    assert drift[0] > 5 * drift[1], drift
