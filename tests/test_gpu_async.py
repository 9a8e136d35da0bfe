"""Asynchronous block updates: a layer's fold and rewrite on a second stream.

Two caches see the same rows and queries.  One folds on the caller's stream
(iskv_compress_block), the other enqueues each layer's update on a side stream
right after that layer's decode (iskv_compress_block_async) and keeps decoding
the other layers meanwhile.  The library orders the next call that touches an
updated layer after its update, so every decode output, the counters and the
final reconstructions must agree bit for bit: same kernels, same inputs.
"""

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _pair_of_caches(**kw):
    import online_rank_kv_b200 as ik
    cfg = ik.Config(batch=2, layers=3, kv_heads=2, q_heads=8, rank_k=32, rank_v=64, window=256,
                    max_tokens=4096, kv_dtype=ik.BF16, coef_dtype=ik.BF16, use_rope=1,
                    rope_theta=1e6, max_deferred=8)
    for k, v in kw.items():
        setattr(cfg, k, v)
    return cfg, ik.Cache(cfg), ik.Cache(cfg)


@pytest.mark.parametrize("protect", [0, 70])
def test_async_updates_match_synchronous_ones_bit_for_bit(protect):
    import online_rank_kv_b200 as ik
    cfg, a, b = _pair_of_caches(protect=protect)
    L, B, H, Hq, D = cfg.layers, cfg.batch, cfg.kv_heads, cfg.q_heads, cfg.head_dim
    ks = synth.KVStream(synth.spec_for("qwen3", "K"), L * B * H, seed=11, device="cuda",
                        dtype=torch.bfloat16)
    vs = synth.KVStream(synth.spec_for("qwen3", "V"), L * B * H, seed=12, device="cuda",
                        dtype=torch.bfloat16)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()

    def ready(c, l):
        T, n_c = c.counts(l)
        return (max(0, T - protect) - n_c - cfg.window) // 64

    # prefill both the same way (synchronous folds)
    for _ in range(12):
        k = ks.next(64).view(L, B, H, 64, D)
        v = vs.next(64).view(L, B, H, 64, D)
        for l in range(L):
            for c in (a, b):
                c.append(l, k[l].contiguous(), v[l].contiguous())
                while ready(c, l) >= 1:
                    c.compress_block(l)
    n_async = 0
    for step in range(200):
        k = ks.next(1).view(L, B, H, 1, D)
        v = vs.next(1).view(L, B, H, 1, D)
        q = synth.query_batch(L * B * Hq, D, seed=500 + step, device="cuda",
                              dtype=torch.bfloat16).view(L, B, Hq, D)
        for l in range(L):
            outs = []
            for c in (a, b):
                c.append(l, k[l].contiguous(), v[l].contiguous())
                outs.append(c.decode_attention(l, q[l].contiguous()))
            assert torch.equal(outs[0], outs[1]), (step, l)
            # the layer's block update right after its decode: synchronous on
            # one cache, on the side stream on the other
            if ready(a, l) >= 1:
                a.compress_block(l)
                b.compress_block_async(l, side, after=main)
                n_async += 1
    assert n_async >= 2 * L
    torch.cuda.synchronize()
    for l in range(L):
        assert a.counts(l) == b.counts(l)
        for which in (ik.WHICH_K, ik.WHICH_V):
            assert torch.equal(a.reconstruct(l, which), b.reconstruct(l, which))
    assert a.status() == 0 and b.status() == 0


def test_async_update_with_postponed_rewrite_then_sync():
    """An asynchronous fold that postpones its rewrite, then iskv_sync on the
    caller's stream: ordered after the fold, same result as synchronous."""
    import online_rank_kv_b200 as ik
    cfg, a, b = _pair_of_caches(layers=1)
    D = cfg.head_dim
    ks = synth.KVStream(synth.spec_for("qwen3", "K"), cfg.batch * cfg.kv_heads, seed=21,
                        device="cuda", dtype=torch.bfloat16)
    vs = synth.KVStream(synth.spec_for("qwen3", "V"), cfg.batch * cfg.kv_heads, seed=22,
                        device="cuda", dtype=torch.bfloat16)
    side = torch.cuda.Stream()
    for _ in range(5):
        k = ks.next(128).view(cfg.batch, cfg.kv_heads, 128, D)
        v = vs.next(128).view(cfg.batch, cfg.kv_heads, 128, D)
        for c in (a, b):
            c.append(0, k, v)
        while True:
            T, n_c = a.counts(0)
            if (T - n_c - cfg.window) // 64 < 1:
                break
            a.compress_block(0, defer=True)
            b.compress_block_async(0, side, defer=True)
    a.sync(0)
    b.sync(0)
    torch.cuda.synchronize()
    assert a.counts(0) == b.counts(0) and a.counts(0)[1] > 0
    for which in (ik.WHICH_K, ik.WHICH_V):
        assert torch.equal(a.reconstruct(0, which), b.reconstruct(0, which))
    q = synth.query_batch(cfg.batch * cfg.q_heads, D, seed=9, device="cuda",
                          dtype=torch.bfloat16).view(cfg.batch, cfg.q_heads, D)
    assert np.array_equal(a.decode_attention(0, q).cpu().numpy(), b.decode_attention(0, q).cpu().numpy())


def test_async_updates_against_the_oracle():
    """The asynchronous path against the float64 oracle, not only against the
    synchronous cache: every layer folds on the side stream right after its
    decode, and the decode outputs and reconstructions of sampled heads stay
    within the bf16-coefficient tolerance of dense attention over the
    oracle's factors (which fold at the same points)."""
    import online_rank_kv_b200 as ik
    from iskv_testlib import SampledCache, rel_err
    from oracle import dense_decode

    cfg = ik.Config(batch=2, layers=3, kv_heads=2, q_heads=8, rank_k=32, rank_v=64, window=256,
                    max_tokens=4096, kv_dtype=ik.BF16, coef_dtype=ik.BF16, use_rope=1,
                    rope_theta=1e6, max_deferred=8, ring_extra=512)
    sample = [(0, 0, 0), (1, 1, 1), (2, 0, 1), (2, 1, 0)]
    s = SampledCache(cfg, "qwen3", sample, seed=33)
    s.prefill(1024, chunk=256, defer_every=0)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    g = cfg.q_heads // cfg.kv_heads
    worst, n_async, checks = 0.0, 0, 0
    for step in range(160):
        s.append(1)
        q = synth.query_batch(cfg.layers * cfg.batch * cfg.q_heads, cfg.head_dim, seed=900 + step,
                              dtype=torch.bfloat16).view(cfg.layers, cfg.batch, cfg.q_heads,
                                                         cfg.head_dim)
        for l in range(cfg.layers):
            out = s.cache.decode_attention(l, q[l].contiguous().cuda())
            if step % 8 == 0:
                got = out.cpu().numpy()
                qn = q[l].double().numpy()
                for (ll, b, h) in sample:
                    if ll != l:
                        continue
                    want = dense_decode(qn[b, h * g:(h + 1) * g], s.ok[(ll, b, h)].full(),
                                        s.ov[(ll, b, h)].full(), cfg.rope_theta)
                    worst = max(worst, rel_err(got[b, h * g:(h + 1) * g], want))
                    checks += 1
            T, n_c = s.cache.counts(l)
            if (T - n_c - cfg.window) // 64 >= 1:
                s.cache.compress_block_async(l, side, after=main)
                for x in sample:
                    if x[0] == l:
                        s.ok[x].fold()
                        s.ov[x].fold()
                n_async += 1
    assert n_async >= 2 * cfg.layers and checks > 0
    assert worst < 2e-2, worst
    s.check(tol=2e-2)
    assert s.cache.status() == 0
