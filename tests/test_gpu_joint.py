"""Joint-head factors on the GPU against the oracle: one K and one V factor per
sequence and layer over all KV heads, their rows side by side (D = kv_heads *
128), at the explainer's worked-example ranks 64, 96 and 128.

Data: one seeded low-rank stream per sequence over the joint row (a 48-dim
latent with decaying scales shared by all heads, noise 1e-6), split into the
heads' rows for the cache and fed whole to the oracle's HeadFactor(D, r): the
truncation then has a clear spectral gap, so the two sides keep the same
subspace.  Reconstructions C B^T (each head's 128 columns) and decode outputs
are compared with the oracle's joint factor (oracle.joint_head_decode):
1e-4 with fp32 coefficients, 2e-2 with bf16 ones (tensor-core decode); the
counters are exact.
"""

import numpy as np
import pytest
import torch

import synth
from iskv_testlib import rel_err
from oracle import HeadFactor, joint_head_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _one_blas_thread():
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        yield


def _joint_stream(D, n_seq, seed, decay):
    return synth.KVStream(synth.StreamSpec(d=D, rank=48, decay=decay, noise=1e-6), n_seq, seed=seed,
                          dtype=torch.float64)


def _run(rk, rv, coef, H=8, batch=2, tokens=1280, window=256, tol=1e-4, defer=False):
    import online_rank_kv_b200 as ik
    D = H * 128
    cfg = ik.Config(batch=batch, layers=1, kv_heads=H, q_heads=4 * H, rank_k=rk, rank_v=rv,
                    window=window, max_tokens=tokens + 256, kv_dtype=ik.BF16, coef_dtype=coef,
                    use_rope=1, rope_theta=1e6, joint=1, max_deferred=8 if defer else 0)
    cache = ik.Cache(cfg)
    ks = _joint_stream(D, batch, 61, 0.9)
    vs = _joint_stream(D, batch, 62, 0.95)
    rnd = "bf16" if coef == ik.BF16 else "f32"
    ok = [HeadFactor(D, rk, window, coef_round=rnd) for _ in range(batch)]
    ov = [HeadFactor(D, rv, window, coef_round=rnd) for _ in range(batch)]
    done, folds = 0, 0
    while done < tokens:
        k = ks.next(64).to(torch.bfloat16)          # [batch, 64, D]
        v = vs.next(64).to(torch.bfloat16)
        kh = k.view(batch, 64, H, 128).permute(0, 2, 1, 3).contiguous()
        vh = v.view(batch, 64, H, 128).permute(0, 2, 1, 3).contiguous()
        ready = cache.append(0, kh.cuda(), vh.cuda())
        for b in range(batch):
            ok[b].append(k[b].double().numpy())
            ov[b].append(v[b].double().numpy())
        done += 64
        for _ in range(ready):
            cache.compress_block(0, defer=defer)
            for b in range(batch):
                ok[b].fold(defer=defer)
                ov[b].fold(defer=defer)
            folds += 1
            if defer and folds % 8 == 0:       # max_deferred postponed folds, then the rewrite
                cache.sync(0)
                for b in range(batch):
                    ok[b].sync()
                    ov[b].sync()
    if defer:
        cache.sync(0)
        for b in range(batch):
            ok[b].sync()
            ov[b].sync()
    T, n_c = cache.counts(0)
    assert (T, n_c) == (ok[0].T, ok[0].n_c) and folds >= 10
    worst = 0.0
    for which, of in ((ik.WHICH_K, ok), (ik.WHICH_V, ov)):
        got = cache.reconstruct(0, which).cpu().numpy()     # [batch, H, n_c, 128]
        for b in range(batch):
            want = of[b].reconstruct()                      # [n_c, D]
            joint = got[b].transpose(1, 0, 2).reshape(n_c, D)
            e = rel_err(joint, want)
            assert e < tol, (which, b, e)
            worst = max(worst, e)
    basis, sigma, coef_t = cache.factors(0, ik.WHICH_K)
    assert tuple(basis.shape) == (batch, D, rk) and tuple(coef_t.shape) == (batch, n_c, rk)
    Bt = basis.cpu().double().numpy()
    for b in range(batch):
        assert np.abs(Bt[b].T @ Bt[b] - np.eye(rk)).max() < 1e-5
    q = synth.query_batch(batch * 4 * H, 128, seed=63, dtype=torch.bfloat16).view(batch, 4 * H, 128)
    out = cache.decode_attention(0, q.cuda()).cpu().numpy()
    for b in range(batch):
        want = joint_head_decode(q[b].double().numpy(), ok[b].full(), ov[b].full(), H, 1e6)
        e = rel_err(out[b], want)
        assert e < tol, (b, e)
        worst = max(worst, e)
    assert cache.status() == 0
    cache.close()
    return worst


@pytest.mark.parametrize("rk,rv", [(64, 96), (96, 64)])
def test_joint_factor_fp32_paper_ranks(rk, rv):
    import online_rank_kv_b200 as ik
    _run(rk, rv, ik.F32, tol=1e-4)


def test_joint_factor_bf16_rank_128_tensor_core_decode():
    import online_rank_kv_b200 as ik
    _run(128, 128, ik.BF16, tol=2e-2)


def test_joint_factor_query_side_decode(monkeypatch):
    """The query-side RoPE kernel on joint-head factors (r_K 32, g 4: N = 128):
    each head's A_h from its 128 rows of the layer-wide basis, coefficient
    tiles shared by the sequence's heads."""
    import online_rank_kv_b200 as ik
    monkeypatch.setenv("ISKV_DECODE_KERNEL", "u")
    _run(32, 64, ik.BF16, tol=2e-2)


def test_joint_factor_postponed_rewrites_four_heads():
    import online_rank_kv_b200 as ik
    _run(64, 64, ik.BF16, H=4, batch=3, tol=2e-2, defer=True)


def test_joint_persistent_bytes():
    """Coefficients, basis (D rows) and sigma are kept once per sequence."""
    import online_rank_kv_b200 as ik
    H, batch, D = 8, 2, 1024
    cfg = ik.Config(batch=batch, layers=1, kv_heads=H, q_heads=32, rank_k=64, rank_v=96, window=256,
                    max_tokens=1024, kv_dtype=ik.BF16, coef_dtype=ik.BF16, joint=1)
    cache = ik.Cache(cfg)
    for _ in range(8):
        k = torch.randn(batch, H, 64, 128, dtype=torch.bfloat16, device="cuda")
        ready = cache.append(0, k, k.clone())
        for _ in range(ready):
            cache.compress_block(0)
    T, n_c = cache.counts(0)
    kept, full = cache.kv_bytes()
    want = batch * (n_c * (64 + 96) * 2 + (D + 1) * (64 + 96) * 4) + batch * H * 2 * (T - n_c) * 128 * 2
    assert (kept, full) == (want, batch * H * 2 * T * 128 * 2)
    cache.close()
