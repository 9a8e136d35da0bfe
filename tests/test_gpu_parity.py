"""GPU parity: the CUDA library against the float64 oracle, element by element.

Tolerances (max |a - b| / max |b| per compared tensor and head): 1e-4 where
the coefficients are stored in fp32, 2e-2 where they are stored in bf16 (the
oracle emulates the bf16 storage at the same points).  Window and block
counters must match exactly.  Singular vectors are compared only through
basis-invariant quantities: reconstructions C B^T, projectors onto leading
well-separated columns, and decode outputs.
"""

import numpy as np
import pytest
import torch

from iskv_testlib import Pair, rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def _ik():
    import online_rank_kv_b200 as ik
    return ik


def tiny_cfg(**kw):
    ik = _ik()
    c = ik.Config(batch=1, layers=1, kv_heads=1, q_heads=1, rank_k=16, rank_v=16, window=128,
                  max_tokens=1024 + 64 + 64, kv_dtype=ik.F32, coef_dtype=ik.F32, use_rope=0)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def qwen_cfg(**kw):
    ik = _ik()
    c = ik.Config(batch=1, layers=1, kv_heads=8, q_heads=32, rank_k=32, rank_v=64, window=1024,
                  max_tokens=16384 + 256, kv_dtype=ik.BF16, coef_dtype=ik.F32, use_rope=1,
                  rope_theta=1e6)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_tiny_single_head_1024_then_64_decode_steps():
    """One head, d=128, r=16, W=128, fp32, no RoPE; rank-8 signal + 1e-3 noise.
    1024 tokens, then 64 decode steps each appending one token."""
    p = Pair(tiny_cfg(), "tiny", seed=0)
    p.prefill(1024, chunk=64)
    p.check_counts()
    assert p.cache.counts(0) == (1024, 896)
    for k, e in p.recon_errors(0).items():
        assert e < TOL_F32, (k, e)
    worst = 0.0
    for step in range(64):
        p.append(1)
        p.fold_ready()
        errs, _ = p.decode(0, p.query())
        worst = max(worst, max(errs.values()))
        p.check_counts()
    assert p.cache.counts(0) == (1088, 960)
    assert worst < TOL_F32, worst
    for k, e in p.recon_errors(0).items():
        assert e < TOL_F32, (k, e)
    assert p.cache.status() == 0


def test_tiny_signal_projector_matches_oracle():
    """The 8 signal directions are separated from the noise by ~1000x: the
    projector onto the leading 8 basis columns is basis-invariant."""
    ik = _ik()
    p = Pair(tiny_cfg(), "tiny", seed=3)
    p.prefill(1024)
    basis, sigma, _ = p.cache.factors(0, ik.WHICH_K)
    Bg = basis[0, 0].cpu().double().numpy()
    Bo = p.ok[(0, 0, 0)].B
    Pg = Bg[:, :8] @ Bg[:, :8].T
    Po = Bo[:, :8] @ Bo[:, :8].T
    assert np.abs(Pg - Po).max() < 1e-5
    assert np.abs(Bg.T @ Bg - np.eye(16)).max() < 1e-5
    assert rel_err(sigma[0, 0].cpu().numpy(), p.ok[(0, 0, 0)].S) < 1e-5


@pytest.mark.parametrize("T", [64 * 5 + 17, 2048 + 33])
def test_qwen_layer_short_ragged(T):
    """8 KV / 32 Q heads, r_K 32, r_V 64, bf16 K/V, fp32 C, RoPE; a context
    that is not a multiple of 64 and (for the first case) shorter than W."""
    p = Pair(qwen_cfg(max_tokens=4096), "qwen3", seed=1)
    p.prefill(T, chunk=128)
    p.check_counts()
    for k, e in p.recon_errors(0).items():
        assert e < TOL_F32, (k, e)
    for _ in range(3):
        p.append(1)
        p.fold_ready()
        errs, _ = p.decode(0, p.query())
        assert max(errs.values()) < TOL_F32, errs


def test_qwen_layer_16k_full_size():
    """The one-layer 16K-context workload at full size: 240 folds per head."""
    p = Pair(qwen_cfg(), "qwen3", seed=2)
    p.prefill(16384, chunk=512)
    p.check_counts()
    assert p.cache.counts(0) == (16384, 15360)
    rec = p.recon_errors(0)
    assert max(rec.values()) < TOL_F32, max(rec.items(), key=lambda x: x[1])
    errs, _ = p.decode(0, p.query())
    assert max(errs.values()) < TOL_F32, errs
    assert p.cache.status() == 0


@pytest.mark.parametrize("defer_every", [0, 8])
def test_bf16_coefficients_multi_layer(defer_every):
    """bf16-stored coefficients over two layers and batch 2; with postponed
    rewrites (prefill) or a rewrite at every fold."""
    ik = _ik()
    cfg = qwen_cfg(batch=2, layers=2, kv_heads=2, q_heads=8, window=256, max_tokens=3072,
                   coef_dtype=ik.BF16, max_deferred=8 if defer_every else 0)
    p = Pair(cfg, "qwen3", seed=4)
    p.prefill(2048 + 40, chunk=256, defer_every=defer_every)
    p.check_counts()
    for l in range(2):
        for k, e in p.recon_errors(l).items():
            assert e < TOL_BF16, (l, k, e)
    for _ in range(2):
        p.append(1)
        p.fold_ready()
        for l in range(2):
            errs, _ = p.decode(l, p.query())
            assert max(errs.values()) < TOL_BF16, errs


@pytest.mark.parametrize("rk,rv", [(64, 96), (128, 128), (16, 48)])
def test_rank_edge_cases(rk, rv):
    """r + 64 > d (k = d - r < 64) and r = d (k = 0, lossless)."""
    cfg = qwen_cfg(kv_heads=2, q_heads=8, rank_k=rk, rank_v=rv, window=256, max_tokens=2048)
    p = Pair(cfg, "qwen3", seed=5)
    p.prefill(1024 + 64 * 3 + 5, chunk=64)
    for k, e in p.recon_errors(0).items():
        assert e < TOL_F32, (k, e)
    errs, _ = p.decode(0, p.query())
    assert max(errs.values()) < TOL_F32, errs
    if rk == 128:
        # lossless: the rebuilt keys are the appended keys
        ik = _ik()
        rec = p.cache.reconstruct(0, ik.WHICH_K).cpu().double().numpy()
        for (l, b, h) in p.heads:
            X = p.ok[(l, b, h)].rows[:rec.shape[2]]
            assert rel_err(rec[b, h], X) < 1e-5


def test_rank_deficient_cores():
    """Exactly rank-8 keys and rank-1 values without noise at r = 16: the core
    has numerically zero singular values among the kept r, whose directions
    an orthonormal completion represents.  Reconstructions stay exact
    (rank <= r) and the bases orthonormal."""
    import dataclasses

    import synth
    ik = _ik()
    exact8 = dataclasses.replace(synth.spec_for("tiny", "K"), noise=0.0)
    exact1 = dataclasses.replace(synth.spec_for("tiny", "V"), noise=0.0, decay=0.0)
    p = Pair(tiny_cfg(), "tiny", seed=9, specs=(exact8, exact1))
    p.prefill(1024, chunk=64)
    p.check_counts()
    for k, e in p.recon_errors(0).items():
        assert e < TOL_F32, (k, e)
    for which, of in ((ik.WHICH_K, p.ok), (ik.WHICH_V, p.ov)):
        rec = p.cache.reconstruct(0, which).cpu().double().numpy()
        X = of[(0, 0, 0)].rows[:rec.shape[2]]
        assert rel_err(rec[0, 0], X) < 1e-5
        basis, sigma, coef = p.cache.factors(0, which)
        Bg = basis[0, 0].cpu().double().numpy()
        assert np.isfinite(Bg).all() and np.isfinite(coef.cpu().numpy()).all()
        assert np.abs(Bg.T @ Bg - np.eye(16)).max() < 1e-5
    errs, _ = p.decode(0, p.query())
    assert max(errs.values()) < TOL_F32, errs
    assert p.cache.status() == 0


def test_all_zero_stream():
    """All-zero keys and values: every singular value of every core is zero,
    the reconstruction is exactly zero and the bases stay orthonormal."""
    ik = _ik()
    cfg = tiny_cfg(rank_k=32, rank_v=64)
    cache = ik.Cache(cfg)
    z = torch.zeros(1, 1, 64, 128, device="cuda")
    for _ in range(8):
        for _ in range(cache.append(0, z, z)):
            cache.compress_block(0)
    assert cache.counts(0) == (512, 384)
    for which, r in ((ik.WHICH_K, 32), (ik.WHICH_V, 64)):
        rec = cache.reconstruct(0, which)
        assert torch.isfinite(rec).all() and rec.abs().max().item() == 0.0
        basis, sigma, coef = cache.factors(0, which)
        Bg = basis[0, 0].cpu().double().numpy()
        assert np.abs(Bg.T @ Bg - np.eye(r)).max() < 1e-5
        assert sigma.abs().max().item() == 0.0
    q = torch.randn(1, 1, 128, device="cuda")
    out = cache.decode_attention(0, q)
    assert torch.isfinite(out).all() and out.abs().max().item() == 0.0
    assert cache.status() == 0


def test_no_sync_ablation():
    """The no-synchronization ablation keeps every old coefficient row in the
    basis it was written in.  Reading such rows in a later basis is not
    basis-invariant: it depends on the sign and rotation choices of each core
    SVD, which differ between any two correct SVD codes.  So only what is
    unique is compared with the oracle's ablation: the stored rows' norms (a
    row is never rewritten, and its norm is that of the block's projection at
    its fold), the singular values, and the newest block's reconstruction
    (written in the current basis).  The basis itself must be identical to the
    synchronized cache's (the fold does not read C), and the drift against the
    appended rows must be clearly larger than with synchronization."""
    ik = _ik()
    cfg_s = qwen_cfg(kv_heads=2, q_heads=8, window=128, max_tokens=2048)
    cfg_n = qwen_cfg(kv_heads=2, q_heads=8, window=128, max_tokens=2048, sync=0)
    ps = Pair(cfg_s, "qwen3", seed=6)
    pn = Pair(cfg_n, "qwen3", seed=6)
    ps.prefill(1536)
    pn.prefill(1536)
    for which, of_s, of_n in ((ik.WHICH_K, ps.ok, pn.ok), (ik.WHICH_V, ps.ov, pn.ov)):
        bs, ss, _ = ps.cache.factors(0, which)
        bn, sn, cn = pn.cache.factors(0, which)
        assert torch.equal(bs, bn) and torch.equal(ss, sn)
        rs = ps.cache.reconstruct(0, which).cpu().double().numpy()
        rn = pn.cache.reconstruct(0, which).cpu().double().numpy()
        cn = cn.cpu().double().numpy()
        for (l, b, h) in ps.heads:
            X = of_s[(l, b, h)].rows[:rs.shape[2]]
            ds = np.linalg.norm(rs[b, h] - X) / np.linalg.norm(X)
            dn = np.linalg.norm(rn[b, h] - X) / np.linalg.norm(X)
            assert dn > 1.5 * ds, (which, ds, dn)
            fn = of_n[(l, b, h)]
            assert rel_err(np.linalg.norm(cn[b, h], axis=1), np.linalg.norm(fn.C, axis=1)) < TOL_F32
            assert rel_err(sn[b, h].cpu().numpy(), fn.S) < TOL_F32
            last = slice(fn.n_c - 64, fn.n_c)
            assert rel_err(rn[b, h][last], (fn.C @ fn.B.T)[last]) < TOL_F32


def test_decode_before_any_fold_and_host_buffers():
    """All rows exact (T < W + 64); k/v/q/out in host memory go through the
    library's staging path and give the same answer as device buffers."""
    ik = _ik()
    cfg = qwen_cfg(kv_heads=2, q_heads=8, window=512, max_tokens=1024)
    p = Pair(cfg, "qwen3", seed=7)
    p.prefill(300, chunk=100)
    assert p.cache.counts(0) == (300, 0)
    q = p.query()
    errs, out_dev = p.decode(0, q)
    assert max(errs.values()) < TOL_F32
    out_host = torch.empty(cfg.batch, cfg.q_heads, cfg.head_dim, dtype=torch.float32).pin_memory()
    p.cache.decode_attention(0, q.cpu(), out=out_host)
    torch.cuda.synchronize()
    assert np.array_equal(out_host.numpy(), out_dev)
    # host-memory append (pageable) then decode again
    k = torch.randn(cfg.batch, cfg.kv_heads, 5, cfg.head_dim).to(torch.bfloat16)
    v = torch.randn(cfg.batch, cfg.kv_heads, 5, cfg.head_dim).to(torch.bfloat16)
    p.cache.append(0, k, v)
    for (l, b, h) in p.heads:
        p.ok[(l, b, h)].append(k[b, h].double().numpy())
        p.ov[(l, b, h)].append(v[b, h].double().numpy())
    errs, _ = p.decode(0, p.query())
    assert max(errs.values()) < TOL_F32


def _offset_view(x: torch.Tensor, elems: int, device=None, pinned=False) -> torch.Tensor:
    """A contiguous copy of x that starts `elems` elements into a fresh buffer
    (an odd offset puts it off the 16-byte alignment)."""
    buf = torch.zeros(x.numel() + 16, dtype=x.dtype, device=device)
    if pinned:
        buf = buf.pin_memory()
    view = buf[elems:elems + x.numel()].view(x.shape)
    view.copy_(x)
    return view


BUFFER_KINDS = {
    "pageable": lambda x: x.clone(),
    "pinned": lambda x: x.pin_memory(),
    "pinned, unaligned": lambda x: _offset_view(x, 1, pinned=True),
    "device, unaligned": lambda x: _offset_view(x, 1, device="cuda"),
}


@pytest.mark.parametrize("coef", ["f32", "bf16"])
def test_caller_buffers_of_every_kind(coef):
    """Page-locked host buffers are read and written in place by the library's
    kernels; pageable ones, another alignment than 16 bytes (host or device)
    and device buffers the bulk copies cannot take are staged.  Rows appended
    from every kind reach the oracle's factors, and the decode writes the same
    output bits into every kind of buffer from every kind of query buffer."""
    ik = _ik()
    cfg = qwen_cfg(kv_heads=2, q_heads=8, window=256, max_tokens=2048,
                   coef_dtype=ik.F32 if coef == "f32" else ik.BF16)
    tol = TOL_F32 if coef == "f32" else TOL_BF16
    p = Pair(cfg, "qwen3", seed=11)
    p.prefill(600, chunk=100)
    g = torch.Generator().manual_seed(3)
    for kind, make in BUFFER_KINDS.items():
        for t in (1, 37):
            k = torch.randn(cfg.batch, cfg.kv_heads, t, cfg.head_dim, generator=g).to(torch.bfloat16)
            v = torch.randn(cfg.batch, cfg.kv_heads, t, cfg.head_dim, generator=g).to(torch.bfloat16)
            kx, vx = make(k), make(v)
            p.cache.append(0, kx, vx)
            torch.cuda.synchronize()        # the sources outlive the enqueued reads
            for (l, b, h) in p.heads:
                p.ok[(l, b, h)].append(k[b, h].double().numpy())
                p.ov[(l, b, h)].append(v[b, h].double().numpy())
            p.fold_ready()
    p.check_counts()
    assert p.cache.counts(0)[1] > 0
    q = p.query()
    errs, out_dev = p.decode(0, q)
    assert max(errs.values()) < tol, errs
    out_kinds = dict(BUFFER_KINDS, device=lambda x: x.cuda())
    for qkind, make_q in BUFFER_KINDS.items():
        for okind, make_o in out_kinds.items():
            qx = make_q(q)
            ox = make_o(torch.full(tuple(q.shape), float("nan"), dtype=torch.float32))
            p.cache.decode_attention(0, qx, out=ox)
            torch.cuda.synchronize()
            assert np.array_equal(ox.cpu().numpy(), out_dev), (qkind, okind)
    assert p.cache.status() == 0


def test_error_codes():
    ik = _ik()
    cfg = qwen_cfg(kv_heads=1, q_heads=4, window=128, max_tokens=1024)   # ring: 128 + 128 rows
    c = ik.Cache(cfg)
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 200, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ik.IskvError) as e:       # empty cache
        c.decode_attention(0, q)
    assert e.value.name == "STATE"
    with pytest.raises(ik.IskvError) as e:       # nothing to fold
        c.compress_block(0)
    assert e.value.name == "STATE"
    assert c.append(0, k, k) == 1                # (200 - 128) // 64
    with pytest.raises(ik.IskvError) as e:       # the exact-window ring would overflow
        c.append(0, k[:, :, :100], k[:, :, :100])
    assert e.value.name == "CAPACITY"
    assert c.counts(0) == (200, 0)               # a refused call changes nothing
    assert c.append(0, k[:, :, :56], k[:, :, :56]) == 2
    c.compress_block(0)
    c.compress_block(0)
    assert c.counts(0) == (256, 128)
    with pytest.raises(ik.IskvError) as e:       # postponing not enabled
        c.append(0, k[:, :, :64], k[:, :, :64])
        c.compress_block(0, defer=True)
    assert e.value.name == "STATE"
    small = ik.Cache(qwen_cfg(kv_heads=1, q_heads=4, window=128, max_tokens=100))
    with pytest.raises(ik.IskvError) as e:       # max_tokens
        small.append(0, k[:, :, :101], k[:, :, :101])
    assert e.value.name == "CAPACITY"
    with pytest.raises(ik.IskvError) as e:
        c.append(3, k, k)
    assert e.value.name == "INVALID_ARG"
    assert c.status() == 0


def test_jacobi_sweep_limit_reports_noconverge():
    """A sweep limit of 1 cannot converge: the sticky status says so, the
    results stay finite, and nothing hangs."""
    ik = _ik()
    cfg = qwen_cfg(kv_heads=1, q_heads=4, window=128, max_tokens=512, jacobi_max_sweeps=1)
    p = Pair(cfg, "qwen3", seed=8)
    p.prefill(256)
    assert p.cache.status() == -5   # ISKV_ERR_NOCONVERGE
    rec = p.cache.reconstruct(0, ik.WHICH_K)
    assert torch.isfinite(rec).all()
