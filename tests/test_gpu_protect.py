"""GPU parity with protected rows: positions 0..P-1 kept exact, never folded.

The CUDA cache and the float64 oracle see the same appended rows; the
protected count P is not a multiple of the 64-row block in most cases, so
appends cross P inside a chunk and the protected rows end in a partial tile.
Both decode paths are covered: the CUDA-core split-K kernel (fp32
coefficients) and the tensor-core kernel (bf16 coefficients).  Tolerances as
in the other parity tests; counters exact.  Also checks the persistent-KV
byte count of the library against the oracle's.
"""

import numpy as np
import pytest
import torch

from iskv_testlib import Pair
from oracle import full_kv_bytes, persistent_kv_bytes

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def _cfg(**kw):
    import online_rank_kv_b200 as ik
    c = ik.Config(batch=2, layers=1, kv_heads=2, q_heads=8, rank_k=32, rank_v=64, window=256,
                  max_tokens=4096, kv_dtype=ik.BF16, coef_dtype=ik.F32, use_rope=1,
                  rope_theta=1e6)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("coef", ["f32", "bf16", "bf16-u"])
@pytest.mark.parametrize("P", [1, 37, 64, 100, 300])
def test_protected_rows_parity(P, coef, monkeypatch):
    """bf16-u: the query-side RoPE kernel, whose position table has a second
    part for the protected positions and whose folded rows sit at P + j."""
    import online_rank_kv_b200 as ik
    if coef == "bf16-u":
        monkeypatch.setenv("ISKV_DECODE_KERNEL", "u")
    cdt = ik.F32 if coef == "f32" else ik.BF16
    tol = TOL_F32 if coef == "f32" else TOL_BF16
    p = Pair(_cfg(protect=P, coef_dtype=cdt), "qwen3", seed=200 + P)
    p.prefill(P + 1500 + 33, chunk=128)
    p.check_counts()
    T, n_c = p.cache.counts(0)
    assert n_c == ((T - P - 256) // 64) * 64 > 0
    for k, e in p.recon_errors(0).items():
        assert e < tol, (k, e)
    for _ in range(3):
        p.append(1)
        p.fold_ready()
        errs, _ = p.decode(0, p.query())
        assert max(errs.values()) < tol, errs
    assert p.cache.status() == 0


@pytest.mark.parametrize("coef", ["f32", "bf16", "bf16-u"])
def test_decode_while_only_protected_rows(coef, monkeypatch):
    """T below P: every row is a protected row (no window, nothing folded),
    then the stream crosses P and the first blocks fold."""
    import online_rank_kv_b200 as ik
    if coef == "bf16-u":
        monkeypatch.setenv("ISKV_DECODE_KERNEL", "u")
    cdt = ik.F32 if coef == "f32" else ik.BF16
    tol = TOL_F32 if coef == "f32" else TOL_BF16
    P = 300
    p = Pair(_cfg(protect=P, coef_dtype=cdt), "qwen3", seed=310)
    p.prefill(200, chunk=70)
    assert p.cache.counts(0) == (200, 0)
    errs, _ = p.decode(0, p.query())
    assert max(errs.values()) < tol, errs
    p.prefill(P + 256 + 64 * 2 + 5 - 200, chunk=90)
    p.check_counts()
    assert p.cache.counts(0)[1] == 128
    errs, _ = p.decode(0, p.query())
    assert max(errs.values()) < tol, errs


def test_protected_rows_from_host_memory():
    """Host (pageable) K/V go through the staging path; the split between
    protected rows and the window ring is the same as for device inputs."""
    P = 50
    cfg = _cfg(protect=P)
    p = Pair(cfg, "qwen3", seed=320)
    g = torch.Generator().manual_seed(5)
    for n in (30, 45, 300, 100, 7):
        k = torch.randn(cfg.batch, cfg.kv_heads, n, cfg.head_dim, generator=g).to(torch.bfloat16)
        v = torch.randn(cfg.batch, cfg.kv_heads, n, cfg.head_dim, generator=g).to(torch.bfloat16)
        p.cache.append(0, k, v)
        for (l, b, h) in p.heads:
            p.ok[(l, b, h)].append(k[b, h].double().numpy())
            p.ov[(l, b, h)].append(v[b, h].double().numpy())
        p.fold_ready()
    p.check_counts()
    errs, _ = p.decode(0, p.query())
    assert max(errs.values()) < TOL_F32, errs


@pytest.mark.parametrize("P", [0, 100])
def test_kv_bytes_match_the_oracle_count(P):
    import online_rank_kv_b200 as ik
    cfg = _cfg(protect=P, coef_dtype=ik.BF16, layers=2)
    p = Pair(cfg, "qwen3", seed=330)
    assert p.cache.kv_bytes() == (0, 0)
    p.prefill(P + 256 + 64 * 5 + 11, chunk=128)
    kept, full = p.cache.kv_bytes()
    want_kept = 0
    for (l, b, h) in p.heads:
        fk, fv = p.ok[(l, b, h)], p.ov[(l, b, h)]
        want_kept += persistent_kv_bytes(fk.n_c, fk.exact().shape[0], 128, cfg.rank_k, cfg.rank_v,
                                         2, 2, 4, n_p=fk.protected().shape[0])
    T, _ = p.cache.counts(0)
    assert kept == want_kept
    assert full == full_kv_bytes(T, cfg.layers, cfg.batch * cfg.kv_heads, 128, 2)
    assert full / kept > 1.0
