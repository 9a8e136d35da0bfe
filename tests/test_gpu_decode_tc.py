"""Tensor-core decode over the folded rows (bf16 coefficients) against the
float64 oracle (bf16 storage emulated) and against the CUDA-core decode on an
identical cache.  Covers the shapes the kernel's layouts depend on: value MMA
with M=64 and M=128 (r_V <= 64 and > 64), r = d, the smallest ranks, query
groups 1..8, no exact rows at all, CTAs whose tile ranges span several heads,
and sharply peaked ("recall") queries aimed at a folded token.
"""

import os

import numpy as np
import pytest
import torch

import synth
from iskv_testlib import Pair, rel_err

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def _cfg(**kw):
    import online_rank_kv_b200 as ik
    c = ik.Config(batch=2, layers=1, kv_heads=2, q_heads=8, rank_k=32, rank_v=64, window=256,
                  max_tokens=4096, kv_dtype=ik.BF16, coef_dtype=ik.BF16, use_rope=1,
                  rope_theta=1e6, max_deferred=8)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _pair(tc: bool, cfg, seed, kernel=None):
    """A cache built with the tensor-core decode on or off; `kernel` picks the
    tensor-core decode: "u" the query-side RoPE kernel (r_K g <= 128), "rot"
    the kernel that rebuilds and rotates the keys, None the library's default."""
    env = {"ISKV_TENSOR_CORES": "1" if tc else "0", "ISKV_DECODE_KERNEL": kernel}
    old = {k: os.environ.get(k) for k in env}
    for k, v in env.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v
    try:
        return Pair(cfg, "qwen3", seed=seed)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


@pytest.mark.parametrize("rk,rv,g,W,T,kernel", [
    (32, 64, 4, 256, 2048 + 40, "u"),      # query-side RoPE kernel (r_K g = 128)
    (32, 64, 4, 256, 2048 + 40, "rot"),    # the same shape through the rotation kernel
    (64, 96, 4, 256, 1500, None),          # r_K g = 256: rotation kernel
    (128, 128, 2, 128, 900, None),
    (16, 16, 1, 128, 700, "u"),            # query-side, g = 1, N = 16
    (16, 16, 1, 128, 700, "rot"),
    (64, 64, 2, 128, 900, "u"),            # query-side, g = 2
    (16, 32, 8, 0, 1024, "u"),             # query-side, g = 8, no exact rows
    (32, 48, 8, 0, 1024, None),            # r_K g = 256: rotation kernel
])
def test_tc_decode_matches_oracle_and_cuda_core(rk, rv, g, W, T, kernel):
    cfg = _cfg(rank_k=rk, rank_v=rv, q_heads=2 * g, window=W, max_tokens=T + 256)
    pt = _pair(True, cfg, seed=31 + rk + rv, kernel=kernel)
    pc = _pair(False, cfg, seed=31 + rk + rv)
    pt.prefill(T, chunk=64, defer_every=8)
    pc.prefill(T, chunk=64, defer_every=8)
    T_, n_c = pt.cache.counts(0)
    assert n_c > 0
    for _ in range(2):
        q = pt.query()
        errs, out_t = pt.decode(0, q)
        out_c = pc.cache.decode_attention(0, q.cuda()).cpu().numpy()
        assert max(errs.values()) < TOL_BF16, errs
        assert rel_err(out_t, out_c) < 5e-3
    assert pt.cache.status() == 0


@pytest.mark.parametrize("kernel", ["rot", "u"])
def test_tc_decode_ctas_span_heads(kernel):
    """64 (sequence, KV head) pairs with 3 tiles each: 192 tiles on 148 SMs,
    so most CTAs cover parts of two heads."""
    cfg = _cfg(batch=8, kv_heads=8, q_heads=32, window=128, max_tokens=1024)
    p = _pair(True, cfg, seed=41, kernel=kernel)
    p.prefill(128 + 3 * 128 - 64 + 17, chunk=64)
    T, n_c = p.cache.counts(0)
    assert n_c == 320                       # 2.5 tiles: last tile half full
    errs, _ = p.decode(0, p.query())
    assert max(errs.values()) < TOL_BF16, errs
    assert p.cache.status() == 0


@pytest.mark.parametrize("kernel", ["rot", "u"])
def test_tc_decode_recall_query(kernel):
    """A query aimed at one folded token (its score ~25 above the rest):
    the sharpest attention the decode has to reproduce."""
    cfg = _cfg(kv_heads=2, q_heads=8, window=256)
    p = _pair(True, cfg, seed=43, kernel=kernel)
    p.prefill(2048)
    q = p.query().double()
    pos = 333
    for b in range(cfg.batch):
        for h in range(cfg.kv_heads):
            kp = torch.from_numpy(p.ok[(0, b, h)].reconstruct()[pos])
            # score of token pos = beta |k| / sqrt(d) = 25
            beta = 25.0 * np.sqrt(128) / float(torch.linalg.vector_norm(kp))
            for j in range(4):
                q[b, h * 4 + j] = synth.recall_query(kp, pos, cfg.rope_theta, beta)
    q = q.to(torch.bfloat16)
    errs, _ = p.decode(0, q)
    assert max(errs.values()) < TOL_BF16, errs


@pytest.mark.parametrize("kernel", ["rot", "u"])
def test_tc_decode_without_folded_rows(kernel):
    """Nothing folded yet (T < W + 64): only exact-row tiles, including a
    ragged last tile, go through the tensor-core kernel."""
    cfg = _cfg(window=512, max_tokens=1024)
    pt = _pair(True, cfg, seed=47, kernel=kernel)
    pc = _pair(False, cfg, seed=47)
    pt.prefill(300, chunk=100)
    pc.prefill(300, chunk=100)
    assert pt.cache.counts(0) == (300, 0)
    q = pt.query()
    errs, out_t = pt.decode(0, q)
    out_c = pc.cache.decode_attention(0, q.cuda()).cpu().numpy()
    assert max(errs.values()) < 1e-3, errs
    assert rel_err(out_t, out_c) < 5e-3


def test_tc_decode_single_basis_buffer_heads_split_across_runs():
    """r_K 64, r_V 96 leave room for one basis buffer; at this shape (16 heads
    of 49 tiles on 148 SMs) eight CTA runs end with a head of which they hold
    a single tile, so one epilogue group has no tile there.  That group's
    release of the basis buffer must stay behind the producer's refill (an
    early second release would look like no release to the producer's parity
    wait): the decode completes with status OK and matches the oracle."""
    cfg = _cfg(batch=2, kv_heads=8, q_heads=32, rank_k=64, rank_v=96, window=256,
               max_tokens=6144)
    p = _pair(True, cfg, seed=49)
    p.prefill(5864, chunk=64, defer_every=16)
    T, n_c = p.cache.counts(0)
    assert (T, n_c) == (5864, 5568)
    for _ in range(2):
        errs, _ = p.decode(0, p.query())
        assert max(errs.values()) < TOL_BF16, errs
    assert p.cache.status() == 0


def test_decode_kernel_choice(monkeypatch):
    """iskv_decode_kernel names the kernel the next decode call runs: the
    CUDA-core kernel for fp32 coefficients or with tensor cores off; between
    the tensor-core kernels the query-side one only where r_K g <= 128, by
    request, or by default once a call has >= 200 folded tiles per SM (none
    at n_c = 0)."""
    import online_rank_kv_b200 as ik

    def kernel(env=None, **kw):
        for k in ("ISKV_DECODE_KERNEL", "ISKV_TENSOR_CORES"):
            monkeypatch.delenv(k, raising=False)
        for k, v in (env or {}).items():
            monkeypatch.setenv(k, v)
        c = ik.Cache(_cfg(**kw))
        try:
            return c.decode_kernel(0)
        finally:
            c.close()

    assert kernel(coef_dtype=ik.F32) == "cuda_core"
    assert kernel({"ISKV_TENSOR_CORES": "0"}) == "cuda_core"
    assert kernel() == "rotate"                                  # n_c = 0: no folded tiles yet
    assert kernel({"ISKV_DECODE_KERNEL": "u"}) == "query_rope"   # r_K g = 32 * 4 = 128
    assert kernel({"ISKV_DECODE_KERNEL": "rot"}) == "rotate"
    assert kernel({"ISKV_DECODE_KERNEL": "u"}, rank_k=64) == "rotate"   # r_K g = 256
    with pytest.raises(ik.IskvError):
        c = ik.Cache(_cfg())
        try:
            c.decode_kernel(5)                                   # layer out of range
        finally:
            c.close()
