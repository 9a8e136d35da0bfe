"""The allocation-free decode entry point against the regular one.

``iskv_decode_attention_noalloc`` serves callers that cannot call cudaMalloc
(a serving engine that owns and plans all device memory, or a latency-critical
path that must avoid cudaMalloc's device-wide synchronization): they pass the
factors from their own buffers and the split-K partials use a library-owned
static device array.  This test builds a cache with the regular API, copies
its factors (row-major, as ``iskv_get_factors`` returns them) and exact rows
into test-owned device buffers, and checks that the allocation-free call gives
the regular call's output within the parity tolerance, on two calls in a row
(the shared scratch keeps the first call's contents; the second call must not
depend on them).  Cases: fp32 and bf16 coefficients, RoPE on and off (a NULL
table), and an empty exact window (every row folded, T == n_c).

Kept in its own file, named to be collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

from iskv_testlib import Pair, rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def _rope_table(T, d, theta):
    inv = np.power(float(theta), -2.0 * np.arange(d // 2) / d)
    ang = np.arange(T, dtype=np.float64)[:, None] * inv[None, :]
    tab = np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)
    return torch.from_numpy(tab).contiguous()


CASES = {
    # name: coefficient type, RoPE, window, tokens appended
    "f32-rope": ("f32", 1, 256, 1000),
    "bf16-rope": ("bf16", 1, 256, 1000),
    "f32-norope": ("f32", 0, 256, 1000),
    "f32-empty-window": ("f32", 1, 0, 1024),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_decode_matches_regular_decode_twice(case):
    import online_rank_kv_b200 as ik
    coef, use_rope, window, tokens = CASES[case]
    coef_dt = ik.BF16 if coef == "bf16" else ik.F32
    tol = TOL_BF16 if coef == "bf16" else TOL_F32
    cfg = ik.Config(batch=2, layers=1, kv_heads=2, q_heads=8, rank_k=32, rank_v=64, window=window,
                    max_tokens=2048, kv_dtype=ik.BF16, coef_dtype=coef_dt, use_rope=use_rope,
                    rope_theta=1e6)
    p = Pair(cfg, "qwen3", seed=21)
    p.prefill(tokens, chunk=64)
    T, n_c = p.cache.counts(0)
    assert n_c > 0
    if window == 0:
        assert T == n_c
    else:
        assert T > n_c
    dev = "cuda"
    bk, _, ck = p.cache.factors(0, ik.WHICH_K)
    bv, _, cv = p.cache.factors(0, ik.WHICH_V)
    BH = cfg.batch * cfg.kv_heads
    ring_rows = 512
    rk = torch.zeros(BH, ring_rows, 128, dtype=torch.bfloat16)
    rv = torch.zeros(BH, ring_rows, 128, dtype=torch.bfloat16)
    for b in range(cfg.batch):
        for h in range(cfg.kv_heads):
            ek = p.ok[(0, b, h)].exact()
            ev = p.ov[(0, b, h)].exact()
            for j in range(n_c, T):
                rk[b * cfg.kv_heads + h, j % ring_rows] = torch.from_numpy(ek[j - n_c])
                rv[b * cfg.kv_heads + h, j % ring_rows] = torch.from_numpy(ev[j - n_c])
    rk, rv = rk.to(dev), rv.to(dev)
    rope = _rope_table(T, 128, cfg.rope_theta).to(dev) if use_rope else None
    bk, ck, bv, cv = (x.contiguous() for x in (bk, ck, bv, cv))

    ops = ik.DecodeOperands()
    ops.batch, ops.kv_heads, ops.q_heads, ops.head_dim = cfg.batch, cfg.kv_heads, cfg.q_heads, 128
    ops.rank_k, ops.rank_v, ops.kv_dtype, ops.coef_dtype = 32, 64, ik.BF16, coef_dt
    ops.T, ops.n_c, ops.coef_rows, ops.ring_rows = T, n_c, n_c, ring_rows
    ops.coef_k, ops.basis_k = ck.data_ptr(), bk.data_ptr()
    ops.coef_v, ops.basis_v = cv.data_ptr(), bv.data_ptr()
    ops.ring_k, ops.ring_v = rk.data_ptr(), rv.data_ptr()
    ops.rope = rope.data_ptr() if rope is not None else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    for call in range(2):
        q = p.query().to(dev)
        want = p.cache.decode_attention(0, q).cpu().numpy()
        out = torch.full((cfg.batch, cfg.q_heads, 128), float("nan"), device=dev)
        rc = ik.LIB.iskv_decode_attention_noalloc(ctypes.byref(ops), ctypes.c_void_p(q.data_ptr()),
                                                  ctypes.c_void_p(out.data_ptr()), stream)
        assert rc == 0, ik.LIB.iskv_strerror(rc)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_err(got, want) < tol, (case, call, rel_err(got, want))

    # host memory is refused (nothing is staged), and so is an oversized batch
    qh = p.query()
    out = torch.empty(cfg.batch, cfg.q_heads, 128, device=dev)
    assert ik.LIB.iskv_decode_attention_noalloc(ctypes.byref(ops), ctypes.c_void_p(qh.data_ptr()),
                                                ctypes.c_void_p(out.data_ptr()), stream) == -1
    big = ik.DecodeOperands.from_buffer_copy(ops)
    big.batch, big.kv_heads, big.q_heads = 1024, 1, 8
    assert ik.LIB.iskv_decode_attention_noalloc(ctypes.byref(big), ctypes.c_void_p(q.data_ptr()),
                                                ctypes.c_void_p(out.data_ptr()), stream) == -2
    p.cache.close()
