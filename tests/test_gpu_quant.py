"""Low-bit latent-channel coefficient codes on the GPU against the oracle.

The format (iskv_quant_format; the SVDq page's latent channels with more bits
for the leading ones) is applied at every coefficient write: a fold's new rows
and every rewrite.  Parity is taken in two parts:

  * the coding step itself, bit for bit: the library's coder and the oracle's
    float32-decision quantizer (LatentQuant(fp32=True)) give identical codes
    and scales for the same float32 rows;
  * the whole path, where GPU and oracle code slightly different values (fp32
    against fp64 folds, and bases that may turn inside nearly equal singular
    values), so codes may differ by a step: the coded GPU factor must lose as
    much against the exact rows as the coded oracle factor (ratio of the two
    reconstruction errors within [0.8, 1.25]), the two coded reconstructions
    may differ by at most twice the oracle's own coding error, and decode
    outputs may differ from the oracle's by at most 2e-2 plus twice the effect
    coding has on the oracle's decode.
"""

import numpy as np
import pytest
import torch

import synth
from iskv_testlib import rel_err
from oracle import HeadFactor, LatentQuant, dense_decode, persistent_kv_bytes

pytestmark = pytest.mark.gpu

QK = ((16, 8), (16, 4))                 # r_K = 32: 6 bits per coefficient
QV = ((16, 8), (16, 4), (32, 2))        # r_V = 64: 4 bits per coefficient


def _unpack(codes, groups):
    """uint32 words (int32 tensor) -> signed codes [n, r] by the documented
    packing: per group, b-bit fields from the lowest bit up, offset 2^(b-1)-1."""
    w = codes.cpu().numpy().astype(np.int64) & 0xFFFFFFFF
    out = []
    word = 0
    for n, b in groups:
        if b == 0:
            out.append(np.zeros((w.shape[0], n), dtype=np.int64))
            continue
        per, qmax = 32 // b, 2 ** (b - 1) - 1
        cols = []
        for c in range(n):
            ww = w[:, word + c // per]
            cols.append(((ww >> ((c % per) * b)) & ((1 << b) - 1)) - qmax)
        out.append(np.stack(cols, 1))
        word += n * b // 32
    return np.concatenate(out, 1)


@pytest.mark.parametrize("groups", [QK, QV, ((32, 2), (32, 0)), ((64, 8), (64, 4))])
def test_coder_matches_the_float32_oracle_bit_for_bit(groups):
    import online_rank_kv_b200 as ik
    r = sum(n for n, _ in groups)
    g = np.random.default_rng(5)
    C = (g.standard_normal((3000, r)) * (0.9 ** np.arange(r)) * 3).astype(np.float32)
    C[7] = 0.0                                      # an all-zero row: scales 0
    C[11, :16] = 0.0                                # an all-zero group
    C[13, 3] = 1e-30                                # tiny values
    codes, scales = ik.quantize_rows(groups, torch.from_numpy(C).cuda())
    torch.cuda.synchronize()
    want_c, want_s = LatentQuant(groups, fp32=True).quantize(C)
    got_c = _unpack(codes, groups)
    np.testing.assert_array_equal(got_c, want_c)
    np.testing.assert_array_equal(scales.cpu().numpy()[:, :len(groups)].astype(np.float64), want_s)


def _cfg(**kw):
    import online_rank_kv_b200 as ik
    c = ik.Config(batch=2, layers=1, kv_heads=2, q_heads=8, rank_k=32, rank_v=64, window=256,
                  max_tokens=4096, kv_dtype=ik.BF16, coef_dtype=ik.F32, use_rope=1, rope_theta=1e6,
                  coef_quant=1, quant_k=QK, quant_v=QV)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("tensor_cores", ["1", "0", "u"])
def test_coded_cache_tracks_the_coded_oracle_through_many_rewrites(tensor_cores, monkeypatch):
    """Decode through the tensor-core kernels (the layer's codes expanded to
    bf16 tiles per call; "u" forces the query-side RoPE kernel) and through the
    CUDA-core kernel (codes read in place)."""
    import online_rank_kv_b200 as ik
    monkeypatch.setenv("ISKV_TENSOR_CORES", "0" if tensor_cores == "0" else "1")
    if tensor_cores == "u":
        monkeypatch.setenv("ISKV_DECODE_KERNEL", "u")
    cfg = _cfg()
    cache = ik.Cache(cfg)
    H = cfg.batch * cfg.kv_heads
    ks = synth.KVStream(synth.spec_for("qwen3", "K"), H, seed=41, dtype=torch.bfloat16)
    vs = synth.KVStream(synth.spec_for("qwen3", "V"), H, seed=42, dtype=torch.bfloat16)
    qk, qv = LatentQuant(QK, fp32=True), LatentQuant(QV, fp32=True)
    coded = [(HeadFactor(128, 32, 256, coef_round=qk), HeadFactor(128, 64, 256, coef_round=qv))
             for _ in range(H)]
    plain = [(HeadFactor(128, 32, 256, coef_round="f32"), HeadFactor(128, 64, 256, coef_round="f32"))
             for _ in range(H)]
    folds = 0
    for _ in range(40):
        k, v = ks.next(64), vs.next(64)
        ready = cache.append(0, k.view(2, 2, 64, 128).cuda(), v.view(2, 2, 64, 128).cuda())
        for i in range(H):
            for f in coded[i] + plain[i]:
                f.append((k if f.r == 32 else v)[i].double().numpy())
        for _ in range(ready):
            cache.compress_block(0)                 # the rewrite of every stored row, coded again
            for i in range(H):
                for f in coded[i] + plain[i]:
                    f.fold()
            folds += 1
    assert folds >= 30
    T, n_c = cache.counts(0)
    assert (T, n_c) == (coded[0][0].T, coded[0][0].n_c)
    for which, idx in ((ik.WHICH_K, 0), (ik.WHICH_V, 1)):
        got = cache.reconstruct(0, which).cpu().numpy().reshape(H, n_c, 128)
        for i in range(H):
            exact = coded[i][idx].rows[:n_c]
            rec_c = coded[i][idx].reconstruct()
            rec_p = plain[i][idx].reconstruct()
            e_gpu = np.linalg.norm(got[i] - exact) / np.linalg.norm(exact)
            e_orc = np.linalg.norm(rec_c - exact) / np.linalg.norm(exact)
            coding = np.linalg.norm(rec_c - rec_p) / np.linalg.norm(rec_p)
            assert 0.8 < e_gpu / e_orc < 1.25, (which, i, e_gpu, e_orc)
            assert np.linalg.norm(got[i] - rec_c) / np.linalg.norm(rec_c) <= 2 * coding, (which, i)
    q = synth.query_batch(cfg.batch * cfg.q_heads, 128, seed=43, dtype=torch.bfloat16).view(2, 8, 128)
    out = cache.decode_attention(0, q.cuda()).cpu().numpy()
    for i in range(H):
        b, h = divmod(i, 2)
        qn = q[b, 4 * h:4 * h + 4].double().numpy()
        want = dense_decode(qn, coded[i][0].full(), coded[i][1].full(), 1e6)
        ref = dense_decode(qn, plain[i][0].full(), plain[i][1].full(), 1e6)
        tol = 2e-2 + 2 * rel_err(want, ref)
        assert rel_err(out[b, 4 * h:4 * h + 4], want) < tol, (i, rel_err(out[b, 4 * h:4 * h + 4], want), tol)
    # persistent bytes: codes and scales per row instead of 4-byte coefficients
    kept, full = cache.kv_bytes()
    want_kept = H * persistent_kv_bytes(n_c, T - n_c, 128, 32, 64, 4, 2,
                                        coef_row_bytes=qk.row_bytes() + qv.row_bytes())
    assert kept == want_kept and full == H * 2 * T * 128 * 2
    assert cache.status() == 0
    cache.close()


def test_coded_factor_values_are_on_their_grids():
    """Every stored value is code * scale with |code| <= 2^(b-1) - 1: coding
    the library's own stored rows again returns the same values."""
    import online_rank_kv_b200 as ik
    cfg = _cfg(batch=1, kv_heads=2, q_heads=8)
    cache = ik.Cache(cfg)
    ks = synth.KVStream(synth.spec_for("qwen3", "K"), 2, seed=51, dtype=torch.bfloat16)
    vs = synth.KVStream(synth.spec_for("qwen3", "V"), 2, seed=52, dtype=torch.bfloat16)
    for _ in range(12):
        ready = cache.append(0, ks.next(64)[None].cuda(), vs.next(64)[None].cuda())
        for _ in range(ready):
            cache.compress_block(0)
    for which, groups in ((ik.WHICH_K, QK), (ik.WHICH_V, QV)):
        _, _, coef = cache.factors(0, which)
        rows = coef.reshape(-1, coef.shape[-1]).contiguous()
        codes, scales = ik.quantize_rows(groups, rows)
        again = torch.from_numpy(LatentQuant(groups, fp32=True).dequantize(
            _unpack(codes, groups), scales.cpu().numpy().astype(np.float64)[:, :len(groups)]))
        np.testing.assert_allclose(again.numpy(), rows.cpu().numpy().astype(np.float64),
                                   rtol=2e-6, atol=0)
    cache.close()
