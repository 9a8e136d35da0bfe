"""Failure reporting of the tensor-core decode, made to happen on purpose
without faulting or hanging the GPU.

  * fp16 range: the rotation kernel's score MMA takes rotated keys as fp16,
    finite only below 65504.  One exact key element far beyond that (or
    infinite) must not pass silently: the call's scores are not finite and the
    sticky status reads RANGE; a cache fed keys inside the range reads OK.
    The query-side RoPE kernel scores exact rows in fp32 (a key of 1e5 is
    fine there) and rounds only the products of queries and basis to fp16: an
    infinite key, or a query far beyond fp16's range, reads RANGE.
  * bounded waits: every pipeline wait of the kernel gives up after a limit
    and the call reports DEVICE_TIMEOUT, with the context still usable.  The
    test shortens only the pipeline waits (ISKV_TEST_PIPELINE_WAIT_CYCLES, read
    when a cache is created) so that they run out at once; the drain waits
    that let in-flight copies and MMAs finish keep their full limit.  A fresh
    cache afterwards decodes normally.
"""

import os

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _cfg():
    import online_rank_kv_b200 as ik
    return ik.Config(batch=1, layers=1, kv_heads=2, q_heads=8, rank_k=32, rank_v=64, window=128,
                     max_tokens=1024, kv_dtype=ik.BF16, coef_dtype=ik.BF16, use_rope=1,
                     rope_theta=1e6)


def _fill(cache, seed, huge=None):
    ks = synth.KVStream(synth.spec_for("qwen3", "K"), 2, seed=seed, device="cuda",
                        dtype=torch.bfloat16)
    vs = synth.KVStream(synth.spec_for("qwen3", "V"), 2, seed=seed + 1, device="cuda",
                        dtype=torch.bfloat16)
    for chunk in range(6):
        k = ks.next(64)
        v = vs.next(64)
        if huge is not None and chunk == 5:
            k[0, 63, 5] = huge            # position 383: in the exact window
        ready = cache.append(0, k[None].contiguous(), v[None].contiguous())
        for _ in range(ready):
            cache.compress_block(0)


@pytest.mark.parametrize("huge", [1.0e5, float("inf")])
def test_key_beyond_fp16_range_is_reported(huge, monkeypatch):
    import online_rank_kv_b200 as ik
    monkeypatch.setenv("ISKV_DECODE_KERNEL", "rot")
    q = synth.query_batch(8, 128, seed=4, device="cuda", dtype=torch.bfloat16).view(1, 8, 128)
    ok = ik.Cache(_cfg())
    _fill(ok, 3, huge=1.0e4)              # inside fp16's range
    out = ok.decode_attention(0, q)
    assert torch.isfinite(out).all() and ok.status() == 0
    ok.close()

    bad = ik.Cache(_cfg())
    _fill(bad, 3, huge=huge)
    bad.decode_attention(0, q)
    assert bad.status() == -9, ik.LIB.iskv_strerror(bad.status())
    bad.close()


def test_query_side_kernel_range(monkeypatch):
    """Query-side RoPE kernel (r_K g = 128 here): a key of 1e5 in the window
    decodes to finite output with status OK; an infinite key, or a query
    element of 1e6 (its products with the basis overflow fp16), reads RANGE."""
    import online_rank_kv_b200 as ik
    monkeypatch.setenv("ISKV_DECODE_KERNEL", "u")
    q = synth.query_batch(8, 128, seed=4, device="cuda", dtype=torch.bfloat16).view(1, 8, 128)
    fine = ik.Cache(_cfg())
    _fill(fine, 3, huge=1.0e5)
    out = fine.decode_attention(0, q)
    assert torch.isfinite(out).all() and fine.status() == 0, ik.LIB.iskv_strerror(fine.status())
    fine.close()

    inf_key = ik.Cache(_cfg())
    _fill(inf_key, 3, huge=float("inf"))
    inf_key.decode_attention(0, q)
    assert inf_key.status() == -9, ik.LIB.iskv_strerror(inf_key.status())
    inf_key.close()

    big_q = q.clone()
    big_q[0, 1, 7] = 1.0e6
    loud = ik.Cache(_cfg())
    _fill(loud, 3)
    loud.decode_attention(0, big_q)
    assert loud.status() == -9, ik.LIB.iskv_strerror(loud.status())
    loud.close()


@pytest.mark.parametrize("kernel", ["rot", "u"])
def test_pipeline_wait_limit_reports_timeout_and_context_survives(kernel, monkeypatch):
    import online_rank_kv_b200 as ik
    monkeypatch.setenv("ISKV_DECODE_KERNEL", kernel)
    monkeypatch.setenv("ISKV_TEST_PIPELINE_WAIT_CYCLES", "1")
    short = ik.Cache(_cfg())
    monkeypatch.delenv("ISKV_TEST_PIPELINE_WAIT_CYCLES")
    _fill(short, 5)
    q = synth.query_batch(8, 128, seed=6, device="cuda", dtype=torch.bfloat16).view(1, 8, 128)
    short.decode_attention(0, q)
    assert short.status() == -8, ik.LIB.iskv_strerror(short.status())
    short.close()
    # the context is still usable: a normal cache decodes and reports OK
    fresh = ik.Cache(_cfg())
    _fill(fresh, 5)
    out = fresh.decode_attention(0, q)
    torch.cuda.synchronize()
    assert np.isfinite(out.cpu().numpy()).all()
    assert fresh.status() == 0
    fresh.close()
    assert "ISKV_TEST_PIPELINE_WAIT_CYCLES" not in os.environ
