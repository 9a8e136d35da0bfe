"""The seeded input generator against the recipe it states (CPU): determinism
by seed, the low-rank latent and its decay, the key outlier channels, the
drift of the subspace at its cadence, and queries (plain and aimed at one
position).  The generator draws data only; these checks make sure the inputs
every parity test and the bench use have the structure the recipe claims.
"""

import math

import numpy as np
import torch

import synth


def _svals(x: torch.Tensor) -> np.ndarray:
    return np.linalg.svd(x.double().numpy(), compute_uv=False)


def test_streams_are_determined_by_the_seed():
    spec = synth.spec_for("qwen3", "K")
    a = synth.KVStream(spec, 3, seed=5).next(700)
    b = synth.KVStream(spec, 3, seed=5).next(700)
    c = synth.KVStream(spec, 3, seed=6).next(700)
    assert a.shape == (3, 700, 128)
    assert torch.equal(a, b)
    assert not torch.equal(a, c)
    bf = synth.KVStream(spec, 3, seed=5, dtype=torch.bfloat16).next(700)
    assert bf.dtype == torch.bfloat16
    assert torch.equal(bf, a.to(torch.bfloat16))


def test_tiny_stream_has_rank_eight_plus_small_noise():
    """Flat rank-8 latent, noise 1e-3: eight singular values of order sqrt(n),
    the rest at the noise floor."""
    x = synth.KVStream(synth.spec_for("tiny", "K"), 1, seed=0).next(1024)[0]
    s = _svals(x)
    assert s[7] > 0.5 * math.sqrt(1024)
    assert s[8] < 1e-3 * (math.sqrt(1024) + math.sqrt(128)) * 1.5
    # flat latent: the eight leading values agree within sampling spread
    assert s[0] / s[7] < 1.6


def test_value_stream_spectrum_follows_the_latent_decay():
    """V of the qwen3 recipe (no outliers, no drift within 512 tokens): the
    l-th singular value over n tokens is about sqrt(n) * 0.95**l."""
    spec = synth.spec_for("qwen3", "V")
    x = synth.KVStream(spec, 1, seed=3).next(512)[0]
    s = _svals(x)
    for l in (5, 10, 20):
        want = spec.decay ** l
        assert abs(s[l] / s[0] - want) < 0.2 * want, (l, s[l] / s[0], want)
    # rank 48 latent over a noise floor of 0.05 per entry
    floor = spec.noise * (math.sqrt(512) + math.sqrt(128))
    assert s[48] < 1.2 * floor
    assert s[30] > 2 * floor                       # sqrt(512) 0.95**30 = 4.9


def test_key_streams_have_four_outlier_channels_per_head():
    spec = synth.spec_for("qwen3", "K")
    st = synth.KVStream(spec, 4, seed=9)
    x = st.next(512)
    rms = x.pow(2).mean(dim=1).sqrt()                  # H x d channel RMS
    for h in range(4):
        r = rms[h].sort(descending=True).values
        med = r.median()
        assert r[3] > 4 * med and r[4] < 3 * med, (h, r[:6] / med)
        top = set(torch.topk(rms[h], 4).indices.tolist())
        assert top == set(st.outlier_idx[h].tolist())


def test_subspace_turns_by_one_givens_rotation_at_the_drift_cadence():
    spec = synth.spec_for("qwen3", "V")                  # drift every 512 tokens
    st = synth.KVStream(spec, 2, seed=4)
    st.next(300)
    g0 = st.G.clone()
    st.next(212)                                        # t = 512: no drift drawn yet
    assert torch.equal(st.G, g0)
    st.next(1)                                          # the draw at t = 512 turns G first
    g1 = st.G.clone()
    for h in range(2):
        moved = (g1[h] - g0[h]).abs().amax(dim=0) > 0   # which of the d coordinates changed
        assert int(moved.sum()) == 2
        i, j = torch.nonzero(moved).flatten().tolist()
        # a rotation by +-0.05 rad in the (i, j) plane
        a, b = g0[h][:, i], g0[h][:, j]
        c, s = math.cos(spec.drift_angle), math.sin(spec.drift_angle)
        ok = any(torch.allclose(g1[h][:, i], c * a - sg * s * b, atol=1e-12) and
                 torch.allclose(g1[h][:, j], sg * s * a + c * b, atol=1e-12) for sg in (1, -1))
        assert ok
        # rows stay orthonormal
        gram = g1[h] @ g1[h].T
        assert torch.allclose(gram, torch.eye(spec.rank, dtype=gram.dtype), atol=1e-12)
    st.next(511)                                        # t = 1024: nothing new inside the period
    assert torch.equal(st.G, g1)


def test_query_batch_is_standard_normal():
    q = synth.query_batch(4096, 128, seed=1)
    assert q.shape == (4096, 128)
    assert abs(float(q.mean())) < 0.01
    assert abs(float(q.std()) - 1.0) < 0.01
    assert torch.equal(q, synth.query_batch(4096, 128, seed=1))
    q2 = synth.query_batch(64, 128, seed=1, scale=3.0)
    assert torch.allclose(q2, 3.0 * q[:64])


def _rope_complex(k: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotate-half RoPE written with complex numbers: pair (i, i + d/2) is the
    complex number k_i + 1j k_{i+d/2}, turned by pos * theta**(-2i/d)."""
    d = k.shape[-1]
    h = d // 2
    z = k[:h] + 1j * k[h:]
    w = z * np.exp(1j * pos * theta ** (-2.0 * np.arange(h) / d))
    return np.concatenate([w.real, w.imag])


def test_recall_query_aims_at_the_rotated_key():
    """q = beta RoPE(k, p) / |k|: |q| = beta and q . RoPE(k, p) = beta |k|,
    the largest score any key of that norm can get at position p."""
    rng = np.random.default_rng(2)
    theta, beta = 1e6, 7.5
    for pos in (0, 1, 333, 65_000):
        k = rng.standard_normal(128)
        q = synth.recall_query(torch.from_numpy(k), pos, theta, beta).numpy()
        kr = _rope_complex(k, pos, theta)
        assert abs(np.linalg.norm(q) - beta) < 1e-12 * beta
        assert abs(q @ kr - beta * np.linalg.norm(k)) < 1e-9 * beta * np.linalg.norm(k)
    ks = rng.standard_normal((5, 128))
    ps = torch.tensor([3, 90, 1000, 4096, 131_071])
    many = synth.recall_queries(torch.from_numpy(ks), ps, theta, beta).numpy()
    for i in range(5):
        one = synth.recall_query(torch.from_numpy(ks[i]), int(ps[i]), theta, beta).numpy()
        assert np.allclose(many[i], one, rtol=0, atol=1e-12)
