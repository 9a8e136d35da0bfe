"""Pins of the float64 oracle against things other than itself.

Each test checks the oracle against what the pages or the mathematics fix:
brute force on tiny inputs, closed forms, invariants, the covariance route to
a batch SVD (KV-CoRE summary, section 2 Methodology), the exactness of Brand's
update on histories of rank <= r, losslessness at r = d, and the one number
the pages print that is pure arithmetic (the A40 full-cache size).  The
mutation tests at the end plant mistakes in a copy of the oracle's fold and
check that the pins catch them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import iskv_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _low_rank_rows(n, d, rank, seed, noise=0.0):
    g = _rng(seed)
    G, _ = np.linalg.qr(g.standard_normal((d, rank)))
    Z = g.standard_normal((n, rank)) * (2.0 ** -np.arange(rank) * 4 + 1)
    return Z @ G.T + noise * g.standard_normal((n, d))


def _cov_projector(H, m):
    """Projector onto the top-m right singular subspace of H via the
    eigenvectors of H^T H (the covariance route of the KV-CoRE summary)."""
    w, V = np.linalg.eigh(H.T @ H)
    idx = np.argsort(w)[::-1][:m]
    Vm = V[:, idx]
    return Vm @ Vm.T


def _fold_all(f):
    while f.ready() > 0:
        f.fold()


# ----------------------------------------------------------------------------
# storage rounding
# ----------------------------------------------------------------------------


def test_bf16_round_matches_torch_on_float32_inputs():
    x = _rng(0).standard_normal(200000).astype(np.float32) * 37.0
    x = np.concatenate([x, np.float32([0.0, -0.0, 1e-30, -3e-39, 3.3e38])])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_round_ties_and_direct_rounding():
    one = 1.0
    # exact tie between 1 and 1 + 2^-7: to even (1)
    assert O.bf16_round(one + 2.0 ** -8) == 1.0
    # tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even): to 1 + 2^-6
    assert O.bf16_round(one + 3 * 2.0 ** -8) == one + 2.0 ** -6
    # just above a tie: rounds up.  A detour through float32 would first make
    # it an exact tie and then round down; the oracle rounds float64 directly.
    assert O.bf16_round(one + 2.0 ** -8 + 2.0 ** -40) == one + 2.0 ** -7
    assert O.bf16_round(-(one + 2.0 ** -8 + 2.0 ** -40)) == -(one + 2.0 ** -7)
    # carry into the exponent
    assert O.bf16_round(2.0 - 2.0 ** -9) == 2.0
    assert np.isinf(O.bf16_round(3.5e38))


# ----------------------------------------------------------------------------
# bookkeeping
# ----------------------------------------------------------------------------


def test_ready_blocks_brute_force():
    for W in (0, 64, 128, 192):
        for T in range(0, 400):
            for n_c in range(0, T + 1, 64):
                # count by simulating the window: pop blocks while enough
                # rows are older than the newest W
                n, cnt = n_c, 0
                while True:
                    old = [j for j in range(n, T) if j < T - W]
                    if len(old) >= 64:
                        n += 64
                        cnt += 1
                    else:
                        break
                assert O.ready_blocks(T, n_c, W) == cnt, (T, n_c, W)


def test_headfactor_counters_and_window_bounds():
    f = O.HeadFactor(d=16, r=4, W=64)
    g = _rng(1)
    for step in range(700):
        f.append(g.standard_normal((1, 16)))
        _fold_all(f)
        n_w = f.T - f.n_c
        assert f.n_c % 64 == 0
        assert (f.T < 64 + 64 and f.n_c == 0) or 64 <= n_w <= 127
        assert 0 <= n_w < 64 + 64
    assert f.T == 700 and f.n_c == 576


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------


def test_rope_hand_computed_d4():
    # d = 4, theta = 10000: inv_freq = [1, 0.01]; pairs (0, 2) and (1, 3)
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    got = O.rope_rotate(x, [1], 10000.0)[0]
    c0, s0, c1, s1 = math.cos(1.0), math.sin(1.0), math.cos(0.01), math.sin(0.01)
    want = [1 * c0 - 3 * s0, 2 * c1 - 4 * s1, 1 * s0 + 3 * c0, 2 * s1 + 4 * c1]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)


def test_rope_invariants():
    g = _rng(2)
    d, theta = 128, 1e6
    x = g.standard_normal((5, d))
    pos = np.array([0, 1, 1000, 65535, 262143])
    y = O.rope_rotate(x, pos, theta)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    np.testing.assert_array_equal(O.rope_rotate(x[:1], [0], theta), x[:1])
    q, k = g.standard_normal((1, d)), g.standard_normal((1, d))
    for a, b in [(3, 10), (1000, 4000), (200000, 262000)]:
        lhs = (O.rope_rotate(q, [a], theta) @ O.rope_rotate(k, [b], theta).T).item()
        rhs = (q @ O.rope_rotate(k, [b - a], theta).T).item()
        assert abs(lhs - rhs) < 1e-9 * (1 + abs(rhs))


# ----------------------------------------------------------------------------
# one fold
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("r", [16, 64, 96, 128])
def test_fold_identities(r):
    d = 128
    g = _rng(3 + r)
    B, _ = np.linalg.qr(g.standard_normal((d, r)))
    S = np.sort(g.uniform(1, 10, r))[::-1]
    X = g.standard_normal((64, d))
    res = O.fold_block(B, S, X)
    k = min(64, d - r)
    assert res.Q.shape == (d, k) and res.R_E.shape == (k, 64)
    # [B, Q] orthonormal
    BQ = np.concatenate([B, res.Q], axis=1)
    np.testing.assert_allclose(BQ.T @ BQ, np.eye(r + k), atol=1e-13)
    # the block is represented exactly: X = P B^T + R_E^T Q^T
    np.testing.assert_allclose(res.P @ B.T + res.R_E.T @ res.Q.T, X, atol=1e-12)
    # new basis orthonormal, singular values sorted
    np.testing.assert_allclose(res.B_new.T @ res.B_new, np.eye(r), atol=1e-12)
    assert np.all(np.diff(res.sigma) <= 1e-12)
    # energy balance: ||core||^2 = ||S||^2 + ||X||^2, discarded = tail sigma^2
    e_core = np.sum(res.core ** 2)
    np.testing.assert_allclose(e_core, np.sum(S ** 2) + np.sum(X ** 2), rtol=1e-12)
    kept = np.sum(res.S_new ** 2)
    np.testing.assert_allclose(e_core - kept, np.sum(res.sigma[r:] ** 2), rtol=1e-9, atol=1e-9)


def test_one_fold_is_eckart_young_of_exact_history():
    """History of rank <= r held exactly: one fold must give the best rank-r
    approximation of [history; block] (batch SVD via the covariance route)."""
    d, r = 128, 24
    g = _rng(7)
    H = _low_rank_rows(200, d, 10, 7)            # rank 10 <= r history
    U, s, Vt = np.linalg.svd(H, full_matrices=False)
    B = Vt[:r].T
    S = s[:r]
    C = U[:, :r] * S                              # C B^T = H exactly
    X = g.standard_normal((64, d))
    res = O.fold_block(B, S, X)
    C_all = np.concatenate([C @ res.W_top, res.C_new], axis=0)
    A = np.concatenate([H, X], axis=0)
    P = _cov_projector(A, r)
    np.testing.assert_allclose(res.B_new @ res.B_new.T, P, atol=1e-9)
    np.testing.assert_allclose(C_all @ res.B_new.T, A @ P, atol=1e-9)


def test_sync_closed_form():
    """Old rows after (e): C' B'^T = (C B^T) B' B'^T, for any history."""
    d, r = 128, 32
    g = _rng(9)
    f = O.HeadFactor(d, r, W=64)
    f.append(_low_rank_rows(64 * 6, d, 48, 9, noise=0.05))
    _fold_all(f)
    before = f.reconstruct()
    n_old = f.n_c
    f.append(g.standard_normal((64, d)))
    f.fold()
    after = (f.C @ f.B.T)[:n_old]
    np.testing.assert_allclose(after, before @ f.B @ f.B.T, atol=1e-11)


# ----------------------------------------------------------------------------
# whole-history pins
# ----------------------------------------------------------------------------


def test_exact_rank_history_is_reproduced():
    """Rank 8 <= r = 16, no noise: zero residual and the batch projector."""
    d, r = 128, 16
    rows = _low_rank_rows(1024, d, 8, 11)
    f = O.HeadFactor(d, r, W=128)
    f.append(rows)
    _fold_all(f)
    assert f.n_c == 896
    H = rows[:f.n_c]
    err = np.abs(f.reconstruct() - H).max() / np.abs(H).max()
    assert err < 1e-12
    np.testing.assert_allclose(f.B[:, :8] @ f.B[:, :8].T, _cov_projector(H, 8), atol=1e-10)
    np.testing.assert_allclose(f.B.T @ f.B, np.eye(r), atol=1e-10)


@pytest.mark.parametrize("seed", [0, 1])
def test_full_rank_is_lossless(seed):
    d = 128
    rows = _rng(seed).standard_normal((64 * 7 + 30, d))
    f = O.HeadFactor(d, d, W=64)
    f.append(rows)
    _fold_all(f)
    np.testing.assert_allclose(f.reconstruct(), rows[:f.n_c], atol=1e-11)
    q = _rng(seed + 100).standard_normal((4, d))
    got = O.dense_decode(q, f.full(), rows, theta=1e6)
    want = O.dense_decode(q, rows, rows, theta=1e6)
    np.testing.assert_allclose(got, want, atol=1e-11)


@pytest.mark.parametrize("r", [16, 96, 128])
def test_orthonormal_after_many_folds_and_degenerate_blocks(r):
    d = 128
    g = _rng(r)
    f = O.HeadFactor(d, r, W=0)
    blocks = [np.zeros((64, d)), np.tile(g.standard_normal((1, d)), (64, 1)),
              _low_rank_rows(64, d, 3, 1)]
    blocks += [g.standard_normal((64, d)) * 10 ** g.uniform(-3, 3) for _ in range(20)]
    blocks += [np.zeros((64, d))]
    for Xb in blocks:
        f.append(Xb)
        f.fold()
        assert np.linalg.norm(f.B.T @ f.B - np.eye(r)) < 1e-10


def test_deferred_sync_equals_per_fold_sync():
    d, r = 128, 32
    rows = _low_rank_rows(64 * 12, d, 48, 13, noise=0.05)
    a = O.HeadFactor(d, r, W=0)
    b = O.HeadFactor(d, r, W=0)
    a.append(rows)
    b.append(rows)
    while a.ready():
        a.fold()
        b.fold(defer=True)
        if len(b.pending) == 5:
            b.sync()
    b.sync()
    np.testing.assert_allclose(b.C, a.C, atol=1e-12)


def test_no_sync_ablation_drifts():
    """The explainer reports far larger drift when only the basis is updated;
    the ablation must show it on a drifting low-rank stream."""
    d, r = 128, 16
    rows = _low_rank_rows(64 * 12, d, 12, 100, noise=0.01)
    s = O.HeadFactor(d, r, W=0)
    n = O.HeadFactor(d, r, W=0, sync=False)
    s.append(rows)
    n.append(rows)
    _fold_all(s)
    _fold_all(n)
    H = rows[:s.n_c]
    e_sync = np.linalg.norm(s.reconstruct() - H) / np.linalg.norm(H)
    e_none = np.linalg.norm(n.C @ n.B.T - H) / np.linalg.norm(H)
    assert e_sync < 0.05
    assert e_none > 20 * e_sync


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------


def _brute_decode(q, K, V, theta, use_rope):
    """Pure-Python loops: rotate, score, softmax, weighted sum."""
    T, d = len(K), len(K[0])
    h = d // 2
    out = []
    for qh in q:
        scores = []
        for j in range(T):
            kr = list(K[j])
            if use_rope:
                for i in range(h):
                    a = j * theta ** (-2.0 * i / d)
                    kr[i] = K[j][i] * math.cos(a) - K[j][i + h] * math.sin(a)
                    kr[i + h] = K[j][i] * math.sin(a) + K[j][i + h] * math.cos(a)
            scores.append(sum(qh[i] * kr[i] for i in range(d)) / math.sqrt(d))
        m = max(scores)
        w = [math.exp(s - m) for s in scores]
        z = sum(w)
        out.append([sum(w[j] * V[j][i] for j in range(T)) / z for i in range(d)])
    return np.array(out)


@pytest.mark.parametrize("use_rope", [False, True])
def test_dense_decode_brute_force(use_rope):
    g = _rng(21)
    d, T = 8, 37
    q = g.standard_normal((3, d)) * 2
    K = g.standard_normal((T, d))
    V = g.standard_normal((T, d))
    got = O.dense_decode(q, K, V, theta=10000.0, use_rope=use_rope)
    want = _brute_decode(q.tolist(), K.tolist(), V.tolist(), 10000.0, use_rope)
    np.testing.assert_allclose(got, want, atol=1e-13)


def test_dense_decode_special_cases():
    g = _rng(22)
    K = g.standard_normal((50, 16))
    V = g.standard_normal((50, 16))
    np.testing.assert_allclose(O.dense_decode(np.zeros((1, 16)), K, V, 1e6)[0], V.mean(0),
                               atol=1e-14)
    q = 1e4 * O.rope_rotate(K[17:18], [17], 1e6)
    np.testing.assert_allclose(O.dense_decode(q, K, V, 1e6)[0], V[17], atol=1e-12)


# ----------------------------------------------------------------------------
# memory accounting
# ----------------------------------------------------------------------------


def test_full_kv_bytes_matches_a40_figure():
    with open(os.path.join(GOLDEN, "a40_memory.json")) as fh:
        gd = json.load(fh)
    got = O.full_kv_bytes(gd["tokens"], gd["layers"], gd["kv_heads"], gd["head_dim"],
                          gd["elem_bytes"]) / 2 ** 30
    assert got == gd["full_gib"]


# ----------------------------------------------------------------------------
# protected rows (positions 0..P-1 kept exact, never folded)
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("P", [1, 37, 64, 200])
def test_protected_factor_is_the_unprotected_factor_of_the_shifted_stream(P):
    """With P protected positions the factor sees the stream from row P on:
    block counts, folds, coefficients and basis equal those of an
    unprotected factor fed rows P, P+1, ...; attention sees the protected
    rows first, unchanged."""
    d, r, W = 128, 16, 128
    rows = _low_rank_rows(P + 700, d, 12, seed=50 + P, noise=1e-3)
    a = O.HeadFactor(d, r, W, protect=P)
    b = O.HeadFactor(d, r, W)
    for lo in range(0, rows.shape[0], 50):
        chunk = rows[lo:lo + 50]
        a.append(chunk)
        tail = rows[max(lo, P):lo + 50]
        if tail.shape[0]:
            b.append(tail)
        assert a.ready() == b.ready()
        while a.ready() >= 1:
            a.fold()
            b.fold()
    assert a.n_c == b.n_c > 0
    np.testing.assert_array_equal(a.C, b.C)
    np.testing.assert_array_equal(a.B, b.B)
    np.testing.assert_array_equal(a.protected(), rows[:P])
    np.testing.assert_array_equal(a.full()[:P], rows[:P])
    np.testing.assert_array_equal(a.full()[P:], b.full())
    assert a.full().shape[0] == rows.shape[0]


def test_protected_ready_counts_brute_force():
    """ready = floor((T - P - n_c - W) / b) when positive, by counting the
    whole blocks that have left the window after the protected positions."""
    W, bsz = 128, 64
    for P in (0, 5, 64, 130):
        for T in range(0, 900, 7):
            for n_c in range(0, max(0, T - P) + 1, 64):
                f = O.HeadFactor(128, 16, W, protect=P)
                f.rows = np.zeros((T, 128))
                f.n_c = n_c
                free = [j for j in range(P + n_c, T) if j < T - W]   # folded-eligible rows
                whole = 0
                while (whole + 1) * bsz <= len(free):
                    whole += 1
                assert f.ready() == whole, (P, T, n_c)


def test_protected_lossless_decode_equals_dense_attention():
    """At r = d every row is reproduced, so decode over protected + folded +
    window rows is dense attention over the raw rows, whatever P is."""
    d, W, P = 128, 64, 70
    g = _rng(61)
    K = g.standard_normal((P + 400, d))
    V = g.standard_normal((P + 400, d))
    fk = O.HeadFactor(d, d, W, protect=P)
    fv = O.HeadFactor(d, d, W, protect=P)
    fk.append(K)
    fv.append(V)
    while fk.ready() >= 1:
        fk.fold()
        fv.fold()
    assert fk.n_c >= 256
    q = g.standard_normal((4, d))
    np.testing.assert_allclose(O.dense_decode(q, fk.full(), fv.full(), 1e6),
                               O.dense_decode(q, K, V, 1e6), atol=1e-10)


def test_persistent_bytes_count_the_kept_arrays():
    """The kept-byte formula equals a count of the arrays the oracle keeps
    (elements times their stored width), for K and V factors with protected
    rows, before and after the first fold."""
    d, rk, rv, W, P = 128, 32, 64, 128, 40
    g = _rng(62)
    for n_rows in (100, P + W + 64 * 3 + 17):
        fk = O.HeadFactor(d, rk, W, protect=P, coef_round="bf16")
        fv = O.HeadFactor(d, rv, W, protect=P, coef_round="bf16")
        X = g.standard_normal((n_rows, d))
        fk.append(X)
        fv.append(X)
        while fk.ready() >= 1:
            fk.fold()
            fv.fold()
        counted = 0
        for f in (fk, fv):
            prot, win = f.protected(), f.exact()
            counted += (prot.size + win.size) * 2          # bf16 K/V rows
            if f.n_c:
                counted += f.C.size * 2 + (f.B.size + f.S.size) * 4   # bf16 C, fp32 B and S
        n_w = fk.exact().shape[0]
        n_p = fk.protected().shape[0]
        assert O.persistent_kv_bytes(fk.n_c, n_w, d, rk, rv, 2, 2, 4, n_p=n_p) == counted


# ----------------------------------------------------------------------------
# low-bit coefficients in latent channels (oracle only)
# ----------------------------------------------------------------------------


def test_latent_quant_is_the_nearest_grid_point():
    """Per row and channel group the stored value is the nearest point of the
    symmetric uniform grid {k * scale : |k| <= 2^(b-1) - 1}, found here by
    brute force over every level; dropped groups are zero."""
    g = _rng(70)
    C = g.standard_normal((40, 32)) * (2.0 ** -np.arange(32) * 8 + 0.1)
    C[3] = 0.0
    q = O.LatentQuant([(4, 8), (12, 4), (8, 2), (8, 0)])
    got = q(C)
    codes, scales = q.quantize(C)
    spans = [(0, 4, 8), (4, 16, 4), (16, 24, 2), (24, 32, 0)]
    for gi, (lo, hi, b) in enumerate(spans):
        for i in range(C.shape[0]):
            if b == 0:
                assert np.all(got[i, lo:hi] == 0)
                continue
            qmax = 2 ** (b - 1) - 1
            sc = np.abs(C[i, lo:hi]).max() / qmax
            assert scales[i, gi] == sc
            if sc == 0:
                assert np.all(got[i, lo:hi] == 0)
                continue
            levels = np.arange(-qmax, qmax + 1) * sc
            for j in range(lo, hi):
                d = np.abs(levels - C[i, j])
                best = levels[np.argmin(d)]
                assert abs(got[i, j] - C[i, j]) <= d.min() + 1e-15
                assert abs(got[i, j] - best) <= 1e-15 or np.isclose(d[np.argsort(d)[:2]], d.min()).all()
                assert abs(codes[i, j]) <= qmax
    assert q.bits_per_coefficient() == (4 * 8 + 12 * 4 + 8 * 2) / 32


def test_latent_quant_grid_values_round_trip_and_high_bits_converge():
    q16 = O.LatentQuant([(16, 16)])
    g = _rng(71)
    C = g.standard_normal((20, 16))
    codes, scales = q16.quantize(C)
    np.testing.assert_array_equal(q16(q16(C)), q16(C))    # grid values are fixed points
    assert np.max(np.abs(q16(C) - C)) <= np.max(scales) / 2 + 1e-15
    assert np.max(np.abs(q16(C) - C)) / np.abs(C).max() < 2 ** -14


def test_latent_channels_quantize_better_than_original_space():
    """The premise the SVDq page states: when the latent channels' values decay
    quickly, quantizing the coefficients with more bits for the leading
    channels loses far less than quantizing the original 128 channels (per
    token or per channel) with the same average bits."""
    d, r, n = 128, 32, 512
    g = _rng(72)
    G, _ = np.linalg.qr(g.standard_normal((d, d)))
    K = (g.standard_normal((n, d)) * (0.75 ** np.arange(d)) * 10) @ G.T
    _, _, Vt = np.linalg.svd(K, full_matrices=False)
    B = Vt[:r].T
    C = K @ B
    lat = O.LatentQuant([(8, 8), (8, 4), (16, 2)])        # 4 bits per coefficient
    err_lat = np.linalg.norm(lat(C) @ B.T - C @ B.T)
    per_token = O.LatentQuant([(d, 4)])(K)
    per_channel = O.LatentQuant([(n, 4)])(K.T).T
    err_orig = min(np.linalg.norm(per_token @ B @ B.T - C @ B.T),
                   np.linalg.norm(per_channel @ B @ B.T - C @ B.T))
    assert lat.bits_per_coefficient() == 4.0
    assert err_lat < 0.3 * err_orig, (err_lat, err_orig)


def test_factor_with_latent_quant_storage_tracks_the_exact_factor():
    """Applied at every write (new rows and rewrites), a 12-bit-or-more schedule
    keeps the reconstruction near the unquantized factor's."""
    d, r, W = 128, 16, 128
    rows = _low_rank_rows(900, d, 10, seed=73, noise=1e-3)
    exact = O.HeadFactor(d, r, W)
    quant = O.HeadFactor(d, r, W, coef_round=O.LatentQuant([(8, 16), (8, 12)]))
    for f in (exact, quant):
        f.append(rows)
        while f.ready() >= 1:
            f.fold()
    ref = exact.reconstruct()
    assert np.abs(quant.reconstruct() - ref).max() / np.abs(ref).max() < 1e-3


# ----------------------------------------------------------------------------
# joint-head factor (one factor over all KV heads of a layer; oracle only)
# ----------------------------------------------------------------------------


def test_joint_head_factor_lossless_decode_equals_per_head_attention():
    """At r = kv_heads*d the joint factor reproduces every row, so its decode
    is dense attention of each query head over its own KV head's raw rows
    (brute-force loops over heads and tokens)."""
    H, d, g, W = 2, 16, 2, 64
    gen = _rng(80)
    T = 64 * 6 + 9
    K = gen.standard_normal((T, H * d))
    V = gen.standard_normal((T, H * d))
    fk = O.HeadFactor(H * d, H * d, W)
    fv = O.HeadFactor(H * d, H * d, W)
    fk.append(K)
    fv.append(V)
    while fk.ready() >= 1:
        fk.fold()
        fv.fold()
    assert fk.n_c > 0
    q = gen.standard_normal((H * g, d))
    got = O.joint_head_decode(q, fk.full(), fv.full(), H, 1e4)
    for h in range(H * g):
        k = h // g
        Kr = O.rope_rotate(K[:, k * d:(k + 1) * d], np.arange(T), 1e4)
        s = np.array([q[h] @ Kr[t] for t in range(T)]) / np.sqrt(d)
        p = np.exp(s - s.max())
        p /= p.sum()
        want = sum(p[t] * V[t, k * d:(k + 1) * d] for t in range(T))
        np.testing.assert_allclose(got[h], want, atol=1e-10)


def test_joint_factor_uses_directions_shared_by_heads():
    """Heads whose keys share a 12-dim subspace: one joint factor of rank 12
    is exact (rank <= r), while per-head factors of rank 6 each (the same 12
    coefficients per token) are not."""
    H, d, W = 2, 32, 64
    gen = _rng(81)
    G, _ = np.linalg.qr(gen.standard_normal((H * d, 12)))
    Z = gen.standard_normal((64 * 8, 12))
    X = Z @ G.T
    joint = O.HeadFactor(H * d, 12, W)
    joint.append(X)
    heads = [O.HeadFactor(d, 6, W) for _ in range(H)]
    for k, f in enumerate(heads):
        f.append(X[:, k * d:(k + 1) * d])
    for f in [joint] + heads:
        while f.ready() >= 1:
            f.fold()
    n = joint.n_c
    err_joint = np.abs(joint.reconstruct() - X[:n]).max()
    err_heads = max(np.abs(f.reconstruct() - X[:n, k * d:(k + 1) * d]).max() for k, f in enumerate(heads))
    assert err_joint < 1e-10 * np.abs(X).max()
    assert err_heads > 1e-3 * np.abs(X).max()


# ----------------------------------------------------------------------------
# mutation tests: plant mistakes in a copy of the fold, check the pins fail
# ----------------------------------------------------------------------------


def _mutated_fold(kind):
    def fold(B, S, X):
        B = np.asarray(B, float)
        S = np.asarray(S, float)
        X = np.asarray(X, float)
        d, r = B.shape
        b = X.shape[0]
        k = min(b, d - r)
        P = X @ B if kind != "negP" else -(X @ B)
        E = X - (X @ B) @ B.T
        M = np.concatenate([B, E.T], axis=1)
        Qf, _ = np.linalg.qr(M, mode="complete")
        Q = Qf[:, r:r + k] if kind != "index" else Qf[:, r - 1:r - 1 + k]
        R_E = Q.T @ E.T
        core = np.zeros((r + b, r + k))
        core[:r, :r] = np.diag(S) if kind != "dropS" else 0.0
        core[r:, :r] = P
        core[r:, r:] = R_E.T
        _, sigma, Wt = np.linalg.svd(core)
        W = Wt.T if kind != "transpose" else Wt
        W_r = W[:, :r] if kind != "smallest" else W[:, -r:]
        return O.FoldResult(B_new=np.concatenate([B, Q], 1) @ W_r, S_new=sigma[:r],
                            W_top=W_r[:r], C_new=core[r:] @ W_r, W_r=W_r, sigma=sigma,
                            P=P, E=E, Q=Q, R_E=R_E, core=core)
    return fold


@pytest.mark.parametrize("kind", ["negP", "index", "dropS", "transpose", "smallest"])
def test_pins_catch_planted_mistakes(kind, monkeypatch):
    monkeypatch.setattr(O, "fold_block", _mutated_fold(kind))
    caught = []
    for check in (test_exact_rank_history_is_reproduced,
                  lambda: test_fold_identities(64),
                  test_sync_closed_form,
                  lambda: test_full_rank_is_lossless(0)):
        try:
            check()
        except (AssertionError, ValueError, np.linalg.LinAlgError):
            caught.append(check)
    assert caught, f"planted mistake {kind!r} went unnoticed"


def test_residual_sign_is_absorbed_by_rule_q():
    """Rule Q takes R_E = Q^T E^T with Q orthogonal to B, so any multiple of
    the B-components in E cancels: a residual formed with the wrong sign
    gives the same fold.  (Documents why that mutation is not a mistake.)"""
    g = _rng(31)
    B, _ = np.linalg.qr(g.standard_normal((128, 32)))
    S = np.sort(g.uniform(1, 5, 32))[::-1]
    X = g.standard_normal((64, 128))
    good = O.fold_block(B, S, X)
    Ebad = X + (X @ B) @ B.T
    Qf, _ = np.linalg.qr(np.concatenate([B, Ebad.T], 1), mode="complete")
    np.testing.assert_allclose(np.abs(Qf[:, 32:96].T @ Ebad.T), np.abs(good.R_E), atol=1e-11)


def test_oracle_exports():
    for name in ("bf16_round", "ready_blocks", "rope_rotate", "fold_block", "HeadFactor",
                 "dense_decode", "full_kv_bytes", "persistent_kv_bytes", "LatentQuant"):
        assert hasattr(oracle, name)
    _ = itertools


# mutations of the protected-row bookkeeping, the kept-byte formula and the
# latent quantizer: each planted mistake must fail one of their pins


class _FoldFromWrongRow(O.HeadFactor):
    """Protected-row mistake: the block is taken at n_c instead of P + n_c."""

    def fold(self, defer=False, keep_history=False):
        res = O.fold_block(self.B, self.S, self.rows[self.n_c:self.n_c + self.b])
        if self.sync_enabled and self.n_c > 0:
            self.C[:self.n_c] = self.C[:self.n_c] @ res.W_top
        self._Cbuf = self._grown(self._Cbuf, self.n_c + self.b)
        self._Cbuf[self.n_c:self.n_c + self.b] = res.C_new
        self.B, self.S = res.B_new, res.S_new
        self.n_c += self.b
        return res


class _ReadyIgnoresProtect(O.HeadFactor):
    """Protected-row mistake: blocks counted from position 0."""

    def ready(self):
        return O.ready_blocks(self.T, self.n_c, self.W, self.b)


@pytest.mark.parametrize("cls", [_FoldFromWrongRow, _ReadyIgnoresProtect])
def test_protected_row_pins_catch_planted_mistakes(cls, monkeypatch):
    monkeypatch.setattr(O, "HeadFactor", cls)
    with pytest.raises(AssertionError):
        test_protected_factor_is_the_unprotected_factor_of_the_shifted_stream(37)


def test_kept_bytes_pin_catches_a_dropped_term(monkeypatch):
    real = O.persistent_kv_bytes

    def no_protected(n_c, n_w, d, r_k, r_v, coef_bytes, kv_bytes, basis_bytes=4, n_p=0):
        return real(n_c, n_w, d, r_k, r_v, coef_bytes, kv_bytes, basis_bytes, 0)

    monkeypatch.setattr(O, "persistent_kv_bytes", no_protected)
    with pytest.raises(AssertionError):
        test_persistent_bytes_count_the_kept_arrays()


def test_latent_quant_pin_catches_a_wrong_level_count(monkeypatch):
    def wide(self, C):
        # mistake: 2^b - 1 levels on each side instead of 2^(b-1) - 1
        C = np.atleast_2d(np.asarray(C, dtype=np.float64))
        codes = np.zeros(C.shape, dtype=np.int64)
        scales = np.zeros((C.shape[0], len(self.groups)))
        for g, (lo, hi, bits) in enumerate(self._spans(C.shape[1])):
            if bits == 0:
                continue
            qmax = 2 ** bits - 1
            sc = np.abs(C[:, lo:hi]).max(axis=1) / qmax
            scales[:, g] = sc
            safe = np.where(sc > 0, sc, 1.0)[:, None]
            codes[:, lo:hi] = np.clip(np.round(C[:, lo:hi] / safe), -qmax, qmax)
        return codes, scales

    monkeypatch.setattr(O.LatentQuant, "quantize", wide)
    with pytest.raises(AssertionError):
        test_latent_quant_is_the_nearest_grid_point()


def test_joint_head_pin_catches_a_wrong_head_slice(monkeypatch):
    real = O.joint_head_decode

    def shifted(q, K_full, V_full, kv_heads, theta, use_rope=True):
        # mistake: query heads read the next KV head's columns
        d = np.atleast_2d(q).shape[1]
        return real(q, np.roll(K_full, -d, axis=1), np.roll(V_full, -d, axis=1), kv_heads, theta,
                    use_rope)

    monkeypatch.setattr(O, "joint_head_decode", shifted)
    with pytest.raises(AssertionError):
        test_joint_head_factor_lossless_decode_equals_per_head_attention()


# ----------------------------------------------------------------------------
# where bf16 coefficient storage rounds: new rows, each per-fold rewrite, and
# once per postponed segment.  Pinned by two facts independent of the code:
# a stored value is a bf16 number, and one round-to-nearest step moves a value
# by at most the unit roundoff u = 2^-8 of bf16's 8-bit significand.
# ----------------------------------------------------------------------------

_U_BF16 = 2.0 ** -8


def _is_bf16(x):
    return np.array_equal(O.bf16_round(x), x)


def _within_one_rounding(stored, exact):
    return bool(np.all(np.abs(stored - exact) <= _U_BF16 * np.abs(exact)))


def _storage_rows(seed):
    return _low_rank_rows(64 * 14, 128, 24, seed=seed, noise=0.05)


def test_bf16_storage_rounds_new_rows_and_every_rewrite_once():
    """Per-fold rewrites: after every fold all stored coefficients are bf16
    values, the block's rows are fold_block's C_new rounded once, and the old
    rows are the previously stored rows times W_top rounded once."""
    rows = _storage_rows(5)
    f = O.HeadFactor(128, 16, 64, coef_round="bf16")
    f.append(rows)
    folds = 0
    while f.ready() > 0:
        prev = f.C.copy()
        res = f.fold()
        C = f.C
        assert _is_bf16(C)
        assert _within_one_rounding(C[prev.shape[0]:], res.C_new)
        if prev.shape[0]:
            assert _within_one_rounding(C[:prev.shape[0]], prev @ res.W_top)
        folds += 1
    assert folds >= 10


def test_bf16_storage_rounds_a_postponed_segment_once():
    """Postponed rewrites: new rows are rounded when written; iskv's postponed
    segment is applied as one product per row and rounded once, so every row
    stays within one rounding of (stored row) x W_top(i) ... W_top(k)."""
    rows = _storage_rows(6)
    f = O.HeadFactor(128, 16, 64, coef_round="bf16")
    f.append(rows[:64 * 4])
    _fold_all(f)
    before = f.C.copy()
    f.append(rows[64 * 4:])
    tops, starts = [], []
    while f.ready() > 0:
        starts.append(f.n_c)
        res = f.fold(defer=True)
        tops.append(res.W_top)
        assert _is_bf16(f.C)                      # new rows rounded at once
    assert len(tops) >= 8
    written = f.C.copy()                          # rows as stored before the rewrite
    f.sync()
    C = f.C
    assert _is_bf16(C)
    for i, n0 in enumerate(starts):
        lo = starts[i - 1] if i > 0 else 0
        if n0 <= lo:
            continue
        chain = np.eye(16)
        for W_top in tops[i:]:
            chain = chain @ W_top
        src = before[lo:n0] if i == 0 else written[lo:n0]
        assert _within_one_rounding(C[lo:n0], src @ chain), i


def _skip_rounding(which):
    real = O._store

    def store(x, coef_round):
        new_rows = np.shape(x)[0] == 64
        if (which == "new" and new_rows) or (which == "rewrite" and not new_rows):
            return np.asarray(x, dtype=np.float64)
        return real(x, coef_round)
    return store


class _RoundsEveryPostponedStep(O.HeadFactor):
    """Storage mistake: the postponed chain is rounded after every factor."""

    def sync(self):
        lo = 0
        for i, (n_rows, _) in enumerate(self.pending):
            if n_rows > lo:
                for _, W_top in self.pending[i:]:
                    self.C[lo:n_rows] = O.bf16_round(self.C[lo:n_rows] @ W_top)
                lo = n_rows
        self.pending = []


@pytest.mark.parametrize("which", ["new", "rewrite"])
def test_storage_pins_catch_a_dropped_rounding(which, monkeypatch):
    monkeypatch.setattr(O, "_store", _skip_rounding(which))
    with pytest.raises(AssertionError):
        test_bf16_storage_rounds_new_rows_and_every_rewrite_once()


def test_storage_pins_catch_a_rounding_per_postponed_step(monkeypatch):
    monkeypatch.setattr(O, "HeadFactor", _RoundsEveryPostponedStep)
    with pytest.raises(AssertionError):
        test_bf16_storage_rounds_a_postponed_segment_once()


# ----------------------------------------------------------------------------
# the float32-decision latent quantizer (the precision of the CUDA format)
# ----------------------------------------------------------------------------


def test_latent_quant_fp32_is_the_nearest_float32_grid_point():
    """In float32 mode, per row and group: the scale is the float32 quotient
    amax / qmax of the float32 values, and each stored value is the float32
    product code * scale of the grid point nearest the float32 value (checked
    by brute force over every level; a quotient within one float32 rounding
    of a half-way point may go either way)."""
    g = _rng(80)
    C = g.standard_normal((64, 32)) * (2.0 ** -np.arange(32) * 8 + 0.1)
    C[5] = 0.0
    q = O.LatentQuant([(8, 8), (8, 4), (16, 2)], fp32=True)
    codes, scales = q.quantize(C)
    got = q.dequantize(codes, scales)
    C32 = C.astype(np.float32)
    for gi, (lo, hi, b) in enumerate([(0, 8, 8), (8, 16, 4), (16, 32, 2)]):
        qmax = 2 ** (b - 1) - 1
        for i in range(C.shape[0]):
            amax = np.float32(np.abs(C32[i, lo:hi]).max())
            sc = np.float32(amax / np.float32(qmax))
            assert np.float32(scales[i, gi]) == sc and scales[i, gi] == float(sc)
            if sc == 0:
                assert np.all(got[i, lo:hi] == 0)
                continue
            for j in range(lo, hi):
                x = float(C32[i, j])
                k = codes[i, j]
                assert abs(k) <= qmax
                assert got[i, j] == float(np.float32(np.float32(k) * sc))
                dist = np.abs(np.arange(-qmax, qmax + 1) * float(sc) - x)
                near_half = abs(abs(x / float(sc)) % 1.0 - 0.5) < 1e-6
                assert dist[k + qmax] <= dist.min() + 1e-12 or near_half


def test_latent_quant_fp32_agrees_with_float64_away_from_half_way_points():
    """float32 and float64 decisions differ only where the quotient x / scale
    lies within float32 rounding of a half-way point, and then by one code."""
    g = _rng(81)
    C = g.standard_normal((400, 32)) * (2.0 ** -np.arange(32) * 8 + 0.1)
    q64 = O.LatentQuant([(8, 8), (8, 4), (16, 2)])
    q32 = O.LatentQuant([(8, 8), (8, 4), (16, 2)], fp32=True)
    c64, s64 = q64.quantize(C)
    c32, s32 = q32.quantize(C)
    np.testing.assert_allclose(s32, s64, rtol=2 ** -22, atol=0)
    diff = c32 != c64
    assert np.abs(c32 - c64).max() <= 1
    assert diff.mean() < 1e-3
    for i, j in zip(*np.nonzero(diff)):
        gi = 0 if j < 8 else (1 if j < 16 else 2)
        u = abs(C[i, j] / s64[i, gi])
        assert abs(u % 1.0 - 0.5) < 1e-5, (i, j, u)


def test_latent_quant_fp32_pin_catches_float64_decisions(monkeypatch):
    """A quantizer that divides in float64 instead of float32 is caught."""
    real = O.LatentQuant.quantize

    def f64_division(self, C):
        keep = self.fp32
        self.fp32 = False
        try:
            return real(self, np.asarray(C, dtype=np.float32).astype(np.float64))
        finally:
            self.fp32 = keep

    monkeypatch.setattr(O.LatentQuant, "quantize", f64_division)
    with pytest.raises(AssertionError):
        test_latent_quant_fp32_is_the_nearest_float32_grid_point()


def test_latent_quant_row_bytes_counts_codes_and_scales():
    """A coded row keeps bits x channels of codes per group and one 4-byte
    scale per group with codes (none for dropped groups)."""
    q = O.LatentQuant([(8, 8), (8, 4), (16, 2)])
    assert q.row_bytes() == 8 + 4 + 4 + 3 * 4
    assert O.LatentQuant([(16, 8), (16, 0)]).row_bytes() == 16 + 4
    codes, scales = q.quantize(np.ones((3, 32)))
    per_row_bits = sum(n * b for n, b in q.groups)
    assert per_row_bits // 8 + 4 * np.count_nonzero(scales[0]) == q.row_bytes()
    assert O.persistent_kv_bytes(64, 10, 128, 32, 32, 2, 2, coef_row_bytes=100) == \
        64 * 100 + 129 * 64 * 4 + 2 * 10 * 128 * 2
