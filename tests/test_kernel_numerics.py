"""The algebra and the number formats the decode and rewrite kernels rest on,
checked on the CPU in float64 against the oracle's plain definitions.  The
GPU parity tests compare the kernels' outputs with the oracle; these pin the
rearrangements themselves, so that a wrong sign or index in a derivation
shows up here as well as there:

* the query-side RoPE identity: q . R_p B c = sum_m c_m (T_p A)_m;
* the per-tile query pre-rotation: q . R_j k = (R_t^T q) . R_(j-t) k;
* split-K softmax with a lazily kept running maximum, merged by log-sum-exp;
* the three-part bf16 split of an fp32 matrix (exact) and the hi + lo
  splits of the basis (bf16) and the queries (fp16);
* the CUDA-core decode's RoPE by stepped fp32 rotations, R(j) R(4t) R(1)^u.
"""

import numpy as np
import pytest
import torch

import oracle as O

D = 128
THETA = 1e6


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _fp16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float16).double().numpy()


@pytest.mark.parametrize("pos", [0, 7, 4095, 262_143])
def test_query_side_rope_identity(pos):
    """For a folded row k = B c at position p: q . R_p k equals
    sum_m c_m U_m with U = T_p A, T_p = [cos(p w_i), sin(p w_i)]_i and
    A = [alpha; beta], alpha[i, m] = q_i B[i, m] + q_(i+64) B[i+64, m],
    beta[i, m] = q_(i+64) B[i, m] - q_i B[i+64, m]."""
    rng = np.random.default_rng(pos)
    r = 32
    B = np.linalg.qr(rng.standard_normal((D, r)))[0]
    c = rng.standard_normal(r) * 3
    q = rng.standard_normal(D)
    h = D // 2
    alpha = q[:h, None] * B[:h] + q[h:, None] * B[h:]
    beta = q[h:, None] * B[:h] - q[:h, None] * B[h:]
    w = O.rope_inv_freq(D, THETA)
    T = np.concatenate([np.cos(pos * w), np.sin(pos * w)])          # 128
    U = T @ np.vstack([alpha, beta])                                 # r
    want = q @ O.rope_rotate((B @ c)[None, :], [pos], THETA)[0]
    assert abs(c @ U - want) <= 1e-12 * np.linalg.norm(q) * np.linalg.norm(B @ c)


def test_query_pre_rotation_leaves_only_the_in_tile_angle():
    """The rotation kernel turns q' = R_t^T q once per tile starting at t and
    each row j of the tile by j - t only: q . R_j k = q' . R_(j-t) k."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal(D)
    t = 40_960
    for j in (t, t + 1, t + 63, t + 127):
        k = rng.standard_normal(D)
        # R_t^T q = R_(-t) q
        q_pre = O.rope_rotate(q[None, :], [-t], THETA)[0]
        lhs = q @ O.rope_rotate(k[None, :], [j], THETA)[0]
        rhs = q_pre @ O.rope_rotate(k[None, :], [j - t], THETA)[0]
        assert abs(lhs - rhs) < 1e-10 * np.linalg.norm(q) * np.linalg.norm(k)


def _lazy_tile_softmax(s, v, lazy=8.0):
    """One split's online softmax over tiles of 128 scores, the way the
    epilogue keeps it: the running max moves only when a tile's max passes
    it by more than `lazy` (then the sums are rescaled exactly)."""
    m, l, acc = -np.inf, 0.0, np.zeros(v.shape[1])
    for a in range(0, len(s), 128):
        st, vt = s[a:a + 128], v[a:a + 128]
        tmax = st.max()
        if not np.isfinite(m) or tmax > m + lazy:
            m_new = max(m, tmax)
            scale = np.exp(m - m_new) if np.isfinite(m) else 0.0
            l, acc, m = l * scale, acc * scale, m_new
        p = np.exp(st - m)
        l += p.sum()
        acc += p @ vt
    return m, l, acc


def test_split_softmax_with_lazy_max_merges_to_the_dense_softmax():
    rng = np.random.default_rng(2)
    n, dv = 5000, 16
    s = rng.standard_normal(n) * 3
    s[1234] += 30                      # one dominant score (a recall query)
    s[4321] += 9                       # a jump of more than the lazy margin later on
    v = rng.standard_normal((n, dv))
    cuts = [0, 700, 701, 2222, 4000, n]            # uneven splits, one of a single row
    parts = [_lazy_tile_softmax(s[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    M = max(p[0] for p in parts)
    L = sum(p[1] * np.exp(p[0] - M) for p in parts)
    acc = sum(p[2] * np.exp(p[0] - M) for p in parts)
    e = np.exp(s - s.max())
    want = (e / e.sum()) @ v
    assert np.max(np.abs(acc / L - want)) < 1e-12 * np.max(np.abs(want))
    # the lazily kept sums stay far from overflow: p <= e^8 within a split
    for a, b in zip(cuts[:-1], cuts[1:]):
        m, l, _ = _lazy_tile_softmax(s[a:b], v[a:b])
        assert np.max(s[a:b]) - m <= 8.0


def test_three_bf16_parts_hold_an_fp32_matrix_exactly():
    """W_top of the rewrite as hi + mid + lo, each rounded to bf16 from the
    remainder: their sum is the fp32 value exactly (8 + 8 + 8 significand
    bits), so three bf16 MMAs with fp32 accumulation see W itself."""
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((96, 96)) * np.exp(rng.uniform(-20, 20, (96, 96)))).astype(np.float32)
    W = W.astype(np.float64)
    hi = _bf16(W)
    mid = _bf16(W - hi)
    lo = _bf16(W - hi - mid)
    assert np.array_equal(hi + mid + lo, W)
    # two parts are not enough: a plausible shortcut fails
    assert not np.array_equal(hi + mid, W)


def test_hi_lo_splits_of_basis_and_queries():
    """The basis enters the key rebuild as bf16 hi + lo (16 significand bits:
    relative error <= 2^-16); the queries enter the score MMA as fp16 hi + lo
    (22 bits: error <= 2^-22 of the element, or half fp16's subnormal spacing,
    2^-25, where the low part falls below fp16's normal range)."""
    rng = np.random.default_rng(4)
    B = np.linalg.qr(rng.standard_normal((D, 64)))[0].astype(np.float32).astype(np.float64)
    hi = _bf16(B)
    lo = _bf16(B - hi)
    assert np.max(np.abs(hi + lo - B) / np.abs(B)) <= 2.0 ** -16
    assert np.max(np.abs(hi - B) / np.abs(B)) > 2.0 ** -10        # one bf16 part alone is coarse
    q = (rng.standard_normal(4096) * 4).astype(np.float32).astype(np.float64)
    qh = _fp16(q)
    ql = _fp16(q - qh)
    err = np.abs(qh + ql - q)
    assert np.all(err <= np.maximum(2.0 ** -22 * np.abs(q), 2.0 ** -25))
    assert np.max(np.abs(qh - q) / np.abs(q)) > 2.0 ** -13       # one fp16 part alone is coarse


def _cmul32(a, b):
    """(a.x + i a.y)(b.x + i b.y) with every product and sum rounded to fp32."""
    f = np.float32
    ax, ay, bx, by = (np.asarray(v, dtype=f) for v in (a[0], a[1], b[0], b[1]))
    return (f(ax * bx) - f(ay * by)).astype(f), (f(ax * by) + f(ay * bx)).astype(f)


def test_stepped_fp32_rope_stays_within_a_few_ulps():
    """The CUDA-core decode turns row j + 4t + u of a 64-row tile starting at
    j by R(j) R(4t) R(1)^u: the tile's base rotation and the steps R(4t),
    R(1) are fp32 roundings of float64 tables, the products fp32.  Four
    complex products keep cos and sin within 1.5e-6 of the float64 values at
    any position up to 2^18, far inside the 1e-4 parity bar of fp32
    coefficients (fp32 angles at such positions would be off by ~1e-2 rad)."""
    rng = np.random.default_rng(5)
    w = O.rope_inv_freq(D, THETA)
    tab = lambda pos: (np.cos(pos * w).astype(np.float32), np.sin(pos * w).astype(np.float32))
    worst = 0.0
    for j in list(rng.integers(0, 2 ** 18 // 64, 40) * 64) + [2 ** 18 - 64]:
        rj = tab(j)
        r1 = tab(1)
        for t in range(16):
            rb = _cmul32(rj, tab(4 * t))
            for u in range(4):
                pos = j + 4 * t + u
                worst = max(worst, np.max(np.abs(rb[0] - np.cos(pos * w))),
                            np.max(np.abs(rb[1] - np.sin(pos * w))))
                rb = _cmul32(rb, r1)
    assert worst < 1.5e-6, worst
    # the shortcut the table avoids: the angle formed in fp32
    pos = np.float32(2 ** 18 - 1)
    ang32 = (pos * w.astype(np.float32)).astype(np.float32)
    assert np.max(np.abs(np.cos(ang32.astype(np.float64)) - np.cos(float(pos) * w))) > 1e-3
