"""Float64 restatement of iS-KV's per-head state machine.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  Nothing here is blocked,
fused or reordered beyond the method's own steps; numpy's LAPACK SVD and QR
serve as library primitives for the two factorizations the method names.

Notation follows the iS-KV explainer ("iS-KV -- Basis-synchronized online
low-rank KV compression -- What does it mean?"):
  d  head dimension, r rank, b = 64 block rows, W exact recent window,
  B  d x r orthonormal basis, S r singular values, C n_c x r coefficients,
  T  tokens appended, n_c tokens folded into (B, S, C).  The exact window is
  rows [n_c, T).

Readings of points the pages leave open (each one is stated where used):
  * a block is folded once T - n_c >= W + b (Jargon: Block-incremental SVD;
    body paragraph on folding 64 tokens as they leave the recent window);
  * initial state B = I_d[:, :r], S = 0, n_c = 0;
  * the residual is re-orthogonalized against B once more (twice is enough);
  * the complement basis Q comes from a Householder QR of [B | E^T] with
    k = min(b, d - r) columns ("rule Q"); it equals the QR of E^T when E has
    full rank and k = b, and keeps [B, Q] orthonormal when r + b > d;
  * truncation keeps the r largest singular values (fixed rank);
  * RoPE is the rotate-half form on pairs (i, i + d/2) with
    inv_freq_i = theta^(-2i/d) at absolute 0-based positions; keys are stored
    pre-RoPE and rotated when attention reads them (Jargon: Pre-RoPE keys);
  * bf16 coefficient storage is emulated by rounding to the nearest bf16
    value (ties to even) wherever the stored coefficients are written.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = [
    "bf16_round",
    "ready_blocks",
    "rope_inv_freq",
    "rope_rotate",
    "fold_block",
    "FoldResult",
    "HeadFactor",
    "dense_decode",
    "full_kv_bytes",
    "persistent_kv_bytes",
    "LatentQuant",
    "joint_head_decode",
]

# ----------------------------------------------------------------------------
# Storage rounding
# ----------------------------------------------------------------------------

_BF16_MAX = float.fromhex("0x1.fep127")


def bf16_round(x):
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits and float32's exponent range.  For
    |x| = m * 2^e with 0.5 <= m < 1 the quantum is 2^(e - 8) (bf16 subnormals:
    2^-133).  Scaling by a power of two is exact, and ``np.round`` rounds half
    to even, so the result is exact.  Pinned in the tests against torch's own
    float32 -> bfloat16 conversion and against hand-built tie cases.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0)
    if np.any(fin):
        xv = x[fin]
        _, e = np.frexp(xv)
        e = np.maximum(e, -125)
        q_exp = e - 8
        scaled = np.ldexp(xv, -q_exp)
        rv = np.ldexp(np.round(scaled), q_exp)
        rv = np.where(np.abs(rv) > _BF16_MAX, np.copysign(np.inf, rv), rv)
        out[fin] = rv
    return out


class LatentQuant:
    """Low-bit storage of coefficient rows, channel by channel (SVDq page,
    Abstract: the key cache is moved into SVD latent channels, whose values
    decay quickly, and the more significant channels get more precision).

    Reading, for iS-KV's coefficients: column j of C is latent channel j, and
    the factor keeps its columns in descending singular-value order, so
    significance falls with j.  ``groups`` lists (channels, bits) from the
    first channel on, bits 2..16; 0 bits drops the channels (stored as zero, the page's
    compression of negligible channels).  Each row is quantized per group,
    symmetrically and uniformly: scale = max |x| / (2^(b-1) - 1), code =
    round-half-even(x / scale) in [-(2^(b-1) - 1), 2^(b-1) - 1]; a group of
    zeros keeps scale 0.  The pages give no scale rule or bit schedule; this is
    the plainest per-token choice.  Used as a coefficient storage format
    (``coef_round``): applied at every write, new rows and every rewrite.

    ``fp32=True`` takes every rounding decision in IEEE float32, the precision
    of the CUDA kernels that store this format: the values are first rounded
    to float32, the group maximum and the scale amax / qmax are float32
    (a correctly rounded division), each code is the float32 quotient x / scale
    rounded half to even, and a stored value is the float32 product
    code * scale.  Codes then agree bit for bit with a float32 quantizer fed
    the same float32 values.
    """

    def __init__(self, groups, fp32: bool = False):
        self.groups = [(int(n), int(b)) for n, b in groups]
        self.fp32 = bool(fp32)
        if any(n <= 0 or not (b == 0 or 2 <= b <= 16) for n, b in self.groups):
            raise ValueError("invalid channel groups")

    def _spans(self, r):
        if sum(n for n, _ in self.groups) != r:
            raise ValueError("channel groups must cover the rank")
        lo = 0
        for n, b in self.groups:
            yield lo, lo + n, b
            lo += n

    def quantize(self, C):
        """Integer codes (same shape as C) and scales (rows x groups)."""
        C = np.atleast_2d(np.asarray(C, dtype=np.float64))
        if self.fp32:
            C = C.astype(np.float32)
        codes = np.zeros(C.shape, dtype=np.int64)
        scales = np.zeros((C.shape[0], len(self.groups)), dtype=C.dtype)
        for g, (lo, hi, b) in enumerate(self._spans(C.shape[1])):
            if b == 0:
                continue
            qmax = 2 ** (b - 1) - 1
            amax = np.abs(C[:, lo:hi]).max(axis=1)
            sc = amax / C.dtype.type(qmax)
            scales[:, g] = sc
            safe = np.where(sc > 0, sc, C.dtype.type(1.0))[:, None]
            codes[:, lo:hi] = np.clip(np.round(C[:, lo:hi] / safe), -qmax, qmax).astype(np.int64)
        return codes, scales.astype(np.float64)

    def dequantize(self, codes, scales):
        codes = np.atleast_2d(codes)
        out = np.zeros(codes.shape)
        for g, (lo, hi, _) in enumerate(self._spans(codes.shape[1])):
            if self.fp32:
                prod = codes[:, lo:hi].astype(np.float32) * scales[:, g:g + 1].astype(np.float32)
                out[:, lo:hi] = prod.astype(np.float64)
            else:
                out[:, lo:hi] = codes[:, lo:hi] * scales[:, g:g + 1]
        return out

    def __call__(self, C):
        C = np.asarray(C, dtype=np.float64)
        return self.dequantize(*self.quantize(C)).reshape(C.shape)

    def bits_per_coefficient(self) -> float:
        """Average code bits per stored coefficient (scales not counted)."""
        n = sum(n for n, _ in self.groups)
        return sum(n * b for n, b in self.groups) / n

    def row_bytes(self, scale_bytes: int = 4) -> int:
        """Bytes one stored row keeps: its codes (bits per channel, whole
        bytes per group) and one scale per group that has codes."""
        return sum((n * b + 7) // 8 for n, b in self.groups) + scale_bytes * sum(
            1 for _, b in self.groups if b > 0)


def _store(x, coef_round):
    if coef_round is None:
        return np.asarray(x, dtype=np.float64)
    if isinstance(coef_round, LatentQuant):
        return coef_round(x)
    if coef_round == "bf16":
        return bf16_round(x)
    if coef_round == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    raise ValueError(f"unknown coefficient storage {coef_round!r}")


# ----------------------------------------------------------------------------
# Window and block bookkeeping
# ----------------------------------------------------------------------------


def ready_blocks(T: int, n_c: int, W: int, b: int = 64) -> int:
    """Number of whole b-row blocks that have left the exact window.

    The newest W tokens stay exact; the rows [n_c, T - W) are old enough to be
    folded, in whole blocks of b (the explainer's body: the compressed history
    grows by one 64-row block at a time, as blocks age out of the window).  Pinned by brute
    force over all small (T, n_c, W) in the tests.
    """
    if T < 0 or n_c < 0 or W < 0 or b <= 0 or n_c > T:
        raise ValueError("invalid counters")
    excess = T - n_c - W
    return excess // b if excess >= 0 else 0


# ----------------------------------------------------------------------------
# RoPE (Jargon: Pre-RoPE keys)
# ----------------------------------------------------------------------------


def rope_inv_freq(d: int, theta: float) -> np.ndarray:
    """inv_freq_i = theta^(-2i/d) for the d/2 rotation pairs."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * i / d)


def rope_rotate(x, pos, theta: float) -> np.ndarray:
    """Rotate rows of ``x`` (n x d) by RoPE at absolute positions ``pos``.

    Pair i is (x[i], x[i + d/2]) and turns by the angle pos * inv_freq_i.
    Pinned in the tests: norm preservation, R(a)^T R(b) = R(b - a) (scores
    depend only on relative position), identity at position 0 and a
    hand-computed d = 4 case.
    """
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * rope_inv_freq(d, theta)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[:, :h], x[:, h:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=1)


# ----------------------------------------------------------------------------
# One block fold: steps (a)-(d) of the block-incremental SVD
# ----------------------------------------------------------------------------


@dataclass
class FoldResult:
    B_new: np.ndarray   # d x r, new orthonormal basis  [B, Q] W_r
    S_new: np.ndarray   # r, leading singular values of the core
    W_top: np.ndarray   # r x r, W_r[0:r, :], the resync map for old rows
    C_new: np.ndarray   # b x r, coefficients of the folded block
    W_r: np.ndarray     # (r+k) x r
    sigma: np.ndarray   # all r+k singular values of the core, descending
    P: np.ndarray       # b x r projection of the block
    E: np.ndarray       # b x d residual
    Q: np.ndarray       # d x k complement basis
    R_E: np.ndarray     # k x b, Q^T E^T
    core: np.ndarray    # (r+b) x (r+k)


def fold_block(B, S, X) -> FoldResult:
    """Fold one block X (b x d) into the rank-r factorization (B, S).

    Brand's block-incremental SVD as the iS-KV explainer applies it (Jargon:
    Block-incremental SVD; body paragraph on the joint update of basis and
    coefficients, whose decomposition works on a fixed-size core matrix,
    independent of how many rows the history holds):
      (a) P = X B
      (b) E = X - P B^T (re-orthogonalized once more), Q and R_E from rule Q
      (c) core = [[diag S, 0], [P, R_E^T]], SVD core = U Sigma W^T, keep r
      (d) B' = [B, Q] W_r, S' = sigma_1..r, new rows [P, R_E^T] W_r,
          and W_top = W_r[0:r, :] for step (e), done by the caller.
    Pinned in the tests: exactness when the history has rank <= r against the
    covariance-route batch SVD, losslessness at r = d, orthonormality of B',
    the reconstruction identity X = P B^T + R_E^T Q^T and the energy balance of
    the truncation.
    """
    B = np.asarray(B, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    d, r = B.shape
    b = X.shape[0]
    k = min(b, d - r)

    # (a) project the block onto the current basis
    P = X @ B
    # (b) residual, with one re-orthogonalization pass against B
    E = X - P @ B.T
    P2 = E @ B
    E = E - P2 @ B.T
    P = P + P2
    # rule Q: Householder QR of [B | E^T]; columns r..r+k-1 of the full Q
    M = np.concatenate([B, E.T], axis=1)
    Qf, _ = np.linalg.qr(M, mode="complete")
    Q = Qf[:, r:r + k]
    R_E = Q.T @ E.T
    # (c) the small core and its SVD, truncated to rank r
    core = np.zeros((r + b, r + k))
    core[:r, :r] = np.diag(S)
    core[r:, :r] = P
    core[r:, r:] = R_E.T
    _, sigma, Wt = np.linalg.svd(core, full_matrices=True)
    Wfull = Wt.T
    W_r = Wfull[:, :r]
    # (d) new basis, new singular values, coefficients of the new rows
    B_new = np.concatenate([B, Q], axis=1) @ W_r
    C_new = core[r:, :] @ W_r
    return FoldResult(B_new=B_new, S_new=sigma[:r].copy(), W_top=W_r[:r, :].copy(),
                      C_new=C_new, W_r=W_r, sigma=sigma, P=P, E=E, Q=Q, R_E=R_E,
                      core=core)


# ----------------------------------------------------------------------------
# Per head-instance state: exact rows + (B, S, C)
# ----------------------------------------------------------------------------


class HeadFactor:
    """One (sequence, layer, KV head, K-or-V) factor with its exact window.

    ``coef_round`` selects the storage format of C: None (float64, exact
    oracle), "f32" or "bf16" (emulated at every write: new rows at a fold and
    every resync).  ``sync=False`` is the no-synchronization ablation: old
    rows keep the coefficients of the basis they were written in.

    ``protect`` = P leading positions (protected prompt rows, kept exact
    beside the recent window: the explainer's paint-shop section and its
    Persistent-KV compression entry) never enter the factor: the factor's
    stream is rows P, P+1, ..., its blocks are counted and folded as if the
    stream began there, and attention sees positions 0..P-1 exact, then the
    n_c folded rows, then the window.

    ``fold(defer=True)`` postpones step (e) for the rows already stored; the
    postponed rewrites are applied in order by ``sync()``, with one storage
    rounding at the end.  With nothing read in between this equals the
    per-fold rewrite in exact arithmetic (each rewrite is a right
    multiplication of the rows that existed before that fold).
    """

    def __init__(self, d: int, r: int, W: int, b: int = 64, coef_round=None,
                 sync: bool = True, protect: int = 0):
        if not (0 < r <= d) or b <= 0 or W < 0 or protect < 0:
            raise ValueError("invalid factor shape")
        self.d, self.r, self.W, self.b = d, r, W, b
        self.P = protect
        self.coef_round = coef_round
        self.sync_enabled = sync
        self.B = np.eye(d)[:, :r].copy()
        self.S = np.zeros(r)
        # row storage grows by doubling (appending block by block to plain
        # arrays would copy the whole history every time)
        self._Cbuf = np.zeros((0, r))
        self._rowbuf = np.zeros((0, d))
        self._nrows = 0
        self.n_c = 0
        self.pending = []           # [(rows_before_fold, W_top)]
        self.history = []           # FoldResult per fold (for drift studies)

    @property
    def T(self) -> int:
        return self._nrows

    @property
    def rows(self) -> np.ndarray:
        """All appended rows (T x d), oldest first."""
        return self._rowbuf[:self._nrows]

    @property
    def C(self) -> np.ndarray:
        """Stored coefficient rows (n_c x r)."""
        return self._Cbuf[:self.n_c]

    @C.setter
    def C(self, value) -> None:
        # replaces the stored rows; n_c has to be set to match by the caller
        self._Cbuf = np.array(value, dtype=np.float64).reshape(-1, self.r)

    @rows.setter
    def rows(self, value) -> None:
        self._rowbuf = np.array(value, dtype=np.float64).reshape(-1, self.d)
        self._nrows = self._rowbuf.shape[0]

    @staticmethod
    def _grown(buf: np.ndarray, need: int) -> np.ndarray:
        if need <= buf.shape[0]:
            return buf
        out = np.zeros((max(need, 2 * buf.shape[0], 256), buf.shape[1]))
        out[:buf.shape[0]] = buf
        return out

    def append(self, rows) -> int:
        rows = np.asarray(rows, dtype=np.float64).reshape(-1, self.d)
        self._rowbuf = self._grown(self._rowbuf, self._nrows + rows.shape[0])
        self._rowbuf[self._nrows:self._nrows + rows.shape[0]] = rows
        self._nrows += rows.shape[0]
        return self.ready()

    @property
    def T_factor(self) -> int:
        """Rows of the factor's stream (those after the protected positions)."""
        return max(0, self.T - self.P)

    def ready(self) -> int:
        return ready_blocks(self.T_factor, self.n_c, self.W, self.b)

    def fold(self, defer: bool = False, keep_history: bool = False) -> FoldResult:
        if self.ready() < 1:
            raise RuntimeError("no ready block")
        X = self.rows[self.P + self.n_c:self.P + self.n_c + self.b]
        res = fold_block(self.B, self.S, X)
        # (e) basis synchronization of the rows stored so far
        if self.sync_enabled and self.n_c > 0:
            if defer:
                self.pending.append((self.n_c, res.W_top))
            else:
                self.C[:self.n_c] = _store(self.C[:self.n_c] @ res.W_top, self.coef_round)
        self._Cbuf = self._grown(self._Cbuf, self.n_c + self.b)
        self._Cbuf[self.n_c:self.n_c + self.b] = _store(res.C_new, self.coef_round)
        self.B, self.S = res.B_new, res.S_new
        self.n_c += self.b
        if keep_history:
            self.history.append(res)
        return res

    def sync(self) -> None:
        """Apply postponed rewrites, then round once.

        A row stored before postponed fold i (of k) is rewritten by
        W_top(i) W_top(i+1) ... W_top(k), the folds that came after it, in
        order; rows between the row counts of folds i-1 and i take the suffix
        product starting at fold i.  The same matrices as rewriting after each
        fold, grouped so that every row is multiplied once."""
        if not self.pending:
            return
        C = self.C                      # rewritten in place
        k = len(self.pending)
        suffix = [None] * k
        acc = None
        for i in range(k - 1, -1, -1):
            W_top = self.pending[i][1]
            acc = W_top if acc is None else W_top @ acc
            suffix[i] = acc
        lo = 0
        for i, (n_rows, _) in enumerate(self.pending):
            if n_rows > lo:
                C[lo:n_rows] = C[lo:n_rows] @ suffix[i]
                lo = n_rows
        C[:lo] = _store(C[:lo], self.coef_round)
        self.pending = []

    def reconstruct(self) -> np.ndarray:
        """Pre-RoPE reconstruction C B^T of the folded rows (n_c x d)."""
        if self.pending:
            raise RuntimeError("postponed rewrites pending; call sync()")
        return self.C @ self.B.T

    def protected(self) -> np.ndarray:
        """The protected rows (positions 0 .. min(T, P) - 1), as appended."""
        return self.rows[:min(self.T, self.P)]

    def exact(self) -> np.ndarray:
        """The exact window: positions P + n_c .. T - 1."""
        return self.rows[self.P + self.n_c:]

    def full(self) -> np.ndarray:
        """All T rows in position order as attention sees them: protected,
        reconstructed, then the exact window."""
        return np.concatenate([self.protected(), self.reconstruct(), self.exact()], axis=0)

    def kept_arrays(self) -> list:
        """The arrays this factor keeps between decode steps: the protected and
        window rows, and, once a block is folded, C, B and S."""
        out = [self.protected(), self.exact()]
        if self.n_c > 0:
            out += [self.C, self.B, self.S]
        return out


# ----------------------------------------------------------------------------
# Decode attention over the mixed cache
# ----------------------------------------------------------------------------


def dense_decode(q, K_pre, V, theta: float, use_rope: bool = True) -> np.ndarray:
    """Softmax attention of query heads ``q`` (g x d) over T rows.

    ``K_pre`` holds the keys before RoPE (reconstructed rows, then the exact
    window); they are rotated at absolute positions 0..T-1 here, the query is
    taken as already rotated (it belongs to position T-1).  Scale 1/sqrt(d),
    no mask.  This is the plain definition; the method's value-side shortcut
    out = (p^T C_V) B_V^T + p_win^T V_win is the same sum regrouped.  Pinned by
    brute-force loops in the tests.
    """
    q = np.atleast_2d(np.asarray(q, dtype=np.float64))
    K_pre = np.asarray(K_pre, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    T, d = K_pre.shape
    Kr = rope_rotate(K_pre, np.arange(T), theta) if use_rope else K_pre
    s = (q @ Kr.T) / np.sqrt(d)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V


def joint_head_decode(q, K_full, V_full, kv_heads: int, theta: float, use_rope: bool = True):
    """Decode with one factor per layer over all KV heads (the joint-head
    reading of the explainer's ranks 64/96/128, worked-example table): the
    factor's rows are the KV heads' rows side by side (T x kv_heads*d), so a
    HeadFactor of dimension kv_heads*d is the joint factor; query head h
    attends over columns [k d, (k+1) d) of the joint rows, k = h // g.
    ``q`` is (q_heads x d).  Oracle only: the CUDA path factors per head."""
    q = np.atleast_2d(np.asarray(q, dtype=np.float64))
    Hq, d = q.shape
    g = Hq // kv_heads
    out = np.zeros((Hq, d))
    for h in range(Hq):
        k = h // g
        out[h] = dense_decode(q[h:h + 1], K_full[:, k * d:(k + 1) * d], V_full[:, k * d:(k + 1) * d],
                              theta, use_rope)[0]
    return out


# ----------------------------------------------------------------------------
# Memory accounting (Jargon: Persistent-KV compression)
# ----------------------------------------------------------------------------


def full_kv_bytes(tokens: int, layers: int, kv_heads: int, head_dim: int,
                  elem_bytes: int) -> int:
    """Bytes of an uncompressed K and V cache.  Pinned by the A40 memory test
    figure of the explainer (full cache at a 32K input + 1,024 steps)."""
    return tokens * layers * kv_heads * head_dim * 2 * elem_bytes


def persistent_kv_bytes(n_c: int, n_w: int, d: int, r_k: int, r_v: int,
                        coef_bytes: int, kv_bytes: int, basis_bytes: int = 4,
                        n_p: int = 0, coef_row_bytes: int | None = None) -> int:
    """Bytes kept between decode steps for one (sequence, layer, KV head)
    (Jargon: Persistent-KV compression): both factors (C, and B, S once a
    block is folded), both exact windows (n_w rows) and both sets of
    protected rows (n_p).  Excludes temporary buffers, as the explainer's
    definition does.  Pinned against a count of the arrays the oracle keeps;
    the explainer's kept-byte figure itself (1.808 GiB on the A40) cannot be
    re-derived from what the pages state, so that number stays unpinned."""
    factors = 0
    if n_c > 0:
        # coef_row_bytes: one row of K and V coefficients when they are not
        # stored element by element (LatentQuant.row_bytes of both factors)
        row = (r_k + r_v) * coef_bytes if coef_row_bytes is None else coef_row_bytes
        factors = n_c * row + (d + 1) * (r_k + r_v) * basis_bytes
    exact = 2 * (n_w + n_p) * d * kv_bytes
    return factors + exact
