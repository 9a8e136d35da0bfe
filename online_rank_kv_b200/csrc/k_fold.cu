// Block fold engine: one CTA per (layer, sequence*KV head) factor folds the
// oldest 64-row block that left the exact window into (B, S, C).
//
// Method: Brand's block-incremental SVD as the iS-KV explainer applies it
// ("iS-KV -- Basis-synchronized online low-rank KV compression -- What does it
// mean?", Jargon: Block-incremental SVD; body paragraph on the joint update of
// basis and coefficients, decomposed on a fixed-size core matrix independent
// of the history's row count).  Steps inside the CTA, fp32, every intermediate in shared
// memory or registers:
//   (a) P = X B.
//   (b) Householder QR of [B | X^T] (d x (r+64)).  Its first r reflections
//       remove the B-components, i.e. they form the residual E = X - P B^T
//       implicitly; Q = columns r..r+k-1 of the orthogonal factor
//       (k = min(64, d - r)) and R_E = rows r..r+k-1 of the triangular
//       factor over the X^T columns.  This keeps [B, Q] orthonormal even when
//       r + 64 > d or the residual is rank deficient.  Q is formed in place
//       (backward accumulation of the reflectors) and parked in a global
//       scratch slot until step (d).
//   (c) SVD of the core K = [[diag S, 0], [P, R_E^T]] ((r+64) x n, n = r+k):
//         - Householder QR of K, exploiting that column j < r of K has
//           nonzeros only in row j and rows r..r+63: K = Q_K R (R n x n);
//         - one-sided (Hestenes) Jacobi on the columns of R^T.  With
//           R^T J = U Sigma, R = J Sigma U^T, so U holds the right singular
//           vectors of K: no rotation has to be accumulated, and the
//           QR-preconditioned Jacobi needs about 7 sweeps where Jacobi on K
//           itself needs 8 and Jacobi on K^T 11-12;
//         - the columns live in registers, eight per block, two blocks per
//           warp: each round rotates eight disjoint pairs of the warp's two
//           blocks (all pairs inside each block once per sweep, then all
//           cross pairs), and blocks travel between warps in the round-robin
//           (circle) order, so every pair of columns meets once per sweep;
//         - column norms are carried through the sweep by the exact update
//           of the rotation and recomputed at its start; a pair is rotated
//           while |a_p . a_q| > tol |a_p| |a_q|; columns whose energy is
//           below 1e-14 ||K||_F^2 are numerically zero and never rotated.
//       sigma = final column norms, sorted descending; W_r = the matching
//       unit columns.  Directions of numerically zero singular values (rank
//       of K below r) are completed by orthonormal vectors (any completion
//       is a correct truncation: K maps all of them to zero).  One Bjorck
//       step W_r <- W_r (3I - W_r^T W_r)/2 restores orthonormality to fp32
//       rounding (a no-op in exact arithmetic).
//   (d) S' = sigma_1..r; W_top = W_r[0:r, :] for step (e);
//       B'' = [B, Q] W_r; new coefficient rows = X B'' (equal to
//       [P, R_E^T] W_r in exact arithmetic: X [B, Q] = [P, R_E^T] because
//       [B, Q] spans the rows of X); B' = B'' after one Bjorck step, written
//       as fp32 plus bf16 hi/lo parts.
// Step (e), the rewrite of the stored coefficients, runs in the resync
// kernels.
#include <utility>

#include "iskv_internal.cuh"

namespace iskv {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;

// smallest stride >= cols that is 8 (mod 32): 4 row-parts x 8 consecutive
// columns of one warp then hit 32 distinct banks
__host__ __device__ constexpr int stride8(int cols) { return cols + ((8 - cols % 32) + 32) % 32; }

template <int R>
struct Geo {
    static constexpr int d = kHeadDim;
    static constexpr int b = kBlock;
    static constexpr int k = (d - R) < b ? (d - R) : b;   // Q columns
    static constexpr int m = R + b;                         // core rows
    static constexpr int n = R + k;                         // core columns
    static constexpr int c = R + b;                         // columns of [B | X^T]
    static constexpr int ldm = stride8(c);
    static constexpr int ldk = stride8(n);
    static constexpr int NR = n <= 96 ? 3 : 4;              // Jacobi rows per lane
    static constexpr int npad = 32 * NR;
    static constexpr int nwj = n / 16;                      // Jacobi warps (two 8-column blocks each)
    static constexpr int nb = n / 8;                        // Jacobi blocks
    static constexpr int ldw = R + 4;                       // W_r / B' staging stride (16-byte rows)
    static constexpr int ldp = R + 4;                       // P stride
    // region A: [B | X^T], then the core, the Jacobi exchange buffer, two
    // d x R staging slots
    static constexpr int regA0 = d * ldm > n * ldk ? d * ldm : n * ldk;   // >= n * d (reflectors)
    static constexpr int regA1 = n * npad > 2 * d * ldw ? n * npad : 2 * d * ldw;
    static constexpr int regA = regA0 > regA1 ? regA0 : regA1;
    // aux: P and R_E, later the r x r Gram matrices of the Bjorck steps
    static constexpr int aux0 = b * ldp + k * b;
    static constexpr int aux = aux0 > R * ldw ? aux0 : R * ldw;
    // small arrays (floats): tau/vd/al of both QRs, 2 norms, sigma^2, rank,
    // per-warp norms and rotation parameters, exchanged norms, flags
    static constexpr int small = 6 * 128 + 4 + 128 + 128 + kWarps * 16 + kWarps * 16 + 128 + 16 + 128 + 384;
    static constexpr int floats = regA + aux + small;
    static_assert(n % 16 == 0 && n <= 128 && npad >= n, "core shape");
    static_assert(R % 16 == 0 && R >= 16 && R <= 128, "rank");
};

// Off-diagonal threshold of the one-sided Jacobi: a pair (p, q) is rotated
// while |a_p . a_q| > tol * |a_p| |a_q|.
__device__ __forceinline__ float jacobi_tol(int len) { return 4.0e-7f * sqrtf((float)len); }

// ---------------------------------------------------------------------------
// Register-resident Householder QR.  Thread (warp w, lane l) owns the matrix
// columns cs + 64 t (cs = 8 w + (l & 7), t < CPT) over the rows
// p RPP .. p RPP + RPP - 1 (p = l >> 3): the four row parts of a column share
// a warp, so every column dot product is a register FMA chain plus two
// shuffles.  Reflector j, H_j = I - tau_j v v^T, is published once as a full
// column v (zeros above row j, vd_j at row j, the subdiagonal entries below)
// in V + slot * ldv, slot = j (keep) or j & 1 (a two-slot ring); al_j = R[j][j].
// Afterwards each thread's registers hold, per owned column c, R above row c,
// the column's value at row c from before its own reflection, and the
// reflector entries below.  Columns at or beyond `cols` must be zero.
// ---------------------------------------------------------------------------
template <int RPP, int CPT, int T1>
__device__ __forceinline__ void make_reflector(float (&x)[CPT][RPP], int jj, float* V, int ldv,
                                               bool keep, float* tau, float* vd, float* al) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, p = lane >> 3;
    const int cs1 = jj & 63;
    if (warp != (cs1 >> 3)) return;   // warp-uniform: the owner warp
    const bool own = (lane & 7) == (cs1 & 7);
    float sp[4] = {0.f, 0.f, 0.f, 0.f}, dg = 0.f;
#pragma unroll
    for (int e = 0; e < RPP; ++e) {
        const float v = x[T1][e];
        const int row = p * RPP + e;
        if (row > jj) sp[e & 3] = fmaf(v, v, sp[e & 3]);
        if (row == jj) dg = v;
    }
    float s = (sp[0] + sp[1]) + (sp[2] + sp[3]);
    if (!own) {
        s = 0.f;
        dg = 0.f;
    }
    s += __shfl_xor_sync(kFull, s, 8);
    s += __shfl_xor_sync(kFull, s, 16);
    dg += __shfl_xor_sync(kFull, dg, 8);
    dg += __shfl_xor_sync(kFull, dg, 16);
    float tj = 0.f, vj = 1.f, aj = dg;
    if (s > 0.f) {
        const float nr = sqrtf(fmaf(dg, dg, s));
        aj = -copysignf(nr, dg);
        vj = dg - aj;
        tj = 2.f / fmaf(vj, vj, s);
    }
    if (own) {
        float* v = V + (keep ? jj : (jj & 1)) * ldv + p * RPP;
#pragma unroll
        for (int e = 0; e < RPP; e += 4) {
            float4 o;
            const int row = p * RPP + e;
            o.x = row < jj ? 0.f : (row == jj ? vj : x[T1][e]);
            o.y = row + 1 < jj ? 0.f : (row + 1 == jj ? vj : x[T1][e + 1]);
            o.z = row + 2 < jj ? 0.f : (row + 2 == jj ? vj : x[T1][e + 2]);
            o.w = row + 3 < jj ? 0.f : (row + 3 == jj ? vj : x[T1][e + 3]);
            *reinterpret_cast<float4*>(v + e) = o;
        }
        if (p == 0) {
            tau[jj] = tj;
            vd[jj] = vj;
            al[jj] = aj;
        }
    }
}

template <int RPP>
__device__ __forceinline__ float dot_split(const float (&a)[RPP], const float (&b)[RPP]) {
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
    for (int e = 0; e < RPP; e += 4) {
        s0 = fmaf(a[e], b[e], s0);
        s1 = fmaf(a[e + 1], b[e + 1], s1);
        s2 = fmaf(a[e + 2], b[e + 2], s2);
        s3 = fmaf(a[e + 3], b[e + 3], s3);
    }
    return (s0 + s1) + (s2 + s3);
}

// Apply the current reflector (vr, tau tj, index j) to column slot t of the thread.
template <int RPP, int CPT>
__device__ __forceinline__ void reflect_slot(float (&x)[CPT][RPP], const float (&vr)[RPP], int t,
                                             int col, int j, int cols, float tj) {
    float w = dot_split<RPP>(vr, x[t]);
    w += __shfl_xor_sync(kFull, w, 8);
    w += __shfl_xor_sync(kFull, w, 16);
    if (col > j && col < cols) {
        const float tw = tj * w;
#pragma unroll
        for (int e = 0; e < RPP; ++e) x[t][e] = fmaf(-tw, vr[e], x[t][e]);
    }
}

// One reflection step j (column j+1 lives in slot TN of its owner threads).
template <int RPP, int CPT, int TN>
__device__ __forceinline__ void qr_step(float (&x)[CPT][RPP], int j, int cols, int nrefl, float* V,
                                        int ldv, bool keep, float* tau, float* vd, float* al) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, p = lane >> 3;
    const int cs = warp * 8 + (lane & 7);
    __syncthreads();
    const float* v = V + (keep ? j : (j & 1)) * ldv + p * RPP;
    const float tj = tau[j];
    auto load_v = [&](float (&vr)[RPP]) {
#pragma unroll
        for (int e = 0; e < RPP; e += 4) {
            const float4 q = *reinterpret_cast<const float4*>(v + e);
            vr[e] = q.x;
            vr[e + 1] = q.y;
            vr[e + 2] = q.z;
            vr[e + 3] = q.w;
        }
    };
    // look-ahead: the warp owning column j+1 brings that column up to date and
    // publishes the next reflector before its other columns (the reflector is
    // reloaded afterwards rather than held across)
    const int jn = j + 1;
    const bool ahead = jn < nrefl && warp == ((jn & 63) >> 3);
    if (ahead) {
        float vr[RPP];
        load_v(vr);
        reflect_slot<RPP, CPT>(x, vr, TN, cs + 64 * TN, j, cols, tj);
        make_reflector<RPP, CPT, TN>(x, jn, V, ldv, keep, tau, vd, al);
    }
    float vr[RPP];
    load_v(vr);
    // slots whose columns (8 per warp) are all finished (<= j) or absent are skipped
    const int cw = warp * 8;
#pragma unroll
    for (int t = 0; t < CPT; ++t)
        if ((t != TN || !ahead) && cw + 7 + 64 * t > j && cw + 64 * t < cols)
            reflect_slot<RPP, CPT>(x, vr, t, cs + 64 * t, j, cols, tj);
}

template <int RPP, int CPT>
__device__ void house_qr_reg(float (&x)[CPT][RPP], int cols, int nrefl, float* V, int ldv, bool keep,
                             float* tau, float* vd, float* al) {
    make_reflector<RPP, CPT, 0>(x, 0, V, ldv, keep, tau, vd, al);
    // step j publishes reflector j+1, whose column sits in slot (j+1) / 64;
    // steps whose j+1 lies beyond the last slot publish nothing (j+1 >= nrefl)
    int j = 0;
    for (; j < nrefl && j < 63; ++j) qr_step<RPP, CPT, 0>(x, j, cols, nrefl, V, ldv, keep, tau, vd, al);
    if constexpr (CPT > 1)
        for (; j < nrefl && j < 127; ++j) qr_step<RPP, CPT, 1>(x, j, cols, nrefl, V, ldv, keep, tau, vd, al);
    if constexpr (CPT > 2)
        for (; j < nrefl && j < 191; ++j) qr_step<RPP, CPT, 2>(x, j, cols, nrefl, V, ldv, keep, tau, vd, al);
    for (; j < nrefl; ++j) qr_step<RPP, CPT, CPT - 1>(x, j, cols, nrefl, V, ldv, keep, tau, vd, al);
    __syncthreads();
}

// Q = H_0 ... H_{n-1} [e_r .. e_{r+k-1}] from the kept reflectors (V, one
// 128-row column per reflector): thread (warp w, lane l) accumulates column
// q = 8 w + (l & 7) < k over rows 32 p .. 32 p + 31 backwards, starting with
// H_{r+q} e_{r+q}; no barrier is needed.  Writes Q (d x k, row-major) to gQ.
__device__ void form_q_reg(const float* V, int r, int k, int n, const float* tau, const float* vd,
                           float* gQ) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, p = lane >> 3;
    const int q = warp * 8 + (lane & 7);
    const bool has = q < k;
    float y[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) y[e] = 0.f;
    for (int j = n - 1; j >= 0; --j) {
        const float* v = V + j * kHeadDim + p * 32;
        float vr[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
            const float4 t4 = *reinterpret_cast<const float4*>(v + e);
            vr[e] = t4.x;
            vr[e + 1] = t4.y;
            vr[e + 2] = t4.z;
            vr[e + 3] = t4.w;
        }
        const float tj = tau[j];
        if (has && j == r + q) {
            const float f0 = -tj * vd[j];
#pragma unroll
            for (int e = 0; e < 32; ++e) y[e] = fmaf(f0, vr[e], (p * 32 + e == j) ? 1.f : 0.f);
        }
        float w = dot_split<32>(vr, y);
        w += __shfl_xor_sync(kFull, w, 8);
        w += __shfl_xor_sync(kFull, w, 16);
        if (has && j < r + q) {
            const float tw = tj * w;
#pragma unroll
            for (int e = 0; e < 32; ++e) y[e] = fmaf(-tw, vr[e], y[e]);
        }
    }
    if (has) {
#pragma unroll
        for (int e = 0; e < 32; ++e) gQ[(p * 32 + e) * k + q] = y[e];
    }
}

// ---------------------------------------------------------------------------
// Register-resident block Jacobi.  Warp g holds blocks "top" (a[0..7]) and
// "bot" (a[8..15]); lane l holds rows l + 32u of each column.
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int circ8(int s, int pos) { return pos == 0 ? 0 : 1 + (pos - 1 + s) % 7; }
// pair i (0..7) of round s: inside the blocks (pairs 0..3 in top, 4..7 in bot)
// or across them
__host__ __device__ constexpr int pair_p(bool within, int s, int i) {
    return within ? (i < 4 ? circ8(s, i) : 8 + circ8(s, i - 4)) : i;
}
__host__ __device__ constexpr int pair_q(bool within, int s, int i) {
    return within ? (i < 4 ? circ8(s, 7 - i) : 8 + circ8(s, 7 - (i - 4))) : 8 + (i + s) % 8;
}

struct JacobiCtx {
    float* nrm;      // this warp's 16 column norms^2
    float2* par;     // this warp's 8 rotation parameters
    int* any;        // this warp's "rotated" flag
    float tol2, tiny;
    int lane;
};

template <int NR, bool WITHIN, int S>
__device__ __forceinline__ void jacobi_round(float (&a)[16][NR], const JacobiCtx& cx) {
    float g[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < NR; ++u) acc = fmaf(a[pair_p(WITHIN, S, i)][u], a[pair_q(WITHIN, S, i)][u], acc);
        g[i] = acc;
    }
    // transpose-reduce: afterwards lane l holds the full dot product of pair (l >> 2) & 7
    const int lane = cx.lane;
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b4 ? g[i] : g[i + 4];
        const float keep = b4 ? g[i + 4] : g[i];
        h[i] = keep + __shfl_xor_sync(kFull, send, 16);
    }
    float h2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b3 ? h[i] : h[i + 2];
        const float keep = b3 ? h[i + 2] : h[i];
        h2[i] = keep + __shfl_xor_sync(kFull, send, 8);
    }
    float gm;
    {
        const float send = b2 ? h2[0] : h2[1];
        const float keep = b2 ? h2[1] : h2[0];
        gm = keep + __shfl_xor_sync(kFull, send, 4);
    }
    gm += __shfl_xor_sync(kFull, gm, 2);
    gm += __shfl_xor_sync(kFull, gm, 1);

    const int ip = (lane >> 2) & 7;
    const int p = pair_p(WITHIN, S, ip), q = pair_q(WITHIN, S, ip);
    const float al = cx.nrm[p], be = cx.nrm[q];
    // rotate while |g| > tol sqrt(al be), i.e. g^2 > tol^2 al be
    const bool need = fminf(al, be) > cx.tiny && gm * gm > cx.tol2 * (al * be);
    if (!__any_sync(kFull, need)) return;   // warp-uniform: nothing to rotate this round
    float cs = 1.f, sn = 0.f, nal = al, nbe = be;
    if (need) {
        // zeta and t set the angle only; c and s are formed from t with
        // correctly rounded operations, so c^2 + s^2 = 1 to rounding
        const float zeta = __fdividef(be - al, 2.f * gm);
        const float t = __fdividef(copysignf(1.f, zeta), fabsf(zeta) + sqrtf(fmaf(zeta, zeta, 1.f)));
        cs = 1.f / sqrtf(fmaf(t, t, 1.f));
        sn = cs * t;
        nal = fmaf(-t, gm, al);
        nbe = fmaf(t, gm, be);
    }
    __syncwarp();
    if ((lane & 3) == 0) {
        cx.par[ip] = make_float2(cs, sn);
        if (need) {
            cx.nrm[p] = nal;
            cx.nrm[q] = nbe;
            *cx.any = 1;
        }
    }
    __syncwarp();
    const float4* pv = reinterpret_cast<const float4*>(cx.par);
    float c8[8], s8[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 v = pv[i];
        c8[2 * i] = v.x;
        s8[2 * i] = v.y;
        c8[2 * i + 1] = v.z;
        s8[2 * i + 1] = v.w;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (s8[i] != 0.f) {   // warp-uniform
#pragma unroll
            for (int u = 0; u < NR; ++u) {
                const float x = a[pair_p(WITHIN, S, i)][u], y = a[pair_q(WITHIN, S, i)][u];
                a[pair_p(WITHIN, S, i)][u] = fmaf(c8[i], x, -s8[i] * y);
                a[pair_q(WITHIN, S, i)][u] = fmaf(s8[i], x, c8[i] * y);
            }
        }
    }
}

template <int NR, bool WITHIN, int... Ss>
__device__ __forceinline__ void jacobi_rounds(float (&a)[16][NR], const JacobiCtx& cx,
                                              std::integer_sequence<int, Ss...>) {
    (jacobi_round<NR, WITHIN, Ss>(a, cx), ...);
}

// Squared norms of the warp's 16 columns; lane l (even) gets column (l >> 1) & 15.
template <int NR>
__device__ __forceinline__ float col_norms16(const float (&a)[16][NR], int lane) {
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float s = 0.f;
#pragma unroll
        for (int u = 0; u < NR; ++u) s = fmaf(a[i][u], a[i][u], s);
        x[i] = s;
    }
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float send = b4 ? x[i] : x[i + 8];
        y[i] = (b4 ? x[i + 8] : x[i]) + __shfl_xor_sync(kFull, send, 16);
    }
    float z[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b3 ? y[i] : y[i + 4];
        z[i] = (b3 ? y[i + 4] : y[i]) + __shfl_xor_sync(kFull, send, 8);
    }
    float w2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b2 ? z[i] : z[i + 2];
        w2[i] = (b2 ? z[i + 2] : z[i]) + __shfl_xor_sync(kFull, send, 4);
    }
    float v;
    {
        const float send = b1 ? w2[0] : w2[1];
        v = (b1 ? w2[1] : w2[0]) + __shfl_xor_sync(kFull, send, 2);
    }
    v += __shfl_xor_sync(kFull, v, 1);
    return v;
}

__device__ __forceinline__ void jbar(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Blocks move one position along the circle top_1 .. top_{G-1}, bot_{G-1} ..
// bot_0 (top_0 stays): every pair of blocks shares a warp once in nb-1 moves,
// after which every block is back at its start.
template <int NR>
__device__ __forceinline__ void block_move(float (&a)[16][NR], float* nrm, float* xbuf, float* xnrm,
                                           int g, int G, int lane, int npad) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int u = 0; u < NR; ++u) xbuf[(16 * g + i) * npad + lane + 32 * u] = a[i][u];
    if (lane < 16) xnrm[16 * g + lane] = nrm[lane];
    jbar(G * 32);
    const int st = g == 0 ? 0 : (g == 1 ? 1 : 2 * (g - 1));     // source position of the new top
    const int sb = g == G - 1 ? 2 * (G - 1) : 2 * (g + 1) + 1;  // and of the new bottom
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int u = 0; u < NR; ++u) {
            a[i][u] = xbuf[(8 * st + i) * npad + lane + 32 * u];
            a[8 + i][u] = xbuf[(8 * sb + i) * npad + lane + 32 * u];
        }
    const float nv = lane < 8 ? xnrm[8 * st + lane] : (lane < 16 ? xnrm[8 * sb + lane - 8] : 0.f);
    jbar(G * 32);
    if (lane < 16) nrm[lane] = nv;
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Small dense products on shared-memory operands.
// ---------------------------------------------------------------------------

// G = A^T A for the rows x R matrix A (stride ld); G: R x R, stride ld.
template <int R>
__device__ void gram(const float* A, int rows, int ld, float* G) {
    constexpr int chunks = R / 4;
    for (int e = threadIdx.x; e < R * chunks; e += kThreads) {
        const int a = e / chunks, c4 = (e % chunks) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < rows; ++i) {
            const float x = A[i * ld + a];
            const float4 y = *reinterpret_cast<const float4*>(A + i * ld + c4);
            acc.x = fmaf(x, y.x, acc.x);
            acc.y = fmaf(x, y.y, acc.y);
            acc.z = fmaf(x, y.z, acc.z);
            acc.w = fmaf(x, y.w, acc.w);
        }
        *reinterpret_cast<float4*>(G + a * ld + c4) = acc;
    }
}

// Row i of the Bjorck step: out[j] = 1.5 A[i][j] - 0.5 sum_a A[i][a] G[a][j],
// for the half j in [h R/2, (h+1) R/2).
template <int R>
__device__ __forceinline__ void bjorck_row(const float* A, const float* G, int ld, int i, int h,
                                           float (&out)[R / 2]) {
    constexpr int H = R / 2;
#pragma unroll
    for (int v = 0; v < H; ++v) out[v] = 0.f;
    for (int a = 0; a < R; ++a) {
        const float x = A[i * ld + a];
        const float4* gr = reinterpret_cast<const float4*>(G + a * ld + h * H);
#pragma unroll
        for (int v = 0; v < H / 4; ++v) {
            const float4 y = gr[v];
            out[4 * v] = fmaf(x, y.x, out[4 * v]);
            out[4 * v + 1] = fmaf(x, y.y, out[4 * v + 1]);
            out[4 * v + 2] = fmaf(x, y.z, out[4 * v + 2]);
            out[4 * v + 3] = fmaf(x, y.w, out[4 * v + 3]);
        }
    }
#pragma unroll
    for (int v = 0; v < H; ++v) out[v] = fmaf(-0.5f, out[v], 1.5f * A[i * ld + h * H + v]);
}

template <typename KvT>
__device__ __forceinline__ float ring_at(const void* ring, int blocked, int64_t slot, int i) {
    return to_f32(reinterpret_cast<const KvT*>(ring)[coef_index(blocked, kHeadDim, slot, i)]);
}

__device__ __forceinline__ float x_at(const FactorView& f, const void* ring, int64_t slot, int i) {
    return f.kv_bf16 ? ring_at<__nv_bfloat16>(ring, f.ring_blocked, slot, i)
                     : ring_at<float>(ring, f.ring_blocked, slot, i);
}

template <int R>
__global__ void __launch_bounds__(kThreads, (R <= 64 ? 2 : 1))
fold_kernel(FactorView f, FoldLaunch fl, int* status) {
    using Gm = Geo<R>;
    constexpr int d = Gm::d, b = Gm::b, k = Gm::k, m = Gm::m, n = Gm::n, c = Gm::c;
    constexpr int ldm = Gm::ldm, ldk = Gm::ldk, ldw = Gm::ldw, ldp = Gm::ldp;
    constexpr int NR = Gm::NR, npad = Gm::npad, G = Gm::nwj, nb = Gm::nb;
    const int bh = blockIdx.x;
    const int task = blockIdx.y;
    const int layer = fl.layer[task];
    const int64_t n_c = fl.n_c[task];
    const int slot = fl.slot[task];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    extern __shared__ __align__(16) float smem[];
    float* A = smem;                           // region A
    float* aux = A + Gm::regA;                 // P (b x ldp) and R_E (k x b); later Gram matrices
    float* Pb = aux;
    float* REb = aux + b * ldp;
    float* sm = aux + Gm::aux;
    float* tau1 = sm;
    float* vd1 = sm + 128;
    float* al1 = sm + 256;
    float* tau2 = sm + 384;
    float* vd2 = sm + 512;
    float* al2 = sm + 640;
    float* sig2 = sm + 772;                    // 128
    int* rnk = reinterpret_cast<int*>(sm + 900);   // 128
    float* wnrm = sm + 1028;                   // kWarps x 16
    float2* wpar = reinterpret_cast<float2*>(sm + 1028 + kWarps * 16);   // kWarps x 8
    float* xnrm = sm + 1028 + kWarps * 32;     // 128
    int* flags = reinterpret_cast<int*>(sm + 1156 + kWarps * 32);       // 16
    int* wany = flags;                         // kWarps
    int* ncomp = flags + 8;
    float* fro = reinterpret_cast<float*>(flags + 10);
    int* cflag = flags + 16;                   // 128: rank slot awaiting completion
    float* vring = reinterpret_cast<float*>(flags + 144);   // 2 x 192: reflectors of the core QR

    const int64_t hidx = (int64_t)layer * f.BH + bh;
    const float* gB = f.basis + hidx * d * R;
    const float* gS = f.sigma + hidx * R;
    const void* ring = reinterpret_cast<const uint8_t*>(f.ring) + hidx * f.cap * d * (f.kv_bf16 ? 2 : 4);
    const int64_t slot0 = n_c % f.cap;
    float* gQ = fl.qscratch + hidx * d * k;

    // ---- load [B | X^T]
    for (int e = tid; e < d * R; e += kThreads) {
        const int i = e / R, j = e - (e / R) * R;
        A[i * ldm + j] = gB[e];
    }
    for (int e = tid; e < b * d; e += kThreads) {
        const int t = e / d, i = e - (e / d) * d;
        A[i * ldm + R + t] = x_at(f, ring, slot0 + t, i);
    }
    if (tid < 16 + 128) flags[tid] = 0;
    __syncthreads();

    // ---- (a) P = X B: thread -> (row t, quarter of the columns)
    {
        constexpr int Q4 = R / 4;
        const int t = tid >> 2, h = tid & 3;
        float acc[Q4];
#pragma unroll
        for (int v = 0; v < Q4; ++v) acc[v] = 0.f;
        for (int i = 0; i < d; ++i) {
            const float x = A[i * ldm + R + t];
            const float4* br = reinterpret_cast<const float4*>(A + i * ldm + h * Q4);
#pragma unroll
            for (int v = 0; v < Q4 / 4; ++v) {
                const float4 y = br[v];
                acc[4 * v] = fmaf(x, y.x, acc[4 * v]);
                acc[4 * v + 1] = fmaf(x, y.y, acc[4 * v + 1]);
                acc[4 * v + 2] = fmaf(x, y.z, acc[4 * v + 2]);
                acc[4 * v + 3] = fmaf(x, y.w, acc[4 * v + 3]);
            }
        }
#pragma unroll
        for (int v = 0; v < Q4; ++v) Pb[t * ldp + h * Q4 + v] = acc[v];
    }
    __syncthreads();

    // ---- (b) Householder QR of [B | X^T] in registers; R_E; Q to global scratch
    const int cs = warp * 8 + (lane & 7), prt = lane >> 3;
    {
        constexpr int CPT1 = (c + 63) / 64;
        float x[CPT1][32];
#pragma unroll
        for (int t = 0; t < CPT1; ++t)
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int col = cs + 64 * t;
                x[t][e] = col < c ? A[(prt * 32 + e) * ldm + col] : 0.f;
            }
        __syncthreads();   // region A now holds the reflectors (n x d)
        house_qr_reg<32, CPT1>(x, c, n, A, d, true, tau1, vd1, al1);
#pragma unroll
        for (int t = 0; t < CPT1; ++t) {
            const int col = cs + 64 * t;
            if (col >= R && col < R + b) {
                const int tt = col - R;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = prt * 32 + e - R;
                    if (i >= 0 && i < k) REb[i * b + tt] = (i < tt) ? x[t][e] : ((i == tt) ? al1[col] : 0.f);
                }
            }
        }
    }
    if constexpr (k > 0) form_q_reg(A, R, k, n, tau1, vd1, gQ);
    __syncthreads();   // R_E complete; reflectors no longer read

    // ---- (c) QR of the core K = [[diag S, 0], [P, R_E^T]] in registers; R to region A
    {
        constexpr int RPP2 = ((m + 3) / 4 + 3) / 4 * 4;
        constexpr int CPT2 = (n + 63) / 64;
        float x[CPT2][RPP2];
#pragma unroll
        for (int t = 0; t < CPT2; ++t)
#pragma unroll
            for (int e = 0; e < RPP2; ++e) {
                const int col = cs + 64 * t, row = prt * RPP2 + e;
                float v = 0.f;
                if (col < n && row < m) {
                    if (row < R) {
                        v = (row == col) ? gS[row] : 0.f;
                    } else {
                        const int tt = row - R;
                        v = (col < R) ? Pb[tt * ldp + col] : REb[(col - R) * b + tt];
                    }
                }
                x[t][e] = v;
            }
        house_qr_reg<RPP2, CPT2>(x, n, n, vring, 4 * RPP2, false, tau2, vd2, al2);
#pragma unroll
        for (int t = 0; t < CPT2; ++t)
#pragma unroll
            for (int e = 0; e < RPP2; ++e) {
                const int col = cs + 64 * t, row = prt * RPP2 + e;
                if (col < n && row <= col) A[row * ldk + col] = (row == col) ? al2[col] : x[t][e];
            }
    }
    __syncthreads();

    // ---- one-sided Jacobi on the columns of R^T (warps 0..G-1)
    float a[16][NR];
    if (warp < G) {
        const int g = warp;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int cc = 16 * g + i;
#pragma unroll
            for (int u = 0; u < NR; ++u) {
                const int row = lane + 32 * u;
                a[i][u] = (row == cc) ? al2[cc] : ((row > cc && row < n) ? A[cc * ldk + row] : 0.f);
            }
        }
        float* nrm = wnrm + g * 16;
        JacobiCtx cx{nrm, wpar + g * 8, wany + g, jacobi_tol(n) * jacobi_tol(n), 0.f, lane};
        {
            const float v = col_norms16<NR>(a, lane);
            float s = ((lane & 1) == 0) ? v : 0.f;
            s = warp_sum(s);
            if (lane == 0) atomicAdd(fro, s);
        }
        jbar(G * 32);   // R fully read before the first block move; fro complete
        cx.tiny = fmaf(1e-14f, *fro, 1e-35f);
        bool converged = false;
        for (int sweep = 0; sweep < fl.max_sweeps; ++sweep) {
            {
                const float v = col_norms16<NR>(a, lane);
                if ((lane & 1) == 0) nrm[(lane >> 1) & 15] = v;
                if (lane == 0) *cx.any = 0;
                __syncwarp();
            }
            for (int br = 0; br < nb - 1; ++br) {
                if (br == 0) jacobi_rounds<NR, true>(a, cx, std::make_integer_sequence<int, 7>{});
                jacobi_rounds<NR, false>(a, cx, std::make_integer_sequence<int, 8>{});
                block_move<NR>(a, nrm, A, xnrm, g, G, lane, npad);
            }
            jbar(G * 32);
            int any = 0;
            for (int w = 0; w < G; ++w) any |= wany[w];
            jbar(G * 32);
            if (!any) {
                converged = true;
                break;
            }
        }
        if (!converged && g == 0 && lane == 0) atomicOr(status, kStatusNoConverge);
        const float v = col_norms16<NR>(a, lane);
        if ((lane & 1) == 0) sig2[16 * g + ((lane >> 1) & 15)] = v;
    }
    __syncthreads();
    // ---- descending order of sigma (ties: lower column first)
    const float tiny = fmaf(1e-14f, *fro, 1e-35f);
    if (tid < n) {
        const float v = sig2[tid];
        int rk = 0;
        for (int j = 0; j < n; ++j) {
            const float u = sig2[j];
            rk += (u > v) || (u == v && j < tid);
        }
        rnk[tid] = rk;
    }
    __syncthreads();
    // ---- W (n x R, slot 0 of region A): unit columns at their rank
    float* W = A;
    float* W2 = A + d * ldw;
    float* sigR = xnrm;   // sigma of rank slot j < R
    if (warp < G) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int cc = 16 * warp + i;
            const int rk = rnk[cc];
            if (rk < R) {
                const float s2 = sig2[cc];
                const bool ok = s2 > tiny;
                const float inv = ok ? 1.f / sqrtf(s2) : 0.f;
#pragma unroll
                for (int u = 0; u < NR; ++u) {
                    const int row = lane + 32 * u;
                    if (row < n) W[row * ldw + rk] = a[i][u] * inv;
                }
                if (lane == 0) {
                    sigR[rk] = sqrtf(s2);
                    if (!ok) {
                        cflag[rk] = 1;
                        atomicAdd(ncomp, 1);
                    }
                }
            }
        }
    }
    __syncthreads();
    // ---- completion of numerically zero directions (rank of K below R): one
    // warp, slot by slot: e_i with the largest residual against the accepted
    // columns, orthogonalized twice (classical Gram-Schmidt) and normalized
    if (*ncomp > 0 && warp == 0) {
        for (int sl = 0; sl < R; ++sl) {
            if (!cflag[sl]) continue;
            float best = -1.f;
            int bi = 0;
            for (int i = lane; i < n; i += 32) {
                float acc = 0.f;
                for (int j = 0; j < R; ++j)
                    if (!cflag[j]) acc = fmaf(W[i * ldw + j], W[i * ldw + j], acc);
                if (1.f - acc > best) {
                    best = 1.f - acc;
                    bi = i;
                }
            }
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_xor_sync(kFull, best, o);
                const int oi = __shfl_xor_sync(kFull, bi, o);
                if (ob > best || (ob == best && oi < bi)) {
                    best = ob;
                    bi = oi;
                }
            }
            float y[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) y[u] = (lane + 32 * u == bi) ? 1.f : 0.f;
            for (int pass = 0; pass < 2; ++pass) {
                for (int j = 0; j < R; ++j) {
                    if (cflag[j]) continue;
                    float dp = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int row = lane + 32 * u;
                        if (row < n) dp = fmaf(W[row * ldw + j], y[u], dp);
                    }
                    dp = warp_sum(dp);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int row = lane + 32 * u;
                        if (row < n) y[u] = fmaf(-dp, W[row * ldw + j], y[u]);
                    }
                }
            }
            float nn = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) nn = fmaf(y[u], y[u], nn);
            const float inv = 1.f / sqrtf(warp_sum(nn));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int row = lane + 32 * u;
                if (row < n) W[row * ldw + sl] = y[u] * inv;
            }
            __syncwarp();
            if (lane == 0) cflag[sl] = 0;   // accepted from now on
            __syncwarp();
        }
    }
    __syncthreads();

    // ---- Bjorck step on W: W2 = 1.5 W - 0.5 W (W^T W)
    float* Gm_ = aux;   // R x ldw (P and R_E are dead)
    gram<R>(W, n, ldw, Gm_);
    __syncthreads();
    if (tid < 2 * n) {
        float o[R / 2];
        bjorck_row<R>(W, Gm_, ldw, tid >> 1, tid & 1, o);
#pragma unroll
        for (int v = 0; v < R / 2; ++v) W2[(tid >> 1) * ldw + (tid & 1) * (R / 2) + v] = o[v];
    }
    __syncthreads();

    // ---- (d) outputs: S', W_top, B'' = [B, Q] W (slot 0), new rows X B''
    float* gSw = f.sigma + hidx * R;
    float* gW = f.pend + (hidx * f.D + slot) * (int64_t)R * R;
    for (int e = tid; e < R * R; e += kThreads) {
        const int i = e / R, j = e - (e / R) * R;
        gW[e] = W2[i * ldw + j];
    }
    if (tid == 0 && bh == 0) f.seg_rows[layer * f.D + slot] = (int)n_c;
    float* Bn = A;   // slot 0: B'' (d x R)
    {
        constexpr int H = R / 2;
        const int i = tid >> 1, h = tid & 1;
        float acc[H];
#pragma unroll
        for (int v = 0; v < H; ++v) acc[v] = 0.f;
#pragma unroll 4
        for (int j = 0; j < n; ++j) {
            const float x = (j < R) ? gB[i * R + j] : gQ[i * k + (j - R)];
            const float4* wr = reinterpret_cast<const float4*>(W2 + j * ldw + h * H);
#pragma unroll
            for (int v = 0; v < H / 4; ++v) {
                const float4 y = wr[v];
                acc[4 * v] = fmaf(x, y.x, acc[4 * v]);
                acc[4 * v + 1] = fmaf(x, y.y, acc[4 * v + 1]);
                acc[4 * v + 2] = fmaf(x, y.z, acc[4 * v + 2]);
                acc[4 * v + 3] = fmaf(x, y.w, acc[4 * v + 3]);
            }
        }
        __syncthreads();   // every thread is done with W (slot 0 is overwritten next)
#pragma unroll
        for (int v = 0; v < H; ++v) Bn[i * ldw + h * H + v] = acc[v];
    }
    if (tid < R) gSw[tid] = sigR[tid];
    __syncthreads();
    {
        // new coefficient rows n_c .. n_c+63 = X B''
        constexpr int Q4 = R / 4;
        const int t = tid >> 2, h = tid & 3;
        float acc[Q4];
#pragma unroll
        for (int v = 0; v < Q4; ++v) acc[v] = 0.f;
        for (int i = 0; i < d; ++i) {
            const float x = x_at(f, ring, slot0 + t, i);
            const float4* br = reinterpret_cast<const float4*>(Bn + i * ldw + h * Q4);
#pragma unroll
            for (int v = 0; v < Q4 / 4; ++v) {
                const float4 y = br[v];
                acc[4 * v] = fmaf(x, y.x, acc[4 * v]);
                acc[4 * v + 1] = fmaf(x, y.y, acc[4 * v + 1]);
                acc[4 * v + 2] = fmaf(x, y.z, acc[4 * v + 2]);
                acc[4 * v + 3] = fmaf(x, y.w, acc[4 * v + 3]);
            }
        }
        const int64_t row = n_c + t;
        if (f.quant) {
            // coded storage: the fp32 rows wait in newrows for the coding kernel
            float* gN = f.newrows + hidx * kBlock * R;
#pragma unroll
            for (int v = 0; v < Q4; ++v) gN[t * R + h * Q4 + v] = acc[v];
        } else if (f.coef_bf16) {
            __nv_bfloat16* gC = reinterpret_cast<__nv_bfloat16*>(f.coef) + hidx * f.n_max * R;
#pragma unroll
            for (int v = 0; v < Q4; ++v)
                gC[coef_index(f.coef_blocked, R, row, h * Q4 + v)] = __float2bfloat16_rn(acc[v]);
        } else {
            float* gC = reinterpret_cast<float*>(f.coef) + hidx * f.n_max * R;
#pragma unroll
            for (int v = 0; v < Q4; ++v) gC[coef_index(f.coef_blocked, R, row, h * Q4 + v)] = acc[v];
        }
    }
    // ---- Bjorck step on B'' and the stores of B' (fp32, bf16 hi/lo blocked)
    gram<R>(Bn, d, ldw, Gm_);
    __syncthreads();
    {
        float o[R / 2];
        const int i = tid >> 1, h = tid & 1;
        bjorck_row<R>(Bn, Gm_, ldw, i, h, o);
        float* gBw = f.basis + hidx * d * R;
        __nv_bfloat16* gHi = f.bsplit + hidx * 2 * d * R;
        __nv_bfloat16* gLo = gHi + d * R;
        __syncthreads();   // gB (the old basis) was read by every thread above
#pragma unroll
        for (int v = 0; v < R / 2; ++v) {
            const int j = h * (R / 2) + v;
            const float x = o[v];
            gBw[i * R + j] = x;
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const int64_t bo = coef_index(1, R, i, j);
            gHi[bo] = hi;
            gLo[bo] = __float2bfloat16_rn(x - __bfloat162float(hi));
        }
    }
}

template <int R>
cudaError_t launch_fold_r(const FactorView& f, const FoldLaunch& fl, int* status, cudaStream_t s) {
    const size_t bytes = (size_t)Geo<R>::floats * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(fold_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid(f.BH, fl.n_tasks);
    fold_kernel<R><<<grid, kThreads, bytes, s>>>(f, fl, status);
    return cudaGetLastError();
}

}  // namespace

size_t fold_smem_bytes(int r) {
    switch (r) {
        case 16: return Geo<16>::floats * sizeof(float);
        case 32: return Geo<32>::floats * sizeof(float);
        case 48: return Geo<48>::floats * sizeof(float);
        case 64: return Geo<64>::floats * sizeof(float);
        case 80: return Geo<80>::floats * sizeof(float);
        case 96: return Geo<96>::floats * sizeof(float);
        case 112: return Geo<112>::floats * sizeof(float);
        case 128: return Geo<128>::floats * sizeof(float);
        default: return 0;
    }
}

int fold_q_cols(int r) { return (kHeadDim - r) < kBlock ? (kHeadDim - r) : kBlock; }

cudaError_t launch_fold(const FactorView& f, const FoldLaunch& fl, int* status, cudaStream_t s) {
    if (fl.n_tasks <= 0) return cudaSuccess;
    switch (f.r) {
        case 16: return launch_fold_r<16>(f, fl, status, s);
        case 32: return launch_fold_r<32>(f, fl, status, s);
        case 48: return launch_fold_r<48>(f, fl, status, s);
        case 64: return launch_fold_r<64>(f, fl, status, s);
        case 80: return launch_fold_r<80>(f, fl, status, s);
        case 96: return launch_fold_r<96>(f, fl, status, s);
        case 112: return launch_fold_r<112>(f, fl, status, s);
        case 128: return launch_fold_r<128>(f, fl, status, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace iskv
