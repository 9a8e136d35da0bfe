// Block fold of a joint-head factor: one factor per sequence and layer whose
// rows are the KV heads' rows side by side (D = kv_heads * 128 columns).
//
// Method: the same Brand block-incremental SVD as the per-head fold ("iS-KV --
// Basis-synchronized online low-rank KV compression -- What does it mean?",
// Jargon: Block-incremental SVD), applied to the layer-wide rows; the
// explainer's worked-example ranks (64, 96, 128 with 128-dim heads) read most
// plainly as ranks of such a factor.  One CTA of 512 threads per factor:
//   (a) P = X B (64 x r), tiled through shared memory;
//   (b) Householder QR of [B | X^T] (D x (r + 64)), column by column in a
//       global scratch matrix (its first r reflections take out the
//       B-components, so the remaining ones factor the residual: rule Q);
//       Q = columns r .. r+k-1 of the orthogonal factor (k = min(64, D - r)),
//       formed by applying the reflectors backwards to unit vectors;
//       R_E = rows r .. r+k-1 of the triangular factor over the X^T columns;
//   (c) the core K = [[diag S, 0], [P, R_E^T]] ((r+64) x (r+k)) as K^T in
//       shared memory; one-sided (Hestenes) Jacobi on the r+64 columns of
//       K^T orthogonalizes them, K^T J = W Sigma, so the normalized columns
//       are K's right singular vectors and nothing is accumulated; pairs
//       follow the round-robin (circle) order, every pair once per sweep;
//       sigma sorted descending, W_r the matching unit columns, directions of
//       numerically zero singular values completed by unit vectors
//       orthogonalized twice (any completion is a correct truncation);
//   (d) B'' = [B, Q] W_r; new rows = X B''; S' = sigma_1..r; W_top =
//       W_r[0:r, :]; B' = B'' after one Bjorck step, written fp32 and as
//       bf16 hi/lo parts per KV head (the decode's operand layout).
// Step (e), the rewrite of the stored rows, is the per-factor resync kernel
// (coefficients and W_top are per sequence).
#include "iskv_internal.cuh"

namespace iskv {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCols = 192;   // r + 64 for r <= 128
constexpr unsigned kFull = 0xffffffffu;

struct WideGeo {
    int D, r, k, nA, n, m, ldn;
};

__host__ __device__ inline WideGeo wide_geo(int D, int r) {
    WideGeo g;
    g.D = D;
    g.r = r;
    g.k = (D - r) < kBlock ? (D - r) : kBlock;
    g.nA = r + kBlock;      // columns of [B | X^T]
    g.n = r + g.k;          // core columns
    g.m = r + kBlock;       // core rows = columns of K^T
    g.ldn = g.n + 1;
    return g;
}

// global scratch floats per factor: [B | X^T] (D x (r+64)), Q (D x 64), B'' (D x r)
__host__ __device__ inline size_t wide_scratch(int D, int r) {
    const WideGeo g = wide_geo(D, r);
    return (size_t)D * g.nA + (size_t)D * kBlock + (size_t)D * r;
}

// shared memory (floats): K^T (m x ldn), the P region, then small arrays
__host__ __device__ inline size_t wide_kt_floats(int D, int r) {
    const WideGeo g = wide_geo(D, r);
    size_t kt = (size_t)g.m * g.ldn;
    const size_t tile = (size_t)64 * 64 + (size_t)64 * r;   // (a) and new-row tiles alias K^T
    if (kt < tile) kt = tile;
    if (kt < (size_t)r * r) kt = (size_t)r * r;             // Bjorck Gram matrix
    return kt;
}
// the P region: P (64 x r), later 32-row tiles of [B | Q] (32 x n) and of B''
__host__ __device__ inline size_t wide_p_floats(int D, int r) {
    const WideGeo g = wide_geo(D, r);
    const size_t p = (size_t)64 * r, t = (size_t)32 * g.n;
    return p > t ? p : t;
}
__host__ __device__ inline size_t wide_smem_floats(int D, int r) {
    return wide_kt_floats(D, r) + wide_p_floats(D, r) + 6 * kMaxCols + 64;
}

__device__ __forceinline__ float block_sum(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += red[w];
    return t;
}

template <typename KvT>
__device__ __forceinline__ float ring_val(const void* ring, int blocked, int64_t slot, int i) {
    return to_f32(reinterpret_cast<const KvT*>(ring)[coef_index(blocked, kHeadDim, slot, i)]);
}

// Row t (0..63) of the block, joint column i (head i / 128, dim i % 128).
__device__ __forceinline__ float block_x(const FactorView& f, int64_t head0, int64_t slot, int i) {
    const int64_t hh = head0 + (i >> 7);
    const void* ring = reinterpret_cast<const char*>(f.ring) +
                       hh * f.cap * kHeadDim * (f.kv_bf16 ? 2 : 4);
    return f.kv_bf16 ? ring_val<__nv_bfloat16>(ring, f.ring_blocked, slot, i & 127)
                     : ring_val<float>(ring, f.ring_blocked, slot, i & 127);
}

__global__ void __launch_bounds__(kThreads, 1)
fold_wide_kernel(FactorView f, FoldLaunch fl, int* status) {
    const int seq = blockIdx.x, task = blockIdx.y;
    const int layer = fl.layer[task];
    const int64_t n_c = fl.n_c[task];
    const int slot = fl.slot[task];
    const int H = f.coef_div;
    const int D = H * kHeadDim;
    const int r = f.r;
    const WideGeo G = wide_geo(D, r);
    const int k = G.k, nA = G.nA, n = G.n, m = G.m, ldn = G.ldn;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t head0 = (int64_t)layer * f.BH + (int64_t)seq * H;   // first KV head instance
    const int64_t fidx = (int64_t)layer * (f.BH / H) + seq;            // factor instance
    const int64_t slot0 = n_c % f.cap;                                  // ring slot of row n_c

    extern __shared__ __align__(16) float smem[];
    float* KT = smem;                                  // K^T, column c at KT + c * ldn
    float* Pm = smem + wide_kt_floats(D, r);
    float* tau = Pm + wide_p_floats(D, r);
    float* vd = tau + kMaxCols;
    float* al = vd + kMaxCols;
    float* sig2 = al + kMaxCols;
    int* order = reinterpret_cast<int*>(sig2 + kMaxCols);
    float* red = sig2 + 2 * kMaxCols;                  // kWarps floats + flags
    int* flags = reinterpret_cast<int*>(red + 32);

    float* A = f.wide + fidx * wide_scratch(D, r);               // D x nA, column-major
    float* Y = A + (size_t)D * nA;                               // D x k, column-major (Q)
    float* Bn = Y + (size_t)D * kBlock;                          // D x r, row-major (B'')
    const float* Bold = f.basis + fidx * (int64_t)D * r;          // D x r, row-major

    // ---- load [B | X^T]
    for (int e = tid; e < D * r; e += kThreads) {
        const int i = e / r, j = e % r;
        A[(size_t)j * D + i] = Bold[e];
    }
    for (int e = tid; e < kBlock * D; e += kThreads) {
        const int t = e / D, i = e % D;
        A[(size_t)(r + t) * D + i] = block_x(f, head0, (slot0 + t) % f.cap, i);
    }
    __syncthreads();

    // ---- (a) P = X B, tiles of 64 joint columns through shared memory
    {
        float* Xs = KT;              // [64 i][64 t]
        float* Bs = KT + 64 * 64;    // [64 i][r]
        const int t = tid & 63, j0 = tid >> 6;   // outputs (t, j0 + 8 u)
        float acc[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) acc[u] = 0.f;
        for (int i0 = 0; i0 < D; i0 += 64) {
            for (int e = tid; e < 64 * 64; e += kThreads) {
                const int tt = e / 64, ii = e % 64;
                Xs[ii * 64 + tt] = A[(size_t)(r + tt) * D + i0 + ii];
            }
            for (int e = tid; e < 64 * r; e += kThreads) Bs[e] = Bold[(size_t)i0 * r + e];
            __syncthreads();
            for (int ii = 0; ii < 64; ++ii) {
                const float x = Xs[ii * 64 + t];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (j0 + 8 * u < r) acc[u] = fmaf(x, Bs[ii * r + j0 + 8 * u], acc[u]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int u = 0; u < 16; ++u)
            if (j0 + 8 * u < r) Pm[t * r + j0 + 8 * u] = acc[u];
    }

    // ---- (b) Householder QR of A, reflectors 0 .. r+k-1
    for (int j = 0; j < r + k; ++j) {
        float part = 0.f;
        for (int i = j + tid; i < D; i += kThreads) {
            const float x = A[(size_t)j * D + i];
            part = fmaf(x, x, part);
        }
        const float nrm2 = block_sum(part, red);
        if (tid == 0) {
            const float x0 = A[(size_t)j * D + j];
            float beta = 0.f, v0 = 0.f, t = 0.f;
            if (nrm2 > 0.f) {
                beta = -copysignf(__fsqrt_rn(nrm2), x0);
                v0 = x0 - beta;
                t = __frcp_rn(beta * (beta - x0));
            }
            tau[j] = t;
            vd[j] = v0;
            al[j] = beta;
            A[(size_t)j * D + j] = beta;   // R[j][j]; the reflector keeps v0 in vd[j]
        }
        __syncthreads();
        const float t = tau[j], v0 = vd[j];
        if (t != 0.f) {
            for (int c = j + 1 + warp; c < nA; c += kWarps) {
                float* col = A + (size_t)c * D;
                const float* v = A + (size_t)j * D;
                const float cj = col[j];   // read by every lane before lane 0 rewrites it
                float w = 0.f;
                for (int i = j + 1 + lane; i < D; i += 32) w = fmaf(v[i], col[i], w);
                w = warp_sum(w) + v0 * cj;
                const float tw = t * w;
                if (lane == 0) col[j] = cj - tw * v0;
                for (int i = j + 1 + lane; i < D; i += 32) col[i] = fmaf(-tw, v[i], col[i]);
            }
        }
        __syncthreads();
    }

    // ---- Q = H_0 ... H_{r+k-1} [e_r .. e_{r+k-1}], one warp per column
    for (int a = warp; a < k; a += kWarps) {
        float* y = Y + (size_t)a * D;
        for (int i = lane; i < D; i += 32) y[i] = (i == r + a) ? 1.f : 0.f;
        __syncwarp();
        for (int j = r + a; j >= 0; --j) {
            const float t = tau[j];
            if (t == 0.f) continue;
            const float* v = A + (size_t)j * D;
            const float yj = y[j];
            float w = 0.f;
            for (int i = j + 1 + lane; i < D; i += 32) w = fmaf(v[i], y[i], w);
            w = warp_sum(w) + vd[j] * yj;
            const float tw = t * w;
            if (lane == 0) y[j] = yj - tw * vd[j];
            for (int i = j + 1 + lane; i < D; i += 32) y[i] = fmaf(-tw, v[i], y[i]);
            __syncwarp();
        }
    }

    // ---- (c) K^T in shared memory: column c < r is S_c e_c; column r + t is
    // [P[t][0..r-1]; R_E[0..k-1][t]]
    const float* Sold = f.sigma + fidx * r;
    for (int e = tid; e < m * n; e += kThreads) {
        const int c = e / n, row = e % n;
        float v;
        if (c < r) {
            v = (row == c) ? Sold[c] : 0.f;
        } else {
            const int t = c - r;
            if (row < r) {
                v = Pm[t * r + row];
            } else {
                const int a = row - r;
                v = (a < t) ? A[(size_t)(r + t) * D + r + a] : (a == t ? al[r + a] : 0.f);
            }
        }
        KT[c * ldn + row] = v;
    }
    __syncthreads();
    float part = 0.f;
    for (int e = tid; e < m * n; e += kThreads) {
        const float v = KT[(e / n) * ldn + e % n];
        part = fmaf(v, v, part);
    }
    const float energy = block_sum(part, red);
    const float eps_e = 1e-14f * energy;
    const float tol = 4.0e-7f * sqrtf((float)n);

    // one-sided Jacobi on the m columns of K^T
    bool converged = false;
    for (int sweep = 0; sweep < fl.max_sweeps && !converged; ++sweep) {
        if (tid == 0) flags[0] = 0;
        __syncthreads();
        for (int rho = 0; rho < m - 1; ++rho) {
            for (int pi = warp; pi < m / 2; pi += kWarps) {
                const int p = pi == 0 ? m - 1 : (rho + pi) % (m - 1);
                const int q = pi == 0 ? rho : (rho - pi + m - 1) % (m - 1);
                float* ap = KT + p * ldn;
                float* aq = KT + q * ldn;
                float al2 = 0.f, be2 = 0.f, ga = 0.f;
                for (int i = lane; i < n; i += 32) {
                    const float x = ap[i], y = aq[i];
                    al2 = fmaf(x, x, al2);
                    be2 = fmaf(y, y, be2);
                    ga = fmaf(x, y, ga);
                }
                al2 = warp_sum(al2);
                be2 = warp_sum(be2);
                ga = warp_sum(ga);
                if (al2 > eps_e && be2 > eps_e && fabsf(ga) > tol * sqrtf(al2) * sqrtf(be2)) {
                    const float zeta = __fdiv_rn(be2 - al2, 2.f * ga);
                    const float tt = copysignf(1.f, zeta) / (fabsf(zeta) + __fsqrt_rn(fmaf(zeta, zeta, 1.f)));
                    const float cs = __frcp_rn(__fsqrt_rn(fmaf(tt, tt, 1.f)));
                    const float sn = cs * tt;
                    for (int i = lane; i < n; i += 32) {
                        const float x = ap[i], y = aq[i];
                        ap[i] = cs * x - sn * y;
                        aq[i] = sn * x + cs * y;
                    }
                    if (lane == 0) flags[0] = 1;
                }
            }
            __syncthreads();
        }
        converged = flags[0] == 0;
        __syncthreads();
    }
    if (!converged && tid == 0) atomicOr(status, kStatusNoConverge);

    // ---- sigma, order (descending), unit columns, completion
    for (int c = tid; c < m; c += kThreads) {
        float s2 = 0.f;
        for (int i = 0; i < n; ++i) s2 = fmaf(KT[c * ldn + i], KT[c * ldn + i], s2);
        sig2[c] = s2;
    }
    __syncthreads();
    for (int c = tid; c < m; c += kThreads) {
        const float s = sig2[c];
        int rk = 0;
        for (int c2 = 0; c2 < m; ++c2) rk += (sig2[c2] > s || (sig2[c2] == s && c2 < c)) ? 1 : 0;
        order[rk] = c;
    }
    __syncthreads();
    int nz = 0;
    for (int c = 0; c < m; ++c) nz += sig2[c] > eps_e ? 1 : 0;
    for (int e = tid; e < m * n; e += kThreads) {
        const int c = e / n, i = e % n;
        if (sig2[c] > eps_e) KT[c * ldn + i] /= __fsqrt_rn(sig2[c]);
    }
    __syncthreads();
    if (warp == 0) {
        for (int j = nz; j < r; ++j) {
            // the unit vector with the largest residual against W[:, 0..j-1]
            float best = -1.f;
            int bi = 0;
            for (int i = lane; i < n; i += 32) {
                float res = 1.f;
                for (int l = 0; l < j; ++l) {
                    const float w = KT[order[l] * ldn + i];
                    res -= w * w;
                }
                if (res > best) {
                    best = res;
                    bi = i;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_xor_sync(kFull, best, o);
                const int oi = __shfl_xor_sync(kFull, bi, o);
                if (ob > best || (ob == best && oi < bi)) {
                    best = ob;
                    bi = oi;
                }
            }
            float* y = KT + order[j] * ldn;
            for (int i = lane; i < n; i += 32) y[i] = (i == bi) ? 1.f : 0.f;
            __syncwarp();
            for (int pass = 0; pass < 2; ++pass) {
                for (int l = 0; l < j; ++l) {
                    const float* w = KT + order[l] * ldn;
                    float dt = 0.f;
                    for (int i = lane; i < n; i += 32) dt = fmaf(w[i], y[i], dt);
                    dt = warp_sum(dt);
                    for (int i = lane; i < n; i += 32) y[i] = fmaf(-dt, w[i], y[i]);
                    __syncwarp();
                }
            }
            float nn = 0.f;
            for (int i = lane; i < n; i += 32) nn = fmaf(y[i], y[i], nn);
            nn = warp_sum(nn);
            const float inv = __frcp_rn(__fsqrt_rn(nn));
            for (int i = lane; i < n; i += 32) y[i] *= inv;
            __syncwarp();
        }
    }
    __syncthreads();

    // ---- (d) S', W_top, B'' = [B, Q] W_r
    float* gS = f.sigma + fidx * r;
    for (int j = tid; j < r; j += kThreads) gS[j] = j < nz ? __fsqrt_rn(sig2[order[j]]) : 0.f;
    float* gW = f.pend + (fidx * f.D + slot) * (int64_t)r * r;
    for (int e = tid; e < r * r; e += kThreads) {
        const int c = e / r, j = e % r;
        gW[e] = KT[order[j] * ldn + c];
    }
    if (tid == 0 && seq == 0) f.seg_rows[layer * f.D + slot] = (int)n_c;
    {
        // 32-row tiles of [B | Q] through shared memory (the P region, free now)
        float* At = Pm;              // [32 rows][n]
        const int jj = tid % r, i_off = tid / r, i_step = kThreads / r;
        const float* w = KT + order[jj] * ldn;
        for (int i0 = 0; i0 < D; i0 += 32) {
            __syncthreads();
            for (int e = tid; e < 32 * n; e += kThreads) {
                const int ii = e / n, c = e % n;
                At[e] = c < r ? Bold[(size_t)(i0 + ii) * r + c] : Y[(size_t)(c - r) * D + i0 + ii];
            }
            __syncthreads();
            for (int ii = i_off; ii < 32; ii += i_step) {
                float acc = 0.f;
                for (int c = 0; c < n; ++c) acc = fmaf(At[ii * n + c], w[c], acc);
                Bn[(size_t)(i0 + ii) * r + jj] = acc;
            }
        }
    }
    __syncthreads();

    // new coefficient rows n_c .. n_c+63 = X B'' (tiles through shared memory)
    {
        float* Xs = KT;              // [64 i][64 t]
        float* Bs = KT + 64 * 64;    // [64 i][r]
        const int t = tid & 63, j0 = tid >> 6;
        float acc[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) acc[u] = 0.f;
        for (int i0 = 0; i0 < D; i0 += 64) {
            for (int e = tid; e < 64 * 64; e += kThreads) {
                const int tt = e / 64, ii = e % 64;
                Xs[ii * 64 + tt] = block_x(f, head0, (slot0 + tt) % f.cap, i0 + ii);
            }
            for (int e = tid; e < 64 * r; e += kThreads) Bs[e] = Bn[(size_t)i0 * r + e];
            __syncthreads();
            for (int ii = 0; ii < 64; ++ii) {
                const float x = Xs[ii * 64 + t];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (j0 + 8 * u < r) acc[u] = fmaf(x, Bs[ii * r + j0 + 8 * u], acc[u]);
            }
            __syncthreads();
        }
        const int64_t row = n_c + t;
        if (f.coef_bf16) {
            __nv_bfloat16* gC = reinterpret_cast<__nv_bfloat16*>(f.coef) + fidx * f.n_max * r;
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (j0 + 8 * u < r)
                    gC[coef_index(f.coef_blocked, r, row, j0 + 8 * u)] = __float2bfloat16_rn(acc[u]);
        } else {
            float* gC = reinterpret_cast<float*>(f.coef) + fidx * f.n_max * r;
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (j0 + 8 * u < r) gC[coef_index(f.coef_blocked, r, row, j0 + 8 * u)] = acc[u];
        }
    }

    // ---- one Bjorck step on B'' and the stores of B' (fp32; bf16 hi/lo per KV head)
    float* Gm = KT;   // r x r
    {
        // Gram matrix over 32-row tiles of B'' in shared memory (the P region)
        float* Bt = Pm;              // [32 rows][r]
        float gacc[32];
        const int ne = (r * r + kThreads - 1) / kThreads;   // entries per thread, <= 32
#pragma unroll
        for (int u = 0; u < 32; ++u) gacc[u] = 0.f;
        for (int i0 = 0; i0 < D; i0 += 32) {
            __syncthreads();
            for (int e = tid; e < 32 * r; e += kThreads) Bt[e] = Bn[(size_t)i0 * r + e];
            __syncthreads();
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int e = tid + u * kThreads;
                if (u >= ne || e >= r * r) break;
                const int a = e / r, b = e % r;
                float acc = gacc[u];
                for (int ii = 0; ii < 32; ++ii) acc = fmaf(Bt[ii * r + a], Bt[ii * r + b], acc);
                gacc[u] = acc;
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const int e = tid + u * kThreads;
            if (u >= ne || e >= r * r) break;
            Gm[e] = gacc[u];
        }
    }
    __syncthreads();
    float* gB = f.basis + fidx * (int64_t)D * r;
    for (int e = tid; e < D * r; e += kThreads) {
        const int i = e / r, j = e % r;
        float acc = 0.f;
        for (int c = 0; c < r; ++c) acc = fmaf(Bn[(size_t)i * r + c], Gm[c * r + j], acc);
        const float x = 1.5f * Bn[e] - 0.5f * acc;
        gB[e] = x;
        const int64_t hh = head0 + (i >> 7);
        __nv_bfloat16* gHi = f.bsplit + hh * 2 * kHeadDim * r;
        const int64_t bo = coef_index(1, r, i & 127, j);
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        gHi[bo] = hi;
        gHi[kHeadDim * r + bo] = __float2bfloat16_rn(x - __bfloat162float(hi));
    }
}

}  // namespace

size_t fold_wide_scratch_floats(int D, int r) { return wide_scratch(D, r); }

cudaError_t launch_fold_wide(const FactorView& f, const FoldLaunch& fl, int* status, cudaStream_t s) {
    if (fl.n_tasks <= 0) return cudaSuccess;
    const int H = f.coef_div > 0 ? f.coef_div : 1;
    const int D = H * kHeadDim;
    if (f.r % 8 != 0 || f.r > 128 || f.r + kBlock > kMaxCols || D < f.r) return cudaErrorInvalidValue;
    const size_t bytes = wide_smem_floats(D, f.r) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(fold_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    fold_wide_kernel<<<dim3(f.BH / H, fl.n_tasks), kThreads, bytes, s>>>(f, fl, status);
    return cudaGetLastError();
}

}  // namespace iskv
