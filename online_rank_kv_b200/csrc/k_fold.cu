// Block fold engine: one CTA per (layer, sequence*KV head) factor folds the
// oldest 64-row block that left the exact window into (B, S, C).
//
// Method: Brand's block-incremental SVD as the iS-KV explainer applies it
// ("iS-KV -- Basis-synchronized online low-rank KV compression -- What does it
// mean?", Jargon: Block-incremental SVD; body paragraph on the joint update of
// basis and coefficients on a small core whose size does not depend on the
// history length).  Steps inside the CTA, all in shared memory, fp32:
//   (a) P = X B                                   (warp dot products)
//   (b) Householder QR of [B | X^T] (d x (r+64)); its first r reflections
//       remove the B-components, i.e. they form the residual E = X - P B^T
//       implicitly.  Q = columns r..r+k-1 of the orthogonal factor
//       (k = min(64, d - r)), R_E = rows r..r+k-1 of the triangular factor
//       over the X^T columns; this keeps [B, Q] orthonormal even when
//       r + 64 > d or the residual is rank deficient.
//   (c) core A = [[diag S, 0], [P, R_E^T]] ((r+64) x (r+k)); one-sided
//       (Hestenes) Jacobi with accumulated right vectors V: each warp rotates
//       one column pair, n/2 disjoint pairs per round (circle ordering),
//       sweeps until no pair needs a rotation.  Singular values are the final
//       column norms, sorted descending.
//       fp32 rotations [[c, s], [-s, c]] keep the two columns exactly
//       orthogonal but scale them by c^2 + s^2 (a few ulp off 1); after the
//       sweeps every column of V is renormalized (and its column of A = K V
//       with it) so this scaling does not compound over hundreds of folds.
//   (d) S' = sigma_1..r, new coefficient rows = rows r.. of A V (first r
//       sorted columns), W_top = V[0:r, perm[0:r]] for step (e),
//       B' = [B, Q] V[:, perm[0:r]], followed by one Bjorck step
//       B' <- B' (3I - B'^T B') / 2 that restores orthonormality to fp32
//       rounding (a no-op in exact arithmetic), written as fp32 plus bf16
//       hi/lo parts.
#include "iskv_internal.cuh"

namespace iskv {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

struct Dims {
    int r, k, m, n, c, nrefl;
};

__host__ __device__ inline Dims dims_for(int r) {
    Dims x;
    x.r = r;
    x.k = (kHeadDim - r) < kBlock ? (kHeadDim - r) : kBlock;
    x.m = r + kBlock;      // core rows
    x.n = r + x.k;         // core columns
    x.c = r + kBlock;      // columns of [B | X^T]
    x.nrefl = r + x.k;     // reflections needed (<= d)
    return x;
}

struct Layout {
    size_t R1, R2, Q, small;
};

__host__ __device__ inline Layout layout_for(const Dims& x) {
    Layout L;
    size_t qr = (size_t)kHeadDim * x.c;
    size_t vv = (size_t)x.n * x.n;
    L.R1 = qr > vv ? qr : vv;               // [B|X^T] during QR, V afterwards
    L.R2 = (size_t)x.m * x.n;               // core A, then B' staging
    L.Q = (size_t)kHeadDim * x.k;
    L.small = 2 * (size_t)x.c + 2 * (size_t)x.n + 8;
    return L;
}

// Off-diagonal threshold of the one-sided Jacobi: a pair (p, q) is rotated
// while |a_p . a_q| > tol * |a_p| |a_q|.
__device__ __forceinline__ float jacobi_tol(int m) { return 4.0e-7f * sqrtf((float)m); }

template <typename KvT, typename CoefT>
__global__ void __launch_bounds__(kThreads, 1)
fold_kernel(FactorView f, FoldLaunch fl, int* status) {
    const int bh = blockIdx.x;
    const int task = blockIdx.y;
    const int layer = fl.layer[task];
    const int64_t n_c = fl.n_c[task];
    const int slot = fl.slot[task];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int d = kHeadDim;
    constexpr int b = kBlock;
    const Dims x = dims_for(f.r);
    const int r = x.r, k = x.k, m = x.m, n = x.n, c = x.c, nrefl = x.nrefl;
    const Layout L = layout_for(x);

    extern __shared__ float smem[];
    float* sM = smem;                 // d x c, column-major (stride d)
    float* sV = smem;                 // n x n, column-major (stride n), after QR
    float* sA = smem + L.R1;          // m x n, column-major (stride m)
    float* sQ = sA + L.R2;            // d x k, column-major (stride d)
    float* tau = sQ + L.Q;
    float* vdiag = tau + c;
    float* nrm = vdiag + c;
    int* perm = reinterpret_cast<int*>(nrm + n);
    int* flag = perm + n;

    const int64_t hidx = (int64_t)layer * f.BH + bh;
    const float* gB = f.basis + hidx * d * r;
    const float* gS = f.sigma + hidx * r;
    const KvT* ring = reinterpret_cast<const KvT*>(f.ring) + hidx * f.cap * d;
    const int64_t slot0 = n_c % f.cap;

    // ---- load B (columns 0..r-1) and X^T (columns r..r+63); zero the core
    for (int e = tid; e < d * r; e += kThreads) {
        int i = e % d, j = e / d;
        sM[j * d + i] = gB[(int64_t)i * r + j];
    }
    for (int e = tid; e < b * d; e += kThreads) {
        int t = e / d, i = e % d;
        sM[(r + t) * d + i] = to_f32(ring[coef_index(f.ring_blocked, d, slot0 + t, i)]);
    }
    for (int e = tid; e < m * n; e += kThreads) sA[e] = 0.f;
    __syncthreads();
    for (int j = tid; j < r; j += kThreads) sA[j * m + j] = gS[j];

    // ---- (a) P = X B into core rows r..r+63, columns 0..r-1
    for (int t = warp; t < b; t += kWarps) {
        float xv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) xv[u] = sM[(r + t) * d + lane + 32 * u];
        for (int j = 0; j < r; ++j) {
            float p = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) p = fmaf(xv[u], sM[j * d + lane + 32 * u], p);
            p = warp_sum(p);
            if (lane == 0) sA[j * m + r + t] = p;
        }
    }
    __syncthreads();

    // ---- (b) Householder QR of [B | X^T], reflections 0..nrefl-1
    for (int j = 0; j < nrefl; ++j) {
        if (warp == 0) {
            float below = 0.f;
            for (int i = j + 1 + lane; i < d; i += 32) {
                float v = sM[j * d + i];
                below = fmaf(v, v, below);
            }
            below = warp_sum(below);
            if (lane == 0) {
                float xj = sM[j * d + j];
                if (below == 0.f) {
                    tau[j] = 0.f;
                    vdiag[j] = 1.f;
                } else {
                    float nr = sqrtf(fmaf(xj, xj, below));
                    float alpha = -copysignf(nr, xj);
                    float vj = xj - alpha;
                    tau[j] = 2.f / fmaf(vj, vj, below);
                    vdiag[j] = vj;
                    sM[j * d + j] = alpha;
                }
            }
        }
        __syncthreads();
        const float tj = tau[j];
        if (tj != 0.f) {
            const float vj = vdiag[j];
            for (int col = j + 1 + warp; col < c; col += kWarps) {
                float w = 0.f;
                for (int i = j + lane; i < d; i += 32) {
                    float vi = (i == j) ? vj : sM[j * d + i];
                    w = fmaf(vi, sM[col * d + i], w);
                }
                w = warp_sum(w) * tj;
                for (int i = j + lane; i < d; i += 32) {
                    float vi = (i == j) ? vj : sM[j * d + i];
                    sM[col * d + i] = fmaf(-w, vi, sM[col * d + i]);
                }
            }
        }
        __syncthreads();
    }

    // ---- R_E^T into the core, Q = H_0 ... H_{r+k-1} e_{r..r+k-1}
    for (int e = tid; e < k * b; e += kThreads) {
        int i = e / b, t = e % b;
        sA[(r + i) * m + r + t] = (i <= t) ? sM[(r + t) * d + r + i] : 0.f;
    }
    for (int qi = warp; qi < k; qi += kWarps) {
        float y[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) y[u] = (lane + 32 * u == r + qi) ? 1.f : 0.f;
        for (int j = r + qi; j >= 0; --j) {
            const float tj = tau[j];
            if (tj == 0.f) continue;
            float w = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                int i = lane + 32 * u;
                float vi = (i < j) ? 0.f : ((i == j) ? vdiag[j] : sM[j * d + i]);
                w = fmaf(vi, y[u], w);
            }
            w = warp_sum(w) * tj;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                int i = lane + 32 * u;
                float vi = (i < j) ? 0.f : ((i == j) ? vdiag[j] : sM[j * d + i]);
                y[u] = fmaf(-w, vi, y[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) sQ[qi * d + lane + 32 * u] = y[u];
    }
    __syncthreads();

    // ---- (c) one-sided Jacobi on the core; V = I
    for (int e = tid; e < n * n; e += kThreads) sV[e] = (e / n == e % n) ? 1.f : 0.f;
    __syncthreads();

    const float tol = jacobi_tol(m);
    const int ru = (m + 31) / 32;   // rows of A per lane (<= 6)
    const int rv = (n + 31) / 32;   // rows of V per lane (<= 6)
    float* fro = reinterpret_cast<float*>(flag + 1);   // Frobenius norm^2 of the core
    bool converged = false;
    for (int sweep = 0; sweep < fl.max_sweeps; ++sweep) {
        for (int col = warp; col < n; col += kWarps) {
            float s = 0.f;
            for (int u = 0; u < ru; ++u) {
                int i = lane + 32 * u;
                float v = (i < m) ? sA[col * m + i] : 0.f;
                s = fmaf(v, v, s);
            }
            s = warp_sum(s);
            if (lane == 0) nrm[col] = s;
        }
        if (tid == 0) *flag = 0;
        __syncthreads();
        if (sweep == 0 && tid == 0) {
            float t = 0.f;
            for (int col = 0; col < n; ++col) t += nrm[col];
            *fro = t;
        }
        __syncthreads();
        // columns below this energy are numerically zero and never rotated
        const float tiny = fmaf(1e-14f, *fro, 1e-35f);
        for (int round = 0; round < n - 1; ++round) {
            for (int pi = warp; pi < n / 2; pi += kWarps) {
                const int p = (pi == 0) ? 0 : 1 + (pi - 1 + round) % (n - 1);
                const int qq = n - 1 - pi;
                const int q = 1 + (qq - 1 + round) % (n - 1);
                const float al = nrm[p], be = nrm[q];
                float gm = 0.f;
                for (int u = 0; u < ru; ++u) {
                    int i = lane + 32 * u;
                    if (i < m) gm = fmaf(sA[p * m + i], sA[q * m + i], gm);
                }
                gm = warp_sum(gm);
                if (fminf(al, be) > tiny && fabsf(gm) > tol * sqrtf(fmaxf(al * be, 0.f))) {
                    const float zeta = (be - al) / (2.f * gm);
                    const float t = copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(fmaf(zeta, zeta, 1.f)));
                    const float cs = 1.f / sqrtf(fmaf(t, t, 1.f));
                    const float sn = cs * t;
                    for (int u = 0; u < ru; ++u) {
                        int i = lane + 32 * u;
                        if (i < m) {
                            float ap = sA[p * m + i], aq = sA[q * m + i];
                            sA[p * m + i] = fmaf(cs, ap, -sn * aq);
                            sA[q * m + i] = fmaf(sn, ap, cs * aq);
                        }
                    }
                    for (int u = 0; u < rv; ++u) {
                        int i = lane + 32 * u;
                        if (i < n) {
                            float vp = sV[p * n + i], vq = sV[q * n + i];
                            sV[p * n + i] = fmaf(cs, vp, -sn * vq);
                            sV[q * n + i] = fmaf(sn, vp, cs * vq);
                        }
                    }
                    if (lane == 0) {
                        nrm[p] = fmaf(-t, gm, al);
                        nrm[q] = fmaf(t, gm, be);
                        *flag = 1;
                    }
                }
            }
            __syncthreads();
        }
        const int any = *flag;
        __syncthreads();
        if (!any) {
            converged = true;
            break;
        }
    }
    if (!converged && tid == 0) atomicOr(status, kStatusNoConverge);

    // ---- unit columns of V, with A = K V scaled alike
    for (int col = warp; col < n; col += kWarps) {
        float s = 0.f;
        for (int u = 0; u < rv; ++u) {
            int i = lane + 32 * u;
            float v = (i < n) ? sV[col * n + i] : 0.f;
            s = fmaf(v, v, s);
        }
        const float inv = 1.f / sqrtf(warp_sum(s));
        for (int u = 0; u < rv; ++u) {
            int i = lane + 32 * u;
            if (i < n) sV[col * n + i] *= inv;
        }
        for (int u = 0; u < ru; ++u) {
            int i = lane + 32 * u;
            if (i < m) sA[col * m + i] *= inv;
        }
    }
    __syncthreads();

    // ---- singular values (exact column norms) and descending order
    for (int col = warp; col < n; col += kWarps) {
        float s = 0.f;
        for (int u = 0; u < ru; ++u) {
            int i = lane + 32 * u;
            float v = (i < m) ? sA[col * m + i] : 0.f;
            s = fmaf(v, v, s);
        }
        s = warp_sum(s);
        if (lane == 0) nrm[col] = sqrtf(s);
    }
    __syncthreads();
    for (int col = tid; col < n; col += kThreads) {
        const float v = nrm[col];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
            const float u = nrm[j];
            rank += (u > v) || (u == v && j < col);
        }
        perm[rank] = col;
    }
    __syncthreads();

    // ---- (d) outputs: S', new coefficient rows, W_top
    float* gSw = f.sigma + hidx * r;
    for (int t = tid; t < r; t += kThreads) gSw[t] = nrm[perm[t]];
    CoefT* gC = reinterpret_cast<CoefT*>(f.coef) + hidx * f.n_max * r;
    for (int e = tid; e < b * r; e += kThreads) {
        int t = e / r, cc = e % r;
        gC[coef_index(f.coef_blocked, r, n_c + t, cc)] = from_f32<CoefT>(sA[perm[cc] * m + r + t]);
    }
    float* gW = f.pend + (hidx * f.D + slot) * (int64_t)r * r;
    for (int e = tid; e < r * r; e += kThreads) {
        int i = e / r, cc = e % r;
        gW[e] = sV[perm[cc] * n + i];
    }
    if (bh == 0 && tid == 0) f.seg_rows[layer * f.D + slot] = (int)n_c;
    __syncthreads();

    // ---- B' = [B, Q] V[:, perm[0:r]] staged in the core's space
    float* sBn = sA;
    for (int e = tid; e < d * r; e += kThreads) {
        const int i = e % d, cc = e / d;
        const float* vcol = sV + perm[cc] * n;
        float acc = 0.f;
        for (int j = 0; j < r; ++j) acc = fmaf(gB[(int64_t)i * r + j], vcol[j], acc);
        for (int j = 0; j < k; ++j) acc = fmaf(sQ[j * d + i], vcol[r + j], acc);
        sBn[i * r + cc] = acc;
    }
    __syncthreads();
    // Bjorck step: G = B'^T B' (r x r, in V's space, no longer needed)
    float* sG = sV;
    for (int e = tid; e < r * r; e += kThreads) {
        const int a = e / r, cc = e % r;
        float acc = 0.f;
        for (int i = 0; i < d; ++i) acc = fmaf(sBn[i * r + a], sBn[i * r + cc], acc);
        sG[e] = acc;
    }
    __syncthreads();
    float* gBw = f.basis + hidx * d * r;
    __nv_bfloat16* gHi = f.bsplit + hidx * 2 * d * r;
    __nv_bfloat16* gLo = gHi + d * r;
    for (int e = tid; e < d * r; e += kThreads) {
        const int i = e / r, cc = e % r;
        // v = sum_j B'[i][j] (1.5 delta_jc - 0.5 G[j][c])
        float corr = 0.f;
        for (int j = 0; j < r; ++j) corr = fmaf(sBn[i * r + j], sG[j * r + cc], corr);
        const float v = fmaf(-0.5f, corr, 1.5f * sBn[e]);
        gBw[e] = v;
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        const int64_t bo = coef_index(1, r, i, cc);
        gHi[bo] = h;
        gLo[bo] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
}

template <typename KvT, typename CoefT>
cudaError_t launch_fold_t(const FactorView& f, const FoldLaunch& fl, int* status,
                          cudaStream_t s) {
    const Dims x = dims_for(f.r);
    const Layout L = layout_for(x);
    const size_t bytes = (L.R1 + L.R2 + L.Q + L.small) * sizeof(float);
    auto kern = fold_kernel<KvT, CoefT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid(f.BH, fl.n_tasks);
    kern<<<grid, kThreads, bytes, s>>>(f, fl, status);
    return cudaGetLastError();
}

}  // namespace

size_t fold_smem_bytes(int r) {
    const Dims x = dims_for(r);
    const Layout L = layout_for(x);
    return (L.R1 + L.R2 + L.Q + L.small) * sizeof(float);
}

cudaError_t launch_fold(const FactorView& f, const FoldLaunch& fl, int* status,
                        cudaStream_t s) {
    if (fl.n_tasks <= 0) return cudaSuccess;
    if (f.kv_bf16) {
        return f.coef_bf16 ? launch_fold_t<__nv_bfloat16, __nv_bfloat16>(f, fl, status, s)
                           : launch_fold_t<__nv_bfloat16, float>(f, fl, status, s);
    }
    return f.coef_bf16 ? launch_fold_t<float, __nv_bfloat16>(f, fl, status, s)
                       : launch_fold_t<float, float>(f, fl, status, s);
}

}  // namespace iskv
