// Basis synchronization, step (e) of the fold: every stored coefficient row is
// rewritten in the new basis, C <- C W_r[0:r, :] ("iS-KV -- Basis-synchronized
// online low-rank KV compression -- What does it mean?", the body paragraph on
// basis synchronization and drift: without it old coefficients would rebuild
// different vectors; the rewrite grows with the history).
//
// Rows are grouped in segments: segment s holds the rows that existed before
// postponed fold s but not before fold s-1, and is multiplied by the product
// of the W_top of folds s..m-1 (built in place by compose_kernel).  A per-fold
// rewrite is the one-segment case.  This file holds the CUDA-core path; the
// bf16 tensor-core path lives in k_resync_tc.cu.
#include "iskv_internal.cuh"

namespace iskv {

namespace {

constexpr int kComposeThreads = 256;

// pend[s] <- pend[s] * pend[s+1] for s = m-2 .. 0 (suffix products).
__global__ void __launch_bounds__(kComposeThreads)
compose_kernel(FactorView f, ResyncLaunch rl) {
    const int bh = blockIdx.x, task = blockIdx.y;
    const int layer = rl.layer[task];
    const int nseg = rl.n_seg[task];
    if (nseg < 2) return;
    const int r = f.r;
    extern __shared__ float sm[];
    float* sNext = sm;            // r x r
    float* sOut = sm + r * r;     // r x r
    const int64_t hidx = (int64_t)layer * f.BH + bh;
    float* base = f.pend + hidx * f.D * (int64_t)r * r;
    for (int e = threadIdx.x; e < r * r; e += kComposeThreads) sNext[e] = base[(int64_t)(nseg - 1) * r * r + e];
    __syncthreads();
    for (int s = nseg - 2; s >= 0; --s) {
        const float* W = base + (int64_t)s * r * r;
        for (int e = threadIdx.x; e < r * r; e += kComposeThreads) {
            const int i = e / r, cc = e % r;
            float acc = 0.f;
            for (int j = 0; j < r; ++j) acc = fmaf(W[i * r + j], sNext[j * r + cc], acc);
            sOut[e] = acc;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < r * r; e += kComposeThreads) {
            sNext[e] = sOut[e];
            base[(int64_t)s * r * r + e] = sOut[e];
        }
        __syncthreads();
    }
}

constexpr int kResyncRows = 64;
constexpr int kResyncThreads = 256;

template <typename CoefT>
__global__ void __launch_bounds__(kResyncThreads)
resync_kernel(FactorView f, ResyncLaunch rl) {
    const int task = blockIdx.z, bh = blockIdx.y;
    const int layer = rl.layer[task];
    const int64_t row0 = (int64_t)blockIdx.x * kResyncRows;
    if (row0 >= rl.n_rows[task]) return;
    const int nseg = rl.n_seg[task];
    const int* bounds = f.seg_rows + layer * f.D;
    int seg = 0;
    while (seg < nseg && row0 >= bounds[seg]) ++seg;
    if (seg >= nseg) return;
    const int r = f.r;
    extern __shared__ float sm[];
    float* sW = sm;                    // r x r
    float* sC = sm + r * r;            // rows x r
    const int64_t hidx = (int64_t)layer * f.BH + bh;
    const float* W = f.pend + (hidx * f.D + seg) * (int64_t)r * r;
    CoefT* C = reinterpret_cast<CoefT*>(f.coef) + hidx * f.n_max * r;
    const int bl = f.coef_blocked;
    for (int e = threadIdx.x; e < r * r; e += kResyncThreads) sW[e] = W[e];
    for (int e = threadIdx.x; e < kResyncRows * r; e += kResyncThreads)
        sC[e] = to_f32(C[coef_index(bl, r, row0 + e / r, e % r)]);
    __syncthreads();
    for (int e = threadIdx.x; e < kResyncRows * r; e += kResyncThreads) {
        const int t = e / r, cc = e % r;
        float acc = 0.f;
        for (int j = 0; j < r; ++j) acc = fmaf(sC[t * r + j], sW[j * r + cc], acc);
        C[coef_index(bl, r, row0 + t, cc)] = from_f32<CoefT>(acc);
    }
}

}  // namespace

cudaError_t launch_compose(const FactorView& f, const ResyncLaunch& rl, cudaStream_t s) {
    if (rl.n_tasks <= 0) return cudaSuccess;
    const size_t bytes = 2 * (size_t)f.r * f.r * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(compose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    compose_kernel<<<dim3(f.BH, rl.n_tasks), kComposeThreads, bytes, s>>>(f, rl);
    return cudaGetLastError();
}

cudaError_t launch_resync(const FactorView& f, const ResyncLaunch& rl, cudaStream_t s) {
    if (rl.n_tasks <= 0) return cudaSuccess;
    int max_rows = 0;
    for (int i = 0; i < rl.n_tasks; ++i) max_rows = rl.n_rows[i] > max_rows ? rl.n_rows[i] : max_rows;
    if (max_rows <= 0) return cudaSuccess;
    const size_t bytes = ((size_t)f.r * f.r + (size_t)kResyncRows * f.r) * sizeof(float);
    dim3 grid((max_rows + kResyncRows - 1) / kResyncRows, f.BH, rl.n_tasks);
    if (f.coef_bf16) {
        auto k = resync_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        k<<<grid, kResyncThreads, bytes, s>>>(f, rl);
    } else {
        auto k = resync_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        k<<<grid, kResyncThreads, bytes, s>>>(f, rl);
    }
    return cudaGetLastError();
}

}  // namespace iskv
