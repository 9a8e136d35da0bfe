// Small kernels of the cache: factor initialization, appending exact rows to
// the window ring, rebuilding folded rows (C B^T, before RoPE), and moving a
// call's operands to and from page-locked host memory.
#include "iskv_internal.cuh"

namespace iskv {

namespace {

// B = I_d[:, :r] (fp32 and its bf16 hi/lo parts), S = 0.
__global__ void init_factor_kernel(FactorView f, int layers) {
    const int64_t heads = (int64_t)layers * f.BH;
    const int r = f.r;
    const int64_t per = (int64_t)kHeadDim * r;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < heads * per;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t h = e / per, w = e % per;
        const int i = (int)(w / r), j = (int)(w % r);
        // joint-head factor: basis row i of head h is joint row (h mod heads) * 128 + i
        const int hrow = f.coef_div > 1 ? (int)(h % f.coef_div) * kHeadDim + i : i;
        const float v = (hrow == j) ? 1.f : 0.f;
        f.basis[e] = v;
        const int64_t bo = coef_index(1, r, i, j);
        f.bsplit[h * 2 * per + bo] = __float2bfloat16_rn(v);
        f.bsplit[h * 2 * per + per + bo] = __float2bfloat16_rn(0.f);
        if (w < r) f.sigma[h * r + w] = 0.f;
    }
}

// ring[bh][(T0 + t) mod cap][:] = src[bh][t][:], 16-byte vectors; with
// `blocked` (bf16 rows of 128) the destination is the 8x8 core-matrix layout:
// vector v of slot s lands at ((s / 8) * 16 + v) * 8 + s % 8.
// Rows src_row0 .. src_row0 + t - 1 of every head of src ([BH][src_t][d]) to
// slots (T0 + i) % cap of the per-head ring ([BH][cap][d], blocked or not).
__global__ void append_kernel(uint4* ring, const uint4* src, int BH, int t, int src_t, int src_row0,
                              int64_t T0, int64_t cap, int vec_per_row, int blocked) {
    const int64_t total = (int64_t)BH * t * vec_per_row;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t v = e % vec_per_row;
        const int64_t row = e / vec_per_row;
        const int64_t bh = row / t, tt = row % t;
        const int64_t slot = (T0 + tt) % cap;
        const int64_t dst = blocked ? bh * cap * vec_per_row + ((slot >> 3) * vec_per_row + v) * 8 + (slot & 7)
                                    : (bh * cap + slot) * vec_per_row + v;
        ring[dst] = src[(bh * src_t + src_row0 + tt) * vec_per_row + v];
    }
}

constexpr int kRecRows = 64;

// out[bh][row][i] = sum_j C[row0 + row][j] B[i][j] for rows of one chunk.
template <typename CoefT>
__global__ void __launch_bounds__(256) reconstruct_kernel(FactorView f, int layer, int64_t row0,
                                                          int64_t rows, float* out) {
    const int bh = blockIdx.y;
    const int64_t t0 = (int64_t)blockIdx.x * kRecRows;
    if (t0 >= rows) return;
    const int r = f.r;
    extern __shared__ float sm[];
    float* sB = sm;                       // d x (r+1), padded rows
    float* sC = sm + kHeadDim * (r + 1);  // kRecRows x r
    const int64_t hidx = (int64_t)layer * f.BH + bh;
    const float* B = f.basis + hidx * kHeadDim * r;
    const CoefT* C = reinterpret_cast<const CoefT*>(f.coef) + coef_inst(f, hidx) * f.n_max * r;
    const int nt = (int)((rows - t0) < kRecRows ? (rows - t0) : kRecRows);
    for (int e = threadIdx.x; e < kHeadDim * r; e += blockDim.x) sB[(e / r) * (r + 1) + e % r] = B[e];
    for (int e = threadIdx.x; e < kRecRows * r; e += blockDim.x) {
        const int t = e / r, c = e % r;
        const int64_t row = row0 + t0 + t;
        sC[e] = (t >= nt) ? 0.f
              : f.quant ? quant_value(f, hidx, row, c)
                        : to_f32(C[coef_index(f.coef_blocked, r, row, c)]);
    }
    __syncthreads();
    float* o = out + ((int64_t)bh * rows + t0) * kHeadDim;
    for (int e = threadIdx.x; e < nt * kHeadDim; e += blockDim.x) {
        const int t = e / kHeadDim, i = e % kHeadDim;
        float acc = 0.f;
        for (int j = 0; j < r; ++j) acc = fmaf(sC[t * r + j], sB[i * (r + 1) + j], acc);
        o[e] = acc;
    }
}

// dst[bh][row][c] (row-major, coefficient dtype) = C[row0 + row][c], any layout.
template <typename CoefT>
__global__ void copy_coef_kernel(FactorView f, int layer, int64_t row0, int64_t rows, CoefT* dst) {
    const int r = f.r;
    const int64_t total = (int64_t)f.BH * rows * r;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(e % r);
        const int64_t row = (e / r) % rows;
        const int64_t bh = e / ((int64_t)r * rows);
        const int64_t hidx = (int64_t)layer * f.BH + bh;
        if (f.quant) {
            dst[e] = from_f32<CoefT>(quant_value(f, hidx, row0 + row, c));
        } else {
            const CoefT* C = reinterpret_cast<const CoefT*>(f.coef) + hidx * f.n_max * r;
            dst[e] = C[coef_index(f.coef_blocked, r, row0 + row, c)];
        }
    }
}

// dst[i] = src[i] over n 16-byte vectors.  Either side may be page-locked
// host memory mapped into the device's address space: its loads or stores
// then cross PCIe in place, with no copy-engine hand-off between the kernels
// of a call on the same stream.
__global__ void copy_vec_kernel(uint4* dst, const uint4* src, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = src[i];
}

}  // namespace

cudaError_t launch_copy_vec(void* dst, const void* src, size_t bytes, cudaStream_t s) {
    if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | bytes) & 15) != 0)
        return cudaErrorInvalidValue;
    const int64_t n = (int64_t)(bytes / 16);
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 592) blocks = 592;
    copy_vec_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<uint4*>(dst),
                                                     reinterpret_cast<const uint4*>(src), n);
    return cudaGetLastError();
}

cudaError_t launch_copy_coef(const FactorView& f, int layer, int64_t row0, int64_t rows, void* dst,
                             cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    const int64_t total = (int64_t)f.BH * rows * f.r;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 4736) blocks = 4736;
    if (f.coef_bf16 && !f.quant)
        copy_coef_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            f, layer, row0, rows, reinterpret_cast<__nv_bfloat16*>(dst));
    else
        copy_coef_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(f, layer, row0, rows,
                                                                 reinterpret_cast<float*>(dst));
    return cudaGetLastError();
}

cudaError_t launch_init_factor(const FactorView& f, int layers, cudaStream_t s) {
    init_factor_kernel<<<1184, 256, 0, s>>>(f, layers);
    return cudaGetLastError();
}

cudaError_t launch_append(void* ring, const void* src, int BH, int t, int src_t, int src_row0,
                          int64_t T0, int64_t cap, int elem_bytes, int blocked, cudaStream_t s) {
    if (t <= 0) return cudaSuccess;
    const int vec_per_row = kHeadDim * elem_bytes / 16;
    const int64_t total = (int64_t)BH * t * vec_per_row;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 4736) blocks = 4736;
    if (blocks < 1) blocks = 1;
    append_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<uint4*>(ring),
                                                   reinterpret_cast<const uint4*>(src), BH, t, src_t,
                                                   src_row0, T0, cap, vec_per_row, blocked);
    return cudaGetLastError();
}

cudaError_t launch_reconstruct(const FactorView& f, int layer, int64_t row0, int64_t rows,
                               float* out, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    const size_t bytes = ((size_t)kHeadDim * (f.r + 1) + (size_t)kRecRows * f.r) * sizeof(float);
    dim3 grid((unsigned)((rows + kRecRows - 1) / kRecRows), f.BH);
    if (f.coef_bf16 && !f.quant) {
        auto k = reconstruct_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        k<<<grid, 256, bytes, s>>>(f, layer, row0, rows, out);
    } else {
        auto k = reconstruct_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        k<<<grid, 256, bytes, s>>>(f, layer, row0, rows, out);
    }
    return cudaGetLastError();
}

}  // namespace iskv
