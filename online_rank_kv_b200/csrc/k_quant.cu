// Low-bit coefficient codes in latent channels: coding a fold's new rows and
// the rewrite C <- C W of coded rows.
//
// Format and method: the SVDq page ("SVDq: 1.25-bit and 410x Key Cache
// Compression for LLM Attention", Abstract) stores a key cache in SVD latent
// channels with more bits for the more significant channels; here the latent
// channels are the columns of a factor's coefficients C (kept in descending
// singular-value order), coded per row and per channel group (see
// iskv_quant_format in include/iskv.h).  The iS-KV explainer (body paragraph
// on GQA and quantization) leaves the combination untried: the rewrite of
// step (e) here decodes each stored row, multiplies it by W_top (or the
// product of postponed ones) in fp32 and codes the result again, so coded
// rows stay in the current basis like bf16 rows do.
#include "iskv_internal.cuh"

namespace iskv {

namespace {

constexpr int kRows = 64;
constexpr int kThreads = 256;

// Rows n_c .. n_c + 63 of every listed layer's factors from the fold's fp32
// new rows.
__global__ void __launch_bounds__(kThreads) quant_new_rows_kernel(FactorView f, FoldLaunch fl) {
    const int bh = blockIdx.x, task = blockIdx.y;
    const int layer = fl.layer[task];
    const int64_t n_c = fl.n_c[task];
    const int64_t hidx = (int64_t)layer * f.BH + bh;
    __shared__ float sScale[kRows * 4];
    const float* src = f.newrows + hidx * kRows * f.r;
    quant_rows_block(f, src, f.r, kRows, f.qcodes + (hidx * f.n_max + n_c) * f.qwords,
                     f.qscales + (hidx * f.n_max + n_c) * 4, sScale);
}

// The rewrite of coded rows, one block of 64 rows per CTA: decode, multiply by
// the block's segment matrix (W_top of one fold, or the product of the
// postponed ones from compose_kernel), code again in place.
__global__ void __launch_bounds__(kThreads) resync_quant_kernel(FactorView f, ResyncLaunch rl) {
    const int task = blockIdx.z, bh = blockIdx.y;
    const int layer = rl.layer[task];
    const int64_t row0 = (int64_t)blockIdx.x * kRows;
    if (row0 >= rl.n_rows[task]) return;
    const int nseg = rl.n_seg[task];
    const int* bounds = f.seg_rows + layer * f.D;
    int seg = 0;
    while (seg < nseg && row0 >= bounds[seg]) ++seg;
    if (seg >= nseg) return;
    const int r = f.r;
    extern __shared__ float sm[];
    float* sW = sm;                    // r x r
    float* sC = sW + r * r;            // kRows x r, decoded rows
    float* sO = sC + kRows * r;        // kRows x r, rewritten rows
    float* sScale = sO + kRows * r;    // kRows x 4
    const int64_t hidx = (int64_t)layer * f.BH + bh;
    const float* W = f.pend + (hidx * f.D + seg) * (int64_t)r * r;
    for (int e = threadIdx.x; e < r * r; e += kThreads) sW[e] = W[e];
    for (int e = threadIdx.x; e < kRows * r; e += kThreads)
        sC[e] = quant_value(f, hidx, row0 + e / r, e % r);
    __syncthreads();
    for (int e = threadIdx.x; e < kRows * r; e += kThreads) {
        const int t = e / r, cc = e % r;
        float acc = 0.f;
        for (int j = 0; j < r; ++j) acc = fmaf(sC[t * r + j], sW[j * r + cc], acc);
        sO[e] = acc;
    }
    __syncthreads();
    quant_rows_block(f, sO, r, kRows, f.qcodes + (hidx * f.n_max + row0) * f.qwords,
                     f.qscales + (hidx * f.n_max + row0) * 4, sScale);
}

// Caller rows (iskv_quantize_rows): rows [n][r] fp32 -> codes, scales.
__global__ void __launch_bounds__(kThreads) quant_rows_kernel(FactorView f, const float* rows, int64_t n,
                                                               uint32_t* codes, float* scales) {
    const int64_t row0 = (int64_t)blockIdx.x * kRows;
    const int nr = (int)((n - row0) < kRows ? (n - row0) : kRows);
    __shared__ float sScale[kRows * 4];
    quant_rows_block(f, rows + row0 * f.r, f.r, nr, codes + row0 * f.qwords, scales + row0 * 4, sScale);
}

// The decode workspace of a coded layer: rows [0, rows) of every head as bf16
// values code * scale, in the 8 x 8 blocked layout the tensor-core decode
// bulk-copies.  One thread per (head, row, 8 columns): one 16-byte store.
__global__ void __launch_bounds__(kThreads) expand_codes_kernel(FactorView f, int layer, int64_t rows,
                                                                 __nv_bfloat16* dst) {
    const int r = f.r;
    const int cg = r / 8;
    const int64_t total = (int64_t)f.BH * rows * cg;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int c0 = (int)(e % cg) * 8;
        const int64_t row = (e / cg) % rows;
        const int64_t bh = e / ((int64_t)cg * rows);
        const int64_t hidx = (int64_t)layer * f.BH + bh;
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __nv_bfloat16 lo = __float2bfloat16_rn(quant_value(f, hidx, row, c0 + 2 * u));
            const __nv_bfloat16 hi = __float2bfloat16_rn(quant_value(f, hidx, row, c0 + 2 * u + 1));
            w[u] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
        }
        *reinterpret_cast<uint4*>(dst + bh * f.n_max * r + coef_index(1, r, row, c0)) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace

cudaError_t launch_expand_codes(const FactorView& f, int layer, int64_t rows, __nv_bfloat16* dst,
                                cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    const int64_t total = (int64_t)f.BH * rows * (f.r / 8);
    int64_t blocks = (total + kThreads - 1) / kThreads;
    if (blocks > 8 * 148) blocks = 8 * 148;
    expand_codes_kernel<<<(unsigned)blocks, kThreads, 0, s>>>(f, layer, rows, dst);
    return cudaGetLastError();
}

cudaError_t launch_quant_new_rows(const FactorView& f, const FoldLaunch& fl, cudaStream_t s) {
    if (fl.n_tasks <= 0) return cudaSuccess;
    quant_new_rows_kernel<<<dim3(f.BH, fl.n_tasks), kThreads, 0, s>>>(f, fl);
    return cudaGetLastError();
}

cudaError_t launch_resync_quant(const FactorView& f, const ResyncLaunch& rl, cudaStream_t s) {
    if (rl.n_tasks <= 0) return cudaSuccess;
    int max_rows = 0;
    for (int i = 0; i < rl.n_tasks; ++i) max_rows = rl.n_rows[i] > max_rows ? rl.n_rows[i] : max_rows;
    if (max_rows <= 0) return cudaSuccess;
    const size_t bytes = ((size_t)f.r * f.r + 2 * (size_t)kRows * f.r + kRows * 4) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(resync_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((max_rows + kRows - 1) / kRows, f.BH, rl.n_tasks);
    resync_quant_kernel<<<grid, kThreads, bytes, s>>>(f, rl);
    return cudaGetLastError();
}

cudaError_t launch_quant_rows(const FactorView& f, const float* rows, int64_t n, uint32_t* codes,
                              float* scales, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    quant_rows_kernel<<<(unsigned)((n + kRows - 1) / kRows), kThreads, 0, s>>>(f, rows, n, codes, scales);
    return cudaGetLastError();
}

}  // namespace iskv
