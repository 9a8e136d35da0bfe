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
constexpr int kChunks = 4;   // 64-row chunks per rewrite block (W loaded once per segment)

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

// The rewrite of coded rows, four chunks of 64 rows per CTA: decode, multiply
// by the chunk's segment matrix (W_top of one fold, or the product of the
// postponed ones from compose_kernel; loaded once while the segment lasts),
// code again in place.  The product is
// register-tiled: each thread owns 4 rows x r/16 columns (columns tx, tx + 16,
// ...), so a k-step reads 4 + r/16 shared values for 4 r/16 FMAs; rows are
// padded to r + 1 floats so the 4-row reads of a warp's two row groups fall in
// different banks.
__global__ void __launch_bounds__(kThreads) resync_quant_kernel(FactorView f, ResyncLaunch rl) {
    const int task = blockIdx.z, bh = blockIdx.y;
    const int layer = rl.layer[task];
    const int64_t base = (int64_t)blockIdx.x * kRows * kChunks;
    if (base >= rl.n_rows[task]) return;
    const int nseg = rl.n_seg[task];
    const int* bounds = f.seg_rows + layer * f.D;
    const int r = f.r, ld = r + 1, cg = r >> 3;
    extern __shared__ float sm[];
    float* sW = sm;                    // r x r
    float* sC = sW + r * r;            // kRows x ld, decoded rows
    float* sO = sC + kRows * ld;       // kRows x ld, rewritten rows
    float* sScale = sO + kRows * ld;   // kRows x 4
    const int64_t hidx = (int64_t)layer * f.BH + bh;
    int loaded = -1;                   // segment whose matrix sits in sW
    for (int ch = 0; ch < kChunks; ++ch) {
        const int64_t row0 = base + ch * kRows;
        if (row0 >= rl.n_rows[task]) break;
        int seg = 0;
        while (seg < nseg && row0 >= bounds[seg]) ++seg;
        if (seg >= nseg) break;
        if (seg != loaded) {
            __syncthreads();           // the previous chunk's product has read sW
            const float* W = f.pend + (hidx * f.D + seg) * (int64_t)r * r;
            for (int e = threadIdx.x; e < r * r; e += kThreads) sW[e] = W[e];
            loaded = seg;
        }
        const uint32_t* codes = f.qcodes + (hidx * f.n_max + row0) * f.qwords;
        const float* scales = f.qscales + (hidx * f.n_max + row0) * 4;
        for (int e = threadIdx.x; e < kRows * cg; e += kThreads) {
            const int t = e / cg, c0 = (e - t * cg) * 8;
            float v[8];
            quant_decode8(f, codes + (int64_t)t * f.qwords, scales + t * 4, c0, v);
#pragma unroll
            for (int k = 0; k < 8; ++k) sC[t * ld + c0 + k] = v[k];
        }
        __syncthreads();
        {
            const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;   // rows 4 ty.., columns tx + 16 k
            const int nk = r >> 4;                                    // 1..8
            float acc[4][8];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[i][k] = 0.f;
            const float* cr = sC + (4 * ty) * ld;
            for (int j = 0; j < r; ++j) {
                float a[4], w[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = cr[i * ld + j];
#pragma unroll
                for (int k = 0; k < 8; ++k) w[k] = k < nk ? sW[j * r + tx + 16 * k] : 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        if (k < nk) acc[i][k] = fmaf(a[i], w[k], acc[i][k]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < nk) sO[(4 * ty + i) * ld + tx + 16 * k] = acc[i][k];
        }
        __syncthreads();
        // (its last reads of sO come before the next chunk's barrier after decoding)
        quant_rows_block(f, sO, ld, kRows, f.qcodes + (hidx * f.n_max + row0) * f.qwords,
                         f.qscales + (hidx * f.n_max + row0) * 4, sScale);
    }
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
// bulk-copies.  One thread per row: a warp reads 32 consecutive rows' code
// words and scales (contiguous runs), and writes each 8-column block of its
// rows as 16-byte words (8 rows of a block are one contiguous 128 bytes).
// Rows of the last 8-row group past `rows` are written as zeros.
__global__ void __launch_bounds__(kThreads) expand_codes_kernel(FactorView f, int layer, int rows,
                                                                 __nv_bfloat16* dst) {
    const int r = f.r, cg = r >> 3;
    const int bh = blockIdx.y;
    const int64_t hidx = (int64_t)layer * f.BH + bh;
    const uint32_t* codes = f.qcodes + hidx * f.n_max * f.qwords;
    const float* scales = f.qscales + hidx * f.n_max * 4;
    uint4* out = reinterpret_cast<uint4*>(dst + (int64_t)bh * f.n_max * r);
    const int total = (rows + 7) & ~7;
    for (int row = blockIdx.x * blockDim.x + threadIdx.x; row < total; row += gridDim.x * blockDim.x) {
        const uint32_t* rc = codes + (int64_t)row * f.qwords;
        const float* rs = scales + (int64_t)row * 4;
        for (int cb = 0; cb < cg; ++cb) {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            if (row < rows) {
                float v[8];
                quant_decode8(f, rc, rs, cb * 8, v);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const __nv_bfloat16 lo = __float2bfloat16_rn(v[2 * u]);
                    const __nv_bfloat16 hi = __float2bfloat16_rn(v[2 * u + 1]);
                    w[u] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
                }
            }
            out[((row >> 3) * cg + cb) * 8 + (row & 7)] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace

cudaError_t launch_expand_codes(const FactorView& f, int layer, int64_t rows, __nv_bfloat16* dst,
                                cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    if (rows > f.n_max || f.BH > 65535) return cudaErrorInvalidValue;
    const int64_t per_head = (rows + 7) / 8 * 8;   // one thread per row
    int64_t bx = (per_head + kThreads - 1) / kThreads;
    // about 8 resident CTAs per SM over all heads; each thread loops over the rest
    const int64_t want = (8 * 148 + f.BH - 1) / f.BH;
    if (bx > want) bx = want;
    expand_codes_kernel<<<dim3((unsigned)bx, (unsigned)f.BH), kThreads, 0, s>>>(f, layer, (int)rows, dst);
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
    const size_t bytes = ((size_t)f.r * f.r + 2 * (size_t)kRows * (f.r + 1) + kRows * 4) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(resync_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((max_rows + kRows * kChunks - 1) / (kRows * kChunks), f.BH, rl.n_tasks);
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
