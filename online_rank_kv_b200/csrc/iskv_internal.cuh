// Internal declarations of the iS-KV CUDA library (sm_100a).  Not part of the
// C ABI: only the .cu files of this library include it.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <vector>

#include "../../include/iskv.h"

namespace iskv {

constexpr int kHeadDim = 128;     // d
constexpr int kBlock = 64;        // rows folded at once (b)
constexpr int kMaxLayers = 128;   // layers per cache (bounds kernel params)
constexpr int kMaxDeferred = 64;  // postponed folds per layer
constexpr int kMaxGroup = 8;      // query heads per KV head in the decode

// Status bits of the sticky device word (bit 2, a bounded wait that gave up,
// is defined with the waits in tc_util.cuh).
constexpr int kStatusNoConverge = 1;
constexpr int kStatusRange = 4;   // a score of the tensor-core decode was not finite

// ---------------------------------------------------------------------------
// Element conversions (explicit round-to-nearest-even for bf16 stores).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Element offset of coefficient (row, c) inside one head's coefficient
// array.  Row-major, or (the cache's bf16 layout) 8-row x 8-column core
// matrices of 16 bytes per row, 8-row groups outermost: a tile of whole
// 8-row groups is contiguous and lands in shared memory, by one bulk copy,
// in the layout the tensor cores read without swizzling.
__host__ __device__ __forceinline__ int64_t coef_index(int blocked, int r, int64_t row, int c) {
    return blocked ? ((row >> 3) * (r >> 3) + (c >> 3)) * 64 + (row & 7) * 8 + (c & 7)
                   : row * r + c;
}

// ---------------------------------------------------------------------------
// Launch descriptors (passed by value; sized well under the 4 KB limit).
// ---------------------------------------------------------------------------

// One factor (K or V) of every layer: element pointers of layer 0 and the
// per-layer strides, so kernels address any (layer, sequence*head) pair.
struct FactorView {
    void* coef;          // [L][BH][n_max][r], coef dtype
    float* basis;        // [L][BH][d][r]
    __nv_bfloat16* bsplit;  // [L][BH][2][d x r blocked 8x8]: bf16 hi and lo parts of basis
    float* sigma;        // [L][BH][r]
    float* pend;         // [L][BH][D][r*r]: W_r[0:r,:] of postponed folds
    int* seg_rows;       // [L][D]: n_c before each postponed fold
    const void* ring;    // [L][BH][cap][d], kv dtype (exact window rows; factor
                         // position j = absolute position - P sits at slot j % cap)
    const void* prot;    // [L][BH][pcap][d], kv dtype (protected rows 0..P-1), or null
    int64_t P;           // protected leading positions
    int64_t pcap;        // protected rows per head (P rounded up to 64)
    int r;
    int coef_bf16;       // 1: coef stored as bf16
    int coef_blocked;    // 1: coef rows in 8x8 core-matrix blocks (see coef_index)
    int ring_blocked;    // 1: exact rows in the same blocked layout (128 columns)
    int kv_bf16;         // 1: ring stored as bf16
    int64_t n_max;       // coefficient rows per head
    int64_t cap;         // ring rows per head
    int D;               // postponed-fold slots per head
    int BH;              // batch * kv_heads
    // low-bit latent-channel codes (iskv_quant_format) instead of coef
    int quant;           // 1: coefficients live in qcodes / qscales
    uint32_t* qcodes;    // [L][BH][n_max][qwords]
    float* qscales;      // [L][BH][n_max][4]
    float* newrows;      // [L][BH][64][r] fp32: a fold's new rows before they are coded
    int qwords;          // code words per row
    int qgroups;         // groups in use (1..4)
    int qbits[4], qlo[4], qhi[4], qword0[4];   // bits, channel range and first word per group
    // joint-head factors: one factor (coefficients, singular values, postponed
    // W_top) per sequence over its `coef_div` KV heads, whose rows sit side by
    // side (D = coef_div * 128); basis rows, their bf16 parts and the exact
    // rows stay addressed per KV head (head h of a sequence holds basis rows
    // h * 128 .. h * 128 + 127).  0 or 1: one factor per head.
    int coef_div;
    float* wide;         // joint fold scratch: per factor [D x (r+64)] + [D x 64] + [D x r]
    int coef_ws;         // 1: coef holds one layer only (a decode workspace): instance = head
};

// Factor instance (coefficients, sigma, postponed W_top) of head instance hidx.
__host__ __device__ __forceinline__ int64_t coef_inst(const FactorView& f, int64_t hidx) {
    return f.coef_div > 1 ? hidx / f.coef_div : hidx;
}

// ---------------------------------------------------------------------------
// Latent-channel codes (iskv_quant_format): fp32 decisions throughout.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int quant_group_of(const FactorView& f, int c) {
    int g = 0;
#pragma unroll
    for (int i = 1; i < 4; ++i) g += (i < f.qgroups && c >= f.qlo[i]) ? 1 : 0;
    return g;
}

// The stored value of coefficient (row, c) of factor instance hidx.
__device__ __forceinline__ float quant_value(const FactorView& f, int64_t hidx, int64_t row, int c) {
    const int g = quant_group_of(f, c);
    const int b = f.qbits[g];
    if (b == 0) return 0.f;
    const int idx = c - f.qlo[g];
    const int64_t rbase = hidx * f.n_max + row;
    const uint32_t w = f.qcodes[rbase * f.qwords + f.qword0[g] + ((idx * b) >> 5)];
    const int qmax = (1 << (b - 1)) - 1;
    const int code = (int)((w >> ((idx * b) & 31)) & ((1u << b) - 1u)) - qmax;
    return (float)code * f.qscales[rbase * 4 + g];
}

// The stored values of coefficients (row, c0 .. c0 + 7) of one row, given
// that row's code words and group scales; c0 a multiple of 8.  Channel groups
// start at multiples of 16, so the 8 channels share one group and their codes
// are 8 b consecutive bits starting at a multiple of 8 b: two whole words for
// b = 8, one for b = 4, one half word for b = 2.  Same values as quant_value.
__device__ __forceinline__ void quant_decode8(const FactorView& f, const uint32_t* row_codes,
                                              const float* row_scales, int c0, float (&v)[8]) {
    const int g = quant_group_of(f, c0);
    const int b = f.qbits[g];
    if (b == 0) {
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = 0.f;
        return;
    }
    const int bit0 = (c0 - f.qlo[g]) * b;
    const uint32_t* wp = row_codes + f.qword0[g] + (bit0 >> 5);
    uint64_t bits = wp[0];
    if (b == 8) bits |= (uint64_t)wp[1] << 32;
    bits >>= (bit0 & 31);
    const uint32_t mask = (1u << b) - 1u;
    const int qmax = (1 << (b - 1)) - 1;
    const float sc = row_scales[g];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = (float)((int)((uint32_t)(bits >> (k * b)) & mask) - qmax) * sc;
}

// Code rows of r fp32 values: src[row * ld + c] for rows [0, nrows) of a
// block, written to codes[row * qwords + w] and scales[row * 4 + g]; sScale
// holds nrows * 4 floats of block scratch.  Called by every thread of the
// block (blockDim.x threads); ends with the codes written.
__device__ __forceinline__ void quant_rows_block(const FactorView& f, const float* src, int ld, int nrows,
                                                 uint32_t* codes, float* scales, float* sScale) {
    for (int e = threadIdx.x; e < nrows * 4; e += blockDim.x) {
        const int row = e >> 2, g = e & 3;
        float sc = 0.f;
        if (g < f.qgroups && f.qbits[g] > 0) {
            float amax = 0.f;
            for (int c = f.qlo[g]; c < f.qhi[g]; ++c) amax = fmaxf(amax, fabsf(src[row * ld + c]));
            sc = __fdiv_rn(amax, (float)((1 << (f.qbits[g] - 1)) - 1));
        }
        sScale[e] = sc;
        scales[(int64_t)row * 4 + g] = sc;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nrows * f.qwords; e += blockDim.x) {
        const int row = e / f.qwords, w = e % f.qwords;
        int g = 0;
#pragma unroll
        for (int i = 1; i < 4; ++i) g += (i < f.qgroups && w >= f.qword0[i]) ? 1 : 0;
        const int b = f.qbits[g];
        uint32_t word = 0u;
        if (b > 0) {
            const int qmax = (1 << (b - 1)) - 1;
            const float sc = sScale[row * 4 + g];
            const int per = 32 / b;
            const int c0 = f.qlo[g] + (w - f.qword0[g]) * per;
            for (int e2 = 0; e2 < per; ++e2) {
                int code = 0;
                if (sc > 0.f) {
                    code = __float2int_rn(__fdiv_rn(src[row * ld + c0 + e2], sc));
                    code = code > qmax ? qmax : (code < -qmax ? -qmax : code);
                }
                word |= (uint32_t)(code + qmax) << (e2 * b);
            }
        }
        codes[(int64_t)row * f.qwords + w] = word;
    }
}

struct FoldLaunch {
    int n_tasks;                 // layers folded by this launch
    int layer[kMaxLayers];
    int n_c[kMaxLayers];         // n_c before the fold
    int slot[kMaxLayers];        // postponed-fold slot receiving W_r[0:r,:]
    int max_sweeps;
    float* qscratch;             // [L][BH][d][k] fp32: Q of the fold in flight
};

struct ResyncLaunch {
    int n_tasks;
    int layer[kMaxLayers];
    int n_seg[kMaxLayers];       // postponed folds to apply (segments)
    int n_rows[kMaxLayers];      // rows to visit (n_c before the last fold)
};

struct DecodeArgs {
    FactorView K, V;
    const void* q;               // [B][Hq][d], kv dtype
    float* partial;              // [B][Hq][splits][2 + r_V + d]
    const float2* rope;          // [max_tokens][d/2] (cos, sin), or null
    int layer, B, Hkv, Hq, g;
    int64_t T, n_c;
    int splits;
    int64_t tokens_per_split;
    float scale;                 // 1/sqrt(d)
    // token range and partial slots of this launch (0 = [0, T), slots 0..splits-1)
    int64_t j_begin;             // first token of split 0
    int split_base;              // partial slot of split 0
    int splits_total;            // partial slots per query head (0: splits)
};

// Tensor-core decode over the folded rows (bf16 blocked coefficients).
constexpr int kDecodeMaxCtas = 160;   // persistent decode grid: at most one CTA per SM

struct DecodeTcArgs {
    FactorView K, V;
    const void* q;               // [B][Hq][d] bf16
    float* partial;              // [B][Hq][splits_total][2 + r_V + d]
    const float2* rope;          // [>= 128 positions][d/2], or null
    int* status;
    float* out;                  // [B][Hq][d] fp32: written by the last CTA of each head
    int* done;                   // [BH] arrival counters, zero between calls
    int layer, B, Hkv, Hq, g;
    int64_t n_c, T;
    int tiles_c;                 // folded-row tiles per head: ceil(n_c / 128)
    int tiles_w;                 // exact window tiles of 64: ceil((T - P - n_c) / 64)
    int tiles_per_head;          // tiles_c + tiles_w + protected tiles of 64: ceil(min(T, P) / 64)
    int64_t total_tiles;         // BH * tiles_per_head
    int ncta;
    // CTA i takes the flattened tiles [cta_start[i], cta_start[i + 1])
    int64_t cta_start[kDecodeMaxCtas + 1];
    int slots_c;                 // compressed partial slots per query head
    int splits_total;
    int stages;                  // shared-memory pipeline depth (2..6)
    int win_rows;                // rows of an exact-row tile: 64, or 32 when 64 would enlarge a stage
    int basis_bufs;              // bf16 basis buffers (1 or 2 heads in flight)
    int q_bufs;                  // q' buffers per epilogue group (1 or 2)
    float scale;
    long long pipe_wait;         // clock cycles a pipeline wait may take before the
                                 // call gives up (drain waits keep their own limit)
    uint32_t idle_hint_ns;       // suspend hint of the single-lane warps' waits
    const void* ptab;            // fp16 [ptab_rows + P rounded to 64][128], 8 x 8 blocked:
                                 // cos, sin of pos w_i interleaved; row j < ptab_rows is
                                 // factor row j (pos = P + j), row ptab_rows + p is pos p
    int64_t ptab_rows;
    uint32_t* aq;                // [BH][128 * 64] words: each head's query-basis products
};

// ---------------------------------------------------------------------------
// Host launchers (one per kernel file).
// ---------------------------------------------------------------------------
cudaError_t launch_init_factor(const FactorView& f, int layers, cudaStream_t s);
cudaError_t launch_append(void* ring, const void* src, int BH, int t, int src_t, int src_row0,
                          int64_t T0, int64_t cap, int elem_bytes, int blocked, cudaStream_t s);
// bytes from src to dst by a kernel (both 16-byte aligned, bytes a multiple
// of 16, else cudaErrorInvalidValue); either may be mapped page-locked host
// memory (the decode call's host queries)
cudaError_t launch_copy_vec(void* dst, const void* src, size_t bytes, cudaStream_t s);
cudaError_t launch_fold(const FactorView& f, const FoldLaunch& fl, int* status,
                        cudaStream_t s);
cudaError_t launch_fold_wide(const FactorView& f, const FoldLaunch& fl, int* status,
                             cudaStream_t s);
size_t fold_wide_scratch_floats(int D, int r);
cudaError_t launch_compose(const FactorView& f, const ResyncLaunch& rl, cudaStream_t s);
cudaError_t launch_resync(const FactorView& f, const ResyncLaunch& rl, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_combine(const DecodeArgs& a, float* out, cudaStream_t s);
cudaError_t launch_reconstruct(const FactorView& f, int layer, int64_t row0, int64_t rows,
                               float* out, cudaStream_t s);
cudaError_t launch_copy_coef(const FactorView& f, int layer, int64_t row0, int64_t rows, void* dst,
                             cudaStream_t s);
cudaError_t launch_resync_tc(const FactorView& f, const ResyncLaunch& rl, int* status,
                             cudaStream_t s);
cudaError_t launch_resync_quant(const FactorView& f, const ResyncLaunch& rl, cudaStream_t s);
cudaError_t launch_quant_new_rows(const FactorView& f, const FoldLaunch& fl, cudaStream_t s);
cudaError_t launch_quant_rows(const FactorView& f, const float* rows, int64_t n, uint32_t* codes,
                              float* scales, cudaStream_t s);
cudaError_t launch_expand_codes(const FactorView& f, int layer, int64_t rows, __nv_bfloat16* dst,
                                cudaStream_t s);
cudaError_t launch_decode_tc(const DecodeTcArgs& a, cudaStream_t s);
bool decode_tc_supports_group(int g);
cudaError_t launch_decode_u(const DecodeTcArgs& a, cudaStream_t s);
bool decode_u_supports(int g, int rK);
size_t decode_u_smem_bytes(int rK, int rV, int ns, int wt);
size_t decode_tc_smem_bytes(int rK, int rV, int ns, int nbk, int nqb, int wt);

size_t fold_smem_bytes(int r);
int fold_q_cols(int r);   // k = min(64, d - r): columns of Q

}  // namespace iskv
