// Basis synchronization (step (e) of the fold) for bf16-stored coefficients
// on the 5th-generation tensor cores: every stored row is rewritten in the new
// basis, C <- C M, with M = W_r[0:r, :] of the fold (or, for postponed folds,
// the product of the W_r[0:r, :] that came after the row was written).
// Method source: "iS-KV -- Basis-synchronized online low-rank KV compression
// -- What does it mean?", body paragraph on basis synchronization and drift.
//
// HBM-streaming design (one CTA = one chunk of rows of one head, 128 threads):
//   * 128-row tiles of the blocked coefficient array are contiguous, so one
//     bulk copy (TMA engine, no tensor map) per tile lands them in shared
//     memory already in the no-swizzle UMMA K-major layout; two tile buffers
//     keep the next tile in flight while the current one is rewritten;
//   * M (fp32) is split into three bf16 parts M1 + M2 + M3 (24 significant
//     bits, i.e. fp32 accuracy); with C exact in bf16 the three kind::f16 MMAs
//     (M=128 rows, N=r, K=r) accumulate C M in fp32 in tensor memory;
//   * each thread owns one row: tcgen05.ld its r accumulators, round to bf16
//     (nearest-even) and store 16-byte chunks back in the blocked layout.
// Rows of a segment boundary that falls inside a tile are left to the CTA
// that owns that segment (a tile may read past its segment but never writes
// past it).
#include "iskv_internal.cuh"
#include "tc_util.cuh"

namespace iskv {

namespace {

using namespace tc;

constexpr int kTileRows = 128;
constexpr int kChunkRows = 4096;
constexpr int kThreads = 128;

struct __align__(16) Shared {
    uint64_t full[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

__host__ __device__ inline size_t smem_bytes(int r) {
    // header, 3 transform splits (r x r bf16), 2 tile buffers (128 x r bf16)
    return 128 + 3 * (size_t)r * r * 2 + 2 * (size_t)kTileRows * r * 2;
}

__device__ __forceinline__ uint32_t tmem_cols_for(int r) {
    uint32_t n = 32;
    while (n < (uint32_t)r) n <<= 1;
    return n;
}

__global__ void __launch_bounds__(kThreads)
resync_tc_kernel(FactorView f, ResyncLaunch rl, int* status) {
    const int task = blockIdx.z, bh = blockIdx.y;
    const int layer = rl.layer[task];
    const int nseg = rl.n_seg[task];
    const int64_t n_rows = rl.n_rows[task];
    const int64_t row_begin = (int64_t)blockIdx.x * kChunkRows;
    if (row_begin >= n_rows) return;                 // whole CTA leaves together
    const int64_t row_end = row_begin + kChunkRows < n_rows ? row_begin + kChunkRows : n_rows;
    const int r = f.r;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    extern __shared__ __align__(1024) uint8_t smem[];
    Shared* sh = reinterpret_cast<Shared*>(smem);
    __nv_bfloat16* xform = reinterpret_cast<__nv_bfloat16*>(smem + 128);
    __nv_bfloat16* tiles = xform + 3 * r * r;
    const uint32_t tile_bytes = (uint32_t)kTileRows * r * 2;

    const int64_t hidx = (int64_t)layer * f.BH + bh;
    __nv_bfloat16* C = reinterpret_cast<__nv_bfloat16*>(f.coef) + hidx * f.n_max * r;
    const int* bounds = f.seg_rows + layer * f.D;
    const uint32_t ncols = tmem_cols_for(r);

    if (warp == 0) {
        tmem_alloc(&sh->tmem_base, ncols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&sh->full[0], 1);
        mbar_init(&sh->full[1], 1);
        mbar_init(&sh->mma_done, 1);
        sh->abort = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    const uint32_t idesc = idesc_f32acc(1, kTileRows, r, 0, 0);
    const uint32_t sbo = (uint32_t)(r / 8) * 128;
    const long long deadline = clock64() + kWaitCycles;

    auto seg_of = [&](int64_t row) {
        int s = 0;
        while (s < nseg && row >= bounds[s]) ++s;
        return s;
    };
    auto tile_end_of = [&](int64_t t0) {
        int64_t e = t0 + kTileRows;
        const int s = seg_of(t0);
        if (s < nseg && bounds[s] < e) e = bounds[s];
        return e < row_end ? e : row_end;
    };

    bool in_flight[2] = {false, false};
    if (tid == 0) {
        mbar_arrive_expect_tx(&sh->full[0], tile_bytes);
        bulk_g2s(tiles, C + row_begin * r, tile_bytes, &sh->full[0]);
    }
    in_flight[0] = true;

    int cur_seg = -1;
    int iter = 0;
    for (int64_t t0 = row_begin; t0 < row_end; ++iter) {
        const int b = iter & 1;
        const int64_t t1 = tile_end_of(t0);
        const int seg = seg_of(t0);
        // prefetch the next tile into the other buffer (its last MMA is done)
        if (t1 < row_end) {
            if (tid == 0) {
                mbar_arrive_expect_tx(&sh->full[b ^ 1], tile_bytes);
                bulk_g2s(tiles + (size_t)(b ^ 1) * kTileRows * r, C + t1 * r, tile_bytes,
                         &sh->full[b ^ 1]);
            }
            in_flight[b ^ 1] = true;
        }
        if (seg != cur_seg) {
            // rewrite map of this segment, split into three bf16 parts, as the
            // K-major B operand: element (n, k) = M[k][n]
            const float* M = f.pend + (hidx * f.D + seg) * (int64_t)r * r;
            for (int e = tid; e < r * r; e += kThreads) {
                const int k = e / r, n = e % r;
                const float x = M[e];
                const __nv_bfloat16 s1 = __float2bfloat16_rn(x);
                const float x1 = x - __bfloat162float(s1);
                const __nv_bfloat16 s2 = __float2bfloat16_rn(x1);
                const __nv_bfloat16 s3 = __float2bfloat16_rn(x1 - __bfloat162float(s2));
                const int64_t o = blocked8(n, k, r);
                xform[o] = s1;
                xform[r * r + o] = s2;
                xform[2 * r * r + o] = s3;
            }
            fence_async_smem();
            __syncthreads();
            cur_seg = seg;
        }
        if (tid == 0) {
            bool ok = mbar_wait(&sh->full[b], (uint32_t)(iter >> 1) & 1u, deadline);
            if (!ok) {
                sh->abort = 1;
                atomicOr(status, kStatusTimeout);
            } else {
                tc_fence_after();
                const uint32_t a0 = smem_u32(tiles + (size_t)b * kTileRows * r);
                const uint32_t x0 = smem_u32(xform);
                for (int s = 0; s < 3; ++s)
                    for (int ks = 0; ks < r / 16; ++ks) {
                        const uint64_t ad = desc_noswizzle(a0 + ks * 256, 128, sbo);
                        const uint64_t bd = desc_noswizzle(x0 + s * r * r * 2 + ks * 256, 128, sbo);
                        mma_f16_ss(tmem, ad, bd, idesc, (s | ks) != 0);
                    }
            }
            mma_commit(&sh->mma_done);   // arrives even when nothing was issued
        }
        in_flight[b] = false;
        if (!mbar_wait(&sh->mma_done, (uint32_t)iter & 1u, deadline)) {
            sh->abort = 1;
            atomicOr(status, kStatusTimeout);
        }
        tc_fence_after();
        __syncthreads();
        if (sh->abort) break;
        // epilogue: this thread's row
        const int64_t row = t0 + tid;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        for (int c0 = 0; c0 < r; c0 += 16) {
            uint32_t v[16];
            tmem_ld16(lane_addr + c0, v);
            tmem_wait_ld();
            if (row < t1) {
                uint32_t pk[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[2 * u]),
                                                              __uint_as_float(v[2 * u + 1]));
                    pk[u] = *reinterpret_cast<uint32_t*>(&h2);
                }
                uint4* dst0 = reinterpret_cast<uint4*>(C + blocked8(row, c0, r));
                uint4* dst1 = reinterpret_cast<uint4*>(C + blocked8(row, c0 + 8, r));
                *dst0 = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *dst1 = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
        tc_fence_before();
        __syncthreads();
        t0 = t1;
        (void)lane;
    }

    // drain: a prefetched tile may still be landing in shared memory
    if (tid == 0) {
        for (int bb = 0; bb < 2; ++bb)
            if (in_flight[bb]) {
                const int uses = (iter + (bb == (iter & 1) ? 0 : 1)) >> 1;
                mbar_wait(&sh->full[bb], (uint32_t)uses & 1u, deadline + kWaitCycles);
            }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace

cudaError_t launch_resync_tc(const FactorView& f, const ResyncLaunch& rl, int* status,
                             cudaStream_t s) {
    if (rl.n_tasks <= 0) return cudaSuccess;
    int max_rows = 0;
    for (int i = 0; i < rl.n_tasks; ++i) max_rows = rl.n_rows[i] > max_rows ? rl.n_rows[i] : max_rows;
    if (max_rows <= 0) return cudaSuccess;
    const size_t bytes = smem_bytes(f.r);
    cudaError_t e = cudaFuncSetAttribute(resync_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((max_rows + kChunkRows - 1) / kChunkRows, f.BH, rl.n_tasks);
    resync_tc_kernel<<<grid, kThreads, bytes, s>>>(f, rl, status);
    return cudaGetLastError();
}

}  // namespace iskv
