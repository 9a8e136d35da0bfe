// Decode attention over the folded (compressed) rows on the 5th-generation
// tensor cores, for bf16-stored coefficients.
//
// Method: "iS-KV -- Basis-synchronized online low-rank KV compression -- What
// does it mean?" (Jargon: Pre-RoPE keys -- folded keys are rebuilt before
// RoPE and rotated when read) and the ASKV design report (Design
// requirements: values are never rebuilt on the decode path).  For query
// head h of KV head h/g and folded token j < n_c:
//   k_j = C_K[j] B_K^T,  s_j = q_h . RoPE(k_j, j) / sqrt(d),
//   partial softmax (m, l) and acc_h = sum_j p_j C_V[j]   (r_V wide);
// and, for the exact rows j >= n_c (64-token tiles of the window ring),
//   s_j = q_h . RoPE(K_j, j) / sqrt(d) and acc_d = sum_j p_j V_j (d wide),
// all under one online softmax per head; combine_kernel (k_decode.cu) merges
// the per-CTA partials and applies B_V^T once per query head.
//
// Persistent design, one CTA per SM, the flattened (head, 128-token tile)
// space cut into equal contiguous ranges; per CTA 10 warps:
//   warp 0  producer: 1-D bulk copies (TMA engine) of the C_K and C_V tiles
//           or of the exact K and V rows (all contiguous in the blocked
//           layout) into an NS-stage ring, and of the bf16 hi/lo basis of
//           each head it visits;
//   warp 1  MMA issuer: K^ = C_K (B_hi + B_lo)^T, kind::f16, M=128 tokens,
//           N=128 dims, fp32 accumulator in TMEM (two buffers);
//   warps 2-9 epilogue, two ping-pong groups of 4 warps (group = tile
//           parity), one token row per thread:
//           * rotate its row of K^ by R_t (t = row within the tile; the
//             row's cos/sin(t w_i) sit in spare TMEM columns) and write it
//             back to TMEM rounded to tf32; the query is pre-rotated per tile
//             by R_{j0}^T (j0 = tile start), so q'.(R_t k) = q.(R_{j0+t} k);
//           * scores S = K_rot q'^T on the tensor cores (kind::tf32, A from
//             TMEM, q' as tf32 hi+lo parts in the N dimension);
//           * online softmax per query head and group; at the end of each
//             head the two groups' states are merged by log-sum-exp;
//           * p as bf16 hi+lo parts -> O = C_V^T P (kind::f16, C_V tile read
//             MN-major in place; for exact rows O = V^T P with M = d),
//             accumulated with the running rescale.
// Every mbarrier wait is bounded; on timeout the CTA records
// ISKV status bit 2, stops, drains its copies and frees its TMEM.
#include "iskv_internal.cuh"
#include "tc_util.cuh"

#include <type_traits>

namespace iskv {

namespace {

using namespace tc;

constexpr int kTile = 128;
constexpr int kWinTile = 64;     // exact-row tiles: 64 rows never wrap the ring
constexpr int kThreads = 384;
constexpr int kEpi = 256;        // epilogue threads (warps 2-9, two groups of 4)
constexpr int kQN = 16;          // N of the score MMA (q' hi and lo of g <= 8 heads)
constexpr int kPN = 16;          // N of the value MMA (p hi and lo of g <= 8 heads)
constexpr int kBufCols = 160;    // per TMEM buffer: K^ 128 | S 16 | O 16
constexpr int kCsCol = 2 * kBufCols;   // per-row RoPE table: cos 64 | sin 64 | -sin 64 columns
constexpr uint32_t kTmemCols = 512;

struct __align__(8) Bars {
    uint64_t full[4], empty[4];
    uint64_t bk_full[2], bk_empty[4];      // bk_empty[buffer * 2 + group]
    uint64_t kh_full[2], kfree[2], s_full[2], o_full[2];
    uint64_t krot_ready[2], krot_b[2], p_ready[2];   // epilogue -> group issuer: K_rot halves, P written
    uint64_t drain[3];   // abort path: completion of each issuer's outstanding MMAs
};

struct SmemPlan {
    uint32_t bk, stage, stage_k, stage_bytes, qb, pb, total;
};

__host__ __device__ inline SmemPlan plan_smem(int rK, int rV, int ns, int nbk, int nqb) {
    SmemPlan p;
    uint32_t off = 1024;                                        // barriers, scratch
    p.bk = off;                off += nbk * (2 * kTile * rK * 2);  // nbk heads x (hi, lo)
    p.stage_k = (uint32_t)kTile * rK * 2;
    uint32_t sb = p.stage_k + kTile * rV * 2;
    if (sb < 2 * kWinTile * kHeadDim * 2) sb = 2 * kWinTile * kHeadDim * 2;   // exact K and V rows
    p.stage_bytes = sb + 1024;
    p.stage = off;             off += ns * p.stage_bytes;
    p.qb = off;                off += 2 * nqb * (kQN * kTile * 4);   // [group][nqb] q' buffers
    p.pb = off;                off += 2 * (kPN * kTile * 2);
    p.total = off;
    return p;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// barrier of one ping-pong group (ids 2 and 3, 128 threads)
__device__ __forceinline__ void group_sync(int grp) {
    asm volatile("bar.sync %0, 128;" ::"r"(2 + grp) : "memory");
}
// the same barrier, returning whether any of the group's threads passed true
__device__ __forceinline__ bool group_sync_or(int grp, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, p;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(2 + grp)
        : "memory");
    return r != 0;
}
// a tile's probabilities use the running max while no score passes it by
// more than this (p <= e^8); otherwise the tile takes the exact rescale
constexpr float kLazyMax = 8.f;

// offsets of the tf32 (K-major, 8 x 4 core matrices) and bf16 (8 x 8) B operands
__device__ __forceinline__ int qb_off(int n, int k) {
    return ((n >> 3) * (kTile / 4) + (k >> 2)) * 32 + (n & 7) * 4 + (k & 3);
}
// p as the value MMA's B operand, MN-major: [token][16] in 8 x 8 blocks, so one
// thread's (token's) 8 values of an n-block are one 16-byte row
__device__ __forceinline__ int pb_off(int n, int k) {
    return ((k >> 3) * (kPN / 8) + (n >> 3)) * 64 + (k & 7) * 8 + (n & 7);
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(DecodeTcArgs a) {
    const int cta = blockIdx.x;
    const int64_t f0 = (int64_t)cta * a.tiles_per_cta;
    int64_t f1 = f0 + a.tiles_per_cta;
    if (f1 > a.total_tiles) f1 = a.total_tiles;
    if (f0 >= f1) return;
    const int ntiles = (int)(f1 - f0);
    const int tph = a.tiles_per_head;
    const int rK = a.K.r, rV = a.V.r, ns = a.stages, nbk = a.basis_bufs, nqb = a.q_bufs;
    constexpr int g = G;
    constexpr int kQItems = (G * 64 + 127) / 128;   // q' items per epilogue thread
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int d = kHeadDim;

    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + sizeof(Bars));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 4);
    // the epilogue's copy of the flag, taken by one thread before a named
    // barrier so that all 256 epilogue threads leave the loop together
    volatile int* epi_abort = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 8);
    volatile int* flag_max = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 16);   // [2]
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 24);
    float* red = reinterpret_cast<float*>(smem + 512);          // [2 groups][max 4x8 | l 4x8]
    float* mlx = reinterpret_cast<float*>(smem + 256);          // [2 groups][m 8 | l 8]
    const SmemPlan P = plan_smem(rK, rV, ns, nbk, nqb);
    float* sq = reinterpret_cast<float*>(smem + P.total);       // queries of the head, g x d fp32
    uint8_t* bk = smem + P.bk;
    uint8_t* stage = smem + P.stage;
    uint32_t* qb = reinterpret_cast<uint32_t*>(smem + P.qb);
    __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(smem + P.pb);
    const uint32_t stage_bytes = P.stage_bytes;
    const int tiles_c = a.tiles_c;
    constexpr uint32_t kWinBytes = kWinTile * kHeadDim * 2;   // one of K, V
    const uint32_t bk_bytes = 2 * kTile * rK * 2;

    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&bars->bk_empty[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->bk_full[i], 1);
            mbar_init(&bars->kh_full[i], 1);
            mbar_init(&bars->kfree[i], 1);
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->o_full[i], 1);
            mbar_init(&bars->krot_ready[i], kEpi / 2);
            mbar_init(&bars->krot_b[i], kEpi / 2);
            mbar_init(&bars->p_ready[i], 1);
        }
        for (int i = 0; i < 3; ++i) mbar_init(&bars->drain[i], 1);
        *abort_flag = 0;
        flag_max[0] = 0;
        flag_max[1] = 0;
        fence_mbar_init();
    }
    // zero the padding rows (n >= 2g) of the q' and p operands once
    for (int e = tid; e < 2 * nqb * kQN * kTile; e += kThreads) {
        const int buf = e / (kQN * kTile), w = e % (kQN * kTile);
        const int n = w / kTile, k = w % kTile;
        if (n >= 2 * g) qb[buf * kQN * kTile + qb_off(n, k)] = 0u;
    }
    for (int e = tid; e < 2 * kPN * kTile; e += kThreads) {
        const int buf = e / (kPN * kTile), w = e % (kPN * kTile);
        const int n = w / kTile, k = w % kTile;
        if (n >= 2 * g) pb[buf * kPN * kTile + pb_off(n, k)] = __float2bfloat16_rn(0.f);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const long long deadline = clock64() + kWaitCycles;
    const int BH = a.K.BH;

    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kStatusTimeout);
    };

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            int hs = -1, prev = -1, issued = 0;
            for (int n = 0; n < ntiles && !*abort_flag; ++n) {
                const int64_t fi = f0 + n;
                const int head = (int)(fi / tph), tile = (int)(fi % tph);
                const int64_t hidx = (int64_t)a.layer * BH + head;
                if (head != prev) {
                    ++hs;
                    const int hb = hs % nbk;
                    if (hs >= nbk && (!mbar_wait(&bars->bk_empty[2 * hb], ((hs / nbk) - 1) & 1, deadline) ||
                                      !mbar_wait(&bars->bk_empty[2 * hb + 1], ((hs / nbk) - 1) & 1, deadline))) {
                        fail();
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->bk_full[hb], bk_bytes);
                    bulk_g2s(bk + hb * bk_bytes, a.K.bsplit + hidx * 2 * d * rK, bk_bytes, &bars->bk_full[hb]);
                    prev = head;
                }
                const int st = n % ns;
                if (n >= ns && !mbar_wait(&bars->empty[st], ((n / ns) - 1) & 1, deadline)) {
                    fail();
                    break;
                }
                uint8_t* sk = stage + st * stage_bytes;
                if (tile < tiles_c) {
                    const __nv_bfloat16* gk = reinterpret_cast<const __nv_bfloat16*>(a.K.coef) +
                                              hidx * a.K.n_max * rK + (int64_t)tile * kTile * rK;
                    const __nv_bfloat16* gv = reinterpret_cast<const __nv_bfloat16*>(a.V.coef) +
                                              hidx * a.V.n_max * rV + (int64_t)tile * kTile * rV;
                    mbar_arrive_expect_tx(&bars->full[st], P.stage_k + kTile * rV * 2);
                    bulk_g2s(sk, gk, P.stage_k, &bars->full[st]);
                    bulk_g2s(sk + P.stage_k, gv, kTile * rV * 2, &bars->full[st]);
                } else {
                    // exact rows j0..j0+63 sit in ring slots j0 % cap.. (no wrap: cap % 64 == 0)
                    const int64_t j0 = a.n_c + (int64_t)(tile - tiles_c) * kWinTile;
                    const int64_t slot0 = j0 % a.K.cap;
                    const __nv_bfloat16* rk = reinterpret_cast<const __nv_bfloat16*>(a.K.ring) +
                                              (hidx * a.K.cap + slot0) * d;
                    const __nv_bfloat16* rv = reinterpret_cast<const __nv_bfloat16*>(a.V.ring) +
                                              (hidx * a.V.cap + slot0) * d;
                    mbar_arrive_expect_tx(&bars->full[st], 2 * kWinBytes);
                    bulk_g2s(sk, rk, kWinBytes, &bars->full[st]);
                    bulk_g2s(sk + kWinBytes, rv, kWinBytes, &bars->full[st]);
                }
                issued = n + 1;
            }
            if (*abort_flag) {
                // drain the copies this thread issued (bounded)
                for (int n = issued - ns > 0 ? issued - ns : 0; n < issued; ++n)
                    mbar_wait(&bars->full[n % ns], (n / ns) & 1, deadline + kWaitCycles);
            }
        }
    } else if (warp >= 2 && warp < 10) {
        // ---------------- epilogue: two groups of 4 warps, alternate tiles ----------------
        const int ept = tid - 64;                 // 0..255
        const int nc32 = (int)a.n_c, T32 = (int)a.T;
        const int grp = ept >> 7;                 // tiles n with n % 2 == grp
        const int gt = ept & 127;                 // thread within the group
        const int sp = warp & 3;                  // TMEM sub-partition of this warp
        const int row = sp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
        const uint32_t tcs = tmem + kCsCol;
        // this row's in-tile RoPE table (cos, sin of row * w_i) into TMEM
        if (grp == 0) {
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 16) {
                uint32_t vc[16], vs[16], vn[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    float2 v = make_float2(1.f, 0.f);
                    if (a.rope) v = a.rope[row * 64 + c0 + u];
                    vc[u] = __float_as_uint(v.x);
                    vs[u] = __float_as_uint(v.y);
                    vn[u] = __float_as_uint(-v.y);
                }
                tmem_st16(tcs + lane_base + c0, vc);
                tmem_st16(tcs + lane_base + 64 + c0, vs);
                tmem_st16(tcs + lane_base + 128 + c0, vn);
            }
            tmem_wait_st();
        }
        const int MV = rV <= 64 ? 64 : 128;
        const int c_acc = (MV == 64) ? (lane < 16 ? sp * 16 + lane : -1) : row;
        const bool acc_ok = c_acc >= 0 && c_acc < rV;
        float* gred = red + grp * 64;             // [max 4 x 8 | l 4 x 8] of this group
        const uint32_t kh = tmem + grp * kBufCols;   // K^ / S / O buffer of this group
        uint32_t* qbb = qb + nqb * grp * kQN * kTile;   // the group's first q' buffer (head-end exchange)
        __nv_bfloat16* pbb = pb + grp * kPN * kTile;
        // q' operand offsets of this thread's items (hi of dims i, i + 64; lo likewise)
        int qoff[kQItems][4];
#pragma unroll
        for (int k = 0; k < kQItems; ++k) {
            const int item = gt + 128 * k;
            const int h = (item >> 6) < G ? (item >> 6) : 0, i = item & 63;
            qoff[k][0] = qb_off(h, i);
            qoff[k][1] = qb_off(h, i + 64);
            qoff[k][2] = qb_off(G + h, i);
            qoff[k][3] = qb_off(G + h, i + 64);
        }

        float m_run[G], l_thr[G], acc[G], accd[G], alpha[G];
        // acc <- acc * alpha + (p^T C_V of a folded tile); accd likewise for exact tiles
        // (both rescaled every tile: they share the running max)
        auto accumulate = [&](const uint32_t (&o)[16], bool was_win) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float add = __uint_as_float(o[h]) + __uint_as_float(o[G + h]);
                acc[h] = (acc_ok && !was_win) ? fmaf(acc[h], alpha[h], add) : acc[h] * alpha[h];
                accd[h] = was_win ? fmaf(accd[h], alpha[h], add) : accd[h] * alpha[h];
            }
        };
        bool stop = false;
        int n0 = 0;
        while (n0 < ntiles) {
            const int head = (int)((f0 + n0) / tph);
            int s1 = (int)(((int64_t)head + 1) * tph - f0);
            if (s1 > ntiles) s1 = ntiles;
            // queries of the head, fresh softmax state; uniform abort check
            {
                const int bq = head / a.Hkv, kvh = head % a.Hkv;
                const __nv_bfloat16* qg = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                          ((int64_t)bq * a.Hq + (int64_t)kvh * g) * d;
                for (int e = ept; e < g * d; e += kEpi) sq[e] = __bfloat162float(qg[e]);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m_run[h] = -INFINITY;
                l_thr[h] = 0.f;
                acc[h] = 0.f;
                accd[h] = 0.f;
                alpha[h] = 0.f;
            }
            if (ept == 0) *epi_abort = *abort_flag;
            tc_fence_before();
            epi_sync();
            tc_fence_after();
            stop = *epi_abort;                    // latched after the barrier: uniform
            if (stop) break;
            bool have_prev = false, prev_win = false;
            int last = -1;
            // first position of a tile (folded tiles of 128 rows, then exact tiles of 64)
            const int64_t hbase = (int64_t)head * tph;   // flattened index of the head's tile 0
            auto tile_j0 = [&](int nn) {   // positions fit in 32 bits (max_tokens is an int32)
                const int lc = (int)(f0 + nn - hbase);
                return lc >= tiles_c ? nc32 + (lc - tiles_c) * kWinTile : lc * kTile;
            };
            // q' = R_{j0}^T q of tile nn as tf32 hi / lo parts (the score MMA's B
            // operand), in the group's q' buffer (nn >> 1) & 1; rv = cos / sin(j0 w_i)
            // for i = gt & 63, the only frequency this thread rotates by
            // this thread's items (head h, frequency i): item gt + 128 k; their
            // query pair (q_i, q_{i+64}) stays in registers for the whole head
            float qx1[kQItems], qx2[kQItems];
#pragma unroll
            for (int k = 0; k < kQItems; ++k) {
                const int item = gt + 128 * k;
                const int h = (item >> 6) < G ? (item >> 6) : 0, i = item & 63;
                qx1[k] = sq[h * d + i];
                qx2[k] = sq[h * d + i + 64];
            }
            auto build_q = [&](int nn, float2 rv) {
                uint32_t* qd = qbb + (nqb == 2 ? ((nn >> 1) & 1) : 0) * kQN * kTile;
#pragma unroll
                for (int k = 0; k < kQItems; ++k) {
                    if (gt + 128 * k >= G * 64) break;
                    const float y1 = fmaf(rv.x, qx1[k], rv.y * qx2[k]);
                    const float y2 = fmaf(rv.x, qx2[k], -rv.y * qx1[k]);
                    const uint32_t t1 = to_tf32(y1), t2 = to_tf32(y2);
                    qd[qoff[k][0]] = t1;
                    qd[qoff[k][1]] = t2;
                    qd[qoff[k][2]] = to_tf32(y1 - __uint_as_float(t1));
                    qd[qoff[k][3]] = to_tf32(y2 - __uint_as_float(t2));
                }
                fence_async_smem();
            };
            auto rope_of = [&](int nn) {
                return a.rope ? a.rope[(int64_t)tile_j0(nn) * 64 + (gt & 63)] : make_float2(1.f, 0.f);
            };
            const int n_first = n0 + ((n0 & 1) != grp ? 1 : 0);
            // two q' buffers: tile n + 2's q' is built while tile n's scores run;
            // one buffer: each tile builds its own before its RoPE
            if (nqb == 2 && n_first < s1) build_q(n_first, rope_of(n_first));
            for (int n = n_first; n < s1; n += 2) {
                const int st = n % ns;
                const int local = (int)(f0 + n - hbase);
                const bool win = local >= tiles_c;    // exact rows (64-token tile)
                const int j0 = tile_j0(n);
                const int lim = win ? T32 : nc32;
                const int span = win ? kWinTile : kTile;
                const int valid = (lim - j0) < span ? (lim - j0) : span;
                // the next tile's query rotation, loaded now, used after this tile's RoPE
                const float2 rq_next = (nqb == 2 && n + 2 < s1) ? rope_of(n + 2) : make_float2(1.f, 0.f);
                if (nqb == 1) build_q(n, rope_of(n));
                // rotate this row of K^ by R_t, store back as tf32
                if (!mbar_wait(&bars->kh_full[grp], (n >> 1) & 1, deadline)) fail();
                tc_fence_after();
                if (win && !mbar_wait(&bars->full[st], (n / ns) & 1, deadline)) fail();
                const uint4* krow = reinterpret_cast<const uint4*>(stage + st * stage_bytes);
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 16) {
                    uint32_t x1[16], x2[16], cc[16], ss[16];
                    if (!win) {
                        tmem_ld16(kh + lane_base + c0, x1);
                        tmem_ld16(kh + lane_base + 64 + c0, x2);
                    } else {
                        // this row's exact key, dims c0.. and 64 + c0.. (blocked 8 x 8 layout)
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
#pragma unroll
                            for (int v = 0; v < 2; ++v) {
                                uint4 q4 = make_uint4(0u, 0u, 0u, 0u);
                                if (row < valid)
                                    q4 = krow[((row >> 3) * 16 + ((half * 64 + c0) >> 3) + v) * 8 + (row & 7)];
                                uint32_t* dst = half ? x2 : x1;
                                const uint32_t w4[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    dst[v * 8 + 2 * e] = w4[e] << 16;            // low bf16 -> fp32
                                    dst[v * 8 + 2 * e + 1] = w4[e] & 0xFFFF0000u; // high bf16 -> fp32
                                }
                            }
                        }
                    }
                    uint32_t nn[16];
                    tmem_ld16(tcs + lane_base + c0, cc);
                    tmem_ld16(tcs + lane_base + 64 + c0, ss);
                    tmem_ld16(tcs + lane_base + 128 + c0, nn);
                    tmem_wait_ld();
                    // (k1, k2) -> (k1 c - k2 s, k1 s + k2 c), two columns per packed
                    // fp32 op; the tf32 score MMA reads the fp32 bits truncated
#pragma unroll
                    for (int u = 0; u < 16; u += 2) {
                        const float2 k1 = make_float2(__uint_as_float(x1[u]), __uint_as_float(x1[u + 1]));
                        const float2 k2 = make_float2(__uint_as_float(x2[u]), __uint_as_float(x2[u + 1]));
                        const float2 co = make_float2(__uint_as_float(cc[u]), __uint_as_float(cc[u + 1]));
                        const float2 si = make_float2(__uint_as_float(ss[u]), __uint_as_float(ss[u + 1]));
                        const float2 ns = make_float2(__uint_as_float(nn[u]), __uint_as_float(nn[u + 1]));
                        const float2 y1 = __ffma2_rn(k1, co, __fmul2_rn(k2, ns));
                        const float2 y2 = __ffma2_rn(k1, si, __fmul2_rn(k2, co));
                        x1[u] = __float_as_uint(y1.x);
                        x1[u + 1] = __float_as_uint(y1.y);
                        x2[u] = __float_as_uint(y2.x);
                        x2[u + 1] = __float_as_uint(y2.y);
                    }
                    tmem_st16(kh + lane_base + c0, x1);
                    tmem_st16(kh + lane_base + 64 + c0, x2);
                    if (c0 == 16 || c0 == 48) {
                        // dims 0..31 and 64..95 of this row are rotated (first barrier),
                        // then the rest (second): the score MMA starts on the first half
                        // while the second is rotated.  One barrier per half, so every
                        // phase counts each thread exactly once.
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(c0 == 16 ? &bars->krot_ready[grp] : &bars->krot_b[grp]);
                    }
                }
                // the next tile's q' goes to the other buffer while this tile's scores run
                if (nqb == 2 && n + 2 < s1) build_q(n + 2, rq_next);
                // this group's previous tile: p^T C_V accumulated (before O is reused)
                if (have_prev) {
                    if (!mbar_wait(&bars->o_full[grp], ((n - 2) >> 1) & 1, deadline)) fail();
                    tc_fence_after();
                    uint32_t o[16];
                    tmem_ld16(kh + 144 + lane_base, o);
                    tmem_wait_ld();
                    accumulate(o, prev_win);
                }
                // scores and the tile max of each head
                if (!mbar_wait(&bars->s_full[grp], (n >> 1) & 1, deadline)) fail();
                tc_fence_after();
                uint32_t sv[16];
                tmem_ld16(kh + 128 + lane_base, sv);
                tmem_wait_ld();
                float sc[G];
                bool over = false;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    sc[h] = (row < valid) ? (__uint_as_float(sv[h]) + __uint_as_float(sv[G + h])) * a.scale
                                          : -INFINITY;
                    over |= sc[h] > m_run[h] + kLazyMax;   // always true while m_run = -inf
                }
                // p of this row, bf16 hi parts then lo parts, one or two 16-byte rows
                auto store_p = [&](const float (&pv)[G]) {
                    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                    __nv_bfloat16 hv[2 * G];
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        hv[h] = __float2bfloat16_rn(pv[h]);
                        hv[G + h] = __float2bfloat16_rn(pv[h] - __bfloat162float(hv[h]));
                    }
#pragma unroll
                    for (int e = 0; e < 2 * G; ++e) {
                        const uint32_t bits = (uint32_t)__bfloat16_as_ushort(hv[e]);
                        w[e >> 1] |= (e & 1) ? (bits << 16) : bits;
                    }
                    uint4* dst = reinterpret_cast<uint4*>(pbb + pb_off(0, row));
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    if (2 * G > 8) reinterpret_cast<uint4*>(pbb + pb_off(8, row))[0] = make_uint4(w[4], w[5], w[6], w[7]);
                };
                float pv[G];
#pragma unroll
                for (int h = 0; h < G; ++h)
                    pv[h] = (sc[h] == -INFINITY || m_run[h] == -INFINITY) ? 0.f : __expf(sc[h] - m_run[h]);
                store_p(pv);
                fence_async_smem();
                tc_fence_before();
                if (group_sync_or(grp, over)) {          // P complete; rare: exact rescale
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float wm = warp_max(sc[h]);
                        if (lane == 0) gred[sp * 8 + h] = wm;
                    }
                    group_sync(grp);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float tmax = fmaxf(fmaxf(gred[h], gred[8 + h]), fmaxf(gred[16 + h], gred[24 + h]));
                        const float m_new = fmaxf(m_run[h], tmax);
                        const float al = (m_run[h] == -INFINITY) ? 0.f : __expf(m_run[h] - m_new);
                        pv[h] = (sc[h] == -INFINITY) ? 0.f : __expf(sc[h] - m_new);
                        l_thr[h] = fmaf(l_thr[h], al, pv[h]);
                        m_run[h] = m_new;
                        alpha[h] = al;
                    }
                    store_p(pv);
                    fence_async_smem();
                    tc_fence_before();
                    group_sync(grp);                  // rescaled P complete, maxima read
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        l_thr[h] += pv[h];
                        alpha[h] = 1.f;
                    }
                }
                if (gt == 0) mbar_arrive(&bars->p_ready[grp]);   // P of tile n complete
                have_prev = true;
                prev_win = win;
                last = n;
            }
            // close this group's share of the head
            if (have_prev) {
                if (!mbar_wait(&bars->o_full[grp], (last >> 1) & 1, deadline)) fail();
                tc_fence_after();
                uint32_t o[16];
                tmem_ld16(kh + 144 + lane_base, o);
                tmem_wait_ld();
                accumulate(o, prev_win);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float ws = warp_sum(l_thr[h]);
                if (lane == 0) gred[32 + sp * 8 + h] = ws;
            }
            tc_fence_before();
            group_sync(grp);
            // a group's softmax state goes to its own q' buffer, idle now that
            // its last score MMA of the head has completed: [m 8 | l 8 | acc 8 x 128]
            static_assert(2 * kMaxGroup * kHeadDim <= kQN * kTile, "exchange fits");
            float* xg = reinterpret_cast<float*>(qbb);       // [acc 8 x 128 | accd 8 x 128]
            float* xml = mlx + grp * 2 * kMaxGroup;          // [m 8 | l 8]
            if (gt == 0) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    xml[h] = m_run[h];
                    xml[kMaxGroup + h] = gred[32 + h] + gred[40 + h] + gred[48 + h] + gred[56 + h];
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                if (acc_ok) xg[h * kHeadDim + c_acc] = acc[h];
                xg[(kMaxGroup + h) * kHeadDim + row] = accd[h];
            }
            epi_sync();                               // both groups published
            if (grp == 0) {
                // log-sum-exp merge of the two groups, one partial slot per head
                const float* x0 = reinterpret_cast<const float*>(qb);
                const float* x1 = reinterpret_cast<const float*>(qb + nqb * kQN * kTile);
                const float* ml0 = mlx;
                const float* ml1 = mlx + 2 * kMaxGroup;
                const int bq = head / a.Hkv, kvh = head % a.Hkv;
                const int c_first = (int)(((int64_t)head * tph) / a.tiles_per_cta);
                const int slot = cta - c_first;
                const int stride = 2 + rV + d;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float m0 = ml0[h], m1 = ml1[h];
                    const float M = fmaxf(m0, m1);
                    const float w0 = (m0 == -INFINITY) ? 0.f : __expf(m0 - M);
                    const float w1 = (m1 == -INFINITY) ? 0.f : __expf(m1 - M);
                    float* Pp = a.partial + (((int64_t)bq * a.Hq + kvh * g + h) * a.splits_total + slot) * stride;
                    if (acc_ok)
                        Pp[2 + c_acc] = x0[h * kHeadDim + c_acc] * w0 + x1[h * kHeadDim + c_acc] * w1;
                    // d = 128 = group size: thread gt owns dim gt of the exact-row sum
                    Pp[2 + rV + gt] = x0[(kMaxGroup + h) * kHeadDim + gt] * w0 +
                                      x1[(kMaxGroup + h) * kHeadDim + gt] * w1;
                    if (gt == 0) {
                        Pp[0] = M;
                        Pp[1] = ml0[kMaxGroup + h] * w0 + ml1[kMaxGroup + h] * w1;
                    }
                }
            }
            // the last CTA to publish a partial of this head merges all of them
            // (log-sum-exp), applies B_V^T once per query head and writes out;
            // no CTA waits for another, so no ordering between CTAs is assumed
            __threadfence();
            epi_sync();
            {
                const int c_first = (int)(((int64_t)head * tph) / a.tiles_per_cta);
                const int c_last = (int)((((int64_t)head + 1) * tph - 1) / a.tiles_per_cta);
                if (ept == 0) {
                    const int before = atomicAdd(a.done + head, 1);
                    const int last = before == c_last - c_first;
                    if (last) a.done[head] = 0;   // ready for the next call
                    *last_flag = last;
                }
                epi_sync();
                if (*last_flag) {
                    __threadfence();
                    const int bq = head / a.Hkv, kvh = head % a.Hkv;
                    const int nsl = c_last - c_first + 1;
                    const int stride = 2 + rV + d;
                    // exchange area (q' buffers, 16 KB): merged acc [8][128], slot
                    // weights [8][256], 1/L [8]
                    static_assert((kMaxGroup * 128 + kMaxGroup * 256 + kMaxGroup) * 4 <= 2 * kQN * kTile * 4,
                                  "combine scratch fits");
                    float* sacc = reinterpret_cast<float*>(qb);
                    float* sw = sacc + kMaxGroup * 128;
                    float* sinv = sw + kMaxGroup * 256;
                    const float* Pbase = a.partial + ((int64_t)bq * a.Hq + (int64_t)kvh * g) * a.splits_total * stride;
                    if (ept < g) {
                        const float* Ph = Pbase + (int64_t)ept * a.splits_total * stride;
                        float M = -INFINITY;
                        for (int sl = 0; sl < nsl; ++sl) M = fmaxf(M, __ldcg(Ph + sl * stride));
                        float L = 0.f;
                        for (int sl = 0; sl < nsl; ++sl) {
                            const float m = __ldcg(Ph + sl * stride);
                            const float w = (m == -INFINITY) ? 0.f : __expf(m - M);
                            sw[ept * 256 + sl] = w;
                            L = fmaf(w, __ldcg(Ph + sl * stride + 1), L);
                        }
                        sinv[ept] = 1.f / L;
                    }
                    epi_sync();
                    for (int e = ept; e < g * rV; e += kEpi) {
                        const int h = e / rV, c = e - (e / rV) * rV;
                        const float* Ph = Pbase + (int64_t)h * a.splits_total * stride;
                        float v = 0.f;
                        for (int sl = 0; sl < nsl; ++sl) v = fmaf(sw[h * 256 + sl], __ldcg(Ph + sl * stride + 2 + c), v);
                        sacc[h * 128 + c] = v;
                    }
                    epi_sync();
                    const float* Bv = a.V.basis + ((int64_t)a.layer * BH + head) * d * rV;
                    for (int e = ept; e < g * d; e += kEpi) {
                        const int h = e / d, i = e - (e / d) * d;
                        const float* Ph = Pbase + (int64_t)h * a.splits_total * stride;
                        float v = 0.f;
                        for (int sl = 0; sl < nsl; ++sl) v = fmaf(sw[h * 256 + sl], __ldcg(Ph + sl * stride + 2 + rV + i), v);
                        const float* br = Bv + (int64_t)i * rV;
                        for (int c = 0; c < rV; c += 4) {
                            const float4 b4 = *reinterpret_cast<const float4*>(br + c);
                            v = fmaf(sacc[h * 128 + c], b4.x, v);
                            v = fmaf(sacc[h * 128 + c + 1], b4.y, v);
                            v = fmaf(sacc[h * 128 + c + 2], b4.z, v);
                            v = fmaf(sacc[h * 128 + c + 3], b4.w, v);
                        }
                        a.out[((int64_t)bq * a.Hq + (int64_t)kvh * g + h) * d + i] = v * sinv[h];
                    }
                }
            }
            epi_sync();                               // exchange area free again
            n0 = s1;
        }
    } else if (warp >= 10) {
        // ---------------- MMA issuer of group warp - 10 ----------------
        // per tile n of the group: K^ = C_K (B_hi + B_lo)^T (issued as soon as the
        // group's previous score MMA has released the K^ buffer), scores once the
        // epilogue has rotated K^ and written q', values once P is written
        const int grp = warp - 10;
        if (lane == 0) {
            const int MV = rV <= 64 ? 64 : 128;
            const uint32_t idesc_k = idesc_f32acc(1, kTile, d, 0, 0);
            const uint32_t idesc_s = idesc_f32acc(2, kTile, kQN, 0, 0);
            const uint32_t idesc_o = idesc_f32acc(1, MV, kPN, 1, 1);
            const uint32_t idesc_ow = idesc_f32acc(1, kTile, kPN, 1, 1);   // exact rows: M = d
            const uint32_t sbo_k = (uint32_t)(rK / 8) * 128;
            const uint32_t sbo_q = (kTile / 4) * 128;
            const uint32_t lbo_v = (uint32_t)(rV / 8) * 128;
            const uint32_t kh = tmem + grp * kBufCols;
            const uint32_t qg = smem_u32(qb + nqb * grp * kQN * kTile);
            const uint32_t p0 = smem_u32(pb + grp * kPN * kTile);
            // K^ of tile n into this group's buffer; exact-row tiles need none
            auto recon = [&](int n, int hb, bool win) -> bool {
                const int st = n % ns;
                if (!mbar_wait(&bars->full[st], (n / ns) & 1, deadline)) return false;
                if (win) {
                    mbar_arrive(&bars->kh_full[grp]);
                    return true;
                }
                tc_fence_after();
                const uint32_t a0 = smem_u32(stage + st * stage_bytes);
                const uint32_t b0 = smem_u32(bk + hb * bk_bytes);
                for (int ks = 0; ks < rK / 16; ++ks)
                    for (int part = 0; part < 2; ++part)
                        mma_f16_ss(kh, desc_noswizzle(a0 + ks * 256, 128, sbo_k),
                                   desc_noswizzle(b0 + part * (kTile * rK * 2) + ks * 256, 128, sbo_k),
                                   idesc_k, (ks | part) != 0);
                mma_commit(&bars->kh_full[grp]);
                return true;
            };
            bool ok = true;
            int hs = -1, n0 = 0;
            while (ok && n0 < ntiles && !*abort_flag) {
                const int head = (int)((f0 + n0) / tph);
                const int64_t hbase = (int64_t)head * tph;
                int s1 = (int)(hbase + tph - f0);
                if (s1 > ntiles) s1 = ntiles;
                ++hs;
                const int hb = hs % nbk;
                const int n_first = n0 + ((n0 & 1) != grp ? 1 : 0);
                if (n_first < s1) {
                    ok = mbar_wait(&bars->bk_full[hb], (hs / nbk) & 1, deadline) &&
                         (n_first < 2 || mbar_wait(&bars->kfree[grp], ((n_first >> 1) - 1) & 1, deadline)) &&
                         recon(n_first, hb, (int)(f0 + n_first - hbase) >= tiles_c);
                }
                for (int n = n_first; ok && n < s1; n += 2) {
                    const int st = n % ns;
                    const bool win = (int)(f0 + n - hbase) >= tiles_c;
                    // scores in two halves of the head dimension, each once the epilogue
                    // has rotated it: dims 0..31 and 64..95 (k-steps 0..3, 8..11), then
                    // 32..63 and 96..127 (k-steps 4..7, 12..15)
                    const uint32_t q0 = qg + (nqb == 2 ? ((n >> 1) & 1) : 0) * (kQN * kTile * 4);
                    bool got = true;
                    for (int half = 0; half < 2; ++half) {
                        if (!mbar_wait(half ? &bars->krot_b[grp] : &bars->krot_ready[grp], (n >> 1) & 1,
                                       deadline)) {
                            got = false;
                            break;
                        }
                        tc_fence_after();
                        for (int j = 0; j < 8; ++j) {
                            const int ks = (j < 4 ? j : j + 4) + 4 * half;
                            mma_tf32_ts(kh + 128, kh + ks * 8, desc_noswizzle(q0 + ks * 256, 128, sbo_q),
                                        idesc_s, (half | j) != 0);
                        }
                    }
                    if (!got) {
                        ok = false;
                        break;
                    }
                    mma_commit(&bars->s_full[grp]);
                    mma_commit(&bars->kfree[grp]);
                    // K_rot of tile n consumed: rebuild tile n + 2 while the epilogue runs
                    // this tile's softmax.  Its data sits in stage (n + 2) % ns, which with
                    // two stages is tile n's own: then it has to wait for value(n) below.
                    auto next_recon = [&]() {
                        return mbar_wait(&bars->kfree[grp], (n >> 1) & 1, deadline) &&
                               recon(n + 2, hb, (int)(f0 + n + 2 - hbase) >= tiles_c);
                    };
                    if (ns >= 3 && n + 2 < s1 && !next_recon()) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&bars->p_ready[grp], (n >> 1) & 1, deadline)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (!win) {
                        const uint32_t v0 = smem_u32(stage + st * stage_bytes + P.stage_k);
                        for (int ks = 0; ks < kTile / 16; ++ks)
                            mma_f16_ss(kh + 144, desc_noswizzle(v0 + ks * 2 * lbo_v, lbo_v, 128),
                                       desc_noswizzle(p0 + ks * 512, 256, 128), idesc_o, ks != 0);
                    } else {
                        // O = V^T P over 64 exact rows: A = V tile, MN-major, M = d
                        const uint32_t v0 = smem_u32(stage + st * stage_bytes + kWinBytes);
                        for (int ks = 0; ks < kWinTile / 16; ++ks)
                            mma_f16_ss(kh + 144, desc_noswizzle(v0 + ks * 2 * 2048, 2048, 128),
                                       desc_noswizzle(p0 + ks * 512, 256, 128), idesc_ow, ks != 0);
                    }
                    mma_commit(&bars->o_full[grp]);
                    mma_commit(&bars->empty[st]);
                    if (ns < 3 && n + 2 < s1 && !next_recon()) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                mma_commit(&bars->bk_empty[2 * hb + grp]);   // this group is done with the basis
                n0 = s1;
            }
            if (!ok) fail();
            if (*abort_flag) {                        // let issued MMAs finish (bounded)
                mma_commit(&bars->drain[1 + grp]);
                mbar_wait(&bars->drain[1 + grp], 0, deadline + kWaitCycles);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

size_t decode_tc_smem_bytes(int rK, int rV, int ns, int nbk, int nqb) {
    // + queries of the head (g x d fp32)
    return plan_smem(rK, rV, ns, nbk, nqb).total + (size_t)kMaxGroup * kHeadDim * 4;
}

template <int G>
cudaError_t launch_g(const DecodeTcArgs& a, cudaStream_t s) {
    const size_t bytes = decode_tc_smem_bytes(a.K.r, a.V.r, a.stages, a.basis_bufs, a.q_bufs);
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    decode_tc_kernel<G><<<a.ncta, kThreads, bytes, s>>>(a);
    return cudaGetLastError();
}

bool decode_tc_supports_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

cudaError_t launch_decode_tc(const DecodeTcArgs& a, cudaStream_t s) {
    switch (a.g) {
        case 1: return launch_g<1>(a, s);
        case 2: return launch_g<2>(a, s);
        case 4: return launch_g<4>(a, s);
        case 8: return launch_g<8>(a, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace iskv
