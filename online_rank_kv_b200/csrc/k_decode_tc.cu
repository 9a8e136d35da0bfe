// Decode attention over the folded (compressed) rows on the 5th-generation
// tensor cores, for bf16-stored coefficients.
//
// Method: "iS-KV -- Basis-synchronized online low-rank KV compression -- What
// does it mean?" (Jargon: Pre-RoPE keys -- folded keys are rebuilt before
// RoPE and rotated when read) and the ASKV design report (Design
// requirements: values are never rebuilt on the decode path).  For query
// head h of KV head h/g and folded row j < n_c (position P + j after the P
// protected positions):
//   k_j = C_K[j] B_K^T,  s_j = q_h . RoPE(k_j, P + j) / sqrt(d),
//   partial softmax (m, l) and acc_h = sum_j p_j C_V[j]   (r_V wide);
// and, for the exact rows (tiles of 64 or 32 tokens: the window ring after
// the folded rows, and the protected rows before them),
//   s_j = q_h . RoPE(K_j, j) / sqrt(d) and acc_d = sum_j p_j V_j (d wide),
// all under one online softmax per head.
//
// Persistent design, one CTA per SM; the flattened (head, tile) space is cut
// into contiguous runs of equal cost (tiles, plus a fixed charge for every
// head a run enters after its first), one run per CTA.  Per CTA 12 warps:
//   warp 0  producer: 1-D bulk copies (TMA engine) of the C_K and C_V tiles
//           or of the exact K and V rows (all contiguous in the blocked
//           layout) into an NS-stage ring, and of the bf16 hi/lo basis and
//           the bf16 queries of each head it visits;
//   warp 1  TMEM allocation;
//   warps 2-9 epilogue, two ping-pong groups of 4 warps (group = tile
//           parity), one token row per thread:
//           * rotate its row of K^ by R_t (t = row within the tile; the
//             row's cos/sin(t w_i) sit in spare TMEM columns) and write it
//             back to TMEM as fp16 pairs (dim i, dim 64 + i) per column; the
//             query is pre-rotated per tile by R_{j0}^T (j0 = tile start), so
//             q'.(R_t k) = q.(R_{j0+t} k);
//           * online softmax per query head with a lazily updated maximum;
//           * p as bf16 hi+lo parts for the value MMA;
//           * at the end of a head the group publishes its own partial
//             (m, l, r_V-wide and d-wide sums); the last group to publish
//             a head's partial merges them all by log-sum-exp, applies
//             B_V^T once per query head and writes the output.  The two
//             groups never wait for each other.
//   warps 10-11 MMA issuer of group 0 / 1:
//           * K^ = C_K (B_hi + B_lo)^T, kind::f16, M=128 tokens, N=128 dims,
//             fp32 accumulator in TMEM, rebuilt two tiles ahead;
//           * scores S = K_rot q'^T, kind::f16 with A from TMEM and q' as
//             fp16 hi+lo parts in the N dimension, issued in two halves of
//             the head dimension as the epilogue finishes rotating them;
//           * O = C_V^T P (kind::f16, C_V tile read MN-major in place; for
//             exact rows O = V^T P with M = d).
// Rotated keys are held in fp16 (finite for |k| < 65504; the same 11-bit
// significand as tf32); the query as fp16 hi + lo parts keeps ~22 bits.
// Every mbarrier wait is bounded; on timeout the CTA records
// ISKV status bit 2, stops, drains its copies and frees its TMEM.  A score
// that is not finite (a rotated key or query outside the fp16 range) sets
// status bit 4.
#include "iskv_internal.cuh"
#include "tc_util.cuh"

#include <type_traits>

namespace iskv {

namespace {

using namespace tc;

constexpr int kTile = 128;
// exact-row tiles have 64 or 32 rows (the host's choice, win_rows): either
// divides the ring and the protected-row capacity, so a tile never wraps
constexpr int kThreads = 384;
constexpr int kEpi = 256;        // epilogue threads (warps 2-9, two groups of 4)
constexpr int kQN = 16;          // N of the score MMA (q' hi and lo of g <= 8 heads)
constexpr int kPN = 16;          // N of the value MMA (p hi and lo of g <= 8 heads)
constexpr int kBufCols = 160;    // per TMEM buffer: K^ 128 | S 16 | O 16
constexpr int kCsCol = 2 * kBufCols;   // per-row RoPE table: cos 64 | sin 64 | -sin 64 columns
constexpr uint32_t kTmemCols = 512;

struct __align__(8) Bars {
    uint64_t full[6], empty[6];
    uint64_t bk_full[2], bk_empty[4];      // bk_empty[buffer * 2 + group]
    uint64_t kh_full[2], kfree[2], s_full[2], o_full[2];
    uint64_t krot_ready[2], krot_b[2], p_ready[2];   // epilogue -> group issuer: K_rot halves, P written
    uint64_t drain[3];   // abort path: completion of each issuer's outstanding MMAs
};

// one basis buffer: B_hi, B_lo (bf16, 128 x r each), then the head's g <= 8
// queries (bf16, g x d)
__host__ __device__ inline uint32_t bk_stride(int rK) {
    return (uint32_t)(2 * kTile * rK * 2 + kMaxGroup * kHeadDim * 2);
}

struct SmemPlan {
    uint32_t bk, stage, stage_k, stage_bytes, qb, pb, total;
};

constexpr int kQWords = kQN * 64;   // one q' buffer: kQN rows of 128 fp16 (64 words)

__host__ __device__ inline SmemPlan plan_smem(int rK, int rV, int ns, int nbk, int nqb, int wt) {
    SmemPlan p;
    uint32_t off = 1024;                                        // barriers, scratch
    p.bk = off;                off += nbk * bk_stride(rK);        // nbk heads x (hi, lo, queries)
    p.stage_k = (uint32_t)kTile * rK * 2;
    uint32_t sb = p.stage_k + kTile * rV * 2;
    if (sb < 2 * wt * kHeadDim * 2) sb = 2 * wt * kHeadDim * 2;   // exact K and V rows
    p.stage_bytes = sb + 1024;
    p.stage = off;             off += ns * p.stage_bytes;
    p.qb = off;                off += 2 * nqb * (kQWords * 4);   // [group][nqb] q' buffers
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

// q' as the score MMA's B operand: fp16, K-major 8 x 8 core matrices over
// K = 128 positions k, where k = 2u holds dim u and k = 2u + 1 dim 64 + u
// (the order of the packed rotated keys in TMEM).  Word (32-bit) offset of
// the pair (k = 2u, 2u + 1) of row n.
__device__ __forceinline__ int qb_off(int n, int u) {
    return ((n >> 3) * (kTile / 8) + (u >> 2)) * 32 + (n & 7) * 4 + (u & 3);
}
// p as the value MMA's B operand, MN-major: [token][16] in 8 x 8 blocks, so one
// thread's (token's) 8 values of an n-block are one 16-byte row
__device__ __forceinline__ int pb_off(int n, int k) {
    return ((k >> 3) * (kPN / 8) + (n >> 3)) * 64 + (k & 7) * 8 + (n & 7);
}

// the CTA whose tile range holds flattened tile f
__device__ __forceinline__ int cta_of(const DecodeTcArgs& a, int64_t f) {
    int lo = 0, hi = a.ncta - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.cta_start[mid] <= f) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ DecodeTcArgs a) {
    const int cta = blockIdx.x;
    const int64_t f0 = a.cta_start[cta];
    const int64_t f1 = a.cta_start[cta + 1];
    if (f0 >= f1) return;
    const int ntiles = (int)(f1 - f0);
    const int tph = a.tiles_per_head;
    const int rK = a.K.r, rV = a.V.r, ns = a.stages, nbk = a.basis_bufs, nqb = a.q_bufs;
    const int wt = a.win_rows;      // rows of an exact-row tile (64 or 32)
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
    volatile int* epi_abort = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 8);    // [2 groups]
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 16);   // [2 groups]
    static_assert(sizeof(Bars) + 24 <= 512, "scratch words fit below the reduction area");
    float* red = reinterpret_cast<float*>(smem + 512);          // [2 groups][max 4x8 | l 4x8]
    const SmemPlan P = plan_smem(rK, rV, ns, nbk, nqb, wt);
    uint8_t* bk = smem + P.bk;
    uint8_t* stage = smem + P.stage;
    uint32_t* qb = reinterpret_cast<uint32_t*>(smem + P.qb);
    __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(smem + P.pb);
    const uint32_t stage_bytes = P.stage_bytes;
    const int tiles_c = a.tiles_c, tiles_cw = a.tiles_c + a.tiles_w;
    const uint32_t win_bytes = (uint32_t)wt * kHeadDim * 2;   // one of K, V
    const uint32_t bk_bytes = 2 * kTile * rK * 2;   // B_hi, B_lo of one head
    const uint32_t bks = bk_stride(rK);
    const uint32_t q_bytes = (uint32_t)g * d * 2;    // the head's queries, bf16

    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) {
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
        fence_mbar_init();
    }
    // zero the padding rows (n >= 2g) of the q' and p operands once
    for (int e = tid; e < 2 * nqb * kQN * 64; e += kThreads) {
        const int buf = e / (kQN * 64), w = e % (kQN * 64);
        const int n = w / 64, u = w % 64;
        if (n >= 2 * g) qb[buf * kQWords + qb_off(n, u)] = 0u;
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
    const long long deadline = clock64() + a.pipe_wait;
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
                    if (hs >= nbk && (!mbar_wait_idle(&bars->bk_empty[2 * hb], ((hs / nbk) - 1) & 1, deadline, a.idle_hint_ns) ||
                                      !mbar_wait_idle(&bars->bk_empty[2 * hb + 1], ((hs / nbk) - 1) & 1, deadline, a.idle_hint_ns))) {
                        fail();
                        break;
                    }
                    const int bq = head / a.Hkv, kvh = head % a.Hkv;
                    const __nv_bfloat16* qg = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                              ((int64_t)bq * a.Hq + (int64_t)kvh * g) * d;
                    mbar_arrive_expect_tx(&bars->bk_full[hb], bk_bytes + q_bytes);
                    bulk_g2s(bk + hb * bks, a.K.bsplit + hidx * 2 * d * rK, bk_bytes, &bars->bk_full[hb]);
                    bulk_g2s(bk + hb * bks + bk_bytes, qg, q_bytes, &bars->bk_full[hb]);
                    prev = head;
                }
                const int st = n % ns;
                if (n >= ns && !mbar_wait_idle(&bars->empty[st], ((n / ns) - 1) & 1, deadline, a.idle_hint_ns)) {
                    fail();
                    break;
                }
                uint8_t* sk = stage + st * stage_bytes;
                if (tile < tiles_c) {
                    // a joint-head factor's coefficients are shared by its heads
                    const int64_t cidx = a.K.coef_ws ? head : coef_inst(a.K, hidx);
                    const __nv_bfloat16* gk = reinterpret_cast<const __nv_bfloat16*>(a.K.coef) +
                                              cidx * a.K.n_max * rK + (int64_t)tile * kTile * rK;
                    const __nv_bfloat16* gv = reinterpret_cast<const __nv_bfloat16*>(a.V.coef) +
                                              cidx * a.V.n_max * rV + (int64_t)tile * kTile * rV;
                    mbar_arrive_expect_tx(&bars->full[st], P.stage_k + kTile * rV * 2);
                    bulk_g2s(sk, gk, P.stage_k, &bars->full[st]);
                    bulk_g2s(sk + P.stage_k, gv, kTile * rV * 2, &bars->full[st]);
                } else {
                    const __nv_bfloat16 *rk, *rv;
                    if (tile < tiles_cw) {
                        // window rows at factor positions j0..j0+63 sit in ring slots
                        // j0 % cap.. (no wrap: cap % 64 == 0)
                        const int64_t j0 = a.n_c + (int64_t)(tile - tiles_c) * wt;
                        const int64_t slot0 = j0 % a.K.cap;
                        rk = reinterpret_cast<const __nv_bfloat16*>(a.K.ring) + (hidx * a.K.cap + slot0) * d;
                        rv = reinterpret_cast<const __nv_bfloat16*>(a.V.ring) + (hidx * a.V.cap + slot0) * d;
                    } else {
                        // protected rows j0..j0+63 (positions below P)
                        const int64_t j0 = (int64_t)(tile - tiles_cw) * wt;
                        rk = reinterpret_cast<const __nv_bfloat16*>(a.K.prot) + (hidx * a.K.pcap + j0) * d;
                        rv = reinterpret_cast<const __nv_bfloat16*>(a.V.prot) + (hidx * a.V.pcap + j0) * d;
                    }
                    mbar_arrive_expect_tx(&bars->full[st], 2 * win_bytes);
                    bulk_g2s(sk, rk, win_bytes, &bars->full[st]);
                    bulk_g2s(sk + win_bytes, rv, win_bytes, &bars->full[st]);
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
        // positions: protected [0, P), folded [P, P + n_c), window [P + n_c, T)
        const int nc32 = (int)a.n_c, T32 = (int)a.T, P32 = (int)a.K.P;
        const int Pe32 = T32 < P32 ? T32 : P32;
        const int grp = ept >> 7;                 // tiles n with n % 2 == grp
        const int gt = ept & 127;                 // thread within the group
        const int sp = warp & 3;                  // TMEM sub-partition of this warp
        const int row = sp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
        const uint32_t tcs = tmem + kCsCol;
        // this row's in-tile RoPE table (cos, sin, -sin of row * w_i) into TMEM:
        // group grp writes frequencies 32 grp .. 32 grp + 31, all loads issued first
        {
            float4 tv[16];
            if (a.rope) {
                const float4* src = reinterpret_cast<const float4*>(a.rope + row * 64 + grp * 32);
#pragma unroll
                for (int u = 0; u < 16; ++u) tv[u] = src[u];
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) tv[u] = make_float4(1.f, 0.f, 1.f, 0.f);
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t vc[16], vs[16], vn[16];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float4 v = tv[hh * 8 + u];
                    vc[2 * u] = __float_as_uint(v.x);
                    vs[2 * u] = __float_as_uint(v.y);
                    vn[2 * u] = __float_as_uint(-v.y);
                    vc[2 * u + 1] = __float_as_uint(v.z);
                    vs[2 * u + 1] = __float_as_uint(v.w);
                    vn[2 * u + 1] = __float_as_uint(-v.w);
                }
                const int c0 = grp * 32 + hh * 16;
                tmem_st16(tcs + lane_base + c0, vc);
                tmem_st16(tcs + lane_base + 64 + c0, vs);
                tmem_st16(tcs + lane_base + 128 + c0, vn);
            }
            tmem_wait_st();
        }
        // both halves of the table written before either group's first RoPE
        tc_fence_before();
        epi_sync();
        tc_fence_after();
        const int MV = rV <= 64 ? 64 : 128;
        const int c_acc = (MV == 64) ? (lane < 16 ? sp * 16 + lane : -1) : row;
        const bool acc_ok = c_acc >= 0 && c_acc < rV;
        float* gred = red + grp * 64;             // [max 4 x 8 | l 4 x 8] of this group
        const uint32_t kh = tmem + grp * kBufCols;   // K^ / S / O buffer of this group
        uint32_t* qbb = qb + nqb * grp * kQWords;   // the group's first q' buffer (head-end exchange)
        __nv_bfloat16* pbb = pb + grp * kPN * kTile;
        // q' operand offsets of this thread's items (hi of dims i, i + 64; lo likewise)
        int qoff[kQItems][2];
#pragma unroll
        for (int k = 0; k < kQItems; ++k) {
            const int item = gt + 128 * k;
            const int h = (item >> 6) < G ? (item >> 6) : 0, i = item & 63;
            qoff[k][0] = qb_off(h, i);       // hi parts of dims i, 64 + i
            qoff[k][1] = qb_off(G + h, i);   // lo parts
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
        bool range_bad = false;                   // a non-finite score seen by this thread
        int n0 = 0, hs = -1;
        // the two groups run through the heads independently: each keeps its own
        // softmax state and publishes its own partial slot per head
        while (n0 < ntiles) {
            const int head = (int)((f0 + n0) / tph);
            int s1 = (int)(((int64_t)head + 1) * tph - f0);
            if (s1 > ntiles) s1 = ntiles;
            ++hs;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m_run[h] = -INFINITY;
                l_thr[h] = 0.f;
                acc[h] = 0.f;
                accd[h] = 0.f;
                alpha[h] = 0.f;
            }
            // group-uniform abort check
            if (gt == 0) epi_abort[grp] = *abort_flag;
            group_sync(grp);
            stop = epi_abort[grp];                // latched after the barrier: uniform
            if (stop) break;
            // this group's first tile of the head; none: only the empty partial
            const int n_first = n0 + ((n0 & 1) != grp ? 1 : 0);
            // the head's queries arrived with its basis (the group's own tiles keep
            // the buffer from being reused before this read)
            const __nv_bfloat16* sq = reinterpret_cast<const __nv_bfloat16*>(bk + (hs % nbk) * bks + bk_bytes);
            if (n_first < s1 && !mbar_wait(&bars->bk_full[hs % nbk], (hs / nbk) & 1, deadline)) fail();
            bool have_prev = false, prev_win = false;
            int last = -1;
            // first position of a tile: folded tiles of 128 rows, then window tiles
            // of 64, then protected tiles of 64
            const int64_t hbase = (int64_t)head * tph;   // flattened index of the head's tile 0
            auto tile_j0 = [&](int nn) {   // positions fit in 32 bits (max_tokens is an int32)
                const int lc = (int)(f0 + nn - hbase);
                return lc < tiles_c ? P32 + lc * kTile
                                    : lc < tiles_cw ? P32 + nc32 + (lc - tiles_c) * wt
                                                    : (lc - tiles_cw) * wt;
            };
            // q' = R_{j0}^T q of tile nn as fp16 hi / lo parts (the score MMA's B
            // operand), in the group's q' buffer (nn >> 1) & 1; rv = cos / sin(j0 w_i)
            // for i = gt & 63, the only frequency this thread rotates by
            // this thread's items (head h, frequency i): item gt + 128 k; their
            // query pair (q_i, q_{i+64}) stays in registers for the whole head
            float qx1[kQItems], qx2[kQItems];
#pragma unroll
            for (int k = 0; k < kQItems; ++k) {
                const int item = gt + 128 * k;
                const int h = (item >> 6) < G ? (item >> 6) : 0, i = item & 63;
                qx1[k] = n_first < s1 ? __bfloat162float(sq[h * d + i]) : 0.f;
                qx2[k] = n_first < s1 ? __bfloat162float(sq[h * d + i + 64]) : 0.f;
            }
            auto build_q = [&](int nn, float2 rv) {
                uint32_t* qd = qbb + (nqb == 2 ? ((nn >> 1) & 1) : 0) * kQWords;
#pragma unroll
                for (int k = 0; k < kQItems; ++k) {
                    if (gt + 128 * k >= G * 64) break;
                    const float y1 = fmaf(rv.x, qx1[k], rv.y * qx2[k]);
                    const float y2 = fmaf(rv.x, qx2[k], -rv.y * qx1[k]);
                    const __half2 hi = __floats2half2_rn(y1, y2);
                    const float2 hf = __half22float2(hi);
                    const __half2 lo = __floats2half2_rn(y1 - hf.x, y2 - hf.y);
                    qd[qoff[k][0]] = *reinterpret_cast<const uint32_t*>(&hi);
                    qd[qoff[k][1]] = *reinterpret_cast<const uint32_t*>(&lo);
                }
                fence_async_smem();
            };
            auto rope_of = [&](int nn) {
                return a.rope ? a.rope[(int64_t)tile_j0(nn) * 64 + (gt & 63)] : make_float2(1.f, 0.f);
            };
            // two q' buffers: tile n + 2's q' is built while tile n's scores run;
            // one buffer: each tile builds its own before its RoPE
            if (nqb == 2 && n_first < s1) build_q(n_first, rope_of(n_first));
            for (int n = n_first; n < s1; n += 2) {
                const int st = n % ns;
                const int local = (int)(f0 + n - hbase);
                const bool win = local >= tiles_c;    // exact rows (a tile of wt tokens)
                const int j0 = tile_j0(n);
                const int lim = !win ? P32 + nc32 : local < tiles_cw ? T32 : Pe32;
                const int span = win ? wt : kTile;
                const int valid = (lim - j0) < span ? (lim - j0) : span;
                // the next tile's query rotation, loaded now, used after this tile's RoPE
                const float2 rq_next = (nqb == 2 && n + 2 < s1) ? rope_of(n + 2) : make_float2(1.f, 0.f);
                if (nqb == 1) build_q(n, rope_of(n));
                // rotate this row of K^ by R_t, store back as fp16 pairs
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
                    // fp32 op, rounded to fp16 pairs for the score MMA
#pragma unroll
                    for (int u = 0; u < 16; u += 2) {
                        const float2 k1 = make_float2(__uint_as_float(x1[u]), __uint_as_float(x1[u + 1]));
                        const float2 k2 = make_float2(__uint_as_float(x2[u]), __uint_as_float(x2[u + 1]));
                        const float2 co = make_float2(__uint_as_float(cc[u]), __uint_as_float(cc[u + 1]));
                        const float2 si = make_float2(__uint_as_float(ss[u]), __uint_as_float(ss[u + 1]));
                        const float2 ns = make_float2(__uint_as_float(nn[u]), __uint_as_float(nn[u + 1]));
                        const float2 y1 = __ffma2_rn(k1, co, __fmul2_rn(k2, ns));
                        const float2 y2 = __ffma2_rn(k1, si, __fmul2_rn(k2, co));
                        // column c0 + u <- fp16 (dim c0 + u, dim 64 + c0 + u): over
                        // the fp32 columns this chunk has just read
                        const __half2 p0 = __floats2half2_rn(y1.x, y2.x);
                        const __half2 p1 = __floats2half2_rn(y1.y, y2.y);
                        x1[u] = *reinterpret_cast<const uint32_t*>(&p0);
                        x1[u + 1] = *reinterpret_cast<const uint32_t*>(&p1);
                    }
                    tmem_st16(kh + lane_base + c0, x1);
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
                    const float raw = __uint_as_float(sv[h]) + __uint_as_float(sv[G + h]);
                    sc[h] = (row < valid) ? raw * a.scale : -INFINITY;
                    range_bad |= row < valid && !(fabsf(raw) <= 3.0e38f);   // inf or NaN
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
            // this group's partial of the head: slot 2 (cta - first cta of the head) + grp
            const int bq = head / a.Hkv, kvh = head % a.Hkv;
            const int c_first = cta_of(a, (int64_t)head * tph);
            const int c_last = cta_of(a, ((int64_t)head + 1) * tph - 1);
            const int stride = 2 + rV + d;
            {
                const int slot = 2 * (cta - c_first) + grp;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float* Pp = a.partial + (((int64_t)bq * a.Hq + kvh * g + h) * a.splits_total + slot) * stride;
                    if (acc_ok) Pp[2 + c_acc] = acc[h];
                    Pp[2 + rV + row] = accd[h];   // d = 128 = group size: row owns dim row
                    if (gt == 0) {
                        Pp[0] = m_run[h];
                        Pp[1] = gred[32 + h] + gred[40 + h] + gred[48 + h] + gred[56 + h];
                    }
                }
            }
            // the last group to publish a partial of this head merges all of them
            // (log-sum-exp), applies B_V^T once per query head and writes out; no
            // group waits for another, so no ordering between CTAs is assumed.
            // Release: the group's writes, then one thread's fence and count.
            group_sync(grp);
            if (gt == 0) {
                __threadfence();
                const int before = atomicAdd(a.done + head, 1);
                const int lst = before == 2 * (c_last - c_first) + 1;
                if (lst) {
                    a.done[head] = 0;   // ready for the next call
                    __threadfence();    // acquire: every slot's writes are visible
                }
                last_flag[grp] = lst;
            }
            group_sync(grp);
            if (last_flag[grp]) {
                const int nsl = 2 * (c_last - c_first + 1);
                const float* Pbase = a.partial + ((int64_t)bq * a.Hq + (int64_t)kvh * g) * a.splits_total * stride;
                const float* br = a.V.basis + (((int64_t)a.layer * BH + head) * d + gt) * rV;
                for (int c = 0; c < rV; c += 32) asm volatile("prefetch.global.L1 [%0];" ::"l"(br + c));
                // scratch: m, l of every (slot, head) in the group's q' buffers
                // (nqb x 4 KB; the host keeps slots x g <= nqb x 512), the [g][r_V]
                // merged sums in its P buffer (4 KB); both idle once the head's last
                // score and value MMAs have completed
                static_assert(kMaxGroup * 128 * 4 <= kPN * kTile * 2, "merge sums fit the P buffer");
                float* sacc = reinterpret_cast<float*>(pbb);
                float* sml = reinterpret_cast<float*>(qbb);   // [slot][G] m, then [slot][G] l
                const int nml = nsl * G;
                for (int e = gt; e < nml; e += 128) {
                    const float* q = Pbase + ((int64_t)(e % G) * a.splits_total + e / G) * stride;
                    sml[e] = __ldcg(q);
                    sml[nml + e] = __ldcg(q + 1);
                }
                // this thread's columns (acc column gt, exact-row dim gt) of kC slots
                // per batch; the first batch is in flight across the barrier
                constexpr int kC = 32 / G;
                float xa[kC][G], xd[kC][G];
                auto load_batch = [&](int s0) {
#pragma unroll
                    for (int j = 0; j < kC; ++j)
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float* q = Pbase + ((int64_t)h * a.splits_total + s0 + j) * stride;
                            const bool in = s0 + j < nsl;
                            xa[j][h] = (in && gt < rV) ? __ldcg(q + 2 + gt) : 0.f;
                            xd[j][h] = in ? __ldcg(q + 2 + rV + gt) : 0.f;
                        }
                };
                load_batch(0);
                group_sync(grp);
                float M[G], L[G], va[G], vd[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    M[h] = -INFINITY;
                    L[h] = 0.f;
                    va[h] = 0.f;
                    vd[h] = 0.f;
                }
                for (int sl = 0; sl < nsl; ++sl)
#pragma unroll
                    for (int h = 0; h < G; ++h) M[h] = fmaxf(M[h], sml[sl * G + h]);
                for (int s0 = 0; s0 < nsl; s0 += kC) {
                    if (s0 > 0) load_batch(s0);
#pragma unroll
                    for (int j = 0; j < kC; ++j)
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            if (s0 + j >= nsl) continue;
                            const float m = sml[(s0 + j) * G + h];
                            const float w = (m == -INFINITY) ? 0.f : __expf(m - M[h]);
                            L[h] = fmaf(w, sml[nml + (s0 + j) * G + h], L[h]);
                            va[h] = fmaf(w, xa[j][h], va[h]);
                            vd[h] = fmaf(w, xd[j][h], vd[h]);   // exact-row sum, dim gt
                        }
                }
#pragma unroll
                for (int h = 0; h < G; ++h)
                    if (gt < rV) sacc[h * rV + gt] = va[h];
                group_sync(grp);
                // out[h][i] = (sum_c acc[h][c] B_V[i][c] + accd[h][i]) / L_h, i = gt
#pragma unroll 4
                for (int c = 0; c < rV; c += 4) {
                    const float4 b4 = *reinterpret_cast<const float4*>(br + c);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float4 s4 = *reinterpret_cast<const float4*>(sacc + h * rV + c);
                        vd[h] = fmaf(s4.x, b4.x, vd[h]);
                        vd[h] = fmaf(s4.y, b4.y, vd[h]);
                        vd[h] = fmaf(s4.z, b4.z, vd[h]);
                        vd[h] = fmaf(s4.w, b4.w, vd[h]);
                    }
                }
#pragma unroll
                for (int h = 0; h < G; ++h)
                    a.out[((int64_t)bq * a.Hq + (int64_t)kvh * g + h) * d + gt] = vd[h] / L[h];
                group_sync(grp);                      // P buffer free again
            }
            n0 = s1;
        }
        if (__any_sync(0xffffffffu, range_bad) && lane == 0) atomicOr(a.status, kStatusRange);
    } else if (warp >= 10) {
        // ---------------- MMA issuer of group warp - 10 ----------------
        // per tile n of the group: K^ = C_K (B_hi + B_lo)^T (issued as soon as the
        // group's previous score MMA has released the K^ buffer), scores once the
        // epilogue has rotated K^ and written q', values once P is written
        const int grp = warp - 10;
        if (lane == 0) {
            const int MV = rV <= 64 ? 64 : 128;
            const uint32_t idesc_k = idesc_f32acc(1, kTile, d, 0, 0);
            const uint32_t idesc_s = idesc_f32acc(0, kTile, kQN, 0, 0);   // fp16 x fp16
            const uint32_t idesc_o = idesc_f32acc(1, MV, kPN, 1, 1);
            const uint32_t idesc_ow = idesc_f32acc(1, kTile, kPN, 1, 1);   // exact rows: M = d
            const uint32_t sbo_k = (uint32_t)(rK / 8) * 128;
            const uint32_t sbo_q = (kTile / 8) * 128;
            const uint32_t lbo_v = (uint32_t)(rV / 8) * 128;
            const uint32_t kh = tmem + grp * kBufCols;
            const uint32_t qg = smem_u32(qb + nqb * grp * kQWords);
            const uint32_t p0 = smem_u32(pb + grp * kPN * kTile);
            // K^ of tile n into this group's buffer; exact-row tiles need none
            auto recon = [&](int n, int hb, bool win) -> bool {
                const int st = n % ns;
                if (!mbar_wait_idle(&bars->full[st], (n / ns) & 1, deadline, a.idle_hint_ns)) return false;
                if (win) {
                    mbar_arrive(&bars->kh_full[grp]);
                    return true;
                }
                tc_fence_after();
                const uint32_t a0 = smem_u32(stage + st * stage_bytes);
                const uint32_t b0 = smem_u32(bk + hb * bks);
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
                    ok = mbar_wait_idle(&bars->bk_full[hb], (hs / nbk) & 1, deadline, a.idle_hint_ns) &&
                         (n_first < 2 || mbar_wait_idle(&bars->kfree[grp], ((n_first >> 1) - 1) & 1, deadline, a.idle_hint_ns)) &&
                         recon(n_first, hb, (int)(f0 + n_first - hbase) >= tiles_c);
                } else {
                    // no tile of this head for the group: its release of the basis
                    // buffer below still waits until the producer has filled the
                    // buffer for this head, so it can never run two releases ahead
                    // of the producer's parity wait on the same barrier
                    ok = mbar_wait_idle(&bars->bk_full[hb], (hs / nbk) & 1, deadline, a.idle_hint_ns);
                }
                for (int n = n_first; ok && n < s1; n += 2) {
                    const int st = n % ns;
                    const bool win = (int)(f0 + n - hbase) >= tiles_c;
                    // scores in two halves of the head dimension, each once the epilogue
                    // has rotated it: dims 0..31 and 64..95 (k-steps 0..3, 8..11), then
                    // 32..63 and 96..127 (k-steps 4..7, 12..15)
                    const uint32_t q0 = qg + (nqb == 2 ? ((n >> 1) & 1) : 0) * (kQWords * 4);
                    bool got = true;
                    for (int half = 0; half < 2; ++half) {
                        if (!mbar_wait_idle(half ? &bars->krot_b[grp] : &bars->krot_ready[grp], (n >> 1) & 1,
                                            deadline, a.idle_hint_ns)) {
                            got = false;
                            break;
                        }
                        tc_fence_after();
                        for (int j = 0; j < 4; ++j) {
                            const int ks = 4 * half + j;   // K = 16: 8 TMEM columns per step
                            mma_f16_ts(kh + 128, kh + ks * 8, desc_noswizzle(q0 + ks * 256, 128, sbo_q),
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
                        return mbar_wait_idle(&bars->kfree[grp], (n >> 1) & 1, deadline, a.idle_hint_ns) &&
                               recon(n + 2, hb, (int)(f0 + n + 2 - hbase) >= tiles_c);
                    };
                    if (ns >= 3 && n + 2 < s1 && !next_recon()) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait_idle(&bars->p_ready[grp], (n >> 1) & 1, deadline, a.idle_hint_ns)) {
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
                        // O = V^T P over wt exact rows: A = V tile, MN-major, M = d
                        const uint32_t v0 = smem_u32(stage + st * stage_bytes + win_bytes);
                        for (int ks = 0; ks < wt / 16; ++ks)
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

size_t decode_tc_smem_bytes(int rK, int rV, int ns, int nbk, int nqb, int wt) {
    return plan_smem(rK, rV, ns, nbk, nqb, wt).total;
}

template <int G>
cudaError_t launch_g(const DecodeTcArgs& a, cudaStream_t s) {
    const size_t bytes = decode_tc_smem_bytes(a.K.r, a.V.r, a.stages, a.basis_bufs, a.q_bufs, a.win_rows);
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
