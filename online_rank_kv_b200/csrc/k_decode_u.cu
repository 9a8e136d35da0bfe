// Decode attention over the folded rows with RoPE folded into the queries:
// the scores of a 128-row tile of coefficients come from one tensor-core
// product per tile and r_K * g fused multiply-adds per row.
//
// Method: "iS-KV -- Basis-synchronized online low-rank KV compression -- What
// does it mean?" (Jargon: Pre-RoPE keys -- folded keys are rebuilt before
// RoPE and rotated when read) and the ASKV design report (Design
// requirements: values are never rebuilt on the decode path).  For query head
// h and folded row j at position p = P + j, with k_j = B_K c_j and RoPE
// rotating the pairs (i, i + 64) by p w_i:
//   q . R_p k_j = sum_m c_j[m] U_j[h, m],
//   U_j[h, m]  = sum_i cos(p w_i) alpha_h[i, m] + sin(p w_i) beta_h[i, m],
//   alpha_h[i, m] = q_i B[i, m] + q_{i+64} B[i+64, m],
//   beta_h[i, m]  = q_{i+64} B[i, m] - q_i B[i+64, m].
// So U = T_p A_h: T_p is a fixed table of the rows' positions (128 fp16
// values per row: cos, sin of each frequency, interleaved), A_h = [alpha;
// beta] depends only on the head's queries and basis.  Per 128-row tile one
// kind::f16 MMA (M = 128 rows, N = r_K g, K = 128) gives U in TMEM; each
// epilogue thread then needs its row's r_K coefficients and r_K g products.
// No key is rebuilt, rotated or rounded: the only roundings are the fp16
// table and the fp16 A_h, both ~2^-12 relative.  Exact rows (the window and
// the protected rows) are rotated and scored on the CUDA cores in fp32, four
// threads per row, with their rows of the fp16 position table.  Values as in the rebuild kernel:
// acc_h = sum_j p_j C_V[j] by the value MMA, B_V^T once per query head.
//
// Persistent, one CTA per SM over cost-balanced runs of the flattened (head,
// tile) space.  Per CTA 12 warps:
//   warp 0  lane 0: C_K, C_V tiles or exact K, V rows (and their fp16 RoPE
//           table rows) into an ns-stage ring;
//   warp 1  TMEM allocation; lane 0: the position-table slice of each tile
//           (one slot per epilogue group), each head's queries, and each
//           head's A_h (prepared for all heads by aq_kernel before the decode
//           kernel) once both groups are done with the previous head's;
//   warps 2-9 epilogue, two groups of 4 warps (group = tile parity), one
//           row per thread: scores, online softmax with a lazy maximum, p as
//           bf16 hi + lo; per head each group publishes its partial, the
//           last to publish merges them all by log-sum-exp and applies B_V^T;
//   warps 10-11 MMA issuer of group 0 / 1: U = T_p A_h for the group's next
//           tile as soon as the previous U has been read, O = C_V^T P.
// Every mbarrier wait is bounded (status bit 2 on timeout, copies drained,
// TMEM freed); a non-finite score sets status bit 4.
#include "iskv_internal.cuh"
#include "tc_util.cuh"

namespace iskv {

namespace {

using namespace tc;

constexpr int kTile = 128;
constexpr int kThreads = 384;
constexpr int kPN = 16;           // N of the value MMA (p hi and lo of g <= 8 heads)
constexpr int kUN = 128;          // max N of the U product (r_K g)
constexpr int kBufCols = 160;     // per group: U 128 | O 16 (at 128) | spare
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxStages = 6;
constexpr uint32_t kTabBytes = kTile * 128 * 2;   // one tile of the position table (fp16)
constexpr uint32_t kBqBytes = kUN * 128 * 2;      // A_h of one head (fp16, N x K)

struct __align__(8) Bars {
    uint64_t full[kMaxStages], empty[kMaxStages];   // coefficient / exact-row stage ring
    uint64_t tfull[2], tempty[2];                   // position-table slot of each group
    uint64_t qfull[2], qempty[2];                   // a head's bf16 queries (two buffers)
    uint64_t bq_full;                               // A_h of the current head copied in
    uint64_t bq_free;                               // both groups done with the current A_h
    uint64_t u_full[2], ufree[2], o_full[2], p_ready[2];
    uint64_t drain[3];
};

struct SmemPlan {
    uint32_t tab, bq, qraw, stage, stage_k, stage_bytes, pb, ms, total;
};

__host__ __device__ inline SmemPlan plan_smem(int rK, int rV, int ns, int wt) {
    SmemPlan p;
    uint32_t off = 1024;                                     // barriers, scratch
    p.tab = off;    off += 2 * kTabBytes;                    // [group] table slice
    p.bq = off;     off += kBqBytes;                         // A_h
    p.qraw = off;   off += 2 * kMaxGroup * kHeadDim * 2;     // [2] bf16 queries
    p.stage_k = (uint32_t)kTile * rK * 2;
    uint32_t sb = p.stage_k + kTile * rV * 2;
    if (sb < 3 * wt * kHeadDim * 2) sb = 3 * wt * kHeadDim * 2;   // exact: K, V, RoPE rows
    p.stage_bytes = (sb + 1023) / 1024 * 1024;
    p.stage = off;  off += ns * p.stage_bytes;
    p.pb = off;     off += 2 * (kPN * kTile * 2);            // [group] P operand
    p.ms = off;     off += 2 * 4096;                         // [group] merge scratch
    p.total = off;
    return p;
}

__device__ __forceinline__ void group_sync(int grp) {
    asm volatile("bar.sync %0, 128;" ::"r"(2 + grp) : "memory");
}
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
constexpr float kLazyMax = 8.f;

// A_h as the U product's B operand: fp16, K-major 8 x 8 core matrices, N rows
// n = h r_K + m, K = 128 with k = 2i the alpha and k = 2i + 1 the beta of
// frequency i.  Word (32-bit) offset of the pair (alpha, beta) of row n.
__device__ __forceinline__ int bq_off(int n, int i) {
    return ((n >> 3) * 16 + (i >> 2)) * 32 + (n & 7) * 4 + (i & 3);
}
// p as the value MMA's B operand, MN-major: [token][16] in 8 x 8 blocks
__device__ __forceinline__ int pb_off(int n, int k) {
    return ((k >> 3) * (kPN / 8) + (n >> 3)) * 64 + (k & 7) * 8 + (n & 7);
}

__device__ __forceinline__ int cta_of(const DecodeTcArgs& a, int64_t f) {
    int lo = 0, hi = a.ncta - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.cta_start[mid] <= f) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 w, float* x) {
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(v[e] << 16);
        x[2 * e + 1] = __uint_as_float(v[e] & 0xFFFF0000u);
    }
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_u_kernel(const __grid_constant__ DecodeTcArgs a) {
    const int cta = blockIdx.x;
    const int64_t f0 = a.cta_start[cta];
    const int64_t f1 = a.cta_start[cta + 1];
    if (f0 >= f1) return;
    const int ntiles = (int)(f1 - f0);
    const int tph = a.tiles_per_head;
    const int rK = a.K.r, rV = a.V.r, ns = a.stages;
    const int NU = rK * G;             // N of the U product (<= 128)
    const int wt = a.win_rows;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int d = kHeadDim;
    constexpr int g = G;

    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bars = reinterpret_cast<Bars*>(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + sizeof(Bars));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 4);
    volatile int* epi_abort = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 8);    // [2]
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + sizeof(Bars) + 16);   // [2]
    static_assert(sizeof(Bars) + 24 <= 512, "scratch words fit below the reduction area");
    float* red = reinterpret_cast<float*>(smem + 512);          // [2 groups][max 4x8 | l 4x8]
    const SmemPlan P = plan_smem(rK, rV, ns, wt);
    uint8_t* tab = smem + P.tab;
    uint32_t* bqw = reinterpret_cast<uint32_t*>(smem + P.bq);
    __nv_bfloat16* qraw = reinterpret_cast<__nv_bfloat16*>(smem + P.qraw);
    uint8_t* stage = smem + P.stage;
    __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(smem + P.pb);
    float* mscr = reinterpret_cast<float*>(smem + P.ms);
    const uint32_t stage_bytes = P.stage_bytes;
    const int tiles_c = a.tiles_c, tiles_cw = a.tiles_c + a.tiles_w;
    // positions: protected [0, P), folded [P, P + n_c), window [P + n_c, T)
    const int nc32 = (int)a.n_c, T32 = (int)a.T, P32 = (int)a.K.P;
    const uint32_t win_bytes = (uint32_t)wt * kHeadDim * 2;
    const uint32_t q_bytes = (uint32_t)g * d * 2;
    const __half* ptab = reinterpret_cast<const __half*>(a.ptab);

    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < kMaxStages; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->tfull[i], 1);
            mbar_init(&bars->tempty[i], 1);
            mbar_init(&bars->qfull[i], 1);
            mbar_init(&bars->qempty[i], 2);   // both groups, after their tiles of the head
            mbar_init(&bars->u_full[i], 1);
            mbar_init(&bars->ufree[i], 128);
            mbar_init(&bars->o_full[i], 1);
            mbar_init(&bars->p_ready[i], 1);
        }
        mbar_init(&bars->bq_full, 1);
        mbar_init(&bars->bq_free, 2);
        for (int i = 0; i < 3; ++i) mbar_init(&bars->drain[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // zero the padding rows (n >= 2g) of the p operands once
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
        // ---------------- producer: coefficient tiles and exact rows ----------------
        if (lane == 0) {
            // global sources of tile n: C_K and C_V rows, or exact K, V rows and their
            // fp16 RoPE table rows (parts of `bytes` each; the third is 0 for folded tiles)
            struct Src {
                const void* p[3];
                uint32_t bytes[3];
            };
            auto source = [&](int n) {
                Src r;
                const int64_t fi = f0 + n;
                const int head = (int)(fi / tph), tile = (int)(fi % tph);
                const int64_t hidx = (int64_t)a.layer * BH + head;
                if (tile < tiles_c) {
                    const int64_t cidx = a.K.coef_ws ? head : coef_inst(a.K, hidx);
                    r.p[0] = reinterpret_cast<const __nv_bfloat16*>(a.K.coef) + cidx * a.K.n_max * rK +
                             (int64_t)tile * kTile * rK;
                    r.p[1] = reinterpret_cast<const __nv_bfloat16*>(a.V.coef) + cidx * a.V.n_max * rV +
                             (int64_t)tile * kTile * rV;
                    r.p[2] = nullptr;
                    r.bytes[0] = P.stage_k;
                    r.bytes[1] = kTile * rV * 2;
                    r.bytes[2] = 0;
                } else {
                    int64_t trow;
                    if (tile < tiles_cw) {
                        const int64_t j0 = a.n_c + (int64_t)(tile - tiles_c) * wt;
                        const int64_t slot0 = j0 % a.K.cap;
                        r.p[0] = reinterpret_cast<const __nv_bfloat16*>(a.K.ring) + (hidx * a.K.cap + slot0) * d;
                        r.p[1] = reinterpret_cast<const __nv_bfloat16*>(a.V.ring) + (hidx * a.V.cap + slot0) * d;
                        trow = j0;                                   // factor row of the window row
                    } else {
                        const int64_t j0 = (int64_t)(tile - tiles_cw) * wt;
                        r.p[0] = reinterpret_cast<const __nv_bfloat16*>(a.K.prot) + (hidx * a.K.pcap + j0) * d;
                        r.p[1] = reinterpret_cast<const __nv_bfloat16*>(a.V.prot) + (hidx * a.V.pcap + j0) * d;
                        trow = a.ptab_rows + j0;                     // the protected part of the table
                    }
                    r.p[2] = ptab + trow * 128;
                    r.bytes[0] = r.bytes[1] = r.bytes[2] = win_bytes;
                }
                return r;
            };
            int issued = 0;
            for (int n = 0; n < ntiles && !*abort_flag; ++n) {
                const int st = n % ns;
                if (n >= ns && !mbar_wait_idle(&bars->empty[st], ((n / ns) - 1) & 1, deadline, a.idle_hint_ns)) {
                    fail();
                    break;
                }
                uint8_t* sk = stage + st * stage_bytes;
                const Src r = source(n);
                mbar_arrive_expect_tx(&bars->full[st], r.bytes[0] + r.bytes[1] + r.bytes[2]);
                bulk_g2s(sk, r.p[0], r.bytes[0], &bars->full[st]);
                bulk_g2s(sk + r.bytes[0], r.p[1], r.bytes[1], &bars->full[st]);
                if (r.bytes[2]) bulk_g2s(sk + 2 * r.bytes[0], r.p[2], r.bytes[2], &bars->full[st]);
                issued = n + 1;
            }
            if (*abort_flag) {
                for (int n = issued - ns > 0 ? issued - ns : 0; n < issued; ++n)
                    mbar_wait(&bars->full[n % ns], (n / ns) & 1, deadline + kWaitCycles);
            }
        }
    } else if (warp == 1) {
        // ---------------- producer: position-table slices and queries ----------------
        if (lane == 0) {
            int hs = -1, prev = -1, tissued = 0, qissued = 0, bqissued = 0;
            for (int n = 0; n < ntiles && !*abort_flag; ++n) {
                const int64_t fi = f0 + n;
                const int head = (int)(fi / tph), tile = (int)(fi % tph);
                if (head != prev) {
                    ++hs;
                    const int b = hs & 1;
                    if (hs >= 2 && !mbar_wait_idle(&bars->qempty[b], ((hs >> 1) - 1) & 1, deadline, a.idle_hint_ns)) {
                        fail();
                        break;
                    }
                    const int bq = head / a.Hkv, kvh = head % a.Hkv;
                    const __nv_bfloat16* qg = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                              ((int64_t)bq * a.Hq + (int64_t)kvh * g) * d;
                    mbar_arrive_expect_tx(&bars->qfull[b], q_bytes);
                    bulk_g2s(qraw + b * kMaxGroup * d, qg, q_bytes, &bars->qfull[b]);
                    // the head's query-basis products (prepared for every head by
                    // aq_kernel) once both groups are done with the previous head's
                    if (hs >= 1 && !mbar_wait_idle(&bars->bq_free, (hs - 1) & 1, deadline, a.idle_hint_ns)) {
                        fail();
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->bq_full, (uint32_t)NU * 256);
                    bulk_g2s(bqw, a.aq + (int64_t)head * kUN * 64, (uint32_t)NU * 256, &bars->bq_full);
                    bqissued = hs + 1;
                    qissued = hs + 1;
                    prev = head;
                }
                const int s = n & 1;
                if (n >= 2 && !mbar_wait_idle(&bars->tempty[s], ((n >> 1) - 1) & 1, deadline, a.idle_hint_ns)) {
                    fail();
                    break;
                }
                if (tile < tiles_c) {
                    mbar_arrive_expect_tx(&bars->tfull[s], kTabBytes);
                    bulk_g2s(tab + s * kTabBytes, ptab + (int64_t)tile * kTile * 128, kTabBytes, &bars->tfull[s]);
                } else {
                    mbar_arrive(&bars->tfull[s]);   // exact tile: no slice, the phase still advances
                }
                tissued = n + 1;
            }
            if (*abort_flag) {
                for (int n = tissued - 2 > 0 ? tissued - 2 : 0; n < tissued; ++n)
                    mbar_wait(&bars->tfull[n & 1], (n >> 1) & 1, deadline + kWaitCycles);
                for (int h = qissued - 2 > 0 ? qissued - 2 : 0; h < qissued; ++h)
                    mbar_wait(&bars->qfull[h & 1], (h >> 1) & 1, deadline + kWaitCycles);
                if (bqissued > 0) mbar_wait(&bars->bq_full, (bqissued - 1) & 1, deadline + kWaitCycles);
            }
        }
    } else if (warp >= 2 && warp < 10) {
        // ---------------- epilogue: two groups of 4 warps, alternate tiles ----------------
        const int ept = tid - 64;                 // 0..255
        const int grp = ept >> 7;
        const int gt = ept & 127;
        const int sp = warp & 3;
        const int row = sp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
        const uint32_t ub = tmem + grp * kBufCols;        // U of this group; O at ub + 128
        const int MV = rV <= 64 ? 64 : 128;
        const int c_acc = (MV == 64) ? (lane < 16 ? sp * 16 + lane : -1) : row;
        const bool acc_ok = c_acc >= 0 && c_acc < rV;
        float* gred = red + grp * 64;
        __nv_bfloat16* pbb = pb + grp * kPN * kTile;
        float* sml = mscr + grp * 1024;

        float m_run[G], l_thr[G], acc[G], accd[G], alpha[G];
        auto accumulate = [&](const uint32_t (&o)[16], bool was_win) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float add = __uint_as_float(o[h]) + __uint_as_float(o[G + h]);
                acc[h] = (acc_ok && !was_win) ? fmaf(acc[h], alpha[h], add) : acc[h] * alpha[h];
                accd[h] = was_win ? fmaf(accd[h], alpha[h], add) : accd[h] * alpha[h];
            }
        };
        bool range_bad = false;
        int n0 = 0, hs = -1;
        while (n0 < ntiles) {
            const int head = (int)((f0 + n0) / tph);
            int s1 = (int)(((int64_t)head + 1) * tph - f0);
            if (s1 > ntiles) s1 = ntiles;
            ++hs;
            // group-uniform abort check
            if (gt == 0) epi_abort[grp] = *abort_flag;
            group_sync(grp);
            if (epi_abort[grp]) break;
            // the head's bf16 queries (exact rows read them)
            const int qbuf = hs & 1;
            if (!mbar_wait(&bars->qfull[qbuf], (hs >> 1) & 1, deadline)) fail();
            const __nv_bfloat16* sq = qraw + qbuf * kMaxGroup * d;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m_run[h] = -INFINITY;
                l_thr[h] = 0.f;
                acc[h] = 0.f;
                accd[h] = 0.f;
                alpha[h] = 0.f;
            }
            const int n_first = n0 + ((n0 & 1) != grp ? 1 : 0);
            bool have_prev = false, prev_win = false;
            int last = -1;
            const int64_t hbase = (int64_t)head * tph;
            for (int n = n_first; n < s1; n += 2) {
                const int st = n % ns;
                const int local = (int)(f0 + n - hbase);
                const bool win = local >= tiles_c;
                const int j0 = local < tiles_c ? P32 + local * kTile
                                               : local < tiles_cw ? P32 + nc32 + (local - tiles_c) * wt
                                                                  : (local - tiles_cw) * wt;
                const int lim = !win ? P32 + nc32 : local < tiles_cw ? T32 : (T32 < P32 ? T32 : P32);
                const int span = win ? wt : kTile;
                const int valid = (lim - j0) < span ? (lim - j0) : span;
                if (!mbar_wait(&bars->u_full[grp], (n >> 1) & 1, deadline)) fail();
                tc_fence_after();
                if (!mbar_wait(&bars->full[st], (n / ns) & 1, deadline)) fail();
                const uint4* srow = reinterpret_cast<const uint4*>(stage + st * stage_bytes);
                float raw[G];
                if (!win) {
                    // s_h = sum_m c[m] U[h][m]: this row's coefficients (bf16 blocked
                    // rows of the stage) against its U row in TMEM, 16 columns a step
                    float2 s2[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) s2[h] = make_float2(0.f, 0.f);
                    const int cgk = rK >> 3;
                    for (int c0 = 0; c0 < rK; c0 += 16) {
                        float c[16];
                        unpack_bf16x8(srow[((row >> 3) * cgk + (c0 >> 3)) * 8 + (row & 7)], c);
                        unpack_bf16x8(srow[((row >> 3) * cgk + (c0 >> 3) + 1) * 8 + (row & 7)], c + 8);
                        constexpr int HB = G < 4 ? G : (G == 8 ? 2 : 4);   // heads per TMEM batch
#pragma unroll
                        for (int h0 = 0; h0 < G; h0 += HB) {
                            uint32_t u[HB][16];
#pragma unroll
                            for (int hh = 0; hh < HB; ++hh)
                                tmem_ld16(ub + lane_base + (h0 + hh) * rK + c0, u[hh]);
                            tmem_wait_ld();
#pragma unroll
                            for (int hh = 0; hh < HB; ++hh)
#pragma unroll
                                for (int k = 0; k < 16; k += 2)
                                    s2[h0 + hh] = __ffma2_rn(make_float2(c[k], c[k + 1]),
                                                             make_float2(__uint_as_float(u[hh][k]),
                                                                         __uint_as_float(u[hh][k + 1])),
                                                             s2[h0 + hh]);
                        }
                    }
#pragma unroll
                    for (int h = 0; h < G; ++h) raw[h] = s2[h].x + s2[h].y;
                } else {
                    // exact rows: four threads per row, 16 frequencies each (dims
                    // 16 p .. 16 p + 15 and 64 + 16 p ..), RoPE rows staged in the
                    // group's table slot, fp32 throughout; the row's scores meet in
                    // the group's scratch and go to the thread that owns the row
                    const int part = gt & 3;
                    for (int rr = gt >> 2; rr < wt; rr += 32) {
                        float s4[G];
#pragma unroll
                        for (int h = 0; h < G; ++h) s4[h] = 0.f;
                        if (rr < valid) {
                            float x1[16], x2[16];
                            const int rb = ((rr >> 3) * 16) * 8 + (rr & 7);
                            unpack_bf16x8(srow[rb + (2 * part) * 8], x1);
                            unpack_bf16x8(srow[rb + (2 * part + 1) * 8], x1 + 8);
                            unpack_bf16x8(srow[rb + (8 + 2 * part) * 8], x2);
                            unpack_bf16x8(srow[rb + (9 + 2 * part) * 8], x2 + 8);
                            // (cos, sin) of frequencies 16 p + k as fp16 pairs: the
                            // stage's third part, same blocked layout as the K rows
#pragma unroll
                            for (int kg = 0; kg < 4; ++kg) {
                                const uint4 w4 = srow[2 * (wt / 8) * 128 + rb + (4 * part + kg) * 8];
                                const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int k = 4 * kg + e;
                                    const float2 cs = __half22float2(*reinterpret_cast<const __half2*>(&ww[e]));
                                    const float y1 = x1[k] * cs.x - x2[k] * cs.y;
                                    const float y2 = x1[k] * cs.y + x2[k] * cs.x;
                                    x1[k] = y1;
                                    x2[k] = y2;
                                }
                            }
#pragma unroll
                            for (int h = 0; h < G; ++h) {
                                // the query's dims 16 p .. 16 p + 15 and 64 + 16 p .. (bf16)
                                const uint4* q1 = reinterpret_cast<const uint4*>(sq + h * d + 16 * part);
                                const uint4* q2 = reinterpret_cast<const uint4*>(sq + h * d + 64 + 16 * part);
                                float sa = 0.f, sb = 0.f;
#pragma unroll
                                for (int k8 = 0; k8 < 2; ++k8) {
                                    float qa[8], qb8[8];
                                    unpack_bf16x8(q1[k8], qa);
                                    unpack_bf16x8(q2[k8], qb8);
#pragma unroll
                                    for (int e = 0; e < 8; ++e) {
                                        sa = fmaf(qa[e], x1[8 * k8 + e], sa);
                                        sb = fmaf(qb8[e], x2[8 * k8 + e], sb);
                                    }
                                }
                                s4[h] = sa + sb;
                            }
                        }
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            s4[h] += __shfl_xor_sync(0xffffffffu, s4[h], 1);
                            s4[h] += __shfl_xor_sync(0xffffffffu, s4[h], 2);
                        }
                        if (part == 0)
#pragma unroll
                            for (int h = 0; h < G; ++h) sml[rr * G + h] = s4[h];
                    }
                    group_sync(grp);
#pragma unroll
                    for (int h = 0; h < G; ++h) raw[h] = row < valid ? sml[row * G + h] : 0.f;
                }
                // U of this tile read (exact tiles: nothing to read)
                tc_fence_before();
                mbar_arrive(&bars->ufree[grp]);
                // this group's previous tile: p^T C_V accumulated (before O is reused)
                if (have_prev) {
                    if (!mbar_wait(&bars->o_full[grp], ((n - 2) >> 1) & 1, deadline)) fail();
                    tc_fence_after();
                    uint32_t o[16];
                    tmem_ld16(ub + 128 + lane_base, o);
                    tmem_wait_ld();
                    accumulate(o, prev_win);
                }
                float sc[G];
                bool over = false;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    sc[h] = (row < valid) ? raw[h] * a.scale : -INFINITY;
                    range_bad |= row < valid && !(fabsf(raw[h]) <= 3.0e38f);   // inf or NaN
                    over |= sc[h] > m_run[h] + kLazyMax;
                }
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
                if (group_sync_or(grp, over)) {
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
                    group_sync(grp);
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        l_thr[h] += pv[h];
                        alpha[h] = 1.f;
                    }
                }
                if (gt == 0) mbar_arrive(&bars->p_ready[grp]);
                have_prev = true;
                prev_win = win;
                last = n;
            }
            // this group has read every U of the head and its queries: release both
            if (gt == 0) {
                mbar_arrive(&bars->bq_free);
                mbar_arrive(&bars->qempty[qbuf]);
            }
            // close this group's share of the head
            if (have_prev) {
                if (!mbar_wait(&bars->o_full[grp], (last >> 1) & 1, deadline)) fail();
                tc_fence_after();
                uint32_t o[16];
                tmem_ld16(ub + 128 + lane_base, o);
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
                    Pp[2 + rV + row] = accd[h];
                    if (gt == 0) {
                        Pp[0] = m_run[h];
                        Pp[1] = gred[32 + h] + gred[40 + h] + gred[48 + h] + gred[56 + h];
                    }
                }
            }
            // the last group to publish a partial of this head merges them all
            group_sync(grp);
            if (gt == 0) {
                __threadfence();
                const int before = atomicAdd(a.done + head, 1);
                const int lst = before == 2 * (c_last - c_first) + 1;
                if (lst) {
                    a.done[head] = 0;
                    __threadfence();
                }
                last_flag[grp] = lst;
            }
            group_sync(grp);
            if (last_flag[grp]) {
                const int nsl = 2 * (c_last - c_first + 1);
                const float* Pbase = a.partial + ((int64_t)bq * a.Hq + (int64_t)kvh * g) * a.splits_total * stride;
                const float* br = a.V.basis + (((int64_t)a.layer * BH + head) * d + gt) * rV;
                for (int c = 0; c < rV; c += 32) asm volatile("prefetch.global.L1 [%0];" ::"l"(br + c));
                // scratch: m, l of every (slot, head) in the group's merge area (4 KB;
                // the host keeps slots x g <= 512), the [g][r_V] merged sums in its P
                // buffer (4 KB), idle once the head's last value MMA has completed
                static_assert(kMaxGroup * 128 * 4 <= kPN * kTile * 2, "merge sums fit the P buffer");
                float* sacc = reinterpret_cast<float*>(pbb);
                const int nml = nsl * G;
                for (int e = gt; e < nml; e += 128) {
                    const float* q = Pbase + ((int64_t)(e % G) * a.splits_total + e / G) * stride;
                    sml[e] = __ldcg(q);
                    sml[nml + e] = __ldcg(q + 1);
                }
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
                            vd[h] = fmaf(w, xd[j][h], vd[h]);
                        }
                }
#pragma unroll
                for (int h = 0; h < G; ++h)
                    if (gt < rV) sacc[h * rV + gt] = va[h];
                group_sync(grp);
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
                group_sync(grp);
            }
            n0 = s1;
        }
        if (__any_sync(0xffffffffu, range_bad) && lane == 0) atomicOr(a.status, kStatusRange);
    } else if (warp >= 10) {
        // ---------------- MMA issuer of group warp - 10 ----------------
        const int grp = warp - 10;
        if (lane == 0) {
            const int MV = rV <= 64 ? 64 : 128;
            const uint32_t idesc_u = idesc_f32acc(0, kTile, NU, 0, 0);     // fp16 x fp16
            const uint32_t idesc_o = idesc_f32acc(1, MV, kPN, 1, 1);
            const uint32_t idesc_ow = idesc_f32acc(1, kTile, kPN, 1, 1);   // exact rows: M = d
            const uint32_t lbo_v = (uint32_t)(rV / 8) * 128;
            const uint32_t ub = tmem + grp * kBufCols;
            const uint32_t t0 = smem_u32(tab + grp * kTabBytes);
            const uint32_t b0 = smem_u32(bqw);
            const uint32_t p0 = smem_u32(pb + grp * kPN * kTile);
            // U of tile n (this group's): after the epilogue has read U of tile n - 2
            auto issue_u = [&](int n, bool win) -> bool {
                if (n >= 2 && !mbar_wait_idle(&bars->ufree[grp], ((n - 2) >> 1) & 1, deadline, a.idle_hint_ns)) return false;
                if (!mbar_wait_idle(&bars->tfull[grp], (n >> 1) & 1, deadline, a.idle_hint_ns)) return false;
                if (win) {
                    mbar_arrive(&bars->tempty[grp]);
                    mbar_arrive(&bars->u_full[grp]);
                    return true;
                }
                tc_fence_after();
                for (int ks = 0; ks < 8; ++ks)   // K = 128 in steps of 16
                    mma_f16_ss(ub, desc_noswizzle(t0 + ks * 256, 128, 2048),
                               desc_noswizzle(b0 + ks * 256, 128, 2048), idesc_u, ks != 0);
                mma_commit(&bars->tempty[grp]);
                mma_commit(&bars->u_full[grp]);
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
                const int n_first = n0 + ((n0 & 1) != grp ? 1 : 0);
                if (n_first < s1)
                    ok = mbar_wait_idle(&bars->bq_full, hs & 1, deadline, a.idle_hint_ns) &&
                         issue_u(n_first, (int)(f0 + n_first - hbase) >= tiles_c);
                for (int n = n_first; ok && n < s1; n += 2) {
                    const int st = n % ns;
                    const bool win = (int)(f0 + n - hbase) >= tiles_c;
                    if (n + 2 < s1 && !issue_u(n + 2, (int)(f0 + n + 2 - hbase) >= tiles_c)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait_idle(&bars->p_ready[grp], (n >> 1) & 1, deadline, a.idle_hint_ns) ||
                        !mbar_wait_idle(&bars->full[st], (n / ns) & 1, deadline, a.idle_hint_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (!win) {
                        const uint32_t v0 = smem_u32(stage + st * stage_bytes + P.stage_k);
                        for (int ks = 0; ks < kTile / 16; ++ks)
                            mma_f16_ss(ub + 128, desc_noswizzle(v0 + ks * 2 * lbo_v, lbo_v, 128),
                                       desc_noswizzle(p0 + ks * 512, 256, 128), idesc_o, ks != 0);
                    } else {
                        const uint32_t v0 = smem_u32(stage + st * stage_bytes + win_bytes);
                        for (int ks = 0; ks < wt / 16; ++ks)
                            mma_f16_ss(ub + 128, desc_noswizzle(v0 + ks * 2 * 2048, 2048, 128),
                                       desc_noswizzle(p0 + ks * 512, 256, 128), idesc_ow, ks != 0);
                    }
                    mma_commit(&bars->o_full[grp]);
                    mma_commit(&bars->empty[st]);
                }
                n0 = s1;
            }
            if (!ok) fail();
            if (*abort_flag) {
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

// A_h of every (sequence, KV head) of the call, in the word order of the U
// product's B operand (bq_off): alpha, beta of frequency i for row n = h r_K + m
// as an fp16 pair, computed in fp32 from the bf16 queries and the fp32 basis.
// One CTA per head; the decode kernel bulk-copies a head's 32 KB when it
// reaches the head.
__global__ void __launch_bounds__(256) aq_kernel(const __grid_constant__ DecodeTcArgs a) {
    const int head = blockIdx.x;
    const int rK = a.K.r, g = a.g, NU = rK * g;
    constexpr int d = kHeadDim;
    const int bq = head / a.Hkv, kvh = head % a.Hkv;
    __shared__ float sq[kMaxGroup * kHeadDim];
    const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(a.q) + ((int64_t)bq * a.Hq + (int64_t)kvh * g) * d;
    for (int e = threadIdx.x; e < g * d; e += 256) sq[e] = __bfloat162float(q[e]);
    __syncthreads();
    const float* Bk = a.K.basis + ((int64_t)a.layer * a.K.BH + head) * d * rK;
    uint32_t* out = a.aq + (int64_t)head * kUN * 64;
    for (int e = threadIdx.x; e < NU * 64; e += 256) {
        const int i = e / NU, n = e - i * NU;
        const int h = n / rK, m = n - h * rK;
        const float b1 = __ldg(Bk + i * rK + m), b2 = __ldg(Bk + (i + 64) * rK + m);
        const float q1 = sq[h * d + i], q2 = sq[h * d + i + 64];
        const __half2 w = __floats2half2_rn(fmaf(q1, b1, q2 * b2), fmaf(q2, b1, -q1 * b2));
        out[bq_off(n, i)] = *reinterpret_cast<const uint32_t*>(&w);
    }
}

}  // namespace

size_t decode_u_smem_bytes(int rK, int rV, int ns, int wt) { return plan_smem(rK, rV, ns, wt).total; }

bool decode_u_supports(int g, int rK) {
    return (g == 1 || g == 2 || g == 4 || g == 8) && rK % 16 == 0 && rK * g <= kUN && rK * g >= 16;
}

template <int G>
static cudaError_t launch_u(const DecodeTcArgs& a, cudaStream_t s) {
    const size_t bytes = decode_u_smem_bytes(a.K.r, a.V.r, a.stages, a.win_rows);
    cudaError_t e = cudaFuncSetAttribute(decode_u_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    decode_u_kernel<G><<<a.ncta, kThreads, bytes, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode_u(const DecodeTcArgs& a, cudaStream_t s) {
    if (!decode_u_supports(a.g, a.K.r) || a.stages < 2 || a.stages > kMaxStages || a.ptab == nullptr ||
        a.aq == nullptr)
        return cudaErrorNotSupported;
    aq_kernel<<<a.K.BH, 256, 0, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return cudaErrorLaunchFailure;
    switch (a.g) {
        case 1: return launch_u<1>(a, s);
        case 2: return launch_u<2>(a, s);
        case 4: return launch_u<4>(a, s);
        case 8: return launch_u<8>(a, s);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace iskv
