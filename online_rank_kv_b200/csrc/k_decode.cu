// Decode attention over the mixed cache, split over the token axis.
//
// Method: "iS-KV -- Basis-synchronized online low-rank KV compression -- What
// does it mean?" (Jargon: Pre-RoPE keys: folded keys are rebuilt before RoPE
// and rotated when read) and the ASKV design report (Design requirements: no
// reconstruction on the decode path, i.e. values stay in coefficient form).
// For query head h of KV head h/g and token j:
//   s_j = q_h . RoPE(k_j, j) / sqrt(d),  k_j = C_K[j - P] B_K^T for the folded
//   positions P <= j < P + n_c, the exact row otherwise (the P protected
//   positions and the window);  p = softmax(s) over all T tokens;
//   out_h = (sum_folded p_j C_V[j - P]) B_V^T + sum_exact p_j V_j.
// decode_kernel: one CTA per (split, KV head, sequence) streams 64-token
// tiles of its split (never straddling P or P + n_c), keeps an online softmax (m, l)
// per query head and accumulates r_V-wide (folded) and d-wide (exact) sums.
// combine_kernel merges the splits by log-sum-exp and applies B_V^T once.
#include "iskv_internal.cuh"

namespace iskv {

namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;
constexpr int kMaxAcc = kMaxGroup * (kHeadDim + kHeadDim) / kThreads;  // 8

// Shared memory (floats).  Row strides are padded by 4 so that 16-byte
// vector reads stay aligned and the rows a warp touches fall in different banks.
struct Smem {
    int ldc, ldv;                       // row strides of the C_K and C_V / V tiles
    size_t b, q, c, v, s, rt, misc;
};

__host__ __device__ inline Smem smem_layout(int rK, int rV, int g) {
    Smem L;
    L.ldc = (rK > kHeadDim ? rK : kHeadDim) + 4;   // C_K tile, or exact K rows (d wide)
    L.ldv = (rV > kHeadDim ? rV : kHeadDim) + 4;   // C_V tile, or exact V rows
    L.b = (size_t)rK * kHeadDim;                   // B_K^T: row c = basis column c over the dims
    L.q = (size_t)kMaxGroup * kHeadDim;
    L.c = (size_t)kTile * L.ldc;
    L.v = (size_t)kTile * L.ldv;
    L.s = (size_t)kMaxGroup * kTile;
    L.rt = (size_t)17 * 64 * 2;                    // RoPE steps: R(4 t_i) for t_i < 16, R(1)
    L.misc = 4 * (size_t)kMaxGroup;
    return L;
}

__host__ __device__ inline size_t smem_floats(const Smem& L) {
    return L.b + L.q + L.c + L.v + L.s + L.rt + L.misc;
}

__device__ __forceinline__ void store4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

// One CTA per (split, KV head, sequence), 64-token tiles.  Per folded tile the
// key rows are rebuilt on the CUDA cores in fp32, register-tiled: thread
// (ti, tj) = (tid / 16, tid % 16) owns rows 4 ti .. 4 ti + 3 and dims
// 4 tj .. 4 tj + 3 with their RoPE partners 64 + 4 tj .. 64 + 4 tj + 3, so the
// rotation needs no data exchange; each k-step of the rebuild reads one
// 16-byte C_K word per row and two B words for 32 FMAs.  The 16 threads of a
// row group (one half-warp) then reduce their partial dot products with the
// queries by shuffles.
template <typename KvT, typename CoefT>
__global__ void __launch_bounds__(kThreads)
decode_kernel(DecodeArgs a) {
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int d = kHeadDim;
    const int rK = a.K.r, rV = a.V.r, g = a.g;
    const int BH = a.K.BH;
    const int bh = b * a.Hkv + kvh;
    const int64_t hidx = (int64_t)a.layer * BH + bh;
    const int64_t j0 = a.j_begin + (int64_t)split * a.tokens_per_split;
    int64_t j1 = j0 + a.tokens_per_split;
    if (j1 > a.T) j1 = a.T;
    const int slots = a.splits_total > 0 ? a.splits_total : a.splits;
    const int slot = a.split_base + split;

    const Smem L = smem_layout(rK, rV, g);
    extern __shared__ __align__(16) float sm[];
    float* sB = sm;
    float* sQ = sB + L.b;
    float* sC = sQ + L.q;
    float* sV = sC + L.c;
    float* sS = sV + L.v;
    float* sMax = sS + L.s;
    float* sSum = sMax + kMaxGroup;
    float* sScale = sSum + kMaxGroup;
    float2* sR = reinterpret_cast<float2*>(sScale + kMaxGroup);   // [17][64]

    const float* Bk = a.K.basis + hidx * d * rK;   // [d][rK]
    for (int e = tid; e < d * rK; e += kThreads) {
        const int i = e / rK, c = e - i * rK;
        sB[c * d + i] = Bk[e];
    }
    const KvT* q = reinterpret_cast<const KvT*>(a.q) + ((int64_t)b * a.Hq + (int64_t)kvh * g) * d;
    for (int e = tid; e < kMaxGroup * d; e += kThreads) sQ[e] = e < g * d ? to_f32(q[e]) : 0.f;
    if (tid < kMaxGroup) {
        sMax[tid] = -INFINITY;
        sSum[tid] = 0.f;
        sScale[tid] = 1.f;
    }
    // RoPE steps from the table's exact rows: R(4 t_i) (positions 0, 4, .., 60)
    // and R(1); a row at j + 4 t_i + u turns by R(j) R(4 t_i) R(1)^u
    if (a.rope)
        for (int e = tid; e < 17 * 64; e += kThreads) {
            const int rr = e >> 6, fq = e & 63;
            sR[e] = a.rope[(rr < 16 ? 4 * rr : 1) * (d / 2) + fq];
        }
    const int width = rV + d;
    const int n_acc = g * width;
    float acc[kMaxAcc];
#pragma unroll
    for (int u = 0; u < kMaxAcc; ++u) acc[u] = 0.f;

    const CoefT* Ck = reinterpret_cast<const CoefT*>(a.K.coef) + coef_inst(a.K, hidx) * a.K.n_max * rK;
    const CoefT* Cv = reinterpret_cast<const CoefT*>(a.V.coef) + coef_inst(a.V, hidx) * a.V.n_max * rV;
    const KvT* Rk = reinterpret_cast<const KvT*>(a.K.ring) + hidx * a.K.cap * d;
    const KvT* Rv = reinterpret_cast<const KvT*>(a.V.ring) + hidx * a.V.cap * d;
    const KvT* Pk = reinterpret_cast<const KvT*>(a.K.prot) + hidx * a.K.pcap * d;
    const KvT* Pv = reinterpret_cast<const KvT*>(a.V.prot) + hidx * a.V.pcap * d;
    const int64_t P = a.K.P, c_end = P + a.n_c;   // folded positions: [P, P + n_c)
    const int ti = tid >> 4, tj = tid & 15;
    const int dlo = 4 * tj;                       // dims dlo..dlo+3 and 64+dlo..64+dlo+3
    __syncthreads();

    for (int64_t j = j0; j < j1;) {
        // R(j) of this thread's four frequencies: loaded now, used after the rebuild
        float2 rj[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) rj[m] = a.rope ? a.rope[j * (d / 2) + dlo + m] : make_float2(1.f, 0.f);
        const bool prot = j < P;
        const bool comp = !prot && j < c_end;
        int64_t jend = j + kTile;
        if (jend > j1) jend = j1;
        if (prot && jend > P) jend = P;
        if (comp && jend > c_end) jend = c_end;
        const int nt = (int)(jend - j);

        // ---- stage the tile: C_K and C_V rows, or exact K and V rows ----
        if (comp) {
            const int64_t jc = j - P;   // coefficient row
            if (a.K.quant) {
                // latent-channel codes, decoded 8 channels at a time
                for (int e = tid; e < kTile * (rK / 8); e += kThreads) {
                    const int t = e / (rK / 8), c0 = (e - t * (rK / 8)) * 8;
                    float v[8];
                    if (t < nt) {
                        const int64_t rb = hidx * a.K.n_max + jc + t;
                        quant_decode8(a.K, a.K.qcodes + rb * a.K.qwords, a.K.qscales + rb * 4, c0, v);
                    } else {
#pragma unroll
                        for (int k = 0; k < 8; ++k) v[k] = 0.f;
                    }
                    store4(sC + t * L.ldc + c0, v[0], v[1], v[2], v[3]);
                    store4(sC + t * L.ldc + c0 + 4, v[4], v[5], v[6], v[7]);
                }
                for (int e = tid; e < kTile * (rV / 8); e += kThreads) {
                    const int t = e / (rV / 8), c0 = (e - t * (rV / 8)) * 8;
                    float v[8];
                    if (t < nt) {
                        const int64_t rb = hidx * a.V.n_max + jc + t;
                        quant_decode8(a.V, a.V.qcodes + rb * a.V.qwords, a.V.qscales + rb * 4, c0, v);
                    } else {
#pragma unroll
                        for (int k = 0; k < 8; ++k) v[k] = 0.f;
                    }
                    store4(sV + t * L.ldv + c0, v[0], v[1], v[2], v[3]);
                    store4(sV + t * L.ldv + c0 + 4, v[4], v[5], v[6], v[7]);
                }
            } else if (!a.K.coef_blocked && sizeof(CoefT) == 4 &&
                       ((reinterpret_cast<uintptr_t>(Ck) | reinterpret_cast<uintptr_t>(Cv)) & 15) == 0) {
                // fp32 row-major rows: the tile is one contiguous run, read as 16-byte words
                const float4* gk = reinterpret_cast<const float4*>(Ck + jc * rK);
                for (int e = tid; e < kTile * rK / 4; e += kThreads) {
                    const int t = (4 * e) / rK, c = 4 * e - t * rK;
                    const float4 v = t < nt ? gk[e] : make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4*>(sC + t * L.ldc + c) = v;
                }
                const float4* gv = reinterpret_cast<const float4*>(Cv + jc * rV);
                for (int e = tid; e < kTile * rV / 4; e += kThreads) {
                    const int t = (4 * e) / rV, c = 4 * e - t * rV;
                    const float4 v = t < nt ? gv[e] : make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4*>(sV + t * L.ldv + c) = v;
                }
            } else {
                for (int e = tid; e < kTile * rK; e += kThreads) {
                    const int t = e / rK, c = e - t * rK;
                    sC[t * L.ldc + c] =
                        t < nt ? to_f32(Ck[coef_index(a.K.coef_blocked, rK, jc + t, c)]) : 0.f;
                }
                for (int e = tid; e < kTile * rV; e += kThreads) {
                    const int t = e / rV, c = e - t * rV;
                    sV[t * L.ldv + c] =
                        t < nt ? to_f32(Cv[coef_index(a.V.coef_blocked, rV, jc + t, c)]) : 0.f;
                }
            }
        } else {
            for (int e = tid; e < kTile * d; e += kThreads) {
                const int t = e / d, i = e % d;
                float kv = 0.f, vv = 0.f;
                if (t < nt && prot) {
                    kv = to_f32(Pk[coef_index(a.K.ring_blocked, d, j + t, i)]);
                    vv = to_f32(Pv[coef_index(a.V.ring_blocked, d, j + t, i)]);
                } else if (t < nt) {
                    const int64_t slot = (j + t - P) % a.K.cap;   // factor position j - P
                    kv = to_f32(Rk[coef_index(a.K.ring_blocked, d, slot, i)]);
                    vv = to_f32(Rv[coef_index(a.V.ring_blocked, d, slot, i)]);
                }
                sC[t * L.ldc + i] = kv;
                sV[t * L.ldv + i] = vv;
            }
        }
        __syncthreads();

        // ---- this thread's 4 rows x 8 dims of the key tile ----
        float k[4][8];
        if (comp) {
            // packed fp32 FMAs: dims (2e, 2e + 1) of the thread's 8 per instruction
            float2 k2[4][4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int e = 0; e < 4; ++e) k2[u][e] = make_float2(0.f, 0.f);
            const float* crow = sC + (4 * ti) * L.ldc;
            for (int c0 = 0; c0 < rK; c0 += 4) {
                float4 cv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) cv[u] = *reinterpret_cast<const float4*>(crow + u * L.ldc + c0);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const float4 b0 = *reinterpret_cast<const float4*>(sB + (c0 + cc) * d + dlo);
                    const float4 b1 = *reinterpret_cast<const float4*>(sB + (c0 + cc) * d + 64 + dlo);
                    const float2 bp[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w),
                                          make_float2(b1.x, b1.y), make_float2(b1.z, b1.w)};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float cu = cc == 0 ? cv[u].x : cc == 1 ? cv[u].y : cc == 2 ? cv[u].z : cv[u].w;
                        const float2 c2 = make_float2(cu, cu);
#pragma unroll
                        for (int e = 0; e < 4; ++e) k2[u][e] = __ffma2_rn(c2, bp[e], k2[u][e]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    k[u][2 * e] = k2[u][e].x;
                    k[u][2 * e + 1] = k2[u][e].y;
                }
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 x0 = *reinterpret_cast<const float4*>(sC + (4 * ti + u) * L.ldc + dlo);
                const float4 x1 = *reinterpret_cast<const float4*>(sC + (4 * ti + u) * L.ldc + 64 + dlo);
                k[u][0] = x0.x; k[u][1] = x0.y; k[u][2] = x0.z; k[u][3] = x0.w;
                k[u][4] = x1.x; k[u][5] = x1.y; k[u][6] = x1.z; k[u][7] = x1.w;
            }
        }
        // ---- RoPE at the row's position: (k_i, k_{i+64}) by angle pos * w_i ----
        if (a.rope) {
            float2 rb[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float2 r4 = sR[ti * 64 + dlo + m];
                rb[m] = make_float2(rj[m].x * r4.x - rj[m].y * r4.y, rj[m].x * r4.y + rj[m].y * r4.x);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float2 r = rb[m];
                    const float x1 = k[u][m], x2 = k[u][m + 4];
                    k[u][m] = x1 * r.x - x2 * r.y;
                    k[u][m + 4] = x1 * r.y + x2 * r.x;
                    const float2 r1 = sR[16 * 64 + dlo + m];
                    rb[m] = make_float2(r.x * r1.x - r.y * r1.y, r.x * r1.y + r.y * r1.x);
                }
            }
        }
        // ---- scores: partial dot products over this thread's 8 dims, then
        // a butterfly over the 16 threads of the row group ----
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h < g) {
                const float4 q0 = *reinterpret_cast<const float4*>(sQ + h * d + dlo);
                const float4 q1 = *reinterpret_cast<const float4*>(sQ + h * d + 64 + dlo);
                float s4[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float s = k[u][0] * q0.x;
                    s = fmaf(k[u][1], q0.y, s);
                    s = fmaf(k[u][2], q0.z, s);
                    s = fmaf(k[u][3], q0.w, s);
                    s = fmaf(k[u][4], q1.x, s);
                    s = fmaf(k[u][5], q1.y, s);
                    s = fmaf(k[u][6], q1.z, s);
                    s = fmaf(k[u][7], q1.w, s);
                    s4[u] = s;
                }
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
                    for (int u = 0; u < 4; ++u) s4[u] += __shfl_xor_sync(0xffffffffu, s4[u], off);
                if (tj < 4) {
                    const int t = 4 * ti + tj;
                    const float sv = tj == 0 ? s4[0] : tj == 1 ? s4[1] : tj == 2 ? s4[2] : s4[3];
                    sS[h * kTile + t] = (t < nt) ? sv * a.scale : -INFINITY;
                }
            }
        }
        __syncthreads();

        if (warp < g) {
            const int h = warp;
            const float s0 = sS[h * kTile + lane], s1 = sS[h * kTile + lane + 32];
            const float tmax = warp_max(fmaxf(s0, s1));
            const float m_old = sMax[h];
            const float m_new = fmaxf(m_old, tmax);
            const float sc = (m_old == -INFINITY) ? 0.f : __expf(m_old - m_new);
            const float p0 = (s0 == -INFINITY) ? 0.f : __expf(s0 - m_new);
            const float p1 = (s1 == -INFINITY) ? 0.f : __expf(s1 - m_new);
            const float ps = warp_sum(p0 + p1);
            sS[h * kTile + lane] = p0;
            sS[h * kTile + lane + 32] = p1;
            if (lane == 0) {
                sSum[h] = sSum[h] * sc + ps;
                sMax[h] = m_new;
                sScale[h] = sc;
            }
        }
        __syncthreads();

#pragma unroll
        for (int u = 0; u < kMaxAcc; ++u) {
            const int e = tid + u * kThreads;
            if (e < n_acc) {
                const int h = e / width, col = e % width;
                float v = acc[u] * sScale[h];
                const float* ph = sS + h * kTile;
                // rows with t >= nt have p = 0 (their scores were -inf) and zeroed
                // coefficients; whole tiles read four p values per shared load
                const int c = comp ? col : col - rV;
                if ((comp && col < rV) || (!comp && col >= rV)) {
                    float v2 = 0.f;
                    for (int t = 0; t < kTile; t += 4) {
                        const float4 p4 = *reinterpret_cast<const float4*>(ph + t);
                        v = fmaf(p4.x, sV[t * L.ldv + c], v);
                        v2 = fmaf(p4.y, sV[(t + 1) * L.ldv + c], v2);
                        v = fmaf(p4.z, sV[(t + 2) * L.ldv + c], v);
                        v2 = fmaf(p4.w, sV[(t + 3) * L.ldv + c], v2);
                    }
                    v += v2;
                }
                acc[u] = v;
            }
        }
        __syncthreads();
        j = jend;
    }

    const int stride = 2 + width;
    for (int u = 0; u < kMaxAcc; ++u) {
        const int e = tid + u * kThreads;
        if (e < n_acc) {
            const int h = e / width, col = e % width;
            float* Pp = a.partial + (((int64_t)b * a.Hq + kvh * g + h) * slots + slot) * stride;
            Pp[2 + col] = acc[u];
        }
    }
    if (tid < g) {
        float* Pp = a.partial + (((int64_t)b * a.Hq + kvh * g + tid) * slots + slot) * stride;
        Pp[0] = sMax[tid];
        Pp[1] = sSum[tid];
    }
}

// One CTA per (query head, sequence), thread i owns output dim i: the split
// maxima and sums are reduced by the whole block, the weighted sums of the
// partials read with independent (unrolled, predicated) loads, then B_V^T.
__global__ void __launch_bounds__(kHeadDim)
combine_kernel(DecodeArgs a, float* out) {
    const int qh = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int rV = a.V.r, d = kHeadDim, g = a.g;
    const int kvh = qh / g;
    const int64_t hidx = (int64_t)a.layer * a.V.BH + b * a.Hkv + kvh;
    const int stride = 2 + rV + d;
    const int slots = a.splits_total > 0 ? a.splits_total : a.splits;
    extern __shared__ float cs[];
    float* sAcc = cs;                              // rV
    float* sW = sAcc + kHeadDim;                   // slots (<= 256)
    float* sRed = sW + 256;                        // 4 warps
    const float* P = a.partial + ((int64_t)b * a.Hq + qh) * slots * stride;
    float m = -INFINITY;
    for (int s = tid; s < slots; s += kHeadDim) m = fmaxf(m, P[s * stride]);
    m = warp_max(m);
    if (lane == 0) sRed[warp] = m;
    __syncthreads();
    const float M = fmaxf(fmaxf(sRed[0], sRed[1]), fmaxf(sRed[2], sRed[3]));
    float ls = 0.f;
    for (int s = tid; s < slots; s += kHeadDim) {
        const float ms = P[s * stride];
        const float w = (ms == -INFINITY) ? 0.f : __expf(ms - M);
        sW[s] = w;
        // empty slots (weight 0) are skipped: their other entries are not written
        if (w != 0.f) ls = fmaf(w, P[s * stride + 1], ls);
    }
    ls = warp_sum(ls);
    __syncthreads();                               // sRed (maxima) read by every thread
    if (lane == 0) sRed[warp] = ls;
    __syncthreads();
    const float Ls = sRed[0] + sRed[1] + sRed[2] + sRed[3];
    float vd = 0.f, va = 0.f;
#pragma unroll 4
    for (int s = 0; s < slots; ++s) {
        const float w = sW[s];
        const float* ps = P + s * stride;
        const float xd = w != 0.f ? ps[2 + rV + tid] : 0.f;
        const float xa = (w != 0.f && tid < rV) ? ps[2 + tid] : 0.f;
        vd = fmaf(w, xd, vd);
        va = fmaf(w, xa, va);
    }
    if (tid < rV) sAcc[tid] = va;
    __syncthreads();
    const float* bv = a.V.basis + (hidx * d + tid) * rV;
    float o = vd;
    if ((reinterpret_cast<uintptr_t>(a.V.basis) & 15) == 0) {
        for (int c = 0; c < rV; c += 4) {
            const float4 b4 = __ldg(reinterpret_cast<const float4*>(bv + c));
            o = fmaf(sAcc[c], b4.x, o);
            o = fmaf(sAcc[c + 1], b4.y, o);
            o = fmaf(sAcc[c + 2], b4.z, o);
            o = fmaf(sAcc[c + 3], b4.w, o);
        }
    } else {
        for (int c = 0; c < rV; ++c) o = fmaf(sAcc[c], __ldg(bv + c), o);
    }
    out[((int64_t)b * a.Hq + qh) * d + tid] = o / Ls;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    const Smem L = smem_layout(a.K.r, a.V.r, a.g);
    const size_t bytes = smem_floats(L) * sizeof(float);
    dim3 grid(a.splits, a.Hkv, a.B);
    if (a.K.kv_bf16) {
        if (a.K.coef_bf16) {
            auto k = decode_kernel<__nv_bfloat16, __nv_bfloat16>;
            cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
            if (e != cudaSuccess) return e;
            k<<<grid, kThreads, bytes, s>>>(a);
        } else {
            auto k = decode_kernel<__nv_bfloat16, float>;
            cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
            if (e != cudaSuccess) return e;
            k<<<grid, kThreads, bytes, s>>>(a);
        }
    } else {
        if (a.K.coef_bf16) {
            auto k = decode_kernel<float, __nv_bfloat16>;
            cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
            if (e != cudaSuccess) return e;
            k<<<grid, kThreads, bytes, s>>>(a);
        } else {
            auto k = decode_kernel<float, float>;
            cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
            if (e != cudaSuccess) return e;
            k<<<grid, kThreads, bytes, s>>>(a);
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_combine(const DecodeArgs& a, float* out, cudaStream_t s) {
    const size_t bytes = ((size_t)kHeadDim + 256 + 4) * sizeof(float);
    combine_kernel<<<dim3(a.Hq, a.B), kHeadDim, bytes, s>>>(a, out);
    return cudaGetLastError();
}

}  // namespace iskv
