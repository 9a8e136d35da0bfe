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
constexpr int kWarps = kThreads / 32;
constexpr int kTile = 64;
constexpr int kMaxAcc = kMaxGroup * (kHeadDim + kHeadDim) / kThreads;  // 8

struct Smem {
    size_t bk, q, kt, ck, cv, s, misc;
};

__host__ __device__ inline Smem smem_layout(int rK, int rV, int g) {
    Smem L;
    L.bk = (size_t)kHeadDim * (rK + 1);
    L.q = (size_t)g * kHeadDim;
    L.kt = (size_t)kTile * kHeadDim;
    L.ck = (size_t)kTile * rK;
    L.cv = (size_t)kTile * (rV > kHeadDim ? rV : kHeadDim);
    L.s = (size_t)g * kTile;
    L.misc = 4 * (size_t)kMaxGroup;
    return L;
}

__host__ __device__ inline size_t smem_floats(const Smem& L) {
    return L.bk + L.q + L.kt + L.ck + L.cv + L.s + L.misc;
}

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
    extern __shared__ float sm[];
    float* sBk = sm;
    float* sQ = sBk + L.bk;
    float* sK = sQ + L.q;
    float* sCk = sK + L.kt;
    float* sCv = sCk + L.ck;
    float* sS = sCv + L.cv;
    float* sMax = sS + L.s;
    float* sSum = sMax + kMaxGroup;
    float* sScale = sSum + kMaxGroup;

    const float* Bk = a.K.basis + hidx * d * rK;
    for (int e = tid; e < d * rK; e += kThreads) sBk[(e / rK) * (rK + 1) + e % rK] = Bk[e];
    const KvT* q = reinterpret_cast<const KvT*>(a.q) + ((int64_t)b * a.Hq + (int64_t)kvh * g) * d;
    for (int e = tid; e < g * d; e += kThreads) sQ[e] = to_f32(q[e]);
    if (tid < kMaxGroup) {
        sMax[tid] = -INFINITY;
        sSum[tid] = 0.f;
        sScale[tid] = 1.f;
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
    __syncthreads();

    for (int64_t j = j0; j < j1;) {
        const bool prot = j < P;
        const bool comp = !prot && j < c_end;
        int64_t jend = j + kTile;
        if (jend > j1) jend = j1;
        if (prot && jend > P) jend = P;
        if (comp && jend > c_end) jend = c_end;
        const int nt = (int)(jend - j);

        if (comp) {
            const int64_t jc = j - P;   // coefficient row
            if (a.K.quant) {
                // latent-channel codes: decoded to fp32 while staged
                for (int e = tid; e < kTile * rK; e += kThreads)
                    sCk[e] = (e / rK < nt) ? quant_value(a.K, hidx, jc + e / rK, e % rK) : 0.f;
                for (int e = tid; e < kTile * rV; e += kThreads)
                    sCv[e] = (e / rV < nt) ? quant_value(a.V, hidx, jc + e / rV, e % rV) : 0.f;
            } else {
                for (int e = tid; e < kTile * rK; e += kThreads)
                    sCk[e] = (e / rK < nt) ? to_f32(Ck[coef_index(a.K.coef_blocked, rK, jc + e / rK, e % rK)])
                                           : 0.f;
                for (int e = tid; e < kTile * rV; e += kThreads)
                    sCv[e] = (e / rV < nt) ? to_f32(Cv[coef_index(a.V.coef_blocked, rV, jc + e / rV, e % rV)])
                                           : 0.f;
            }
            __syncthreads();
            for (int e = tid; e < kTile * d; e += kThreads) {
                const int t = e / d, i = e % d;
                float s = 0.f;
                for (int c = 0; c < rK; ++c) s = fmaf(sCk[t * rK + c], sBk[i * (rK + 1) + c], s);
                sK[e] = s;
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
                sK[e] = kv;
                sCv[e] = vv;
            }
        }
        __syncthreads();

        if (a.rope) {
            for (int e = tid; e < kTile * (d / 2); e += kThreads) {
                const int t = e / (d / 2), i = e % (d / 2);
                if (t < nt) {
                    const float2 cs = a.rope[(j + t) * (d / 2) + i];
                    const float x1 = sK[t * d + i], x2 = sK[t * d + i + d / 2];
                    sK[t * d + i] = x1 * cs.x - x2 * cs.y;
                    sK[t * d + i + d / 2] = x1 * cs.y + x2 * cs.x;
                }
            }
            __syncthreads();
        }

        for (int pidx = warp; pidx < g * kTile; pidx += kWarps) {
            const int h = pidx / kTile, t = pidx % kTile;
            float s = 0.f;
#pragma unroll
            for (int u = 0; u < d / 32; ++u) s = fmaf(sQ[h * d + lane + 32 * u], sK[t * d + lane + 32 * u], s);
            s = warp_sum(s);
            if (lane == 0) sS[h * kTile + t] = (t < nt) ? s * a.scale : -INFINITY;
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
                if (comp && col < rV) {
                    for (int t = 0; t < nt; ++t) v = fmaf(sS[h * kTile + t], sCv[t * rV + col], v);
                } else if (!comp && col >= rV) {
                    const int i = col - rV;
                    for (int t = 0; t < nt; ++t) v = fmaf(sS[h * kTile + t], sCv[t * d + i], v);
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
            float* P = a.partial + (((int64_t)b * a.Hq + kvh * g + h) * slots + slot) * stride;
            P[2 + col] = acc[u];
        }
    }
    if (tid < g) {
        float* P = a.partial + (((int64_t)b * a.Hq + kvh * g + tid) * slots + slot) * stride;
        P[0] = sMax[tid];
        P[1] = sSum[tid];
    }
}

// One CTA per (sequence, KV head): B_V is staged once (coalesced) for the
// query group; thread i owns output dim i.
__global__ void __launch_bounds__(kHeadDim)
combine_kernel(DecodeArgs a, float* out) {
    const int kvh = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int rV = a.V.r, d = kHeadDim, g = a.g;
    const int64_t hidx = (int64_t)a.layer * a.V.BH + b * a.Hkv + kvh;
    const int stride = 2 + rV + d;
    const int slots = a.splits_total > 0 ? a.splits_total : a.splits;
    extern __shared__ float cs[];
    float* sBv = cs;                               // d x (rV + 1)
    float* sAcc = sBv + d * (rV + 1);              // rV
    float* sW = sAcc + kHeadDim;                   // slots (<= 256)
    const float* Bv = a.V.basis + hidx * d * rV;
    for (int e = tid; e < d * rV; e += blockDim.x) sBv[(e / rV) * (rV + 1) + e % rV] = Bv[e];
    for (int hq = 0; hq < g; ++hq) {
        const int qh = kvh * g + hq;
        const float* P = a.partial + ((int64_t)b * a.Hq + qh) * slots * stride;
        float M = -INFINITY;
        for (int s = 0; s < slots; ++s) M = fmaxf(M, P[s * stride]);
        __syncthreads();                           // sW / sAcc of the previous head consumed
        for (int s = tid; s < slots; s += blockDim.x) {
            const float ms = P[s * stride];
            sW[s] = (ms == -INFINITY) ? 0.f : __expf(ms - M);
        }
        __syncthreads();
        // empty slots (weight 0) are skipped: their other entries are not written
        float Ls = 0.f, vd = 0.f;
        for (int s = 0; s < slots; ++s) {
            const float w = sW[s];
            if (w != 0.f) {
                Ls = fmaf(w, P[s * stride + 1], Ls);
                vd = fmaf(w, P[s * stride + 2 + rV + tid], vd);
            }
        }
        if (tid < rV) {
            float v = 0.f;
            for (int s = 0; s < slots; ++s)
                if (sW[s] != 0.f) v = fmaf(sW[s], P[s * stride + 2 + tid], v);
            sAcc[tid] = v;
        }
        __syncthreads();
        float o = vd;
        for (int c = 0; c < rV; ++c) o = fmaf(sAcc[c], sBv[tid * (rV + 1) + c], o);
        out[((int64_t)b * a.Hq + qh) * d + tid] = o / Ls;
    }
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
    const size_t bytes = ((size_t)kHeadDim * (a.V.r + 1) + kHeadDim + 256) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    combine_kernel<<<dim3(a.Hkv, a.B), kHeadDim, bytes, s>>>(a, out);
    return cudaGetLastError();
}

}  // namespace iskv
