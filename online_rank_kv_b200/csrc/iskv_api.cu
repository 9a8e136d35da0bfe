// C ABI of the iS-KV cache (declared in include/iskv.h): configuration checks,
// device buffers, host counters and the order of kernel launches.
//
// Bookkeeping follows the iS-KV explainer ("iS-KV -- Basis-synchronized online
// low-rank KV compression -- What does it mean?": the newest W tokens stay
// exact; every 64 tokens that leave that window are folded as one block):
// T and n_c are host integers per layer, advanced when a call is enqueued;
// ready blocks = floor((T - n_c - W) / 64) when positive.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "decode_plan.h"
#include "iskv_internal.cuh"
#include "tc_util.cuh"

using namespace iskv;

struct iskv_cache {
    iskv_config cfg{};
    int device = 0;
    int64_t cap = 0;      // ring rows per head
    int64_t n_max = 0;    // coefficient rows per head
    int BH = 0;
    int FH = 0;           // factor instances per layer: BH, or batch for joint-head factors
    int D = 1;            // postponed-fold slots per head
    int kv_bytes = 4, coef_bytes = 4;
    // device memory
    void* ring_k = nullptr;
    void* ring_v = nullptr;
    void* prot_k = nullptr;       // protected rows 0..P-1, blocked like the ring
    void* prot_v = nullptr;
    int64_t pcap = 0;             // protected rows per head (P rounded up to 64)
    void* coef_k = nullptr;
    void* coef_v = nullptr;
    float* basis_k = nullptr;
    float* basis_v = nullptr;
    __nv_bfloat16* bsplit_k = nullptr;
    __nv_bfloat16* bsplit_v = nullptr;
    float* sigma_k = nullptr;
    float* sigma_v = nullptr;
    float* pend_k = nullptr;
    float* pend_v = nullptr;
    float* qscr_k = nullptr;      // fold scratch: Q of every (layer, head)
    float* qscr_v = nullptr;
    int* seg_rows = nullptr;
    // latent-channel codes (coef_quant): codes, scales and the fold's fp32 new rows
    uint32_t* qcodes_k = nullptr;
    uint32_t* qcodes_v = nullptr;
    float* qscales_k = nullptr;
    float* qscales_v = nullptr;
    float* newrows_k = nullptr;
    float* newrows_v = nullptr;
    float* wide = nullptr;        // joint-head fold scratch: K's, then V's
    size_t wide_floats = 0;       // floats of one of the two
    __nv_bfloat16* qws_k = nullptr;   // coded caches: one layer's coefficients as bf16
    __nv_bfloat16* qws_v = nullptr;   // (the tensor-core decode's workspace)
    float* partial = nullptr;
    int* done = nullptr;          // per-head arrival counters of the fused decode combine
    float2* rope = nullptr;
    __half* ptab = nullptr;       // fp16 position table (decode_u): factor rows j at
                                  // P + j, then the protected positions 0 .. P - 1
    int64_t ptab_rows = 0;        // rows of the factor-row part
    uint32_t* aq = nullptr;       // per-call query-basis products of every head (decode_u)
    int* status = nullptr;
    void* stage_in = nullptr;     // host-input staging
    size_t stage_in_bytes = 0;
    float* stage_out = nullptr;   // host-output staging
    size_t stage_out_bytes = 0;
    int max_splits = 256;
    bool use_tc = true;           // tensor-core paths for bf16 coefficients
    int use_u = 2;                // query-side RoPE decode: 0 never, 1 wherever it applies,
                                  // 2 where a call gives each SM enough folded tiles
    int sms = 148;
    // clock cycles a tensor-core pipeline wait may take before the call gives
    // up with DEVICE_TIMEOUT; tests shorten it through the environment to make
    // the wait run out on purpose (ISKV_TEST_PIPELINE_WAIT_CYCLES)
    long long pipe_wait = tc::kWaitCycles;
    // host counters
    std::vector<int64_t> T, n_c;
    std::vector<int> n_pend;
    // asynchronous block updates (iskv_compress_block_async): per layer, the
    // event that completes the layer's last update and whether the next call
    // touching the layer has yet to order its stream after it
    std::vector<cudaEvent_t> upd_evt;
    std::vector<char> upd_wait;
    cudaEvent_t enq_evt = nullptr;   // orders an update's stream after the caller's
    // the V fold of a compress call runs on this stream beside the K fold
    cudaStream_t fold_side = nullptr;
    cudaEvent_t fork_evt = nullptr, join_evt = nullptr;
    DecodeGridPlan grid_plan;        // the last decode grid, reused while its shape holds
};

namespace {

// One NVTX range per API call (a no-op unless a profiler is attached).
struct TraceRange {
    explicit TraceRange(const char* name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
};

constexpr size_t kStageBytes = 16u << 20;
constexpr bool kDecodeTcDefault = true;
// The query-side RoPE decode pays a fixed cost per CTA and head (building the
// head's query-basis products) and keeps four stages instead of six; same-box
// A/B (one layer, 8 KV / 32 query heads) put it ahead from about 200 folded
// tiles per SM (batch 8 at 64K: -4 %; batch 32 at 64K: -17 %) and behind
// below (batch 8 at 32K: +7 %; batch 1 at 128K: +28 %).
constexpr int64_t kDecodeUMinTilesPerSm = 200;

// Fill the code-format fields of a view from `q` for rank r; false if the
// format is invalid (groups 1..4, channels multiples of 16 summing to r, bits
// 0, 2, 4 or 8, at least one group with codes).
bool quant_fill(const iskv_quant_format& q, int r, FactorView* f) {
    if (q.groups < 1 || q.groups > 4) return false;
    int lo = 0, word = 0, coded = 0;
    for (int g = 0; g < 4; ++g) {
        f->qbits[g] = 0;
        f->qlo[g] = f->qhi[g] = r;
        f->qword0[g] = 0;
    }
    for (int g = 0; g < q.groups; ++g) {
        const int n = q.channels[g], b = q.bits[g];
        if (n < 16 || n % 16 != 0 || !(b == 0 || b == 2 || b == 4 || b == 8)) return false;
        f->qbits[g] = b;
        f->qlo[g] = lo;
        f->qhi[g] = lo + n;
        f->qword0[g] = word;
        lo += n;
        word += n * b / 32;
        coded += b > 0;
    }
    if (lo != r || coded == 0) return false;
    f->qgroups = q.groups;
    f->qwords = word;
    return true;
}

// The address at which this device's kernels may dereference caller buffer
// p: p itself for memory of the current device or managed memory, the mapped
// address for page-locked host memory (*mapped = true), nullptr for pageable
// host memory and for another GPU's memory (both staged with cudaMemcpyAsync,
// which also copies between peers).
const void* kernel_addr(const void* p, bool* mapped = nullptr) {
    if (mapped) *mapped = false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (at.type == cudaMemoryTypeManaged) return p;
    if (at.type == cudaMemoryTypeDevice) {
        int dev = -1;
        if (cudaGetDevice(&dev) != cudaSuccess || at.device != dev) return nullptr;
        return p;
    }
    if (at.type == cudaMemoryTypeHost && at.devicePointer != nullptr) {
        if (mapped) *mapped = true;
        return at.devicePointer;
    }
    return nullptr;
}

// memory of the current device (or managed): read and written by kernels as is
bool is_device_ptr(const void* p) {
    bool mapped;
    return kernel_addr(p, &mapped) != nullptr && !mapped;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int validate(const iskv_config* c) {
    if (!c) return ISKV_ERR_INVALID_ARG;
    if (c->batch < 1 || c->layers < 1 || c->layers > kMaxLayers || c->kv_heads < 1 ||
        c->q_heads < 1 || c->q_heads % c->kv_heads != 0)
        return ISKV_ERR_INVALID_ARG;
    if (c->q_heads / c->kv_heads > kMaxGroup) return ISKV_ERR_UNSUPPORTED;
    if (c->head_dim != kHeadDim || c->block != kBlock) return ISKV_ERR_UNSUPPORTED;
    for (int r : {c->rank_k, c->rank_v})
        if (r < 16 || r > kHeadDim || r % 16 != 0) return ISKV_ERR_UNSUPPORTED;
    if (c->window < 0 || c->window % kBlock != 0 || c->max_tokens < 1) return ISKV_ERR_INVALID_ARG;
    if ((c->kv_dtype != ISKV_F32 && c->kv_dtype != ISKV_BF16) ||
        (c->coef_dtype != ISKV_F32 && c->coef_dtype != ISKV_BF16))
        return ISKV_ERR_INVALID_ARG;
    if (c->use_rope != 0 && c->use_rope != 1) return ISKV_ERR_INVALID_ARG;
    if (c->use_rope && !(c->rope_theta > 1.0)) return ISKV_ERR_INVALID_ARG;
    if (c->sync != 0 && c->sync != 1) return ISKV_ERR_INVALID_ARG;
    if (c->max_deferred < 0 || c->max_deferred > kMaxDeferred) return ISKV_ERR_INVALID_ARG;
    if (c->jacobi_max_sweeps < 0 || c->jacobi_max_sweeps > 1000) return ISKV_ERR_INVALID_ARG;
    if (c->ring_extra < 0 || c->ring_extra % kBlock != 0) return ISKV_ERR_INVALID_ARG;
    if (c->protect < 0 || c->protect > c->max_tokens) return ISKV_ERR_INVALID_ARG;
    if (c->coef_quant != 0 && c->coef_quant != 1) return ISKV_ERR_INVALID_ARG;
    if (c->joint != 0 && c->joint != 1) return ISKV_ERR_INVALID_ARG;
    if (c->joint && (c->kv_heads * kHeadDim > 1024 || c->coef_quant)) return ISKV_ERR_UNSUPPORTED;
    if (c->coef_quant) {
        FactorView f{};
        if (!quant_fill(c->quant_k, c->rank_k, &f) || !quant_fill(c->quant_v, c->rank_v, &f))
            return ISKV_ERR_INVALID_ARG;
    }
    return ISKV_OK;
}

FactorView view(const iskv_cache* h, int which) {
    FactorView f{};
    const bool K = which == ISKV_WHICH_K;
    f.coef = K ? h->coef_k : h->coef_v;
    f.basis = K ? h->basis_k : h->basis_v;
    f.bsplit = K ? h->bsplit_k : h->bsplit_v;
    f.sigma = K ? h->sigma_k : h->sigma_v;
    f.pend = K ? h->pend_k : h->pend_v;
    f.seg_rows = h->seg_rows;   // identical for K and V: both fold together
    f.ring = K ? h->ring_k : h->ring_v;
    f.prot = K ? h->prot_k : h->prot_v;
    f.P = h->cfg.protect;
    f.pcap = h->pcap;
    f.r = K ? h->cfg.rank_k : h->cfg.rank_v;
    f.coef_bf16 = h->cfg.coef_dtype == ISKV_BF16;
    f.coef_blocked = f.coef_bf16;   // bf16 rows live in 8x8 core-matrix blocks
    f.kv_bf16 = h->cfg.kv_dtype == ISKV_BF16;
    f.ring_blocked = f.kv_bf16;     // and so do bf16 exact rows
    f.n_max = h->n_max;
    f.cap = h->cap;
    f.D = h->D;
    f.BH = h->BH;
    f.coef_div = h->cfg.joint ? h->cfg.kv_heads : 1;
    f.wide = h->wide ? h->wide + (which == ISKV_WHICH_V ? h->wide_floats : 0) : nullptr;
    if (h->cfg.coef_quant) {
        f.quant = 1;
        f.coef_bf16 = 0;
        f.coef_blocked = 0;
        quant_fill(K ? h->cfg.quant_k : h->cfg.quant_v, f.r, &f);
        f.qcodes = K ? h->qcodes_k : h->qcodes_v;
        f.qscales = K ? h->qscales_k : h->qscales_v;
        f.newrows = K ? h->newrows_k : h->newrows_v;
    }
    return f;
}

// The view of the per-factor arrays (coefficients, sigma, postponed W_top) with
// one instance per factor: kernels that never touch a head's basis rows or
// exact rows (rewrite, composition, coefficient copies) take this one.
FactorView view_factors(const iskv_cache* h, int which) {
    FactorView f = view(h, which);
    f.BH = h->FH;
    f.coef_div = 1;
    return f;
}

// rows of the layer's factor stream: the positions after the protected ones
int64_t factor_rows(const iskv_cache* h, int layer) {
    const int64_t tf = h->T[layer] - h->cfg.protect;
    return tf > 0 ? tf : 0;
}

int64_t ready_of(const iskv_cache* h, int layer) {
    const int64_t excess = factor_rows(h, layer) - h->n_c[layer] - h->cfg.window;
    return excess >= 0 ? excess / kBlock : 0;
}

#define CU(x)                                          \
    do {                                               \
        cudaError_t e_ = (x);                          \
        if (e_ != cudaSuccess) return ISKV_ERR_CUDA;   \
    } while (0)

void free_events(iskv_cache* h) {
    for (cudaEvent_t e : h->upd_evt)
        if (e) cudaEventDestroy(e);
    h->upd_evt.clear();
    if (h->enq_evt) cudaEventDestroy(h->enq_evt);
    h->enq_evt = nullptr;
    if (h->fork_evt) cudaEventDestroy(h->fork_evt);
    if (h->join_evt) cudaEventDestroy(h->join_evt);
    if (h->fold_side) cudaStreamDestroy(h->fold_side);
    h->fork_evt = h->join_evt = nullptr;
    h->fold_side = nullptr;
}

void free_all(iskv_cache* h) {
    free_events(h);
    void* ptrs[] = {h->ring_k, h->ring_v, h->prot_k, h->prot_v, h->coef_k, h->coef_v, h->basis_k, h->basis_v,
                    h->bsplit_k, h->bsplit_v, h->sigma_k, h->sigma_v, h->pend_k, h->pend_v,
                    h->qscr_k, h->qscr_v, h->seg_rows, h->partial, h->done, h->rope, h->status, h->stage_in, h->stage_out,
                    h->qcodes_k, h->qcodes_v, h->qscales_k, h->qscales_v, h->newrows_k, h->newrows_v,
                    h->wide, h->qws_k, h->qws_v, h->ptab, h->aq};
    for (void* p : ptrs)
        if (p) cudaFree(p);
}

template <typename T>
int dalloc(T** p, size_t bytes) {
    void* q = nullptr;
    if (bytes == 0) bytes = 16;
    if (cudaMalloc(&q, bytes) != cudaSuccess) {
        cudaGetLastError();
        return ISKV_ERR_NOMEM;
    }
    *p = reinterpret_cast<T*>(q);
    return ISKV_OK;
}

// The decode kernel of a layer's next decode call (iskv_decode_kernel): tensor
// cores for bf16 K/V with bf16 (or coded, expanded per call) coefficients and
// g in {1, 2, 4, 8}; among those the query-side RoPE kernel where r_K g <= 128
// and it is selected -- by ISKV_DECODE_KERNEL=u, or by default when the folded
// tiles of the call give every SM at least kDecodeUMinTilesPerSm -- else the
// rotation kernel.
int decode_path(const iskv_cache* h, int layer) {
    const iskv_config& c = h->cfg;
    const int g = c.q_heads / c.kv_heads;
    const bool coded_tc = c.coef_quant && h->qws_k != nullptr;
    if (!(h->use_tc && (coded_tc || (!c.coef_quant && c.coef_dtype == ISKV_BF16)) &&
          c.kv_dtype == ISKV_BF16 && decode_tc_supports_group(g)))
        return ISKV_DECODE_CUDA_CORE;
    if (h->use_u == 0 || h->ptab == nullptr || !decode_u_supports(g, c.rank_k)) return ISKV_DECODE_ROTATE;
    if (h->use_u == 1) return ISKV_DECODE_QUERY_ROPE;
    const int64_t tiles = (int64_t)h->BH * ((h->n_c[layer] + 127) / 128);
    return tiles >= kDecodeUMinTilesPerSm * h->sms ? ISKV_DECODE_QUERY_ROPE : ISKV_DECODE_ROTATE;
}

// A call on stream s that touches the listed layers runs after their last
// asynchronous update (the swap to the updated factors happens here, at the
// next call, not at the update's launch).  Callers keep every other call on
// one stream, so one wait per update suffices.
int order_after_updates(iskv_cache* h, const std::vector<int>& ls, cudaStream_t s) {
    for (int l : ls)
        if (h->upd_wait[l]) {
            if (cudaStreamWaitEvent(s, h->upd_evt[l], 0) != cudaSuccess) return ISKV_ERR_CUDA;
            h->upd_wait[l] = 0;
        }
    return ISKV_OK;
}

int order_after_update(iskv_cache* h, int layer, cudaStream_t s) {
    return order_after_updates(h, std::vector<int>{layer}, s);
}

// Layers named by a call: one, or all of them.
bool layers_of(const iskv_cache* h, int layer, std::vector<int>* out) {
    out->clear();
    if (layer == ISKV_ALL_LAYERS) {
        for (int l = 0; l < h->cfg.layers; ++l) out->push_back(l);
        return true;
    }
    if (layer < 0 || layer >= h->cfg.layers) return false;
    out->push_back(layer);
    return true;
}

// Rewrite the rows of the listed layers: compose postponed W_top, then the
// per-segment rewrite.  `nseg`, `rows` per listed layer.
int run_resync(iskv_cache* h, const std::vector<int>& layers, const std::vector<int>& nseg,
               const std::vector<int>& rows, cudaStream_t s) {
    ResyncLaunch rl{};
    for (size_t i = 0; i < layers.size(); ++i) {
        if (nseg[i] <= 0 || rows[i] <= 0) continue;
        rl.layer[rl.n_tasks] = layers[i];
        rl.n_seg[rl.n_tasks] = nseg[i];
        rl.n_rows[rl.n_tasks] = rows[i];
        ++rl.n_tasks;
    }
    if (rl.n_tasks == 0) return ISKV_OK;
    bool chained = false;
    for (int i = 0; i < rl.n_tasks; ++i) chained = chained || rl.n_seg[i] > 1;
    for (int which : {ISKV_WHICH_K, ISKV_WHICH_V}) {
        FactorView f = view_factors(h, which);
        if (chained) CU(launch_compose(f, rl, s));
        if (f.quant)
            CU(launch_resync_quant(f, rl, s));
        else if (f.coef_blocked)
            CU(launch_resync_tc(f, rl, h->status, s));
        else
            CU(launch_resync(f, rl, s));
    }
    return ISKV_OK;
}

}  // namespace

extern "C" {

int iskv_config_default(iskv_config* c) {
    if (!c) return ISKV_ERR_INVALID_ARG;
    std::memset(c, 0, sizeof(*c));
    c->batch = 1;
    c->layers = 1;
    c->kv_heads = 8;
    c->q_heads = 32;
    c->head_dim = kHeadDim;
    c->rank_k = 32;
    c->rank_v = 64;
    c->window = 1024;
    c->block = kBlock;
    c->max_tokens = 16384;
    c->kv_dtype = ISKV_BF16;
    c->coef_dtype = ISKV_F32;
    c->use_rope = 1;
    c->rope_theta = 1e6;
    c->sync = 1;
    c->max_deferred = 0;
    c->jacobi_max_sweeps = 0;
    c->ring_extra = 0;
    c->protect = 0;
    return ISKV_OK;
}

int iskv_create(const iskv_config* cfg, void* stream, iskv_t* out) {
    if (!out) return ISKV_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = validate(cfg);
    if (rc != ISKV_OK) return rc;
    iskv_cache* h = new (std::nothrow) iskv_cache();
    if (!h) return ISKV_ERR_NOMEM;
    h->cfg = *cfg;
    if (h->cfg.jacobi_max_sweeps == 0) h->cfg.jacobi_max_sweeps = 40;
    if (h->cfg.ring_extra == 0) h->cfg.ring_extra = kBlock;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaGetDevice(&h->device) != cudaSuccess) {
        delete h;
        return ISKV_ERR_CUDA;
    }
    const iskv_config& c = h->cfg;
    h->BH = c.batch * c.kv_heads;
    h->FH = c.joint ? c.batch : h->BH;
    h->cap = (int64_t)c.window + kBlock + c.ring_extra;
    h->pcap = ((int64_t)c.protect + kBlock - 1) / kBlock * kBlock;
    int64_t nm = (int64_t)c.max_tokens - c.window;
    if (nm < 0) nm = 0;
    h->n_max = (nm / kBlock) * kBlock + 2 * kBlock;   // slack rows for whole tiles
    h->D = c.max_deferred > 0 ? c.max_deferred : 1;
    h->kv_bytes = c.kv_dtype == ISKV_BF16 ? 2 : 4;
    h->coef_bytes = c.coef_quant ? 4 : (c.coef_dtype == ISKV_BF16 ? 2 : 4);   // as copied out
    {
        // tensor-core decode over folded rows: on unless ISKV_TENSOR_CORES=0
        const char* env = std::getenv("ISKV_TENSOR_CORES");
        h->use_tc = kDecodeTcDefault ? !(env && env[0] == '0') : (env && env[0] == '1');
        cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->device);
        // decode kernel for bf16 coefficient tiles: "rot" always the kernel that
        // rebuilds and rotates the keys, "u" the query-side RoPE kernel wherever
        // r_K g <= 128, unset a choice per call (decode_path)
        const char* dk = std::getenv("ISKV_DECODE_KERNEL");
        h->use_u = dk && std::strcmp(dk, "u") == 0 ? 1 : dk && std::strcmp(dk, "rot") == 0 ? 0 : 2;
        const char* w = std::getenv("ISKV_TEST_PIPELINE_WAIT_CYCLES");
        if (w && std::atoll(w) > 0) h->pipe_wait = std::atoll(w);
    }
    h->T.assign(c.layers, 0);
    h->n_c.assign(c.layers, 0);
    h->n_pend.assign(c.layers, 0);
    h->upd_wait.assign(c.layers, 0);
    h->upd_evt.assign(c.layers, nullptr);

    const size_t heads = (size_t)c.layers * h->BH;
    const size_t facs = (size_t)c.layers * h->FH;   // factor instances (coefficients, W_top)
    const size_t d = kHeadDim;
    size_t ring_bytes = heads * h->cap * d * h->kv_bytes;
    rc = ISKV_OK;
    for (int l = 0; l < c.layers && rc == ISKV_OK; ++l)
        if (cudaEventCreateWithFlags(&h->upd_evt[l], cudaEventDisableTiming) != cudaSuccess)
            rc = ISKV_ERR_CUDA;
    if (rc == ISKV_OK && cudaEventCreateWithFlags(&h->enq_evt, cudaEventDisableTiming) != cudaSuccess)
        rc = ISKV_ERR_CUDA;
    if (rc == ISKV_OK && (cudaEventCreateWithFlags(&h->fork_evt, cudaEventDisableTiming) != cudaSuccess ||
                          cudaEventCreateWithFlags(&h->join_evt, cudaEventDisableTiming) != cudaSuccess ||
                          cudaStreamCreateWithFlags(&h->fold_side, cudaStreamNonBlocking) != cudaSuccess))
        rc = ISKV_ERR_CUDA;
    rc = rc ? rc : dalloc(&h->ring_k, ring_bytes);
    rc = rc ? rc : dalloc(&h->ring_v, ring_bytes);
    const size_t prot_bytes = heads * h->pcap * d * h->kv_bytes;
    if (prot_bytes > 0) {
        rc = rc ? rc : dalloc(&h->prot_k, prot_bytes);
        rc = rc ? rc : dalloc(&h->prot_v, prot_bytes);
    }
    const size_t coef_k_bytes = c.coef_quant ? 0 : facs * h->n_max * c.rank_k * h->coef_bytes;
    const size_t coef_v_bytes = c.coef_quant ? 0 : facs * h->n_max * c.rank_v * h->coef_bytes;
    rc = rc ? rc : dalloc(&h->coef_k, coef_k_bytes);
    rc = rc ? rc : dalloc(&h->coef_v, coef_v_bytes);
    size_t qk_bytes = 0, qv_bytes = 0, qs_bytes = 0;
    if (c.coef_quant) {
        FactorView fk{}, fv{};
        quant_fill(c.quant_k, c.rank_k, &fk);
        quant_fill(c.quant_v, c.rank_v, &fv);
        qk_bytes = heads * h->n_max * fk.qwords * 4;
        qv_bytes = heads * h->n_max * fv.qwords * 4;
        qs_bytes = heads * h->n_max * 4 * sizeof(float);
        rc = rc ? rc : dalloc(&h->qcodes_k, qk_bytes);
        rc = rc ? rc : dalloc(&h->qcodes_v, qv_bytes);
        rc = rc ? rc : dalloc(&h->qscales_k, qs_bytes);
        rc = rc ? rc : dalloc(&h->qscales_v, qs_bytes);
        rc = rc ? rc : dalloc(&h->newrows_k, heads * kBlock * c.rank_k * sizeof(float));
        rc = rc ? rc : dalloc(&h->newrows_v, heads * kBlock * c.rank_v * sizeof(float));
        if (c.kv_dtype == ISKV_BF16) {   // the tensor-core decode reads codes expanded per call
            rc = rc ? rc : dalloc(&h->qws_k, (size_t)h->BH * h->n_max * c.rank_k * 2);
            rc = rc ? rc : dalloc(&h->qws_v, (size_t)h->BH * h->n_max * c.rank_v * 2);
            if (rc == ISKV_OK &&
                (cudaMemsetAsync(h->qws_k, 0, (size_t)h->BH * h->n_max * c.rank_k * 2, s) != cudaSuccess ||
                 cudaMemsetAsync(h->qws_v, 0, (size_t)h->BH * h->n_max * c.rank_v * 2, s) != cudaSuccess))
                rc = ISKV_ERR_CUDA;
        }
    }
    rc = rc ? rc : dalloc(&h->basis_k, heads * d * c.rank_k * 4);
    rc = rc ? rc : dalloc(&h->basis_v, heads * d * c.rank_v * 4);
    rc = rc ? rc : dalloc(&h->bsplit_k, heads * 2 * d * c.rank_k * 2);
    rc = rc ? rc : dalloc(&h->bsplit_v, heads * 2 * d * c.rank_v * 2);
    rc = rc ? rc : dalloc(&h->sigma_k, heads * c.rank_k * 4);
    rc = rc ? rc : dalloc(&h->sigma_v, heads * c.rank_v * 4);
    rc = rc ? rc : dalloc(&h->pend_k, facs * h->D * (size_t)c.rank_k * c.rank_k * 4);
    rc = rc ? rc : dalloc(&h->pend_v, facs * h->D * (size_t)c.rank_v * c.rank_v * 4);
    rc = rc ? rc : dalloc(&h->qscr_k, c.joint ? 0 : heads * d * fold_q_cols(c.rank_k) * 4);
    rc = rc ? rc : dalloc(&h->qscr_v, c.joint ? 0 : heads * d * fold_q_cols(c.rank_v) * 4);
    if (c.joint) {   // K's and V's scratch: their folds run side by side
        h->wide_floats = facs * fold_wide_scratch_floats(c.kv_heads * kHeadDim, std::max(c.rank_k, c.rank_v));
        rc = rc ? rc : dalloc(&h->wide, 2 * h->wide_floats * 4);
    }
    rc = rc ? rc : dalloc(&h->seg_rows, (size_t)c.layers * h->D * 4);
    rc = rc ? rc : dalloc(&h->partial, (size_t)c.batch * c.q_heads * h->max_splits *
                                           (2 + c.rank_v + d) * 4);
    rc = rc ? rc : dalloc(&h->status, 16);
    rc = rc ? rc : dalloc(&h->done, (size_t)h->BH * 4);
    h->stage_in_bytes = kStageBytes;
    h->stage_out_bytes = kStageBytes;
    rc = rc ? rc : dalloc(&h->stage_in, h->stage_in_bytes);
    rc = rc ? rc : dalloc(&h->stage_out, h->stage_out_bytes);
    if (rc == ISKV_OK && c.use_rope) {
        // at least 128 positions: the tensor-core decode reads the in-tile offsets 0..127
        const int64_t npos = c.max_tokens > 128 ? c.max_tokens : 128;
        rc = dalloc(&h->rope, (size_t)npos * (d / 2) * sizeof(float2));
        if (rc == ISKV_OK) {
            // cos/sin of pos * theta^(-2i/d), evaluated in double precision
            std::vector<float2> tab((size_t)npos * (d / 2));
            std::vector<double> inv(d / 2);
            for (size_t i = 0; i < d / 2; ++i) inv[i] = std::pow(c.rope_theta, -2.0 * (double)i / (double)d);
            for (int64_t p = 0; p < npos; ++p)
                for (size_t i = 0; i < d / 2; ++i) {
                    const double ang = (double)p * inv[i];
                    tab[p * (d / 2) + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
                }
            if (cudaMemcpy(h->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) !=
                cudaSuccess)
                rc = ISKV_ERR_CUDA;
        }
    }
    if (rc == ISKV_OK && c.kv_dtype == ISKV_BF16 && (c.coef_quant || c.coef_dtype == ISKV_BF16)) {
        // the query-side RoPE decode's table: coefficient row j sits at position
        // P + j; 128 fp16 per row (cos, sin of each frequency, interleaved) in
        // 8 x 8 blocks, 8-row groups outermost, so a 128-row tile is contiguous
        // rows: every factor position a folded or window row can take; a second
        // table holds the protected positions 0 .. P - 1 (rounded up to 64)
        const int64_t rows = std::max<int64_t>(h->n_max, (c.max_tokens + 63) / 64 * 64 + 128);
        const int64_t prows = (c.protect + 63) / 64 * 64;
        h->ptab_rows = rows;
        rc = dalloc(&h->ptab, (size_t)(rows + prows) * 128 * sizeof(__half));
        rc = rc ? rc : dalloc(&h->aq, (size_t)h->BH * 128 * 64 * sizeof(uint32_t));
        if (rc == ISKV_OK) {
            std::vector<__half> tab((size_t)(rows + prows) * 128);
            std::vector<double> inv(d / 2);
            for (size_t i = 0; i < d / 2; ++i) inv[i] = std::pow(c.rope_theta, -2.0 * (double)i / (double)d);
            for (int64_t j = 0; j < rows + prows; ++j) {
                const int64_t pos = j < rows ? c.protect + j : j - rows;
                for (int i = 0; i < d / 2; ++i) {
                    const double ang = (double)pos * inv[i];
                    const float cs = c.use_rope ? (float)std::cos(ang) : 1.f;
                    const float sn = c.use_rope ? (float)std::sin(ang) : 0.f;
                    tab[tc::blocked8(j, 2 * i, 128)] = __float2half_rn(cs);
                    tab[tc::blocked8(j, 2 * i + 1, 128)] = __float2half_rn(sn);
                }
            }
            if (cudaMemcpy(h->ptab, tab.data(), tab.size() * sizeof(__half), cudaMemcpyHostToDevice) !=
                cudaSuccess)
                rc = ISKV_ERR_CUDA;
        }
    }
    if (rc == ISKV_OK) {
        if (cudaMemsetAsync(h->ring_k, 0, ring_bytes, s) != cudaSuccess ||
            cudaMemsetAsync(h->ring_v, 0, ring_bytes, s) != cudaSuccess ||
            (prot_bytes > 0 && (cudaMemsetAsync(h->prot_k, 0, prot_bytes, s) != cudaSuccess ||
                                cudaMemsetAsync(h->prot_v, 0, prot_bytes, s) != cudaSuccess)) ||
            (coef_k_bytes > 0 && cudaMemsetAsync(h->coef_k, 0, coef_k_bytes, s) != cudaSuccess) ||
            (coef_v_bytes > 0 && cudaMemsetAsync(h->coef_v, 0, coef_v_bytes, s) != cudaSuccess) ||
            (qk_bytes > 0 && (cudaMemsetAsync(h->qcodes_k, 0, qk_bytes, s) != cudaSuccess ||
                              cudaMemsetAsync(h->qcodes_v, 0, qv_bytes, s) != cudaSuccess ||
                              cudaMemsetAsync(h->qscales_k, 0, qs_bytes, s) != cudaSuccess ||
                              cudaMemsetAsync(h->qscales_v, 0, qs_bytes, s) != cudaSuccess)) ||
            cudaMemsetAsync(h->status, 0, 16, s) != cudaSuccess ||
            cudaMemsetAsync(h->done, 0, (size_t)h->BH * 4, s) != cudaSuccess ||
            cudaMemsetAsync(h->seg_rows, 0, (size_t)c.layers * h->D * 4, s) != cudaSuccess ||
            launch_init_factor(view(h, ISKV_WHICH_K), c.layers, s) != cudaSuccess ||
            launch_init_factor(view(h, ISKV_WHICH_V), c.layers, s) != cudaSuccess)
            rc = ISKV_ERR_CUDA;
    }
    if (rc != ISKV_OK) {
        free_all(h);
        delete h;
        return rc;
    }
    *out = h;
    return ISKV_OK;
}

int iskv_destroy(iskv_t h) {
    if (!h) return ISKV_OK;
    cudaDeviceSynchronize();
    free_all(h);
    delete h;
    return ISKV_OK;
}

int iskv_append(iskv_t h, int layer, const void* k, const void* v, int t, void* stream,
                int* ready_blocks) {
    TraceRange trace_("iskv_append");
    if (!h || !k || !v || t < 0 || layer < 0 || layer >= h->cfg.layers) return ISKV_ERR_INVALID_ARG;
    const int64_t T1 = h->T[layer] + t;
    const int64_t P = h->cfg.protect;
    {
        const int rc = order_after_update(h, layer, reinterpret_cast<cudaStream_t>(stream));
        if (rc != ISKV_OK) return rc;
    }
    const int64_t tf1 = T1 > P ? T1 - P : 0;   // factor-stream rows after the call
    if (T1 > h->cfg.max_tokens || tf1 - h->n_c[layer] > h->cap) return ISKV_ERR_CAPACITY;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (t > 0) {
        const size_t row_bytes = (size_t)kHeadDim * h->kv_bytes;
        const size_t head_stride = (size_t)h->cap * row_bytes;
        const size_t prot_stride = (size_t)h->pcap * row_bytes;
        char* rk = reinterpret_cast<char*>(h->ring_k) + (size_t)layer * h->BH * head_stride;
        char* rv = reinterpret_cast<char*>(h->ring_v) + (size_t)layer * h->BH * head_stride;
        char* pk = h->prot_k ? reinterpret_cast<char*>(h->prot_k) + (size_t)layer * h->BH * prot_stride : nullptr;
        char* pv = h->prot_v ? reinterpret_cast<char*>(h->prot_v) + (size_t)layer * h->BH * prot_stride : nullptr;
        const void* srcs[2] = {k, v};
        char* rings[2] = {rk, rv};
        char* prots[2] = {pk, pv};
        const int blocked = h->cfg.kv_dtype == ISKV_BF16;
        // n rows of src ([BH][src_t][d], from src_row0) at absolute positions
        // pos0..: those below P to the protected rows, the rest to the ring at
        // factor position (pos - P)
        auto place = [&](int w, const void* src, int n, int src_t, int src_row0, int64_t pos0) -> int {
            const int np = (int)std::max<int64_t>(0, std::min<int64_t>(pos0 + n, P) - pos0);
            if (np > 0)
                CU(launch_append(prots[w], src, h->BH, np, src_t, src_row0, pos0, h->pcap, h->kv_bytes,
                                 blocked, s));
            if (n > np)
                CU(launch_append(rings[w], src, h->BH, n - np, src_t, src_row0 + np, pos0 + np - P, h->cap,
                                 h->kv_bytes, blocked, s));
            return ISKV_OK;
        };
        for (int w = 0; w < 2; ++w) {
            // device memory and mapped page-locked host memory are read in place
            // by the append kernel (16-byte vectors); everything else is staged
            const void* src = kernel_addr(srcs[w]);
            if (src != nullptr && aligned16(src)) {
                const int rc = place(w, src, t, t, 0, h->T[layer]);
                if (rc != ISKV_OK) return rc;
            } else {
                // stage token chunks of every (sequence, head) through device memory
                const int chunk = (int)std::max<size_t>(1, h->stage_in_bytes / ((size_t)h->BH * row_bytes));
                for (int t0 = 0; t0 < t; t0 += chunk) {
                    const int n = std::min(chunk, t - t0);
                    CU(cudaMemcpy2DAsync(h->stage_in, n * row_bytes,
                                         reinterpret_cast<const char*>(srcs[w]) + t0 * row_bytes,
                                         (size_t)t * row_bytes, n * row_bytes, h->BH,
                                         cudaMemcpyDefault, s));
                    const int rc = place(w, h->stage_in, n, n, 0, h->T[layer] + t0);
                    if (rc != ISKV_OK) return rc;
                }
            }
        }
    }
    h->T[layer] = T1;
    if (ready_blocks) *ready_blocks = (int)ready_of(h, layer);
    return ISKV_OK;
}

namespace {

// Fold (and rewrite) the ready blocks of the listed layers on stream s; the
// layers that were folded go to *folded.
int compress_on(iskv_cache* h, const std::vector<int>& ls, int flags, cudaStream_t s,
                std::vector<int>* folded) {
    const bool want_defer = (flags & ISKV_FOLD_DEFER_SYNC) != 0;
    FoldLaunch fl{};
    fl.max_sweeps = h->cfg.jacobi_max_sweeps;
    std::vector<int> fold_layers;
    for (int l : ls) {
        if (ready_of(h, l) < 1) continue;
        fold_layers.push_back(l);
    }
    if (fold_layers.empty()) return ISKV_ERR_STATE;
    // every layer of this call postpones if asked to, or if it already has
    // postponed folds (their rewrites must come first, in order)
    for (int l : fold_layers) {
        const bool defer = h->cfg.sync && (want_defer || h->n_pend[l] > 0);
        if (defer && h->n_pend[l] >= h->D) return ISKV_ERR_STATE;
        if (defer && h->cfg.max_deferred == 0 && want_defer) return ISKV_ERR_STATE;
    }
    for (int l : fold_layers) {
        const bool defer = h->cfg.sync && (want_defer || h->n_pend[l] > 0);
        fl.layer[fl.n_tasks] = l;
        fl.n_c[fl.n_tasks] = (int)h->n_c[l];
        fl.slot[fl.n_tasks] = defer ? h->n_pend[l] : 0;
        ++fl.n_tasks;
    }
    // the K and V folds share nothing: V's runs on the side stream, forked from
    // and joined back into s, so small launches (few heads) fill the GPU together
    CU(cudaEventRecord(h->fork_evt, s));
    CU(cudaStreamWaitEvent(h->fold_side, h->fork_evt, 0));
    for (int which : {ISKV_WHICH_K, ISKV_WHICH_V}) {
        cudaStream_t fs = which == ISKV_WHICH_K ? s : h->fold_side;
        fl.qscratch = which == ISKV_WHICH_K ? h->qscr_k : h->qscr_v;
        const FactorView f = view(h, which);
        if (h->cfg.joint)
            CU(launch_fold_wide(f, fl, h->status, fs));
        else
            CU(launch_fold(f, fl, h->status, fs));
        if (f.quant) CU(launch_quant_new_rows(f, fl, fs));   // the block's rows, coded
    }
    CU(cudaEventRecord(h->join_evt, h->fold_side));
    CU(cudaStreamWaitEvent(s, h->join_evt, 0));
    std::vector<int> rl_layers, rl_seg, rl_rows;
    for (int l : fold_layers) {
        const bool defer = h->cfg.sync && (want_defer || h->n_pend[l] > 0);
        const int64_t old = h->n_c[l];
        h->n_c[l] += kBlock;
        if (!h->cfg.sync) continue;
        if (defer) {
            h->n_pend[l] += 1;
            if (!want_defer) {   // finish the postponed chain now
                rl_layers.push_back(l);
                rl_seg.push_back(h->n_pend[l]);
                rl_rows.push_back((int)old);
                h->n_pend[l] = 0;
            }
        } else if (old > 0) {
            rl_layers.push_back(l);
            rl_seg.push_back(1);
            rl_rows.push_back((int)old);
        }
    }
    *folded = fold_layers;
    return run_resync(h, rl_layers, rl_seg, rl_rows, s);
}

}  // namespace

int iskv_compress_block(iskv_t h, int layer, int flags, void* stream) {
    TraceRange trace_("iskv_compress_block");
    if (!h || (flags & ~ISKV_FOLD_DEFER_SYNC)) return ISKV_ERR_INVALID_ARG;
    std::vector<int> ls, folded;
    if (!layers_of(h, layer, &ls)) return ISKV_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int rc = order_after_updates(h, ls, s);
    return rc != ISKV_OK ? rc : compress_on(h, ls, flags, s, &folded);
}

int iskv_compress_block_async(iskv_t h, int layer, int flags, void* stream, void* after) {
    TraceRange trace_("iskv_compress_block_async");
    if (!h || (flags & ~ISKV_FOLD_DEFER_SYNC)) return ISKV_ERR_INVALID_ARG;
    std::vector<int> ls, folded;
    if (!layers_of(h, layer, &ls)) return ISKV_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the update sees everything enqueued so far on `after` (the appended rows)
    // and runs after the layers' earlier updates
    CU(cudaEventRecord(h->enq_evt, reinterpret_cast<cudaStream_t>(after)));
    CU(cudaStreamWaitEvent(s, h->enq_evt, 0));
    int rc = order_after_updates(h, ls, s);
    if (rc == ISKV_OK) rc = compress_on(h, ls, flags, s, &folded);
    if (rc != ISKV_OK) return rc;
    for (int l : folded) {
        CU(cudaEventRecord(h->upd_evt[l], s));
        h->upd_wait[l] = 1;
    }
    return ISKV_OK;
}

int iskv_sync(iskv_t h, int layer, void* stream) {
    TraceRange trace_("iskv_sync");
    if (!h) return ISKV_ERR_INVALID_ARG;
    std::vector<int> ls;
    if (!layers_of(h, layer, &ls)) return ISKV_ERR_INVALID_ARG;
    {
        const int rc = order_after_updates(h, ls, reinterpret_cast<cudaStream_t>(stream));
        if (rc != ISKV_OK) return rc;
    }
    std::vector<int> rl_layers, rl_seg, rl_rows;
    for (int l : ls) {
        if (h->n_pend[l] == 0) continue;
        rl_layers.push_back(l);
        rl_seg.push_back(h->n_pend[l]);
        rl_rows.push_back((int)(h->n_c[l] - kBlock));
        h->n_pend[l] = 0;
    }
    return run_resync(h, rl_layers, rl_seg, rl_rows, reinterpret_cast<cudaStream_t>(stream));
}

int iskv_decode_attention(iskv_t h, int layer, const void* q, float* out, void* stream) {
    TraceRange trace_("iskv_decode_attention");
    if (!h || !q || !out || layer < 0 || layer >= h->cfg.layers) return ISKV_ERR_INVALID_ARG;
    if (h->T[layer] == 0 || h->n_pend[layer] > 0) return ISKV_ERR_STATE;
    const iskv_config& c = h->cfg;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    {
        const int rc = order_after_update(h, layer, s);
        if (rc != ISKV_OK) return rc;
    }
    const size_t q_bytes = (size_t)c.batch * c.q_heads * kHeadDim * h->kv_bytes;
    const size_t o_bytes = (size_t)c.batch * c.q_heads * kHeadDim * sizeof(float);
    const void* qd = q;
    // host queries, or device queries off the 16-byte alignment of the bulk
    // copies that fetch them, go through the staging buffer: by a copy kernel
    // from mapped page-locked memory, else by cudaMemcpyAsync
    bool q_mapped = false;
    const void* qk = kernel_addr(q, &q_mapped);
    if (qk == nullptr || q_mapped || !aligned16(qk)) {
        if (q_bytes > h->stage_in_bytes) return ISKV_ERR_UNSUPPORTED;
        if (q_mapped && aligned16(qk)) CU(launch_copy_vec(h->stage_in, qk, q_bytes, s));
        else CU(cudaMemcpyAsync(h->stage_in, q, q_bytes, cudaMemcpyDefault, s));
        qd = h->stage_in;
    }
    // device memory and mapped page-locked memory take the kernels' 4-byte
    // stores of the result in place; anything else gets it through the
    // staging buffer and cudaMemcpyAsync
    void* ok = const_cast<void*>(kernel_addr(out));
    const bool host_out = ok == nullptr || (reinterpret_cast<uintptr_t>(ok) & 3) != 0;
    if (host_out && o_bytes > h->stage_out_bytes) return ISKV_ERR_UNSUPPORTED;
    float* od = host_out ? h->stage_out : static_cast<float*>(ok);
    auto copy_out = [&]() { return cudaMemcpyAsync(out, od, o_bytes, cudaMemcpyDefault, s); };

    DecodeArgs a{};
    a.K = view(h, ISKV_WHICH_K);
    a.V = view(h, ISKV_WHICH_V);
    a.q = qd;
    a.partial = h->partial;
    a.rope = c.use_rope ? h->rope : nullptr;
    a.layer = layer;
    a.B = c.batch;
    a.Hkv = c.kv_heads;
    a.Hq = c.q_heads;
    a.g = c.q_heads / c.kv_heads;
    a.T = h->T[layer];
    a.n_c = h->n_c[layer];
    a.scale = 1.0f / std::sqrt((float)kHeadDim);
    const int sms = h->sms;
    const bool coded_tc = c.coef_quant && h->qws_k != nullptr;
    const int path = decode_path(h, layer);
    if (path != ISKV_DECODE_CUDA_CORE) {
        // one persistent tensor-core kernel, one CTA per SM, over the flattened
        // (head, tile) space: 128-token tiles of folded rows, then 64-token
        // tiles of exact rows, all under one online softmax per head
        DecodeTcArgs t{};
        t.K = a.K;
        t.V = a.V;
        if (coded_tc) {
            // coded coefficients: this layer's rows expanded to bf16 tiles in the
            // workspace, then the same tensor-core decode
            CU(launch_expand_codes(a.K, layer, a.n_c, h->qws_k, s));
            CU(launch_expand_codes(a.V, layer, a.n_c, h->qws_v, s));
            for (FactorView* f : {&t.K, &t.V}) {
                f->coef = f == &t.K ? (void*)h->qws_k : (void*)h->qws_v;
                f->quant = 0;
                f->coef_bf16 = 1;
                f->coef_blocked = 1;
                f->coef_ws = 1;
            }
        }
        t.q = qd;
        t.partial = h->partial;
        t.rope = a.rope;
        t.status = h->status;
        t.out = od;
        t.done = h->done;
        t.layer = layer;
        t.B = c.batch;
        t.Hkv = c.kv_heads;
        t.Hq = c.q_heads;
        t.g = a.g;
        t.n_c = a.n_c;
        t.T = a.T;
        t.scale = a.scale;
        t.pipe_wait = h->pipe_wait;
        t.idle_hint_ns = h->pipe_wait < tc::kWaitCycles ? 0u : 20000u;
        t.ptab = h->ptab;
        t.ptab_rows = h->ptab_rows;
        t.aq = h->aq;
        const int64_t coef_tile = (int64_t)128 * (c.rank_k + c.rank_v) * 2;
        // query-side RoPE kernel where U (r_K g columns) fits one TMEM buffer
        const bool use_u = path == ISKV_DECODE_QUERY_ROPE;
        t.stages = 0;
        if (use_u) {
            // exact tiles also stage their rows' fp16 RoPE table: 3 x wt rows of 256 bytes
            t.win_rows = 3 * 64 * kHeadDim * 2 > coef_tile ? 32 : 64;
            for (int ns = 6; ns >= 2 && t.stages == 0; --ns)
                if (decode_u_smem_bytes(c.rank_k, c.rank_v, ns, t.win_rows) <= 227 * 1024) t.stages = ns;
            t.basis_bufs = 1;
            t.q_bufs = 1;
        } else {
            // deepest pipeline that fits for exact-row tiles of wt rows: stages
            // first, then two basis buffers, then double-buffered q'
            struct Fit { int ns = 0, nbk = 0, nqb = 0; };
            auto fit = [&](int wt) {
                Fit f;
                for (int ns = 6; ns >= 2 && f.ns == 0; --ns)
                    for (int nbk = 2; nbk >= 1 && f.ns == 0; --nbk)
                        for (int nqb = 2; nqb >= 1; --nqb)
                            if (decode_tc_smem_bytes(c.rank_k, c.rank_v, ns, nbk, nqb, wt) <= 227 * 1024) {
                                f = Fit{ns, nbk, nqb};
                                break;
                            }
                return f;
            };
            // exact-row tiles of 64 rows unless that costs a basis or q' buffer, or
            // more than the stages down to four, against 32-row tiles (a same-box
            // A/B at r_K 32, r_V 64: 64-row tiles and five stages 142 us against
            // 32-row tiles and six stages 151 us: half as many exact tiles, each a
            // full pass of the epilogue's per-tile chain)
            const Fit f64 = fit(64), f32 = fit(32);
            const bool wide = f64.ns > 0 && f64.nbk == f32.nbk && f64.nqb == f32.nqb &&
                              f64.ns >= std::min(f32.ns, 4);
            const Fit f = wide ? f64 : f32;
            t.win_rows = wide ? 64 : 32;
            t.stages = f.ns;
            t.basis_bufs = f.nbk;
            t.q_bufs = f.nqb;
        }
        if (t.stages == 0) return ISKV_ERR_UNSUPPORTED;
        const int wt = t.win_rows;
        const int64_t P = c.protect, Pe = std::min<int64_t>(a.T, P);
        t.tiles_c = (int)((a.n_c + 127) / 128);
        t.tiles_w = (int)((factor_rows(h, layer) - a.n_c + wt - 1) / wt);
        t.tiles_per_head = t.tiles_c + t.tiles_w + (int)((Pe + wt - 1) / wt);
        t.total_tiles = (int64_t)h->BH * t.tiles_per_head;
        // each CTA publishes two partials (one per epilogue group) for every head
        // it visits; fewer CTAs when a head would span more slots than the
        // partial buffer holds (few heads, long context)
        const int ncta = (int)std::min<int64_t>(std::min(sms, kDecodeMaxCtas), t.total_tiles);
        // partial slots per query head: the buffer's, and the merge scratch's
        // (slots x g <= 512 per q' buffer of a group; 512 for the query-side kernel)
        const int cap_slots = std::min(h->max_splits, 512 * t.q_bufs / a.g);
        if (!plan_decode_grid(t.total_tiles, t.tiles_per_head, h->BH, ncta, cap_slots, 2, &h->grid_plan))
            return ISKV_ERR_UNSUPPORTED;
        t.ncta = h->grid_plan.nruns;
        std::copy(h->grid_plan.start.begin(), h->grid_plan.start.begin() + t.ncta + 1, t.cta_start);
        const int slots_c = h->grid_plan.slots;
        t.slots_c = slots_c;
        t.splits_total = 2 * slots_c;
        if (t.stages == 0) return ISKV_ERR_UNSUPPORTED;
        if (use_u) CU(launch_decode_u(t, s));   // both merge the partials of each head
        else CU(launch_decode_tc(t, s));
        if (host_out) CU(copy_out());
        return ISKV_OK;
    }
    // split the token axis so that the grid covers the GPU several times
    const int64_t want = (int64_t)4 * sms;
    int64_t splits = (want + h->BH - 1) / h->BH;
    const int64_t max_by_tokens = (a.T + 63) / 64;
    if (splits > max_by_tokens) splits = max_by_tokens;
    if (splits > h->max_splits) splits = h->max_splits;
    if (splits < 1) splits = 1;
    int64_t tps = (a.T + splits - 1) / splits;
    tps = ((tps + 63) / 64) * 64;
    splits = (a.T + tps - 1) / tps;
    a.tokens_per_split = tps;
    a.splits = (int)splits;
    CU(launch_decode(a, s));
    CU(launch_combine(a, od, s));
    if (host_out) CU(copy_out());
    return ISKV_OK;
}

int iskv_reconstruct(iskv_t h, int layer, int which, float* out, void* stream) {
    TraceRange trace_("iskv_reconstruct");
    if (!h || layer < 0 || layer >= h->cfg.layers ||
        (which != ISKV_WHICH_K && which != ISKV_WHICH_V))
        return ISKV_ERR_INVALID_ARG;
    if (h->n_pend[layer] > 0) return ISKV_ERR_STATE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    {
        const int rc = order_after_update(h, layer, s);
        if (rc != ISKV_OK) return rc;
    }
    const FactorView f = view(h, which);
    const int64_t rows = h->n_c[layer];
    if (rows == 0) return ISKV_OK;   // nothing folded: an empty result
    if (!out) return ISKV_ERR_INVALID_ARG;
    if (is_device_ptr(out)) {
        CU(launch_reconstruct(f, layer, 0, rows, out, s));
        return ISKV_OK;
    }
    const size_t row_bytes = (size_t)kHeadDim * sizeof(float);
    int64_t chunk = (int64_t)(h->stage_out_bytes / (row_bytes * h->BH));
    chunk = (chunk / 64) * 64;
    if (chunk < 64) return ISKV_ERR_UNSUPPORTED;
    for (int64_t r0 = 0; r0 < rows; r0 += chunk) {
        const int64_t n = std::min(chunk, rows - r0);
        CU(launch_reconstruct(f, layer, r0, n, h->stage_out, s));
        CU(cudaMemcpy2DAsync(reinterpret_cast<char*>(out) + r0 * row_bytes, rows * row_bytes,
                             h->stage_out, n * row_bytes, n * row_bytes, h->BH, cudaMemcpyDefault, s));
    }
    return ISKV_OK;
}

int iskv_get_factors(iskv_t h, int layer, int which, float* basis, float* sigma, void* coef,
                     void* stream) {
    if (!h || layer < 0 || layer >= h->cfg.layers || (which != ISKV_WHICH_K && which != ISKV_WHICH_V))
        return ISKV_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    {
        const int rc = order_after_update(h, layer, s);
        if (rc != ISKV_OK) return rc;
    }
    const FactorView f = view_factors(h, which);
    const size_t heads = h->FH;   // factor instances: per head, or per sequence (joint)
    const int r = f.r;
    const size_t rows_b = (size_t)h->BH * kHeadDim;   // basis rows of the layer, either way
    if (basis)
        CU(cudaMemcpyAsync(basis, f.basis + (size_t)layer * rows_b * r, rows_b * r * sizeof(float),
                           cudaMemcpyDefault, s));
    if (sigma)
        CU(cudaMemcpyAsync(sigma, f.sigma + (size_t)layer * heads * r, heads * r * sizeof(float),
                           cudaMemcpyDefault, s));
    if (coef && h->n_c[layer] > 0) {
        const int64_t rows = h->n_c[layer];
        const size_t rb = (size_t)r * h->coef_bytes;
        if (is_device_ptr(coef)) {
            CU(launch_copy_coef(f, layer, 0, rows, coef, s));
        } else {
            int64_t chunk = (int64_t)(h->stage_out_bytes / (rb * heads));
            if (chunk < 1) return ISKV_ERR_UNSUPPORTED;
            for (int64_t r0 = 0; r0 < rows; r0 += chunk) {
                const int64_t n = std::min(chunk, rows - r0);
                CU(launch_copy_coef(f, layer, r0, n, h->stage_out, s));
                CU(cudaMemcpy2DAsync(reinterpret_cast<char*>(coef) + r0 * rb, rows * rb, h->stage_out,
                                     n * rb, n * rb, heads, cudaMemcpyDefault, s));
            }
        }
    }
    return ISKV_OK;
}

int iskv_decode_kernel(iskv_t h, int layer, int* kernel) {
    if (!h || !kernel || layer < 0 || layer >= h->cfg.layers) return ISKV_ERR_INVALID_ARG;
    *kernel = decode_path(h, layer);
    return ISKV_OK;
}

int iskv_kv_bytes(iskv_t h, int64_t* persistent_bytes, int64_t* full_bytes) {
    if (!h) return ISKV_ERR_INVALID_ARG;
    const iskv_config& c = h->cfg;
    const int64_t d = kHeadDim, rs = (int64_t)c.rank_k + c.rank_v;
    int64_t kept = 0, full = 0;
    for (int l = 0; l < c.layers; ++l) {
        const int64_t T = h->T[l], n_c = h->n_c[l];
        const int64_t exact = T - n_c;   // protected rows and the window
        int64_t per_head = 2 * exact * d * h->kv_bytes;
        int64_t row_bytes = rs * h->coef_bytes;   // one coefficient row of K and V
        if (c.coef_quant) {
            // codes, plus one fp32 scale per coded group
            FactorView fk{}, fv{};
            quant_fill(c.quant_k, c.rank_k, &fk);
            quant_fill(c.quant_v, c.rank_v, &fv);
            int64_t ng = 0;
            for (int g = 0; g < 4; ++g) ng += (fk.qbits[g] > 0) + (fv.qbits[g] > 0);
            row_bytes = (int64_t)(fk.qwords + fv.qwords) * 4 + ng * 4;
        }
        if (c.joint) {
            // coefficients, basis (D rows) and sigma once per sequence
            kept += per_head * h->BH;
            if (n_c > 0) kept += (n_c * row_bytes + (d * c.kv_heads + 1) * rs * 4) * h->FH;
            full += 2 * T * d * h->kv_bytes * h->BH;
            continue;
        }
        if (n_c > 0) per_head += n_c * row_bytes + (d + 1) * rs * 4;   // C; B and S in fp32
        kept += per_head * h->BH;
        full += 2 * T * d * h->kv_bytes * h->BH;
    }
    if (persistent_bytes) *persistent_bytes = kept;
    if (full_bytes) *full_bytes = full;
    return ISKV_OK;
}

int iskv_get_counts(iskv_t h, int layer, int64_t* T, int64_t* n_c) {
    if (!h || layer < 0 || layer >= h->cfg.layers) return ISKV_ERR_INVALID_ARG;
    if (T) *T = h->T[layer];
    if (n_c) *n_c = h->n_c[layer];
    return ISKV_OK;
}

int iskv_status(iskv_t h) {
    if (!h) return ISKV_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return ISKV_ERR_CUDA;
    int st = 0;
    if (cudaMemcpy(&st, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return ISKV_ERR_CUDA;
    if (st & tc::kStatusTimeout) return ISKV_ERR_DEVICE_TIMEOUT;
    if (st & kStatusRange) return ISKV_ERR_RANGE;
    if (st & kStatusNoConverge) return ISKV_ERR_NOCONVERGE;
    return ISKV_OK;
}

int iskv_quant_words(const iskv_quant_format* fmt) {
    if (!fmt) return -1;
    int r = 0;
    for (int g = 0; g < fmt->groups && g < 4; ++g) r += fmt->channels[g];
    FactorView f{};
    if (r < 16 || r > kHeadDim || !quant_fill(*fmt, r, &f)) return -1;
    return f.qwords;
}

int iskv_quantize_rows(const iskv_quant_format* fmt, int rank, const float* rows, int64_t n,
                       uint32_t* codes, float* scales, void* stream) {
    if (!fmt || n < 0 || rank < 16 || rank > kHeadDim) return ISKV_ERR_INVALID_ARG;
    FactorView f{};
    if (!quant_fill(*fmt, rank, &f)) return ISKV_ERR_INVALID_ARG;
    f.r = rank;
    if (n == 0) return ISKV_OK;
    if (!rows || !codes || !scales || !is_device_ptr(rows) || !is_device_ptr(codes) ||
        !is_device_ptr(scales))
        return ISKV_ERR_INVALID_ARG;
    CU(launch_quant_rows(f, rows, n, codes, scales, reinterpret_cast<cudaStream_t>(stream)));
    return ISKV_OK;
}

const char* iskv_strerror(int code) {
    switch (code) {
        case ISKV_OK: return "ok";
        case ISKV_ERR_INVALID_ARG: return "invalid argument";
        case ISKV_ERR_CAPACITY: return "capacity exceeded (max_tokens or exact-window ring)";
        case ISKV_ERR_STATE: return "invalid state (no ready block, empty cache, or pending rewrites)";
        case ISKV_ERR_CUDA: return "CUDA runtime error";
        case ISKV_ERR_NOCONVERGE: return "core SVD reached its sweep limit";
        case ISKV_ERR_NOMEM: return "device allocation failed";
        case ISKV_ERR_UNSUPPORTED: return "shape not supported by the compiled kernels";
        case ISKV_ERR_DEVICE_TIMEOUT: return "a device-side wait gave up; that call's results are incomplete";
        case ISKV_ERR_RANGE: return "a score of the tensor-core decode was not finite (fp16 range of its keys exceeded, or inf/NaN input)";
        default: return "unknown status";
    }
}

}  // extern "C"
