// Decode attention that allocates nothing: the caller passes every operand
// (its own buffers) and the split-K partial results live in one file-scope
// device array instead of memory obtained from cudaMalloc.
//
// Who needs this: programs whose device memory is planned and owned by a
// host framework -- for example a serving engine that reserves HBM for its
// KV pools at start-up and forbids later driver allocations -- and
// latency-critical paths that must not call cudaMalloc (it may synchronize
// the whole device).  Such callers cannot use iskv_create, which allocates
// the cache; they keep the factors in their own memory and call this.
//
// The scratch array is part of the library image: every GPU that loads the
// library holds it until the process exits.  In host code its name is only a
// host-side stand-in, so its device address is looked up once per device
// with cudaGetSymbolAddress (on the first call on that device) and passed to
// the kernels.  That address is kept for the life of the process: after a
// cudaDeviceReset the library image is loaded again and the array may move,
// so this entry point must not be used across a cudaDeviceReset.  All calls share it: calls whose work overlaps on the GPU
// (different streams, or several host threads) race on it and must be
// serialized by the caller.  Nothing in it has to start at zero: every
// partial a call reads was written earlier by the same call.
#include <mutex>

#include "iskv_internal.cuh"

namespace iskv {

namespace {

constexpr int64_t kScratchFloats = int64_t(1) << 20;   // 4 MiB of partial results
constexpr int kMaxDevices = 64;

__device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

std::mutex g_setup_mutex;
float* g_scratch_dev[kMaxDevices] = {};

// Device address of the scratch array for the current device (set-up once).
cudaError_t scratch_for_current_device(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_dev[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_dev[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_dev[dev];
    return cudaSuccess;
}

// True for memory the kernels on device `dev` may read directly: device
// memory of `dev` itself, or managed memory.  Device memory of another GPU is
// refused (it would fault, or cross NVLink unplanned, if peer access is on).
bool on_device(const void* p, int dev) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (at.type == cudaMemoryTypeManaged) return true;
    return at.type == cudaMemoryTypeDevice && at.device == dev;
}

}  // namespace

}  // namespace iskv

using namespace iskv;

extern "C" int iskv_decode_attention_noalloc(const iskv_decode_operands* o, const void* q,
                                             float* out, void* stream) {
    if (!o || !q || !out) return ISKV_ERR_INVALID_ARG;
    if (o->batch < 1 || o->kv_heads < 1 || o->q_heads < 1 || o->q_heads % o->kv_heads != 0)
        return ISKV_ERR_INVALID_ARG;
    if (o->head_dim != kHeadDim || o->q_heads / o->kv_heads > kMaxGroup) return ISKV_ERR_UNSUPPORTED;
    for (int r : {o->rank_k, o->rank_v})
        if (r < 16 || r > kHeadDim || r % 16 != 0) return ISKV_ERR_UNSUPPORTED;
    if ((o->kv_dtype != ISKV_F32 && o->kv_dtype != ISKV_BF16) ||
        (o->coef_dtype != ISKV_F32 && o->coef_dtype != ISKV_BF16))
        return ISKV_ERR_INVALID_ARG;
    if (o->T < 1 || o->n_c < 0 || o->n_c > o->T || o->n_c % kBlock != 0) return ISKV_ERR_INVALID_ARG;
    // the kernels stage both bases and may touch either store: all are required
    if (!o->coef_k || !o->coef_v || !o->basis_k || !o->basis_v || !o->ring_k || !o->ring_v)
        return ISKV_ERR_INVALID_ARG;
    if (o->coef_rows < o->n_c || o->ring_rows < 1 || o->ring_rows < o->T - o->n_c)
        return ISKV_ERR_INVALID_ARG;
    // every operand must already be in the current device's memory: nothing
    // is staged, and nothing is read across GPUs
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ISKV_ERR_CUDA;
    const void* ptrs[] = {q, out, o->coef_k, o->coef_v, o->basis_k, o->basis_v, o->ring_k,
                          o->ring_v, o->rope};
    for (const void* p : ptrs)
        if (p && !on_device(p, dev)) return ISKV_ERR_INVALID_ARG;

    // split the token axis as far as the scratch array allows
    const int64_t stride = 2 + o->rank_v + kHeadDim;
    const int64_t per_split = (int64_t)o->batch * o->q_heads * stride;
    const int64_t fit = kScratchFloats / per_split;
    if (fit < 1) return ISKV_ERR_CAPACITY;   // batch * q_heads too large for the scratch
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t BH = (int64_t)o->batch * o->kv_heads;
    int64_t splits = (4 * (int64_t)sms + BH - 1) / BH;
    const int64_t by_tokens = (o->T + 63) / 64;
    if (splits > by_tokens) splits = by_tokens;
    if (splits > fit) splits = fit;
    if (splits > 256) splits = 256;
    if (splits < 1) splits = 1;
    int64_t tps = (o->T + splits - 1) / splits;
    tps = ((tps + 63) / 64) * 64;
    splits = (o->T + tps - 1) / tps;

    float* scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return ISKV_ERR_CUDA;

    DecodeArgs a{};
    for (int w = 0; w < 2; ++w) {
        FactorView& f = w == 0 ? a.K : a.V;
        f.coef = const_cast<void*>(w == 0 ? o->coef_k : o->coef_v);
        f.basis = const_cast<float*>(w == 0 ? o->basis_k : o->basis_v);
        f.ring = w == 0 ? o->ring_k : o->ring_v;
        f.r = w == 0 ? o->rank_k : o->rank_v;
        f.coef_bf16 = o->coef_dtype == ISKV_BF16;
        f.kv_bf16 = o->kv_dtype == ISKV_BF16;
        f.n_max = o->coef_rows;
        f.cap = o->ring_rows;
        f.BH = (int)BH;
        f.D = 1;
    }
    a.q = q;
    a.partial = scratch;
    a.rope = reinterpret_cast<const float2*>(o->rope);
    a.layer = 0;
    a.B = o->batch;
    a.Hkv = o->kv_heads;
    a.Hq = o->q_heads;
    a.g = o->q_heads / o->kv_heads;
    a.T = o->T;
    a.n_c = o->n_c;
    a.scale = 1.0f / sqrtf((float)kHeadDim);
    a.tokens_per_split = tps;
    a.splits = (int)splits;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (launch_decode(a, s) != cudaSuccess) return ISKV_ERR_CUDA;
    if (launch_combine(a, out, s) != cudaSuccess) return ISKV_ERR_CUDA;
    return ISKV_OK;
}
