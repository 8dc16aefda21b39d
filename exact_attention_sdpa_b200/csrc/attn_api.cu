// attn_api.cu -- the C ABI of libattn.so (declared in include/attn.h):
// argument validation, TMA tensor-map encoding and kernel dispatch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>

#include "attn.h"
#include "attn_fwd_kernel.cuh"
#include "attn_bwd_tc.cuh"

namespace {

using attn::FwdParams;

__device__ unsigned int g_status_word;
__device__ unsigned int g_status_read;   // the word's value at the last read-and-clear

// Reads the status word and clears it in one atomic exchange, ordered after the kernels
// already enqueued on the stream it runs on.
__global__ void status_exchange_kernel() { g_status_read = atomicExch(&g_status_word, 0u); }

uint64_t g_wait_limit = 1ull << 32;
int g_inject_stall = 0;

// ---------------------------------------------------------------------------
// validation helpers
// ---------------------------------------------------------------------------
bool is_half_type(attn_dtype_t t) { return t == ATTN_F16 || t == ATTN_BF16; }

int64_t span_bytes(const attn_tensor_t* t) {
    // bytes from data to one past the last element (strides are non-negative)
    int64_t last = 0;
    for (int i = 0; i < t->ndim; ++i) last += (t->shape[i] - 1) * t->stride[i];
    return (last + 1) * 2;
}

bool overlaps(const attn_tensor_t* a, const attn_tensor_t* b) {
    if (a == nullptr || b == nullptr) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a->data), a1 = a0 + span_bytes(a);
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(b->data), b1 = b0 + span_bytes(b);
    return a0 < b1 && b0 < a1;
}

// A plain byte range [p, p + n) against a tensor's span.
bool overlaps_bytes(const void* p, size_t n, const attn_tensor_t* t) {
    if (p == nullptr || t == nullptr || n == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p), a1 = a0 + n;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(t->data), b1 = b0 + span_bytes(t);
    return a0 < b1 && b0 < a1;
}

// Common checks of a 16-bit tensor of rank `ndim`: positive shape, unit inner
// stride, other strides positive multiples of 8 elements, 16-byte aligned data.
attn_status_t check_tensor(const attn_tensor_t* t, int ndim) {
    if (t == nullptr || t->data == nullptr) return ATTN_ERR_INVALID_ARG;
    if (t->ndim != ndim) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < ndim; ++i)
        if (t->shape[i] <= 0) return ATTN_ERR_INVALID_ARG;
    if (t->stride[ndim - 1] != 1) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < ndim - 1; ++i) {
        if (t->stride[i] < 0 || (t->stride[i] % 8) != 0) return ATTN_ERR_INVALID_ARG;
        if (t->shape[i] > 1 && t->stride[i] == 0) return ATTN_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(t->data) & 15u) != 0) return ATTN_ERR_INVALID_ARG;
    return ATTN_OK;
}

// A packed [T, H, d] tensor of a ragged batch: non-negative strides, unit inner stride, data
// present (span_bytes and the overlap checks read the strides).
attn_status_t check_packed(const attn_tensor_t* t) {
    if (t->data == nullptr) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        if (t->shape[i] <= 0 || t->stride[i] < 0) return ATTN_ERR_INVALID_ARG;
    if (t->stride[2] != 1) return ATTN_ERR_INVALID_ARG;
    return ATTN_OK;
}

bool same_shape(const attn_tensor_t* a, const attn_tensor_t* b) {
    if (a->ndim != b->ndim) return false;
    for (int i = 0; i < a->ndim; ++i)
        if (a->shape[i] != b->shape[i]) return false;
    return true;
}

// Queries and keys: same batch, heads and head dim (the row counts may differ).
bool same_bhd(const attn_tensor_t* q, const attn_tensor_t* k) {
    return q->ndim == 4 && k->ndim == 4 && q->shape[0] == k->shape[0] && q->shape[1] == k->shape[1] &&
           q->shape[3] == k->shape[3];
}

// ---------------------------------------------------------------------------
// tensor maps (driver entry point fetched through the runtime, so the library
// does not link libcuda directly)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [B, H, N, d] view -> 4-D map with dims {d, N, H, B}, box {min(d,64), rows, 1, 1}
bool encode_qkv_map(CUtensorMap* map, const attn_tensor_t* t, unsigned rows = 128) {
    EncodeTiledFn enc = get_encode_fn();
    if (enc == nullptr) return false;
    const int64_t d = t->shape[3];
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)t->shape[2], (cuuint64_t)t->shape[1],
                                (cuuint64_t)t->shape[0]};
    // a stride of a size-1 dimension is irrelevant; give TMA a legal one
    auto stride_or = [&](int i, int64_t fallback) { return t->shape[i] > 1 ? t->stride[i] : fallback; };
    const int64_t sN = stride_or(2, d);
    const int64_t sH = stride_or(1, sN * t->shape[2]);
    const int64_t sB = stride_or(0, sH * t->shape[1]);
    const cuuint64_t strides[3] = {(cuuint64_t)(sN * 2), (cuuint64_t)(sH * 2), (cuuint64_t)(sB * 2)};
    const cuuint32_t box[4] = {(cuuint32_t)(d >= 64 ? 64 : d), (cuuint32_t)rows, 1u, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUtensorMapDataType dt =
        t->dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const CUtensorMapSwizzle sw = d >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return enc(map, dt, 4, t->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// e4m3 [B, H, N, d] view -> 4-D map {d, N, H, B}, box {d, 128, 1, 1}: one swizzle atom per row
// (64 bytes at d = 64, 128 bytes at d = 128)
bool encode_e4m3_map(CUtensorMap* map, const attn_tensor_t* t) {
    EncodeTiledFn enc = get_encode_fn();
    if (enc == nullptr) return false;
    const int64_t d = t->shape[3];
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)t->shape[2], (cuuint64_t)t->shape[1],
                                (cuuint64_t)t->shape[0]};
    auto stride_or = [&](int i, int64_t fallback) { return t->shape[i] > 1 ? t->stride[i] : fallback; };
    const int64_t sN = stride_or(2, d);
    const int64_t sH = stride_or(1, sN * t->shape[2]);
    const int64_t sB = stride_or(0, sH * t->shape[1]);
    const cuuint64_t strides[3] = {(cuuint64_t)sN, (cuuint64_t)sH, (cuuint64_t)sB};
    const cuuint32_t box[4] = {(cuuint32_t)d, 128u, 1u, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUtensorMapSwizzle sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, t->data, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// e4m3 V^T [B, H, d, Nk] view -> 4-D map {Nk, d, H, B}, box {128, d, 1, 1}, 128-byte swizzle
bool encode_e4m3_vt_map(CUtensorMap* map, const attn_tensor_t* t) {
    EncodeTiledFn enc = get_encode_fn();
    if (enc == nullptr) return false;
    const int64_t d = t->shape[2], nk = t->shape[3];
    const cuuint64_t dims[4] = {(cuuint64_t)nk, (cuuint64_t)d, (cuuint64_t)t->shape[1], (cuuint64_t)t->shape[0]};
    auto stride_or = [&](int i, int64_t fallback) { return t->shape[i] > 1 ? t->stride[i] : fallback; };
    const int64_t sD = stride_or(2, (nk + 15) / 16 * 16);
    const int64_t sH = stride_or(1, sD * d);
    const int64_t sB = stride_or(0, sH * t->shape[1]);
    const cuuint64_t strides[3] = {(cuuint64_t)sD, (cuuint64_t)sH, (cuuint64_t)sB};
    const cuuint32_t box[4] = {128u, (cuuint32_t)d, 1u, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, t->data, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bias [H, N, N] or [B, H, N, N] -> 4-D map {keys, rows, H, B}, box {64, 128, 1, 1}, 128-byte swizzle
bool encode_bias_map(CUtensorMap* map, const attn_tensor_t* b) {
    EncodeTiledFn enc = get_encode_fn();
    if (enc == nullptr) return false;
    const bool has_b = b->ndim == 4;
    const int64_t H = has_b ? b->shape[1] : b->shape[0];
    const int64_t Nq = has_b ? b->shape[2] : b->shape[1];      // rows (queries)
    const int64_t Nk = has_b ? b->shape[3] : b->shape[2];      // columns (keys)
    const int64_t si = has_b ? b->stride[2] : b->stride[1];
    const int64_t sh = has_b ? b->stride[1] : b->stride[0];
    // strides of extent-1 dimensions are free; give them valid (16-byte multiple) values
    const int64_t row = Nq > 1 ? si : (Nk + 7) / 8 * 8;
    const int64_t head = H > 1 ? sh : row * Nq;
    const int64_t batch = (has_b && b->shape[0] > 1) ? b->stride[0] : head * H;
    const cuuint64_t dims[4] = {(cuuint64_t)Nk, (cuuint64_t)Nq, (cuuint64_t)H, (cuuint64_t)(has_b ? b->shape[0] : 1)};
    const cuuint64_t strides[3] = {(cuuint64_t)(row * 2), (cuuint64_t)(head * 2), (cuuint64_t)(batch * 2)};
    const cuuint32_t box[4] = {64u, 128u, 1u, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUtensorMapDataType dt =
        b->dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    return enc(map, dt, 4, b->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Encoded tensor maps, cached per (base pointer, dtype, rank, shape, strides, box rows, map
// kind): a map depends on nothing else, so a call on buffers seen before skips the driver's
// encode.  64 entries replaced round-robin; lookups and inserts under one mutex.
enum MapKind { kMapQkv = 0, kMapE4m3 = 1, kMapE4m3Vt = 2, kMapBias = 3 };
struct MapKey {
    const void* data;
    int64_t shape[4], stride[4];
    int32_t dtype, ndim, kind;
    uint32_t rows;
};
struct MapEntry {
    MapKey key;
    CUtensorMap map;
    bool used;
};
std::mutex g_map_mu;
MapEntry g_maps[64];
unsigned g_map_next = 0;

bool encode_map(MapKind kind, CUtensorMap* map, const attn_tensor_t* t, unsigned rows) {
    MapKey k;
    std::memset(&k, 0, sizeof(k));            // padding included: keys compare with memcmp
    k.data = t->data;
    for (int i = 0; i < t->ndim && i < 4; ++i) {
        k.shape[i] = t->shape[i];
        k.stride[i] = t->stride[i];
    }
    k.dtype = static_cast<int32_t>(t->dtype);
    k.ndim = t->ndim;
    k.kind = kind;
    k.rows = rows;
    {
        std::lock_guard<std::mutex> lock(g_map_mu);
        for (const MapEntry& e : g_maps)
            if (e.used && std::memcmp(&e.key, &k, sizeof(k)) == 0) {
                *map = e.map;
                return true;
            }
    }
    bool ok = false;
    switch (kind) {
        case kMapQkv: ok = encode_qkv_map(map, t, rows); break;
        case kMapE4m3: ok = encode_e4m3_map(map, t); break;
        case kMapE4m3Vt: ok = encode_e4m3_vt_map(map, t); break;
        case kMapBias: ok = encode_bias_map(map, t); break;
    }
    if (!ok) return false;
    std::lock_guard<std::mutex> lock(g_map_mu);
    MapEntry& e = g_maps[g_map_next++ % 64];
    e.key = k;
    e.map = *map;
    e.used = true;
    return true;
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------
// A device attribute of the current device, cached per device.  Host threads may call
// concurrently: the cache entries are atomics (a race only repeats the same query).
int cached_attribute(cudaDeviceAttr attr, std::atomic<int> (&cache)[64]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, attr, dev) != cudaSuccess) return 0;
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

std::atomic<int> g_l2_bytes[64];
std::atomic<int> g_sm_count[64];

int l2_bytes() { return cached_attribute(cudaDevAttrL2CacheSize, g_l2_bytes); }

int sm_count() { return cached_attribute(cudaDevAttrMultiProcessorCount, g_sm_count); }

struct Maps {
    CUtensorMap q, k, v, bias;
};

// Raises a kernel's dynamic shared-memory limit once per device.  `done` is the calling
// launcher's own flag word (one bit per device), so each kernel instantiation is set once;
// concurrent first calls may both set it, which is harmless.
template <typename Kern>
cudaError_t smem_limit_once(Kern kern, int smem, std::atomic<uint64_t>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
}

template <typename T, int D, bool CAUSAL, bool BIAS, bool GATE, bool MODS = false>
cudaError_t launch_t(const Maps& m, const FwdParams& p, cudaStream_t stream) {
    auto kern = attn::attn_fwd_kernel<T, D, CAUSAL, BIAS, GATE, MODS>;
    // At least 116 KB of dynamic shared memory, so that two CTAs (of two kernels running
    // concurrently on different streams) never share an SM: each CTA allocates all 512
    // tensor-memory columns, and a second one would only wait for the first to finish.
    constexpr int smem = attn::BiasCfg<D, BIAS>::kDynBytes > 116 * 1024 ? attn::BiasCfg<D, BIAS>::kDynBytes
                                                                      : 116 * 1024;
    static std::atomic<uint64_t> smem_set{0};
    cudaError_t e = smem_limit_once(kern, smem, smem_set);
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    // persistent: one CTA per SM (tensor memory and registers allow no more)
    const int grid = p.num_units < sms ? p.num_units : sms;
    kern<<<grid, attn::kThreads, smem, stream>>>(m.q, m.k, m.v, m.bias, p);
    return cudaGetLastError();
}

template <typename T, int D, bool CAUSAL>
cudaError_t launch_fp8_t(const Maps& m, const FwdParams& p, cudaStream_t stream) {
    auto kern = attn::attn_fwd_kernel<T, D, CAUSAL, false, false, false, true>;
    constexpr int need = attn::Cfg<D, true>::kDynBytes;
    constexpr int smem = need > 116 * 1024 ? need : 116 * 1024;     // one CTA per SM (all of TMEM)
    static std::atomic<uint64_t> smem_set{0};
    cudaError_t e = smem_limit_once(kern, smem, smem_set);
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const int grid = p.num_units < sms ? p.num_units : sms;
    kern<<<grid, attn::kThreads, smem, stream>>>(m.q, m.k, m.v, m.bias, p);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_d(bool causal, bool bias, bool gate, const Maps& m, const FwdParams& p, cudaStream_t s) {
    if (p.has_mods) {   // score modifications: built without bias and gate only
        if (bias || gate) return cudaErrorInvalidValue;
        return causal ? launch_t<T, D, true, false, false, true>(m, p, s)
                      : launch_t<T, D, false, false, false, true>(m, p, s);
    }
#define ATTN_CASE(C, B_, G_) \
    if (causal == C && bias == B_ && gate == G_) return launch_t<T, D, C, B_, G_>(m, p, s);
    ATTN_CASE(false, false, false)
    ATTN_CASE(false, false, true)
    ATTN_CASE(false, true, false)
    ATTN_CASE(false, true, true)
    ATTN_CASE(true, false, false)
    ATTN_CASE(true, false, true)
    ATTN_CASE(true, true, false)
    ATTN_CASE(true, true, true)
#undef ATTN_CASE
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_dtype(int d, bool causal, bool bias, bool gate, const Maps& m, const FwdParams& p,
                         cudaStream_t s) {
    switch (d) {
        case 32: return launch_d<T, 32>(causal, bias, gate, m, p, s);
        case 64: return launch_d<T, 64>(causal, bias, gate, m, p, s);
        case 128: return launch_d<T, 128>(causal, bias, gate, m, p, s);
        default: return cudaErrorInvalidValue;
    }
}

unsigned int* status_word_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    static unsigned int* ptrs[64] = {nullptr};
    static std::mutex mu;
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<unsigned int*>(ptr);
    }
    return ptrs[dev];
}

// Every host-side check of attn_fwd, in its documented order; sets *empty for a
// problem with B, H or N equal to 0 (valid, nothing to do).
attn_status_t validate_fwd(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                           const attn_tensor_t* bias, const attn_tensor_t* gate, float scale,
                           const attn_tensor_t* out, const float* lse, bool* empty) {
    *empty = false;
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return ATTN_ERR_INVALID_ARG;
    // dtype rules first: fp32 is a valid request this fused kernel does not serve
    if (q->dtype == ATTN_F32 || q->dtype == ATTN_E4M3) return ATTN_ERR_UNSUPPORTED;   // (e4m3: attn_fwd_fp8)
    if (!is_half_type(q->dtype)) return ATTN_ERR_INVALID_ARG;
    if (k->dtype != q->dtype || v->dtype != q->dtype || out->dtype != q->dtype) return ATTN_ERR_UNSUPPORTED;
    if (bias != nullptr && bias->dtype != q->dtype) return ATTN_ERR_UNSUPPORTED;
    if (gate != nullptr && gate->dtype != q->dtype) return ATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;

    // empty problems (B, H or the query count 0): nothing to do
    if (q->ndim == 4 && (q->shape[0] == 0 || q->shape[1] == 0 || q->shape[2] == 0)) {
        if (k->ndim != 4 || v->ndim != 4 || out->ndim != 4) return ATTN_ERR_INVALID_ARG;
        if (!same_shape(k, v) || !same_shape(q, out) || !same_bhd(q, k)) return ATTN_ERR_INVALID_ARG;
        *empty = true;
        return ATTN_OK;
    }
    attn_status_t st;
    if ((st = check_tensor(q, 4)) != ATTN_OK) return st;
    if ((st = check_tensor(k, 4)) != ATTN_OK) return st;   // (a key count of 0 fails here)
    if ((st = check_tensor(v, 4)) != ATTN_OK) return st;
    if ((st = check_tensor(out, 4)) != ATTN_OK) return st;
    if (!same_shape(k, v) || !same_shape(q, out) || !same_bhd(q, k)) return ATTN_ERR_INVALID_ARG;
    const int64_t B = q->shape[0], H = q->shape[1], N = q->shape[2], Nk = k->shape[2], d = q->shape[3];
    if (d != 32 && d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (N > (int64_t(1) << 30) || Nk > (int64_t(1) << 30) || B * H > (int64_t(1) << 24)) return ATTN_ERR_UNSUPPORTED;
    if (gate != nullptr) {
        if ((st = check_tensor(gate, 4)) != ATTN_OK) return st;
        if (!same_shape(q, gate)) return ATTN_ERR_INVALID_ARG;
    }
    if (bias != nullptr) {
        if (bias->ndim == 3) {
            if ((st = check_tensor(bias, 3)) != ATTN_OK) return st;
            if (bias->shape[0] != H || bias->shape[1] != N || bias->shape[2] != Nk) return ATTN_ERR_INVALID_ARG;
        } else if (bias->ndim == 4) {
            if ((st = check_tensor(bias, 4)) != ATTN_OK) return st;
            if (bias->shape[0] != B || bias->shape[1] != H || bias->shape[2] != N || bias->shape[3] != Nk)
                return ATTN_ERR_INVALID_ARG;
        } else {
            return ATTN_ERR_INVALID_ARG;
        }
    }
    if (overlaps(out, q) || overlaps(out, k) || overlaps(out, v) || overlaps(out, bias) || overlaps(out, gate))
        return ATTN_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_INVALID_ARG;

    return ATTN_OK;
}

// Tensor-core backward: D_i into dQ's rows, then dK/dV (one CTA per 128 keys), then dQ (one CTA
// per 128 queries).  m: Q/dO maps with 64-row boxes and K/V with 128 (dK/dV kernel), then
// Q/dO with 128 and K/V with 64 (dQ kernel).
struct BwdMaps {
    CUtensorMap q64, k128, v128, do64, q128, k64, v64, do128;
};

template <typename T, int D, bool CAUSAL, bool MODS>
cudaError_t launch_bwd_tc_t(const BwdMaps& m, const attn::bwdtc::Params& p, cudaStream_t stream) {
    using namespace attn::bwdtc;
    const int64_t threads = static_cast<int64_t>(p.B) * p.H * p.N * (D / 8);
    const int64_t blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    bwd_prep_kernel<T, D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    auto k1 = bwd_dkdv_kernel<T, D, CAUSAL, MODS>;
    constexpr int s1 = DkdvCfg<D>::kDynBytes;
    static std::atomic<uint64_t> set1{0}, set2{0};
    if ((e = smem_limit_once(k1, s1, set1)) != cudaSuccess) return e;
    k1<<<dim3((p.Nk + 127) / 128, p.B * p.H), kThreadsPP, s1, stream>>>(m.q64, m.k128, m.v128, m.do64, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    auto k2 = bwd_dq_kernel<T, D, CAUSAL, MODS>;
    constexpr int s2 = DqCfg<D>::kDynBytes;
    if ((e = smem_limit_once(k2, s2, set2)) != cudaSuccess) return e;
    k2<<<dim3((p.N + 127) / 128, p.B * p.H), kThreadsPP, s2, stream>>>(m.q128, m.k64, m.v64, m.do128, p);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_bwd_tc_d(bool causal, bool mods, const BwdMaps& m, const attn::bwdtc::Params& p, cudaStream_t s) {
    if (mods) return causal ? launch_bwd_tc_t<T, D, true, true>(m, p, s) : launch_bwd_tc_t<T, D, false, true>(m, p, s);
    return causal ? launch_bwd_tc_t<T, D, true, false>(m, p, s) : launch_bwd_tc_t<T, D, false, false>(m, p, s);
}

template <typename T>
cudaError_t launch_bwd_tc_dtype(int d, bool causal, bool mods, const BwdMaps& m, const attn::bwdtc::Params& p,
                                cudaStream_t s) {
    if (d == 32) return launch_bwd_tc_d<T, 32>(causal, mods, m, p, s);
    if (d == 64) return launch_bwd_tc_d<T, 64>(causal, mods, m, p, s);
    return launch_bwd_tc_d<T, 128>(causal, mods, m, p, s);
}


// A host view and its device staging view: same dtype, rank, shape and strides.
bool same_layout(const attn_tensor_t* a, const attn_tensor_t* b) {
    if ((a == nullptr) != (b == nullptr)) return false;
    if (a == nullptr) return true;
    if (a->dtype != b->dtype || !same_shape(a, b)) return false;
    for (int i = 0; i < a->ndim; ++i)
        if (a->stride[i] != b->stride[i]) return false;
    return true;
}

// The checks of attn_fwd_ex's score modifications (nullable: none).
attn_status_t check_mods(const attn_mods_t* mods, const attn_tensor_t* bias, const attn_tensor_t* gate) {
    if (mods == nullptr) return ATTN_OK;
    if (!std::isfinite(mods->softcap) || mods->softcap < 0.f) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(mods->alibi_slopes) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    const bool on = mods->alibi_slopes != nullptr || mods->softcap > 0.f || mods->window_left >= 0;
    if (on && (bias != nullptr || gate != nullptr)) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

// attn_fwd_ex with an optional lse layout (defined below the C entry points)
attn_status_t fwd_impl(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                       const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                       const attn_mods_t* mods, attn_tensor_t* out, float* lse, const int64_t* lse_layout,
                       cudaStream_t stream);

}  // namespace

extern "C" {

attn_status_t attn_fwd(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                       const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                       attn_tensor_t* out, float* lse, cudaStream_t stream) {
    return attn_fwd_ex(q, k, v, bias, gate, causal, scale, nullptr, out, lse, stream);
}

attn_status_t attn_fwd_ex(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                          const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                          const attn_mods_t* mods, attn_tensor_t* out, float* lse, cudaStream_t stream) {
    return fwd_impl(q, k, v, bias, gate, causal, scale, mods, out, lse, nullptr, stream);
}

}  // extern "C"

namespace {
// attn_fwd_ex with an optional lse layout {stride between batches, stride between heads}
attn_status_t fwd_impl(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                       const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                       const attn_mods_t* mods, attn_tensor_t* out, float* lse, const int64_t* lse_layout,
                       cudaStream_t stream) {
    bool empty = false;
    const attn_status_t st = validate_fwd(q, k, v, bias, gate, scale, out, lse, &empty);
    if (st != ATTN_OK) return st;
    const attn_status_t ms = check_mods(mods, bias, gate);
    if (ms != ATTN_OK) return ms;
    if (empty) return ATTN_OK;
    const int64_t B = q->shape[0], H = q->shape[1], N = q->shape[2], Nk = k->shape[2], d = q->shape[3];

    // ---- launch
    Maps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!encode_map(kMapQkv, &maps.q, q, 128) || !encode_map(kMapQkv, &maps.k, k, 128) ||
        !encode_map(kMapQkv, &maps.v, v, 128))
        return ATTN_ERR_CUDA;
    // d <= 64 stages bias tiles through shared memory by TMA; d = 128 reads bias rows directly
    if (bias != nullptr && d <= 64 && !encode_map(kMapBias, &maps.bias, bias, 128)) return ATTN_ERR_CUDA;
    unsigned int* status = status_word_ptr();
    if (status == nullptr) return ATTN_ERR_CUDA;

    FwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = static_cast<int>(B);
    p.H = static_cast<int>(H);
    p.N = static_cast<int>(N);
    p.Nk = static_cast<int>(Nk);
    p.causal_off = static_cast<int>(Nk - N);
    p.num_q_pairs = static_cast<int>((N + attn::kRowsPerUnit - 1) / attn::kRowsPerUnit);
    p.n_kv_tiles = static_cast<int>((Nk + attn::kBlockN - 1) / attn::kBlockN);
    const int64_t units = static_cast<int64_t>(p.num_q_pairs) * B * H;
    if (units > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
    p.num_units = static_cast<int>(units);
    p.scale = scale;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    // unit order: when the K/V of all heads exceed the L2, schedule a few heads at a
    // time (enough query pairs to occupy every SM), else all heads together
    {
        const double kv_bytes = 2.0 * static_cast<double>(B * H) * static_cast<double>(Nk) * d * 2.0;
        const int sms = sm_count();
        int g = static_cast<int>(B * H);
        if (sms > 0 && kv_bytes > static_cast<double>(l2_bytes())) g = (sms + p.num_q_pairs - 1) / p.num_q_pairs;
        p.head_group = g < 1 ? 1 : (g > B * H ? static_cast<int>(B * H) : g);
    }
    if (bias != nullptr) {
        p.bias = bias->data;
        if (bias->ndim == 3) {
            p.bias_sb = 0;
            p.bias_sh = bias->stride[0];
            p.bias_si = bias->stride[1];
        } else {
            p.bias_sb = bias->stride[0];
            p.bias_sh = bias->stride[1];
            p.bias_si = bias->stride[2];
        }
    }
    if (gate != nullptr) {
        p.gate = gate->data;
        p.gate_sb = gate->stride[0];
        p.gate_sh = gate->stride[1];
        p.gate_si = gate->stride[2];
    }
    p.out = out->data;
    p.out_sb = out->stride[0];
    p.out_sh = out->stride[1];
    p.out_si = out->stride[2];
    p.lse = lse;
    p.lse_sh = N;
    p.lse_sb = H * N;
    if (lse_layout != nullptr) {   // (ragged batches: each sequence's rows inside [H, T])
        p.lse_sb = lse_layout[0];
        p.lse_sh = lse_layout[1];
    }
    if (mods != nullptr) {
        p.alibi = mods->alibi_slopes;
        p.softcap = mods->softcap;
        p.window_left = mods->window_left >= 0 ? mods->window_left : -1;
        p.has_mods = (p.alibi != nullptr || p.softcap > 0.f || p.window_left >= 0) ? 1 : 0;
    } else {
        p.window_left = -1;
    }
    p.wait_limit = g_wait_limit;
    p.status = status;
    p.inject_stall = g_inject_stall;

    cudaError_t e;
    if (q->dtype == ATTN_BF16)
        e = launch_dtype<__nv_bfloat16>(static_cast<int>(d), causal != 0, bias != nullptr, gate != nullptr, maps, p,
                                        stream);
    else
        e = launch_dtype<__half>(static_cast<int>(d), causal != 0, bias != nullptr, gate != nullptr, maps, p,
                                 stream);
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Test hook of attn_debug_exp2: thread t evaluates elements 2t and 2t + 1 (one pair, as the
// softmax does) with the exponential selected by `mode`.
__global__ void exp2_probe_kernel(const float* x, float* y, int64_t n, int mode) {
    const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const bool two = i + 1 < n;
    const float x0 = x[i], x1 = two ? x[i + 1] : 0.f;
    float y0, y1;
    if (mode == ATTN_EXP2_FMA_PIPE) {
        attn::ex2_emu2(y0, y1, x0, x1);
    } else if (mode == ATTN_EXP2_MUFU) {
        y0 = attn::sm100::ex2_approx(x0);
        y1 = attn::sm100::ex2_approx(x1);
    } else {
        y0 = exp2f(x0);
        y1 = exp2f(x1);
    }
    y[i] = y0;
    if (two) y[i + 1] = y1;
}

}  // namespace

extern "C" {

attn_status_t attn_debug_exp2(const float* x, float* y, int64_t n, int mode, cudaStream_t stream) {
    if (n < 0 || mode < ATTN_EXP2_FMA_PIPE || mode > ATTN_EXP2_CUDA_EXP2F) return ATTN_ERR_INVALID_ARG;
    if (n == 0) return ATTN_OK;
    if (x == nullptr || y == nullptr) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 3u) != 0 || (reinterpret_cast<uintptr_t>(y) & 3u) != 0)
        return ATTN_ERR_INVALID_ARG;
    const int64_t blocks = ((n + 1) / 2 + 255) / 256;
    if (blocks > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
    exp2_probe_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, y, n, mode);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_fwd_host(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                            const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                            attn_tensor_t* out, float* lse,
                            const attn_tensor_t* q_dev, const attn_tensor_t* k_dev, const attn_tensor_t* v_dev,
                            const attn_tensor_t* bias_dev, const attn_tensor_t* gate_dev,
                            attn_tensor_t* out_dev, float* lse_dev, cudaStream_t stream) {
    return attn_fwd_host_ex(q, k, v, bias, gate, causal, scale, nullptr, out, lse, q_dev, k_dev, v_dev, bias_dev,
                            gate_dev, out_dev, lse_dev, stream);
}

attn_status_t attn_fwd_host_ex(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                               const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                               const attn_mods_t* mods, attn_tensor_t* out, float* lse,
                               const attn_tensor_t* q_dev, const attn_tensor_t* k_dev, const attn_tensor_t* v_dev,
                               const attn_tensor_t* bias_dev, const attn_tensor_t* gate_dev,
                               attn_tensor_t* out_dev, float* lse_dev, cudaStream_t stream) {
    // every check before the first copy is enqueued
    if (q_dev == nullptr || k_dev == nullptr || v_dev == nullptr || out_dev == nullptr) return ATTN_ERR_INVALID_ARG;
    bool empty = false;
    attn_status_t st = validate_fwd(q_dev, k_dev, v_dev, bias_dev, gate_dev, scale, out_dev, lse_dev, &empty);
    if (st != ATTN_OK) return st;
    st = check_mods(mods, bias_dev, gate_dev);
    if (st != ATTN_OK) return st;
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return ATTN_ERR_INVALID_ARG;
    if (!same_layout(q, q_dev) || !same_layout(k, k_dev) || !same_layout(v, v_dev) || !same_layout(out, out_dev) ||
        !same_layout(bias, bias_dev) || !same_layout(gate, gate_dev))
        return ATTN_ERR_INVALID_ARG;
    if ((lse == nullptr) != (lse_dev == nullptr)) return ATTN_ERR_INVALID_ARG;
    if (empty) return ATTN_OK;
    const attn_tensor_t* hosts[6] = {q, k, v, out, bias, gate};
    for (const attn_tensor_t* t : hosts)
        if (t != nullptr && t->data == nullptr) return ATTN_ERR_INVALID_ARG;

    // host -> device, one copy per input (the span from the first to one past the last element)
    const attn_tensor_t* ins[5][2] = {{q, q_dev}, {k, k_dev}, {v, v_dev}, {bias, bias_dev}, {gate, gate_dev}};
    for (auto& io : ins) {
        if (io[0] == nullptr) continue;
        if (cudaMemcpyAsync(io[1]->data, io[0]->data, static_cast<size_t>(span_bytes(io[0])),
                            cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return ATTN_ERR_CUDA;
    }
    st = fwd_impl(q_dev, k_dev, v_dev, bias_dev, gate_dev, causal, scale, mods, out_dev, lse_dev, nullptr, stream);
    if (st != ATTN_OK) return st;
    // device -> host: O, then lse
    if (cudaMemcpyAsync(out->data, out_dev->data, static_cast<size_t>(span_bytes(out)), cudaMemcpyDeviceToHost,
                        stream) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (lse != nullptr) {
        const size_t n = static_cast<size_t>(q->shape[0] * q->shape[1] * q->shape[2]) * sizeof(float);
        if (cudaMemcpyAsync(lse, lse_dev, n, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

attn_status_t attn_fwd_varlen(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch, int causal,
                              float scale, attn_tensor_t* out, float* lse, cudaStream_t stream) {
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return ATTN_ERR_INVALID_ARG;
    if (q->dtype == ATTN_F32) return ATTN_ERR_UNSUPPORTED;
    if (!is_half_type(q->dtype)) return ATTN_ERR_INVALID_ARG;
    if (k->dtype != q->dtype || v->dtype != q->dtype || out->dtype != q->dtype) return ATTN_ERR_UNSUPPORTED;
    if (q->ndim != 3 || k->ndim != 3 || v->ndim != 3 || out->ndim != 3) return ATTN_ERR_INVALID_ARG;
    if (!same_shape(k, v) || !same_shape(q, out)) return ATTN_ERR_INVALID_ARG;
    if (q->shape[1] != k->shape[1] || q->shape[2] != k->shape[2]) return ATTN_ERR_INVALID_ARG;
    if (batch < 0 || cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    const int64_t Tq = q->shape[0], Tk = k->shape[0], H = q->shape[1];
    attn_status_t st0 = ATTN_OK;
    if (cu_seqlens_q[0] != 0 || cu_seqlens_k[0] != 0 || cu_seqlens_q[batch] != Tq || cu_seqlens_k[batch] != Tk)
        return ATTN_ERR_INVALID_ARG;
    for (int32_t b = 0; b < batch; ++b) {
        const int32_t nq = cu_seqlens_q[b + 1] - cu_seqlens_q[b], nk = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        if (nq < 0 || nk < 0) return ATTN_ERR_INVALID_ARG;
        if (nq > 0 && nk == 0) return ATTN_ERR_INVALID_ARG;     // queries with no key at all
    }
    if (Tq == 0 || H == 0) return ATTN_OK;
    // the packed tensors as wholes: O must not overlap any input row of any sequence, and lse
    // ([H, Tq] fp32) must overlap none of the tensors
    if ((st0 = check_packed(q)) != ATTN_OK || (st0 = check_packed(k)) != ATTN_OK ||
        (st0 = check_packed(v)) != ATTN_OK || (st0 = check_packed(out)) != ATTN_OK)
        return st0;
    if (overlaps(out, q) || overlaps(out, k) || overlaps(out, v)) return ATTN_ERR_INVALID_ARG;
    if (lse != nullptr) {
        const size_t lse_bytes = static_cast<size_t>(H * Tq) * sizeof(float);
        if (overlaps_bytes(lse, lse_bytes, q) || overlaps_bytes(lse, lse_bytes, k) ||
            overlaps_bytes(lse, lse_bytes, v) || overlaps_bytes(lse, lse_bytes, out))
            return ATTN_ERR_INVALID_ARG;
    }
    // each sequence: a [1, H, n, d] view of the packed [T, H, d] tensors (strides in elements);
    // every check of attn_fwd runs on the first sequence's views before anything is launched
    auto view = [](const attn_tensor_t* t, int64_t row0, int64_t n) {
        attn_tensor_t x;
        x.data = static_cast<char*>(t->data) + row0 * t->stride[0] * 2;
        x.dtype = t->dtype;
        x.ndim = 4;
        x.shape[0] = 1; x.shape[1] = t->shape[1]; x.shape[2] = n; x.shape[3] = t->shape[2];
        x.stride[0] = n * t->stride[0]; x.stride[1] = t->stride[1]; x.stride[2] = t->stride[0]; x.stride[3] = t->stride[2];
        return x;
    };
    std::vector<int32_t> order;                    // non-empty sequences, every one checked first
    for (int32_t b = 0; b < batch; ++b) {
        const int64_t q0 = cu_seqlens_q[b], nq = cu_seqlens_q[b + 1] - q0;
        const int64_t k0 = cu_seqlens_k[b], nk = cu_seqlens_k[b + 1] - k0;
        if (nq == 0) continue;
        attn_tensor_t vq = view(q, q0, nq), vk = view(k, k0, nk), vv = view(v, k0, nk), vo = view(out, q0, nq);
        bool empty = false;
        attn_status_t st = validate_fwd(&vq, &vk, &vv, nullptr, nullptr, scale, &vo, lse, &empty);
        if (st != ATTN_OK) return st;
        order.push_back(b);
    }
    if (order.empty()) return ATTN_OK;
    // heaviest sequences first (query rows x visible keys), in launches of up to kMaxSeq sequences
    auto work = [&](int32_t b) {
        const double nq = cu_seqlens_q[b + 1] - cu_seqlens_q[b], nk = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        return causal ? nq * (nk - 0.5 * nq) : nq * nk;
    };
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return work(a) > work(b); });
    // packed [1, H, T, d] views of the whole tensors: one tensor map each for every sequence
    attn_tensor_t pq = view(q, 0, Tq), pk = view(k, 0, Tk), pv = view(v, 0, Tk), po = view(out, 0, Tq);
    Maps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!encode_map(kMapQkv, &maps.q, &pq, 128) || !encode_map(kMapQkv, &maps.k, &pk, 128) ||
        !encode_map(kMapQkv, &maps.v, &pv, 128))
        return ATTN_ERR_CUDA;
    unsigned int* status = status_word_ptr();
    if (status == nullptr) return ATTN_ERR_CUDA;
    const int64_t d = q->shape[2];
    for (size_t c0 = 0; c0 < order.size(); c0 += attn::kMaxSeq) {
        const size_t c1 = std::min(order.size(), c0 + attn::kMaxSeq);
        FwdParams p;
        std::memset(&p, 0, sizeof(p));
        p.B = 1;
        p.H = static_cast<int>(H);
        p.N = static_cast<int>(Tq);
        p.Nk = static_cast<int>(Tk);
        p.num_q_pairs = 1;
        p.n_kv_tiles = 1;
        p.head_group = static_cast<int>(H);
        p.n_seq = static_cast<int>(c1 - c0);
        // causal with N_q = N_k everywhere: units ordered by query pair across the sequences (the
        // chunk is sorted by causal work, which for N_q = N_k orders the pair counts, most first)
        bool level = causal != 0;
        for (size_t i = c0; i < c1; ++i)
            level = level && (cu_seqlens_q[order[i] + 1] - cu_seqlens_q[order[i]] ==
                              cu_seqlens_k[order[i] + 1] - cu_seqlens_k[order[i]]);
        p.level_order = level ? 1 : 0;
        auto pairs = [&](int s) { return (p.seq_nq[s] + attn::kRowsPerUnit - 1) / attn::kRowsPerUnit; };
        for (size_t i = c0; i < c1; ++i) {
            const int32_t b = order[i];
            const int s = static_cast<int>(i - c0);
            p.seq_q0[s] = cu_seqlens_q[b];
            p.seq_k0[s] = cu_seqlens_k[b];
            p.seq_nq[s] = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
            p.seq_nk[s] = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        }
        int64_t units = 0;
        for (int s = 0; s < p.n_seq; ++s) {
            p.seq_units[s] = static_cast<int>(units);
            if (level) {
                // segment s: the pairs of sequences 0..s beyond those of sequence s + 1
                const int below = s + 1 < p.n_seq ? pairs(s + 1) : 0;
                units += static_cast<int64_t>(s + 1) * H * (pairs(s) - below);
            } else {
                units += H * pairs(s);
            }
        }
        if (units > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
        p.seq_units[p.n_seq] = static_cast<int>(units);
        p.num_units = static_cast<int>(units);
        p.scale = scale;
        p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
        p.out = po.data;
        p.out_sb = po.stride[0];
        p.out_sh = po.stride[1];
        p.out_si = po.stride[2];
        p.lse = lse;
        p.lse_sb = 0;
        p.lse_sh = Tq;
        p.window_left = -1;
        p.wait_limit = g_wait_limit;
        p.status = status;
        p.inject_stall = g_inject_stall;
        const cudaError_t e = q->dtype == ATTN_BF16
                                  ? launch_dtype<__nv_bfloat16>(static_cast<int>(d), causal != 0, false, false, maps, p, stream)
                                  : launch_dtype<__half>(static_cast<int>(d), causal != 0, false, false, maps, p, stream);
        if (e != cudaSuccess) return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

attn_status_t attn_bwd(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                       const attn_tensor_t* out, const float* lse, const attn_tensor_t* dout, int causal,
                       float scale, attn_tensor_t* dq, attn_tensor_t* dk, attn_tensor_t* dv,
                       cudaStream_t stream) {
    return attn_bwd_ex(q, k, v, out, lse, dout, causal, scale, nullptr, dq, dk, dv, stream);
}

attn_status_t attn_bwd_ex(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                          const attn_tensor_t* out, const float* lse, const attn_tensor_t* dout, int causal,
                          float scale, const attn_mods_t* mods, attn_tensor_t* dq, attn_tensor_t* dk,
                          attn_tensor_t* dv, cudaStream_t stream) {
    bool mods_on = false;
    if (mods != nullptr) {
        if (!std::isfinite(mods->softcap) || mods->softcap < 0.f) return ATTN_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(mods->alibi_slopes) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
        mods_on = mods->alibi_slopes != nullptr || mods->softcap > 0.f || mods->window_left >= 0;
    }
    bool empty = false;
    attn_status_t st = validate_fwd(q, k, v, nullptr, nullptr, scale, out, lse, &empty);
    if (st != ATTN_OK) return st;
    if (dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr) return ATTN_ERR_INVALID_ARG;
    if (dout->dtype != q->dtype || dq->dtype != q->dtype || dk->dtype != q->dtype || dv->dtype != q->dtype)
        return ATTN_ERR_UNSUPPORTED;
    if (!same_shape(dout, q) || !same_shape(dq, q) || !same_shape(dk, k) || !same_shape(dv, k))
        return ATTN_ERR_INVALID_ARG;
    if (empty) return ATTN_OK;
    if (lse == nullptr) return ATTN_ERR_INVALID_ARG;
    if ((st = check_tensor(dout, 4)) != ATTN_OK) return st;
    if ((st = check_tensor(dq, 4)) != ATTN_OK) return st;
    if ((st = check_tensor(dk, 4)) != ATTN_OK) return st;
    if ((st = check_tensor(dv, 4)) != ATTN_OK) return st;
    const attn_tensor_t* outs[3] = {dq, dk, dv};
    const attn_tensor_t* ins[5] = {q, k, v, out, dout};
    for (int a = 0; a < 3; ++a) {
        for (int b = 0; b < 5; ++b)
            if (overlaps(outs[a], ins[b])) return ATTN_ERR_INVALID_ARG;
        for (int b = a + 1; b < 3; ++b)
            if (overlaps(outs[a], outs[b])) return ATTN_ERR_INVALID_ARG;
    }
    const int64_t B = q->shape[0], H = q->shape[1], N = q->shape[2], Nk = k->shape[2], d = q->shape[3];
    {   // lse ([B, H, N] fp32, read) must not overlap a gradient the kernels write
        const size_t lse_bytes = static_cast<size_t>(B * H * N) * sizeof(float);
        for (int a = 0; a < 3; ++a)
            if (overlaps_bytes(lse, lse_bytes, outs[a])) return ATTN_ERR_INVALID_ARG;
    }
    if (B * H > 65535) return ATTN_ERR_UNSUPPORTED;

    attn::bwdtc::Params tp;
    std::memset(&tp, 0, sizeof(tp));
    tp.B = static_cast<int>(B);
    tp.H = static_cast<int>(H);
    tp.N = static_cast<int>(N);
    tp.Nk = static_cast<int>(Nk);
    tp.causal_off = static_cast<int>(Nk - N);
    tp.scale = scale;
    tp.scale_log2 = scale * 1.4426950408889634f;
    tp.o = out->data; tp.o_sb = out->stride[0]; tp.o_sh = out->stride[1]; tp.o_si = out->stride[2];
    tp.dout = dout->data; tp.do_sb = dout->stride[0]; tp.do_sh = dout->stride[1]; tp.do_si = dout->stride[2];
    tp.lse = lse;
    tp.dq = dq->data; tp.dq_sb = dq->stride[0]; tp.dq_sh = dq->stride[1]; tp.dq_si = dq->stride[2];
    tp.dk = dk->data; tp.dk_sb = dk->stride[0]; tp.dk_sh = dk->stride[1]; tp.dk_si = dk->stride[2];
    tp.dv = dv->data; tp.dv_sb = dv->stride[0]; tp.dv_sh = dv->stride[1]; tp.dv_si = dv->stride[2];
    tp.wait_limit = g_wait_limit;
    tp.status = status_word_ptr();
    tp.alibi = mods_on ? mods->alibi_slopes : nullptr;
    tp.softcap = mods_on ? mods->softcap : 0.f;
    tp.window_left = (mods_on && mods->window_left >= 0) ? mods->window_left : -1;
    if (tp.status == nullptr) return ATTN_ERR_CUDA;
    BwdMaps m;
    if (!encode_map(kMapQkv, &m.q64, q, 64) || !encode_map(kMapQkv, &m.k128, k, 128) ||
        !encode_map(kMapQkv, &m.v128, v, 128) || !encode_map(kMapQkv, &m.do64, dout, 64) ||
        !encode_map(kMapQkv, &m.q128, q, 128) || !encode_map(kMapQkv, &m.k64, k, 64) ||
        !encode_map(kMapQkv, &m.v64, v, 64) || !encode_map(kMapQkv, &m.do128, dout, 128))
        return ATTN_ERR_CUDA;
    cudaError_t e = q->dtype == ATTN_BF16
                        ? launch_bwd_tc_dtype<__nv_bfloat16>(static_cast<int>(d), causal != 0, mods_on, m, tp, stream)
                        : launch_bwd_tc_dtype<__half>(static_cast<int>(d), causal != 0, mods_on, m, tp, stream);
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

const char* attn_status_string(attn_status_t status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument (null, shape/stride mismatch, misalignment, aliasing or non-finite scale)";
        case ATTN_ERR_UNSUPPORTED: return "unsupported (fp32, mixed dtypes, or head dim not in {32, 64, 128})";
        case ATTN_ERR_CUDA: return "CUDA error (launch, tensor-map encoding or device query failed)";
        case ATTN_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        case ATTN_ERR_CHECK: return "a debug build's device-side index or range check failed";
        default: return "unknown status";
    }
}

attn_status_t attn_last_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
    status_exchange_kernel<<<1, 1, 0, stream>>>();
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_status_read, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
    if (v & attn::kStatusTimeout) return ATTN_ERR_TIMEOUT;
    return (v & attn::kStatusCheck) ? ATTN_ERR_CHECK : ATTN_OK;
}

void attn_set_wait_limit(uint64_t cycles) { g_wait_limit = cycles < 1024 ? 1024 : cycles; }

void attn_debug_inject_stall(int enable) { g_inject_stall = enable != 0; }

const char* attn_version(void) { return "0.2.0"; }

int attn_build_flags(void) { return ATTN_DEBUG ? ATTN_BUILD_DEBUG_CHECKS : 0; }

}  // extern "C"

namespace {
// e4m3 tensor: positive shape, unit inner stride, other strides multiples of 16 elements (bytes),
// 16-byte aligned data
attn_status_t check_e4m3(const attn_tensor_t* t) {
    if (t == nullptr || t->data == nullptr || t->dtype != ATTN_E4M3 || t->ndim != 4) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 4; ++i)
        if (t->shape[i] <= 0) return ATTN_ERR_INVALID_ARG;
    if (t->stride[3] != 1) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i) {
        if (t->stride[i] < 0 || (t->stride[i] % 16) != 0) return ATTN_ERR_INVALID_ARG;
        if (t->shape[i] > 1 && t->stride[i] == 0) return ATTN_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(t->data) & 15u) != 0) return ATTN_ERR_INVALID_ARG;
    return ATTN_OK;
}

int64_t span_bytes_e(const attn_tensor_t* t, int64_t esize) {
    int64_t last = 0;
    for (int i = 0; i < t->ndim; ++i) last += (t->shape[i] - 1) * t->stride[i];
    return (last + 1) * esize;
}

bool overlaps_e(const attn_tensor_t* a, int64_t ea, const attn_tensor_t* b, int64_t eb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a->data), a1 = a0 + span_bytes_e(a, ea);
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(b->data), b1 = b0 + span_bytes_e(b, eb);
    return a0 < b1 && b0 < a1;
}
}  // namespace

extern "C" {

attn_status_t attn_fwd_fp8(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v_t, float q_scale,
                           float k_scale, float v_scale, int causal, float scale, attn_tensor_t* out, float* lse,
                           cudaStream_t stream) {
    if (q == nullptr || k == nullptr || v_t == nullptr || out == nullptr) return ATTN_ERR_INVALID_ARG;
    if (q->dtype != ATTN_E4M3 || k->dtype != ATTN_E4M3 || v_t->dtype != ATTN_E4M3) return ATTN_ERR_UNSUPPORTED;
    if (!is_half_type(out->dtype)) return ATTN_ERR_UNSUPPORTED;
    for (float f : {q_scale, k_scale, v_scale, scale})
        if (!std::isfinite(f)) return ATTN_ERR_INVALID_ARG;
    if (q_scale <= 0.f || k_scale <= 0.f || v_scale <= 0.f) return ATTN_ERR_INVALID_ARG;
    attn_status_t st;
    if ((st = check_e4m3(q)) != ATTN_OK || (st = check_e4m3(k)) != ATTN_OK || (st = check_e4m3(v_t)) != ATTN_OK)
        return st;
    if ((st = check_tensor(out, 4)) != ATTN_OK) return st;
    if (!same_shape(q, out) || !same_bhd(q, k)) return ATTN_ERR_INVALID_ARG;
    // V transposed: [B, H, d, Nk]
    if (v_t->shape[0] != k->shape[0] || v_t->shape[1] != k->shape[1] || v_t->shape[2] != k->shape[3] ||
        v_t->shape[3] != k->shape[2])
        return ATTN_ERR_INVALID_ARG;
    const int64_t B = q->shape[0], H = q->shape[1], N = q->shape[2], Nk = k->shape[2], d = q->shape[3];
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (N > (int64_t(1) << 30) || Nk > (int64_t(1) << 30) || B * H > (int64_t(1) << 24)) return ATTN_ERR_UNSUPPORTED;
    if (overlaps_e(out, 2, q, 1) || overlaps_e(out, 2, k, 1) || overlaps_e(out, 2, v_t, 1)) return ATTN_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_INVALID_ARG;

    Maps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!encode_map(kMapE4m3, &maps.q, q, 128) || !encode_map(kMapE4m3, &maps.k, k, 128) ||
        !encode_map(kMapE4m3Vt, &maps.v, v_t, 128))
        return ATTN_ERR_CUDA;
    unsigned int* status = status_word_ptr();
    if (status == nullptr) return ATTN_ERR_CUDA;
    FwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = static_cast<int>(B);
    p.H = static_cast<int>(H);
    p.N = static_cast<int>(N);
    p.Nk = static_cast<int>(Nk);
    p.causal_off = static_cast<int>(Nk - N);
    p.num_q_pairs = static_cast<int>((N + attn::kRowsPerUnit - 1) / attn::kRowsPerUnit);
    p.n_kv_tiles = static_cast<int>((Nk + attn::kBlockN - 1) / attn::kBlockN);
    const int64_t units = static_cast<int64_t>(p.num_q_pairs) * B * H;
    if (units > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
    p.num_units = static_cast<int>(units);
    // the query and key scales fold into the score scale; the value scale into the epilogue
    const double s_all = static_cast<double>(scale) * q_scale * k_scale;
    p.scale = static_cast<float>(s_all);
    p.scale_log2 = static_cast<float>(s_all * 1.4426950408889634);
    p.v_scale = v_scale;
    {
        const double kv_bytes = 2.0 * static_cast<double>(B * H) * static_cast<double>(Nk) * d;
        const int sms = sm_count();
        int g = static_cast<int>(B * H);
        if (sms > 0 && kv_bytes > static_cast<double>(l2_bytes())) g = (sms + p.num_q_pairs - 1) / p.num_q_pairs;
        p.head_group = g < 1 ? 1 : (g > B * H ? static_cast<int>(B * H) : g);
    }
    p.out = out->data;
    p.out_sb = out->stride[0];
    p.out_sh = out->stride[1];
    p.out_si = out->stride[2];
    p.lse = lse;
    p.lse_sh = N;
    p.lse_sb = H * N;
    p.window_left = -1;
    p.wait_limit = g_wait_limit;
    p.status = status;
    p.inject_stall = g_inject_stall;
    cudaError_t e;
    const bool bf = out->dtype == ATTN_BF16;
    if (d == 64)
        e = bf ? (causal ? launch_fp8_t<__nv_bfloat16, 64, true>(maps, p, stream) : launch_fp8_t<__nv_bfloat16, 64, false>(maps, p, stream))
               : (causal ? launch_fp8_t<__half, 64, true>(maps, p, stream) : launch_fp8_t<__half, 64, false>(maps, p, stream));
    else
        e = bf ? (causal ? launch_fp8_t<__nv_bfloat16, 128, true>(maps, p, stream) : launch_fp8_t<__nv_bfloat16, 128, false>(maps, p, stream))
               : (causal ? launch_fp8_t<__half, 128, true>(maps, p, stream) : launch_fp8_t<__half, 128, false>(maps, p, stream));
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"