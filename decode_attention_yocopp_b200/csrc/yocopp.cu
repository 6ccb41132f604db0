// yocopp C ABI: host-side argument checks, TMA descriptor encoding, split
// planning and kernel launches for the YOCO++ compose/append and the shared-
// cache decode attention.  One translation unit holds every kernel so the
// device status word is a single symbol.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "compose_append.cuh"
#include "decode_attn.cuh"
#include "decode_attn_tc.cuh"
#include "prefill_attn_tc.cuh"

namespace yocopp {
namespace {

constexpr int kMaxBatch = 8192;
constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s

// Process-wide settings written by the setters below and read at every launch;
// atomics, since launches may run on other host threads (relaxed: each value
// stands alone).
std::atomic<int> g_test_drop_tile{-1};
std::atomic<int> g_test_prefetch{1};
std::atomic<int> g_decode_kernel{0};  // 0 / 2: tensor-core scores where supported, 1: CUDA-core scores
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elem_bytes(int dtype) { return dtype == YOCOPP_BF16 ? 2 : (dtype == YOCOPP_F32 ? 4 : 0); }

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

int sm_count(int dev) {
    static int cache[kMaxDevices] = {0};
    if (dev < 0 || dev >= kMaxDevices) return -1;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
        cache[dev] = n;
    }
    return cache[dev];
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

// 2-D view of a cache (or query) tensor: rows of head_dim elements; 128-byte
// swizzled boxes of (128 / elem) x box_rows.
bool encode_rows(CUtensorMap* map, const void* base, int dtype, int head_dim, int64_t rows, int box_rows) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    const int eb = elem_bytes(dtype);
    cuuint64_t gdim[2] = {cuuint64_t(head_dim), cuuint64_t(rows)};
    cuuint64_t gstride[1] = {cuuint64_t(head_dim) * eb};
    cuuint32_t box[2] = {cuuint32_t(128 / eb), cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dtype == YOCOPP_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
              const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shape checks shared by both entry points; returns YOCOPP_OK or an error.
int32_t check_cache(const yocopp_cache* c) {
    if (c == nullptr || c->k == nullptr || c->v == nullptr) return YOCOPP_EINVAL;
    if (elem_bytes(c->dtype) == 0) return YOCOPP_EDTYPE;
    if (c->head_dim != 64 && c->head_dim != 128) return YOCOPP_EINVAL;
    if (c->batch < 1 || c->batch > kMaxBatch || c->num_kv_heads < 1 || c->capacity < 1) return YOCOPP_EINVAL;
    if (!aligned(c->k, 16) || !aligned(c->v, 16)) return YOCOPP_EINVAL;
    int64_t rows;
    if (c->block_table != nullptr) {
        const int bs = c->block_size;
        if (bs != 16 && bs != 32 && bs != 64 && bs != 128 && bs != 256) return YOCOPP_EINVAL;
        if (c->max_blocks_per_seq < 1 || c->num_blocks < 1) return YOCOPP_EINVAL;
        if (int64_t(bs) * c->max_blocks_per_seq != c->capacity) return YOCOPP_EINVAL;
        rows = int64_t(c->num_blocks) * c->num_kv_heads * bs;
    } else {
        rows = int64_t(c->batch) * c->num_kv_heads * c->capacity;
    }
    if (rows >= (int64_t(1) << 31)) return YOCOPP_EINVAL;  // 32-bit row coordinates
    return YOCOPP_OK;
}

int32_t cuda_status(cudaError_t e) { return e == cudaSuccess ? YOCOPP_OK : YOCOPP_ECUDA; }

// ---------------------------------------------------------------- compose
template <typename T, int ROWB>
int32_t launch_compose(ComposeParams& p, cudaStream_t st) {
    const int dev = current_device();
    const int sms = sm_count(dev);
    if (sms <= 0) return YOCOPP_ECUDA;
    const int64_t nchunks = p.total_rows * (ROWB / 16);
    constexpr int64_t per_cta = int64_t(YOCOPP_COMPOSE_THREADS) * YOCOPP_COMPOSE_UNROLL;
    int64_t grid = (nchunks + per_cta - 1) / per_cta;
    if (grid > int64_t(sms) * YOCOPP_COMPOSE_CTAS_PER_SM) grid = int64_t(sms) * YOCOPP_COMPOSE_CTAS_PER_SM;
    if (grid < 1) grid = 1;
    const size_t smem = p.cu_new ? size_t(p.batch + 1) * sizeof(int) : 0;
    compose_append_kernel<T, ROWB><<<unsigned(grid), YOCOPP_COMPOSE_THREADS, smem, st>>>(p);
    return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------- decode
// Launch shape of the split kernel: consumer warps per CTA, pipeline stages,
// CTAs per SM (compile-time; the defaults are the measured best on B200).
#ifndef YOCOPP_DECODE_WARPS
#define YOCOPP_DECODE_WARPS 4
#endif
#ifndef YOCOPP_DECODE_STAGES
#define YOCOPP_DECODE_STAGES 3
#endif
#ifndef YOCOPP_DECODE_CTAS_PER_SM
#define YOCOPP_DECODE_CTAS_PER_SM 2
#endif
// Split plan: what closing a segment (flush, arrival, merge) costs a CTA, in tiles.
#ifndef YOCOPP_DECODE_SEG_UNITS
#define YOCOPP_DECODE_SEG_UNITS 3
#endif

struct DecodeLaunch {
    int w, stages, tile, ctas_per_sm;
};

template <typename T, int D, bool FUSED>
constexpr DecodeLaunch decode_cfg() {
    return DecodeLaunch{YOCOPP_DECODE_WARPS, YOCOPP_DECODE_STAGES, DecodeShape<D, T, FUSED>::TILE,
                        YOCOPP_DECODE_CTAS_PER_SM};
}

template <typename T, int D, int G, bool FUSED>
int32_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tk1, const CUtensorMap& tv1,
                      const DecodeParams& p, cudaStream_t st) {
    constexpr DecodeLaunch cfg = decode_cfg<T, D, FUSED>();
    constexpr int W = cfg.w, STAGES = cfg.stages;
    auto kern = decode_split_kernel<T, D, G, W, STAGES, cfg.ctas_per_sm, FUSED>;
    const size_t smem = DecodeSmem<T, D, G, W, STAGES, FUSED>::bytes(p.batch);
    static bool attr_set[kMaxDevices] = {false};
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return YOCOPP_ECUDA;
    static size_t max_dyn[kMaxDevices] = {0};
    if (!attr_set[dev]) {
        int maxopt = 0;
        cudaFuncAttributes fa;
        if (cudaDeviceGetAttribute(&maxopt, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
            return YOCOPP_ECUDA;
        max_dyn[dev] = size_t(maxopt) - fa.sharedSizeBytes;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(max_dyn[dev])) != cudaSuccess)
            return YOCOPP_ECUDA;
        attr_set[dev] = true;
    }
    if (smem > max_dyn[dev]) return YOCOPP_EINVAL;  // batch too large for the shared-memory plan
    // launched as a programmatic dependent of the previous kernel in the stream:
    // its launch and prologue overlap that kernel's tail (it waits before reading inputs)
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(unsigned(p.num_ctas), 1, 1);
    lc.blockDim = dim3((W + 1) * 32, 1, 1);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&lc, kern, tk, tv, tk1, tv1, p));
}

template <int G>
int32_t launch_decode_tc(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq, const DecodeParams& p,
                         cudaStream_t st) {
    constexpr int STAGES = 3;
    auto kern = decode_tc_kernel<G, STAGES>;
    const size_t smem = TcSmem<G, STAGES>::bytes(p.batch);
    static bool attr_set[kMaxDevices] = {false};
    static size_t max_dyn[kMaxDevices] = {0};
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return YOCOPP_ECUDA;
    if (!attr_set[dev]) {
        int maxopt = 0;
        cudaFuncAttributes fa;
        if (cudaDeviceGetAttribute(&maxopt, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
            return YOCOPP_ECUDA;
        max_dyn[dev] = size_t(maxopt) - fa.sharedSizeBytes;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(max_dyn[dev])) != cudaSuccess)
            return YOCOPP_ECUDA;
        attr_set[dev] = true;
    }
    if (smem > max_dyn[dev]) return YOCOPP_EINVAL;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(unsigned(p.num_ctas), 1, 1);
    lc.blockDim = dim3(TcShape::THREADS, 1, 1);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&lc, kern, tk, tv, tq, p));
}

// ---------------------------------------------------------------- prefill
// 3-D view of token-major queries [rows][heads][head_dim] (bf16): one box is
// 64 channels x 1 head x box_rows tokens, 128-byte swizzled.
bool encode_q3d(CUtensorMap* map, const void* base, int heads, int head_dim, int64_t rows, int box_rows) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3] = {cuuint64_t(head_dim), cuuint64_t(heads), cuuint64_t(rows)};
    cuuint64_t gstride[2] = {cuuint64_t(head_dim) * 2, cuuint64_t(heads) * head_dim * 2};
    cuuint32_t box[3] = {64, 1, cuuint32_t(box_rows)};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool FUSED>
int32_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const PrefillParams& p,
                       int64_t grid, cudaStream_t st) {
    auto kern = prefill_tc_kernel<FUSED>;
    static bool attr_set[kMaxDevices] = {false};
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return YOCOPP_ECUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PfShape::SMEM) != cudaSuccess)
            return YOCOPP_ECUDA;
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(unsigned(grid), 1, 1);
    lc.blockDim = dim3(PfShape::THREADS, 1, 1);
    lc.dynamicSmemBytes = PfShape::SMEM;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&lc, kern, tq, tk, tv, p));
}

// Decode workspace: a 256-byte header (call generation + call arrivals), the
// split partials m [slots][G], l [slots][G], o [slots][G][D] (fp32) from offset
// 256 upwards, and the per-plane arrival counters at the END of the buffer.
// Slots are sized for the larger of the two decode grids (plane + CTA index),
// so the partials' extent depends only on (planes, G, D) and grows with the
// plane count.  Counters of a call therefore never land on bytes an earlier
// call with the same G and D (and the same buffer size) used for partials:
// a call with more planes has its counters lower down, but its partials, and
// every earlier call's, end below them.
struct WorkspaceLayout {
    size_t gen, m, l, o, partial_end, cnt;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// planes = batch * hkv; max_ctas = the larger decode grid; buf_bytes = the
// buffer's size; cnt_words = counter words reserved at its end (>= planes).
WorkspaceLayout workspace_layout(size_t planes, int G, int D, int max_ctas, size_t buf_bytes, size_t cnt_words) {
    const size_t slots = size_t(max_ctas) + planes;
    WorkspaceLayout w;
    w.gen = 0;
    w.m = 256;
    w.l = w.m + up256(slots * G * sizeof(float));
    w.o = w.l + up256(slots * G * sizeof(float));
    w.partial_end = w.o + up256(slots * G * D * sizeof(float));
    const size_t cnt_bytes = up256(cnt_words * sizeof(unsigned long long));
    const size_t top = buf_bytes & ~size_t(255);
    w.cnt = top >= cnt_bytes ? top - cnt_bytes : 0;
    return w;
}

// Bytes yocopp_decode_attn_workspace_size reports: partials plus the counters right after.
size_t workspace_bytes_needed(size_t planes, int G, int D, int max_ctas) {
    const WorkspaceLayout w = workspace_layout(planes, G, D, max_ctas, 0, 0);
    return w.partial_end + up256(planes * sizeof(unsigned long long));
}

int32_t check_decode_shape(const yocopp_cache* cache, int32_t num_q_heads, int* G) {
    const int32_t rc = check_cache(cache);
    if (rc != YOCOPP_OK) return rc;
    if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads != 0) return YOCOPP_EINVAL;
    *G = num_q_heads / cache->num_kv_heads;
    if (*G != 1 && *G != 2 && *G != 4) return YOCOPP_EINVAL;
    const int tile = (cache->head_dim * elem_bytes(cache->dtype)) <= 256 ? 64 : 32;
    if (cache->block_table != nullptr && cache->block_size % tile != 0 && tile % cache->block_size != 0)
        return YOCOPP_EINVAL;
    const int64_t tiles = int64_t(cache->batch) * cache->num_kv_heads * ((cache->capacity + tile - 1) / tile);
    if (tiles >= (int64_t(1) << 31)) return YOCOPP_EINVAL;
    return YOCOPP_OK;
}

}  // namespace

// ---------------------------------------------------------------- decode without allocation
// Scratch for yocopp_decode_attn_static: a fixed device array in this library's
// image, so callers that cannot allocate device memory still get a workspace.
// Every device that loads the library holds it until the process exits.
constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr size_t kStaticCounterWords = 8192;              // planes (batch x kv heads) a static call may have
static __device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

namespace {
// Device address of g_decode_scratch per device, looked up once with that
// device current (host code must not pass the symbol itself to a kernel).
void* static_scratch_ptr(int dev) {
    static std::mutex mu;
    static void* ptrs[kMaxDevices] = {nullptr};
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
        ptrs[dev] = p;
    }
    return ptrs[dev];
}
}  // namespace
}  // namespace yocopp

using namespace yocopp;

extern "C" {

int32_t yocopp_version(void) { return 100; }

const char* yocopp_status_string(int32_t s) {
    switch (s) {
        case YOCOPP_OK: return "YOCOPP_OK";
        case YOCOPP_EINVAL: return "YOCOPP_EINVAL";
        case YOCOPP_EDTYPE: return "YOCOPP_EDTYPE";
        case YOCOPP_ECAPACITY: return "YOCOPP_ECAPACITY";
        case YOCOPP_EWORKSPACE: return "YOCOPP_EWORKSPACE";
        case YOCOPP_ECUDA: return "YOCOPP_ECUDA";
        case YOCOPP_EDEVICE_CHECK: return "YOCOPP_EDEVICE_CHECK";
        case YOCOPP_ETIMEOUT: return "YOCOPP_ETIMEOUT";
        default: return "YOCOPP_UNKNOWN";
    }
}

int32_t yocopp_get_device_status(int32_t reset) {
    int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return YOCOPP_ECUDA;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return YOCOPP_ECUDA;
    if (reset) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return YOCOPP_ECUDA;
    }
    return v;
}

int32_t yocopp_set_decode_kernel(int32_t which) {
    if (which < 0 || which > 2) return YOCOPP_EINVAL;
    g_decode_kernel.store(which, std::memory_order_relaxed);
    return YOCOPP_OK;
}

int32_t yocopp_testing_set_decode_fault(int32_t drop_tile, int64_t wait_limit_ns) {
    if (wait_limit_ns <= 0) return YOCOPP_EINVAL;
    g_test_drop_tile.store(drop_tile < 0 ? -1 : drop_tile, std::memory_order_relaxed);
    g_wait_limit_ns.store(uint64_t(wait_limit_ns), std::memory_order_relaxed);
    return YOCOPP_OK;
}

int32_t yocopp_testing_set_decode_prefetch(int32_t enabled) {
    if (enabled != 0 && enabled != 1) return YOCOPP_EINVAL;
    g_test_prefetch.store(enabled, std::memory_order_relaxed);
    return YOCOPP_OK;
}

int32_t yocopp_compose_append(const void* K1, const void* V1, const void* Ki, const void* Vi,
                              const float alpha[4], float lambda, const yocopp_cache* cache,
                              const int32_t* pos, const int32_t* cu_new, int32_t n_uniform,
                              int64_t total_new, void* stream) {
    const int32_t rc = check_cache(cache);
    if (rc != YOCOPP_OK) return rc;
    if (alpha == nullptr || pos == nullptr || total_new < 0) return YOCOPP_EINVAL;
    if (!std::isfinite(lambda) || !std::isfinite(alpha[0]) || !std::isfinite(alpha[1]) ||
        !std::isfinite(alpha[2]) || !std::isfinite(alpha[3]))
        return YOCOPP_EINVAL;
    if (cu_new == nullptr) {
        if (n_uniform < 0 || int64_t(n_uniform) * cache->batch != total_new) return YOCOPP_EINVAL;
    }
    if (total_new == 0) return YOCOPP_OK;
    if (K1 == nullptr || V1 == nullptr || Ki == nullptr || Vi == nullptr) return YOCOPP_EINVAL;
    if (!aligned(K1, 16) || !aligned(V1, 16) || !aligned(Ki, 16) || !aligned(Vi, 16)) return YOCOPP_EINVAL;
    if (total_new > (int64_t(1) << 40)) return YOCOPP_EINVAL;

    ComposeParams p;
    p.k1 = static_cast<const uint8_t*>(K1);
    p.v1 = static_cast<const uint8_t*>(V1);
    p.ki = static_cast<const uint8_t*>(Ki);
    p.vi = static_cast<const uint8_t*>(Vi);
    p.ck = static_cast<uint8_t*>(cache->k);
    p.cv = static_cast<uint8_t*>(cache->v);
    p.block_table = cache->block_table;
    p.pos = pos;
    p.cu_new = cu_new;
    p.ak1 = alpha[0];
    p.ak2 = alpha[1];
    p.av1 = alpha[2];
    p.av2 = alpha[3];
    p.lam = lambda;
    p.total_rows = total_new * cache->num_kv_heads;
    p.hkv = cache->num_kv_heads;
    p.batch = cache->batch;
    p.n_uniform = n_uniform;
    p.capacity = cache->capacity;
    p.block_size = cache->block_table ? cache->block_size : 0;
    p.mbps = cache->block_table ? cache->max_blocks_per_seq : 0;
    p.num_blocks = cache->block_table ? cache->num_blocks : 0;
    const FastDiv dh = make_fast_div(uint32_t(cache->num_kv_heads)), dn = make_fast_div(uint32_t(n_uniform > 0 ? n_uniform : 1));
    p.hkv_m = dh.m;
    p.hkv_s = dh.s;
    p.nu_m = dn.m;
    p.nu_s = dn.s;
    p.bs_log2 = 0;
    while (cache->block_table && (1 << p.bs_log2) < cache->block_size) ++p.bs_log2;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int rowb = cache->head_dim * elem_bytes(cache->dtype);
    if (cache->dtype == YOCOPP_BF16)
        return rowb == 256 ? launch_compose<__nv_bfloat16, 256>(p, st) : launch_compose<__nv_bfloat16, 128>(p, st);
    return rowb == 512 ? launch_compose<float, 512>(p, st) : launch_compose<float, 256>(p, st);
}

int64_t yocopp_decode_attn_workspace_size(const yocopp_cache* cache, int32_t num_q_heads) {
    int G = 0;
    const int32_t rc = check_decode_shape(cache, num_q_heads, &G);
    if (rc != YOCOPP_OK) return rc;
    const int sms = sm_count(current_device());
    if (sms <= 0) return YOCOPP_ECUDA;
    return int64_t(workspace_bytes_needed(size_t(cache->batch) * cache->num_kv_heads, G, cache->head_dim,
                                          sms * YOCOPP_DECODE_CTAS_PER_SM));
}

// fused != nullptr: the read-time composition variant; `cache` holds raw K_i, V_i,
// fused->cache1 raw K_1, V_1 (same shape and layout), fused->coef = lambda * alpha.
struct FusedArgs {
    const yocopp_cache* cache1;
    float coef[4];
};

// cnt_words: arrival-counter words reserved at the end of the workspace (0: one per
// plane of this call, the caller-workspace layout).
static int32_t decode_attn_impl(const void* q, const yocopp_cache* cache, const int32_t* seq_lens, void* out,
                                float* part_out, int32_t num_q_heads, float scale, void* workspace,
                                int64_t workspace_bytes, void* stream, const FusedArgs* fused = nullptr,
                                size_t cnt_words = 0) {
    int G = 0;
    int32_t rc = check_decode_shape(cache, num_q_heads, &G);
    if (rc != YOCOPP_OK) return rc;
    if (fused != nullptr) {
        const yocopp_cache* c1 = fused->cache1;
        rc = check_cache(c1);
        if (rc != YOCOPP_OK) return rc;
        if (c1->dtype != cache->dtype || c1->batch != cache->batch || c1->num_kv_heads != cache->num_kv_heads ||
            c1->head_dim != cache->head_dim || c1->capacity != cache->capacity ||
            c1->block_table != cache->block_table ||
            (cache->block_table != nullptr && (c1->block_size != cache->block_size ||
                                               c1->max_blocks_per_seq != cache->max_blocks_per_seq ||
                                               c1->num_blocks != cache->num_blocks)))
            return YOCOPP_EINVAL;
    }
    if (q == nullptr || (out == nullptr && part_out == nullptr) || seq_lens == nullptr) return YOCOPP_EINVAL;
    if (!aligned(q, 16) || !aligned(out != nullptr ? out : static_cast<void*>(part_out), 16)) return YOCOPP_EINVAL;
    if (!(scale >= 0.f) || !std::isfinite(scale)) return YOCOPP_EINVAL;
    const int sms = sm_count(current_device());
    if (sms <= 0) return YOCOPP_ECUDA;
    // tensor-core scores: bf16, head_dim 128, no read-time composition, block size >= 16, and the
    // batch's tile table fits next to the 3-stage ring
    const bool use_tc = g_decode_kernel.load(std::memory_order_relaxed) != 1 && fused == nullptr && cache->dtype == YOCOPP_BF16 &&
                        cache->head_dim == 128 && TcSmem<4, 3>::bytes(cache->batch) <= 232448 - 1024;
    const int num_ctas = use_tc ? sms : sms * YOCOPP_DECODE_CTAS_PER_SM;
    const size_t planes = size_t(cache->batch) * cache->num_kv_heads;
    if (cnt_words == 0) cnt_words = planes;
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes <= 0 || cnt_words < planes)
        return YOCOPP_EWORKSPACE;
    const WorkspaceLayout wl = workspace_layout(planes, G, cache->head_dim, sms * YOCOPP_DECODE_CTAS_PER_SM,
                                                size_t(workspace_bytes), cnt_words);
    if (wl.cnt < wl.partial_end) return YOCOPP_EWORKSPACE;

    const int D = cache->head_dim;
    const int tile = use_tc ? TcShape::TILE : ((D * elem_bytes(cache->dtype)) <= 256 ? 64 : 32) / (fused != nullptr ? 2 : 1);
    const bool paged = cache->block_table != nullptr;
    const int boxr = paged ? (cache->block_size < tile ? cache->block_size : tile) : tile;
    const int64_t rows = paged ? int64_t(cache->num_blocks) * cache->num_kv_heads * cache->block_size
                               : int64_t(cache->batch) * cache->num_kv_heads * cache->capacity;
    alignas(64) CUtensorMap tk, tv, tk1, tv1;
    if (!encode_rows(&tk, cache->k, cache->dtype, D, rows, boxr) ||
        !encode_rows(&tv, cache->v, cache->dtype, D, rows, boxr))
        return YOCOPP_ECUDA;
    if (fused != nullptr) {
        if (!encode_rows(&tk1, fused->cache1->k, cache->dtype, D, rows, boxr) ||
            !encode_rows(&tv1, fused->cache1->v, cache->dtype, D, rows, boxr))
            return YOCOPP_ECUDA;
    } else {
        tk1 = tk;
        tv1 = tv;
    }

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    DecodeParams p;
    p.q = static_cast<const uint8_t*>(q);
    p.out = static_cast<uint8_t*>(out);
    p.seq_lens = seq_lens;
    p.block_table = cache->block_table;
    p.ws_gen = reinterpret_cast<unsigned long long*>(ws + wl.gen);
    p.ws_cnt = reinterpret_cast<unsigned long long*>(ws + wl.cnt);
    p.ws_m = reinterpret_cast<float*>(ws + wl.m);
    p.ws_l = reinterpret_cast<float*>(ws + wl.l);
    p.ws_o = reinterpret_cast<float*>(ws + wl.o);
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(float(D));
    p.qscale = sc * 1.4426950408889634f;
    p.batch = cache->batch;
    p.hkv = cache->num_kv_heads;
    p.hq = num_q_heads;
    p.capacity = cache->capacity;
    p.block_size = paged ? cache->block_size : 0;
    p.mbps = paged ? cache->max_blocks_per_seq : 0;
    p.num_blocks = paged ? cache->num_blocks : 0;
    p.boxr = boxr;
    p.num_ctas = num_ctas;
    p.seg_units = YOCOPP_DECODE_SEG_UNITS;
    p.drop_tile = g_test_drop_tile.load(std::memory_order_relaxed);
    p.prefetch = g_test_prefetch.load(std::memory_order_relaxed);
    p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    p.part_out = part_out;
    p.fa1k = fused ? fused->coef[0] : 0.f;
    p.fa2k = fused ? fused->coef[1] : 0.f;
    p.fa1v = fused ? fused->coef[2] : 0.f;
    p.fa2v = fused ? fused->coef[3] : 0.f;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (use_tc) {
        alignas(64) CUtensorMap tq;
        if (!encode_rows(&tq, q, cache->dtype, D, int64_t(cache->batch) * num_q_heads, TcShape::QROWS))
            return YOCOPP_ECUDA;
        switch (G) {
            case 1: return launch_decode_tc<1>(tk, tv, tq, p, st);
            case 2: return launch_decode_tc<2>(tk, tv, tq, p, st);
            default: return launch_decode_tc<4>(tk, tv, tq, p, st);
        }
    }

#define YOCOPP_DECODE_CASE(TT, DD, FF)                                                 \
    switch (G) {                                                                       \
        case 1: return launch_decode<TT, DD, 1, FF>(tk, tv, tk1, tv1, p, st);          \
        case 2: return launch_decode<TT, DD, 2, FF>(tk, tv, tk1, tv1, p, st);          \
        default: return launch_decode<TT, DD, 4, FF>(tk, tv, tk1, tv1, p, st);         \
    }
    if (fused != nullptr) {
        if (cache->dtype == YOCOPP_BF16) {
            if (D == 128) { YOCOPP_DECODE_CASE(__nv_bfloat16, 128, true) }
            YOCOPP_DECODE_CASE(__nv_bfloat16, 64, true)
        }
        if (D == 128) { YOCOPP_DECODE_CASE(float, 128, true) }
        YOCOPP_DECODE_CASE(float, 64, true)
    }
    if (cache->dtype == YOCOPP_BF16) {
        if (D == 128) { YOCOPP_DECODE_CASE(__nv_bfloat16, 128, false) }
        YOCOPP_DECODE_CASE(__nv_bfloat16, 64, false)
    }
    if (D == 128) { YOCOPP_DECODE_CASE(float, 128, false) }
    YOCOPP_DECODE_CASE(float, 64, false)
#undef YOCOPP_DECODE_CASE
}

int32_t yocopp_decode_attn(const void* q, const yocopp_cache* cache, const int32_t* seq_lens, void* out,
                           int32_t num_q_heads, float scale, void* workspace, int64_t workspace_bytes,
                           void* stream) {
    if (out == nullptr) return YOCOPP_EINVAL;
    return decode_attn_impl(q, cache, seq_lens, out, nullptr, num_q_heads, scale, workspace, workspace_bytes,
                            stream);
}

int32_t yocopp_decode_attn_partial(const void* q, const yocopp_cache* cache, const int32_t* seq_lens,
                                   float* partial, int32_t num_q_heads, float scale, void* workspace,
                                   int64_t workspace_bytes, void* stream) {
    if (partial == nullptr) return YOCOPP_EINVAL;
    return decode_attn_impl(q, cache, seq_lens, nullptr, partial, num_q_heads, scale, workspace,
                            workspace_bytes, stream);
}

int32_t yocopp_decode_attn_fused(const void* q, const yocopp_cache* cache_i, const yocopp_cache* cache_1,
                                 const float alpha[4], float lambda, const int32_t* seq_lens, void* out,
                                 int32_t num_q_heads, float scale, void* workspace, int64_t workspace_bytes,
                                 void* stream) {
    if (out == nullptr || alpha == nullptr || cache_1 == nullptr) return YOCOPP_EINVAL;
    if (!std::isfinite(lambda) || !std::isfinite(alpha[0]) || !std::isfinite(alpha[1]) ||
        !std::isfinite(alpha[2]) || !std::isfinite(alpha[3]))
        return YOCOPP_EINVAL;
    FusedArgs f;
    f.cache1 = cache_1;
    for (int j = 0; j < 4; ++j) f.coef[j] = lambda * alpha[j];
    return decode_attn_impl(q, cache_i, seq_lens, out, nullptr, num_q_heads, scale, workspace, workspace_bytes,
                            stream, &f);
}

int32_t yocopp_decode_combine(const float* partials, int32_t num_parts, int64_t rows, int32_t head_dim,
                              int32_t dtype, void* out, void* stream) {
    if (partials == nullptr || out == nullptr || num_parts < 1 || rows < 0) return YOCOPP_EINVAL;
    if (elem_bytes(dtype) == 0) return YOCOPP_EDTYPE;
    if (head_dim != 64 && head_dim != 128) return YOCOPP_EINVAL;
    if (rows == 0) return YOCOPP_OK;
    if (rows > (int64_t(1) << 31) - 1) return YOCOPP_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* o = static_cast<uint8_t*>(out);
    if (dtype == YOCOPP_BF16) {
        if (head_dim == 128) combine_parts_kernel<__nv_bfloat16, 128><<<unsigned(rows), 128, 0, st>>>(partials, num_parts, rows, o);
        else combine_parts_kernel<__nv_bfloat16, 64><<<unsigned(rows), 64, 0, st>>>(partials, num_parts, rows, o);
    } else {
        if (head_dim == 128) combine_parts_kernel<float, 128><<<unsigned(rows), 128, 0, st>>>(partials, num_parts, rows, o);
        else combine_parts_kernel<float, 64><<<unsigned(rows), 64, 0, st>>>(partials, num_parts, rows, o);
    }
    return cuda_status(cudaGetLastError());
}

// Decode attention whose workspace is the library's own static device array
// (no allocation anywhere).  Argument meaning as yocopp_decode_attn.
// The counter region sits at a fixed place (the array's last kStaticCounterWords
// words) whatever the shape, so no call's partials ever overlap another call's
// counters.
int32_t yocopp_decode_attn_static(const void* q, const yocopp_cache* cache, const int32_t* seq_lens, void* out,
                                  int32_t num_q_heads, float scale, void* stream) {
    const int64_t need = yocopp_decode_attn_workspace_size(cache, num_q_heads);
    if (need < 0) return int32_t(need);
    if (out == nullptr) return YOCOPP_EINVAL;
    if (int64_t(cache->batch) * cache->num_kv_heads > int64_t(kStaticCounterWords)) return YOCOPP_EWORKSPACE;
    void* scratch = static_scratch_ptr(current_device());
    if (scratch == nullptr) return YOCOPP_ECUDA;
    // too large a shape fails the partials-below-counters check with YOCOPP_EWORKSPACE
    return decode_attn_impl(q, cache, seq_lens, out, nullptr, num_q_heads, scale, scratch,
                            int64_t(kStaticScratchBytes), stream, nullptr, kStaticCounterWords);
}

// Causal prefill attention of a self-decoder layer over its own cache
// (tcgen05 for both products); with `fused`, the same launch first composes
// the rows it attends over from raw inputs.  Argument meaning in yocopp.h.
struct PrefillFused {
    const void *k1, *v1, *ki, *vi;
    const float* alpha;
    float lambda;
    void* workspace;
    int64_t workspace_bytes;
};

static int64_t prefill_fused_ws_bytes(int32_t batch, int q_tiles) {
    return int64_t(256) + ((int64_t(batch) * q_tiles * 8 + 255) & ~int64_t(255));
}

static int32_t prefill_attn_impl(const void* q, const yocopp_cache* cache, const int32_t* pos, const int32_t* cu_q,
                                 int32_t n_uniform, int64_t total_q, int32_t max_q, void* out, int32_t num_q_heads,
                                 float scale, void* stream, const PrefillFused* fused) {
    const int32_t rc = check_cache(cache);
    if (rc != YOCOPP_OK) return rc;
    if (cache->dtype != YOCOPP_BF16) return YOCOPP_EDTYPE;
    if (cache->head_dim != 128) return YOCOPP_EINVAL;
    const bool paged = cache->block_table != nullptr;
    if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads != 0) return YOCOPP_EINVAL;
    if (q == nullptr || out == nullptr || !aligned(q, 16) || !aligned(out, 16)) return YOCOPP_EINVAL;
    if (!(scale >= 0.f) || !std::isfinite(scale)) return YOCOPP_EINVAL;
    if (total_q < 0 || total_q >= (int64_t(1) << 31)) return YOCOPP_EINVAL;
    if (cu_q == nullptr) {
        if (n_uniform < 0 || int64_t(n_uniform) * cache->batch != total_q) return YOCOPP_EINVAL;
        max_q = n_uniform;
    } else if (max_q < 0) {
        return YOCOPP_EINVAL;
    }
    if (int64_t(max_q) > int64_t(cache->capacity)) return YOCOPP_EINVAL;
    const int64_t rows = paged ? int64_t(cache->num_blocks) * cache->num_kv_heads * cache->block_size
                               : int64_t(cache->batch) * cache->num_kv_heads * cache->capacity;
    if (rows + PfShape::TK >= (int64_t(1) << 31)) return YOCOPP_EINVAL;  // tile row coordinates stay 32-bit
    const int boxr = paged ? (cache->block_size < PfShape::TK ? cache->block_size : PfShape::TK) : PfShape::TK;
    const int q_tiles = (max_q + PfShape::TQ - 1) / PfShape::TQ;
    if (fused != nullptr) {
        if (fused->alpha == nullptr || !std::isfinite(fused->lambda) || !std::isfinite(fused->alpha[0]) ||
            !std::isfinite(fused->alpha[1]) || !std::isfinite(fused->alpha[2]) || !std::isfinite(fused->alpha[3]))
            return YOCOPP_EINVAL;
        if (total_q > 0 && (fused->k1 == nullptr || fused->v1 == nullptr || fused->ki == nullptr ||
                            fused->vi == nullptr || !aligned(fused->k1, 16) || !aligned(fused->v1, 16) ||
                            !aligned(fused->ki, 16) || !aligned(fused->vi, 16)))
            return YOCOPP_EINVAL;
        if (fused->workspace == nullptr || !aligned(fused->workspace, 256) ||
            fused->workspace_bytes < prefill_fused_ws_bytes(cache->batch, q_tiles))
            return YOCOPP_EWORKSPACE;
    }
    if (total_q == 0 || max_q == 0) return YOCOPP_OK;
    const int heads_per_cta = (num_q_heads / cache->num_kv_heads) % 2 == 0 ? 2 : 1;
    int64_t grid = int64_t(q_tiles) * cache->batch * (num_q_heads / heads_per_cta);
    if (fused != nullptr) grid += int64_t(q_tiles) * cache->batch;  // the composition CTAs
    if (grid >= (int64_t(1) << 31)) return YOCOPP_EINVAL;
    if (fused != nullptr && grid >= (int64_t(1) << 20)) return YOCOPP_EINVAL;  // the call-arrival count field
    alignas(64) CUtensorMap tq, tk, tv;
    if (!encode_q3d(&tq, q, num_q_heads, 128, total_q, PfShape::TQ) ||
        !encode_rows(&tk, cache->k, YOCOPP_BF16, 128, rows, boxr) ||
        !encode_rows(&tv, cache->v, YOCOPP_BF16, 128, rows, boxr))
        return YOCOPP_ECUDA;
    PrefillParams p = {};
    p.out = static_cast<uint8_t*>(out);
    p.pos = pos;
    p.cu_q = cu_q;
    p.block_table = cache->block_table;
    p.block_size = paged ? cache->block_size : 0;
    p.mbps = paged ? cache->max_blocks_per_seq : 0;
    p.num_blocks = paged ? cache->num_blocks : 0;
    p.boxr = boxr;
    p.n_uniform = cu_q ? 0 : n_uniform;
    p.batch = cache->batch;
    p.hq = num_q_heads;
    p.hkv = cache->num_kv_heads;
    p.capacity = cache->capacity;
    p.q_tiles = q_tiles;
    p.heads_per_cta = heads_per_cta;
    const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(128.f);
    p.qscale = sc * 1.4426950408889634f;
    p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    p.drop_k_tile = g_test_drop_tile.load(std::memory_order_relaxed);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (fused == nullptr) return launch_prefill<false>(tq, tk, tv, p, grid, st);
    p.k1 = static_cast<const uint8_t*>(fused->k1);
    p.v1 = static_cast<const uint8_t*>(fused->v1);
    p.ki = static_cast<const uint8_t*>(fused->ki);
    p.vi = static_cast<const uint8_t*>(fused->vi);
    p.ck = static_cast<uint8_t*>(cache->k);
    p.cv = static_cast<uint8_t*>(cache->v);
    p.ak1 = fused->alpha[0];
    p.ak2 = fused->alpha[1];
    p.av1 = fused->alpha[2];
    p.av2 = fused->alpha[3];
    p.lam = fused->lambda;
    uint8_t* ws = static_cast<uint8_t*>(fused->workspace);
    p.ws_gen = reinterpret_cast<unsigned long long*>(ws);
    p.flags = reinterpret_cast<unsigned long long*>(ws + 256);
    return launch_prefill<true>(tq, tk, tv, p, grid, st);
}

int32_t yocopp_prefill_attn(const void* q, const yocopp_cache* cache, const int32_t* pos, const int32_t* cu_q,
                            int32_t n_uniform, int64_t total_q, int32_t max_q, void* out, int32_t num_q_heads,
                            float scale, void* stream) {
    return prefill_attn_impl(q, cache, pos, cu_q, n_uniform, total_q, max_q, out, num_q_heads, scale, stream,
                             nullptr);
}

int64_t yocopp_prefill_compose_attn_workspace_size(const yocopp_cache* cache, int32_t max_q) {
    if (cache == nullptr || cache->batch < 1 || cache->batch > kMaxBatch || max_q < 0) return YOCOPP_EINVAL;
    return prefill_fused_ws_bytes(cache->batch, (max_q + PfShape::TQ - 1) / PfShape::TQ);
}

int32_t yocopp_prefill_compose_attn(const void* K1, const void* V1, const void* Ki, const void* Vi,
                                    const float alpha[4], float lambda, const void* q, const yocopp_cache* cache,
                                    const int32_t* pos, const int32_t* cu_q, int32_t n_uniform, int64_t total_q,
                                    int32_t max_q, void* out, int32_t num_q_heads, float scale, void* workspace,
                                    int64_t workspace_bytes, void* stream) {
    PrefillFused f;
    f.k1 = K1;
    f.v1 = V1;
    f.ki = Ki;
    f.vi = Vi;
    f.alpha = alpha;
    f.lambda = lambda;
    f.workspace = workspace;
    f.workspace_bytes = workspace_bytes;
    return prefill_attn_impl(q, cache, pos, cu_q, n_uniform, total_q, max_q, out, num_q_heads, scale, stream, &f);
}

}  // extern "C"
