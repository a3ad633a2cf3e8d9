// The C ABI declared in include/mqa_logits.h: host-side checks, tensor-map
// encoding and kernel launches. Nothing here computes logits; every step of
// the path runs in the kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "mqa_logits_diag.h"

namespace mqa {

// defined in diag_gather.cu
int launch_fp8_gather(int D, const LaunchSpec& ls, const CUtensorMap& tm_k, const CUtensorMap& tm_q,
                      const KernelArgs& args);

// defined in schedule.cu
int launch_schedule(const int32_t* context_lens, int batch, int num_ctas, int32_t* schedule,
                    void* stream);
// defined in topk.cu
int launch_topk(const float* logits, const int32_t* context_lens, int batch, int next_n, int L,
                int k, int flags, int32_t* out, float* values, void* stream, int cluster_force);
int launch_topk_merge(const float* cand_values, const int32_t* cand_tokens, int shards, int rows,
                      int k_in, const int32_t* offsets, int k, int flags, int32_t* out,
                      float* values, void* stream);

constexpr int kMaxBatchSchedule = 32768;
constexpr int kMaxCtas = 4096;
constexpr int kMaxStages = 16;  // cap on the MQA_LOGITS_STAGES override
// Default K ring depths (units of 256 tokens).
constexpr int kDefaultStages = 3;     // FP4 kernels (three producer warps)
constexpr int kDefaultStagesFp8 = 5;  // FP8 kernel (one producer, units issued in order)

// The library's own status word: one per device that loads the library
// (each device gets its own copy of a __device__ variable). Logits kernels OR
// MQA_STATUS_* bits into it through the pointer in KernelArgs.
__device__ uint32_t g_lib_status;

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(MQA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Compute capability 10.0 check, cached per device; on the first success on
// a device it also looks up that device's copy of g_lib_status.
int check_arch(int* device_out, uint32_t** lib_status = nullptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    static std::mutex mu;
    static int cache[64];  // 0 unknown, 1 ok, 2 bad
    static uint32_t* status_ptr[64];
    if (dev < 0 || dev >= 64) return fail(MQA_ERR_ARCH, "device index %d out of range", dev);
    {
        std::lock_guard<std::mutex> lk(mu);
        if (cache[dev] == 0) {
            int major = 0, minor = 0;
            e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
            if (e == cudaSuccess)
                e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
            if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
            if (major == 10 && minor == 0) {
                void* p = nullptr;
                e = cudaGetSymbolAddress(&p, g_lib_status);
                if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
                status_ptr[dev] = static_cast<uint32_t*>(p);
                cache[dev] = 1;
            } else {
                cache[dev] = 2;
            }
        }
        if (cache[dev] != 1)
            return fail(MQA_ERR_ARCH, "device %d is not compute capability 10.0 (sm_100a build)", dev);
        if (lib_status) *lib_status = status_ptr[dev];
    }
    if (device_out) *device_out = dev;
    return MQA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tiled map over bytes (uint8 elements) or 16-bit elements; dims[0] innermost.
int encode_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* addr,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
               CUtensorMapSwizzle swz, const char* what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MQA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void*>(addr),
                    reinterpret_cast<const cuuint64_t*>(dims),
                    reinterpret_cast<const cuuint64_t*>(strides_bytes),
                    reinterpret_cast<const cuuint32_t*>(box), estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MQA_ERR_CUDA, "tensor map for %s rejected (CUresult %d)", what, (int)r);
    return MQA_OK;
}

CUtensorMapSwizzle swizzle_for_bytes(int row_bytes) {
    return row_bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
         : row_bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                            : CU_TENSOR_MAP_SWIZZLE_32B;
}

int max_optin_smem(int dev, int* out) {
    cudaError_t e = cudaDeviceGetAttribute(out, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(smem)");
    return MQA_OK;
}

bool env_flag(const char* name) {
    const char* v = std::getenv(name);
    return v && v[0] && std::strcmp(v, "0") != 0;
}

int env_int(const char* name, int dflt) {
    const char* v = std::getenv(name);
    if (!v || !v[0]) return dflt;
    return std::atoi(v);
}

enum class Kind { FP8, FP4, NVFP4 };

// Host checks shared by both logits entry points.
int check_common(Kind kind, const void* q, const void* kv, const int32_t* bt, const int32_t* ctx,
                 const float* w, const int32_t* sched, const float* out,
                 const mqa_logits_params* p) {
    if (!p) return fail(MQA_ERR_INVALID_ARG, "params is NULL");
    if (p->batch < 0) return fail(MQA_ERR_INVALID_ARG, "batch must be >= 0 (got %d)", p->batch);
    if (p->next_n < 1 || p->next_n > 4)
        return fail(MQA_ERR_INVALID_ARG, "next_n must be in 1..4 (got %d)", p->next_n);
    const int H = p->num_heads;
    if (!(H == 4 || H == 8 || H == 16 || H == 32 || H == 64 || H == 128))
        return fail(MQA_ERR_UNSUPPORTED, "num_heads must be 4, 8, 16, 32, 64 or 128 (got %d)", H);
    if (H * p->next_n > 256)
        return fail(MQA_ERR_UNSUPPORTED, "num_heads * next_n must be <= 256 (got %d)", H * p->next_n);
    if (kind != Kind::FP8 && H * p->next_n > 128)
        return fail(MQA_ERR_UNSUPPORTED, "fp4: num_heads * next_n must be <= 128 (got %d)",
                    H * p->next_n);
    const int D = p->head_dim;
    if (kind == Kind::FP8 && !(D == 32 || D == 64 || D == 128))
        return fail(MQA_ERR_UNSUPPORTED, "fp8 head_dim must be 32, 64 or 128 (got %d)", D);
    if (kind != Kind::FP8 && !(D == 64 || D == 128))
        return fail(MQA_ERR_UNSUPPORTED, "fp4 head_dim must be 64 or 128 (got %d)", D);
    const int ps = p->page_size;
    const int ps_min = kind == Kind::FP8 ? 8 : 16;
    if (!pow2(ps) || ps < ps_min || ps > 256)
        return fail(MQA_ERR_INVALID_ARG, "page_size must be a power of two in [%d, 256] (got %d)",
                    ps_min, ps);
    if (p->num_pages < 1) return fail(MQA_ERR_INVALID_ARG, "num_pages must be >= 1");
    if (p->max_pages_per_row < 1) return fail(MQA_ERR_INVALID_ARG, "max_pages_per_row must be >= 1");
    if (p->out_len < 0 || (p->out_len % 4) != 0)
        return fail(MQA_ERR_INVALID_ARG, "out_len must be a non-negative multiple of 4 (got %d)",
                    p->out_len);
    if (p->num_ctas < 1 || p->num_ctas > kMaxCtas)
        return fail(MQA_ERR_INVALID_ARG, "num_ctas must be in 1..%d (got %d)", kMaxCtas, p->num_ctas);
    if (p->batch == 0 || p->out_len == 0) return MQA_OK;
    if (!q || !kv || !bt || !ctx || !w || !sched || !out)
        return fail(MQA_ERR_INVALID_ARG, "a tensor pointer is NULL");
    if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(w, 16) || !aligned(out, 16))
        return fail(MQA_ERR_INVALID_ARG, "q, kv_cache, weights and out must be 16-byte aligned");
    if (!aligned(bt, 4) || !aligned(ctx, 4) || !aligned(sched, 4))
        return fail(MQA_ERR_INVALID_ARG, "block_table, context_lens and schedule must be 4-byte aligned");
    if (p->status && !aligned(p->status, 4))
        return fail(MQA_ERR_INVALID_ARG, "status must be 4-byte aligned");
    return MQA_OK;
}

KernelArgs make_args(Kind kind, const void* q, const void* kv, const int32_t* bt, const int32_t* ctx,
                     const float* w, const int32_t* sched, float* out,
                     const mqa_logits_params* p) {
    KernelArgs a{};
    a.kv = static_cast<const uint8_t*>(kv);
    a.q = static_cast<const uint8_t*>(q);
    a.block_table = bt;
    a.context_lens = ctx;
    a.weights = w;
    a.schedule = sched;
    a.out = out;
    a.status = p->status;
    const int D = p->head_dim;
    a.page_bytes = kind == Kind::FP8 ? (int64_t)p->page_size * (D + 4)
                                     : (int64_t)p->page_size * (D / 2 + D / 16);
    a.batch = p->batch;
    a.next_n = p->next_n;
    a.heads = p->num_heads;
    a.head_dim = D;
    a.page_size = p->page_size;
    a.num_pages = p->num_pages;
    a.max_pages = p->max_pages_per_row;
    a.out_len = p->out_len;
    a.num_ctas = p->num_ctas;
    a.hn = p->num_heads * p->next_n;
    a.npad = (a.hn + 15) / 16 * 16;
    a.q_bytes = (int64_t)p->batch * a.hn *
                (kind == Kind::FP8 ? D : kind == Kind::FP4 ? 2 * D : D / 2 + D / 16);
    const int64_t cap = (int64_t)p->max_pages_per_row * p->page_size;
    a.ctx_cap = (int32_t)(cap < p->out_len ? cap : p->out_len);
    a.ps_shift = 0;
    while ((1 << a.ps_shift) < p->page_size) ++a.ps_shift;
    a.flags = p->flags | (env_flag("MQA_LOGITS_VALIDATE") ? MQA_FLAG_VALIDATE : 0u);
    a.timeout_ns = p->timeout_ns ? p->timeout_ns : 2000000000ull;
    return a;
}

int run_logits(Kind kind, const void* q, const void* kv, const int32_t* bt, const int32_t* ctx,
               const float* w, const int32_t* sched, float* out, const mqa_logits_params* p,
               void* stream, bool gather_only = false) {
    int rc = check_common(kind, q, kv, bt, ctx, w, sched, out, p);
    if (rc != MQA_OK) return rc;
    int dev = 0;
    uint32_t* lib_status = nullptr;
    rc = check_arch(&dev, &lib_status);
    if (rc != MQA_OK) return rc;
    if (p->batch == 0 || p->out_len == 0) return MQA_OK;

    KernelArgs a = make_args(kind, q, kv, bt, ctx, w, sched, out, p);
    a.lib_status = lib_status;
    const int D = p->head_dim;
    int smem_max = 0;
    rc = max_optin_smem(dev, &smem_max);
    if (rc != MQA_OK) return rc;
#ifdef MQA_DEBUG
    smem_max -= 256;  // the debug counters' static shared memory
#endif

    // ring depth: the kernel's default, or as many as fit if fewer (env
    // MQA_LOGITS_STAGES overrides); at least as many as the kernel has producer
    // warps (see producer_warp)
    const int min_stages = kind == Kind::FP8 ? 2 : kProducers;
    int stages = env_int("MQA_LOGITS_STAGES", kind == Kind::FP8 ? kDefaultStagesFp8 : kDefaultStages);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < min_stages) stages = min_stages;
    auto bytes_for = [&](int s) -> uint32_t {
        return kind == Kind::FP8   ? fp8_smem_layout(D, a.npad, s).total
             : kind == Kind::FP4   ? fp4_smem_layout(D, a.npad, s, p->page_size).total
                                   : nvfp4_smem_layout(D, a.npad, s).total;
    };
    while (stages > min_stages && bytes_for(stages) > (uint32_t)smem_max) --stages;
    if (kind == Kind::NVFP4) {
        // the stages' scale blocks share TMEM with the accumulators: keep >= 2 of those
        const int astride = acc_stride(a.npad);
        while (stages > kProducers && (512 - (stages * 2 + 2) * (D / 64) * 4) / astride < 2)
            --stages;
    }
    if (bytes_for(stages) > (uint32_t)smem_max)
        return fail(MQA_ERR_UNSUPPORTED, "shared memory does not fit (%u > %d bytes)",
                    bytes_for(stages), smem_max);
    a.num_stages = stages;
    const uint32_t smem = bytes_for(stages);

    CUtensorMap tm_k, tm_q;
    const int box_rows = p->page_size < kUnit ? p->page_size : kUnit;
    if (kind == Kind::FP8) {
        uint64_t kd[3] = {(uint64_t)D, (uint64_t)p->page_size, (uint64_t)p->num_pages};
        uint64_t ks[2] = {(uint64_t)D, (uint64_t)a.page_bytes};
        uint32_t kb[3] = {(uint32_t)D, (uint32_t)box_rows, 1};
        rc = encode_map(&tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, kv, kd, ks, kb,
                        swizzle_for_bytes(D), "kv_cache");
        if (rc != MQA_OK) return rc;
        uint64_t qd[2] = {(uint64_t)D, (uint64_t)p->batch * a.hn};
        uint64_t qs[1] = {(uint64_t)D};
        uint32_t qb[2] = {(uint32_t)D, (uint32_t)a.npad};
        rc = encode_map(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, qd, qs, qb,
                        swizzle_for_bytes(D), "q");
        if (rc != MQA_OK) return rc;
    } else if (kind == Kind::NVFP4) {
        // packed e2m1 rows (D/2 bytes), swizzled in the MMA's K-major layout
        uint64_t kd[3] = {(uint64_t)(D / 2), (uint64_t)p->page_size, (uint64_t)p->num_pages};
        uint64_t ks[2] = {(uint64_t)(D / 2), (uint64_t)a.page_bytes};
        uint32_t kb[3] = {(uint32_t)(D / 2), (uint32_t)box_rows, 1};
        rc = encode_map(&tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, kv, kd, ks, kb,
                        swizzle_for_bytes(D / 2), "kv_cache");
        if (rc != MQA_OK) return rc;
        // q codes: per (b, n) row [H][D/2], rows H * (D/2 + D/16) bytes apart;
        // one box holds every draft of a batch row
        uint64_t qd[3] = {(uint64_t)(D / 2), (uint64_t)p->num_heads,
                          (uint64_t)p->batch * p->next_n};
        uint64_t qs[2] = {(uint64_t)(D / 2), (uint64_t)p->num_heads * (D / 2 + D / 16)};
        uint32_t qb[3] = {(uint32_t)(D / 2), (uint32_t)p->num_heads, (uint32_t)p->next_n};
        rc = encode_map(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q, qd, qs, qb,
                        swizzle_for_bytes(D / 2), "q");
        if (rc != MQA_OK) return rc;
    } else {
        // a whole page (codes, then scales) as 9 ps / 16 rows of D bytes: one
        // tensor copy per page, swizzled so the dequant reads are conflict-free
        const uint32_t prow = (uint32_t)(9 * p->page_size / 16);
        uint64_t kd[3] = {(uint64_t)D, (uint64_t)prow, (uint64_t)p->num_pages};
        uint64_t ks[2] = {(uint64_t)D, (uint64_t)a.page_bytes};
        uint32_t kb[3] = {(uint32_t)D, prow, 1};
        rc = encode_map(&tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, kv, kd, ks, kb,
                        swizzle_for_bytes(D), "kv_cache");
        if (rc != MQA_OK) return rc;
        // bf16 q as 64-element (128-byte) column blocks: dims {64, rows, D/64}
        uint64_t qd[3] = {64, (uint64_t)p->batch * a.hn, (uint64_t)(D / 64)};
        uint64_t qs[2] = {(uint64_t)D * 2, 128};
        uint32_t qb[3] = {64, (uint32_t)a.npad, (uint32_t)(D / 64)};
        rc = encode_map(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, qd, qs, qb,
                        CU_TENSOR_MAP_SWIZZLE_128B, "q");
        if (rc != MQA_OK) return rc;
    }

    LaunchSpec ls;
    ls.grid = p->num_ctas;
    ls.smem = smem;
    ls.stream = stream;
    ls.pdl = (a.flags & MQA_FLAG_NO_PDL) == 0;
    if (gather_only) {
        const int e = launch_fp8_gather(D, ls, tm_k, tm_q, a);
        if (e != (int)cudaSuccess) return cuda_fail((cudaError_t)e, "gather launch");
        return MQA_OK;
    }
    const int e = kind == Kind::FP8 ? launch_fp8_logits(p->num_heads, D, ls, tm_k, tm_q, a)
                : kind == Kind::FP4 ? launch_fp4_logits(p->num_heads, D, ls, tm_k, tm_q, a)
                                    : launch_nvfp4_logits(p->num_heads, D, ls, tm_k, tm_q, a);
    if (e != (int)cudaSuccess) return cuda_fail((cudaError_t)e, "logits launch");
    return MQA_OK;
}

}  // namespace
}  // namespace mqa

extern "C" {

int mqa_logits_num_ctas(int device, int32_t* num_ctas) {
    if (!num_ctas) return mqa::fail(MQA_ERR_INVALID_ARG, "num_ctas is NULL");
    int n = 0;
    cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device);
    if (e != cudaSuccess) return mqa::cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    *num_ctas = n;
    return MQA_OK;
}

int mqa_logits_schedule(const int32_t* context_lens, int32_t batch, int32_t num_ctas,
                        int32_t* schedule, void* stream) {
    using namespace mqa;
    if (batch < 0 || batch > kMaxBatchSchedule)
        return fail(MQA_ERR_INVALID_ARG, "batch must be in 0..%d (got %d)", kMaxBatchSchedule, batch);
    if (num_ctas < 1 || num_ctas > kMaxCtas)
        return fail(MQA_ERR_INVALID_ARG, "num_ctas must be in 1..%d (got %d)", kMaxCtas, num_ctas);
    if (!schedule || (batch > 0 && !context_lens))
        return fail(MQA_ERR_INVALID_ARG, "context_lens / schedule is NULL");
    if (!aligned(schedule, 4) || !aligned(context_lens, 4))
        return fail(MQA_ERR_INVALID_ARG, "context_lens and schedule must be 4-byte aligned");
    int rc = check_arch(nullptr);
    if (rc != MQA_OK) return rc;
    const int e = launch_schedule(context_lens, batch, num_ctas, schedule, stream);
    if (e != (int)cudaSuccess) return cuda_fail((cudaError_t)e, "schedule launch");
    return MQA_OK;
}

int paged_mqa_logits_fp8(const void* q, const void* kv_cache, const int32_t* block_table,
                         const int32_t* context_lens, const float* weights,
                         const int32_t* schedule, float* out, const mqa_logits_params* params,
                         void* stream) {
    return mqa::run_logits(mqa::Kind::FP8, q, kv_cache, block_table, context_lens, weights,
                           schedule, out, params, stream);
}

int mqa_diag_fp8_gather(const void* q, const void* kv_cache, const int32_t* block_table,
                        const int32_t* context_lens, const float* weights,
                        const int32_t* schedule, float* out, const mqa_logits_params* params,
                        void* stream) {
    return mqa::run_logits(mqa::Kind::FP8, q, kv_cache, block_table, context_lens, weights,
                           schedule, out, params, stream, true);
}

int paged_mqa_logits_fp4(const void* q, const void* kv_cache, const int32_t* block_table,
                         const int32_t* context_lens, const float* weights,
                         const int32_t* schedule, float* out, const mqa_logits_params* params,
                         void* stream) {
    return mqa::run_logits(mqa::Kind::FP4, q, kv_cache, block_table, context_lens, weights,
                           schedule, out, params, stream);
}

int paged_mqa_logits_nvfp4(const void* q, const void* kv_cache, const int32_t* block_table,
                           const int32_t* context_lens, const float* weights,
                           const int32_t* schedule, float* out, const mqa_logits_params* params,
                           void* stream) {
    return mqa::run_logits(mqa::Kind::NVFP4, q, kv_cache, block_table, context_lens, weights,
                           schedule, out, params, stream);
}

int mqa_logits_topk(const float* logits, const int32_t* context_lens, int32_t batch,
                    int32_t next_n, int32_t out_len, int32_t k, int32_t flags, int32_t* indices,
                    float* values, void* stream) {
    using namespace mqa;
    if (batch < 0 || next_n < 1 || next_n > 4 || out_len < 0)
        return fail(MQA_ERR_INVALID_ARG, "need batch >= 0, 1 <= next_n <= 4, out_len >= 0");
    if (k < 1 || k > MQA_TOPK_MAX)
        return fail(MQA_ERR_INVALID_ARG, "k must be in 1..%d (got %d)", MQA_TOPK_MAX, k);
    if (flags & ~MQA_TOPK_BY_TOKEN) return fail(MQA_ERR_INVALID_ARG, "unknown top-k flag bits");
    if ((int64_t)batch * next_n > (int64_t)2147483647)
        return fail(MQA_ERR_INVALID_ARG, "too many rows");
    if (batch == 0) return MQA_OK;
    if (!logits || !context_lens || !indices)
        return fail(MQA_ERR_INVALID_ARG, "logits / context_lens / indices is NULL");
    if (!aligned(logits, 4) || !aligned(context_lens, 4) || !aligned(indices, 4) ||
        !aligned(values, 4))
        return fail(MQA_ERR_INVALID_ARG,
                    "logits, context_lens, indices and values must be 4-byte aligned");
    int rc = check_arch(nullptr);
    if (rc != MQA_OK) return rc;
    // MQA_TOPK_CLUSTER: 1 keeps one CTA per row, 2 or 4 splits every row over
    // a cluster of that many CTAs; unset or 0 lets the launcher choose
    const int e = launch_topk(logits, context_lens, batch, next_n, out_len, k, flags, indices,
                              values, stream, env_int("MQA_TOPK_CLUSTER", 0));
    if (e != (int)cudaSuccess) return cuda_fail((cudaError_t)e, "top-k launch");
    return MQA_OK;
}

int mqa_logits_topk_merge(const float* cand_values, const int32_t* cand_tokens, int32_t shards,
                          int32_t rows, int32_t k_in, const int32_t* token_offsets,
                          const int32_t* token_counts, int32_t k, int32_t flags,
                          int32_t* indices, float* values, void* stream) {
    using namespace mqa;
    if (shards < 1 || shards > MQA_TOPK_MERGE_MAX_SHARDS || rows < 0 || k_in < 1)
        return fail(MQA_ERR_INVALID_ARG, "need 1 <= shards <= %d, rows >= 0, k_in >= 1",
                    MQA_TOPK_MERGE_MAX_SHARDS);
    if ((int64_t)shards * k_in > MQA_TOPK_MERGE_MAX)
        return fail(MQA_ERR_INVALID_ARG, "shards * k_in must be <= %d", MQA_TOPK_MERGE_MAX);
    if (k < 1 || k > MQA_TOPK_MAX)
        return fail(MQA_ERR_INVALID_ARG, "k must be in 1..%d (got %d)", MQA_TOPK_MAX, k);
    if (flags & ~MQA_TOPK_BY_TOKEN) return fail(MQA_ERR_INVALID_ARG, "unknown top-k flag bits");
    if (!token_offsets || !token_counts)
        return fail(MQA_ERR_INVALID_ARG, "token_offsets / token_counts is NULL");
    for (int s = 0; s < shards; ++s) {
        if (token_offsets[s] < 0 || token_counts[s] < 0)
            return fail(MQA_ERR_INVALID_ARG, "token_offsets and token_counts must be >= 0");
        if ((int64_t)token_offsets[s] + token_counts[s] > 2147483647LL)
            return fail(MQA_ERR_INVALID_ARG, "shard %d's token range passes 2^31", s);
        if (s + 1 < shards && (int64_t)token_offsets[s] + token_counts[s] > token_offsets[s + 1])
            return fail(MQA_ERR_INVALID_ARG,
                        "token ranges overlap or descend: shard %d covers [%d, %lld), shard %d "
                        "starts at %d",
                        s, token_offsets[s], (long long)token_offsets[s] + token_counts[s], s + 1,
                        token_offsets[s + 1]);
    }
    if (rows == 0) return MQA_OK;
    if (!cand_values || !cand_tokens || !indices)
        return fail(MQA_ERR_INVALID_ARG, "cand_values / cand_tokens / indices is NULL");
    if (!aligned(cand_values, 4) || !aligned(cand_tokens, 4) || !aligned(indices, 4) ||
        !aligned(values, 4))
        return fail(MQA_ERR_INVALID_ARG, "device arrays must be 4-byte aligned");
    int rc = check_arch(nullptr);
    if (rc != MQA_OK) return rc;
    const int e = launch_topk_merge(cand_values, cand_tokens, shards, rows, k_in, token_offsets,
                                    k, flags, indices, values, stream);
    if (e != (int)cudaSuccess) return cuda_fail((cudaError_t)e, "top-k merge launch");
    return MQA_OK;
}

int mqa_logits_get_status(uint32_t* bits, void* stream) {
    using namespace mqa;
    if (!bits) return fail(MQA_ERR_INVALID_ARG, "bits is NULL");
    uint32_t* word = nullptr;
    int rc = check_arch(nullptr, &word);
    if (rc != MQA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, word, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
    *bits = v;
    return MQA_OK;
}

int mqa_logits_check_status(void* stream) {
    using namespace mqa;
    uint32_t v = 0;
    const int rc = mqa_logits_get_status(&v, stream);
    if (rc != MQA_OK) return rc;
    if (v == 0) return MQA_OK;
    static const char* const names[] = {"TIMEOUT", "BAD_PAGE", "BAD_CONTEXT", "STALE_SCHEDULE",
                                        "Q_RANGE", "DEBUG_INVARIANT"};
    std::string msg;
    for (int i = 0; i < 6; ++i)
        if (v & (1u << i)) msg += std::string(" ") + names[i];
    if (v >> 6) msg += " (unknown bits)";
    return fail(MQA_ERR_DEVICE_CHECK, "device status 0x%x:%s", v, msg.c_str());
}

int mqa_logits_clear_status(void* stream) {
    using namespace mqa;
    uint32_t* word = nullptr;
    int rc = check_arch(nullptr, &word);
    if (rc != MQA_OK) return rc;
    cudaError_t e = cudaMemsetAsync(word, 0, sizeof(uint32_t), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
    return MQA_OK;
}

const char* mqa_logits_last_error(void) { return mqa::g_err.c_str(); }

#ifdef MQA_DEBUG
const char* mqa_logits_version(void) { return "0.1.0-debug"; }
#else
const char* mqa_logits_version(void) { return "0.1.0"; }
#endif

}  // extern "C"
