// libpa.so: the C ABI declared in include/pa.h.
//
// Host side only: argument checks, launch geometry and template dispatch.
// Every step of the computation runs in the kernels this file includes.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <atomic>

#include "pa_common.cuh"
#include "decode.cuh"
#include "prefill_sm100.cuh"
#include "block_copy.cuh"
#include "reshape_and_cache.cuh"

namespace {

thread_local int g_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    int n = __atomic_load_n(&g_sm_count[dev], __ATOMIC_ACQUIRE);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        __atomic_store_n(&g_sm_count[dev], n, __ATOMIC_RELEASE);
    }
    return n;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int cuda_fail(cudaError_t e) {
    g_last_cuda_error = static_cast<int>(e);
    return PA_ERR_CUDA;
}

int check_launch() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PA_OK : cuda_fail(e);
}

int check_shape(const pa_shape *s) {
    if (!s) return PA_ERR_INVALID_ARGUMENT;
    if (s->num_heads <= 0 || s->num_kv_heads <= 0 || s->num_blocks <= 0) return PA_ERR_INVALID_ARGUMENT;
    if (s->num_heads % s->num_kv_heads != 0) return PA_ERR_INVALID_ARGUMENT;
    if (s->block_size != PA_BLOCK_SIZE) return PA_ERR_UNSUPPORTED;
    if (s->head_dim != 64 && s->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (s->dtype != PA_DTYPE_F32 && s->dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
    const int g = s->num_heads / s->num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return PA_ERR_UNSUPPORTED;
    if (s->num_blocks >= (int64_t{1} << 31) / PA_BLOCK_SIZE) return PA_ERR_UNSUPPORTED;  // rows fit in int32 math
    if (s->kv_fp8 != 0 && s->kv_fp8 != 1) return PA_ERR_INVALID_ARGUMENT;
    if (s->kv_fp8) {
        if (s->dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
        if (!(s->k_scale > 0.f) || !(s->v_scale > 0.f) || !std::isfinite(s->k_scale) || !std::isfinite(s->v_scale))
            return PA_ERR_INVALID_ARGUMENT;
    }
    return PA_OK;
}

int elem_bytes(const pa_shape *s) { return s->dtype == PA_DTYPE_BF16 ? 2 : 4; }
int cache_elem_bytes(const pa_shape *s) { return s->kv_fp8 ? 1 : elem_bytes(s); }

// CTAs of the decode kernel one SM holds, for this shape: the occupancy the
// runtime reports on the current device (with the kernel's shared memory and
// the largest shared-memory carveout, set here once per device), or, without
// a device, the compile-time estimate. The grid is sized from it, so every
// slice's CTA is resident from the start.
template <typename Tq, typename Tc, int D, int G>
int resident_of() {
    using C = pa::DecodeCfg<Tc, D, G>;
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return C::RESIDENT;
    }
    int n = cached[dev].load(std::memory_order_acquire);
    if (n > 0) return n;
    auto kernel = pa::decode_kernel<Tq, Tc, D, G>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, C::THREADS, C::SMEM) != cudaSuccess ||
        n < 1) {
        cudaGetLastError();
        return C::RESIDENT;
    }
    cached[dev].store(n, std::memory_order_release);
    return n;
}

// CTAs per SM and warps per CTA of the decode kernel for one shape.
struct DecodeFit {
    int resident;
    int warps;
};

template <typename Tq, typename Tc, int D, int G>
DecodeFit fit_of() {
    return DecodeFit{resident_of<Tq, Tc, D, G>(), pa::DecodeCfg<Tc, D, G>::WARPS};
}

template <typename Tq, typename Tc, int D>
DecodeFit fit_g(int g) {
    switch (g) {
        case 1: return fit_of<Tq, Tc, D, 1>();
        case 2: return fit_of<Tq, Tc, D, 2>();
        case 4: return fit_of<Tq, Tc, D, 4>();
        default: return fit_of<Tq, Tc, D, 8>();
    }
}

DecodeFit decode_fit(const pa_shape *s) {
    const int g = s->num_heads / s->num_kv_heads;
    if (s->kv_fp8)
        return s->head_dim == 128 ? fit_g<__nv_bfloat16, pa::fp8e4m3, 128>(g)
                                  : fit_g<__nv_bfloat16, pa::fp8e4m3, 64>(g);
    if (s->dtype == PA_DTYPE_BF16)
        return s->head_dim == 128 ? fit_g<__nv_bfloat16, __nv_bfloat16, 128>(g)
                                  : fit_g<__nv_bfloat16, __nv_bfloat16, 64>(g);
    return s->head_dim == 128 ? fit_g<float, float, 128>(g) : fit_g<float, float, 64>(g);
}

struct DecodeGeometry {
    int ctas;          // grid of the persistent decode kernel (one slice per warp)
    int64_t slots;     // partial (m, l, O) slots: slice index + unit index
    int64_t ws_bytes;  // workspace bytes
};

int64_t round16(int64_t n) { return (n + 15) / 16 * 16; }

// The decode kernel cuts the flat (sequence, KV head, block) list into
// warps * ctas equal slices, one per warp. Automatic: the CTAs all SMs hold at once
// (each warp streams one slice; balance comes from equal slices, not from many
// waves), but no more than one warp per 4 blocks of the largest possible list.
// With partition_tokens given: slices of about that many tokens of a context
// of max_context_len. Workspace: fp32 partial outputs [slots][G][D], partial
// maxima and sums [slots][G] each, then int32 (first slice, slices) records
// [B][Hk]; each part 16-byte aligned.
int decode_geometry(int32_t num_seqs, int32_t max_context_len, int32_t requested, const pa_shape *s,
                    DecodeGeometry *g) {
    if (num_seqs < 0 || max_context_len < 0) return PA_ERR_INVALID_ARGUMENT;
    if (requested < 0 || (requested > 0 && (requested % 64 != 0))) return PA_ERR_INVALID_ARGUMENT;
    const int64_t units = static_cast<int64_t>(num_seqs) * s->num_kv_heads;
    const int64_t n_max = units * ((max_context_len + PA_BLOCK_SIZE - 1) / PA_BLOCK_SIZE);
    const DecodeFit fit = decode_fit(s);
    int64_t slices;
    if (requested > 0) {
        slices = (n_max * PA_BLOCK_SIZE + requested - 1) / requested;
    } else {
        const int64_t sms = sm_count() > 0 ? sm_count() : 148;
        slices = std::min<int64_t>(sms * fit.resident * fit.warps, (n_max + 3) / 4);
    }
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>((slices + fit.warps - 1) / fit.warps, 65535));
    g->ctas = static_cast<int>(ctas);
    if (units == 0) {
        g->slots = 0;
        g->ws_bytes = 0;
    } else {
        const int gq = s->num_heads / s->num_kv_heads;
        g->slots = ctas * fit.warps + units - 1;
        g->ws_bytes = g->slots * gq * s->head_dim * 4 + round16(g->slots * gq * 4) * 2 + round16(units * 8);
    }
    return PA_OK;
}

// The two launches of a decode: the partition pass and the merge.
enum DecodeParts { kPartials = 1, kMerge = 2, kBoth = 3 };

template <typename Tq, typename Tc, int D, int G>
int launch_decode(const pa::DecodeParams &prm, const DecodeGeometry &geo, int parts, cudaStream_t st) {
    using C = pa::DecodeCfg<Tc, D, G>;
    // Both kernels are programmatic dependent launches: each starts launching
    // while the kernel before it drains, and waits for it (griddepcontrol.wait)
    // before reading what it wrote.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    pa::DecodeParams p = prm;
    p.warps_total = geo.ctas * C::WARPS;
    if (parts & kPartials) {
        resident_of<Tq, Tc, D, G>();  // sets the kernel's shared-memory attributes on this device
        CUtensorMap tm_k{}, tm_v{};
        const uint64_t rows = static_cast<uint64_t>(prm.num_blocks) * pa::kBlockSize;
        if (!pa::encode_3d(&tm_k, prm.k_cache, D, prm.num_kv_heads, rows, sizeof(Tc), D, 1, pa::kBlockSize,
                           CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !pa::encode_3d(&tm_v, prm.v_cache, D, prm.num_kv_heads, rows, sizeof(Tc), D, 1, pa::kBlockSize,
                           CU_TENSOR_MAP_SWIZZLE_NONE))
            return PA_ERR_UNSUPPORTED;
        cfg.gridDim = dim3(geo.ctas);
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = C::SMEM;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, pa::decode_kernel<Tq, Tc, D, G>, p, tm_k, tm_v);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    if (parts & kMerge) {
        // Four warps per unit when units average 16 slices or more (long
        // contexts): their slices are merged four ways at once. One otherwise:
        // fewer, smaller CTAs launch and finish sooner.
        const int64_t units = static_cast<int64_t>(prm.num_seqs) * prm.num_kv_heads;
        const bool wide = static_cast<int64_t>(geo.ctas) * C::WARPS >= 16 * units;
        cfg.gridDim = dim3(static_cast<unsigned>(units), (G * D + 127) / 128);
        cfg.blockDim = dim3(wide ? 128 : 32);
        cfg.dynamicSmemBytes = 0;
        const cudaError_t e = wide ? cudaLaunchKernelEx(&cfg, pa::decode_merge_kernel<Tq, G, D, 4>, p)
                                   : cudaLaunchKernelEx(&cfg, pa::decode_merge_kernel<Tq, G, D, 1>, p);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return PA_OK;
}

template <typename Tq, typename Tc, int D>
int dispatch_g(int g, const pa::DecodeParams &prm, const DecodeGeometry &geo, int parts, cudaStream_t st) {
    switch (g) {
        case 1: return launch_decode<Tq, Tc, D, 1>(prm, geo, parts, st);
        case 2: return launch_decode<Tq, Tc, D, 2>(prm, geo, parts, st);
        case 4: return launch_decode<Tq, Tc, D, 4>(prm, geo, parts, st);
        case 8: return launch_decode<Tq, Tc, D, 8>(prm, geo, parts, st);
        default: return PA_ERR_UNSUPPORTED;
    }
}

}  // namespace

extern "C" {

int pa_abi_version(void) { return PA_ABI_VERSION; }

const char *pa_strerror(int code) {
    switch (code) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARGUMENT: return "invalid argument";
        case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case PA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case PA_ERR_WORKSPACE: return "workspace missing or too small";
        case PA_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
        case PA_ERR_DEVICE: return "no usable sm_100 device";
        case PA_ERR_SCRATCH_LIMIT: return "request needs more scratch than pa_decode_noalloc's built-in array";
        default: return "unknown error";
    }
}

int pa_last_cuda_error(void) { return g_last_cuda_error; }

int pa_reshape_and_cache(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                         int64_t num_tokens, const pa_shape *shape, void *stream) {
    int rc = check_shape(shape);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0) return PA_ERR_INVALID_ARGUMENT;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARGUMENT;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned(slot_mapping, 8))
        return PA_ERR_ALIGNMENT;
    const int row_bytes = shape->num_kv_heads * shape->head_dim * elem_bytes(shape);  // one input row
    if (row_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
    const int row_vecs = row_bytes / 16;
    const int64_t total = num_tokens * row_vecs;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int sms = sm_count() > 0 ? sm_count() : 148;
    if (blocks > int64_t{sms} * 16) blocks = int64_t{sms} * 16;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (shape->kv_fp8) {
        pa::reshape_and_cache_fp8_kernel<<<static_cast<unsigned>(blocks), threads, 0, st>>>(
            static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint2 *>(k_cache),
            static_cast<uint2 *>(v_cache), slot_mapping, num_tokens, shape->num_blocks * PA_BLOCK_SIZE, row_vecs,
            1.0f / shape->k_scale, 1.0f / shape->v_scale);
        return check_launch();
    }
    pa::reshape_and_cache_kernel<<<static_cast<unsigned>(blocks), threads, 0, st>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint4 *>(k_cache),
        static_cast<uint4 *>(v_cache), slot_mapping, num_tokens, shape->num_blocks * PA_BLOCK_SIZE, row_vecs);
    return check_launch();
}

int64_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t max_context_len, int32_t partition_tokens,
                                  const pa_shape *shape) {
    int rc = check_shape(shape);
    if (rc != PA_OK) return rc;
    DecodeGeometry g;
    rc = decode_geometry(num_seqs, max_context_len, partition_tokens, shape, &g);
    if (rc != PA_OK) return rc;
    return g.ws_bytes;
}

}  // extern "C"

namespace {

// pa_decode (or one of its two launches) after its argument checks.
int decode_call(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
                float scale, int32_t partition_tokens, void *workspace, int64_t workspace_bytes,
                const pa_shape *shape, void *stream, int parts = kBoth) {
    int rc = check_shape(shape);
    if (rc != PA_OK) return rc;
    if (num_seqs < 0 || max_context_len < 0 || max_blocks_per_seq < 0) return PA_ERR_INVALID_ARGUMENT;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_INVALID_ARGUMENT;
    if (max_blocks_per_seq < 1 || !std::isfinite(scale)) return PA_ERR_INVALID_ARGUMENT;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned(block_tables, 4) ||
        !aligned(context_lens, 4))
        return PA_ERR_ALIGNMENT;
    if (static_cast<int64_t>(num_seqs) * shape->num_kv_heads > 0x7fffffff) return PA_ERR_UNSUPPORTED;
    DecodeGeometry g;
    rc = decode_geometry(num_seqs, max_context_len, partition_tokens, shape, &g);
    if (rc != PA_OK) return rc;
    pa::DecodeParams prm{};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!workspace || workspace_bytes < g.ws_bytes) return PA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return PA_ERR_ALIGNMENT;
    {
        const int gq = shape->num_heads / shape->num_kv_heads;
        char *w = static_cast<char *>(workspace);
        const int64_t o_bytes = g.slots * gq * shape->head_dim * 4, ml_bytes = round16(g.slots * gq * 4);
        prm.ws_o = reinterpret_cast<float *>(w);
        prm.ws_m = reinterpret_cast<float *>(w + o_bytes);
        prm.ws_l = reinterpret_cast<float *>(w + o_bytes + ml_bytes);
        prm.ws_unit = reinterpret_cast<int *>(w + o_bytes + 2 * ml_bytes);
    }
    prm.out = out;
    prm.q = q;
    prm.k_cache = k_cache;
    prm.v_cache = v_cache;
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.num_blocks = shape->num_blocks;
    prm.num_seqs = num_seqs;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_heads = shape->num_heads;
    prm.num_kv_heads = shape->num_kv_heads;
    prm.max_context_len = max_context_len;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.v_scale = 1.f;
    if (shape->kv_fp8) {
        prm.scale_log2 *= shape->k_scale;
        prm.v_scale = shape->v_scale;
    }
    const int G = shape->num_heads / shape->num_kv_heads;
    if (shape->kv_fp8) {
        return shape->head_dim == 128 ? dispatch_g<__nv_bfloat16, pa::fp8e4m3, 128>(G, prm, g, parts, st)
                                      : dispatch_g<__nv_bfloat16, pa::fp8e4m3, 64>(G, prm, g, parts, st);
    }
    if (shape->dtype == PA_DTYPE_BF16) {
        return shape->head_dim == 128 ? dispatch_g<__nv_bfloat16, __nv_bfloat16, 128>(G, prm, g, parts, st)
                                      : dispatch_g<__nv_bfloat16, __nv_bfloat16, 64>(G, prm, g, parts, st);
    }
    return shape->head_dim == 128 ? dispatch_g<float, float, 128>(G, prm, g, parts, st)
                                  : dispatch_g<float, float, 64>(G, prm, g, parts, st);
}

}  // namespace

extern "C" {

int pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
              int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
              float scale, int32_t partition_tokens, void *workspace, int64_t workspace_bytes, const pa_shape *shape,
              void *stream) {
    return decode_call(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                       max_context_len, scale, partition_tokens, workspace, workspace_bytes, shape, stream);
}

int pa_decode_partials(void *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
                       int32_t num_seqs, int32_t max_context_len, float scale, int32_t partition_tokens,
                       void *workspace, int64_t workspace_bytes, const pa_shape *shape, void *stream) {
    return decode_call(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                       max_context_len, scale, partition_tokens, workspace, workspace_bytes, shape, stream, kPartials);
}

int pa_decode_merge(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                    int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
                    int32_t max_context_len, float scale, int32_t partition_tokens, void *workspace,
                    int64_t workspace_bytes, const pa_shape *shape, void *stream) {
    return decode_call(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                       max_context_len, scale, partition_tokens, workspace, workspace_bytes, shape, stream, kMerge);
}

int pa_prefill_chunk(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                     int32_t max_blocks_per_seq, const int32_t *cu_q_lens, const int32_t *context_lens,
                     int32_t num_seqs, int32_t max_q_len, int32_t num_q_tokens, float scale, const pa_shape *shape,
                     void *stream) {
    int rc = check_shape(shape);
    if (rc != PA_OK) return rc;
    if (shape->dtype != PA_DTYPE_BF16 || shape->head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (num_seqs < 0 || max_q_len < 0 || num_q_tokens < 0 || max_blocks_per_seq < 0) return PA_ERR_INVALID_ARGUMENT;
    if (num_seqs == 0 || num_q_tokens == 0 || max_q_len == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !cu_q_lens || !context_lens)
        return PA_ERR_INVALID_ARGUMENT;
    if (max_blocks_per_seq < 1 || !std::isfinite(scale) || !(scale > 0.f)) return PA_ERR_INVALID_ARGUMENT;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned(block_tables, 4) ||
        !aligned(cu_q_lens, 4) || !aligned(context_lens, 4))
        return PA_ERR_ALIGNMENT;
    rc = pa::launch_prefill(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, cu_q_lens, context_lens,
                            num_seqs, max_q_len, num_q_tokens, scale, shape, static_cast<cudaStream_t>(stream));
    return rc == PA_ERR_CUDA ? cuda_fail(cudaGetLastError()) : rc;  // keep the CUDA error for pa_last_cuda_error
}

}  // extern "C"

// ---- pa_decode_noalloc: decode with a scratch array compiled into the library ----

namespace {

// Scratch for the split-context partials of pa_decode_noalloc. Each device
// that loads this module holds it until the process exits. Host code must not
// use the symbol itself as a device address: the address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

// Per device: the context the address was looked up in, and the address. A
// context change (cudaDeviceReset, then a new primary context) reloads the
// module, possibly elsewhere, so the address is looked up again.
struct NoallocSlot {
    std::atomic<void *> ctx{nullptr};
    std::atomic<void *> ptr{nullptr};
};
NoallocSlot g_noalloc[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

void *current_context() {
    static CtxGetCurrentFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<CtxGetCurrentFn>(nullptr);
        return reinterpret_cast<CtxGetCurrentFn>(p);
    }();
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return static_cast<void *>(c);
}

int noalloc_scratch(void **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_DEVICE;
    NoallocSlot &slot = g_noalloc[dev];
    void *ctx = current_context();
    // ctx is stored after ptr and loaded before it: a matching ctx comes with its ptr
    const void *seen_ctx = slot.ctx.load(std::memory_order_acquire);
    void *p = slot.ptr.load(std::memory_order_acquire);
    if (!p || !ctx || seen_ctx != ctx) {
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // with `dev` current
        if (e != cudaSuccess) return cuda_fail(e);
        if (!ctx) ctx = current_context();  // the lookup made the primary context current
        slot.ptr.store(p, std::memory_order_release);
        slot.ctx.store(ctx, std::memory_order_release);
    }
    *ptr = p;
    return PA_OK;
}

}  // namespace

extern "C" {

int pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
                      int32_t num_seqs, int32_t max_context_len, float scale, int32_t partition_tokens,
                      const pa_shape *shape, void *stream) {
    const int64_t need = pa_decode_workspace_bytes(num_seqs, max_context_len, partition_tokens, shape);
    if (need < 0) return static_cast<int>(need);
    if (need > static_cast<int64_t>(PA_NOALLOC_SCRATCH_BYTES)) return PA_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if (need > 0) {
        const int rc = noalloc_scratch(&scratch);
        if (rc != PA_OK) return rc;
    }
    if (need == 0) return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                    num_seqs, max_context_len, scale, partition_tokens, nullptr, 0, shape, stream);
    // Every partial and record a call reads, it has written first: no earlier
    // call's contents matter.
    return decode_call(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                       max_context_len, scale, partition_tokens, scratch, need, shape, stream);
}

static int launch_copy(void *dst, const void *src, const int64_t *pairs, int64_t num_pairs, int64_t src_blocks,
                       int64_t dst_blocks, int64_t block_bytes, cudaStream_t st) {
    if (block_bytes <= 0 || block_bytes % 16 != 0 || block_bytes / 16 > (int64_t{1} << 30)) return PA_ERR_UNSUPPORTED;
    const int sms = sm_count() > 0 ? sm_count() : 148;
    int64_t grid = num_pairs < int64_t{sms} * 8 ? num_pairs : int64_t{sms} * 8;
    pa::copy_blocks_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
        static_cast<uint4 *>(dst), static_cast<const uint4 *>(src), pairs, num_pairs, src_blocks, dst_blocks,
        static_cast<int>(block_bytes / 16));
    return check_launch();
}

int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_pairs, int64_t num_pairs,
                   const pa_shape *shape, void *stream) {
    int rc = check_shape(shape);
    if (rc != PA_OK) return rc;
    if (num_pairs < 0) return PA_ERR_INVALID_ARGUMENT;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !block_pairs) return PA_ERR_INVALID_ARGUMENT;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned(block_pairs, 8)) return PA_ERR_ALIGNMENT;
    const int64_t bb = int64_t{PA_BLOCK_SIZE} * shape->num_kv_heads * shape->head_dim * cache_elem_bytes(shape);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = launch_copy(k_cache, k_cache, block_pairs, num_pairs, shape->num_blocks, shape->num_blocks, bb, st);
    if (rc != PA_OK) return rc;
    return launch_copy(v_cache, v_cache, block_pairs, num_pairs, shape->num_blocks, shape->num_blocks, bb, st);
}

// Device address of memory a kernel may touch: device memory, or pinned host
// memory through its mapping. Pageable host memory is refused.
static int device_view(const void *p, void **dev) {
    cudaPointerAttributes a;
    const cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return PA_ERR_INVALID_ARGUMENT;
    }
    if (a.type == cudaMemoryTypeUnregistered || a.devicePointer == nullptr) return PA_ERR_INVALID_ARGUMENT;
    *dev = a.devicePointer;
    return PA_OK;
}

int pa_swap_blocks(void *dst, const void *src, const int64_t *block_pairs, int64_t num_pairs, int64_t src_blocks,
                   int64_t dst_blocks, int64_t block_bytes, void *stream) {
    if (num_pairs < 0 || src_blocks <= 0 || dst_blocks <= 0) return PA_ERR_INVALID_ARGUMENT;
    if (num_pairs == 0) return PA_OK;
    if (!dst || !src || !block_pairs) return PA_ERR_INVALID_ARGUMENT;
    void *d = nullptr, *s = nullptr, *pr = nullptr;
    int rc = device_view(dst, &d);
    if (rc == PA_OK) rc = device_view(src, &s);
    if (rc == PA_OK) rc = device_view(block_pairs, &pr);
    if (rc != PA_OK) return rc;
    if (!aligned16(d) || !aligned16(s) || !aligned(pr, 8)) return PA_ERR_ALIGNMENT;
    return launch_copy(d, s, static_cast<const int64_t *>(pr), num_pairs, src_blocks, dst_blocks, block_bytes,
                       static_cast<cudaStream_t>(stream));
}

int pa_get_status(uint32_t *status, void *stream) {
    if (!status) return PA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned int v = 0;
    e = cudaMemcpyFromSymbol(&v, pa::g_status, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e);
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(pa::g_status, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e);
    *status = v;
    return PA_OK;
}

}  // extern "C"
