// Device helpers shared by the paged-attention kernels (sm_100a only).
//
// Hand-written PTX for the asynchronous-copy machinery: mbarriers, 1-D bulk
// copies from global to shared memory, and the packed two-wide fp32 FMA.
// Every wait here has a time limit. A wait that runs out sets a flag in the
// library's device status word and returns false, so a kernel can never spin
// forever.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/pa.h"

namespace pa {

// Device status word of this library (PA_STATUS_* flags); read by pa_get_status.
// The library is a single translation unit, so this is its one definition.
__device__ unsigned int g_status = 0;

constexpr int kBlockSize = PA_BLOCK_SIZE;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s for any single wait

__device__ __forceinline__ void flag_status(unsigned int f) { atomicOr(&g_status, f); }

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier ---------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of an mbarrier to complete, for at most kWaitLimitNs.
// Returns false (and flags PA_STATUS_WAIT_TIMEOUT) if it did not.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) {
            flag_status(PA_STATUS_WAIT_TIMEOUT);
            return false;
        }
    }
}

// ---- bulk async copy (TMA, non-tensor) ---------------------------------------

// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) from global
// memory into this CTA's shared memory; completion is counted on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Same, with an L2 eviction-priority policy (createpolicy result).
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// The normal L2 eviction priority as an explicit policy (createpolicy result).
__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---- arithmetic ---------------------------------------------------------------

// Packed pairs of fp32 in one 64-bit register, for the two-wide fp32 ops
// (fma/mul .f32x2, sm_100). Each lane of a pair is an IEEE op with
// round-to-nearest, so results equal two scalar ops.
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void unpack2(f32x2 v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// d += a * b
__device__ __forceinline__ void fma2(f32x2 &d, f32x2 a, f32x2 b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

// d *= a
__device__ __forceinline__ void mul2(f32x2 &d, f32x2 a) { asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(d) : "l"(a)); }

// d += a
__device__ __forceinline__ void add2(f32x2 &d, f32x2 a) { asm("add.rn.f32x2 %0, %0, %1;" : "+l"(d) : "l"(a)); }

// 2^x with the hardware approximation (ex2.approx.ftz.f32): 2^-inf = 0,
// subnormal results flush to zero. Used where the result is rounded to bf16.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One FP8 E4M3 code (cache storage type).
struct fp8e4m3 {
    uint8_t bits;
};

// Two E4M3 codes (low byte = element 0) to two fp32 values, exactly.
__device__ __forceinline__ f32x2 e4m3x2_to_f32x2(uint32_t two_codes) {
    uint32_t h2;
    asm("{\n\t.reg .b16 c;\n\t"
        "cvt.u16.u32 c, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, c;\n\t}"
        : "=r"(h2)
        : "r"(two_codes));
    float lo, hi;
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.f32.f16 %0, l;\n\t"
        "cvt.f32.f16 %1, h;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(h2));
    return pack2(lo, hi);
}

// Two fp32 values to two E4M3 codes in the low 16 bits (low byte = x0):
// nearest, ties to even, saturating at +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float x0, float x1) {
    uint32_t r;
    asm("{\n\t.reg .b16 c;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 c, %2, %1;\n\t"
        "cvt.u32.u16 %0, c;\n\t}"
        : "=r"(r)
        : "f"(x0), "f"(x1));
    return r;
}

// Widen 16 bytes of storage to fp32: 16 fp8, 8 bf16 or 4 fp32 values.
template <typename T>
struct Widen;

template <>
struct Widen<fp8e4m3> {
    static constexpr int N = 16;
    __device__ __forceinline__ static void apply2(const uint4 &r, f32x2 *f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = e4m3x2_to_f32x2(w[i] & 0xffffu);
            f[2 * i + 1] = e4m3x2_to_f32x2(w[i] >> 16);
        }
    }
};

template <>
struct Widen<__nv_bfloat16> {
    static constexpr int N = 8;
    // pairs (element 2i, element 2i+1) for i < 4
    __device__ __forceinline__ static void apply2(const uint4 &r, f32x2 *f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = pack2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
    }
    __device__ __forceinline__ static void apply(const uint4 &r, float *f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

template <>
struct Widen<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void apply2(const uint4 &r, f32x2 *f) {
        f[0] = (static_cast<f32x2>(r.y) << 32) | r.x;
        f[1] = (static_cast<f32x2>(r.w) << 32) | r.z;
    }
    __device__ __forceinline__ static void apply(const uint4 &r, float *f) {
        f[0] = __uint_as_float(r.x);
        f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z);
        f[3] = __uint_as_float(r.w);
    }
};

__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// Four consecutive outputs (p 16-byte aligned for fp32, 8-byte for bf16).
__device__ __forceinline__ void store_out4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void store_out4(__nv_bfloat16 *p, float4 v) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 r;
    r.x = *reinterpret_cast<const uint32_t *>(&a);
    r.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = r;
}

__device__ __forceinline__ float load_in(const float *p) { return *p; }
__device__ __forceinline__ float load_in(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// Context length as the kernels use it: negative lengths count as 0 and
// lengths over the table's capacity or the host's bound are clamped; both
// set PA_STATUS_BAD_CONTEXT (only `report` callers flag, to flag once).
__device__ __forceinline__ int clamp_context(int c, int cap, bool report) {
    if (c < 0 || c > cap) {
        if (report) flag_status(PA_STATUS_BAD_CONTEXT);
        c = c < 0 ? 0 : cap;
    }
    return c;
}

}  // namespace pa
