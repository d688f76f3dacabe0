// Shared device helpers of libw4a8 (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "w4a8.h"

namespace w4a8 {

// One status word per device. Kernels record the first internal fault here
// (a bounded wait that ran out) instead of trapping, so the context stays
// usable and the host can read the code back. The library is one
// translation unit (w4a8_abi.cu includes every kernel header), so this is the
// only definition.
__device__ int g_device_status = 0;

__device__ __forceinline__ void record_fault(int code) {
    atomicCAS(&g_device_status, 0, code);
}

// Programmatic dependent launch: wait for the grids this one depends on to
// finish (their writes are then visible), and let dependents start launching.
// Both are no-ops when the launch carries no programmatic dependency.
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Loads of values that a grid this launch depends on may write (activations,
// scales, bias; the weights too, as far as the kernel can tell). The kernels
// here are launched with a programmatic dependency, so they can be running
// while their predecessor still writes: such values are not constant for the
// kernel's lifetime, which the read-only (.nc, __ldg) path requires, and a
// load the compiler treats as invariant may be scheduled above
// griddepcontrol.wait. These are plain coherent loads in volatile asm, which
// stays in program order with the (volatile) wait.
//   ld_dep*   : cached at all levels (reused operands);
//   ld_dep_cg*: cached in L2 only, for bytes that are used once.
__device__ __forceinline__ float ld_dep(const float *p) {
    float v;
    asm volatile("ld.global.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_dep_u8(const uint8_t *p) {
    uint32_t v;
    asm volatile("ld.global.u8 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ int32_t ld_dep_s32(const int32_t *p) {
    int32_t v;
    asm volatile("ld.global.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ int32_t ld_dep_s8(const int8_t *p) {
    int32_t v;
    asm volatile("ld.global.s8 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ float4 ld_dep_f4(const float *p) {
    float4 v;
    asm volatile("ld.global.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ld_dep_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ld_dep_cg_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Streaming load (evict-first in L1 and L2) for bytes read once per call.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Activation quantization (step 3 of "How it works"): the row scale from the
// row's abs-max (1 for an all-zero row), and one code as a byte.
__device__ __forceinline__ float act_scale_from_amax(float a) {
    return a == 0.0f ? 1.0f : __fdiv_rn(127.0f, a);
}
__device__ __forceinline__ uint32_t act_code8(float v, float s, bool in) {
    const int q = in ? min(max(__float2int_rn(__fmul_rn(v, s)), -127), 127) : 0;
    return (uint32_t)(q & 0xFF);
}

// Warm L2 with [p, p + bytes) (bytes a multiple of 16, p 16-byte aligned)
// without returning data: safe to issue before griddepcontrol.wait, because
// L2 is the point of coherence and no stale value reaches a register.
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Sign-extend the eight 4-bit two's-complement codes of one packed word.
// Byte b of `p` holds codes k = 2b (low nibble) and k = 2b + 1 (high nibble).
// Returns lo = bytes {k0, k2, k4, k6} and hi = bytes {k1, k3, k5, k7} as INT8.
// Nibble v becomes v | 0xF0 when its sign bit (bit 3) is set: the product
// (bit3 << 3) * 0x1E = 0xF0 stays inside its byte, so one multiply sets the
// high nibbles of all four bytes at once.
__device__ __forceinline__ void unpack_s4x8(uint32_t p, uint32_t &lo, uint32_t &hi) {
    const uint32_t m = 0x0F0F0F0Fu, s = 0x08080808u;
    uint32_t t = p >> 4;
    lo = (p & m) + (p & s) * 0x1Eu;
    hi = (t & m) + (t & s) * 0x1Eu;
}

// Dequantize one INT32 accumulator and apply the Dense epilogue, in the same
// float32 operations and order as the method's statement:
//   y = float(acc) / (sx * sw); y += bias; y = y > 0 ? y : +0.
__device__ __forceinline__ float dequant_value(int32_t acc, float sxm, float swn, bool has_bias, float b,
                                               bool relu) {
    float d = __fmul_rn(sxm, swn);
    float y = __fdiv_rn(__int2float_rn(acc), d);
    if (has_bias) y = __fadd_rn(y, b);
    if (relu) y = y > 0.0f ? y : 0.0f;
    return y;
}

// Write output (m, n) in the format `flags` selects; b is bias[n] when a
// bias is given.
__device__ __forceinline__ void store_value(void *__restrict__ Y, int ldy, int m, int n, int32_t acc, float sxm,
                                            float swn, bool has_bias, float b, unsigned flags) {
    size_t off = (size_t)m * (size_t)ldy + (size_t)n;
    unsigned fmt = flags & W4A8_OUT_MASK;
    if (fmt == W4A8_OUT_S32) {
        static_cast<int32_t *>(Y)[off] = acc;
        return;
    }
    float y = dequant_value(acc, sxm, swn, has_bias, b, (flags & W4A8_RELU) != 0);
    if (fmt == W4A8_OUT_BF16)
        static_cast<__nv_bfloat16 *>(Y)[off] = __float2bfloat16_rn(y);
    else
        static_cast<float *>(Y)[off] = y;
}

__device__ __forceinline__ void store_out(void *__restrict__ Y, int ldy, int m, int n,
                                          int32_t acc, float sxm, float swn,
                                          const float *__restrict__ bias, unsigned flags) {
    const bool has_bias = bias != nullptr && (flags & W4A8_OUT_MASK) != W4A8_OUT_S32;
    store_value(Y, ldy, m, n, acc, sxm, swn, has_bias, has_bias ? ld_dep(bias + n) : 0.0f, flags);
}

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return min(max(v, lo), hi); }

// The zero-point form of the weights stores each code q in [0, 15] as the
// signed nibble q - 8, so the W4A8 product gives acc' = sum_k xq (q - 8) and
// the layer's accumulator is acc = acc' - (zp[n] - 8) * rowsum[m], rowsum[m]
// = sum_k xq[m][k] (the "INT4" concept page, section 4.1). Product kernels
// take these two arrays and correct in their epilogue (64-bit, then the
// INT32 result, which the method's accumulator holds); null zp: no
// correction (the symmetric layer).
struct ZpArgs {
    const int32_t *zp;
    const int32_t *rowsum;
};
__device__ __forceinline__ int32_t zp_fix(int32_t acc, const ZpArgs &z, int m, int n) {
    if (z.zp == nullptr) return acc;
    return (int32_t)((long long)acc - ((long long)ld_dep_s32(z.zp + n) - 8) * (long long)ld_dep_s32(z.rowsum + m));
}

}  // namespace w4a8
