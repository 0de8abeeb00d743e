// gspn_lane.cuh -- small per-lane helpers of the TMA-fed compact kernels:
// shared-memory accesses through ordinary pointers, bf16 packing, the packed
// fp32x2 subtract and the mixed-precision bf16 FMA of sm_100.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace gspn {
namespace lane {

constexpr unsigned FULL = 0xffffffffu;

// Shared memory is addressed through ordinary pointers into the dynamic
// shared array, so the compiler folds constant offsets into the accesses; the
// TMA-written data is read only after the mbarrier wait (an asm with a memory
// clobber), which orders these loads behind it.
__device__ __forceinline__ uint4 lds128(const unsigned char* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ float4 lds128f(const unsigned char* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ uint32_t lds32(const unsigned char* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ float2 lds64f(const unsigned char* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ void sts64f(unsigned char* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void stg_cs32(__nv_bfloat16* p, uint32_t v) {
    __stcs(reinterpret_cast<unsigned int*>(p), v);
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// a - b, exactly rounded (sm_100 has packed add and fma but no packed subtract)
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }

// c + a*b with a, b the low / high bf16 halves of two 32-bit words: the bf16
// operands feed the fp32 FMA directly (mixed-precision fma of sm_100), exact
// products and one rounding, like the fp32 FMA of the widened values.
__device__ __forceinline__ float fma_bf_lo(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.bf16 %0, a0, b0, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_bf_hi(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.bf16 %0, a1, b1, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
// `half` is a compile-time constant at every (unrolled) call site
__device__ __forceinline__ float fma_bf(int half, uint32_t a, uint32_t b, float c) {
    return half ? fma_bf_hi(a, b, c) : fma_bf_lo(a, b, c);
}

// Scratch that lives in L2 between two phases of a kernel: stored with the
// evict-last priority, read back once, then discarded (the dead lines are
// dropped without a write-back to DRAM).
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void stg128_keep(float* p, float4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ float2 ldg64_keep(const float* p, uint64_t pol) {
    float2 v;
    asm volatile("ld.global.L2::cache_hint.v2.f32 {%0, %1}, [%2], %3;" : "=f"(v.x), "=f"(v.y) : "l"(p), "l"(pol) : "memory");
    return v;
}
__device__ __forceinline__ void stg64_keep(float* p, float2 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(v.x), "f"(v.y), "l"(pol) : "memory");
}
__device__ __forceinline__ float4 ldg128_keep(const float* p, uint64_t pol) {
    float4 v;
    asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol)
                 : "memory");
    return v;
}
// drop one 128-byte L2 line (128-byte aligned address); its contents become undefined
__device__ __forceinline__ void l2_discard128(const void* p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

}  // namespace lane
}  // namespace gspn
