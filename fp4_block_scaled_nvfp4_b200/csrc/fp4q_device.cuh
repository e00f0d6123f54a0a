// fp4q_device.cuh -- device-side building blocks for the sm_100a kernels: packed f32x2
// arithmetic, the hardware E2M1 / E4M3 conversions, and the bf16 unpacking.  Every helper
// is one IEEE binary32 operation (round to nearest even) per lane, so the kernels follow
// the library's arithmetic contract exactly.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace fp4q {

typedef unsigned long long u64;

// ---- packed pairs of floats (sm_100 f32x2 instructions) ---------------------------------
// Caution (measured on B200 with CUDA 12.9): a mul.rn.f32x2 whose result feeds an
// add/sub.rn.f32x2 can be contracted by the assembler into one fused multiply-add, dropping
// the rounding of the product despite the .rn qualifiers.  Where the contract rounds a
// product before adding it, use the scalar __fmul_rn/__fadd_rn/__fsub_rn intrinsics.
__device__ __forceinline__ u64 pk(float a, float b) {
    u64 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk(u64 v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
    u64 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
    u64 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ u64 add2(u64 a, u64 b) {
    u64 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ u64 sub2(u64 a, u64 b) {
    u64 r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// ---- E2M1 ---------------------------------------------------------------------------------
// Round two floats to E2M1 (nearest even, saturating at +-6, sign kept); the result byte
// holds `lo` in bits 0..3 and `hi` in bits 4..7.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint16_t r;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; mov.b16 %0, {t, 0}; }"
        : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t e2m1x2(u64 v) {
    float a, b;
    upk(v, a, b);
    return e2m1x2(a, b);
}
// Values of the two E2M1 codes in the low byte of c (low nibble -> g0).
__device__ __forceinline__ void e2m1x2_decode(uint32_t c, float& g0, float& g1) {
    asm("{ .reg .b8 t, z; .reg .b16 c16; .reg .b32 h; .reg .f16 a, b;\n"
        "  cvt.u16.u32 c16, %2; mov.b16 {t, z}, c16;\n"
        "  cvt.rn.f16x2.e2m1x2 h, t; mov.b32 {a, b}, h;\n"
        "  cvt.f32.f16 %0, a; cvt.f32.f16 %1, b; }"
        : "=f"(g0), "=f"(g1) : "r"(c));
}
__device__ __forceinline__ u64 e2m1x2_decode(uint32_t c) {
    float a, b;
    e2m1x2_decode(c, a, b);
    return pk(a, b);
}

// ---- E4M3 (FN) ----------------------------------------------------------------------------
// Bit pattern of the nearest E4M3 value (ties to even, saturating at 448) of a finite v >= 0.
__device__ __forceinline__ int e4m3_rne(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0x7F;
}
// Value of E4M3 pattern p in [0, 126] (exact).
__device__ __forceinline__ float e4m3_value(int p) {
    const int E = p >> 3, M = p & 7;
    if (E == 0) return (float)M * 0x1p-9f;
    return (float)(8 + M) * __int_as_float((E - 10 + 127) << 23);
}

// ---- bf16 ---------------------------------------------------------------------------------
// Two bf16 values packed in one 32-bit word (element 2k in the low half) as a float pair.
__device__ __forceinline__ u64 bf16x2_to_pair(uint32_t w) {
    return pk(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// The magnitudes of the pair (sign bits cleared).
__device__ __forceinline__ u64 bf16x2_to_abs_pair(uint32_t w) {
    return pk(__uint_as_float((w & 0x7FFFu) << 16), __uint_as_float(w & 0x7FFF0000u));
}
// The sign bits of 8 bf16 values (value 2j in the low half of word wj, 2j + 1 in the high half)
// where E2M1 codes keep them: value i at bit 4 i + 3.  The high bytes of the eight values are
// gathered, split into even and odd values, and their bit 7 moved to bit 3 (even values).
__device__ __forceinline__ uint32_t bf16_sign_nibbles8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
    const uint32_t t = __byte_perm(w0, w1, 0x7531), u = __byte_perm(w2, w3, 0x7531);
    const uint32_t ev = __byte_perm(t, u, 0x6420), od = __byte_perm(t, u, 0x7531);
    return ((ev >> 4) & 0x08080808u) | (od & 0x80808080u);
}
// The same from 4 pairs of binary32 values (sign bit 31 of each).
__device__ __forceinline__ uint32_t f32_sign_nibbles8(u64 p0, u64 p1, u64 p2, u64 p3) {
    float a[8];
    upk(p0, a[0], a[1]);
    upk(p1, a[2], a[3]);
    upk(p2, a[4], a[5]);
    upk(p3, a[6], a[7]);
    uint32_t u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = __float_as_uint(a[i]);
    const uint32_t ev = __byte_perm(__byte_perm(u[0], u[2], 0x0073), __byte_perm(u[4], u[6], 0x0073), 0x5410);
    const uint32_t od = __byte_perm(__byte_perm(u[1], u[3], 0x0073), __byte_perm(u[5], u[7], 0x0073), 0x5410);
    return ((ev >> 4) & 0x08080808u) | (od & 0x80808080u);
}
// 2^k as a float for k in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2i(int k) {
    return k >= -126 ? __int_as_float((k + 127) << 23) : __int_as_float(0x00400000);
}

}  // namespace fp4q
