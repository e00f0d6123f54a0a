// fp4q.cu -- sm_100a kernels and the C ABI of libfp4q (declared in include/fp4q.h).
//
// Kernels (one CUDA thread owns one quantization block, so the per-block search runs in
// registers without any cross-thread reduction):
//   amax_kernel          tensor max|x| as an integer max over magnitude bit patterns
//                        (NaN/Inf sort above every finite value), one atomicMax per CTA;
//                        the last CTA to arrive computes S = RN(amax/1536) and the data
//                        flags.  ScaleSweep (gist.science/ko/paper/2606.07618),
//                        "Methodology", global scale S = max|x|/(256*6).
//   quant16_kernel<OBJ>  base scale, candidate sweep, RTN, block error, argmin, nibble
//                        pack, scale write.  ScaleSweep "Methodology" (offsets [-3,+7] MSE,
//                        [-8,+7] WMSE), 4/6 (Adaptive Block-Scaled Data Types,
//                        gist.science/ko/paper/2603.28765, "Problem").
//   if4_kernel           FP4 vs scaled-INT4 per block, indicator in the scale sign bit.
//                        Adaptive Block-Scaled Data Types, "Methodology", IF4 structure.
//   mxfp4_kernel<HAD>    E8M0 scale + RTN over 32-element blocks, optional in-register
//                        32-point fast Walsh-Hadamard rotation.  Bridging the Gap ...
//                        Microscaling FP4 (gist.science/ko/paper/2509.23202),
//                        "Methodology"; TORQ (gist.science/ko/paper/2605.19561) S-step.
//   HAD16 variants       amax, NVFP4 and IF4 kernels on blocks rotated by the normalized
//                        16-point Hadamard H_16/4 (in registers, before the scale is chosen);
//                        Bridging the Gap ..., "Methodology", block-wise Hadamard transforms,
//                        which rotates for both NVFP4 and MXFP4.
//   dequant kernels      codes + scales (+S) -> fp32 / bf16 (+ the inverse rotation).
// Status protocol (workspace words): each quantize kernel ORs its data flags into
// PENDING, counts its CTAs in an arrival counter, and the last CTA publishes
// STATUS = PENDING and zeroes PENDING and the counter, so the workspace is clean again
// after every call.
#include <cmath>
#include <cstdint>
#include <mutex>
#include <vector>
#include <cuda_runtime.h>

#include "fp4q.h"
#include "fp4q_device.cuh"

namespace fp4q {

enum : int { WS_STATUS = 0, WS_PENDING = 1, WS_AMAX = 2, WS_CNT_AMAX = 3, WS_CNT_Q = 4 };
constexpr size_t kWorkspaceBytes = 64;
constexpr int kThreads = 256;
constexpr float kRintMagic = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ bool scale_range_ok(float S) {
    if (S == 0.0f) return true;
    return S >= 0x1p-117f && S <= __fdiv_rn(0x1p125f, 1536.0f);
}

// Data flags implied by the tensor scale: NaN/Inf S -> NONFINITE, S outside the supported
// range -> RANGE (every candidate scale must stay normal and every reciprocal finite).
__device__ __forceinline__ uint32_t scale_flags(float S) {
    if (!isfinite(S)) return FP4Q_DEVSTAT_NONFINITE;
    return scale_range_ok(S) ? 0u : (uint32_t)FP4Q_DEVSTAT_RANGE;
}

// Publish this CTA's data flags; the last CTA of the grid writes the call's status word.
__device__ __forceinline__ void finish_status(uint32_t* ws, uint32_t flag, int cnt) {
    __shared__ uint32_t s_flag;
    if (threadIdx.x == 0) s_flag = 0u;
    __syncthreads();
    if (flag) atomicOr(&s_flag, flag);
    __syncthreads();
    if (threadIdx.x == 0) {
        if (s_flag) atomicOr(&ws[WS_PENDING], s_flag);
        __threadfence();
        const unsigned prev = atomicAdd(&ws[cnt], 1u);
        if (prev == gridDim.x - 1) {
            __threadfence();
            const uint32_t all = atomicExch(&ws[WS_PENDING], 0u);
            atomicExch(&ws[WS_STATUS], all);
            atomicExch(&ws[cnt], 0u);
        }
    }
}

// Byte offset of the scale of block (r, j) -- row r, column block j of jblocks -- in the tiled
// layout that block-scaled tensor-core GEMMs read their scale factors in: 128-row x 4-column
// tiles of 512 bytes, tiles row-major over (r / 128, j / 4), and inside a tile row r%32 at
// 16 (r%32) + 4 ((r/32)%4) + j%4.  The scale tensor is padded to whole tiles.
template <typename IDX>
__device__ __forceinline__ int64_t tiled_scale_offset(IDX r, IDX j, IDX jblocks) {
    const int64_t jt = ((int64_t)jblocks + 3) >> 2;
    return ((int64_t)r >> 7) * (jt * 512) + ((int64_t)j >> 2) * 512 + ((int64_t)r & 31) * 16 +
           (((int64_t)r >> 5) & 3) * 4 + ((int64_t)j & 3);
}
// Scale offset of linear block index blk of a tensor with jblocks blocks per row.
template <typename IDX>
__device__ __forceinline__ int64_t scale_offset(IDX blk, IDX jblocks, bool tiled) {
    if (!tiled) return (int64_t)blk;
    const IDX r = blk / jblocks;
    return tiled_scale_offset<IDX>(r, blk - r * jblocks, jblocks);
}

// ------------------------------------------------------------------------------------------
// amax
// ------------------------------------------------------------------------------------------
// Combine the per-thread maxima m (magnitude bit patterns) of the CTA, fold them into the
// workspace word, and let the last CTA write S = RN(RN(amax * post) / div) (NaN when any
// element was NaN or infinite) and, when publish is set, the status word.  div = 256 times the
// element format's largest magnitude: 1536 for FP4 (NVFP4, IF4), 1920 for FP6 (IF6).
__device__ __forceinline__ void amax_finish(uint32_t m, float post, uint32_t* ws, float* gscale, int publish,
                                            float div = 1536.0f) {
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    __shared__ uint32_t red[kThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w) m = max(m, red[w]);
        atomicMax(&ws[WS_AMAX], m);
        __threadfence();
        const unsigned prev = atomicAdd(&ws[WS_CNT_AMAX], 1u);
        if (prev == gridDim.x - 1) {
            __threadfence();
            const uint32_t bits = atomicExch(&ws[WS_AMAX], 0u);
            atomicExch(&ws[WS_CNT_AMAX], 0u);
            const float S = bits >= 0x7F800000u ? __uint_as_float(0x7FC00000u)
                                                : __fdiv_rn(__fmul_rn(__uint_as_float(bits), post), div);
            *gscale = S;
            if (publish) atomicExch(&ws[WS_STATUS], scale_flags(S));
        }
    }
}

// Fold one 16-byte vector into a running maximum of magnitude bit patterns: per 16-bit half for
// bf16 (amax_bits turns the pair into float bits), per word for fp32.
template <int IN>
__device__ __forceinline__ void amax_fold(uint32_t& m, const uint4 v) {
    if (IN == FP4Q_IN_BF16) {
        uint32_t t;
        const uint32_t mk = 0x7FFF7FFFu;
        asm("max.u16x2 %0, %1, %2;" : "=r"(t) : "r"(v.x & mk), "r"(v.y & mk));
        asm("max.u16x2 %0, %0, %1;" : "+r"(t) : "r"(v.z & mk));
        asm("max.u16x2 %0, %0, %1;" : "+r"(t) : "r"(v.w & mk));
        asm("max.u16x2 %0, %0, %1;" : "+r"(m) : "r"(t));
    } else {
        const uint32_t mk = 0x7FFFFFFFu;
        m = max(m, max(max(v.x & mk, v.y & mk), max(v.z & mk, v.w & mk)));
    }
}
template <int IN>
__device__ __forceinline__ uint32_t amax_bits(uint32_t m) {
    return IN == FP4Q_IN_BF16 ? max(m & 0xFFFFu, m >> 16) << 16 : m;   // bf16 bits -> f32 bits
}

// Largest magnitude of the elements in the 16-byte vectors first, first + step, ... of a
// rows x cols tensor with row pitch ld, as float bits (NaN and Inf order above every finite
// value as integers).  U loads are kept in flight per thread on contiguous tensors.
template <int IN, int U>
__device__ __forceinline__ uint32_t amax_partial(const void* __restrict__ xv, int64_t rows, int64_t cols, int64_t ld,
                                                 int64_t first, int64_t step) {
    const int64_t vpr = cols * (IN == FP4Q_IN_BF16 ? 2 : 4) / 16;   // 16-byte vectors per row
    const int64_t total = rows * vpr;
    uint32_t m = 0;
    const uint4* base = reinterpret_cast<const uint4*>(xv);
    const int64_t ldv = ld * (IN == FP4Q_IN_BF16 ? 2 : 4) / 16;
    auto fold = [&](const uint4 v) { amax_fold<IN>(m, v); };
    auto at = [&](int64_t i) -> const uint4* {
        if (ldv == vpr) return base + i;
        const int64_t r = i / vpr;
        return base + r * ldv + (i - r * vpr);
    };
    int64_t i = first;
    if (ldv == vpr) {   // contiguous tensor: U independent 16-byte loads in flight per thread
        for (; i + (U - 1) * step < total; i += U * step) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {   // read-only, no L1 allocation, 256-byte L2 fetches
                const uint4* src = base + i + u * step;
                asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v[u].x), "=r"(v[u].y), "=r"(v[u].z), "=r"(v[u].w) : "l"(src));
            }
#pragma unroll
            for (int u = 0; u < U; ++u) fold(v[u]);
        }
    } else {
        for (; i + 3 * step < total; i += 4 * step) {
            const uint4 v0 = __ldg(at(i)), v1 = __ldg(at(i + step)), v2 = __ldg(at(i + 2 * step)),
                        v3 = __ldg(at(i + 3 * step));
            fold(v0); fold(v1); fold(v2); fold(v3);
        }
    }
    for (; i < total; i += step) fold(__ldg(at(i)));
    return amax_bits<IN>(m);
}

template <int IN>
__global__ void __launch_bounds__(kThreads, 4) amax_kernel(const void* __restrict__ xv, int64_t rows, int64_t cols,
                                                        int64_t ld, uint32_t* __restrict__ ws,
                                                        float* __restrict__ gscale, int publish, float div) {
    const uint32_t m = amax_partial<IN, 8>(xv, rows, cols, ld, (int64_t)blockIdx.x * blockDim.x + threadIdx.x,
                                           (int64_t)gridDim.x * blockDim.x);
    amax_finish(m, 1.0f, ws, gscale, publish, div);
}

// ------------------------------------------------------------------------------------------
// Shared pieces of the NVFP4 / IF4 kernels
// ------------------------------------------------------------------------------------------
// Per-pattern scale table {inv, e} with e = the E4M3 value of pattern p and inv = RN(1/sv),
// sv = RN(e S), indexed by p + kTabPad for p = -kTabPad .. 126 + kTabPad, so that a candidate
// window [p0 - 8, p0 + 7] never leaves it.  Entries for patterns that are not candidates (p < 0 or
// p >= 127) hold inv = 0 and e = NaN: every score built from e is NaN and never wins, so the
// candidate loops need no bounds.  Pattern 0, the zero scale, holds inv = 0 and e = 0: its codes
// are the signs of the elements and its reconstruction is 0.
constexpr int kTabPad = 8;
constexpr int kTabLen = 127 + 2 * kTabPad;
__device__ __forceinline__ void build_scale_table(float S, float2* tab) {
    for (int i = threadIdx.x; i < kTabLen; i += blockDim.x) {
        const int p = i - kTabPad;
        float2 t = make_float2(0.0f, __uint_as_float(0x7FC00000u));
        if (p == 0) t.y = 0.0f;
        if (p >= 1 && p <= 126) {
            const float e = e4m3_value(p);
            t = make_float2(__frcp_rn(__fmul_rn(e, S)), e);
        }
        tab[i] = t;
    }
    __syncthreads();
}

// Raw 16-byte vectors of one 16-element block (2 for bf16, 4 for fp32), loaded ahead of the
// scale table so that their latency overlaps it, and their conversion to 8 float pairs.
template <int IN>
struct RawBlock16 {
    uint4 v[IN == FP4Q_IN_BF16 ? 2 : 4];
};
template <int IN>
__device__ __forceinline__ void load_raw16(const void* xv, int64_t off, RawBlock16<IN>& rb) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(xv) + off * (IN == FP4Q_IN_BF16 ? 2 : 4));
#pragma unroll
    for (int q = 0; q < (IN == FP4Q_IN_BF16 ? 2 : 4); ++q) rb.v[q] = __ldg(p + q);
}
// The same loads marked evict-first in L2: in a batch the block's second read (the first was
// the previous kernel's amax read, marked evict-last) is its last use.
template <int IN>
__device__ __forceinline__ void load_raw16_last_use(const void* xv, int64_t off, RawBlock16<IN>& rb) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(xv) + off * (IN == FP4Q_IN_BF16 ? 2 : 4));
#pragma unroll
    for (int q = 0; q < (IN == FP4Q_IN_BF16 ? 2 : 4); ++q)
        asm("{ .reg .b64 pol;\n"
            "  createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n"
            "  ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], pol; }"
            : "=r"(rb.v[q].x), "=r"(rb.v[q].y), "=r"(rb.v[q].z), "=r"(rb.v[q].w) : "l"(p + q));
}
template <int IN, bool LAST_USE>
__device__ __forceinline__ void load_block(const void* xv, int64_t off, RawBlock16<IN>& rb) {
    if constexpr (LAST_USE) load_raw16_last_use<IN>(xv, off, rb);
    else load_raw16<IN>(xv, off, rb);
}
template <int IN>
__device__ __forceinline__ void unpack16(const RawBlock16<IN>& rb, u64 (&xp)[8]) {
    if (IN == FP4Q_IN_BF16) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            xp[4 * q] = bf16x2_to_pair(rb.v[q].x); xp[4 * q + 1] = bf16x2_to_pair(rb.v[q].y);
            xp[4 * q + 2] = bf16x2_to_pair(rb.v[q].z); xp[4 * q + 3] = bf16x2_to_pair(rb.v[q].w);
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            xp[2 * q] = pk(__uint_as_float(rb.v[q].x), __uint_as_float(rb.v[q].y));
            xp[2 * q + 1] = pk(__uint_as_float(rb.v[q].z), __uint_as_float(rb.v[q].w));
        }
    }
}

// Where block blk of a rows x cols tensor with row pitch ld lives: element offset of its
// first value, its column block b, and its byte offset in the codes.  Contiguous rows
// (ld == cols) need no division.
template <typename IDX>
struct BlockAt {
    int64_t xoff, coff;
    IDX b;
};
template <typename IDX, bool NEED_COL>
__device__ __forceinline__ BlockAt<IDX> block_at(IDX blk, IDX cols, IDX ld, IDX nb) {
    BlockAt<IDX> a;
    if (ld == cols) {
        a.xoff = (int64_t)blk * 16;
        a.coff = (int64_t)blk * 8;
        a.b = NEED_COL ? blk % nb : 0;
    } else {
        const IDX r = blk / nb, b = blk - r * nb;
        a.xoff = (int64_t)r * ld + (int64_t)b * 16;
        a.coff = (int64_t)blk * 8;
        a.b = b;
    }
    return a;
}

__device__ __forceinline__ float block_absmax(const u64 (&xp)[8]) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a, b;
        upk(xp[j], a, b);
        m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
    }
    return m;
}

// Fast Walsh-Hadamard butterflies h = 1, 2, 4, 8 over one 16-element block held as 8
// (even, odd) pairs, without the normalization: h = 1 combines the two halves of a pair
// (scalar), h = 2, 4, 8 combine whole pairs k and k + h/2 (packed).
__device__ __forceinline__ void fwht16_butterflies(u64 (&xp)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a, b;
        upk(xp[j], a, b);
        xp[j] = pk(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {   // h counts pairs: element stride 2h
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if ((j & h) == 0) {
                const u64 a = xp[j], b = xp[j + h];
                xp[j] = add2(a, b);
                xp[j + h] = sub2(a, b);
            }
        }
    }
}

// Normalized 16-point Hadamard H_16 / 4 of one block: the butterflies, then each value times
// 1/sqrt(16) = 1/4 (a single rounding, exact unless the product is subnormal).
__device__ __forceinline__ void fwht16(u64 (&xp)[8]) {
    fwht16_butterflies(xp);
    const u64 q = pk(0.25f, 0.25f);
#pragma unroll
    for (int j = 0; j < 8; ++j) xp[j] = mul2(xp[j], q);
}

template <int IN>
__device__ __forceinline__ uint32_t amax_had16_partial(const void* __restrict__ xv, int64_t rows, int64_t cols,
                                                       int64_t ld, int64_t first, int64_t step) {
    constexpr int VPB = IN == FP4Q_IN_BF16 ? 2 : 4;   // 16-byte vectors per block
    constexpr int U = 8 / VPB;                        // blocks in flight per thread
    const int64_t nb = cols / 16;
    const int64_t total = rows * nb;
    uint32_t m = 0;
    auto src = [&](int64_t blk) {
        const int64_t r = blk / nb;
        const int64_t off = r * ld + (blk - r * nb) * 16;   // elements
        return reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(xv) + off * (IN == FP4Q_IN_BF16 ? 2 : 4));
    };
    auto fold = [&](const uint4 (&v)[VPB]) {
        u64 xp[8];
        if (IN == FP4Q_IN_BF16) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                xp[4 * q] = bf16x2_to_pair(v[q].x); xp[4 * q + 1] = bf16x2_to_pair(v[q].y);
                xp[4 * q + 2] = bf16x2_to_pair(v[q].z); xp[4 * q + 3] = bf16x2_to_pair(v[q].w);
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                xp[2 * q] = pk(__uint_as_float(v[q].x), __uint_as_float(v[q].y));
                xp[2 * q + 1] = pk(__uint_as_float(v[q].z), __uint_as_float(v[q].w));
            }
        }
        fwht16_butterflies(xp);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float a, b;
            upk(xp[j], a, b);
            m = max(m, max(__float_as_uint(a) & 0x7FFFFFFFu, __float_as_uint(b) & 0x7FFFFFFFu));
        }
    };
    auto load = [&](int64_t blk, uint4 (&v)[VPB]) {
        const uint4* p = src(blk);
#pragma unroll
        for (int q = 0; q < VPB; ++q)   // read-only, no L1 allocation, 256-byte L2 fetches
            asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v[q].x), "=r"(v[q].y), "=r"(v[q].z), "=r"(v[q].w) : "l"(p + q));
    };
    int64_t blk = first;
    for (; blk + (U - 1) * step < total; blk += U * step) {
        uint4 v[U][VPB];
#pragma unroll
        for (int u = 0; u < U; ++u) load(blk + u * step, v[u]);
#pragma unroll
        for (int u = 0; u < U; ++u) fold(v[u]);
    }
    for (; blk < total; blk += step) {
        uint4 v[VPB];
        load(blk, v);
        fold(v);
    }
    return m;
}

// Tensor amax of the rotated blocks.  Every thread rotates whole 16-element blocks and keeps
// the largest unnormalized magnitude; the factor 1/4 is applied once to the maximum, which
// gives the maximum of the normalized values because RN(a/4) is non-decreasing in a and
// |RN(v/4)| = RN(|v|/4).  The raw 16-byte vectors of several blocks (eight loads for bf16,
// the same bytes for fp32) are issued before any of them is converted, so the registers hold
// the loads in flight rather than unpacked pairs.
template <int IN>
__global__ void __launch_bounds__(kThreads, 4) amax_had16_kernel(const void* __restrict__ xv, int64_t rows,
                                                              int64_t cols, int64_t ld, uint32_t* __restrict__ ws,
                                                              float* __restrict__ gscale, int publish) {
    const uint32_t m = amax_had16_partial<IN>(xv, rows, cols, ld, (int64_t)blockIdx.x * blockDim.x + threadIdx.x,
                                              (int64_t)gridDim.x * blockDim.x);
    amax_finish(m, 0.25f, ws, gscale, publish);
}

// ------------------------------------------------------------------------------------------
// Exact block errors
// ------------------------------------------------------------------------------------------
// A candidate with grid step g (FP4: sv; INT4: RN(RN(6/7) sv); MXFP4: 2^e) gives element i the
// code magnitude m_i, and the block error is
//   E = sum (|x_i| - m_i g)^2 = sum x_i^2 + g (g Q - 2 X),   Q = sum m_i^2,  X = sum |x_i| m_i.
// The kernels evaluate it in fixed point.  Per block a shift k puts the magnitudes on integers
// A_i = |x_i| 2^k (exact for every element that any candidate of the window can give a nonzero
// code: those lie within a factor 2^7 of the block maximum, and bf16 values carry 8 significant
// bits, so 15-bit integers hold them; binary32 values need 31 bits), and M_i = 2 m_i is a byte
// (E2M1: 0,1,2,3,4,6,8,12; INT4: 0,2,...,14).  Q4 = sum M_i^2 and Xi = sum A_i M_i are exact
// integer dot products (dp4a / dp2a), and with sigma4 = g 2^(k-2),
//   G = sigma4 (sigma4 Q4 - Xi) = (E - sum x^2) 2^(2k) / 4,
// the same positive multiple of E - sum x^2 for every candidate of the block, so candidates are
// ranked by G.  In binary32, t = fma(sigma4, Q4, -Xi) and G~ = sigma4 t are each one rounding of
// an exact value, so |G~ - G| <= 2^-22.9 |G|: a candidate whose G~ exceeds min G~ + 2^-20 |min G~|
// is certainly worse.  When two or more candidates lie inside that margin (exact ties among
// them), the block is decided on the exact G = hi + lo held in binary64: u = sigma4 Q4 - Xi is
// exact there (fewer than 45 significant bits), hi = RN(sigma4 u), lo = fma(sigma4, u, -hi).
// ScaleSweep (gist.science/ko/paper/2606.07618), Methodology: the objective is the block's
// reconstruction error.

constexpr uint32_t kLutE2M1Lo = 0x03020100u, kLutE2M1Hi = 0x0C080604u;   // 2 m for E2M1 codes 0..7
constexpr uint32_t kMagicInt = 0x4B000000u;                              // bits of 2^23: ints < 2^23 ride in the mantissa
constexpr float kTwo23 = 8388608.0f;

// floor(log2 a) of a finite a > 0 (subnormals included).
__device__ __forceinline__ int ilog2f(float a) {
    const uint32_t u = __float_as_uint(a);
    return u >= 0x00800000u ? (int)(u >> 23) - 127 : -118 - __clz(u);
}
// 2^k as two factors that are normal floats for k in [-250, 250].
__device__ __forceinline__ void pow2_split(int k, float& fa, float& fb) {
    const int ka = k >> 1;
    fa = pow2i(ka);
    fb = pow2i(k - ka);
}

// Fixed-point magnitudes of one block of 2 NP elements.  B16 (bf16 values): w[j] = A_{2j} | A_{2j+1} << 16
// (15-bit integers).  Otherwise (binary32 values, 31-bit integers): w[4g + b] = byte b of A_{4g},
// A_{4g+1}, A_{4g+2}, A_{4g+3} (byte planes, so that each plane is one dp4a operand).
template <bool B16, int NP = 8>
struct Fixed16 {
    uint32_t w[B16 ? NP : 2 * NP];
};

// xp: the block's values (pairs; their magnitudes are used), k: the shift, from a block maximum a
// with a 2^k in [2^14, 2^15) (B16) or [2^30, 2^31).
// ABS: xp holds magnitudes (bf16 values: packed multiplies, exact as the scalar ones).
template <bool B16, int NP = 8, bool ABS = false>
__device__ __forceinline__ void fixed_point(const u64 (&xp)[NP], int k, Fixed16<B16, NP>& A) {
    float fa, fb;
    pow2_split(k, fa, fb);
    if (B16 && ABS) {
        const u64 fa2 = pk(fa, fa), fb2 = pk(fb, fb), m2 = pk(kTwo23, kTwo23);
#pragma unroll
        for (int j = 0; j < NP; ++j) {   // |x| 2^k + 2^23 (every step exact for the elements that count)
            float v0, v1;
            upk(fma2(mul2(xp[j], fa2), fb2, m2), v0, v1);
            A.w[j] = __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x5410);
        }
    } else if (B16) {
#pragma unroll
        for (int j = 0; j < NP; ++j) {   // RN(|x| 2^k + 2^23): the integer sits in the low mantissa bits
            float x0, x1;
            upk(xp[j], x0, x1);
            const float v0 = __fmaf_rn(__fmul_rn(fabsf(x0), fa), fb, kTwo23);
            const float v1 = __fmaf_rn(__fmul_rn(fabsf(x1), fa), fb, kTwo23);
            A.w[j] = __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x5410);
        }
    } else {
#pragma unroll
        for (int g = 0; g < NP / 2; ++g) {
            uint32_t a[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float v0, v1;
                upk(xp[2 * g + h], v0, v1);
                a[2 * h] = __float2uint_rz(__fmul_rn(__fmul_rn(fabsf(v0), fa), fb));   // exact integers below 2^31
                a[2 * h + 1] = __float2uint_rz(__fmul_rn(__fmul_rn(fabsf(v1), fa), fb));
            }
            const uint32_t t01 = __byte_perm(a[0], a[1], 0x5140), t23 = __byte_perm(a[2], a[3], 0x5140);
            const uint32_t u01 = __byte_perm(a[0], a[1], 0x7362), u23 = __byte_perm(a[2], a[3], 0x7362);
            A.w[4 * g + 0] = __byte_perm(t01, t23, 0x5410);
            A.w[4 * g + 1] = __byte_perm(t01, t23, 0x7632);
            A.w[4 * g + 2] = __byte_perm(u01, u23, 0x5410);
            A.w[4 * g + 3] = __byte_perm(u01, u23, 0x7632);
        }
    }
}

// 2m of the E2M1 codes of four quotients (bytes in element order): two conversions to E2M1 (round
// to nearest even, saturating, sign in bit 3 of each code), the two code bytes joined over a zero
// high half into the selector, and one byte-permute lookup of the magnitude index.  ABS: the
// quotients are magnitudes, so the sign bits are clear; otherwise they are masked off first.
template <bool ABS>
__device__ __forceinline__ uint32_t mags4_fp4(u64 y01, u64 y23) {
    float y0, y1, y2, y3;
    upk(y01, y0, y1);
    upk(y23, y2, y3);
    uint32_t m;
    if (ABS) {
        asm("{ .reg .b8 c0, c1; .reg .b16 h0, h1; .reg .b32 s;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n"
            "  mov.b16 h0, {c0, c1};\n"
            "  mov.b16 h1, 0;\n"
            "  mov.b32 s, {h0, h1};\n"
            "  prmt.b32 %0, %5, %6, s; }"
            : "=r"(m) : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "r"(kLutE2M1Lo), "r"(kLutE2M1Hi));
    } else {
        asm("{ .reg .b8 c0, c1; .reg .b16 h0, h1; .reg .b32 s;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n"
            "  mov.b16 h0, {c0, c1};\n"
            "  mov.b16 h1, 0;\n"
            "  mov.b32 s, {h0, h1};\n"
            "  and.b32 s, s, 0x7777;\n"
            "  prmt.b32 %0, %5, %6, s; }"
            : "=r"(m) : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "r"(kLutE2M1Lo), "r"(kLutE2M1Hi));
    }
    return m;
}

// 2|n| of the INT4 codes of four quotients y: |n| = min(rint(RN(|y| RN(7/6))), 7), each step a
// separate binary32 rounding (scalar intrinsics are never contracted); adding 1.5 2^23 rounds to
// an integer (ties to even) that sits in the low mantissa bits.
__device__ __forceinline__ uint32_t mags4_int4(u64 y01, u64 y23, float K76) {
    float y[4];
    upk(y01, y[0], y[1]);
    upk(y23, y[2], y[3]);
    uint32_t t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        t[i] = __float_as_uint(fminf(__fadd_rn(__fmul_rn(fabsf(y[i]), K76), kRintMagic), kRintMagic + 7.0f));
    const uint32_t n = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
    return (n & 0x07070707u) << 1;
}

// Exact integer sums of one candidate: Q4 = sum M^2 and the X partials (B16: one sum; binary32
// values: one per byte plane).  q and x start at the caller's value (kMagicInt for B16).
// ABS: xp holds magnitudes.
template <bool B16, bool INT4, int NP = 8, bool ABS = false>
__device__ __forceinline__ void cand_sums(const u64 (&xp)[NP], const Fixed16<B16, NP>& A, float inv, float K76, uint32_t& q,
                                          uint32_t (&x)[B16 ? 1 : 4]) {
    const u64 inv2 = pk(inv, inv);
#pragma unroll
    for (int g = 0; g < NP / 2; ++g) {
        const u64 y01 = mul2(xp[2 * g], inv2), y23 = mul2(xp[2 * g + 1], inv2);
        const uint32_t m4 = INT4 ? mags4_int4(y01, y23, K76) : mags4_fp4<ABS>(y01, y23);
        q = __dp4a(m4, m4, q);
        if (B16) {
            x[0] = __dp2a_lo(A.w[2 * g], m4, x[0]);
            x[0] = __dp2a_hi(A.w[2 * g + 1], m4, x[0]);
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b) x[b] = __dp4a(A.w[4 * g + b], m4, x[b]);
        }
    }
}

// IF4 at one scale, bf16 values.  The FP4 sums of cand_sums, and the block's signed E2M1 code word
// (the conversions the sums already made, before their sign bits are masked off).
__device__ __forceinline__ uint2 fp4_sums_codes(const u64 (&xp)[8], const Fixed16<true>& A, float inv, uint32_t& q,
                                                uint32_t& x) {
    const u64 inv2 = pk(inv, inv);
    uint32_t h[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float y0, y1, y2, y3;
        upk(mul2(xp[2 * g], inv2), y0, y1);
        upk(mul2(xp[2 * g + 1], inv2), y2, y3);
        uint32_t m4;
        asm("{ .reg .b8 c0, c1; .reg .b16 h0, h1; .reg .b32 t;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c0, %3, %2;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c1, %5, %4;\n"
            "  mov.b16 h0, {c0, c1};\n"
            "  mov.b16 h1, 0;\n"
            "  mov.b32 %1, {h0, h1};\n"
            "  and.b32 t, %1, 0x7777;\n"
            "  prmt.b32 %0, %6, %7, t; }"
            : "=r"(m4), "=r"(h[g]) : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "r"(kLutE2M1Lo), "r"(kLutE2M1Hi));
        q = __dp4a(m4, m4, q);
        x = __dp2a_lo(A.w[2 * g], m4, x);
        x = __dp2a_hi(A.w[2 * g + 1], m4, x);
    }
    return make_uint2(__byte_perm(h[0], h[1], 0x5410), __byte_perm(h[2], h[3], 0x5410));
}

// IF4 at one scale, bf16 values: the INT4 sums in binary32 and the block's INT4 code word.
// n = rint(RN(RN(x inv) RN(7/6))) rides in the low mantissa bits of v = RN(z + 1.5 2^23), clamped
// to [-7, 7] when CLAMP (at a normal, unsaturated base pattern |y| <= 6.4 (1 + 2^-21): the E4M3
// rounding of a_b / RN(6 S) is within 1/16, so |z| stays below 7.5 and it needs none); the low
// nibble of v's bits is n's two's complement code.  xs = sum x n and qs = sum n^2 are exact in
// binary32: every product x n with n != 0 is a multiple of ulp(a_b) 2^-4 (|x| >= a_b / 15 there,
// and x has 8 significant bits) and the sum stays below 2^19 such units.  In the fixed point of
// the FP4 sums (A = |x| 2^k, M = 2|n|): X = 2^(k+1) xs and Q4 = 4 qs.
template <bool CLAMP>
__device__ __forceinline__ uint2 int4_sums_f(const u64 (&xp)[8], float inv, float K76, float& qs, float& xs) {
    const u64 inv2 = pk(inv, inv), mag2 = pk(kRintMagic, kRintMagic);
    u64 xa = 0ull, qa = 0ull;   // +0.0f pairs
    uint32_t cw[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float y0, y1;
        upk(mul2(xp[j], inv2), y0, y1);
        float v0 = __fadd_rn(__fmul_rn(y0, K76), kRintMagic), v1 = __fadd_rn(__fmul_rn(y1, K76), kRintMagic);
        if (CLAMP) {
            v0 = fminf(fmaxf(v0, kRintMagic - 7.0f), kRintMagic + 7.0f);
            v1 = fminf(fmaxf(v1, kRintMagic - 7.0f), kRintMagic + 7.0f);
        }
        const u64 n2 = sub2(pk(v0, v1), mag2);   // exact
        xa = fma2(xp[j], n2, xa);
        qa = fma2(n2, n2, qa);
        const uint32_t byte = (__float_as_uint(v0) & 0xFu) | ((__float_as_uint(v1) & 0xFu) << 4);
        cw[j >> 2] |= byte << (8 * (j & 3));
    }
    float a, b;
    upk(xa, a, b);
    xs = __fadd_rn(a, b);
    upk(qa, a, b);
    qs = __fadd_rn(a, b);
    return make_uint2(cw[0], cw[1]);
}

// The fast score G~ of a candidate from its sums, and its exact value in binary64.
template <bool B16>
__device__ __forceinline__ float fast_G(float s4, uint32_t q, const uint32_t (&x)[B16 ? 1 : 4]) {
    if (B16) {
        const float q4 = __fsub_rn(__uint_as_float(q), kTwo23), xi = __fsub_rn(__uint_as_float(x[0]), kTwo23);
        return __fmul_rn(s4, __fmaf_rn(s4, q4, -xi));
    }
    // X = xh + xl exactly (each below 2^24 times a power of two); t = RN(RN(s4 Q4 - xh) - xl) is
    // within 2^-23.9 (1 + 2^-12) |t| of the exact value, since xl < 2^-12 |t| wherever it matters
    const float xh = __fmul_rn((float)(x[3] * 256u + x[2]), 65536.0f), xl = (float)(x[1] * 256u + x[0]);
    return __fmul_rn(s4, __fsub_rn(__fmaf_rn(s4, (float)q, -xh), xl));
}
struct ExactG {
    double hi, lo;
};
template <bool B16>
__device__ __forceinline__ ExactG exact_G(float s4, uint32_t q, const uint32_t (&x)[B16 ? 1 : 4]) {
    double xi;
    double q4;
    if (B16) {
        xi = (double)(x[0] - kMagicInt);
        q4 = (double)(q - kMagicInt);
    } else {
        xi = (double)x[3] * 16777216.0 + (double)x[2] * 65536.0 + (double)x[1] * 256.0 + (double)x[0];
        q4 = (double)q;
    }
    const double s = (double)s4;
    const double u = __fma_rn(s, q4, -xi);   // exact: fewer than 45 significant bits
    ExactG g;
    g.hi = __dmul_rn(s, u);
    g.lo = __fma_rn(s, u, -g.hi);
    return g;
}
// The same from the binary32 INT4 sums of int4_sums_f (Q4 = 4 qs, X = 2^(k+1) xs, both exact).
__device__ __forceinline__ ExactG exact_G_int4f(float s4, float qs, float xs, int k) {
    const double s = (double)s4;
    const double u = __fma_rn(s, 4.0 * (double)qs, -ldexp((double)xs, k + 1));   // exact, as in exact_G
    ExactG g;
    g.hi = __dmul_rn(s, u);
    g.lo = __fma_rn(s, u, -g.hi);
    return g;
}
__device__ __forceinline__ bool exact_less(const ExactG& a, const ExactG& b) {
    return a.hi < b.hi || (a.hi == b.hi && a.lo < b.lo);
}

// Candidates within 2^-20 of the smallest fast score (NaN scores, which mark patterns outside
// 0..126, are never inside): the index of the smallest when it is the only one, else -1.  The
// count runs on the FMA pipe: d = RN(thr - g) is >= 0 exactly when g <= thr, and
// sat(d 2^126 + 1) is then 1; it is 0 for d <= -2^-126 and for NaN, and in between only for
// candidates that are (barely) outside, which can only raise the count -- a count of exactly 1
// therefore means the smallest is alone inside the margin, and the weighted sum is its index.
template <int N>
__device__ __forceinline__ int near_min_unique(const float (&g)[N]) {
    float m = g[0];
#pragma unroll
    for (int c = 1; c < N; ++c) m = fminf(m, g[c]);
    const float thr = __fmaf_rn(fabsf(m), 0x1p-20f, m);
    float cnt = 0.0f, idx = 0.0f;
#pragma unroll
    for (int c = 0; c < N; ++c) {
        const float st = __saturatef(__fmaf_rn(__fsub_rn(thr, g[c]), 0x1p126f, 1.0f));
        cnt = __fadd_rn(cnt, st);
        idx = __fmaf_rn(st, (float)c, idx);
    }
    return cnt == 1.0f ? (int)idx : -1;
}

// The same candidates as a bit mask (the exact decision's input).
template <int N>
__device__ __forceinline__ uint32_t near_min_mask(const float (&g)[N]) {
    float m = g[0];
#pragma unroll
    for (int c = 1; c < N; ++c) m = fminf(m, g[c]);
    const float thr = __fmaf_rn(fabsf(m), 0x1p-20f, m);
    uint32_t mask = 0;
#pragma unroll
    for (int c = 0; c < N; ++c) mask |= (g[c] <= thr ? 1u : 0u) << c;
    return mask;
}

// Per-block context of the searches: magnitudes, fixed point, the per-tensor table base.
// Table entry of pattern p: {inv = RN(1/sv), e = the E4M3 value}, sv = RN(e S); patterns outside
// 1..126 hold inv = 0 and e = NaN (pattern 0, the zero scale, holds e = 0).
template <bool B16>
struct BlockCtx {
    u64 xp[8];          // the block's values (pairs); the searches use their magnitudes
    Fixed16<B16> A;
    float T;            // S 2^(k-2): sigma4 of pattern p is RN(e(p) T) = sv(p) 2^(k-2)
    int k;              // the fixed-point shift: A = |x| 2^k
};

template <bool B16, bool ABS = false>
__device__ __forceinline__ void block_ctx(const u64 (&xp)[8], float ab, float S, BlockCtx<B16>& c) {
#pragma unroll
    for (int j = 0; j < 8; ++j) c.xp[j] = xp[j];
    // an element reaches a nonzero code only from |x| >= sv/4 >= 2^-11 S, so a maximum below that
    // is raised to it (all codes are zero then, and the integers need not be exact)
    const float aeff = fmaxf(ab, __fmul_rn(S, 0x1p-11f));
    const int k = (B16 ? 14 : 30) - ilog2f(aeff);
    fixed_point<B16, 8, ABS>(c.xp, k, c.A);
    float fa, fb;
    pow2_split(k - 2, fa, fb);
    c.T = __fmul_rn(__fmul_rn(S, fa), fb);
    c.k = k;
}

// Exact comparison of the candidates in `mask` (bit c = window offset c, INT4 at odd bits when
// TWO_TYPES), their sums recomputed; the lowest index wins a tie.  The branch that reaches it is
// rare; inlined, it needs no call frame and no spills around a call.  ABS: c.xp holds magnitudes.
template <bool B16, bool TWO_TYPES, bool ABS>
__device__ __forceinline__ int exact_pick(const BlockCtx<B16>& c, const float2* t, uint32_t mask, float K76, float K67) {
    int best = -1;
    ExactG bg = {0.0, 0.0};
    for (; mask; mask &= mask - 1) {
        const int i = __ffs(mask) - 1;
        const int off = TWO_TYPES ? i >> 1 : i;
        const bool int4 = TWO_TYPES && (i & 1);
        const float2 e = t[off];
        uint32_t q = B16 ? kMagicInt : 0u, x[B16 ? 1 : 4];
#pragma unroll
        for (int b = 0; b < (B16 ? 1 : 4); ++b) x[b] = B16 ? kMagicInt : 0u;
        float s4 = __fmul_rn(e.y, c.T);
        if (int4) {
            cand_sums<B16, true, 8, ABS>(c.xp, c.A, e.x, K76, q, x);
            s4 = __fmul_rn(K67, s4);
        } else {
            cand_sums<B16, false, 8, ABS>(c.xp, c.A, e.x, K76, q, x);
        }
        const ExactG g = exact_G<B16>(s4, q, x);
        if (best < 0 || exact_less(g, bg)) {
            bg = g;
            best = i;
        }
    }
    return best;
}

// The window search of the NVFP4 MSE sweep (offsets 0..NOFF-1 from table entry t = base + p0 - 3)
// or of the IF4 sweep (TWO_TYPES: FP4 and INT4 at each offset, FP4 first); returns the winning
// index.  Each candidate's fast score is kept; only when another candidate lies within the
// margin of the smallest are the close ones' sums recomputed and compared exactly.  ABS: c.xp
// holds magnitudes.
template <bool B16, bool TWO_TYPES, int NOFF, bool ABS = false>
__device__ __forceinline__ int window_search(const BlockCtx<B16>& c, const float2* t, float K76, float K67) {
    constexpr int N = TWO_TYPES ? 2 * NOFF : NOFF;
    float g[N];
#pragma unroll
    for (int o = 0; o < NOFF; ++o) {
        const float2 e = t[o];
        const float s4 = __fmul_rn(e.y, c.T);
        uint32_t q = B16 ? kMagicInt : 0u, x[B16 ? 1 : 4];
#pragma unroll
        for (int b = 0; b < (B16 ? 1 : 4); ++b) x[b] = B16 ? kMagicInt : 0u;
        cand_sums<B16, false, 8, ABS>(c.xp, c.A, e.x, K76, q, x);
        g[TWO_TYPES ? 2 * o : o] = fast_G<B16>(s4, q, x);
        if (TWO_TYPES) {
            const float s4i = __fmul_rn(K67, s4);
            q = B16 ? kMagicInt : 0u;
#pragma unroll
            for (int b = 0; b < (B16 ? 1 : 4); ++b) x[b] = B16 ? kMagicInt : 0u;
            cand_sums<B16, true, 8, ABS>(c.xp, c.A, e.x, K76, q, x);
            g[2 * o + 1] = fast_G<B16>(s4i, q, x);
        }
    }
    const int unique = near_min_unique<N>(g);
    if (unique >= 0) return unique;
    return exact_pick<B16, TWO_TYPES, ABS>(c, t, near_min_mask<N>(g), K76, K67);
}

// Packed codes of a block (signed values xp) at reciprocal scale inv: 8 bytes, elements 0..15; the
// code bytes of each 8 elements are joined with two half-word packs.
__device__ __forceinline__ uint2 block_codes(const u64 (&xp)[8], float inv) {
    const u64 inv2 = pk(inv, inv);
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float y[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) upk(mul2(xp[4 * h + j], inv2), y[2 * j], y[2 * j + 1]);
        asm("{ .reg .b8 c0, c1, c2, c3; .reg .b16 h0, h1;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n"
            "  cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n"
            "  mov.b16 h0, {c0, c1};\n"
            "  mov.b16 h1, {c2, c3};\n"
            "  mov.b32 %0, {h0, h1}; }"
            : "=r"(w[h]) : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
    }
    return make_uint2(w[0], w[1]);
}
// INT4 codes of a block at reciprocal scale inv: n = clamp(rint(RN(RN(x inv) RN(7/6))), -7, 7) as
// 4-bit two's complement nibbles (the low bits of 1.5 2^23 + n).
__device__ __forceinline__ uint2 block_codes_int4(const u64 (&xp)[8], float inv, float K76) {
    const u64 inv2 = pk(inv, inv);
    uint32_t ci[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float y0, y1;
        upk(mul2(xp[j], inv2), y0, y1);
        const float t0 = fminf(fmaxf(__fadd_rn(__fmul_rn(y0, K76), kRintMagic), kRintMagic - 7.0f), kRintMagic + 7.0f);
        const float t1 = fminf(fmaxf(__fadd_rn(__fmul_rn(y1, K76), kRintMagic), kRintMagic - 7.0f), kRintMagic + 7.0f);
        ci[j] = (__float_as_uint(t0) & 0xFu) | ((__float_as_uint(t1) & 0xFu) << 4);
    }
    return make_uint2(ci[0] | (ci[1] << 8) | (ci[2] << 16) | (ci[3] << 24),
                      ci[4] | (ci[5] << 8) | (ci[6] << 16) | (ci[7] << 24));
}

// WMSE error of one candidate, binary32 with one accumulator in element order:
// xhat = RN(q sv), d = RN(|x| - xhat), acc = fma(RN(w d), d, acc) (on magnitudes: RN is odd, so
// d, RN(w d) d and the sum equal those of the signed values).
__device__ __forceinline__ float wmse_error(const u64 (&ap)[8], const u64 (&wp)[8], float inv, float sv) {
    const u64 inv2 = pk(inv, inv);
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a0, a1, w0, w1, q0, q1;
        upk(ap[j], a0, a1);
        upk(wp[j], w0, w1);
        e2m1x2_decode(e2m1x2(mul2(ap[j], inv2)), q0, q1);
        const float d0 = __fsub_rn(a0, __fmul_rn(q0, sv));
        acc = __fmaf_rn(__fmul_rn(w0, d0), d0, acc);
        const float d1 = __fsub_rn(a1, __fmul_rn(q1, sv));
        acc = __fmaf_rn(__fmul_rn(w1, d1), d1, acc);
    }
    return acc;
}

// ------------------------------------------------------------------------------------------
// NVFP4: AbsMax / 4-over-6 / ScaleSweep MSE [-3,+7] / ScaleSweep WMSE [-8,+7] of one block.
// The block stays in registers for the whole candidate search.  ScaleSweep
// (gist.science/ko/paper/2606.07618), Methodology; 4/6: Adaptive Block-Scaled Data Types
// (gist.science/ko/paper/2603.28765), Problem.
// ------------------------------------------------------------------------------------------
// ABS (the MSE sweep): xp holds the magnitudes and sgn the sign bits at their code positions
// (bit 4 i + 3), put back into the codes at the end.
template <int OBJ, bool B16, bool ABS>
__device__ __forceinline__ void nvfp4_block(const u64 (&xp)[8], uint2 sgn, const float* __restrict__ imp,
                                            int64_t colblk, float S, float d6, float d4, const float2* tab,
                                            uint2* cdst, uint8_t* sdst) {
    static_assert(!ABS || OBJ == FP4Q_SWEEP_MSE, "magnitude inputs serve the MSE sweep");
    int bp = 0;
    if (S > 0.0f) {
        const float ab = block_absmax(xp);
        const int p0 = e4m3_rne(__fdiv_rn(ab, d6));
        bp = p0;
        if (OBJ == FP4Q_FOUR_OVER_SIX) {
            const int p4 = e4m3_rne(__fdiv_rn(ab, d4));   // p4 >= p0
            if (p4 != p0) {   // the two scales compared exactly; a tie keeps max -> 6
                BlockCtx<B16> c;
                block_ctx<B16>(xp, ab, S, c);
                ExactG g[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float2 e = tab[i ? p4 : p0];
                    uint32_t q = B16 ? kMagicInt : 0u, x[B16 ? 1 : 4];
#pragma unroll
                    for (int b = 0; b < (B16 ? 1 : 4); ++b) x[b] = B16 ? kMagicInt : 0u;
                    cand_sums<B16, false>(c.xp, c.A, e.x, 0.0f, q, x);
                    g[i] = exact_G<B16>(__fmul_rn(e.y, c.T), q, x);
                }
                if (exact_less(g[1], g[0])) bp = p4;
            }
        } else if (OBJ == FP4Q_SWEEP_MSE) {
            // below 2^-11 S no element reaches a nonzero code at any candidate: every candidate
            // ties with the zero scale (p0 is 0 there), the lowest offset
            if (__fmul_rn(ab, 0x1p11f) >= S) {
                BlockCtx<B16> c;
                block_ctx<B16, ABS>(xp, ab, S, c);
                bp = p0 - 3 + window_search<B16, false, 11, ABS>(c, tab + p0 - 3, 0.0f, 0.0f);
            }
        } else if (OBJ == FP4Q_SWEEP_WMSE) {
            // candidates p0 - 8 .. p0 + 7 in increasing offset with strict improvement (ties keep
            // the lowest offset); patterns outside 0..126 score NaN and are never taken; if every
            // error is +inf the first candidate is kept
            u64 wp[8], ap[8];
            const float4* w4 = reinterpret_cast<const float4*>(imp + colblk * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float4 v = __ldg(w4 + j);
                wp[2 * j] = pk(v.x, v.y);
                wp[2 * j + 1] = pk(v.z, v.w);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float a, b;
                upk(xp[j], a, b);
                ap[j] = pk(fabsf(a), fabsf(b));
            }
            float best = INFINITY;
            int kb = max(-8, -p0);
            const float2* t = tab + p0;
#pragma unroll
            for (int k = -8; k <= 7; ++k) {
                const float2 e = t[k];
                const float err = wmse_error(ap, wp, e.x, __fmul_rn(e.y, S));
                if (err < best) {
                    best = err;
                    kb = k;
                }
            }
            bp = p0 + kb;
        }
    }
    uint2 cw = block_codes(xp, tab[bp].x);
    if (ABS) cw = make_uint2(cw.x | sgn.x, cw.y | sgn.y);
    *cdst = cw;
    *sdst = (uint8_t)bp;
}

// ------------------------------------------------------------------------------------------
// IF4 of one block: FP4 (E2M1) vs scaled INT4 at the shared AbsMax scale, the lower exact block
// error kept (a tie keeps FP4), indicator in bit 7 of the scale byte.  Adaptive Block-Scaled Data
// Types (gist.science/ko/paper/2603.28765), Methodology, IF4 structure and the 6/7 method.
// SWEEP: IF4 x ScaleSweep, every candidate scale of the MSE window p0 - 3 .. p0 + 7 under both
// element types, the lowest (error, offset, FP4 before INT4) -- the IF4 page's type choice
// searched jointly with ScaleSweep (gist.science/ko/paper/2606.07618), Methodology (MSE window).
// ------------------------------------------------------------------------------------------
template <bool SWEEP, bool B16>
__device__ __forceinline__ void if4_block(const u64 (&xp)[8], float S, float d6, float K76, float K67,
                                          const float2* tab, uint2* cdst, uint8_t* sdst) {
    int bp = 0;
    bool use_int = false;
    if (S > 0.0f) {
        const float ab = block_absmax(xp);
        const int p0 = e4m3_rne(__fdiv_rn(ab, d6));
        bp = p0;
        if (__fmul_rn(ab, 0x1p11f) >= S) {   // otherwise every candidate ties: FP4 at the lowest offset
            BlockCtx<B16> c;
            block_ctx<B16>(xp, ab, S, c);
            if (SWEEP) {
                const int i = window_search<B16, true, 11>(c, tab + p0 - 3, K76, K67);
                bp = p0 - 3 + (i >> 1);
                use_int = (i & 1) != 0;
            } else if constexpr (B16) {
                // both element types at p0, each type's codes taken from its own evaluation
                const float2 e = tab[p0];
                const float s4 = __fmul_rn(e.y, c.T);
                uint32_t q = kMagicInt, x[1] = {kMagicInt};
                const uint2 cw_fp = fp4_sums_codes(c.xp, c.A, e.x, q, x[0]);
                const ExactG gf = exact_G<true>(s4, q, x);
                float qs, xs;
                // below pattern 8 (subnormal) and at 126 (where a_b / RN(6 S) may exceed the largest
                // E4M3 value when S is given) |y| can pass 6.4, so the INT4 codes are clamped there
                const uint2 cw_int = p0 >= 8 && p0 < 126 ? int4_sums_f<false>(c.xp, e.x, K76, qs, xs)
                                                         : int4_sums_f<true>(c.xp, e.x, K76, qs, xs);
                const ExactG gi = exact_G_int4f(__fmul_rn(K67, s4), qs, xs, c.k);
                use_int = exact_less(gi, gf);
                *cdst = use_int ? cw_int : cw_fp;
                *sdst = (uint8_t)(bp | (use_int ? 0x80 : 0));
                return;
            } else {
                const float2 e = tab[p0];
                const float s4 = __fmul_rn(e.y, c.T);
                uint32_t q = 0u, x[4] = {0u, 0u, 0u, 0u};
                cand_sums<B16, false>(c.xp, c.A, e.x, K76, q, x);
                const ExactG gf = exact_G<B16>(s4, q, x);
                q = 0u;
#pragma unroll
                for (int b = 0; b < 4; ++b) x[b] = 0u;
                cand_sums<B16, true>(c.xp, c.A, e.x, K76, q, x);
                const ExactG gi = exact_G<B16>(__fmul_rn(K67, s4), q, x);
                use_int = exact_less(gi, gf);
            }
        } else if (SWEEP) {
            bp = max(p0 - 3, 0);
        }
    }
    const float inv = tab[bp].x;
    *cdst = use_int ? block_codes_int4(xp, inv, K76) : block_codes(xp, inv);
    *sdst = (uint8_t)(bp | (use_int ? 0x80 : 0));
}

// ------------------------------------------------------------------------------------------
// The NVFP4 / IF4 quantize kernel (KIND = the NVFP4 objective, or KIND_IF4).  Each thread
// walks the blocks tid, tid + G, ... (G threads in the grid) with the next block's loads in
// flight while the current one is searched; the CTA builds its scale table once.  The host
// picks the grid per kind: one block per thread (G >= blocks: the loop runs once) for the WMSE
// search, one persistent wave (the CTAs that fit on the SMs) for the other kinds, whose per-CTA
// start-up (S, table, first loads) would otherwise not be amortized.  The status word depends
// only on S, so CTA 0 writes it.
// ------------------------------------------------------------------------------------------
enum : int { KIND_IF4 = 4, KIND_IF4_SWEEP = 5 };   // kinds 0..3 are the NVFP4 objectives

template <int KIND>
__host__ __device__ constexpr bool q16_persistent() {
    return KIND != FP4Q_SWEEP_WMSE;
}
template <int KIND>
__host__ __device__ constexpr int q16_min_ctas() {   // register cap: CTAs per SM the kernel is compiled for
    return KIND == FP4Q_SWEEP_MSE || KIND == KIND_IF4_SWEEP ? 3 : (KIND == FP4Q_ABSMAX ? 5 : 4);
}

// The next tensor of a batch (fp4q_quantize_batch): same element type; its S is written to gs.
template <typename IDX>
struct NextTensor {
    const void* x;
    IDX rows, cols, ld;
    float* gs;
};

// 16-byte vector i of a tensor, counted row by row.
template <int IN, typename IDX>
__device__ __forceinline__ const uint4* vec_at(const NextTensor<IDX>& t, IDX i) {
    constexpr int es = IN == FP4Q_IN_BF16 ? 2 : 4;
    const IDX vpr = t.cols * es / 16, ldv = t.ld * es / 16;
    const uint4* base = reinterpret_cast<const uint4*>(t.x);
    if (ldv == vpr) return base + i;
    const IDX r = i / vpr;
    return base + r * ldv + (i - r * vpr);
}

// The next tensor's amax, folded while this tensor is quantized.  Thread t owns the vectors
// t, t + G, t + 2G, ... of the next tensor and takes two of them per block it quantizes: the
// pair is copied into the thread's own shared-memory slots by cp.async one block ahead and
// folded after the following block, so its HBM reads overlap the candidate search and hold
// no registers meanwhile.  Only the issuing thread reads a slot, so the group wait orders it.
// For AbsMax, which is bound by HBM, the copies are marked evict-last in L2 and the kernel's own
// reads evict-first, so that a tensor that fits in L2 is still there when the next kernel
// quantizes it (cfg3: 25.5 -> 21.0 us per tensor); the arithmetic-bound searches measured
// slightly slower with the hints and go without.
template <int IN, bool EVICT_LAST, typename IDX>
__device__ __forceinline__ void next_stage(const NextTensor<IDX>& t, IDX ntot, IDX v, IDX G, uint4* s) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const IDX i = v + (IDX)u * G;
        if (i < ntot) {
            const uint32_t dst = (uint32_t)__cvta_generic_to_shared(s + u * kThreads + threadIdx.x);
            if constexpr (EVICT_LAST)
                asm volatile("{ .reg .b64 pol;\n"
                             "  createpolicy.fractional.L2::evict_last.b64 pol, 1.0;\n"
                             "  cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, pol; }"
                             ::"r"(dst), "l"(vec_at<IN>(t, i)) : "memory");
            else
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(vec_at<IN>(t, i)) : "memory");
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int IN, typename IDX>
__device__ __forceinline__ void next_fold(IDX ntot, IDX v, IDX G, const uint4* s, uint32_t& m) {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
    for (int u = 0; u < 2; ++u)
        if (v + (IDX)u * G < ntot) amax_fold<IN>(m, s[u * kThreads + threadIdx.x]);
}

template <int IN, int KIND, bool HAD, typename IDX, bool NEXT>
__global__ void __launch_bounds__(kThreads, q16_min_ctas<KIND>())
    q16_kernel(const void* __restrict__ xv, IDX rows, IDX cols, IDX ld, const float* __restrict__ imp,
               uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, const float* __restrict__ gscale,
               uint32_t* __restrict__ ws, int tiled, NextTensor<IDX> nx, int status_or) {
    static_assert(!NEXT || (q16_persistent<KIND>() && !HAD), "the next tensor's amax rides on the persistent loop");
    __shared__ float2 s_tab[kTabLen];
    __shared__ uint4 s_nx[NEXT ? 2 * kThreads : 1];
    constexpr bool kL2Keep = NEXT && KIND == FP4Q_ABSMAX;   // keep the next tensor in L2
    const IDX nb = cols / 16;
    const IDX total = rows * nb;
    const IDX G = (IDX)gridDim.x * blockDim.x;
    IDX blk = (IDX)blockIdx.x * blockDim.x + threadIdx.x;
    // bf16 blocks (8 registers) are loaded before S and the table so the load latency overlaps
    // them; fp32 blocks (16 registers) would not fit the register cap across the table build
    RawBlock16<IN> rb;
    if (IN == FP4Q_IN_BF16 && blk < total) load_block<IN, kL2Keep>(xv, block_at<IDX, false>(blk, cols, ld, nb).xoff, rb);
    const float S = *gscale;
    const uint32_t flags = scale_flags(S);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (status_or) atomicOr(&ws[WS_STATUS], flags);
        else ws[WS_STATUS] = flags;
    }
    build_scale_table(S, s_tab);
    const float2* tab = s_tab + kTabPad;
    const float d6 = __fmul_rn(6.0f, S), d4 = __fmul_rn(4.0f, S);
    const float K76 = __fdiv_rn(7.0f, 6.0f), K67 = __fdiv_rn(6.0f, 7.0f);
    auto one_block = [&](IDX b) {
        const BlockAt<IDX> at = block_at<IDX, KIND == FP4Q_SWEEP_WMSE>(b, cols, ld, nb);
        uint2* cdst = reinterpret_cast<uint2*>(codes + at.coff);
        uint8_t* sdst = scales + scale_offset<IDX>(b, nb, tiled != 0);
        if (flags) {   // data out of contract: zero-filled outputs
            *cdst = make_uint2(0u, 0u);
            *sdst = 0;
            return;
        }
        if (IN != FP4Q_IN_BF16) load_block<IN, kL2Keep>(xv, at.xoff, rb);
        // the MSE sweep searches on magnitudes and puts the signs back into the codes at the end
        constexpr bool kAbs = KIND == FP4Q_SWEEP_MSE;
        constexpr bool kRawSigns = kAbs && IN == FP4Q_IN_BF16 && !HAD;
        u64 xp[8];
        uint2 sgn = make_uint2(0u, 0u);
        if constexpr (kRawSigns) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint4 v = rb.v[q];
                (q ? sgn.y : sgn.x) = bf16_sign_nibbles8(v.x, v.y, v.z, v.w);
                xp[4 * q] = bf16x2_to_abs_pair(v.x);
                xp[4 * q + 1] = bf16x2_to_abs_pair(v.y);
                xp[4 * q + 2] = bf16x2_to_abs_pair(v.z);
                xp[4 * q + 3] = bf16x2_to_abs_pair(v.w);
            }
        } else {
            unpack16<IN>(rb, xp);
        }
        if (q16_persistent<KIND>() && IN == FP4Q_IN_BF16 && b + G < total)   // next block's loads in flight
            load_block<IN, kL2Keep>(xv, block_at<IDX, false>(b + G, cols, ld, nb).xoff, rb);
        if (HAD) fwht16(xp);
        if constexpr (kAbs && !kRawSigns) {
            sgn = make_uint2(f32_sign_nibbles8(xp[0], xp[1], xp[2], xp[3]), f32_sign_nibbles8(xp[4], xp[5], xp[6], xp[7]));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float a0, a1;
                upk(xp[j], a0, a1);
                xp[j] = pk(fabsf(a0), fabsf(a1));
            }
        }
        constexpr bool B16 = IN == FP4Q_IN_BF16 && !HAD;   // bf16 values: 15-bit fixed point
        if (KIND == KIND_IF4) if4_block<false, B16>(xp, S, d6, K76, K67, tab, cdst, sdst);
        else if (KIND == KIND_IF4_SWEEP) if4_block<true, B16>(xp, S, d6, K76, K67, tab, cdst, sdst);
        else nvfp4_block<KIND, B16, kAbs>(xp, sgn, imp, at.b, S, d6, d4, tab, cdst, sdst);
    };
    if constexpr (NEXT) {
        const IDX ntot = nx.rows * (nx.cols * (IN == FP4Q_IN_BF16 ? 2 : 4) / 16);
        IDX nv = blk;
        uint32_t nm = 0;
        next_stage<IN, kL2Keep>(nx, ntot, nv, G, s_nx);
        for (; blk < total; blk += G) {
            one_block(blk);
            next_fold<IN>(ntot, nv, G, s_nx, nm);
            nv += 2 * G;
            next_stage<IN, kL2Keep>(nx, ntot, nv, G, s_nx);
        }
        next_fold<IN>(ntot, nv, G, s_nx, nm);
        for (nv += 2 * G; nv < ntot; nv += G) amax_fold<IN>(nm, __ldg(vec_at<IN>(nx, nv)));
        amax_finish(amax_bits<IN>(nm), 1.0f, ws, nx.gs, 0);
    } else if (q16_persistent<KIND>()) {
        for (; blk < total; blk += G) one_block(blk);
    } else if (blk < total) {
        one_block(blk);
    }
}

// ------------------------------------------------------------------------------------------
// IF6: FP6 E2M3 vs scaled INT6 per 16-element block, the IF4 idea at 6 bits.  Adaptive
// Block-Scaled Data Types (gist.science/ko/paper/2603.28765), Methodology ("extensibility" to
// 6-bit formats): one E4M3 scale per block, p0 = E4M3(RN(a_b / RN(7.5 S))), S = RN(amax / 1920);
// FP6 codes E2M3(RN(x inv)) reconstructed as q sv; INT6 codes n = clamp(rint(RN(RN(x inv) RN(62/15))),
// -31, 31) reconstructed as n RN(RN(15/62) sv); INT6 (bit 7 of the scale byte) when its exact block
// error is lower.  Codes: 6-bit fields, element i at bits 6i..6i+5 of the block's 12 bytes.
// The exact comparison is the NVFP4 one with M = 8m (FP6, multiples of 1/8 up to 7.5) and
// M = |n| (INT6): for M = c m the common multiple of E - sum x^2 is a (a Q - X), a = g 2^k / (2c).
// ------------------------------------------------------------------------------------------
// 8m of four FP6 codes (bytes, sign bit 5 ignored): e = bits 3..4, f = bits 0..2;
// 8m = f for e = 0, (8 + f) 2^(e-1) otherwise.
__device__ __forceinline__ uint32_t e2m3_m8(uint32_t c) {
    const uint32_t e = (c >> 3) & 3u, f = c & 7u;
    return e == 0 ? f : (8u + f) << (e - 1);
}

// 8m of the FP6 codes of four non-negative quotients (bytes in element order): two conversions to
// E2M3, their decode to f16 pairs, RN(8 m + 1024) in f16 (exact: 8m is an integer below 64, so
// the sum sits in [1024, 2048) where the f16 step is 1) leaves 8m in the low byte of each half,
// and one byte permute gathers the four bytes.
__device__ __forceinline__ uint32_t m8x4_fp6(float y0, float y1, float y2, float y3) {
    uint32_t m;
    asm("{ .reg .b16 c01, c23; .reg .b32 h01, h23, e8, k;\n"
        "  cvt.rn.satfinite.e2m3x2.f32 c01, %2, %1;\n"
        "  cvt.rn.satfinite.e2m3x2.f32 c23, %4, %3;\n"
        "  cvt.rn.f16x2.e2m3x2 h01, c01;\n"
        "  cvt.rn.f16x2.e2m3x2 h23, c23;\n"
        "  mov.b32 e8, 0x48004800;\n"
        "  mov.b32 k, 0x64006400;\n"
        "  fma.rn.f16x2 h01, h01, e8, k;\n"
        "  fma.rn.f16x2 h23, h23, e8, k;\n"
        "  prmt.b32 %0, h01, h23, 0x6420; }"
        : "=r"(m) : "f"(y0), "f"(y1), "f"(y2), "f"(y3));
    return m;
}

template <bool B16>
__device__ __forceinline__ void if6_block(const u64 (&xp)[8], float S, float d75, float K62, float K15,
                                          const float2* tab, uint8_t* cdst, uint8_t* sdst) {
    int p0 = 0;
    bool use_int = false;
    const float ab = block_absmax(xp);
    if (S > 0.0f) p0 = e4m3_rne(__fdiv_rn(ab, d75));
    const float2 te = tab[p0];
    const float inv = te.x;
    // below S/(16 * 512) every code of both types is zero: the tie keeps FP6
    if (S > 0.0f && __fmul_rn(ab, 0x1p13f) >= S) {
        u64 ap[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float a, b;
            upk(xp[j], a, b);
            ap[j] = pk(fabsf(a), fabsf(b));
        }
        // A = |x| 2^k with ab 2^k in [2^15, 2^16) (bf16) or [2^31, 2^32): every element with a
        // nonzero code of either type (|x| >= sv/16, ab <= 12 sv) is an exact integer
        const int k = (B16 ? 15 : 31) - ilog2f(ab);
        Fixed16<B16> A;
        fixed_point<B16>(ap, k, A);
        const u64 inv2 = pk(inv, inv);
        uint32_t qf = 0, qi = 0, xf[B16 ? 1 : 4] = {}, xi[B16 ? 1 : 4] = {};
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            float y[4];
            upk(mul2(ap[2 * g], inv2), y[0], y[1]);
            upk(mul2(ap[2 * g + 1], inv2), y[2], y[3]);
            const uint32_t mf = m8x4_fp6(y[0], y[1], y[2], y[3]);
            uint32_t t[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                t[i] = __float_as_uint(fminf(__fadd_rn(__fmul_rn(y[i], K62), kRintMagic), kRintMagic + 31.0f));
            const uint32_t mi = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410) &
                                0x1F1F1F1Fu;
            qf = __dp4a(mf, mf, qf);
            qi = __dp4a(mi, mi, qi);
            if (B16) {
                xf[0] = __dp2a_lo(A.w[2 * g], mf, xf[0]);
                xf[0] = __dp2a_hi(A.w[2 * g + 1], mf, xf[0]);
                xi[0] = __dp2a_lo(A.w[2 * g], mi, xi[0]);
                xi[0] = __dp2a_hi(A.w[2 * g + 1], mi, xi[0]);
            } else {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    xf[b] = __dp4a(A.w[4 * g + b], mf, xf[b]);
                    xi[b] = __dp4a(A.w[4 * g + b], mi, xi[b]);
                }
            }
        }
        auto xsum = [](const uint32_t (&x)[B16 ? 1 : 4]) {
            return B16 ? (double)x[0]
                       : (double)x[3] * 16777216.0 + (double)x[2] * 65536.0 + (double)x[1] * 256.0 + (double)x[0];
        };
        const float sv = __fmul_rn(te.y, S), gi = __fmul_rn(K15, sv);
        float fa, fb;
        pow2_split(k - 4, fa, fb);   // FP6: a = sv 2^k / 16
        const double af = (double)__fmul_rn(__fmul_rn(sv, fa), fb);
        pow2_split(k - 1, fa, fb);   // INT6: a = RN(RN(15/62) sv) 2^k / 2
        const double ai = (double)__fmul_rn(__fmul_rn(gi, fa), fb);
        ExactG g6, gn;
        const double uf = __fma_rn(af, (double)qf, -xsum(xf)), ui = __fma_rn(ai, (double)qi, -xsum(xi));
        g6.hi = __dmul_rn(af, uf);
        g6.lo = __fma_rn(af, uf, -g6.hi);
        gn.hi = __dmul_rn(ai, ui);
        gn.lo = __fma_rn(ai, ui, -gn.hi);
        use_int = exact_less(gn, g6);
    }
    // codes of the chosen type from the signed values, packed 6 bits each
    const u64 inv2 = pk(inv, inv);
    uint32_t fld[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float y0, y1;
        upk(mul2(xp[j], inv2), y0, y1);
        if (use_int) {
            const float t0 = fminf(fmaxf(__fadd_rn(__fmul_rn(y0, K62), kRintMagic), kRintMagic - 31.0f), kRintMagic + 31.0f);
            const float t1 = fminf(fmaxf(__fadd_rn(__fmul_rn(y1, K62), kRintMagic), kRintMagic - 31.0f), kRintMagic + 31.0f);
            fld[2 * j] = __float_as_uint(t0) & 0x3Fu;
            fld[2 * j + 1] = __float_as_uint(t1) & 0x3Fu;
        } else {
            uint16_t c;
            asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(y1), "f"(y0));
            fld[2 * j] = c & 0x3Fu;
            fld[2 * j + 1] = (c >> 8) & 0x3Fu;
        }
    }
    uint32_t w[3] = {0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int bit = 6 * i;
        w[bit >> 5] |= fld[i] << (bit & 31);
        if ((bit & 31) > 26) w[(bit >> 5) + 1] |= fld[i] >> (32 - (bit & 31));
    }
    uint32_t* d32 = reinterpret_cast<uint32_t*>(cdst);
    d32[0] = w[0];
    d32[1] = w[1];
    d32[2] = w[2];
    *sdst = (uint8_t)(p0 | (use_int ? 0x80 : 0));
}

template <int IN>
__global__ void __launch_bounds__(kThreads, 4)
    if6_kernel(const void* __restrict__ xv, int64_t rows, int64_t cols, int64_t ld, uint8_t* __restrict__ codes,
               uint8_t* __restrict__ scales, const float* __restrict__ gscale, uint32_t* __restrict__ ws) {
    __shared__ float2 s_tab[kTabLen];
    const int64_t nb = cols / 16;
    const int64_t total = rows * nb;
    const float S = *gscale;
    const uint32_t flags = scale_flags(S);
    if (blockIdx.x == 0 && threadIdx.x == 0) ws[WS_STATUS] = flags;
    build_scale_table(S, s_tab);
    const float2* tab = s_tab + kTabPad;
    const float d75 = __fmul_rn(7.5f, S);
    const float K62 = __fdiv_rn(62.0f, 15.0f), K15 = __fdiv_rn(15.0f, 62.0f);
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < total;
         blk += (int64_t)gridDim.x * blockDim.x) {
        // codes and scales are dense (12 bytes and 1 byte per block); the input row pitch needs
        // the row index only when rows are padded
        int64_t xoff = blk * 16;
        if (ld != cols) {
            const int64_t r = blk / nb;
            xoff = r * ld + (blk - r * nb) * 16;
        }
        uint8_t* cdst = codes + blk * 12;
        uint8_t* sdst = scales + blk;
        if (flags) {   // data out of contract: zero-filled outputs
            reinterpret_cast<uint32_t*>(cdst)[0] = 0u;
            reinterpret_cast<uint32_t*>(cdst)[1] = 0u;
            reinterpret_cast<uint32_t*>(cdst)[2] = 0u;
            *sdst = 0;
            continue;
        }
        RawBlock16<IN> rb;
        load_raw16<IN>(xv, xoff, rb);
        u64 xp[8];
        unpack16<IN>(rb, xp);
        if6_block<IN == FP4Q_IN_BF16>(xp, S, d75, K62, K15, tab, cdst, sdst);
    }
}

// ------------------------------------------------------------------------------------------
// MXFP4 (+ 32-point Hadamard)
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void fwht32(float (&v)[32]) {
    // h = 1 pairs neighbours within a register pair: scalar adds
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
        const float a = v[j], b = v[j + 1];
        v[j] = __fadd_rn(a, b);
        v[j + 1] = __fsub_rn(a, b);
    }
    // h = 2, 4, 8, 16: (v_j, v_j+1) and (v_j+h, v_j+h+1) butterfly as packed pairs
    u64 w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = pk(v[2 * j], v[2 * j + 1]);
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {   // h counts pairs: element stride 2h
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if ((j & h) == 0) {
                const u64 a = w[j], b = w[j + h];
                w[j] = add2(a, b);
                w[j + h] = sub2(a, b);
            }
        }
    }
    const float KH = (float)0.17677669529663688110021109052621;   // RN(1/sqrt(32))
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        upk(w[j], v[2 * j], v[2 * j + 1]);
        v[2 * j] = __fmul_rn(v[2 * j], KH);
        v[2 * j + 1] = __fmul_rn(v[2 * j + 1], KH);
    }
}

// Smallest e with a <= 6*2^e (ceil rule) or floor(log2 a) - 2 (OCP rule), clamped to [-127,127].
__device__ __forceinline__ int mx_exponent(float a, bool ocp) {
    if (a == 0.0f) return -127;
    int sh = 0;
    if (a < 0x1p-126f) { a = __fmul_rn(a, 0x1p24f); sh = 24; }   // exact rescale of subnormals
    const uint32_t u = __float_as_uint(a);
    const int k = (int)(u >> 23) - 127 - sh;                     // floor(log2 a)
    int e = ocp ? k - 2 : (k - 2 + ((u & 0x7FFFFFu) > 0x400000u ? 1 : 0));
    return min(max(e, -127), 127);
}

// MX scale sweep of one 32-element block (pairs vp, maximum magnitude ab): the exponent among
// e_c - 2 .. e_c (e_c the ceil rule, none below -127) with the lowest exact block error; the
// lowest exponent wins a tie.  In the fixed point of the NVFP4 searches, sigma4 = 2^(e + k - 2) is
// a power of two at least 2^9, so u = sigma4 Q4 - Xi is an integer below 2^41 and
// G = sigma4 u is exact in binary64.  Bridging the Gap ... Microscaling FP4
// (gist.science/ko/paper/2509.23202), Methodology: MXFP4 "Scale Fitting" of the power-of-two scale
// grid to the data.
template <bool B16>
__device__ __forceinline__ int mx_sweep_exponent(const u64 (&vp)[16], float ab, int ec) {
    if (ab == 0.0f) return ec;   // a zero block: every exponent ties, ec = -127 is the only one
    u64 ap[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float a, b;
        upk(vp[j], a, b);
        ap[j] = pk(fabsf(a), fabsf(b));
    }
    const int k = (B16 ? 14 : 30) - ilog2f(ab);
    Fixed16<B16, 16> A;
    fixed_point<B16, 16, true>(ap, k, A);
    int be = max(ec - 2, -127);
    double best = 0.0;
    bool first = true;
#pragma unroll
    for (int d = -2; d <= 0; ++d) {
        const int e = ec + d;
        if (e < -127) continue;
        uint32_t q = 0u, x[B16 ? 1 : 4] = {};
        cand_sums<B16, false, 16, true>(ap, A, pow2i(-e), 0.0f, q, x);
        const double xi = B16 ? (double)x[0]
                              : (double)x[3] * 16777216.0 + (double)x[2] * 65536.0 + (double)x[1] * 256.0 + (double)x[0];
        const double s4 = __longlong_as_double((long long)(1023 + e + k - 2) << 52);
        const double g = __dmul_rn(s4, __fma_rn(s4, (double)q, -xi));
        if (first || g < best) {
            best = g;
            be = e;
            first = false;
        }
    }
    return be;
}

template <int IN, bool HAD, bool SWEEP>
__global__ void __launch_bounds__(kThreads) mxfp4_kernel(const void* __restrict__ xv, int64_t rows, int64_t cols,
                                                         int64_t ld, uint8_t* __restrict__ codes,
                                                         uint8_t* __restrict__ scales, uint32_t* __restrict__ ws,
                                                         int ocp, int tiled) {
    const int64_t nb = cols / 32;
    const int64_t total = rows * nb;
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    uint32_t flag = 0;
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < total; blk += step) {
        const int64_t r = blk / nb, b = blk - r * nb;
        float v[32];
        // magnitude bits compared as unsigned integers (NaN > Inf > every finite value): one
        // maximum gives both the finiteness check and, unrotated, the block maximum
        uint32_t mb;
        if (IN == FP4Q_IN_BF16) {
            const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(xv) + r * ld + b * 32);
            uint32_t m2 = 0;   // two 16-bit maxima
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = __ldg(p + q);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    v[q * 8 + 2 * t] = __uint_as_float(ww[t] << 16);
                    v[q * 8 + 2 * t + 1] = __uint_as_float(ww[t] & 0xFFFF0000u);
                    m2 = __vmaxu2(m2, ww[t] & 0x7FFF7FFFu);
                }
            }
            mb = max(m2 & 0xFFFFu, m2 >> 16) << 16;
        } else {
            const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(xv) + r * ld + b * 32);
            mb = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 w = __ldg(p + q);
                v[4 * q] = w.x; v[4 * q + 1] = w.y; v[4 * q + 2] = w.z; v[4 * q + 3] = w.w;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) mb = max(mb, __float_as_uint(v[i]) & 0x7FFFFFFFu);
        }
        uint4* cdst = reinterpret_cast<uint4*>(codes + r * (cols / 2) + b * 16);
        uint8_t* sdst = scales + (tiled ? tiled_scale_offset<int64_t>(r, b, nb) : blk);
        if (mb >= 0x7F800000u) {   // a NaN or an infinity in the block
            flag = FP4Q_DEVSTAT_NONFINITE;
            *cdst = make_uint4(0u, 0u, 0u, 0u);
            *sdst = 0xFF;
            continue;
        }
        float ab = __uint_as_float(mb);
        if (HAD) {
            // the rotated maximum ignores a NaN that an overflowing butterfly can produce
            fwht32(v);
            ab = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) ab = fmaxf(ab, fabsf(v[i]));
        }
        u64 vp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) vp[j] = pk(v[2 * j], v[2 * j + 1]);
        const int e = SWEEP ? mx_sweep_exponent<IN == FP4Q_IN_BF16 && !HAD>(vp, ab, mx_exponent(ab, false))
                            : mx_exponent(ab, ocp != 0);
        const float m = pow2i(-e);
        const u64 m2 = pk(m, m);
        uint32_t c[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) c[j] = e2m1x2(mul2(vp[j], m2));   // x 2^-e is exact
        *cdst = make_uint4(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24),
                           c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24),
                           c[8] | (c[9] << 8) | (c[10] << 16) | (c[11] << 24),
                           c[12] | (c[13] << 8) | (c[14] << 16) | (c[15] << 24));
        *sdst = (uint8_t)(e + 127);
    }
    finish_status(ws, flag, WS_CNT_Q);
}

// ------------------------------------------------------------------------------------------
// Dequantize
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bf16_bits(float f) {
    if (isnan(f)) return 0x7FC0u;
    const uint32_t u = __float_as_uint(f);
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

template <bool OUT_BF16, int N>
__device__ __forceinline__ void store_values(void* out, int64_t off, const float (&v)[N]) {
    if (OUT_BF16 && N == 4) {
        *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(out) + off) =
            make_uint2(bf16_bits(v[0]) | (bf16_bits(v[1]) << 16), bf16_bits(v[2 % N]) | (bf16_bits(v[3 % N]) << 16));
    } else if (OUT_BF16) {
        uint4* p = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + off);
#pragma unroll
        for (int q = 0; q < N / 8; ++q) {
            uint32_t w[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) w[t] = bf16_bits(v[8 * q + 2 * t]) | (bf16_bits(v[8 * q + 2 * t + 1]) << 16);
            p[q] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
        float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + off);
#pragma unroll
        for (int q = 0; q < N / 4; ++q) p[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
}

// Unrotated dequantization with one thread per 4 consecutive elements of a row: each thread reads
// the 2 bytes of its codes and its block's scale byte and writes one 16-byte (fp32) or 8-byte
// (bf16) store, so a warp's loads and stores each cover one contiguous stretch of memory.
// FMT: FP4Q_NVFP4, FP4Q_IF4 (INT4 blocks: RN(n RN(RN(6/7) sv))) or FP4Q_MXFP4 (RN(q 2^e)).
template <bool OUT_BF16, int FMT>
__global__ void __launch_bounds__(kThreads) dequant_lin_kernel(const uint8_t* __restrict__ codes,
                                                               const uint8_t* __restrict__ scales,
                                                               const float* __restrict__ gscale, int64_t rows,
                                                               int64_t cols, void* __restrict__ out, int tiled) {
    constexpr int B = FMT == FP4Q_MXFP4 ? 32 : 16;
    const float S = FMT == FP4Q_MXFP4 ? 0.0f : *gscale;
    const float K67 = __fdiv_rn(6.0f, 7.0f);
    const int64_t q4 = cols / 4, nb = cols / B;
    const int64_t total = rows * q4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / q4, c = (i - r * q4) * 4, b = c / B;
        const uint32_t cw = __ldg(reinterpret_cast<const uint16_t*>(codes + r * (cols / 2) + c / 2));
        const uint32_t sb = __ldg(scales + (tiled ? tiled_scale_offset<int64_t>(r, b, nb) : r * nb + b));
        float v[4];
        if (FMT == FP4Q_MXFP4) {
            const float m = sb == 0xFFu ? __uint_as_float(0x7FC00000u) : pow2i((int)sb - 127);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float g0, g1;
                e2m1x2_decode((cw >> (8 * h)) & 0xFFu, g0, g1);
                v[2 * h] = __fmul_rn(g0, m);
                v[2 * h + 1] = __fmul_rn(g1, m);
            }
        } else {
            const int p = sb & 0x7F;
            const float sv = p == 0 ? 0.0f : (p == 127 ? __uint_as_float(0x7FC00000u) : __fmul_rn(e4m3_value(p), S));
            if (FMT == FP4Q_IF4 && (sb & 0x80)) {
                const float gi = __fmul_rn(K67, sv);   // the INT4 block scale RN(RN(6/7) sv)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int nib = (cw >> (4 * e)) & 0xF;
                    v[e] = __fmul_rn((float)(nib >= 8 ? nib - 16 : nib), gi);
                }
            } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float g0, g1;
                    e2m1x2_decode((cw >> (8 * h)) & 0xFFu, g0, g1);
                    v[2 * h] = __fmul_rn(g0, sv);
                    v[2 * h + 1] = __fmul_rn(g1, sv);
                }
            }
        }
        store_values<OUT_BF16>(out, r * cols + c, v);
    }
}

template <bool OUT_BF16, bool IF4, bool HAD>
__global__ void __launch_bounds__(kThreads) dequant16_kernel(const uint8_t* __restrict__ codes,
                                                             const uint8_t* __restrict__ scales,
                                                             const float* __restrict__ gscale, int64_t rows,
                                                             int64_t cols, void* __restrict__ out, int tiled) {
    const float S = *gscale;
    const float K67 = __fdiv_rn(6.0f, 7.0f);
    const int64_t nb = cols / 16;
    const int64_t total = rows * nb;
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < total; blk += step) {
        const int64_t r = blk / nb, b = blk - r * nb;
        const uint2 c = __ldg(reinterpret_cast<const uint2*>(codes + r * (cols / 2) + b * 8));
        const uint32_t sb = __ldg(scales + (tiled ? tiled_scale_offset<int64_t>(r, b, nb) : blk));
        const int p = sb & 0x7F;
        const float sv = p == 0 ? 0.0f : (p == 127 ? __uint_as_float(0x7FC00000u) : __fmul_rn(e4m3_value(p), S));
        const float gi = __fmul_rn(K67, sv);   // the INT4 block scale RN(RN(6/7) sv)
        float v[16];
        const uint32_t cw[2] = {c.x, c.y};
        if (IF4 && (sb & 0x80)) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int nib = (cw[i >> 3] >> ((i & 7) * 4)) & 0xF;
                const int n = nib >= 8 ? nib - 16 : nib;
                v[i] = __fmul_rn((float)n, gi);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float g0, g1;
                e2m1x2_decode((cw[j >> 2] >> ((j & 3) * 8)) & 0xFFu, g0, g1);
                v[2 * j] = __fmul_rn(g0, sv);
                v[2 * j + 1] = __fmul_rn(g1, sv);
            }
        }
        if (HAD) {   // inverse rotation: H_16 / 4 is its own inverse
            u64 vp[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) vp[j] = pk(v[2 * j], v[2 * j + 1]);
            fwht16(vp);
#pragma unroll
            for (int j = 0; j < 8; ++j) upk(vp[j], v[2 * j], v[2 * j + 1]);
        }
        store_values<OUT_BF16>(out, r * cols + b * 16, v);
    }
}

template <bool OUT_BF16, bool HAD>
__global__ void __launch_bounds__(kThreads) dequant_mx_kernel(const uint8_t* __restrict__ codes,
                                                              const uint8_t* __restrict__ scales, int64_t rows,
                                                              int64_t cols, void* __restrict__ out, int tiled) {
    const int64_t nb = cols / 32;
    const int64_t total = rows * nb;
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < total; blk += step) {
        const int64_t r = blk / nb, b = blk - r * nb;
        const uint4 c = __ldg(reinterpret_cast<const uint4*>(codes + r * (cols / 2) + b * 16));
        const uint32_t sb = __ldg(scales + (tiled ? tiled_scale_offset<int64_t>(r, b, nb) : blk));
        const float m = sb == 0xFFu ? __uint_as_float(0x7FC00000u) : pow2i((int)sb - 127);
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
        float v[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float g0, g1;
            e2m1x2_decode((cw[j >> 2] >> ((j & 3) * 8)) & 0xFFu, g0, g1);
            v[2 * j] = __fmul_rn(g0, m);
            v[2 * j + 1] = __fmul_rn(g1, m);
        }
        if (HAD) fwht32(v);
        store_values<OUT_BF16>(out, r * cols + b * 32, v);
    }
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(kThreads) dequant_if6_kernel(const uint8_t* __restrict__ codes,
                                                               const uint8_t* __restrict__ scales,
                                                               const float* __restrict__ gscale, int64_t rows,
                                                               int64_t cols, void* __restrict__ out) {
    const float S = *gscale;
    const float K15 = __fdiv_rn(15.0f, 62.0f);
    const int64_t nb = cols / 16;
    const int64_t total = rows * nb;
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < total;
         blk += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = blk / nb, b = blk - r * nb;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(codes + r * (cols * 3 / 4) + b * 12);
        const uint64_t lo = (uint64_t)__ldg(src) | ((uint64_t)__ldg(src + 1) << 32);
        const uint32_t hi = __ldg(src + 2);
        const uint32_t sb = __ldg(scales + blk);
        const int p = sb & 0x7F;
        const float sv = p == 0 ? 0.0f : (p == 127 ? __uint_as_float(0x7FC00000u) : __fmul_rn(e4m3_value(p), S));
        const float gi = __fmul_rn(K15, sv);
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int bit = 6 * i;
            const uint32_t f = bit < 64 ? (uint32_t)((bit <= 58 ? lo >> bit : (lo >> bit) | ((uint64_t)hi << (64 - bit))) & 0x3Fu)
                                        : (hi >> (bit - 64)) & 0x3Fu;
            if (sb & 0x80) {
                const int n = f >= 32 ? (int)f - 64 : (int)f;
                v[i] = __fmul_rn((float)n, gi);
            } else {
                const float m = __fmul_rn((float)e2m3_m8(f), 0.125f);   // exact
                v[i] = __fmul_rn((f & 0x20u) ? -m : m, sv);
            }
        }
        store_values<OUT_BF16>(out, r * cols + b * 16, v);
    }
}

// ------------------------------------------------------------------------------------------
// Element codec: the hardware conversions every quantize path uses, applied element by element
// (KIND 0: E2M1 round to nearest even, saturating, the 4-bit code with the sign in bit 3;
// KIND 1: E4M3FN round to nearest even, saturating, the whole byte).  Four elements per thread
// and step, one 4-byte store.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3_byte(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xFFu;
}

template <int KIND>
__global__ void __launch_bounds__(kThreads) encode_kernel(const float* __restrict__ x, int64_t n,
                                                          uint8_t* __restrict__ out) {
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t n4 = n / 4;
    for (int64_t i = tid; i < n4; i += step) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(x) + i);
        uint32_t w;
        if (KIND == 0) {
            const uint32_t c01 = e2m1x2(v.x, v.y), c23 = e2m1x2(v.z, v.w);   // low nibble = first element
            w = (c01 & 0xFu) | ((c01 >> 4) << 8) | ((c23 & 0xFu) << 16) | ((c23 >> 4) << 24);
        } else {
            w = e4m3_byte(v.x) | (e4m3_byte(v.y) << 8) | (e4m3_byte(v.z) << 16) | (e4m3_byte(v.w) << 24);
        }
        reinterpret_cast<uint32_t*>(out)[i] = w;
    }
    for (int64_t i = 4 * n4 + tid; i < n; i += step)
        out[i] = (uint8_t)(KIND == 0 ? (e2m1x2(x[i], 0.0f) & 0xFu) : e4m3_byte(x[i]));
}

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------
thread_local int g_launches = 0;

int sm_count() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    }
    return sms;
}

// Grid for a grid-stride kernel: enough CTAs for the work, at most one full wave (the CTAs
// the kernel's register and shared-memory use let every SM hold, and no more than
// ctas_per_sm per SM).
template <typename K>
int grid_for(K kernel, int64_t work_items, int ctas_per_sm) {
    // per-thread cache of the occupancy query, keyed by kernel address
    thread_local const void* keys[32] = {};
    thread_local int fits[32] = {};
    const void* key = reinterpret_cast<const void*>(kernel);
    int fit = 0, slot = 0;
    for (; slot < 32 && keys[slot]; ++slot)
        if (keys[slot] == key) { fit = fits[slot]; break; }
    if (fit == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, kernel, kThreads, 0) != cudaSuccess || fit <= 0) fit = 1;
        if (slot < 32) { keys[slot] = key; fits[slot] = fit; }
    }
    const int per_sm = fit < ctas_per_sm ? fit : ctas_per_sm;
    const int64_t need = (work_items + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)sm_count() * per_sm;
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

thread_local int g_cuda_error = 0;

int launched(int n) {
    g_launches = n;
    const cudaError_t e = cudaGetLastError();
    g_cuda_error = (int)e;
    return e == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA;
}

int check_common(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, int B, const uint8_t* codes,
                 const uint8_t* scales, const void* workspace) {
    if (dtype != FP4Q_IN_F32 && dtype != FP4Q_IN_BF16) return FP4Q_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols || cols % B) return FP4Q_ERR_SHAPE;
    if (rows > 0 && cols > 0 && rows > ((int64_t)1 << 40) / cols) return FP4Q_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP4Q_OK;
    if (!x || !codes || !scales || !workspace) return FP4Q_ERR_INVALID_ARG;
    const int es = dtype == FP4Q_IN_BF16 ? 2 : 4;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(workspace) || (ld * es) % 16) return FP4Q_ERR_ALIGNMENT;
    return FP4Q_OK;
}

// Batch context of a q16 launch: the next tensor whose amax the launch folds (null: none) and
// whether the status word is ORed (later tensors of a batch) rather than written.
struct BatchLink {
    const NextTensor<int64_t>* next = nullptr;
    int status_or = 0;
};

// The NVFP4 / IF4 kernel; 32-bit index arithmetic when the tensors allow it.
template <int IN, int KIND, bool HAD, typename IDX>
void launch_q16_as(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* imp, uint8_t* codes,
                   uint8_t* scales, float* gs, uint32_t* ws, int tiled, cudaStream_t st, BatchLink bl) {
    const int64_t total = rows * (cols / 16);
    if constexpr (q16_persistent<KIND>() && !HAD) {
        if (bl.next) {
            const NextTensor<int64_t>& n = *bl.next;
            const NextTensor<IDX> nx = {n.x, (IDX)n.rows, (IDX)n.cols, (IDX)n.ld, n.gs};
            const int64_t nvec = n.rows * (n.cols * (IN == FP4Q_IN_BF16 ? 2 : 4) / 16);
            auto kernel = q16_kernel<IN, KIND, HAD, IDX, true>;
            // two of the next tensor's vectors ride on each block: size the wave for the larger need
            const int grid = grid_for(kernel, total > nvec / 2 ? total : nvec / 2, q16_min_ctas<KIND>());
            kernel<<<grid, kThreads, 0, st>>>(x, (IDX)rows, (IDX)cols, (IDX)ld, imp, codes, scales, gs, ws, tiled, nx,
                                              bl.status_or);
            return;
        }
    }
    auto kernel = q16_kernel<IN, KIND, HAD, IDX, false>;
    const int grid = q16_persistent<KIND>() ? grid_for(kernel, total, q16_min_ctas<KIND>())
                                            : (int)((total + kThreads - 1) / kThreads);
    const NextTensor<IDX> none = {nullptr, 0, 0, 0, nullptr};
    kernel<<<grid, kThreads, 0, st>>>(x, (IDX)rows, (IDX)cols, (IDX)ld, imp, codes, scales, gs, ws, tiled, none,
                                      bl.status_or);
}

template <int IN, int KIND, bool HAD>
void launch_q16(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* imp, uint8_t* codes,
                uint8_t* scales, float* gs, uint32_t* ws, int tiled, cudaStream_t st, BatchLink bl) {
    const int64_t total = rows * (cols / 16);
    const bool small_next = !bl.next || bl.next->rows * bl.next->ld < ((int64_t)1 << 31);
    if (total < ((int64_t)1 << 31) && rows * ld < ((int64_t)1 << 31) && small_next)
        launch_q16_as<IN, KIND, HAD, uint32_t>(x, rows, cols, ld, imp, codes, scales, gs, ws, tiled, st, bl);
    else
        launch_q16_as<IN, KIND, HAD, int64_t>(x, rows, cols, ld, imp, codes, scales, gs, ws, tiled, st, bl);
}

// Tensor scale pass: plain amax, or the amax of the 16-point rotated blocks.
template <int IN>
void launch_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, uint32_t* ws, float* gs, int publish,
                 bool had16, cudaStream_t st, float div = 1536.0f) {
    if (had16) {
        amax_had16_kernel<IN><<<grid_for(amax_had16_kernel<IN>, rows * (cols / 16), 4), kThreads, 0, st>>>(
            x, rows, cols, ld, ws, gs, publish);
    } else {
        const int64_t vecs = rows * cols * (IN == FP4Q_IN_BF16 ? 2 : 4) / 16;
        amax_kernel<IN><<<grid_for(amax_kernel<IN>, vecs, 4), kThreads, 0, st>>>(x, rows, cols, ld, ws, gs, publish,
                                                                                  div);
    }
}

template <int IN, bool HAD>
void launch_nvfp4_if4(const void* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int obj, const float* imp,
                      uint8_t* codes, uint8_t* scales, float* gs, uint32_t* ws, uint32_t flags, cudaStream_t st,
                      BatchLink bl = BatchLink()) {
    const int tiled = (flags & FP4Q_F_SCALE_TILED) ? 1 : 0;
    if (fmt == FP4Q_IF4) {
        if (flags & FP4Q_F_IF4_SWEEP)
            launch_q16<IN, KIND_IF4_SWEEP, HAD>(x, rows, cols, ld, imp, codes, scales, gs, ws, tiled, st, bl);
        else
            launch_q16<IN, KIND_IF4, HAD>(x, rows, cols, ld, imp, codes, scales, gs, ws, tiled, st, bl);
        return;
    }
    switch (obj) {
        case FP4Q_ABSMAX:
            launch_q16<IN, FP4Q_ABSMAX, HAD>(x, rows, cols, ld, imp, codes, scales, gs, ws, tiled, st, bl);
            break;
        case FP4Q_FOUR_OVER_SIX:
            launch_q16<IN, FP4Q_FOUR_OVER_SIX, HAD>(x, rows, cols, ld, imp, codes, scales, gs, ws, tiled, st, bl);
            break;
        case FP4Q_SWEEP_MSE:
            launch_q16<IN, FP4Q_SWEEP_MSE, HAD>(x, rows, cols, ld, imp, codes, scales, gs, ws, tiled, st, bl);
            break;
        default:   // WMSE is rejected with the rotation before any launch
            if (!HAD) launch_q16<IN, FP4Q_SWEEP_WMSE, false>(x, rows, cols, ld, imp, codes, scales, gs, ws, tiled, st, bl);
            break;
    }
}

template <int IN>
int launch_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int obj, const float* imp,
                    uint8_t* codes, uint8_t* scales, float* gs, uint32_t* ws, uint32_t flags, cudaStream_t st) {
    if (fmt == FP4Q_MXFP4) {
        const int ocp = (flags & FP4Q_F_MX_OCP_FLOOR) ? 1 : 0;
        const bool had = (flags & FP4Q_F_HADAMARD32) != 0, sweep = (flags & FP4Q_F_MX_SWEEP) != 0;
        const int tiled = (flags & FP4Q_F_SCALE_TILED) ? 1 : 0;
        const int64_t nblk = rows * (cols / 32);
        if (had && sweep)
            mxfp4_kernel<IN, true, true><<<grid_for(mxfp4_kernel<IN, true, true>, nblk, 8), kThreads, 0, st>>>(
                x, rows, cols, ld, codes, scales, ws, ocp, tiled);
        else if (had)
            mxfp4_kernel<IN, true, false><<<grid_for(mxfp4_kernel<IN, true, false>, nblk, 8), kThreads, 0, st>>>(
                x, rows, cols, ld, codes, scales, ws, ocp, tiled);
        else if (sweep)
            mxfp4_kernel<IN, false, true><<<grid_for(mxfp4_kernel<IN, false, true>, nblk, 8), kThreads, 0, st>>>(
                x, rows, cols, ld, codes, scales, ws, ocp, tiled);
        else
            mxfp4_kernel<IN, false, false><<<grid_for(mxfp4_kernel<IN, false, false>, nblk, 8), kThreads, 0, st>>>(
                x, rows, cols, ld, codes, scales, ws, ocp, tiled);
        return launched(1);
    }
    if (fmt == FP4Q_IF6) {
        int n = 0;
        if (!(flags & FP4Q_F_GLOBAL_SCALE_GIVEN)) {
            launch_amax<IN>(x, rows, cols, ld, ws, gs, 0, false, st, 1920.0f);
            ++n;
        }
        if6_kernel<IN><<<grid_for(if6_kernel<IN>, rows * (cols / 16), 4), kThreads, 0, st>>>(x, rows, cols, ld, codes,
                                                                                         scales, gs, ws);
        return launched(n + 1);
    }
    const bool had16 = (flags & FP4Q_F_HADAMARD16) != 0;
    int n = 0;
    if (!(flags & FP4Q_F_GLOBAL_SCALE_GIVEN)) {
        launch_amax<IN>(x, rows, cols, ld, ws, gs, 0, had16, st);
        ++n;
    }
    if (had16) launch_nvfp4_if4<IN, true>(x, rows, cols, ld, fmt, obj, imp, codes, scales, gs, ws, flags, st);
    else launch_nvfp4_if4<IN, false>(x, rows, cols, ld, fmt, obj, imp, codes, scales, gs, ws, flags, st);
    return launched(n + 1);
}

// Scratch for fp4q_quantize_noalloc: the 64 bytes a quantize call keeps on the device
// (status word, amax word, arrival counters) live in this file-scope array instead of a
// caller-allocated workspace.  Every GPU that loads the library holds these 256 bytes until
// the process exits.  In host code the name is only a stand-in for the symbol; the device
// address comes from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) uint32_t g_noalloc_scratch[64];
constexpr size_t kNoAllocScratchBytes = sizeof(g_noalloc_scratch);
static_assert(kWorkspaceBytes <= kNoAllocScratchBytes, "no-alloc scratch smaller than a workspace");
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The first call on a device looks
// it up; later calls check that the cached address still belongs to device memory of this
// device (a cudaDeviceReset ends the context it lived in, and the next context maps the array
// afresh), and look it up again if not.
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP4Q_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FP4Q_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev]) {
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, g_noalloc_addr[dev]) != cudaSuccess || a.type != cudaMemoryTypeDevice ||
            a.device != dev) {
            (void)cudaGetLastError();   // the failed query leaves no error behind
            g_noalloc_addr[dev] = nullptr;
        }
    }
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FP4Q_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return FP4Q_OK;
}

template <bool OUT_BF16, bool IF4, bool HAD>
void launch_dequant16_as(const uint8_t* codes, const uint8_t* scales, const float* gs, int64_t rows, int64_t cols,
                         void* out, int tiled, cudaStream_t st) {
    auto k = dequant16_kernel<OUT_BF16, IF4, HAD>;
    k<<<grid_for(k, rows * (cols / 16), 8), kThreads, 0, st>>>(codes, scales, gs, rows, cols, out, tiled);
}

template <bool OUT_BF16, int FMT>
void launch_dequant_lin(const uint8_t* codes, const uint8_t* scales, const float* gs, int64_t rows, int64_t cols,
                        void* out, int tiled, cudaStream_t st) {
    auto k = dequant_lin_kernel<OUT_BF16, FMT>;
    k<<<grid_for(k, rows * (cols / 4), 8), kThreads, 0, st>>>(codes, scales, gs, rows, cols, out, tiled);
}

template <bool HAD>
void launch_dequant16(const uint8_t* codes, const uint8_t* scales, const float* gs, int64_t rows, int64_t cols,
                      bool if4, bool bf, void* out, int tiled, cudaStream_t st) {
    if (!HAD) {
        if (if4 && bf) launch_dequant_lin<true, FP4Q_IF4>(codes, scales, gs, rows, cols, out, tiled, st);
        else if (if4) launch_dequant_lin<false, FP4Q_IF4>(codes, scales, gs, rows, cols, out, tiled, st);
        else if (bf) launch_dequant_lin<true, FP4Q_NVFP4>(codes, scales, gs, rows, cols, out, tiled, st);
        else launch_dequant_lin<false, FP4Q_NVFP4>(codes, scales, gs, rows, cols, out, tiled, st);
        return;
    }
    if (if4 && bf) launch_dequant16_as<true, true, HAD>(codes, scales, gs, rows, cols, out, tiled, st);
    else if (if4) launch_dequant16_as<false, true, HAD>(codes, scales, gs, rows, cols, out, tiled, st);
    else if (bf) launch_dequant16_as<true, false, HAD>(codes, scales, gs, rows, cols, out, tiled, st);
    else launch_dequant16_as<false, false, HAD>(codes, scales, gs, rows, cols, out, tiled, st);
}

template <bool OUT_BF16, bool HAD>
void launch_dequant_mx(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, void* out, int tiled,
                       cudaStream_t st) {
    auto k = dequant_mx_kernel<OUT_BF16, HAD>;
    k<<<grid_for(k, rows * (cols / 32), 8), kThreads, 0, st>>>(codes, scales, rows, cols, out, tiled);
}

// Format, objective and flag checks shared by fp4q_quantize and fp4q_quantize_noalloc.
int check_quantize_args(int fmt, int objective, uint32_t flags) {
    if (fmt != FP4Q_NVFP4 && fmt != FP4Q_IF4 && fmt != FP4Q_MXFP4 && fmt != FP4Q_IF6) return FP4Q_ERR_INVALID_ARG;
    if (fmt == FP4Q_IF6 && (flags & ~(uint32_t)FP4Q_F_GLOBAL_SCALE_GIVEN)) return FP4Q_ERR_UNSUPPORTED;
    if (flags & ~(FP4Q_F_GLOBAL_SCALE_GIVEN | FP4Q_F_MX_OCP_FLOOR | FP4Q_F_HADAMARD16 | FP4Q_F_HADAMARD32 |
                  FP4Q_F_MX_SWEEP | FP4Q_F_IF4_SWEEP | FP4Q_F_SCALE_TILED))
        return FP4Q_ERR_INVALID_ARG;
    if ((flags & FP4Q_F_SCALE_TILED) && fmt == FP4Q_IF4) return FP4Q_ERR_UNSUPPORTED;
    if ((flags & FP4Q_F_IF4_SWEEP) && fmt != FP4Q_IF4) return FP4Q_ERR_UNSUPPORTED;
    if ((flags & FP4Q_F_MX_SWEEP) && (flags & FP4Q_F_MX_OCP_FLOOR)) return FP4Q_ERR_INVALID_ARG;
    if ((flags & FP4Q_F_MX_SWEEP) && fmt != FP4Q_MXFP4) return FP4Q_ERR_UNSUPPORTED;
    if (fmt == FP4Q_NVFP4 && (objective < FP4Q_ABSMAX || objective > FP4Q_SWEEP_WMSE)) return FP4Q_ERR_INVALID_ARG;
    if (fmt == FP4Q_MXFP4 && (flags & FP4Q_F_GLOBAL_SCALE_GIVEN)) return FP4Q_ERR_INVALID_ARG;
    if (flags & FP4Q_F_HADAMARD16) {
        if (fmt == FP4Q_MXFP4) return FP4Q_ERR_UNSUPPORTED;
        if (fmt == FP4Q_NVFP4 && objective == FP4Q_SWEEP_WMSE) return FP4Q_ERR_UNSUPPORTED;
    }
    if ((flags & FP4Q_F_HADAMARD32) && fmt != FP4Q_MXFP4) return FP4Q_ERR_UNSUPPORTED;
    return FP4Q_OK;
}

}  // namespace fp4q

using namespace fp4q;

extern "C" {

size_t fp4q_workspace_bytes(void) { return kWorkspaceBytes; }

int64_t fp4q_scale_bytes(int64_t rows, int64_t cols, int fmt, uint32_t flags) {
    if (fmt != FP4Q_NVFP4 && fmt != FP4Q_IF4 && fmt != FP4Q_MXFP4 && fmt != FP4Q_IF6) return -1;
    if (fmt == FP4Q_IF6 && (flags & FP4Q_F_SCALE_TILED)) return -1;
    const int64_t B = fmt == FP4Q_MXFP4 ? 32 : 16;
    if (rows < 0 || cols < 0 || cols % B) return -1;
    if (rows > 0 && cols > 0 && rows > ((int64_t)1 << 40) / cols) return -1;
    const int64_t J = cols / B;
    if (!(flags & FP4Q_F_SCALE_TILED)) return rows * J;
    return ((rows + 127) / 128) * 128 * ((J + 3) / 4) * 4;
}

int fp4q_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, int fmt, int objective,
                  const float* importance, uint8_t* codes, uint8_t* scales, float* global_scale, void* workspace,
                  uint32_t flags, void* stream) {
    g_launches = 0;
    int rc = check_quantize_args(fmt, objective, flags);
    if (rc != FP4Q_OK) return rc;
    const int B = fmt == FP4Q_MXFP4 ? 32 : 16;
    rc = check_common(x, dtype, rows, cols, ld, B, codes, scales, workspace);
    if (rc != FP4Q_OK || rows == 0 || cols == 0) return rc;
    if (fmt != FP4Q_MXFP4 && !global_scale) return FP4Q_ERR_INVALID_ARG;
    if (fmt == FP4Q_NVFP4 && objective == FP4Q_SWEEP_WMSE) {
        if (!importance) return FP4Q_ERR_INVALID_ARG;
        if (!aligned16(importance)) return FP4Q_ERR_ALIGNMENT;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* ws = reinterpret_cast<uint32_t*>(workspace);
    if (dtype == FP4Q_IN_BF16)
        return launch_quantize<FP4Q_IN_BF16>(x, rows, cols, ld, fmt, objective, importance, codes, scales, global_scale,
                                             ws, flags, st);
    return launch_quantize<FP4Q_IN_F32>(x, rows, cols, ld, fmt, objective, importance, codes, scales, global_scale, ws,
                                        flags, st);
}

}  // extern "C"

namespace fp4q {
// fp4q_quantize_batch: the non-empty tensors in order.  Without a given S, the first one's amax
// pass is its own kernel and every quantize kernel also folds the following tensor's amax
// (persistent kinds, no rotation); WMSE and the rotated forms run each tensor's amax pass as its
// own kernel.  The status word is cleared first and every quantize kernel ORs its flags into it.
template <int IN>
int batch_impl(const fp4q_tensor* t, const int* live, int m, int fmt, int obj, uint32_t* ws, uint32_t flags,
               cudaStream_t st) {
    if (cudaMemsetAsync(ws + WS_STATUS, 0, sizeof(uint32_t), st) != cudaSuccess) return launched(0);
    const bool given = (flags & FP4Q_F_GLOBAL_SCALE_GIVEN) != 0, had16 = (flags & FP4Q_F_HADAMARD16) != 0;
    const bool fused = !given && !had16 && !(fmt == FP4Q_NVFP4 && obj == FP4Q_SWEEP_WMSE);
    auto rides = [&](int k) { return fused && k > 0; };   // a tensor's amax rides on the previous kernel
    int n = 0;
    for (int k = 0; k < m; ++k) {
        const fp4q_tensor& a = t[live[k]];
        if (!given && !rides(k)) {
            launch_amax<IN>(a.x, a.rows, a.cols, a.ld, ws, a.global_scale, 0, had16, st);
            ++n;
        }
        NextTensor<int64_t> nx = {nullptr, 0, 0, 0, nullptr};
        BatchLink bl;
        bl.status_or = 1;
        if (k + 1 < m && rides(k + 1)) {
            const fp4q_tensor& b = t[live[k + 1]];
            nx = {b.x, b.rows, b.cols, b.ld, b.global_scale};
            bl.next = &nx;
        }
        if (had16)
            launch_nvfp4_if4<IN, true>(a.x, a.rows, a.cols, a.ld, fmt, obj, a.importance, a.codes, a.scales,
                                       a.global_scale, ws, flags, st, bl);
        else
            launch_nvfp4_if4<IN, false>(a.x, a.rows, a.cols, a.ld, fmt, obj, a.importance, a.codes, a.scales,
                                        a.global_scale, ws, flags, st, bl);
        ++n;
    }
    return launched(n);
}
}  // namespace fp4q

extern "C" {

int fp4q_quantize_batch(int n, const fp4q_tensor* tensors, int dtype, int fmt, int objective, void* workspace,
                        uint32_t flags, void* stream) {
    g_launches = 0;
    if (n < 0 || (n > 0 && !tensors)) return FP4Q_ERR_INVALID_ARG;
    int rc = check_quantize_args(fmt, objective, flags);
    if (rc != FP4Q_OK) return rc;
    if (fmt != FP4Q_NVFP4 && fmt != FP4Q_IF4) return FP4Q_ERR_UNSUPPORTED;
    std::vector<int> live;
    for (int i = 0; i < n; ++i) {
        const fp4q_tensor& a = tensors[i];
        rc = check_common(a.x, dtype, a.rows, a.cols, a.ld, 16, a.codes, a.scales, workspace);
        if (rc != FP4Q_OK) return rc;
        if (a.rows == 0 || a.cols == 0) continue;
        if (!a.global_scale) return FP4Q_ERR_INVALID_ARG;
        if (fmt == FP4Q_NVFP4 && objective == FP4Q_SWEEP_WMSE) {
            if (!a.importance) return FP4Q_ERR_INVALID_ARG;
            if (!aligned16(a.importance)) return FP4Q_ERR_ALIGNMENT;
        }
        live.push_back(i);
    }
    if (live.empty()) return FP4Q_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* ws = reinterpret_cast<uint32_t*>(workspace);
    if (dtype == FP4Q_IN_BF16)
        return batch_impl<FP4Q_IN_BF16>(tensors, live.data(), (int)live.size(), fmt, objective, ws, flags, st);
    return batch_impl<FP4Q_IN_F32>(tensors, live.data(), (int)live.size(), fmt, objective, ws, flags, st);
}

}  // extern "C"

namespace fp4q {
// fp4q_global_scale (plain, granule = 16 bytes of a row) and fp4q_hadamard_global_scale
// (rotated blocks, granule = 16 elements).
int global_scale_impl(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, bool had16,
                      float* global_scale, void* workspace, void* stream, float div = 1536.0f) {
    g_launches = 0;
    if (dtype != FP4Q_IN_F32 && dtype != FP4Q_IN_BF16) return FP4Q_ERR_INVALID_ARG;
    const int es = dtype == FP4Q_IN_BF16 ? 2 : 4;
    if (rows < 0 || cols < 0 || ld < cols || (cols * es) % 16 || (had16 && cols % 16)) return FP4Q_ERR_SHAPE;
    if (rows > 0 && cols > 0 && rows > ((int64_t)1 << 40) / cols) return FP4Q_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP4Q_OK;
    if (!x || !global_scale || !workspace) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(workspace) || (ld * es) % 16) return FP4Q_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* ws = reinterpret_cast<uint32_t*>(workspace);
    if (dtype == FP4Q_IN_BF16) launch_amax<FP4Q_IN_BF16>(x, rows, cols, ld, ws, global_scale, 1, had16, st, div);
    else launch_amax<FP4Q_IN_F32>(x, rows, cols, ld, ws, global_scale, 1, had16, st, div);
    return launched(1);
}
}  // namespace fp4q

extern "C" {

int fp4q_global_scale(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, float* global_scale,
                      void* workspace, void* stream) {
    return global_scale_impl(x, dtype, rows, cols, ld, false, global_scale, workspace, stream);
}

int fp4q_if6_global_scale(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, float* global_scale,
                          void* workspace, void* stream) {
    return global_scale_impl(x, dtype, rows, cols, ld, false, global_scale, workspace, stream, 1920.0f);
}

int fp4q_hadamard_global_scale(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, int had_size,
                               float* global_scale, void* workspace, void* stream) {
    g_launches = 0;
    if (had_size != 16) return FP4Q_ERR_UNSUPPORTED;
    return global_scale_impl(x, dtype, rows, cols, ld, true, global_scale, workspace, stream);
}

int fp4q_hadamard_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, int had_size,
                           uint8_t* codes, uint8_t* scales, void* workspace, uint32_t flags, void* stream) {
    g_launches = 0;
    if (had_size != 32) return FP4Q_ERR_UNSUPPORTED;
    if (flags & ~(FP4Q_F_MX_OCP_FLOOR | FP4Q_F_MX_SWEEP | FP4Q_F_SCALE_TILED)) return FP4Q_ERR_INVALID_ARG;
    return fp4q_quantize(x, dtype, rows, cols, ld, FP4Q_MXFP4, 0, nullptr, codes, scales, nullptr, workspace,
                         flags | FP4Q_F_HADAMARD32, stream);
}

int fp4q_dequantize(const uint8_t* codes, const uint8_t* scales, const float* global_scale, int64_t rows,
                    int64_t cols, int fmt, int inverse_hadamard, void* out, uint32_t flags, void* stream) {
    g_launches = 0;
    if (fmt != FP4Q_NVFP4 && fmt != FP4Q_IF4 && fmt != FP4Q_MXFP4 && fmt != FP4Q_IF6) return FP4Q_ERR_INVALID_ARG;
    if (fmt == FP4Q_IF6 && (inverse_hadamard || (flags & FP4Q_F_SCALE_TILED))) return FP4Q_ERR_UNSUPPORTED;
    if (flags & ~(FP4Q_F_OUT_BF16 | FP4Q_F_SCALE_TILED)) return FP4Q_ERR_INVALID_ARG;
    if ((flags & FP4Q_F_SCALE_TILED) && fmt == FP4Q_IF4) return FP4Q_ERR_UNSUPPORTED;
    const int tiled = (flags & FP4Q_F_SCALE_TILED) ? 1 : 0;
    const int B = fmt == FP4Q_MXFP4 ? 32 : 16;
    if (rows < 0 || cols < 0 || cols % B) return FP4Q_ERR_SHAPE;
    if (rows > 0 && cols > 0 && rows > ((int64_t)1 << 40) / cols) return FP4Q_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP4Q_OK;
    if (!codes || !scales || !out || (fmt != FP4Q_MXFP4 && !global_scale)) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(out)) return FP4Q_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = (flags & FP4Q_F_OUT_BF16) != 0;
    if (fmt == FP4Q_IF6) {
        if (reinterpret_cast<uintptr_t>(codes) & 3u) return FP4Q_ERR_ALIGNMENT;
        if (bf)
            dequant_if6_kernel<true><<<grid_for(dequant_if6_kernel<true>, rows * (cols / 16), 8), kThreads, 0, st>>>(
                codes, scales, global_scale, rows, cols, out);
        else
            dequant_if6_kernel<false><<<grid_for(dequant_if6_kernel<false>, rows * (cols / 16), 8), kThreads, 0, st>>>(
                codes, scales, global_scale, rows, cols, out);
        return launched(1);
    }
    if (fmt == FP4Q_MXFP4) {
        if (bf && inverse_hadamard) launch_dequant_mx<true, true>(codes, scales, rows, cols, out, tiled, st);
        else if (bf) launch_dequant_lin<true, FP4Q_MXFP4>(codes, scales, nullptr, rows, cols, out, tiled, st);
        else if (inverse_hadamard) launch_dequant_mx<false, true>(codes, scales, rows, cols, out, tiled, st);
        else launch_dequant_lin<false, FP4Q_MXFP4>(codes, scales, nullptr, rows, cols, out, tiled, st);
    } else if (inverse_hadamard) {
        launch_dequant16<true>(codes, scales, global_scale, rows, cols, fmt == FP4Q_IF4, bf, out, tiled, st);
    } else {
        launch_dequant16<false>(codes, scales, global_scale, rows, cols, fmt == FP4Q_IF4, bf, out, tiled, st);
    }
    return launched(1);
}

int fp4q_quantize_noalloc(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, int fmt,
                          int objective, const float* importance, uint8_t* codes, uint8_t* scales,
                          float* global_scale, uint32_t* device_status, uint32_t flags, void* stream) {
    g_launches = 0;
    // the same argument checks as fp4q_quantize, made before the scratch is touched
    const int rca = check_quantize_args(fmt, objective, flags);
    if (rca != FP4Q_OK) return rca;
    const int B = fmt == FP4Q_MXFP4 ? 32 : 16;
    const void* aligned_stand_in = reinterpret_cast<const void*>(static_cast<uintptr_t>(256));
    int rc0 = check_common(x, dtype, rows, cols, ld, B, codes, scales, aligned_stand_in);
    if (rc0 != FP4Q_OK) return rc0;
    if (device_status && (reinterpret_cast<uintptr_t>(device_status) & 3u)) return FP4Q_ERR_ALIGNMENT;
    if (rows == 0 || cols == 0) {   // nothing to quantize: the status word still reports this call
        if (device_status &&
            cudaMemsetAsync(device_status, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
            return FP4Q_ERR_CUDA;
        return FP4Q_OK;
    }
    if (fmt != FP4Q_MXFP4 && !global_scale) return FP4Q_ERR_INVALID_ARG;
    if (fmt == FP4Q_NVFP4 && objective == FP4Q_SWEEP_WMSE) {
        if (!importance) return FP4Q_ERR_INVALID_ARG;
        if (!aligned16(importance)) return FP4Q_ERR_ALIGNMENT;
    }
    void* scratch = nullptr;
    int rc = noalloc_scratch(&scratch);
    if (rc != FP4Q_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the previous call's words (and anything an interrupted call left) start from zero
    if (cudaMemsetAsync(scratch, 0, kWorkspaceBytes, st) != cudaSuccess) return FP4Q_ERR_CUDA;
    rc = fp4q_quantize(x, dtype, rows, cols, ld, fmt, objective, importance, codes, scales, global_scale, scratch,
                       flags, stream);
    if (rc == FP4Q_OK && device_status &&
        cudaMemcpyAsync(device_status, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    return rc;
}

int fp4q_quantize_host_async(const void* x_host, int dtype, int64_t rows, int64_t cols, int fmt, int objective,
                             const float* importance, uint8_t* codes_host, uint8_t* scales_host, float* S_host,
                             void* x_dev, uint8_t* codes_dev, uint8_t* scales_dev, float* S_dev, void* workspace,
                             uint32_t flags, void* copy_stream, void* compute_stream, void* staged_event,
                             void* free_event) {
    g_launches = 0;
    int rc = check_quantize_args(fmt, objective, flags);
    if (rc != FP4Q_OK) return rc;
    const int B = fmt == FP4Q_MXFP4 ? 32 : 16;
    rc = check_common(x_dev, dtype, rows, cols, cols, B, codes_dev, scales_dev, workspace);
    if (rc != FP4Q_OK || rows == 0 || cols == 0) return rc;
    if (!x_host || !codes_host || !scales_host || !staged_event || !free_event) return FP4Q_ERR_INVALID_ARG;
    if (fmt != FP4Q_MXFP4 && (!S_dev || !S_host)) return FP4Q_ERR_INVALID_ARG;
    if (fmt == FP4Q_NVFP4 && objective == FP4Q_SWEEP_WMSE) {
        if (!importance) return FP4Q_ERR_INVALID_ARG;
        if (!aligned16(importance)) return FP4Q_ERR_ALIGNMENT;
    }
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(copy_stream);
    cudaStream_t ks = reinterpret_cast<cudaStream_t>(compute_stream);
    cudaEvent_t staged = reinterpret_cast<cudaEvent_t>(staged_event);
    cudaEvent_t freed = reinterpret_cast<cudaEvent_t>(free_event);
    const size_t in_bytes = (size_t)rows * (size_t)cols * (dtype == FP4Q_IN_BF16 ? 2 : 4);
    // the staging input is overwritten only once the kernels of its previous use have read it
    if (cudaStreamWaitEvent(cs, freed, 0) != cudaSuccess) return FP4Q_ERR_CUDA;
    if (cudaMemcpyAsync(x_dev, x_host, in_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess) return FP4Q_ERR_CUDA;
    if (cudaEventRecord(staged, cs) != cudaSuccess || cudaStreamWaitEvent(ks, staged, 0) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    rc = fp4q_quantize(x_dev, dtype, rows, cols, cols, fmt, objective, importance, codes_dev, scales_dev,
                       fmt == FP4Q_MXFP4 ? nullptr : S_dev, workspace, flags, compute_stream);
    if (rc != FP4Q_OK) return rc;
    const int n = g_launches;
    if (cudaEventRecord(freed, ks) != cudaSuccess) return FP4Q_ERR_CUDA;
    const size_t code_bytes = (size_t)rows * (size_t)(fmt == FP4Q_IF6 ? cols * 3 / 4 : cols / 2);
    if (cudaMemcpyAsync(codes_host, codes_dev, code_bytes, cudaMemcpyDeviceToHost, ks) !=
            cudaSuccess ||
        cudaMemcpyAsync(scales_host, scales_dev, (size_t)rows * (size_t)(cols / B), cudaMemcpyDeviceToHost, ks) !=
            cudaSuccess)
        return FP4Q_ERR_CUDA;
    if (fmt != FP4Q_MXFP4 &&
        cudaMemcpyAsync(S_host, S_dev, sizeof(float), cudaMemcpyDeviceToHost, ks) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    g_launches = n;
    return FP4Q_OK;
}

int fp4q_encode(const float* x, int64_t n, int kind, uint8_t* out, void* stream) {
    g_launches = 0;
    if (kind != FP4Q_CODEC_E2M1 && kind != FP4Q_CODEC_E4M3) return FP4Q_ERR_INVALID_ARG;
    if (n < 0 || n > ((int64_t)1 << 40)) return FP4Q_ERR_SHAPE;
    if (n == 0) return FP4Q_OK;
    if (!x || !out) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(out) & 3u)) return FP4Q_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t items = n / 4 > 0 ? n / 4 : 1;
    if (kind == FP4Q_CODEC_E2M1)
        encode_kernel<0><<<grid_for(encode_kernel<0>, items, 8), kThreads, 0, st>>>(x, n, out);
    else
        encode_kernel<1><<<grid_for(encode_kernel<1>, items, 8), kThreads, 0, st>>>(x, n, out);
    return launched(1);
}

int fp4q_read_device_status(const void* workspace, uint32_t* status, void* stream) {
    if (!workspace || !status) return FP4Q_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(status, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA;
}

int fp4q_last_launch_count(void) { return g_launches; }

int fp4q_last_cuda_error(void) { return g_cuda_error; }

const char* fp4q_status_string(int s) {
    switch (s) {
        case FP4Q_OK: return "ok";
        case FP4Q_ERR_INVALID_ARG: return "invalid argument";
        case FP4Q_ERR_SHAPE: return "invalid shape";
        case FP4Q_ERR_ALIGNMENT: return "misaligned pointer or row pitch (16 bytes required)";
        case FP4Q_ERR_UNSUPPORTED: return "unsupported combination";
        case FP4Q_ERR_CUDA: return "CUDA launch or runtime error";
        default: return "unknown status";
    }
}

}  // extern "C"
