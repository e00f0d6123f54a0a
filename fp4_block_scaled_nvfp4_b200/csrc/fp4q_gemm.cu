// fp4q_gemm.cu -- block-scaled FP4 GEMMs on the sm_100a tensor cores (tcgen05), the consumer
// of the quantizer's outputs: D[m][n] = S_a S_b sum_k A[m][k] B[n][k] for NVFP4 operands, and
// D[m][n] = sum_k A[m][k] B[n][k] for MXFP4 operands, with A and B stored exactly as
// fp4q_quantize writes them (codes [rows][K/2], element 2j in the low nibble; scales in the
// 128x4-tiled layout of FP4Q_F_SCALE_TILED; NVFP4: one fp32 tensor scale each).  Both operands
// have K contiguous.
//
// Per K stage of 256 elements the A and B tiles (128-byte rows) sit in shared memory in the
// 128-byte-swizzled K-major layout the MMA descriptors describe, and the operands' 512-byte
// scale-factor atoms as they are; one thread moves the atoms into tensor memory (tcgen05.cp
// 32x128b, broadcast to the four lane quarters) and issues four block-scaled MMAs of K = 64
// (tcgen05.mma kind::mxf4nvf4, 16-element E4M3 or 32-element E8M0 scale blocks) accumulating
// fp32 in tensor memory; the epilogue reads the accumulator back with tcgen05.ld (each warp
// its lane quarter), multiplies by RN(S_a S_b) (NVFP4) and stores D.
//   fp4_gemm_kernel<MX, OUT_BF16>: one CTA per SM over 128 x 256 output tiles, a four-stage
//     ring filled by tensor copies, producer / MMA / epilogue warps, two overlapping
//     accumulators so the epilogue of a tile overlaps the next tile's MMAs; D in fp32 or bf16.
// Every wait is bounded; one that runs out sets FP4Q_DEVSTAT_TIMEOUT in the status word and
// stops the CTA's loops.  Before the CTA frees its tensor memory and leaves, the MMA thread waits
// (bounded) for its tensor-core operations to finish and the producer for the copies it armed.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fp4q.h"

// Failure-path test build only (compiled into a separate library by the test suite's build):
// the MMA thread treats its first wait as timed out, before any copy has landed or any MMA has
// been issued, so that the bounded exit path runs; never set in the product library.
#ifndef FP4Q_GEMM_FAIL_FIRST_WAIT
#define FP4Q_GEMM_FAIL_FIRST_WAIT 0
#endif

namespace fp4q {

extern thread_local int g_launches;
extern thread_local int g_cuda_error;

namespace gemm {

constexpr int kTM = 128, kTN = 128, kTK = 256;     // M tile, narrow N tile, K per stage
constexpr int kTileBytes = kTM * kTK / 2;          // 16 KB of A codes per stage
constexpr int kSfBytes = 4 * 512;                  // four 128x4 scale atoms per operand and stage
constexpr uint32_t kWaitPolls = 1u << 22;          // bounded mbarrier wait

// Shared-memory matrix descriptor (sm_100 tensor-core operand): start address, leading and
// stride byte offsets in 16-byte units, descriptor version 1, and the layout type in bits
// 61..63 (0 = no swizzle, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46) | ((uint64_t)layout << 61);
}

// Instruction descriptor of the block-scaled FP4 MMA: E2M1 A and B (format 1), K-major
// operands, N / 8 in bits 17..22, UE4M3 scale factors (bit 23 = 0), M / 16 in bits 24..28,
// dense K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kTN >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        uint32_t done;
        asm volatile(
            "{ .reg .pred p;\n"
            "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            "  selp.u32 %0, 1, 0, p; }"
            : "=r"(done) : "r"(bar), "r"(parity) : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------------------------------
// Pipelined, persistent form (the one fp4q_nvfp4_gemm launches).  Output tiles are 128 x 256
// (the last tile of a row of tiles is 128 x 128 when N is an odd multiple of 128): per K stage
// of 256 elements one MMA of N = 256 (or 128) per K = 64 reads the A tile (128 rows) and the
// B tile (256 rows), so every byte brought into shared memory feeds twice the products of a
// 128 x 128 tile.  The operands sit in a ring of kPStages stages filled by the tensor-memory-
// access engine (A and B tiles as 2-D tensor copies written 128-byte-swizzled by the copy
// engine, B rows past N read as zeros; scale atoms as 2048-byte bulk copies), completing on the
// stage's "full" mbarrier, and released by the MMAs' commit to the stage's "empty" mbarrier.
// One CTA per SM walks the tiles t = blockIdx.x, + gridDim.x, ... (row-major over (m tile,
// n tile)).  192 threads, six warps:
//   warp 0 lane 0 -- producer over the (tile, K stage) sequence;
//   warp 1 lane 0 -- MMA issuer: copies each stage's scale atoms into tensor memory and issues
//     the four MMAs, then commits "acc_full" per tile;
//   warps 2..5 -- epilogue: per tile wait "acc_full", read the accumulator (each warp the lane
//     quarter warp % 4, as tensor memory requires), scale by S_a S_b and store.
// Tensor memory (512 columns): two accumulators of 256 columns cannot both fit beside the
// scale factors, so they overlap: tile j accumulates at column 0 (j even) or 192 (j odd), and
// the 64 columns [192, 256) are shared.  The epilogue of each tile reads its shared 64 columns
// first and then arrives on "acc_free"; the MMAs of the next tile start on that arrival and
// overlap the rest of the epilogue.  Scale factors: A at column 448 (4 per K = 64), B at 464
// (8 per K = 64: B rows 32 c .. 32 c + 31 in column c).
// ------------------------------------------------------------------------------------------
constexpr int kBN = 256;                                   // tile N
constexpr int kPStages = 4;
constexpr int kBTileBytes = kBN * kTK / 2;                 // 32 KB of B codes per stage
constexpr int kPStageBytes = kTileBytes + kBTileBytes + 3 * kSfBytes;   // 54 KB per ring stage
constexpr int kPThreads = 192;
constexpr uint32_t kPTmemCols = 512;
constexpr uint32_t kAcc1 = 192;                            // first column of the odd tiles' accumulator
constexpr uint32_t kPColSFA = 448, kPColSFB = 464;
constexpr int kPersistSmem = kPStages * kPStageBytes + 1024 + 256;   // ring, alignment, barriers
constexpr uint32_t kIdescN256 = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);

// MX = false: NVFP4 operands (E4M3 factor per 16 elements, tensor scales S_a, S_b); MX = true:
// MXFP4 operands (E8M0 factor per 32 elements, no tensor scale).  An MXFP4 scale atom covers
// K = 128 (four 32-element blocks per row), so a stage holds two atoms per 128 rows instead of
// four, and each K = 64 MMA reads two of a 32-bit column's four factor bytes: the byte offset
// (0 or 2) goes into the tensor-memory address's top bits and the instruction descriptor's
// factor-id fields.
template <bool MX, bool OUT_BF16>
__global__ void __launch_bounds__(kPThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                                 const uint8_t* __restrict__ sfa, const float* __restrict__ sa,
                                 const uint8_t* __restrict__ sfb, const float* __restrict__ sb, int K, int m_tiles,
                                 int n_tiles, int n_last_wide, void* __restrict__ dv, int64_t ldd,
                                 uint32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPStages * kPStageBytes);
    uint64_t* empty = full + kPStages;
    uint64_t* acc_full = empty + kPStages;
    uint64_t* acc_free = acc_full + 1;
    uint64_t* drained = acc_free + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
    __shared__ volatile int s_fail;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kAtoms = MX ? 2 : 4;                     // scale atoms per 128 rows and stage
    constexpr uint32_t kSfCopy = kAtoms * 512;
    const int64_t jt = K / (MX ? 128 : 64);                // scale atoms per 128 rows
    const int KT = K / kTK;
    const int tiles = m_tiles * n_tiles;
    // the last tile of each row of tiles is 128 wide unless N is a multiple of 256
    auto wide_tile = [&](int nt) { return nt + 1 < n_tiles || n_last_wide; };

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tmem_slot)), "r"(kPTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        s_fail = 0;
        for (int i = 0; i < kPStages; ++i) {
            mbar_init(smem_u32(full + i), 1);
            mbar_init(smem_u32(empty + i), 1);
        }
        mbar_init(smem_u32(acc_full), 1);
        mbar_init(smem_u32(acc_free), 4);   // one arrival per epilogue warp
        mbar_init(smem_u32(drained), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tma_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tma_b)) : "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    uint32_t issued = 0;   // stages the producer has armed (thread 0)

    if (tid == 0) {
        // producer
        uint32_t& g = issued;
        for (int t = blockIdx.x; t < tiles && !s_fail; t += gridDim.x) {
            const int mt = t / n_tiles, nt = t - mt * n_tiles;
            const bool wide = wide_tile(nt);
            // a tensor copy's transaction count is its whole box, rows past N included
            const uint32_t bytes = (uint32_t)(kTileBytes + kBTileBytes) + (wide ? 3u : 2u) * kSfCopy;
            for (int kt = 0; kt < KT; ++kt, ++g) {
                const uint32_t s = g % kPStages, round = g / kPStages;
                if (!mbar_wait(smem_u32(empty + s), (round & 1u) ^ 1u)) { s_fail = 1; break; }
                uint8_t* st = smem + s * kPStageBytes;
                const uint32_t fb = smem_u32(full + s);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(fb), "r"(bytes) : "memory");
                const int x = kt * (kTK / 2);
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                    :: "r"(smem_u32(st)), "l"(reinterpret_cast<uint64_t>(&tma_a)), "r"(x), "r"(mt * kTM), "r"(fb)
                    : "memory");
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                    :: "r"(smem_u32(st + kTileBytes)), "l"(reinterpret_cast<uint64_t>(&tma_b)), "r"(x), "r"(nt * kBN),
                       "r"(fb)
                    : "memory");
                uint8_t* ssf = st + kTileBytes + kBTileBytes;
                const uint8_t* gsa = sfa + ((int64_t)mt * jt + kAtoms * kt) * 512;
                const uint8_t* gsb = sfb + ((int64_t)(2 * nt) * jt + kAtoms * kt) * 512;
                asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                             :: "r"(smem_u32(ssf)), "l"(gsa), "r"(kSfCopy), "r"(fb) : "memory");
                asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                             :: "r"(smem_u32(ssf + kSfBytes)), "l"(gsb), "r"(kSfCopy), "r"(fb) : "memory");
                if (wide)
                    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                                 :: "r"(smem_u32(ssf + 2 * kSfBytes)), "l"(gsb + jt * 512), "r"(kSfCopy), "r"(fb)
                                 : "memory");
            }
        }
    } else if (tid == 32) {
        // MMA issuer
        uint32_t g = 0;
        int j = 0;
        for (int t = blockIdx.x; t < tiles && !s_fail; t += gridDim.x, ++j) {
            const int nt = t % n_tiles;
            const bool wide = wide_tile(nt);
            const uint32_t idesc = (wide ? kIdescN256 : kIdesc) | (MX ? (1u << 23) : 0u);   // E8M0 factors
            // the previous tile's epilogue has read the columns this accumulator shares with it
            if (j > 0 && !mbar_wait(smem_u32(acc_free), (uint32_t)((j - 1) & 1))) { s_fail = 1; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t tacc = tmem + ((j & 1) ? kAcc1 : 0u);
            for (int kt = 0; kt < KT; ++kt, ++g) {
                const uint32_t s = g % kPStages, round = g / kPStages;
                if ((FP4Q_GEMM_FAIL_FIRST_WAIT && g == 0) || !mbar_wait(smem_u32(full + s), round & 1u)) {
                    s_fail = 1;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                uint8_t* st = smem + s * kPStageBytes;
                uint8_t* ssf = st + kTileBytes + kBTileBytes;
#pragma unroll
                for (int kk = 0; kk < kAtoms; ++kk) {
                    const uint64_t da = smem_desc(smem_u32(ssf + kk * 512), 16, 128, 0);
                    const uint64_t db0 = smem_desc(smem_u32(ssf + kSfBytes + kk * 512), 16, 128, 0);
                    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                 :: "r"(tmem + kPColSFA + 4 * kk), "l"(da) : "memory");
                    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                 :: "r"(tmem + kPColSFB + 8 * kk), "l"(db0) : "memory");
                    if (wide) {
                        const uint64_t db1 = smem_desc(smem_u32(ssf + 2 * kSfBytes + kk * 512), 16, 128, 0);
                        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                     :: "r"(tmem + kPColSFB + 8 * kk + 4), "l"(db1) : "memory");
                    }
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t adesc = smem_desc(smem_u32(st + kk * 32), 16, 1024, 2);
                    const uint64_t bdesc = smem_desc(smem_u32(st + kTileBytes + kk * 32), 16, 1024, 2);
                    const uint32_t accumulate = (kt > 0 || kk > 0) ? 1u : 0u;
                    if constexpr (MX) {
                        const uint32_t id = (uint32_t)(kk & 1) * 2u;   // factor bytes 2 kk % 4 .. + 1
                        const uint32_t sfa_t = (tmem + kPColSFA + 4 * (kk >> 1)) | (id << 30);
                        const uint32_t sfb_t = (tmem + kPColSFB + 8 * (kk >> 1)) | (id << 30);
                        asm volatile(
                            "{ .reg .pred p;\n"
                            "  setp.ne.b32 p, %4, 0;\n"
                            "  tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p; }"
                            :: "r"(tacc), "l"(adesc), "l"(bdesc), "r"(idesc | (id << 29) | (id << 4)), "r"(accumulate),
                               "r"(sfa_t), "r"(sfb_t)
                            : "memory");
                    } else {
                        asm volatile(
                            "{ .reg .pred p;\n"
                            "  setp.ne.b32 p, %4, 0;\n"
                            "  tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p; }"
                            :: "r"(tacc), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate),
                               "r"(tmem + kPColSFA + 4 * kk), "r"(tmem + kPColSFB + 8 * kk)
                            : "memory");
                    }
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                             :: "r"(smem_u32(empty + s)) : "memory");
            }
            // the accumulator is complete once every MMA above has finished (also after a failure,
            // so that the epilogue's wait ends)
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         :: "r"(smem_u32(acc_full)) : "memory");
        }
    } else if (warp >= 2) {
        // epilogue: this warp owns tensor-memory lanes 32 (warp % 4) .. + 31
        const int q = warp & 3;
        const float scale = MX ? 1.0f : __fmul_rn(*sa, *sb);
        int j = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
            // warp-uniform decisions: the tensor-memory loads below are warp-collective
            const int ok = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(acc_full), (uint32_t)(j & 1)) ? 1 : 0);
            const int failed = __shfl_sync(0xFFFFFFFFu, s_fail, 0);
            if (!ok || failed) {
                s_fail = 1;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const int mt = t / n_tiles, nt = t - mt * n_tiles;
            const bool odd = (j & 1) != 0;
            const int nchunks = wide_tile(nt) ? kBN / 32 : kTN / 32;
            // chunks (of 32 columns) shared with the other accumulator are read first: the last
            // two of an even tile's 256 columns, the first two of an odd tile's
            const int first = (!odd && nchunks == 8) ? 6 : 0;
            const int shared_chunks = odd ? 2 : (nchunks == 8 ? 2 : 0);
            const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (odd ? kAcc1 : 0u);
            const int64_t drow = ((int64_t)mt * kTM + q * 32 + lane) * ldd + (int64_t)nt * kBN;
            for (int i = 0; i <= nchunks; ++i) {
                if (i == shared_chunks) {
                    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(acc_free)) : "memory");
                }
                if (i == nchunks) break;
                const int c = (first + i) % nchunks;
                uint32_t v[32];
                tmem_ld32(tbase + (uint32_t)(c * 32), v);
                if constexpr (OUT_BF16) {   // RN(RN(acc * scale)) to bf16, nearest even
                    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(dv) + drow + c * 32);
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint32_t w[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const __nv_bfloat162 p = __floats2bfloat162_rn(
                                __fmul_rn(__uint_as_float(v[e + 2 * h]), scale),
                                __fmul_rn(__uint_as_float(v[e + 2 * h + 1]), scale));
                            w[h] = *reinterpret_cast<const uint32_t*>(&p);
                        }
                        dst[e / 8] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else {
                    float* drp = reinterpret_cast<float*>(dv) + drow + c * 32;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(drp + e) = make_float4(
                            __fmul_rn(__uint_as_float(v[e]), scale), __fmul_rn(__uint_as_float(v[e + 1]), scale),
                            __fmul_rn(__uint_as_float(v[e + 2]), scale), __fmul_rn(__uint_as_float(v[e + 3]), scale));
                }
            }
        }
    }
    __syncwarp();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (s_fail) {
        if (tid == 32) {
            // a wait gave up: the MMA thread's tensor-core operations (MMAs and scale copies into
            // tensor memory) finish before the memory they use is freed; the commit arrives once
            // all of them have (the wait is again bounded)
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         :: "r"(smem_u32(drained)) : "memory");
            mbar_wait(smem_u32(drained), 0u);
        }
        if (tid == 0) {
            atomicOr(status, (uint32_t)FP4Q_DEVSTAT_TIMEOUT);
            // the copies the producer armed land in this CTA's shared memory before it leaves (the
            // last stage armed in each ring slot; each wait is again bounded)
            for (uint32_t i = 0; i < (uint32_t)kPStages && i < issued; ++i) {
                const uint32_t gi = issued - 1 - i;
                mbar_wait(smem_u32(full + gi % kPStages), (gi / kPStages) & 1u);
            }
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    }
    __syncwarp();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kPTmemCols) : "memory");
}

}  // namespace gemm
}  // namespace fp4q

namespace fp4q {
namespace gemm {

// The kernel's dynamic shared-memory limit, raised once per kernel and device (the attribute
// belongs to the current device's context); one bit per device ordinal below 64.
template <auto kernel>
bool smem_attribute_set(int bytes) {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
    if (bit && (done.load(std::memory_order_relaxed) & bit)) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    done.fetch_or(bit, std::memory_order_relaxed);
    return true;
}

// Shared host path of the two entry points: argument checks, tensor maps, launch.
template <bool MX, bool OUT_BF16>
int launch(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global_scale, const uint8_t* b_codes,
           const uint8_t* b_scales, const float* b_global_scale, int64_t M, int64_t N, int64_t K, void* d, int64_t ldd,
           void* workspace, void* stream) {
    g_launches = 0;
    g_cuda_error = 0;
    // a CUDA call that fails leaves its code for fp4q_last_cuda_error
    auto cuda_failed = [](cudaError_t e) {
        g_cuda_error = (int)e;
        return e != cudaSuccess;
    };
    if (M < 0 || N < 0 || K < 0 || M % kTM || N % kTN || K % kTK || ldd < N) return FP4Q_ERR_SHAPE;
    if (M / kTM > 65535 || K > (1 << 30)) return FP4Q_ERR_SHAPE;
    if (M == 0 || N == 0 || K == 0) return FP4Q_OK;
    if (!a_codes || !a_scales || !b_codes || !b_scales || !d || !workspace) return FP4Q_ERR_INVALID_ARG;
    if (!MX && (!a_global_scale || !b_global_scale)) return FP4Q_ERR_INVALID_ARG;
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!al16(a_codes) || !al16(a_scales) || !al16(b_codes) || !al16(b_scales) || !al16(d) || !al16(workspace) ||
        ldd % (OUT_BF16 ? 8 : 4))
        return FP4Q_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* status = reinterpret_cast<uint32_t*>(workspace);
    if (cuda_failed(cudaMemsetAsync(status, 0, sizeof(uint32_t), st))) return FP4Q_ERR_CUDA;
    // the tensor-copy descriptors of A and B: [rows][K/2] bytes, 128-byte-wide boxes of 128 (A) or
    // 256 (B) rows, 128-byte swizzle
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cuda_failed(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q)) ||
            q != cudaDriverEntryPointSuccess || !fn)
            return FP4Q_ERR_CUDA;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (!smem_attribute_set<fp4_gemm_kernel<MX, OUT_BF16>>(kPersistSmem)) {
        g_cuda_error = (int)cudaGetLastError();
        return FP4Q_ERR_CUDA;
    }
    CUtensorMap ta, tb;
    auto make = [&](CUtensorMap* m, const uint8_t* base, int64_t rows, int box_rows) {
        const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
        const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
        const cuuint32_t box[2] = {(cuuint32_t)(kTK / 2), (cuuint32_t)box_rows};
        const cuuint32_t estr[2] = {1, 1};
        return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    if (!make(&ta, a_codes, M, kTM) || !make(&tb, b_codes, N, kBN)) {
        g_cuda_error = -1;   // the tensor-map encoder refused the operands
        return FP4Q_ERR_CUDA;
    }
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return FP4Q_ERR_CUDA;
    }
    const int m_tiles = (int)(M / kTM), n_tiles = (int)((N + kBN - 1) / kBN);
    const int tiles = m_tiles * n_tiles;
    fp4_gemm_kernel<MX, OUT_BF16><<<tiles < sms ? tiles : sms, kPThreads, kPersistSmem, st>>>(
        ta, tb, a_scales, a_global_scale, b_scales, b_global_scale, (int)K, m_tiles, n_tiles, (int)(N % kBN == 0), d,
        ldd, status);
    if (cuda_failed(cudaGetLastError())) return FP4Q_ERR_CUDA;
    g_launches = 1;
    return FP4Q_OK;
}

}  // namespace gemm
}  // namespace fp4q

extern "C" int fp4q_gemm(int fmt, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global_scale,
                         const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global_scale, int64_t M,
                         int64_t N, int64_t K, void* d, int64_t ldd, uint32_t flags, void* workspace, void* stream) {
    fp4q::g_launches = 0;
    if (flags & ~(uint32_t)FP4Q_F_OUT_BF16) return FP4Q_ERR_INVALID_ARG;
    const bool bf = (flags & FP4Q_F_OUT_BF16) != 0;
    if (fmt == FP4Q_NVFP4)
        return bf ? fp4q::gemm::launch<false, true>(a_codes, a_scales, a_global_scale, b_codes, b_scales, b_global_scale,
                                                    M, N, K, d, ldd, workspace, stream)
                  : fp4q::gemm::launch<false, false>(a_codes, a_scales, a_global_scale, b_codes, b_scales,
                                                     b_global_scale, M, N, K, d, ldd, workspace, stream);
    if (fmt == FP4Q_MXFP4)
        return bf ? fp4q::gemm::launch<true, true>(a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, M, N, K, d,
                                                   ldd, workspace, stream)
                  : fp4q::gemm::launch<true, false>(a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, M, N, K, d,
                                                    ldd, workspace, stream);
    return fmt == FP4Q_IF4 ? FP4Q_ERR_UNSUPPORTED : FP4Q_ERR_INVALID_ARG;
}

extern "C" int fp4q_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global_scale,
                               const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global_scale,
                               int64_t M, int64_t N, int64_t K, float* d, int64_t ldd, void* workspace,
                               void* stream) {
    return fp4q_gemm(FP4Q_NVFP4, a_codes, a_scales, a_global_scale, b_codes, b_scales, b_global_scale, M, N, K, d, ldd,
                     0, workspace, stream);
}

extern "C" int fp4q_mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                               const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, float* d, int64_t ldd,
                               void* workspace, void* stream) {
    return fp4q_gemm(FP4Q_MXFP4, a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, M, N, K, d, ldd, 0, workspace,
                     stream);
}
