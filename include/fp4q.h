/*
 * fp4q.h -- C ABI of libfp4q: block-scaled FP4 quantization on NVIDIA B200 (sm_100a), and the
 * block-scaled NVFP4 / MXFP4 GEMMs (tcgen05 tensor cores) that consume the quantized operands.
 *
 * Formats and methods (each entry point cites the passage that defines what it computes):
 *   NVFP4  16-element blocks of E2M1 codes {0,.5,1,1.5,2,3,4,6} with one E4M3 scale per
 *          block and one FP32 scale S per tensor.  S = max|x| / (256*6) and the ScaleSweep
 *          search over E4M3 bit-pattern offsets [-3,+7] (MSE) or [-8,+7] (WMSE):
 *          ScaleSweep (gist.science/ko/paper/2606.07618), "Methodology".  AbsMax is the
 *          base scale itself; 4/6 (max->6 or max->4, lower MSE): Adaptive Block-Scaled Data
 *          Types (gist.science/ko/paper/2603.28765), "Problem".
 *   IF4    NVFP4 layout; per block the lower-MSE of FP4 and scaled INT4 (x 7/6 before
 *          rounding, x 6/7 on dequantization), flagged in the scale byte's sign bit
 *          (1 = INT4): Adaptive Block-Scaled Data Types, "Methodology", IF4 structure.
 *   MXFP4  32-element blocks of E2M1 codes with an E8M0 (power-of-two) scale, optionally
 *          after a normalized 32-point block Hadamard rotation: Bridging the Gap ...
 *          Microscaling FP4 (gist.science/ko/paper/2509.23202), "Methodology"; scale rule
 *          "block maximum onto the largest codeword": TORQ (gist.science/ko/paper/
 *          2605.19561), "Method", S-step.
 *   IF6    16-element blocks of 6-bit codes, per block the lower-MSE of FP6 (E2M3, largest
 *          value 7.5) and scaled INT6 ([-31, 31], x 62/15 before rounding, x 15/62 on
 *          dequantization), indicator in the scale byte's sign bit (1 = INT6): the IF4
 *          construction at 6 bits, Adaptive Block-Scaled Data Types, "Methodology"
 *          (extensibility to 6-bit types).
 *
 * Arithmetic (identical on every path).  RN is one binary32 operation rounded to nearest even,
 * with no contraction and no flush-to-zero:
 *   S = RN(amax/1536) (IF6: RN(amax/1920)); p0 = E4M3_RNE(RN(a_b / RN(6 S))) (IF6: RN(7.5 S));
 *   p4 = E4M3_RNE(RN(a_b / RN(4 S))) (4/6 only).
 *   candidate pattern p: sv = RN(e(p) S), inv = RN(1/sv) (sv = inv = 0 for p = 0);
 *   codes: y = RN(x inv), q = E2M1_RNE_satfinite(y); the reconstruction is q sv (exact).
 *   MSE objectives (4/6, the sweep, IF4, IF6, the IF4 sweep, the MX sweep): the block error
 *   E = sum_i (x_i - xhat_i)^2 of the exact reconstructions, compared EXACTLY (the library
 *   decides it in integer and binary64 arithmetic with no rounding in the comparison); the
 *   lowest offset wins a tie (4/6: the max->6 scale; IF4, IF6: FP first; the IF4 sweep: lowest
 *   offset, then FP4; the MX sweep: the lowest exponent).  ScaleSweep, "Methodology": the
 *   objective is the block's reconstruction error.
 *   WMSE (importance-weighted): binary32, one accumulator per candidate in element order:
 *   xhat = RN(q sv), d = RN(x - xhat), acc = fma(RN(w d), d, acc); the lowest (acc, offset)
 *   wins; NaN never wins; if every acc is +inf the first candidate is kept.
 *   IF4 INT4: n = clamp(rint(RN(y RN(7/6))), -7, 7), reconstruction n g with g = RN(RN(6/7) sv)
 *   (the INT4 block's own binary32 scale); INT4 iff its exact error is lower.
 *   IF4 x ScaleSweep (flag FP4Q_F_IF4_SWEEP): every MSE-window candidate p0-3 .. p0+7 under both
 *   types, exact errors; the lowest (error, offset, type) wins with FP4 before INT4.  Adaptive
 *   Block-Scaled Data Types, "Methodology" (IF4 type choice) searched jointly with ScaleSweep,
 *   "Methodology".
 *   IF6: FP6 codes E2M3_RNE_satfinite(y), reconstruction q sv; INT6 codes
 *   n = clamp(rint(RN(y RN(62/15))), -31, 31), reconstruction n RN(RN(15/62) sv).
 *   MXFP4: e = smallest integer with a_b <= 6 * 2^e (flag FP4Q_F_MX_OCP_FLOOR: floor(log2
 *   a_b) - 2), clamped to [-127,127]; y = RN(x 2^-e), reconstruction q 2^e.
 *   MX scale sweep (flag FP4Q_F_MX_SWEEP): e among e_c - 2 .. e_c (e_c the ceil rule, none
 *   below -127) with the lowest exact block error.  Bridging the Gap ... Microscaling FP4,
 *   "Methodology": MXFP4 "Scale Fitting" of the power-of-two grid to the data, read as
 *   ScaleSweep's block-MSE search over E8M0 neighbours; exponents above e_c can only tie (the
 *   grid at 2^(e_c+1) below 6*2^e_c is a subset of the grid at 2^e_c).
 *
 * Memory layout (all device memory, row-major, owned and allocated by the caller):
 *   x        [rows][ld] bf16 or fp32; ld >= cols elements; x and the row pitch (ld * element
 *            size) 16-byte aligned.
 *   codes    [rows][cols/2] bytes; element 2k in the low nibble of byte k, 2k+1 in the high
 *            nibble; nibble = sign << 3 | E2M1 magnitude index (IF4 INT4 blocks: 4-bit two's
 *            complement of n).  16-byte aligned; cols/2 bytes per row, no padding.
 *            IF6: [rows][cols*3/4] bytes, 12 per block, element i of a block in bits
 *            6i .. 6i+5 of the block's little-endian 96-bit field (FP6: sign << 5 | E2M3
 *            magnitude bits; INT6: 6-bit two's complement of n).
 *   scales   [rows][cols/B] bytes, B = 16 (NVFP4/IF4/IF6: E4M3 pattern, IF4/IF6 indicator in
 *            bit 7) or 32 (MXFP4: E8M0 byte e+127, 0xFF marks a block with a non-finite input).
 *   global_scale  one float (NVFP4/IF4/IF6): written with S, or read when
 *            FP4Q_F_GLOBAL_SCALE_GIVEN is set.
 *   workspace fp4q_workspace_bytes() bytes, 16-byte aligned, ZERO-FILLED ONCE by the caller
 *            before its first use; every call leaves it zeroed again except word 0.  Word 0
 *            (uint32) receives the device status (FP4Q_DEVSTAT_*) of the most recent call that
 *            used it.  One workspace must not be shared by calls that may run concurrently.
 *
 * Errors: argument, shape and alignment problems are detected on the host before anything
 * is launched and returned as fp4q_status; a failed launch returns FP4Q_ERR_CUDA.  Data
 * conditions (a non-finite input, or a tensor scale S outside [2^-117, 2^125/1536]) are found
 * on the device: the outputs of that call are zero-filled and the device status word is
 * set; no call synchronizes the host, and no kernel traps.  Calls are asynchronous on
 * `stream` (a cudaStream_t; NULL = the legacy default stream).
 */
#ifndef FP4Q_H
#define FP4Q_H

#include <stddef.h>
#include <stdint.h>

/* Exported entry points (the library is built with hidden visibility: nothing else is exported,
 * so two builds of it loaded into one process keep their internal state apart). */
#if defined(__GNUC__)
#define FP4Q_API __attribute__((visibility("default")))
#else
#define FP4Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP4Q_OK = 0,
    FP4Q_ERR_INVALID_ARG = 1,   /* null pointer, unknown enum value, bad flag combination */
    FP4Q_ERR_SHAPE = 2,         /* rows/cols/ld out of range or cols not a multiple of B    */
    FP4Q_ERR_ALIGNMENT = 3,     /* a pointer or the row pitch is not 16-byte aligned        */
    FP4Q_ERR_UNSUPPORTED = 4,   /* combination the library does not implement                */
    FP4Q_ERR_CUDA = 5           /* a CUDA launch or runtime call failed                      */
} fp4q_status;

/* Device status bits.  TIMEOUT: fp4q_nvfp4_gemm / fp4q_mxfp4_gemm gave up a bounded wait for
 * its tensor-core work (its output is then incomplete). */
enum { FP4Q_DEVSTAT_OK = 0, FP4Q_DEVSTAT_NONFINITE = 1, FP4Q_DEVSTAT_RANGE = 2, FP4Q_DEVSTAT_TIMEOUT = 4 };
enum { FP4Q_IN_F32 = 0, FP4Q_IN_BF16 = 1 };
enum { FP4Q_NVFP4 = 0, FP4Q_IF4 = 1, FP4Q_MXFP4 = 2, FP4Q_IF6 = 3 };
enum { FP4Q_ABSMAX = 0, FP4Q_FOUR_OVER_SIX = 1, FP4Q_SWEEP_MSE = 2, FP4Q_SWEEP_WMSE = 3 };

#define FP4Q_F_GLOBAL_SCALE_GIVEN 0x1u  /* quantize: read S from *global_scale (no amax pass) */
#define FP4Q_F_MX_OCP_FLOOR       0x2u  /* MXFP4: e = floor(log2 a_b) - 2 instead of the ceil rule */
#define FP4Q_F_OUT_BF16           0x4u  /* dequantize: write bf16 (RNE of the fp32 value)     */
#define FP4Q_F_HADAMARD16         0x8u  /* NVFP4/IF4 quantize: rotate every 16-element block by
                                           H_16/4 first (see fp4q_hadamard_global_scale)      */
#define FP4Q_F_HADAMARD32         0x10u /* MXFP4 quantize: rotate every 32-element block first,
                                           as fp4q_hadamard_quantize does                     */
#define FP4Q_F_MX_SWEEP           0x20u /* MXFP4 quantize (fp4q_quantize, fp4q_hadamard_quantize):
                                           MX scale sweep -- each block's exponent is the one
                                           among e_c-2 .. e_c (e_c = the ceil rule) with the
                                           lowest block error; not with FP4Q_F_MX_OCP_FLOOR    */
#define FP4Q_F_SCALE_TILED        0x80u /* NVFP4/MXFP4 quantize and dequantize: scale bytes in the
                                           128x4-tiled layout of block-scaled tensor-core GEMMs
                                           (see fp4q_scale_bytes) instead of row-major         */
#define FP4Q_F_IF4_SWEEP          0x40u /* IF4 quantize: IF4 x ScaleSweep -- the block scale and
                                           the element type are chosen together over the MSE
                                           window p0-3 .. p0+7 (see the arithmetic above)      */

/* Size in bytes of the workspace every quantize call needs (a small constant). */
FP4Q_API size_t fp4q_workspace_bytes(void);

/*
 * Size in bytes of the scales buffer of a rows x cols tensor in format fmt: rows * cols/B
 * row-major, or with FP4Q_F_SCALE_TILED in flags the tiled layout that block-scaled tensor-core
 * GEMMs (the consumer of these codes and scales on B200) read: the [rows][cols/B] scale matrix
 * padded to whole tiles of 128 rows x 4 scale columns (512 bytes each), tiles row-major over
 * (row/128, col/4), and inside a tile the scale of row r, column c at byte
 * 16*(r%32) + 4*((r/32)%4) + c%4.  A quantize call writes only the entries of real blocks; the
 * padding keeps whatever the caller put there (zero it if the consumer reads it).  The pages
 * give no scale layout; this one is the public layout of NVIDIA's block-scaled GEMMs
 * (cuBLASLt's "32x4x4" scale-factor tiles), kept byte for byte so that a GEMM can read the
 * scales as written (fp4q_nvfp4_gemm and fp4q_mxfp4_gemm do).  IF4 has no tiled form (its indicator bit is not a consumer format).
 * Returns -1 for an unknown format or a bad shape.
 */
FP4Q_API int64_t fp4q_scale_bytes(int64_t rows, int64_t cols, int fmt, uint32_t flags);

/*
 * Quantize x into codes + scales (+ S).
 *   fmt FP4Q_NVFP4 with objective FP4Q_ABSMAX / FP4Q_FOUR_OVER_SIX / FP4Q_SWEEP_MSE /
 *   FP4Q_SWEEP_WMSE (importance: device float[cols], one non-negative finite weight per
 *   column, required for WMSE and ignored otherwise); fmt FP4Q_IF4 (objective ignored);
 *   fmt FP4Q_MXFP4 (objective, importance and global_scale ignored; see also
 *   fp4q_hadamard_quantize).
 *   rows >= 0, cols a multiple of 16 (32 for MXFP4), ld >= cols; rows*cols < 2^40.
 *   flags: FP4Q_F_GLOBAL_SCALE_GIVEN (NVFP4/IF4), FP4Q_F_MX_OCP_FLOOR (MXFP4),
 *   FP4Q_F_HADAMARD16 (NVFP4 with ABSMAX / FOUR_OVER_SIX / SWEEP_MSE, and IF4),
 *   FP4Q_F_HADAMARD32 (MXFP4 only, else FP4Q_ERR_UNSUPPORTED; identical to
 *   fp4q_hadamard_quantize), FP4Q_F_MX_SWEEP (MXFP4 only, else FP4Q_ERR_UNSUPPORTED;
 *   with FP4Q_F_MX_OCP_FLOOR: FP4Q_ERR_INVALID_ARG), FP4Q_F_IF4_SWEEP (IF4 only, else
 *   FP4Q_ERR_UNSUPPORTED; combines with FP4Q_F_HADAMARD16 and FP4Q_F_GLOBAL_SCALE_GIVEN),
 *   FP4Q_F_SCALE_TILED (NVFP4 and MXFP4: scales in the tiled layout of fp4q_scale_bytes; IF4:
 *   FP4Q_ERR_UNSUPPORTED).  fmt FP4Q_IF6 (objective ignored) takes FP4Q_F_GLOBAL_SCALE_GIVEN
 *   only (S = RN(amax/1920) otherwise); every other flag returns FP4Q_ERR_UNSUPPORTED.
 * FP4Q_F_HADAMARD16: every 16-element block is first rotated by the normalized Sylvester
 *   Hadamard matrix H_16 / 4 (butterflies h = 1, 2, 4, 8 in binary32, then one exact
 *   multiplication by 1/4 per value), and the whole method -- S, the block scales, the
 *   scale search and the codes -- runs on the rotated values, so S = RN(max|H x| / 1536).
 *   Bridging the Gap ... Microscaling FP4 (gist.science/ko/paper/2509.23202),
 *   "Methodology", block-wise Hadamard transforms, which rotates NVFP4 as well as MXFP4.
 *   A given S (FP4Q_F_GLOBAL_SCALE_GIVEN) must then be the rotated tensor's, e.g. from
 *   fp4q_hadamard_global_scale.  SWEEP_WMSE with the flag returns FP4Q_ERR_UNSUPPORTED (a
 *   per-column importance has no meaning once the columns of a block are mixed), and so
 *   does MXFP4 (use fp4q_hadamard_quantize).  Dequantize with inverse_hadamard = 1.
 * Launches: NVFP4/IF4 without a given S: an amax kernel then the quantize kernel;
 * otherwise one kernel.  Empty tensors launch nothing.
 */
FP4Q_API int fp4q_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                  int fmt, int objective, const float* importance,
                  uint8_t* codes, uint8_t* scales, float* global_scale,
                  void* workspace, uint32_t flags, void* stream);

/*
 * Tensor scale only: S = RN(max|x| / 1536) written to *global_scale (device float), the
 * ScaleSweep global scale S = max|x|/(256*6) (ScaleSweep, gist.science/ko/paper/2606.07618,
 * "Methodology").  A non-finite element gives S = NaN.  The workspace status word receives
 * FP4Q_DEVSTAT_NONFINITE (S = NaN) or FP4Q_DEVSTAT_RANGE (S outside [2^-117, 2^125/1536]).
 * Passing the result to fp4q_quantize with FP4Q_F_GLOBAL_SCALE_GIVEN performs exactly the
 * work of a call without the flag.  cols * element size must be a multiple of 16 bytes.
 */
FP4Q_API int fp4q_global_scale(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                      float* global_scale, void* workspace, void* stream);

/*
 * One tensor of a batch (fp4q_quantize_batch).  Members as the fp4q_quantize arguments of the
 * same names: x [rows][ld] (device, bf16 or fp32 as the batch's dtype), codes, scales,
 * global_scale (device; written with S, or read under FP4Q_F_GLOBAL_SCALE_GIVEN) and, for
 * SWEEP_WMSE only, importance (device float[cols], else NULL).  Caller-owned.
 */
typedef struct fp4q_tensor {
    const void* x;
    int64_t rows, cols, ld;
    const float* importance;
    uint8_t* codes;
    uint8_t* scales;
    float* global_scale;
} fp4q_tensor;

/*
 * NVFP4 or IF4 quantization of n tensors in order, with the results of n fp4q_quantize calls
 * (same dtype, fmt, objective and flags; every tensor gets its own S = RN(amax/1536) from its
 * own elements, ScaleSweep, "Methodology"): codes, scale bytes and S bit for bit identical.
 * A sequence of tensors (the layers of a model, a stream of activations) leaves the HBM-bound
 * amax pass and the arithmetic-bound search of each tensor side by side: here the quantize
 * kernel of tensor i also reads tensor i+1 and writes its S, so that read overlaps the search
 * instead of running as a pass of its own.
 *   tensors    host array of n descriptors (read during the call only); empty tensors are
 *              skipped.  The inputs must not overlap any output of the batch.
 *   workspace  as fp4q_quantize; word 0 receives the OR of the tensors' device statuses (a
 *              batch of only empty tensors leaves it unchanged).
 *   flags      as fp4q_quantize.
 * Launches (NVFP4 AbsMax, 4/6 and sweep-MSE, IF4 and the IF4 sweep, no rotation, S not given):
 * one amax kernel for the first non-empty tensor, then one quantize kernel per tensor, m + 1
 * for m non-empty tensors.  With FP4Q_F_GLOBAL_SCALE_GIVEN: m quantize kernels.  SWEEP_WMSE and
 * FP4Q_F_HADAMARD16 keep the amax pass as its own kernel per tensor (2m).  MXFP4 and IF6:
 * FP4Q_ERR_UNSUPPORTED.  Errors: as fp4q_quantize, for every tensor, before anything runs.
 */
FP4Q_API int fp4q_quantize_batch(int n, const fp4q_tensor* tensors, int dtype, int fmt, int objective,
                        void* workspace, uint32_t flags, void* stream);

/*
 * IF6's tensor scale: S = RN(max|x| / 1920) (7.5, the FP6 maximum, in place of FP4's 6; Adaptive
 * Block-Scaled Data Types, "Methodology", the IF4 construction at 6 bits).  Status, workspace,
 * shapes and errors as fp4q_global_scale; passing the result to fp4q_quantize(FP4Q_IF6) with
 * FP4Q_F_GLOBAL_SCALE_GIVEN performs exactly the work of a call without the flag.  Use: a
 * row-sharded tensor reduces the per-shard S values by maximum.
 */
FP4Q_API int fp4q_if6_global_scale(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                          float* global_scale, void* workspace, void* stream);

/*
 * Tensor scale of the block-rotated tensor: S = RN(max|H x| / 1536), H x being every
 * 16-element block of every row rotated by H_16 / 4 exactly as fp4q_quantize does under
 * FP4Q_F_HADAMARD16 (so this S with FP4Q_F_GLOBAL_SCALE_GIVEN | FP4Q_F_HADAMARD16
 * reproduces a call without the first flag).  had_size must be 16 (else
 * FP4Q_ERR_UNSUPPORTED); cols a multiple of 16.  A non-finite element, or a rotation that
 * overflows, gives S = NaN.  Status, workspace and errors as fp4q_global_scale.  Use: a
 * row-sharded tensor reduces the per-shard S values by maximum.
 */
FP4Q_API int fp4q_hadamard_global_scale(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                               int had_size, float* global_scale, void* workspace, void* stream);

/*
 * MXFP4 quantization of H x: each 32-element block (along the contiguous dimension) is
 * rotated by the normalized Sylvester Hadamard matrix H_32 / sqrt(32) before the E8M0 scale
 * and the E2M1 codes are chosen (Bridging the Gap ... Microscaling FP4, "Methodology",
 * block-wise Hadamard transforms).  had_size must be 32.  The transform is computed as the
 * fast Walsh-Hadamard butterflies h = 1, 2, 4, 8, 16 followed by one multiplication by
 * RN(1/sqrt(32)).  Same layout, alignment and error rules as fp4q_quantize with
 * fmt = FP4Q_MXFP4.  Dequantized values are in the rotated domain.  flags: 0,
 * FP4Q_F_MX_OCP_FLOOR or FP4Q_F_MX_SWEEP (the MX scale sweep on the rotated blocks).
 */
FP4Q_API int fp4q_hadamard_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                           int had_size, uint8_t* codes, uint8_t* scales,
                           void* workspace, uint32_t flags, void* stream);

/*
 * Quantize a tensor that lives in host memory: copy it in, quantize, copy codes, scales
 * (and S) out, all enqueued asynchronously; the call returns before any of it completes.
 * The pages have no counterpart; this is the end-to-end form of fp4q_quantize for callers
 * whose tensors arrive in host memory, built so that consecutive calls overlap.
 *   x_host [rows][cols] (contiguous, bf16 or fp32), codes_host [rows][cols/2],
 *   scales_host [rows][cols/B], S_host [1] (NVFP4/IF4; may be NULL for MXFP4): host
 *   memory, page-locked (cudaHostAlloc / pinned) for the copies to be asynchronous.
 *   x_dev, codes_dev, scales_dev, S_dev, workspace: one caller-owned device staging set
 *   (same sizes, contiguous; alignment and zeroed workspace as fp4q_quantize).
 *   fmt, objective, importance (device), flags: as fp4q_quantize (S_dev is read, not
 *   written, under FP4Q_F_GLOBAL_SCALE_GIVEN).
 *   copy_stream: carries the host-to-device copy; compute_stream: the kernels and the
 *   device-to-host copies (cudaStream_t; they may be equal, which serialises them).
 *   staged_event, free_event: two cudaEvent_t owned by the staging set (created by the
 *   caller, timing disabled is fine).  The call records staged_event on copy_stream after
 *   the input copy and makes compute_stream wait for it; it records free_event on
 *   compute_stream after the kernels and, on its next use with the same set, makes
 *   copy_stream wait for it before overwriting x_dev.  free_event must have been recorded
 *   once (e.g. on compute_stream) before the set's first use.
 * With two staging sets used alternately, the input copy of one call runs while the
 * previous call's kernels and output copies run, so a stream of calls is bound by the
 * host-to-device bandwidth instead of the sum of both copies.  The host output buffers of
 * a call may be read once compute_stream has passed the call (synchronize or record an
 * event after it).  Errors as fp4q_quantize; the device status lands in the set's
 * workspace.  Launch count as fp4q_quantize (copies are not counted).
 */
FP4Q_API int fp4q_quantize_host_async(const void* x_host, int dtype, int64_t rows, int64_t cols,
                             int fmt, int objective, const float* importance,
                             uint8_t* codes_host, uint8_t* scales_host, float* S_host,
                             void* x_dev, uint8_t* codes_dev, uint8_t* scales_dev, float* S_dev,
                             void* workspace, uint32_t flags, void* copy_stream,
                             void* compute_stream, void* staged_event, void* free_event);

/*
 * Dequantize codes + scales (+ S for NVFP4/IF4) into out [rows][cols], fp32 or (flag
 * FP4Q_F_OUT_BF16) bf16.  NVFP4: RN(q * RN(e(p) S)); IF4 blocks with bit 7 set:
 * RN(n * RN(RN(6/7) * RN(e(p) S))) (the INT4 block scale with the 6/7 dequantization folded
 * in); MXFP4: RN(q * 2^(byte-127)) (byte 0xFF gives NaN); IF6 (codes as fp4q_quantize writes
 * them): RN(q * RN(e(p) S)) for FP6 blocks, RN(n * RN(RN(15/62) * RN(e(p) S))) for INT6 blocks
 * (no inverse_hadamard, no tiled scales).  Each value is the binary32 rounding of the
 * reconstruction the quantizer's objective measures.
 * inverse_hadamard: apply the normalized transform of the format's block size (32-point for
 * MXFP4, 16-point H_16 / 4 for NVFP4/IF4) to each dequantized block, as butterflies then
 * one multiplication per value (it is its own inverse up to rounding).  global_scale is a device
 * pointer (ignored for MXFP4).  out must be 16-byte aligned.  flags: FP4Q_F_OUT_BF16 and
 * FP4Q_F_SCALE_TILED (scales in the tiled layout of fp4q_scale_bytes; NVFP4 and MXFP4).
 */
FP4Q_API int fp4q_dequantize(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                    int64_t rows, int64_t cols, int fmt, int inverse_hadamard,
                    void* out, uint32_t flags, void* stream);

/*
 * fp4q_quantize for callers that cannot allocate device memory.  The pages have no
 * counterpart; this is a deployment convenience.  Some callers run where the allocator is
 * off limits: code inside another framework's stream capture or memory pool, a plugin that
 * gets only the tensors it works on, or an inference engine that plans every allocation
 * ahead of time.  They cannot hand over the zeroed workspace fp4q_quantize wants.  This
 * entry point keeps that scratch (64 bytes: status word, amax word, arrival counters) in a
 * 256-byte array compiled into the library, one per GPU, held until the process exits.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 *   Arguments and results are those of fp4q_quantize, minus `workspace`.  device_status is
 *   an optional device uint32 (4-byte aligned, may be NULL); it receives the call's
 *   FP4Q_DEVSTAT_* word, copied asynchronously on `stream` (FP4Q_DEVSTAT_OK for an empty
 *   tensor, written by a 4-byte memset on `stream`).
 *   The scratch need does not grow with the tensor, so every shape fp4q_quantize accepts
 *   fits; larger tensors (2^40 elements and up) are rejected with FP4Q_ERR_SHAPE as there.
 *   The first call on a device looks up the array's address (cudaGetSymbolAddress) with
 *   that device current.  Make that first call before any stream capture.  Later calls check
 *   the remembered address (cudaPointerGetAttributes) and look it up again after a
 *   cudaDeviceReset of that device, whose new context maps the array afresh.
 *   Every call clears the scratch on `stream` before using it, and all calls on a device
 *   share it: calls that may run at the same time on the GPU (different streams, different
 *   host threads) race and must be serialized by the caller.
 */
FP4Q_API int fp4q_quantize_noalloc(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                          int fmt, int objective, const float* importance,
                          uint8_t* codes, uint8_t* scales, float* global_scale,
                          uint32_t* device_status, uint32_t flags, void* stream);

/*
 * Element codec: the hardware conversions every quantize path uses, applied to n fp32 values.
 *   kind FP4Q_CODEC_E2M1: out[i] = E2M1 code of x[i], round to nearest with ties to the even
 *     code, saturating at +-6, sign kept (-0 -> 0x8): the low nibble holds sign << 3 | index of
 *     the magnitude in {0, .5, 1, 1.5, 2, 3, 4, 6} (ScaleSweep, gist.science/ko/paper/2606.07618,
 *     Contributions: round-to-nearest FP4 codes).
 *   kind FP4Q_CODEC_E4M3: out[i] = E4M3FN byte of x[i], round to nearest even, saturating at
 *     +-448 (the 126 positive finite values the ScaleSweep page counts, Methodology).
 * x: device fp32 [n], 16-byte aligned; out: device uint8 [n], 4-byte aligned.  One launch.
 * Errors: FP4Q_ERR_INVALID_ARG (unknown kind, NULL), FP4Q_ERR_SHAPE (n < 0 or n > 2^40),
 * FP4Q_ERR_ALIGNMENT.  NaN inputs give whatever the hardware conversion gives.
 */
enum { FP4Q_CODEC_E2M1 = 0, FP4Q_CODEC_E4M3 = 1 };
FP4Q_API int fp4q_encode(const float* x, int64_t n, int kind, uint8_t* out, void* stream);

/* Copy the device status word of `workspace` to *status (blocks until `stream` is done). */
FP4Q_API int fp4q_read_device_status(const void* workspace, uint32_t* status, void* stream);

/* Number of kernel launches the most recent successful call on this thread issued. */
FP4Q_API int fp4q_last_launch_count(void);

/* The cudaError_t value behind the most recent FP4Q_ERR_CUDA on this thread from a launching call
 * (0 after a successful launch; -1 when the GEMM's tensor-map encoder refused its operands). */
FP4Q_API int fp4q_last_cuda_error(void);

/* Static description of a status code. */
FP4Q_API const char* fp4q_status_string(int status);

/*
 * Block-scaled NVFP4 GEMM on the B200 tensor cores (tcgen05), the consumer of two quantized
 * operands: d[m][n] = S_a * S_b * sum_k A[m][k] * B[n][k] in fp32, where A (M x K) and B (N x K)
 * are NVFP4 tensors exactly as fp4q_quantize writes them with FP4Q_F_SCALE_TILED:
 *   a_codes [M][K/2], b_codes [N][K/2] (K contiguous, element 2j in the low nibble),
 *   a_scales, b_scales: E4M3 scale bytes in the tiled layout of fp4q_scale_bytes,
 *   a_global_scale, b_global_scale: device pointers to the two tensor scales S.
 * Every product of two element values q_a e_a * q_b e_b is formed exactly by the tensor core
 * and accumulated in fp32; the result is multiplied by RN(S_a S_b) once.  The pages give no
 * GEMM: this is the step after the quantizer (Bridging the Gap ... Microscaling FP4,
 * "Methodology", the FP4 GEMM kernels whose operands the quantizer produces).
 * d: fp32 [M][ldd], ldd >= N, ldd a multiple of 4; all pointers device memory, 16-byte
 * aligned.  M and N multiples of 128, K a multiple of 256 (FP4Q_ERR_SHAPE otherwise).
 * workspace: fp4q_workspace_bytes() bytes; its word 0 receives the device status
 * (FP4Q_DEVSTAT_TIMEOUT if a bounded wait for the tensor cores ran out; the kernel then lets its
 * tensor-core operations and armed copies finish, each again with a bounded wait, frees its
 * tensor memory and returns, so the context stays usable).  One launch.
 */
FP4Q_API int fp4q_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global_scale,
                    const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global_scale,
                    int64_t M, int64_t N, int64_t K, float* d, int64_t ldd, void* workspace,
                    void* stream);

/*
 * The same GEMM for two MXFP4 operands: d[m][n] = sum_k A[m][k] * B[n][k] in fp32, where
 * A and B are MXFP4 tensors as fp4q_quantize or fp4q_hadamard_quantize writes them with
 * FP4Q_F_SCALE_TILED (E8M0 scale bytes, one per 32 elements, in the tiled layout of
 * fp4q_scale_bytes); MXFP4 has no tensor scale.  When both operands were rotated with the
 * same 32-point block Hadamard along K, the rotations cancel in the product (the normalized
 * transform is orthogonal), so d approximates the product of the unrotated tensors (Bridging
 * the Gap ... Microscaling FP4, "Methodology": rotations folded into the adjacent weights).
 * Shapes, alignment, layout of d, workspace and errors as for fp4q_nvfp4_gemm.
 */
FP4Q_API int fp4q_mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                    const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, float* d, int64_t ldd,
                    void* workspace, void* stream);

/*
 * Either GEMM with a choice of output type: fmt FP4Q_NVFP4 (arguments as fp4q_nvfp4_gemm) or
 * FP4Q_MXFP4 (as fp4q_mxfp4_gemm; the global-scale pointers are ignored).  d is fp32 [M][ldd]
 * (ldd a multiple of 4) or, with flags = FP4Q_F_OUT_BF16, bf16 [M][ldd] (ldd a multiple of 8):
 * the fp32 value RN(acc * RN(S_a S_b)) rounded to the nearest bf16, ties to even.  The pages
 * leave the consumer's output type open; bf16 is the usual activation type of the layer after
 * the GEMM and halves the bytes D takes.  Errors: FP4Q_ERR_INVALID_ARG (unknown format or flag),
 * FP4Q_ERR_UNSUPPORTED (FP4Q_IF4: its indicator bit is not a tensor-core operand format), and
 * those of fp4q_nvfp4_gemm.
 */
FP4Q_API int fp4q_gemm(int fmt, const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global_scale,
              const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global_scale,
              int64_t M, int64_t N, int64_t K, void* d, int64_t ldd, uint32_t flags,
              void* workspace, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FP4Q_H */
