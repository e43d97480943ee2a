/*
 * bsp.h — C ABI of libbsp.so: block-scaled GEMM D = A * B^T on one B200 (sm_100a).
 *
 * Operations (the DeepGEMM-style calls the pages list):
 *   - dense GEMM in BF16, FP8 and FP4, and an M-grouped GEMM for mixture-of-experts
 *     layers ("DeepGEMM-Ascend cobre quantas operações no Ascend 950?", section
 *     "Cobertura de operações e a lacuna declarada no repositório"; "DeepSeek lanza
 *     kernels de DeepGEMM para Huawei Ascend 950", section "Qué incluye el lanzamiento");
 *   - the UE8M0 scale-factor layout transform: each pair of UE8M0 factors along K in
 *     one 16-bit integer, stored MN-major ("DeepSeek lanza kernels de DeepGEMM para
 *     Huawei Ascend 950", section "Qué incluye el lanzamiento"; "DeepGEMM-Ascend cobre
 *     quantas operações no Ascend 950?", section "Fatores de escala FP8 e o formato
 *     UE8M0 no Ascend");
 *   - the masked grouped GEMM the pages list as missing, and the FP8 quantiser that
 *     produces the GEMM's operands with their scales already in the packed layout.
 *
 * Conventions shared by every call
 *   - "NT": A is M x K row-major (K contiguous), B is N x K row-major, D is M x N
 *     row-major bf16.  Leading dimensions (lda, ldb, ldd, ld_sf*) are in ELEMENTS of
 *     the stored type (bytes for FP8 and for packed FP4, 2-byte units for bf16/int16).
 *   - Every pointer is a DEVICE pointer owned by the caller; the library never frees
 *     or retains caller memory.  Work is enqueued asynchronously on `stream` (a
 *     cudaStream_t passed as void*; NULL = legacy default stream) on the current device.
 *     Stream order holds as for any kernel: a call's kernels start reading and writing
 *     memory only after the work enqueued before them on `stream` has completed.  (The
 *     scaled GEMMs, the scale transform and the scale-layout pass are launched with
 *     programmatic stream serialisation, so their launch and set-up may overlap the kernel
 *     before them; each waits for it before touching memory.)
 *   - Argument errors are returned synchronously and nothing is launched.  Launch
 *     failures return BSP_ERR_CUDA.  Faults found while the kernels run (a wait that
 *     timed out, a malformed scale or expert index) are latched in a per-device status
 *     word and reported by bsp_get_device_status().
 *   - Alignment: base pointers 16-byte aligned; lda/ldb/ldd/ld_sf* times the element
 *     size a multiple of 16 bytes (the tensor-memory-accelerator copy rule).
 *   - M and N may take any positive value (rows and columns past them are neither
 *     read as data nor written); K has the per-call rule stated below.
 *   - The GEMM calls take their own scratch (the scale layout for the tensor cores, the
 *     partial sums of a split last wave) stream-ordered from a pool the library keeps per
 *     device, and free it on the same stream.  These calls can be captured in a CUDA
 *     graph; under capture the scratch becomes a graph memory node.
 *   - Results are deterministic: the same inputs give the same bytes on every run.
 *
 * Packed scale-factor layout ("SF words"): for a matrix with MN scale rows and KB scale
 * blocks along K, the SF tensor is int16 [ceil(KB/2)][ld], with
 *     word(j, r) = sf[j*ld + r] = e[r][2j] | e[r][2j+1] << 8
 * where e are biased UE8M0 bytes (scale = 2^(e-127)), the lower K block in the low
 * byte (a reading: the pages give no byte order).  ld >= MN; entries r >= MN and the
 * high byte of the last word when KB is odd are 0.
 */
#ifndef BSP_H
#define BSP_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BSP_OK = 0,
    BSP_ERR_ARG = -1,          /* null pointer, negative size, bad enum value */
    BSP_ERR_ALIGN = -2,        /* pointer or leading dimension breaks the 16-byte rule */
    BSP_ERR_SHAPE = -3,        /* K (or M_total) breaks its multiple-of rule, ld too small */
    BSP_ERR_UNSUPPORTED = -4,  /* no B200 (sm_100) device current, or size out of range */
    BSP_ERR_CUDA = -5,         /* a CUDA runtime/driver call failed */
    BSP_ERR_TIMEOUT = -6,      /* device: a pipeline wait gave up (latched) */
    BSP_ERR_DEVICE_CHECK = -7  /* device: bad scale value or expert index seen (latched) */
} bsp_status;

/*
 * gemm_bf16_nt — D[m,n] = bf16( sum_k A[m,k] * B[n,k] ), fp32 accumulation.
 *   A  bf16 [M][lda], B bf16 [N][ldb], D bf16 [M][ldd].
 *   K: any positive multiple of 8 (so that rows stay 16-byte aligned).
 */
int gemm_bf16_nt(const void* A, const void* B, void* D, int M, int N, int K,
                 int64_t lda, int64_t ldb, int64_t ldd, void* stream);

/*
 * gemm_fp8_nt — FP8 E4M3 GEMM with fine-grained UE8M0 scales along K
 * ("DeepGEMM-Ascend cobre quantas operações no Ascend 950?", section "Fatores de
 * escala FP8 e o formato UE8M0 no Ascend"):
 *   D[m,n] = bf16( sum_kb 2^(ea[m,kb]-127) * 2^(eb[n/g,kb]-127)
 *                  * sum_{k in block kb} A[m,k] * B[n,k] ),  blocks of 128 along K.
 *   A   E4M3 bytes [M][lda];  B  E4M3 bytes [N][ldb];  D bf16 [M][ldd].
 *   sfa SF words for MN = M rows, KB = K/128:            int16 [ceil(KB/2)][ld_sfa].
 *   sfb SF words for MN = ceil(N/g) rows, g = sfb_gran_n: int16 [ceil(KB/2)][ld_sfb].
 *       sfb_gran_n = 128: one scale per 128x128 block of B (weights);
 *       sfb_gran_n = 1:   one scale per row of B and 128 K.
 *   K: positive multiple of 128.  fp32 accumulation; one accumulation order.
 */
int gemm_fp8_nt(const void* A, const void* sfa, const void* B, const void* sfb, void* D,
                int M, int N, int K, int64_t lda, int64_t ldb, int64_t ldd,
                int64_t ld_sfa, int64_t ld_sfb, int sfb_gran_n, void* stream);

/*
 * gemm_fp4_nt — FP4 E2M1 GEMM, one UE8M0 scale per 32 K elements for every row of A
 * and of B (pages: FP4 coverage, section "Cobertura de operações ..." of "DeepGEMM-Ascend
 * cobre quantas operações no Ascend 950?"):
 *   D[m,n] = bf16( sum_kb 2^(ea[m,kb]-127) * 2^(eb[n,kb]-127) * sum_{k in kb} A[m,k]*B[n,k] ).
 *   A, B: two E2M1 values per byte, even K index in the low nibble: [M][lda], [N][ldb]
 *         with lda, ldb in BYTES (>= K/2).
 *   sfa SF words for MN = M, KB = K/32; sfb SF words for MN = N, KB = K/32.
 *   K: positive multiple of 64.
 */
int gemm_fp4_nt(const void* A, const void* sfa, const void* B, const void* sfb, void* D,
                int M, int N, int K, int64_t lda, int64_t ldb, int64_t ldd,
                int64_t ld_sfa, int64_t ld_sfb, void* stream);

/*
 * m_grouped_gemm_fp8_nt_contiguous — M-grouped FP8 GEMM for mixture-of-experts layers
 * ("DeepSeek lanza kernels de DeepGEMM para Huawei Ascend 950", section "Qué incluye el
 * lanzamiento": grouped operations for mixture-of-experts models).  The rows of all
 * experts are concatenated along M; row m uses expert g = m_indices[m]:
 *   D[m,n] = FP8 formula above with B := B[g], SFB := SFB[g]   if g >= 0,
 *   D[m,n] = 0                                                  if g == -1 (padding).
 *   A [M_total][K] E4M3 (row stride K); sfa SF words for MN = M_total, ld_sfa.
 *   B [G][N][K] E4M3 (contiguous); sfb [G][ceil(KB/2)][ld_sfb] SF words per expert with
 *     MN = ceil(N/sfb_gran_n); D [M_total][N] bf16 (row stride N).
 *   m_indices int32 [M_total]: every 128-row block [128i, 128i+128) holds one expert's
 *     rows followed by -1 padding rows only; its first row is not padding.
 *   M_total: positive multiple of 128.  K: positive multiple of 128.  1 <= G.
 *   A block that breaks the layout rule (index >= G, < -1, or a second expert in the
 *   block) latches BSP_ERR_DEVICE_CHECK; its rows hold unspecified values.
 */
int m_grouped_gemm_fp8_nt_contiguous(const void* A, const void* sfa, const void* B, const void* sfb,
                                     void* D, const int32_t* m_indices, int M_total, int N, int K,
                                     int G, int64_t ld_sfa, int64_t ld_sfb, int sfb_gran_n,
                                     void* stream);

/*
 * m_grouped_gemm_fp8_nt_masked — M-grouped FP8 GEMM in the masked (decode-time) layout,
 * which the pages list as not yet implemented in their release ("DeepGEMM-Ascend cobre
 * quantas operações no Ascend 950?", section "Cobertura de operações e a lacuna declarada no
 * repositório").  Every expert g owns a slab of max_m rows; only the first masked_m[g] rows of
 * the slab are products, the count being read on the device (so a CUDA graph can be captured
 * before the routing that produces it is known):
 *   D[g][m][n] = FP8 formula above with B := B[g], SFB := SFB[g]   for m < masked_m[g];
 *   rows m >= masked_m[g] of D are not written (they keep whatever they held).
 *   A [G][max_m][K] E4M3; sfa SF words for MN = G*max_m (row g*max_m + m), ld_sfa.
 *   B [G][N][K] E4M3; sfb [G][ceil(KB/2)][ld_sfb] SF words per expert, MN = ceil(N/sfb_gran_n).
 *   D [G][max_m][N] bf16.  masked_m int32 [G] in device memory, values in [0, max_m]; a value
 *   outside latches BSP_ERR_DEVICE_CHECK and is clamped into the range.
 *   1 <= G <= 1024; max_m a positive multiple of 128; K a positive multiple of 128; N*2 a
 *   multiple of 16 bytes.  The work is split by the device-side counts: tiles of rows past
 *   masked_m[g] are neither loaded nor computed.
 */
int m_grouped_gemm_fp8_nt_masked(const void* A, const void* sfa, const void* B, const void* sfb, void* D,
                                 const int32_t* masked_m, int G, int max_m, int N, int K, int64_t ld_sfa,
                                 int64_t ld_sfb, int sfb_gran_n, void* stream);

/*
 * transform_sf_ue8m0 — scale factors [mn][kb] (row stride ld_in) into SF words
 * int16 [ceil(kb/2)][ld_out] (layout above).
 *   in_kind 0: fp32 scales, each an exact positive normal power of two; its biased
 *              exponent (bits 30..23) is the UE8M0 byte.  A value that is not such a
 *              power of two latches BSP_ERR_DEVICE_CHECK (its byte is still written).
 *   in_kind 1: uint8 biased UE8M0 bytes, copied as they are; the byte 0xFF (NaN in UE8M0)
 *              latches BSP_ERR_DEVICE_CHECK (it is still written).
 *   ld_out >= mn and ld_out*2 a multiple of 16 bytes; sf_out must not overlap sf_in.
 * The caller decides whether a tensor is already packed ("reuse or convert",
 * "Fatores de escala FP8 e o formato UE8M0 no Ascend"); this call always converts.
 */
int transform_sf_ue8m0(const void* sf_in, int in_kind, int mn, int kb, int64_t ld_in,
                       void* sf_out, int64_t ld_out, void* stream);

/*
 * transform_sf_ue8m0_pair — two independent conversions of transform_sf_ue8m0 with the same
 * in_kind and kb (a GEMM's A and B scales) in one launch: sf_a [mn_a][kb] (row stride
 * ld_in_a) into out_a int16 [ceil(kb/2)][ld_out_a], and likewise for b.  Each tensor follows
 * the rules of transform_sf_ue8m0; no output may overlap the other output or either input.
 * The results are the bytes the two single calls give.
 */
int transform_sf_ue8m0_pair(const void* sf_a, int mn_a, int64_t ld_in_a, void* out_a, int64_t ld_out_a,
                            const void* sf_b, int mn_b, int64_t ld_in_b, void* out_b, int64_t ld_out_b,
                            int in_kind, int kb, void* stream);

/*
 * transform_sf_ue8m0_batched — transform_sf_ue8m0 of `batch` same-shaped tensors (for example
 * the per-expert B scales [G][mn][kb] of a grouped GEMM) in one launch: tensor z is read at
 * sf_in + z * batch_stride_in (elements of the input kind) and written at
 * sf_out + z * batch_stride_out (int16 words), each with the rules of transform_sf_ue8m0.
 *   1 <= batch <= 65535.  For batch > 1: batch_stride_in >= (mn-1)*ld_in + kb,
 *   batch_stride_out >= ceil(kb/2)*ld_out and batch_stride_out*2 a multiple of 16 bytes (the
 *   strides are ignored when batch == 1).  The whole input and output ranges must not overlap.
 * The results are the bytes `batch` single calls give.
 */
int transform_sf_ue8m0_batched(const void* sf_in, int in_kind, int batch, int mn, int kb, int64_t ld_in,
                               int64_t batch_stride_in, void* sf_out, int64_t ld_out, int64_t batch_stride_out,
                               void* stream);

/*
 * quantize_fp8_ue8m0 — the step before the GEMM: real values to E4M3 codes with one
 * power-of-two UE8M0 scale per block, the scales written straight into the SF-word layout
 * ("DeepGEMM-Ascend cobre quantas operações no Ascend 950?", section "Fatores de escala FP8
 * e o formato UE8M0 no Ascend": a power-of-two scale per block so that the block fits the
 * FP8 range, stored as UE8M0 and packed in pairs along K, MN-major).
 *   x [rows][ld_x]: in_kind 0 fp32, 1 bf16; all values finite (a non-finite value latches
 *     BSP_ERR_DEVICE_CHECK; its block's codes are then unspecified).
 *   block_rows 1: a block is 1 x 128 (activations; scale rows = rows);
 *   block_rows 128: a block is 128 x 128 (weights; scale rows = ceil(rows/128), the last
 *     block may be shorter).
 *   Per block: e = the smallest integer with 448 * 2^e >= max|x| (0 for an all-zero block),
 *     clamped to [-126, 127]; UE8M0 byte e + 127; code = x * 2^-e rounded to the nearest
 *     E4M3 value (ties to even, sign kept).
 *   q [rows][ld_q] uint8 E4M3 codes; sf int16 [ceil(cols/256)][ld_sf] SF words (layout
 *     above, MN = scale rows; words of rows >= MN and the high byte past an odd block count
 *     are 0) — what gemm_fp8_nt takes as sfa (block_rows 1) or sfb (block_rows 128,
 *     sfb_gran_n = 128).
 *   cols: positive multiple of 128.  ld_x >= cols, ld_q >= cols, ld_sf >= scale rows; x, q,
 *   sf 16-byte aligned, ld_x * element size, ld_q and ld_sf * 2 multiples of 16 bytes.  The
 *   buffers must not overlap.  All memory is the caller's; nothing is allocated.
 */
int quantize_fp8_ue8m0(const void* x, int in_kind, int rows, int cols, int64_t ld_x, int block_rows,
                       void* q, int64_t ld_q, void* sf, int64_t ld_sf, void* stream);

/*
 * gemm_fp8_nt_noalloc — the FP8 block-scaled GEMM of gemm_fp8_nt for callers that cannot
 * allocate device memory.  (The pages have no counterpart; this is a deployment variant.)
 *
 * Who needs it: gemm_fp8_nt wants its scale factors already packed and keeps its status word
 * in memory the library cudaMalloc's on first use.  A caller that holds plain UE8M0 bytes
 * and cannot call cudaMalloc — for example code running under a framework whose caching
 * allocator has already reserved the device memory, a loop that cannot afford cudaMalloc's
 * implicit device synchronisation, or a C program that forbids allocation after start-up —
 * would have nowhere to put the packed words.  This call packs them into a 4 MiB scratch
 * array that the library defines statically on the device (every GPU that loads the library
 * holds it until the process exits), then runs the same GEMM kernel.  It calls no cudaMalloc,
 * cudaFree or allocating library routine.
 *
 *   A, B, D, M, N, K, lda, ldb, ldd, sfb_gran_n: as in gemm_fp8_nt.
 *   sfa_e8m0  uint8 UE8M0 bytes [M][ld_sfa_in], one per row of A and 128 K (ld_sfa_in >= K/128).
 *   sfb_e8m0  uint8 UE8M0 bytes [ceil(N/sfb_gran_n)][ld_sfb_in] (ld_sfb_in >= K/128).
 *   status    device int, output: set to 0 by the call, then latched by its kernels like the
 *             status word of the other calls (BSP_ERR_TIMEOUT, BSP_ERR_DEVICE_CHECK); read it
 *             after the stream has finished.
 * Limit: the packed words (round_up(M,8) + round_up(ceil(N/g),8) int16 per K pair) plus the
 * tensor-core layout of them the GEMM loads (one 32-bit word per row and four K blocks, B
 * rows counted per 224-row tile) must fit in 4 MiB — for example M up to about 12000 at
 * N = 7168, K = 16384; larger calls return BSP_ERR_UNSUPPORTED and launch nothing.
 * Every call shares the one scratch array and overwrites it: calls that overlap on the GPU
 * (different streams, or different host threads on one device) race on it and must be
 * ordered by the caller.  The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for the process; make that
 * first call before any stream capture, and do not use this entry point on a device after
 * cudaDeviceReset, or from a context other than the device's primary one (the kept address
 * would then be stale).  A scale byte 0xFF (NaN) latches BSP_ERR_DEVICE_CHECK in `status`.
 */
int gemm_fp8_nt_noalloc(const void* A, const void* sfa_e8m0, const void* B, const void* sfb_e8m0, void* D,
                        int* status, int M, int N, int K, int64_t lda, int64_t ldb, int64_t ldd,
                        int64_t ld_sfa_in, int64_t ld_sfb_in, int sfb_gran_n, void* stream);

/*
 * bsp_get_device_status — synchronises `stream`, then returns and clears the status
 * word latched by kernels on the current device (BSP_OK if nothing was latched).
 */
int bsp_get_device_status(void* stream);

/* bsp_status_string — static description of a status code (never NULL). */
const char* bsp_status_string(int status);

/*
 * bsp_set_wait_timeout_ns — upper bound for every device-side pipeline wait (default
 * 2e9 ns).  A wait that exceeds it latches BSP_ERR_TIMEOUT and the kernel winds down.
 * Returns the previous value.
 */
uint64_t bsp_set_wait_timeout_ns(uint64_t ns);

/*
 * bsp_gemm_plan — how a GEMM of this kind and shape would be launched on the current
 * device, without launching it.  kind: 0 BF16, 1 FP8 (gemm_fp8_nt), 2 FP4, 3 M-grouped FP8
 * (M = M_total), 4 masked M-grouped FP8 (M = max_m; plan[4] then counts the work items of one
 * expert whose count is max_m).  Writes eight int32 to `plan` (caller-owned host memory):
 *   plan[0] rows per tile (128 single CTA, 256 CTA pair)   plan[1] columns per tile
 *   plan[2] K slices per split tile (1: no split)          plan[3] split tiles
 *   plan[4] work items (whole tiles + slices)              plan[5] persistent workers launched
 *   plan[6] 1 if the product is computed transposed, D^T = B A^T (M <= 128: the tile rows
 *           then run along N and the columns along M), else 0
 *   plan[7] 1 if the two K slices of every tile run on the two CTA pairs of one 4-CTA cluster
 *           and are added in distributed shared memory (BF16, FP8 or FP4 at M <= 128, two slices
 *           per tile, all tiles co-resident), else 0; the sums and their order are the same
 *           either way
 * The tiles left after the last full wave of workers are cut along K into slices at
 * scale-group boundaries when that shortens the last wave (at least two slices of eight or
 * more K steps); their fp32 partial sums meet in a workspace and are added in slice order
 * before the bf16 rounding, so results do not change from run to run.
 * Returns BSP_ERR_ARG for a bad kind, sizes <= 0 or a NULL plan; needs an sm_100 device.
 */
int bsp_gemm_plan(int kind, int M, int N, int K, int32_t* plan);

/*
 * bsp_kernel_launches — number of kernels this library has launched in this process
 * (all devices, all calls).  For the bench's launch count.
 */
uint64_t bsp_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* BSP_H */
