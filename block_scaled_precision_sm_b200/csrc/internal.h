// internal.h — launch helpers shared between translation units of libbsp.so.  They take
// the status word from the caller and never allocate device memory.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace bsp {
namespace detail {

// The current device's status word (allocated on first use) and the launch counter of
// bsp_kernel_launches, for entry points outside api.cu.
int status_word(int** out);
void note_launch();

// SF words from two uint8 UE8M0 byte tensors [mn_x][ld_in_x] (the same kb) into int16
// [ceil(kb/2)][ld_out_x], in one launch; faults latch `status`.
int launch_sf_transform_u8_pair(const void* in_a, int mn_a, int64_t ld_in_a, void* out_a, int64_t ld_out_a,
                                const void* in_b, int mn_b, int64_t ld_in_b, void* out_b, int64_t ld_out_b, int kb,
                                int* status, cudaStream_t stream);

// Bytes of scratch the FP8 GEMM lays its scale chunks out in, for this problem.
int64_t gemm_fp8_scale_scratch_bytes(int M, int N, int K, int sfb_gran_n);

// FP8 block-scaled GEMM on packed SF words, same rules as gemm_fp8_nt; faults latch `status`.
// `scratch` (256-aligned, `scratch_bytes` >= gemm_fp8_scale_scratch_bytes) takes the scale
// chunks and, when it has room, the workspace of a split last wave.
int launch_gemm_fp8_packed(const void* A, const void* sfa, const void* B, const void* sfb, void* D, int M, int N,
                           int K, int64_t lda, int64_t ldb, int64_t ldd, int64_t ld_sfa, int64_t ld_sfb,
                           int sfb_gran_n, int* status, void* scratch, int64_t scratch_bytes,
                           cudaStream_t stream);

}  // namespace detail
}  // namespace bsp
