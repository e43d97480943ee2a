// noalloc.cu — gemm_fp8_nt_noalloc: the FP8 block-scaled GEMM for callers that cannot
// allocate device memory.
//
// The regular path needs memory that is neither an input nor an output: the packed int16
// scale words (which a caller holding plain UE8M0 bytes has to produce somewhere) and the
// library's status word (cudaMalloc'd on first use).  Some callers cannot call cudaMalloc:
// code running under a framework whose caching allocator has already reserved the device
// memory, loops where cudaMalloc's implicit device synchronisation is unacceptable, or C
// programs that forbid allocation after start-up.  This entry point keeps its scratch in the
// file-scope array below, which exists on every GPU that loads the library until the process
// exits, and takes the status word from the caller as an output.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "bsp.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB

// Packed SFA words at offset 0, packed SFB words and then the GEMM's scale chunks at the
// next 256-byte boundaries.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDev] = {};

// The array's name in host code is a host-side stand-in, not a device address: the kernels
// get the address cudaGetSymbolAddress returns, looked up once per device with that device
// current (done by the first call on each device).
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSP_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDev) return BSP_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return BSP_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return BSP_OK;
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

}  // namespace

extern "C" int gemm_fp8_nt_noalloc(const void* A, const void* sfa_e8m0, const void* B, const void* sfb_e8m0,
                                   void* D, int* status, int M, int N, int K, int64_t lda, int64_t ldb,
                                   int64_t ldd, int64_t ld_sfa_in, int64_t ld_sfb_in, int sfb_gran_n,
                                   void* stream) {
    if (!A || !sfa_e8m0 || !B || !sfb_e8m0 || !D || !status || M <= 0 || N <= 0 || K <= 0) return BSP_ERR_ARG;
    if (sfb_gran_n != 1 && sfb_gran_n != 128) return BSP_ERR_ARG;
    if (K % 128) return BSP_ERR_SHAPE;
    const auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (misaligned(A) || misaligned(B) || misaligned(D) || (reinterpret_cast<uintptr_t>(status) & 3u))
        return BSP_ERR_ALIGN;
    const int kb = K / 128, words = (kb + 1) / 2;
    const int mn_b = (N + sfb_gran_n - 1) / sfb_gran_n;
    if (lda < K || ldb < K || ldd < N || ld_sfa_in < kb || ld_sfb_in < kb) return BSP_ERR_SHAPE;
    if (lda % 16 || ldb % 16 || (ldd * 2) % 16) return BSP_ERR_ALIGN;
    // scratch: packed words for M and for ceil(N/g) scale rows (leading dimensions rounded to 8),
    // then the tensor-core layout of those words that the GEMM loads
    const int64_t ld_a = round_up(M, 8), ld_b = round_up(mn_b, 8);
    const int64_t off_b = round_up((int64_t)words * ld_a * 2, 256);
    const int64_t off_chunks = round_up(off_b + (int64_t)words * ld_b * 2, 256);
    const int64_t chunk_bytes = bsp::detail::gemm_fp8_scale_scratch_bytes(M, N, K, sfb_gran_n);
    if (off_chunks + chunk_bytes > (int64_t)kScratchBytes) return BSP_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (const int rc = scratch_address(&scratch)) return rc;
    unsigned char* sfa_w = static_cast<unsigned char*>(scratch);
    unsigned char* sfb_w = sfa_w + off_b;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the status word must start at zero for this call; the scratch is fully rewritten below
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return BSP_ERR_CUDA;
    if (const int rc = bsp::detail::launch_sf_transform_u8_pair(sfa_e8m0, M, ld_sfa_in, sfa_w, ld_a, sfb_e8m0, mn_b,
                                                                ld_sfb_in, sfb_w, ld_b, kb, status, st))
        return rc;
    return bsp::detail::launch_gemm_fp8_packed(A, sfa_w, B, sfb_w, D, M, N, K, lda, ldb, ldd, ld_a, ld_b,
                                               sfb_gran_n, status, sfa_w + off_chunks,
                                               (int64_t)kScratchBytes - off_chunks, st);
}
