// quantize.cu — host side of quantize_fp8_ue8m0 (declared in bsp.h): argument checks, the
// tensor map of the input and the launch of the persistent quantiser kernel (quantize.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "bsp.h"
#include "internal.h"
#include "quantize.cuh"

namespace {

constexpr int kMaxDev = 64;
// Each wait of the quantiser is on its own TMA copies (microseconds); this bounds it all the same.
constexpr unsigned long long kQuantWaitNs = 2000000000ull;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int encode_input_map(CUtensorMap* m, bool bf16, const void* x, int rows, int cols, int64_t ld_x, int box_cols) {
    static std::once_flag once;
    static EncodeTiledFn encode = nullptr;
    std::call_once(once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    if (!encode) return BSP_ERR_CUDA;
    const int es = bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld_x * es)};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, 128};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                              const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_CUDA;
}

template <class C>
int launch_quantize(const CUtensorMap& tm, bsp::QuantArgs a, cudaStream_t st) {
    static std::once_flag once[kMaxDev];
    static cudaError_t err[kMaxDev];
    static int sms[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return BSP_ERR_CUDA;
    std::call_once(once[dev], [&] {
        err[dev] = cudaFuncSetAttribute(bsp::quantize_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
        if (err[dev] == cudaSuccess) err[dev] = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    });
    if (err[dev] != cudaSuccess) return BSP_ERR_CUDA;
    const int grid = a.num_tiles < sms[dev] ? a.num_tiles : sms[dev];  // one persistent CTA per SM
    bsp::quantize_kernel<C><<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tm, a);
    bsp::detail::note_launch();
    return cudaGetLastError() == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
}

}  // namespace

extern "C" int quantize_fp8_ue8m0(const void* x, int in_kind, int rows, int cols, int64_t ld_x, int block_rows,
                                  void* q, int64_t ld_q, void* sf, int64_t ld_sf, void* stream) {
    using namespace bsp;
    if (!x || !q || !sf || rows <= 0 || cols <= 0 || (in_kind != 0 && in_kind != 1)) return BSP_ERR_ARG;
    if (block_rows != 1 && block_rows != 128) return BSP_ERR_ARG;
    if (cols % 128) return BSP_ERR_SHAPE;
    const bool bf16 = in_kind == 1;
    const int es = bf16 ? 2 : 4;
    const int kb = cols / 128;
    const int scale_rows = (rows + block_rows - 1) / block_rows;
    if (ld_x < cols || ld_q < cols || ld_sf < scale_rows) return BSP_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sf)) return BSP_ERR_ALIGN;
    if ((ld_x * es) % 16 || ld_q % 16 || (ld_sf * 2) % 16) return BSP_ERR_ALIGN;
    int* status = nullptr;
    if (const int rc = detail::status_word(&status)) return rc;
    const int tile_cols = bf16 ? QuantCfg<true>::TC : QuantCfg<false>::TC;
    QuantArgs a{};
    a.rows = rows;
    a.kb_count = kb;
    a.col_tiles = (cols + tile_cols - 1) / tile_cols;
    const int64_t tiles = (int64_t)((rows + 127) / 128) * a.col_tiles;
    if (tiles > 0x7fffffff) return BSP_ERR_UNSUPPORTED;
    a.num_tiles = (int)tiles;
    a.scale_rows = scale_rows;
    a.block_rows = block_rows;
    a.ld_q = ld_q;
    a.ld_sf = ld_sf;
    a.q = static_cast<uint8_t*>(q);
    a.sf = static_cast<uint8_t*>(sf);
    a.status = status;
    a.timeout_ns = kQuantWaitNs;
    CUtensorMap tm;
    if (const int rc = encode_input_map(&tm, bf16, x, rows, cols, ld_x, tile_cols)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return bf16 ? launch_quantize<QuantCfg<true>>(tm, a, st) : launch_quantize<QuantCfg<false>>(tm, a, st);
}
