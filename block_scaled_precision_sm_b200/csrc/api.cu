// api.cu — host side of libbsp.so: argument validation, tensor-map (TMA descriptor)
// encoding, per-device context, kernel selection and launch for the C ABI in bsp.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "bsp.h"
#include "gemm.cuh"
#include "internal.h"
#include "sf_transform.cuh"

namespace bsp {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceCtx {
    bool ready = false;
    int sms = 0;
    int* status = nullptr;  // device status word (latched by kernels)
};

std::mutex g_mu;
DeviceCtx g_dev[kMaxDevices];
std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
std::atomic<uint64_t> g_launches{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int ensure_ctx(DeviceCtx** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSP_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BSP_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceCtx& c = g_dev[dev];
    if (!c.ready) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BSP_ERR_CUDA;
        if (major != 10) return BSP_ERR_UNSUPPORTED;  // sm_100a code only
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return BSP_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        int* st = nullptr;
        if (cudaMalloc(&st, 256) != cudaSuccess) return BSP_ERR_CUDA;
        if (cudaMemset(st, 0, 256) != cudaSuccess) return BSP_ERR_CUDA;
        c.sms = sms;
        c.status = st;
        c.ready = true;
    }
    *out = &c;
    return BSP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Encode a tiled tensor map; dims/box are innermost first, strides (bytes) for dims 1..rank-1.
int encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
           const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = g_encode(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                                sw == CU_TENSOR_MAP_SWIZZLE_NONE ? CU_TENSOR_MAP_L2_PROMOTION_NONE
                                                                 : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_CUDA;
}

// Operand tile map: rows x row_elems of `dt`, row stride `ld` elements, box = 128 bytes x box_rows.
int operand_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, int64_t row_elems,
                int64_t rows, int64_t ld, int box_rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)row_elems, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld * esize)};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / esize), (cuuint32_t)box_rows};
    return encode(m, dt, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

int operand_map_3d(CUtensorMap* m, const void* base, int64_t row_bytes, int64_t rows, int64_t groups,
                   int box_rows) {
    const cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)groups};
    const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)(row_bytes * rows)};
    const cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Scale-word map: int16 [words][ld], box = box_mn x box_words; rank 3 ([groups][words][ld],
// box depth 1) when `grouped`, since the grouped kernel issues 3-D loads even for one group.
int sf_map(CUtensorMap* m, const void* base, int64_t mn, int64_t words, int64_t ld, int box_mn, int box_words,
           int64_t groups, bool grouped = false) {
    const cuuint64_t dims[3] = {(cuuint64_t)mn, (cuuint64_t)words, (cuuint64_t)groups};
    const cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(ld * 2 * words)};
    const cuuint32_t box[3] = {(cuuint32_t)box_mn, (cuuint32_t)box_words, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, grouped ? 3 : 2, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <class C>
int launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa, const CUtensorMap& tsb,
           GemmArgs a, const DeviceCtx& ctx, cudaStream_t stream) {
    static std::once_flag attr_once[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once[dev], [&] {
        attr_err = cudaFuncSetAttribute(gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return BSP_ERR_CUDA;
    a.m_blocks = (a.M + C::BM - 1) / C::BM;
    a.n_blocks = (a.N + C::BN - 1) / C::BN;
    a.num_tiles = a.m_blocks * a.n_blocks;
    a.group_m = 16;
    a.status = ctx.status;
    a.timeout_ns = g_timeout_ns.load();
    const int grid = a.num_tiles < ctx.sms ? a.num_tiles : ctx.sms;
    gemm_kernel<C><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(ta, tb, tsa, tsb, a);
    g_launches.fetch_add(1);
    return cudaGetLastError() == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
}

using CfgBF16 = GemmCfg<Kind::BF16, 224, 5, false>;
using CfgFP8 = GemmCfg<Kind::FP8, 224, 4, false>;
using CfgFP4 = GemmCfg<Kind::FP4, 224, 4, false>;
using CfgGrouped = GemmCfg<Kind::FP8, 224, 4, true>;

int check_ld(int64_t ld, int64_t min_elems, int esize) {
    if (ld < min_elems) return BSP_ERR_SHAPE;
    if ((ld * esize) % 16) return BSP_ERR_ALIGN;
    return BSP_OK;
}

#define BSP_TRY(x)                     \
    do {                               \
        const int _rc = (x);           \
        if (_rc != BSP_OK) return _rc; \
    } while (0)

// Device facts without the per-device context (which allocates the status word).
int device_facts_noalloc(int* sms) {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSP_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return BSP_ERR_CUDA;
    if (major != 10) return BSP_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return BSP_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return BSP_OK;
}

}  // namespace

namespace detail {

int launch_sf_transform_u8(const void* in, int mn, int kb, int64_t ld_in, void* out, int64_t ld_out, int* status,
                           cudaStream_t stream) {
    const dim3 grid((unsigned)((ld_out + kSfTileMN - 1) / kSfTileMN), (unsigned)((kb + kSfTileKB - 1) / kSfTileKB));
    if (grid.y > 65535u) return BSP_ERR_UNSUPPORTED;
    sf_transform_kernel<1><<<grid, 256, 0, stream>>>(in, mn, kb, ld_in, static_cast<uint16_t*>(out), ld_out, status);
    g_launches.fetch_add(1);
    return cudaGetLastError() == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
}

int launch_gemm_fp8_packed(const void* A, const void* sfa, const void* B, const void* sfb, void* D, int M, int N,
                           int K, int64_t lda, int64_t ldb, int64_t ldd, int64_t ld_sfa, int64_t ld_sfb,
                           int sfb_gran_n, int* status, cudaStream_t stream) {
    DeviceCtx ctx;
    BSP_TRY(device_facts_noalloc(&ctx.sms));
    ctx.ready = true;
    ctx.status = status;
    const int kb = K / 128, words = (kb + 1) / 2;
    const int mn_b = (N + sfb_gran_n - 1) / sfb_gran_n;
    CUtensorMap ta, tb, tsa, tsb;
    BSP_TRY(operand_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, M, lda, CfgFP8::BM));
    BSP_TRY(operand_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, K, N, ldb, CfgFP8::BN));
    BSP_TRY(sf_map(&tsa, sfa, M, words, ld_sfa, CfgFP8::BM, 1, 1));
    BSP_TRY(sf_map(&tsb, sfb, mn_b, words, ld_sfb, sfb_gran_n == 1 ? CfgFP8::BN : 16, 1, 1));
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.num_kb = kb;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = ldd;
    a.sfb_gran = sfb_gran_n;
    return launch<CfgFP8>(ta, tb, tsa, tsb, a, ctx, stream);
}

}  // namespace detail
}  // namespace bsp

using namespace bsp;

extern "C" {

int gemm_bf16_nt(const void* A, const void* B, void* D, int M, int N, int K, int64_t lda, int64_t ldb, int64_t ldd,
                 void* stream) {
    if (!A || !B || !D || M <= 0 || N <= 0 || K <= 0) return BSP_ERR_ARG;
    if (K % 8) return BSP_ERR_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return BSP_ERR_ALIGN;
    BSP_TRY(check_ld(lda, K, 2));
    BSP_TRY(check_ld(ldb, K, 2));
    BSP_TRY(check_ld(ldd, N, 2));
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    CUtensorMap ta, tb;
    BSP_TRY(operand_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, K, M, lda, CfgBF16::BM));
    BSP_TRY(operand_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, K, N, ldb, CfgBF16::BN));
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.num_kb = (K + 63) / 64;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = ldd;
    a.sfb_gran = 1;
    return launch<CfgBF16>(ta, tb, ta, tb, a, *ctx, static_cast<cudaStream_t>(stream));
}

int gemm_fp8_nt(const void* A, const void* sfa, const void* B, const void* sfb, void* D, int M, int N, int K,
                int64_t lda, int64_t ldb, int64_t ldd, int64_t ld_sfa, int64_t ld_sfb, int sfb_gran_n,
                void* stream) {
    if (!A || !sfa || !B || !sfb || !D || M <= 0 || N <= 0 || K <= 0) return BSP_ERR_ARG;
    if (sfb_gran_n != 1 && sfb_gran_n != 128) return BSP_ERR_ARG;
    if (K % 128) return BSP_ERR_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned16(sfb)) return BSP_ERR_ALIGN;
    const int kb = K / 128, words = (kb + 1) / 2;
    const int mn_b = (N + sfb_gran_n - 1) / sfb_gran_n;
    BSP_TRY(check_ld(lda, K, 1));
    BSP_TRY(check_ld(ldb, K, 1));
    BSP_TRY(check_ld(ldd, N, 2));
    BSP_TRY(check_ld(ld_sfa, M, 2));
    BSP_TRY(check_ld(ld_sfb, mn_b, 2));
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    CUtensorMap ta, tb, tsa, tsb;
    BSP_TRY(operand_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, M, lda, CfgFP8::BM));
    BSP_TRY(operand_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, K, N, ldb, CfgFP8::BN));
    BSP_TRY(sf_map(&tsa, sfa, M, words, ld_sfa, CfgFP8::BM, 1, 1));
    BSP_TRY(sf_map(&tsb, sfb, mn_b, words, ld_sfb, sfb_gran_n == 1 ? CfgFP8::BN : 16, 1, 1));
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.num_kb = kb;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = ldd;
    a.sfb_gran = sfb_gran_n;
    return launch<CfgFP8>(ta, tb, tsa, tsb, a, *ctx, static_cast<cudaStream_t>(stream));
}

int gemm_fp4_nt(const void* A, const void* sfa, const void* B, const void* sfb, void* D, int M, int N, int K,
                int64_t lda, int64_t ldb, int64_t ldd, int64_t ld_sfa, int64_t ld_sfb, void* stream) {
    if (!A || !sfa || !B || !sfb || !D || M <= 0 || N <= 0 || K <= 0) return BSP_ERR_ARG;
    if (K % 64) return BSP_ERR_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned16(sfb)) return BSP_ERR_ALIGN;
    const int kb = K / 32, words = kb / 2;
    BSP_TRY(check_ld(lda, K / 2, 1));
    BSP_TRY(check_ld(ldb, K / 2, 1));
    BSP_TRY(check_ld(ldd, N, 2));
    BSP_TRY(check_ld(ld_sfa, M, 2));
    BSP_TRY(check_ld(ld_sfb, N, 2));
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    CUtensorMap ta, tb, tsa, tsb;
    BSP_TRY(operand_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K / 2, M, lda, CfgFP4::BM));
    BSP_TRY(operand_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, K / 2, N, ldb, CfgFP4::BN));
    BSP_TRY(sf_map(&tsa, sfa, M, words, ld_sfa, CfgFP4::BM, 4, 1));
    BSP_TRY(sf_map(&tsb, sfb, N, words, ld_sfb, CfgFP4::BN, 4, 1));
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.num_kb = (K / 2 + 127) / 128;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = ldd;
    a.sfb_gran = 1;
    return launch<CfgFP4>(ta, tb, tsa, tsb, a, *ctx, static_cast<cudaStream_t>(stream));
}

int m_grouped_gemm_fp8_nt_contiguous(const void* A, const void* sfa, const void* B, const void* sfb, void* D,
                                     const int32_t* m_indices, int M_total, int N, int K, int G, int64_t ld_sfa,
                                     int64_t ld_sfb, int sfb_gran_n, void* stream) {
    if (!A || !sfa || !B || !sfb || !D || !m_indices || M_total <= 0 || N <= 0 || K <= 0 || G < 1)
        return BSP_ERR_ARG;
    if (sfb_gran_n != 1 && sfb_gran_n != 128) return BSP_ERR_ARG;
    if (K % 128 || M_total % 128) return BSP_ERR_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned16(sfb)) return BSP_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(m_indices) & 3u) != 0) return BSP_ERR_ALIGN;
    if ((N * 2) % 16) return BSP_ERR_ALIGN;  // rows of D are N bf16 long
    const int kb = K / 128, words = (kb + 1) / 2;
    const int mn_b = (N + sfb_gran_n - 1) / sfb_gran_n;
    BSP_TRY(check_ld(ld_sfa, M_total, 2));
    BSP_TRY(check_ld(ld_sfb, mn_b, 2));
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    CUtensorMap ta, tb, tsa, tsb;
    BSP_TRY(operand_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, M_total, K, CfgGrouped::BM));
    BSP_TRY(operand_map_3d(&tb, B, K, N, G, CfgGrouped::BN));
    BSP_TRY(sf_map(&tsa, sfa, M_total, words, ld_sfa, CfgGrouped::BM, 1, 1));
    BSP_TRY(sf_map(&tsb, sfb, mn_b, words, ld_sfb, sfb_gran_n == 1 ? CfgGrouped::BN : 16, 1, G, true));
    GemmArgs a{};
    a.M = M_total, a.N = N, a.K = K;
    a.num_kb = kb;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = N;
    a.m_indices = m_indices, a.G = G;
    a.sfb_gran = sfb_gran_n;
    return launch<CfgGrouped>(ta, tb, tsa, tsb, a, *ctx, static_cast<cudaStream_t>(stream));
}

int transform_sf_ue8m0(const void* sf_in, int in_kind, int mn, int kb, int64_t ld_in, void* sf_out, int64_t ld_out,
                       void* stream) {
    if (!sf_in || !sf_out || mn <= 0 || kb <= 0 || (in_kind != 0 && in_kind != 1)) return BSP_ERR_ARG;
    if (ld_in < kb || ld_out < mn) return BSP_ERR_SHAPE;
    if ((ld_out * 2) % 16 || !aligned16(sf_out)) return BSP_ERR_ALIGN;
    if (in_kind == 0 && (reinterpret_cast<uintptr_t>(sf_in) & 3u)) return BSP_ERR_ALIGN;
    const int words = (kb + 1) / 2;
    const char* ib = static_cast<const char*>(sf_in);
    const char* ie = ib + ((int64_t)(mn - 1) * ld_in + kb) * (in_kind == 0 ? 4 : 1);
    const char* ob = static_cast<const char*>(sf_out);
    const char* oe = ob + (int64_t)words * ld_out * 2;
    if (ib < oe && ob < ie) return BSP_ERR_ARG;  // overlapping buffers
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    const dim3 grid((unsigned)((ld_out + kSfTileMN - 1) / kSfTileMN), (unsigned)((kb + kSfTileKB - 1) / kSfTileKB));
    if (grid.y > 65535u) return BSP_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint16_t* out = static_cast<uint16_t*>(sf_out);
    if (in_kind == 0)
        sf_transform_kernel<0><<<grid, 256, 0, st>>>(sf_in, mn, kb, ld_in, out, ld_out, ctx->status);
    else
        sf_transform_kernel<1><<<grid, 256, 0, st>>>(sf_in, mn, kb, ld_in, out, ld_out, ctx->status);
    g_launches.fetch_add(1);
    return cudaGetLastError() == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
}

int bsp_get_device_status(void* stream) {
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BSP_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, ctx->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return BSP_ERR_CUDA;
    if (v != 0 && cudaMemset(ctx->status, 0, sizeof v) != cudaSuccess) return BSP_ERR_CUDA;
    return v;
}

const char* bsp_status_string(int status) {
    switch (status) {
        case BSP_OK: return "ok";
        case BSP_ERR_ARG: return "invalid argument";
        case BSP_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
        case BSP_ERR_SHAPE: return "shape rule broken (K multiple, M_total multiple of 128, or ld too small)";
        case BSP_ERR_UNSUPPORTED: return "unsupported device or size (needs sm_100)";
        case BSP_ERR_CUDA: return "CUDA call failed";
        case BSP_ERR_TIMEOUT: return "device pipeline wait timed out";
        case BSP_ERR_DEVICE_CHECK: return "device check failed (bad scale value or expert index)";
        default: return "unknown status";
    }
}

uint64_t bsp_set_wait_timeout_ns(uint64_t ns) { return g_timeout_ns.exchange(ns); }

uint64_t bsp_kernel_launches(void) { return g_launches.load(); }

}  // extern "C"
