// api.cu — host side of libbsp.so: argument validation, tensor-map (TMA descriptor)
// encoding, per-device context, kernel selection and launch for the C ABI in bsp.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "bsp.h"
#include "gemm.cuh"
#include "internal.h"
#include "sf_layout.cuh"
#include "sf_transform.cuh"

#define BSP_TRY(x)                     \
    do {                               \
        const int _rc = (x);           \
        if (_rc != BSP_OK) return _rc; \
    } while (0)

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

int64_t round_up_i(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

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

// Co-resident workers (CTAs or CTA pairs) of config C on the current device: a persistent
// grid larger than this would serialise its last workers.
template <class C>
int max_workers_of(const DeviceCtx& ctx, int* out) {
    static std::once_flag once[kMaxDevices];
    static int workers[kMaxDevices];
    static cudaError_t err[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSP_ERR_CUDA;
    std::call_once(once[dev], [&] {
        err[dev] = cudaFuncSetAttribute(gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C::CLUSTER;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(C::CLUSTER * (ctx.sms / C::CLUSTER));
        int clusters = 0;
        if (err[dev] == cudaSuccess) err[dev] = cudaOccupancyMaxActiveClusters(&clusters, gemm_kernel<C>, &cfg);
        workers[dev] = clusters > 0 ? clusters : ctx.sms / C::CLUSTER;
    });
    if (err[dev] != cudaSuccess) return BSP_ERR_CUDA;
    *out = workers[dev];
    return BSP_OK;
}

// Tail plan: how many whole tiles, and into how many K slices the rest is cut.  The tiles
// left over after the last full wave of workers are split when at least two slices of
// eight or more K steps fit per tile, up to 16 slices and no more than the idle workers
// take in one wave, so that the last wave keeps most workers busy instead of a few.
struct TailPlan {
    int tiles, full_tiles, splits, tail_tiles, num_work;
};

TailPlan plan_tail(int tiles, int num_kb, int period, int workers, bool allow) {
    TailPlan p{tiles, tiles, 1, 0, tiles};
    const int rem = tiles % workers;
    if (!allow || rem == 0) return p;
    const int groups = (num_kb + period - 1) / period;
    int s = workers / rem;
    s = s < 16 ? s : 16;
    s = s < groups ? s : groups;
    while (s >= 2 && num_kb / s < 8) --s;
    if (s < 2) return p;
    p.full_tiles = tiles - rem;
    p.splits = s;
    p.tail_tiles = rem;
    p.num_work = p.full_tiles + rem * s;
    return p;
}

template <class C>
int64_t tail_ws_bytes(const TailPlan& p) {
    return p.splits > 1 ? (int64_t)p.tail_tiles * p.splits * C::TILE_M * C::BN * 4 : 0;
}
// Split-tail counters ([split tiles][CTAs][4 epilogue warps] int) followed by the share
// claims ([split tiles][CTAs][4][splits] int), zeroed before the GEMM runs.
template <class C>
int64_t tail_counters(const TailPlan& p) {
    return (int64_t)p.tail_tiles * C::CTAS * 4;
}
template <class C>
int64_t tail_count_bytes(const TailPlan& p) {
    return p.splits > 1 ? round_up_i(tail_counters<C>(p) * (1 + p.splits) * 4, 256) : 0;
}

// Launch config C with the split-tail plan `p` (ws: its workspace, count: its zeroed counters).
template <class C>
int launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa, const CUtensorMap& tsb,
           GemmArgs a, const TailPlan& p, float* ws, int* count, const DeviceCtx& ctx, cudaStream_t stream) {
    // D: bf16 [M][ldd], stored in 32 x 32 blocks through a 64-byte-swizzled staging buffer; the
    // cluster split of a transposed problem stores 64 rows x 32 columns of D (the swapped
    // problem's N x M) from plain row-major blocks
    CUtensorMap td, tw;
    if constexpr (C::CSPLIT) {
        const cuuint64_t dims[2] = {(cuuint64_t)a.M, (cuuint64_t)a.N};
        const cuuint64_t strides[1] = {(cuuint64_t)(a.ldd * 2)};
        const cuuint32_t box[2] = {32, (cuuint32_t)C::X_COLS};
        BSP_TRY(encode(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.D, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE));
    } else {
        const cuuint64_t dims[2] = {(cuuint64_t)a.N, (cuuint64_t)a.M};
        const cuuint64_t strides[1] = {(cuuint64_t)(a.ldd * 2)};
        const cuuint32_t box[2] = {32, 32};
        BSP_TRY(encode(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.D, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B));
    }
    if (p.splits > 1) {
        // workspace: fp32 [split tiles * splits * TILE_M][BN], stored in 32 x 32 blocks
        const cuuint64_t dims[2] = {(cuuint64_t)C::BN, (cuuint64_t)p.tail_tiles * p.splits * C::TILE_M};
        const cuuint64_t strides[1] = {(cuuint64_t)C::BN * 4};
        const cuuint32_t box[2] = {32, 32};
        BSP_TRY(encode(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, ws, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B));
    } else {
        tw = td;  // not read
    }
    int max_workers = 0;
    BSP_TRY(max_workers_of<C>(ctx, &max_workers));
    a.num_tiles = p.tiles;
    a.full_tiles = p.full_tiles;
    a.splits = p.splits;
    a.num_work = p.num_work;
    a.ws = ws;
    a.tail_count = count;
    a.tail_claim = count ? count + tail_counters<C>(p) : nullptr;
    a.group_m = 8;  // raster groups of 8 row blocks: measured ~1 % faster than 16 or 4 at 4096x7168x16384
    a.status = ctx.status;
    a.timeout_ns = g_timeout_ns.load();
    const int workers = a.num_work < max_workers ? a.num_work : max_workers;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C::CLUSTER;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // Scaled kinds follow their own scale layout pass on the stream: the GEMM may launch while
    // that pass runs (set-up, operand loads) and waits for it only before reading its output.
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = C::SCALED ? 2 : 1;
    cfg.gridDim = dim3(C::CLUSTER * workers);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_kernel<C>, ta, tb, tsa, tsb, td, tw, a);
    g_launches.fetch_add(1);
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? BSP_OK : BSP_ERR_CUDA;
}

//                          kind        BN   stages grouped pair  accumulators
using CfgBF16P224 = GemmCfg<Kind::BF16, 224, 6, false, true>;
using CfgFP8P224 = GemmCfg<Kind::FP8, 224, 6, false, true>;
using CfgFP4P224 = GemmCfg<Kind::FP4, 224, 6, false, true>;
// 256 x 256 pair tiles keep the tensor pipe busier than 256 x 224 ones (measured: about 8%
// more throughput per tile), but two 256-column accumulators leave no TMEM for the scales,
// so these run with one accumulator and an epilogue that empties it into registers at once.
using CfgBF16P256 = GemmCfg<Kind::BF16, 256, 6, false, true, 1>;
using CfgFP8P256 = GemmCfg<Kind::FP8, 256, 6, false, true, 1>;
using CfgFP4P256 = GemmCfg<Kind::FP4, 256, 5, false, true, 1>;
// constants only (M <= 128 runs transposed)
using CfgBF16 = GemmCfg<Kind::BF16, 224, 4, false, false>;
using CfgFP8 = GemmCfg<Kind::FP8, 224, 4, false, false>;
using CfgFP4 = GemmCfg<Kind::FP4, 224, 4, false, false>;
using CfgGrouped = GemmCfg<Kind::FP8, 224, 4, true, false>;
// contiguous grouped layout on CTA pairs (pairs of 128-row blocks of one expert), used while the
// block count fits the kernel's on-device tile list; CfgGrouped (single CTAs) otherwise
using CfgGroupedPair = GemmCfg<Kind::FP8, 224, 6, true, true>;
using CfgGroupedPair256 = GemmCfg<Kind::FP8, 256, 6, true, true, 1>;
// masked layout, transposed: 256 rows of an expert's B on a CTA pair against up to 256 of its
// rows of A as the MMA's N (cut to the valid rows at run time), so B is streamed once per expert
// (per 256 valid rows) instead of once per 128-row block
using CfgMaskedT = GemmCfg<Kind::FP8, 256, 6, true, true, 1, true, true>;
// M <= 128: computed as D^T = B A^T on 256 x 128 pair tiles (B's rows along the pair, A's rows
// across), written transposed.  Per SM and K step: 128 rows of B and 64 of A for 128 x 128
// products, against the same bytes for 128 x 64 in single-CTA narrow tiles: half the bytes per
// product, in a kernel whose loads are latency-bound.
using CfgBF16S = GemmCfg<Kind::BF16, 128, 8, false, true, 2, false, true>;
using CfgFP8S = GemmCfg<Kind::FP8, 128, 8, false, true, 2, false, true>;
using CfgFP4S = GemmCfg<Kind::FP4, 128, 7, false, true, 2, false, true>;
// M <= 128 whose transposed tiles would all be cut into two K slices: the two halves of a tile
// run on the two CTA pairs of a 4-CTA cluster and meet in distributed shared memory instead of
// a global workspace (one tile per cluster)
using CfgFP8S2 = GemmCfg<Kind::FP8, 128, 8, false, true, 2, false, true, true>;
using CfgBF16S2 = GemmCfg<Kind::BF16, 128, 8, false, true, 2, false, true, true>;
using CfgFP4S2 = GemmCfg<Kind::FP4, 128, 7, false, true, 2, false, true, true>;

// Grouped pair tiles 256 columns wide unless 224-wide ones cover N with enough fewer wasted
// columns to make up for being about 8% less efficient.
bool grouped_wide(int N) {
    const int64_t w256 = (int64_t)((N + 255) / 256) * 256, w224 = (int64_t)((N + 223) / 224) * 224;
    return w256 * 23 <= w224 * 25;
}

// Tile shape by problem shape.  M > 128: CTA pairs, 256 or 224 columns wide, whichever
// finishes first by a model of the waves (tile time proportional to its MMA work, 224-wide
// tiles 8% less efficient, a split tail paying for its longest slice plus about four K steps
// of reduction).  M <= 128: the product runs transposed on 256 x 128 pair tiles.
enum class Shape { Pair256, Pair224, Swap };
Shape pick_shape(int M, int N, int num_kb, int period, int sms) {
    if (M <= 128) return Shape::Swap;
    const int workers = sms / 2;
    const auto cost = [&](int bn, double eff) {
        const int tiles = ((M + 255) / 256) * ((N + bn - 1) / bn);
        const TailPlan p = plan_tail(tiles, num_kb, period, workers, true);
        double steps;
        if (p.splits > 1) {
            const int groups = (num_kb + period - 1) / period;
            steps = (double)(p.full_tiles / workers) * num_kb + (double)((groups + p.splits - 1) / p.splits) * period + 4.0;
        } else {
            steps = (double)((tiles + workers - 1) / workers) * num_kb;
        }
        return steps * 256.0 * bn / eff;
    };
    return cost(256, 1.0) <= cost(224, 0.92) ? Shape::Pair256 : Shape::Pair224;
}

// Problem description shared by the GEMM entry points.
struct Operands {
    const void *A, *B, *sfa, *sfb;
    int64_t lda, ldb, ld_sfa, ld_sfb;
    int mn_b;         // scale rows of B (per expert)
    int words;        // int16 scale words along K
    int groups = 1;   // experts (grouped layout)
};

// The swapped problem D^T = B A^T: operands, scale tensors and sizes exchanged; B's scale
// granularity becomes the A-operand's, A's per-row scales the B-operand's.
void swap_operands(Operands& o, GemmArgs& a) {
    std::swap(o.A, o.B);
    std::swap(o.sfa, o.sfb);
    std::swap(o.lda, o.ldb);
    std::swap(o.ld_sfa, o.ld_sfb);
    o.mn_b = a.M;
    std::swap(a.M, a.N);
    a.sfa_gran = a.sfb_gran;
    a.sfb_gran = 1;
}


int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Scale chunks of config C: layouts of the A and B chunk tensors and their bytes.
template <class C>
struct ScaleChunks {
    SfLayout a, b;
    int64_t a_bytes = 0, b_bytes = 0;
    ScaleChunks(const Operands& o, const GemmArgs& g) {
        const int q = (o.words + 2 * C::UT_WORDS - 1) / (2 * C::UT_WORDS);
        if constexpr (C::MT) {
            // A' = B_g (its scales per expert, 128-row tiles), B' = the rows of A (128-row atoms;
            // a tile loads the two atoms of its chunk)
            a = SfLayout{g.N, g.sfb_gran, o.words, o.ld_sfb, (int64_t)o.words * o.ld_sfb, C::BM, 1, C::UT_WORDS,
                         (g.N + C::BM - 1) / C::BM, q, o.groups};
            b = SfLayout{g.M, 1, o.words, o.ld_sfa, 0, 128, 1, C::UT_WORDS, (g.M + 127) / 128, q, 1};
            a_bytes = round_up((int64_t)q * a.tiles * C::SFA_CHUNK * o.groups, 256);
            b_bytes = round_up((int64_t)q * b.tiles * 512 * C::UT_WORDS, 256);
            return;
        }
        a = SfLayout{g.M, g.sfa_gran > 1 ? g.sfa_gran : 1, o.words, o.ld_sfa, 0, C::BM, 1, C::UT_WORDS,
                     (g.M + C::BM - 1) / C::BM, q, 1};
        const int64_t b_gstride = (int64_t)o.words * o.ld_sfb;
        b = SfLayout{g.N, g.sfb_gran, o.words, o.ld_sfb, b_gstride, C::BN, C::SFB_ATOMS, C::UT_WORDS,
                     (g.N + C::BN - 1) / C::BN, q, o.groups};
        a_bytes = round_up((int64_t)q * a.tiles * C::SFA_CHUNK, 256);
        b_bytes = round_up((int64_t)q * b.tiles * C::SFB_CHUNK * o.groups, 256);
    }
    int64_t bytes() const { return a_bytes + b_bytes; }
};

// Scale chunks of both operands, and `zero_bytes` (a multiple of 16) zeroed at `zero`.
int launch_sf_layout(const void* in_a, const SfLayout& pa, void* out_a, const void* in_b, const SfLayout& pb,
                     void* out_b, void* zero, int64_t zero_bytes, cudaStream_t stream) {
    const int64_t total = sf_layout_words(pa) + sf_layout_words(pb) + zero_bytes / 16;
    const int64_t blocks = (total + 255) / 256;
    // a grid that is resident at once (grid-stride loop): every CTA reaches launch_dependents as
    // soon as the kernel before it has completed, so the GEMM after it launches at that moment
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = (int64_t)sms * 4;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(blocks < cap ? blocks : cap));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, sf_tmem_layout_kernel, static_cast<const uint16_t*>(in_a), pa,
                                             static_cast<uint32_t*>(out_a), static_cast<const uint16_t*>(in_b), pb,
                                             static_cast<uint32_t*>(out_b), static_cast<uint4*>(zero), zero_bytes / 16);
    g_launches.fetch_add(1);
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? BSP_OK : BSP_ERR_CUDA;
}

// Stream-ordered scratch from a pool this library owns on each device, which keeps its memory
// mapped between calls (the default pool would hand it back to the driver at every
// synchronisation and map it again on the next call).
int scratch_alloc(void** p, size_t bytes, cudaStream_t stream) {
    // under stream capture the allocation becomes a graph memory node (graph-owned pool)
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return BSP_ERR_CUDA;
    if (cs == cudaStreamCaptureStatusActive)
        return cudaMallocAsync(p, bytes, stream) == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
    static std::mutex mu;
    static cudaMemPool_t pools[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSP_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (pools[dev] == nullptr) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            if (cudaMemPoolCreate(&pools[dev], &props) != cudaSuccess) return BSP_ERR_CUDA;
            uint64_t keep = UINT64_MAX;
            if (cudaMemPoolSetAttribute(pools[dev], cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess)
                return BSP_ERR_CUDA;
        }
    }
    return cudaMallocFromPoolAsync(p, bytes, pools[dev], stream) == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
}

// Chunk tensor map: 8-byte elements, one chunk per (row tile, group [, expert]).
int chunk_map(CUtensorMap* m, const void* base, int chunk_bytes, int tiles, int q, int experts_or_neg) {
    // experts_or_neg < 0: a rank-4 map over -experts_or_neg experts (the grouped kernel's 4-D loads)
    const int experts = experts_or_neg < 0 ? -experts_or_neg : experts_or_neg;
    const cuuint64_t dims[4] = {(cuuint64_t)(chunk_bytes / 8), (cuuint64_t)tiles, (cuuint64_t)q,
                                (cuuint64_t)experts};
    const cuuint64_t strides[3] = {(cuuint64_t)chunk_bytes, (cuuint64_t)chunk_bytes * tiles,
                                   (cuuint64_t)chunk_bytes * tiles * q};
    const cuuint32_t box[4] = {(cuuint32_t)(chunk_bytes / 8), 1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, experts_or_neg < 0 ? 4 : 3, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Tiles, K steps and the tail plan of config C for this problem on this device.
template <class C>
int plan_gemm(GemmArgs& a, const DeviceCtx& ctx, TailPlan* p, int* workers) {
    const int64_t row_bytes = C::kind == Kind::FP4 ? a.K / 2 : (C::kind == Kind::BF16 ? (int64_t)a.K * 2 : a.K);
    a.num_kb = (int)((row_bytes + 127) / 128);
    a.m_blocks = (a.M + C::TILE_M - 1) / C::TILE_M;
    a.n_blocks = (a.N + C::BN - 1) / C::BN;
    int max_workers = 0;
    BSP_TRY(max_workers_of<C>(ctx, &max_workers));
    *p = plan_tail(a.m_blocks * a.n_blocks, a.num_kb, C::SF_PERIOD, max_workers, !C::GROUPED && !C::CSPLIT);
    if constexpr (C::MT) {
        // masked transposed: at most ceil(max_m / 256) chunks per expert, found on the device
        const int g = a.G > 0 ? a.G : 1, mm = a.G > 0 ? a.max_m : a.M;
        p->tiles = p->full_tiles = p->num_work = g * ((mm + C::MCHUNK - 1) / C::MCHUNK) * a.n_blocks;
    }
    if constexpr (C::PAIR_LIST) {
        // the pair tiles are found on the device: between M/256 and M/128 of them per column block;
        // the grid is sized for the most
        p->tiles = p->full_tiles = p->num_work = (a.M / 128) * a.n_blocks;
    }
    *workers = max_workers;
    return BSP_OK;
}

// True when config C would cut every tile of this (transposed) problem into exactly two K
// slices and the tiles fit as co-resident clusters of the cluster-split config C2.
template <class C, class C2>
bool use_cluster_split(const GemmArgs& a, const DeviceCtx& ctx) {
    GemmArgs t = a;
    TailPlan p;
    int max_workers = 0, clusters = 0;
    if (plan_gemm<C>(t, ctx, &p, &max_workers) != BSP_OK) return false;
    if (p.splits != 2 || p.full_tiles != 0) return false;
    if (max_workers_of<C2>(ctx, &clusters) != BSP_OK) return false;
    return p.tiles <= clusters;
}

template <class C>
int describe_plan(int M, int N, int K, const DeviceCtx& ctx, int32_t* out) {
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    TailPlan p;
    int max_workers = 0;
    BSP_TRY(plan_gemm<C>(a, ctx, &p, &max_workers));
    out[0] = C::TILE_M;
    out[1] = C::BN;
    out[2] = p.splits;
    out[3] = p.tail_tiles;
    out[4] = p.num_work;
    out[5] = p.num_work < max_workers ? p.num_work : max_workers;
    out[6] = 0;
    out[7] = 0;
    return BSP_OK;
}

// Encode the tensor maps for config C and launch it.  Scratch (stream-ordered, from the
// caller's stream, unless `fixed` is given): the scale chunks of scaled kinds, then the
// split tail's counters (zeroed by the scale layout pass, or a memset) and workspace.  With
// `fixed` scratch of `fixed_bytes`, the tail is split only if its workspace fits.
template <class C>
int launch_gemm(const Operands& o, GemmArgs a, const DeviceCtx& ctx, cudaStream_t stream, void* fixed = nullptr,
                int64_t fixed_bytes = 0) {
    constexpr bool bf16 = C::kind == Kind::BF16;
    const auto dt = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const int es = bf16 ? 2 : 1;
    const int64_t row_elems = C::kind == Kind::FP4 ? a.K / 2 : a.K;
    CUtensorMap ta, tb, tsa, tsb;
    if constexpr (C::MT) {
        BSP_TRY(operand_map_3d(&ta, o.B, a.K, a.N, o.groups, C::BM));          // B_g: 128 rows per CTA
        BSP_TRY(operand_map(&tb, dt, es, o.A, row_elems, a.M, o.lda, C::BN_CTA));  // rows of A
    } else {
    BSP_TRY(operand_map(&ta, dt, es, o.A, row_elems, a.M, o.lda, C::BM));
    if constexpr (C::GROUPED)
        BSP_TRY(operand_map_3d(&tb, o.B, a.K, a.N, o.groups, C::BN_CTA));
    else
        BSP_TRY(operand_map(&tb, dt, es, o.B, row_elems, a.N, o.ldb, C::BN_CTA));
    }
    TailPlan p;
    int max_workers = 0;
    BSP_TRY(plan_gemm<C>(a, ctx, &p, &max_workers));
    int64_t chunk_bytes = 0;
    SfLayout la{}, lb{};
    if constexpr (C::SCALED) {
        const ScaleChunks<C> sc(o, a);
        chunk_bytes = sc.bytes();
        la = sc.a, lb = sc.b;
    }
    int64_t tail_bytes = tail_count_bytes<C>(p) + tail_ws_bytes<C>(p);
    if (fixed != nullptr && chunk_bytes + tail_bytes > fixed_bytes) {
        p = plan_tail(p.tiles, a.num_kb, C::SF_PERIOD, max_workers, false);
        tail_bytes = 0;
    }
    void* scratch = fixed;
    const bool owned = fixed == nullptr && chunk_bytes + tail_bytes > 0;
    if (owned) BSP_TRY(scratch_alloc(&scratch, (size_t)(chunk_bytes + tail_bytes), stream));
    char* base = static_cast<char*>(scratch);
    int* count = tail_bytes ? reinterpret_cast<int*>(base + chunk_bytes) : nullptr;
    float* ws = tail_bytes ? reinterpret_cast<float*>(base + chunk_bytes + tail_count_bytes<C>(p)) : nullptr;
    int rc = BSP_OK;
    if constexpr (C::SCALED) {
        char* wa = base;
        char* wb = wa + ScaleChunks<C>(o, a).a_bytes;
        rc = launch_sf_layout(C::MT ? o.sfb : o.sfa, la, wa, C::MT ? o.sfa : o.sfb, lb, wb, count,
                              tail_bytes ? tail_count_bytes<C>(p) : 0, stream);
        if constexpr (C::MT) {
            if (rc == BSP_OK) rc = chunk_map(&tsa, wa, C::SFA_CHUNK, la.tiles, la.q, -o.groups);
            if (rc == BSP_OK) rc = chunk_map(&tsb, wb, 512 * C::UT_WORDS, lb.tiles, lb.q, 1);
        } else {
            if (rc == BSP_OK) rc = chunk_map(&tsa, wa, C::SFA_CHUNK, la.tiles, la.q, 1);
            if (rc == BSP_OK) rc = chunk_map(&tsb, wb, C::SFB_CHUNK, lb.tiles, lb.q, C::GROUPED ? -o.groups : 1);
        }
    } else {
        tsa = ta, tsb = tb;  // not read
        if (tail_bytes && cudaMemsetAsync(count, 0, (size_t)tail_count_bytes<C>(p), stream) != cudaSuccess)
            rc = BSP_ERR_CUDA;
    }
    if (rc == BSP_OK) rc = launch<C>(ta, tb, tsa, tsb, a, p, ws, count, ctx, stream);
    if (owned && cudaFreeAsync(scratch, stream) != cudaSuccess && rc == BSP_OK) rc = BSP_ERR_CUDA;
    return rc;
}

int check_ld(int64_t ld, int64_t min_elems, int esize) {
    if (ld < min_elems) return BSP_ERR_SHAPE;
    if ((ld * esize) % 16) return BSP_ERR_ALIGN;
    return BSP_OK;
}


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

int status_word(int** out) {
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    *out = ctx->status;
    return BSP_OK;
}

void note_launch() { g_launches.fetch_add(1); }

int launch_sf_transform_u8_pair(const void* in_a, int mn_a, int64_t ld_in_a, void* out_a, int64_t ld_out_a,
                                const void* in_b, int mn_b, int64_t ld_in_b, void* out_b, int64_t ld_out_b, int kb,
                                int* status, cudaStream_t stream) {
    if ((kb + kSfTileKB - 1) / kSfTileKB > 65535) return BSP_ERR_UNSUPPORTED;
    const SfJob jobs[2] = {{in_a, ld_in_a, static_cast<uint16_t*>(out_a), ld_out_a, mn_a},
                           {in_b, ld_in_b, static_cast<uint16_t*>(out_b), ld_out_b, mn_b}};
    const bool ok = launch_sf_transform(jobs, 2, 1, kb, status, stream);
    g_launches.fetch_add(1);
    return ok ? BSP_OK : BSP_ERR_CUDA;
}

int64_t gemm_fp8_scale_scratch_bytes(int M, int N, int K, int sfb_gran_n) {
    const int kb = K / 128, words = (kb + 1) / 2;
    const Operands o{nullptr, nullptr, nullptr, nullptr, 0, 0, 0, 0, (N + sfb_gran_n - 1) / sfb_gran_n, words};
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K, a.sfb_gran = sfb_gran_n;
    int sms = 0;
    if (device_facts_noalloc(&sms) != BSP_OK) sms = 148;
    switch (pick_shape(M, N, kb, CfgFP8::SF_PERIOD, sms)) {
        case Shape::Pair256: return ScaleChunks<CfgFP8P256>(o, a).bytes();
        case Shape::Pair224: return ScaleChunks<CfgFP8P224>(o, a).bytes();
        default: {  // Swap: M <= 128
            Operands os = o;
            GemmArgs as = a;
            swap_operands(os, as);
            return ScaleChunks<CfgFP8S>(os, as).bytes();
        }
    }
}

int launch_gemm_fp8_packed(const void* A, const void* sfa, const void* B, const void* sfb, void* D, int M, int N,
                           int K, int64_t lda, int64_t ldb, int64_t ldd, int64_t ld_sfa, int64_t ld_sfb,
                           int sfb_gran_n, int* status, void* scratch, int64_t scratch_bytes, cudaStream_t stream) {
    DeviceCtx ctx;
    BSP_TRY(device_facts_noalloc(&ctx.sms));
    ctx.ready = true;
    ctx.status = status;
    const int kb = K / 128, words = (kb + 1) / 2;
    const int mn_b = (N + sfb_gran_n - 1) / sfb_gran_n;
    const Operands o{A, B, sfa, sfb, lda, ldb, ld_sfa, ld_sfb, mn_b, words};
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = ldd;
    a.sfb_gran = sfb_gran_n;
    switch (pick_shape(M, N, kb, CfgFP8::SF_PERIOD, ctx.sms)) {
        case Shape::Pair256: return launch_gemm<CfgFP8P256>(o, a, ctx, stream, scratch, scratch_bytes);
        case Shape::Pair224: return launch_gemm<CfgFP8P224>(o, a, ctx, stream, scratch, scratch_bytes);
        default: {  // Swap: M <= 128
            Operands os = o;
            swap_operands(os, a);
            if (use_cluster_split<CfgFP8S, CfgFP8S2>(a, ctx))
                return launch_gemm<CfgFP8S2>(os, a, ctx, stream, scratch, scratch_bytes);
            return launch_gemm<CfgFP8S>(os, a, ctx, stream, scratch, scratch_bytes);
        }
    }
}

}  // namespace detail
}  // namespace bsp

using namespace bsp;

namespace {

// Argument checks of one conversion; its input and output byte ranges go to `in_r` / `out_r`.
int check_sf_job(const void* sf_in, int in_kind, int mn, int kb, int64_t ld_in, void* sf_out, int64_t ld_out,
                 const char* in_r[2], const char* out_r[2]) {
    if (!sf_in || !sf_out || mn <= 0 || kb <= 0 || (in_kind != 0 && in_kind != 1)) return BSP_ERR_ARG;
    if (ld_in < kb || ld_out < mn) return BSP_ERR_SHAPE;
    if ((ld_out * 2) % 16 || !aligned16(sf_out)) return BSP_ERR_ALIGN;
    if (in_kind == 0 && (reinterpret_cast<uintptr_t>(sf_in) & 3u)) return BSP_ERR_ALIGN;
    const int words = (kb + 1) / 2;
    in_r[0] = static_cast<const char*>(sf_in);
    in_r[1] = in_r[0] + ((int64_t)(mn - 1) * ld_in + kb) * (in_kind == 0 ? 4 : 1);
    out_r[0] = static_cast<const char*>(sf_out);
    out_r[1] = out_r[0] + (int64_t)words * ld_out * 2;
    if (in_r[0] < out_r[1] && out_r[0] < in_r[1]) return BSP_ERR_ARG;  // overlapping buffers
    if ((kb + kSfTileKB - 1) / kSfTileKB > 65535) return BSP_ERR_UNSUPPORTED;
    return BSP_OK;
}

bool overlap(const char* const a[2], const char* const b[2]) { return a[0] < b[1] && b[0] < a[1]; }

}  // namespace

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
    const Operands o{A, B, nullptr, nullptr, lda, ldb, 0, 0, 0, 0};
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = ldd;
    a.sfb_gran = 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (pick_shape(M, N, (K + 63) / 64, CfgBF16::SF_PERIOD, ctx->sms)) {
        case Shape::Pair256: return launch_gemm<CfgBF16P256>(o, a, *ctx, st);
        case Shape::Pair224: return launch_gemm<CfgBF16P224>(o, a, *ctx, st);
        default: {  // Swap: M <= 128
            Operands os = o;
            swap_operands(os, a);
            if (use_cluster_split<CfgBF16S, CfgBF16S2>(a, *ctx)) return launch_gemm<CfgBF16S2>(os, a, *ctx, st);
            return launch_gemm<CfgBF16S>(os, a, *ctx, st);
        }
    }
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
    const Operands o{A, B, sfa, sfb, lda, ldb, ld_sfa, ld_sfb, mn_b, words};
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = ldd;
    a.sfb_gran = sfb_gran_n;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (pick_shape(M, N, kb, CfgFP8::SF_PERIOD, ctx->sms)) {
        case Shape::Pair256: return launch_gemm<CfgFP8P256>(o, a, *ctx, st);
        case Shape::Pair224: return launch_gemm<CfgFP8P224>(o, a, *ctx, st);
        default: {  // Swap: M <= 128
            Operands os = o;
            swap_operands(os, a);
            if (use_cluster_split<CfgFP8S, CfgFP8S2>(a, *ctx)) return launch_gemm<CfgFP8S2>(os, a, *ctx, st);
            return launch_gemm<CfgFP8S>(os, a, *ctx, st);
        }
    }
}

int gemm_fp4_nt(const void* A, const void* sfa, const void* B, const void* sfb, void* D, int M, int N, int K,
                int64_t lda, int64_t ldb, int64_t ldd, int64_t ld_sfa, int64_t ld_sfb, void* stream) {
    if (!A || !sfa || !B || !sfb || !D || M <= 0 || N <= 0 || K <= 0) return BSP_ERR_ARG;
    if (K % 64) return BSP_ERR_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned16(sfb)) return BSP_ERR_ALIGN;
    const int words = K / 64;
    BSP_TRY(check_ld(lda, K / 2, 1));
    BSP_TRY(check_ld(ldb, K / 2, 1));
    BSP_TRY(check_ld(ldd, N, 2));
    BSP_TRY(check_ld(ld_sfa, M, 2));
    BSP_TRY(check_ld(ld_sfb, N, 2));
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    const Operands o{A, B, sfa, sfb, lda, ldb, ld_sfa, ld_sfb, N, words};
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = ldd;
    a.sfb_gran = 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (pick_shape(M, N, K / 256 + (K % 256 ? 1 : 0), CfgFP4::SF_PERIOD, ctx->sms)) {
        case Shape::Pair256: return launch_gemm<CfgFP4P256>(o, a, *ctx, st);
        case Shape::Pair224: return launch_gemm<CfgFP4P224>(o, a, *ctx, st);
        default: {  // Swap: M <= 128
            Operands os = o;
            swap_operands(os, a);
            if (use_cluster_split<CfgFP4S, CfgFP4S2>(a, *ctx)) return launch_gemm<CfgFP4S2>(os, a, *ctx, st);
            return launch_gemm<CfgFP4S>(os, a, *ctx, st);
        }
    }
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
    Operands o{A, B, sfa, sfb, K, K, ld_sfa, ld_sfb, mn_b, words};
    o.groups = G;
    GemmArgs a{};
    a.M = M_total, a.N = N, a.K = K;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = N;
    a.m_indices = m_indices, a.G = G;
    a.sfb_gran = sfb_gran_n;
    if (M_total / 128 <= CfgGroupedPair::MAX_PAIR_TILES) {
        if (grouped_wide(N)) return launch_gemm<CfgGroupedPair256>(o, a, *ctx, static_cast<cudaStream_t>(stream));
        return launch_gemm<CfgGroupedPair>(o, a, *ctx, static_cast<cudaStream_t>(stream));
    }
    return launch_gemm<CfgGrouped>(o, a, *ctx, static_cast<cudaStream_t>(stream));
}

int m_grouped_gemm_fp8_nt_masked(const void* A, const void* sfa, const void* B, const void* sfb, void* D,
                                 const int32_t* masked_m, int G, int max_m, int N, int K, int64_t ld_sfa,
                                 int64_t ld_sfb, int sfb_gran_n, void* stream) {
    if (!A || !sfa || !B || !sfb || !D || !masked_m || G < 1 || max_m <= 0 || N <= 0 || K <= 0) return BSP_ERR_ARG;
    if (sfb_gran_n != 1 && sfb_gran_n != 128) return BSP_ERR_ARG;
    if (G > CfgMaskedT::MAX_MASKED_G) return BSP_ERR_UNSUPPORTED;
    if (K % 128 || max_m % 128) return BSP_ERR_SHAPE;
    if ((int64_t)G * max_m > 0x7fffffff) return BSP_ERR_UNSUPPORTED;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned16(sfb)) return BSP_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(masked_m) & 3u) != 0) return BSP_ERR_ALIGN;
    if ((N * 2) % 16) return BSP_ERR_ALIGN;  // rows of D are N bf16 long
    const int kb = K / 128, words = (kb + 1) / 2;
    const int mn_b = (N + sfb_gran_n - 1) / sfb_gran_n;
    const int M = G * max_m;
    BSP_TRY(check_ld(ld_sfa, M, 2));
    BSP_TRY(check_ld(ld_sfb, mn_b, 2));
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    Operands o{A, B, sfa, sfb, K, K, ld_sfa, ld_sfb, mn_b, words};
    o.groups = G;
    GemmArgs a{};
    a.M = M, a.N = N, a.K = K;
    a.D = static_cast<__nv_bfloat16*>(D), a.ldd = N;
    a.G = G;
    a.masked_m = masked_m, a.max_m = max_m;
    a.sfb_gran = sfb_gran_n;
    return launch_gemm<CfgMaskedT>(o, a, *ctx, static_cast<cudaStream_t>(stream));
}

int transform_sf_ue8m0(const void* sf_in, int in_kind, int mn, int kb, int64_t ld_in, void* sf_out, int64_t ld_out,
                       void* stream) {
    const char *in_r[2], *out_r[2];
    BSP_TRY(check_sf_job(sf_in, in_kind, mn, kb, ld_in, sf_out, ld_out, in_r, out_r));
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    const bool ok = launch_sf_transform(sf_in, in_kind, mn, kb, ld_in, static_cast<uint16_t*>(sf_out), ld_out,
                                        ctx->status, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1);
    return ok ? BSP_OK : BSP_ERR_CUDA;
}

int transform_sf_ue8m0_pair(const void* sf_a, int mn_a, int64_t ld_in_a, void* out_a, int64_t ld_out_a,
                            const void* sf_b, int mn_b, int64_t ld_in_b, void* out_b, int64_t ld_out_b, int in_kind,
                            int kb, void* stream) {
    const char *in_a[2], *oa[2], *in_b[2], *ob[2];
    BSP_TRY(check_sf_job(sf_a, in_kind, mn_a, kb, ld_in_a, out_a, ld_out_a, in_a, oa));
    BSP_TRY(check_sf_job(sf_b, in_kind, mn_b, kb, ld_in_b, out_b, ld_out_b, in_b, ob));
    if (overlap(oa, ob) || overlap(oa, in_b) || overlap(ob, in_a)) return BSP_ERR_ARG;
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    const SfJob jobs[2] = {{sf_a, ld_in_a, static_cast<uint16_t*>(out_a), ld_out_a, mn_a},
                           {sf_b, ld_in_b, static_cast<uint16_t*>(out_b), ld_out_b, mn_b}};
    const bool ok = launch_sf_transform(jobs, 2, in_kind, kb, ctx->status, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1);
    return ok ? BSP_OK : BSP_ERR_CUDA;
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

int bsp_gemm_plan(int kind, int M, int N, int K, int32_t* plan) {
    if (!plan || M <= 0 || N <= 0 || K <= 0 || kind < 0 || kind > 4) return BSP_ERR_ARG;
    DeviceCtx* ctx;
    BSP_TRY(ensure_ctx(&ctx));
    switch (kind) {
        case 0:
            switch (pick_shape(M, N, (K + 63) / 64, CfgBF16::SF_PERIOD, ctx->sms)) {
                case Shape::Pair256: return describe_plan<CfgBF16P256>(M, N, K, *ctx, plan);
                case Shape::Pair224: return describe_plan<CfgBF16P224>(M, N, K, *ctx, plan);
                default: {  // Swap: M <= 128
                    BSP_TRY(describe_plan<CfgBF16S>(N, M, K, *ctx, plan));
                    plan[6] = 1;
                    GemmArgs t{};
                    t.M = N, t.N = M, t.K = K;
                    plan[7] = use_cluster_split<CfgBF16S, CfgBF16S2>(t, *ctx) ? 1 : 0;
                    return BSP_OK;
                }
            }
        case 1:
            switch (pick_shape(M, N, (K + 127) / 128, CfgFP8::SF_PERIOD, ctx->sms)) {
                case Shape::Pair256: return describe_plan<CfgFP8P256>(M, N, K, *ctx, plan);
                case Shape::Pair224: return describe_plan<CfgFP8P224>(M, N, K, *ctx, plan);
                default: {  // Swap: M <= 128
                    BSP_TRY(describe_plan<CfgFP8S>(N, M, K, *ctx, plan));
                    plan[6] = 1;
                    GemmArgs t{};
                    t.M = N, t.N = M, t.K = K;
                    plan[7] = use_cluster_split<CfgFP8S, CfgFP8S2>(t, *ctx) ? 1 : 0;
                    return BSP_OK;
                }
            }
        case 2:
            switch (pick_shape(M, N, (K + 255) / 256, CfgFP4::SF_PERIOD, ctx->sms)) {
                case Shape::Pair256: return describe_plan<CfgFP4P256>(M, N, K, *ctx, plan);
                case Shape::Pair224: return describe_plan<CfgFP4P224>(M, N, K, *ctx, plan);
                default: {  // Swap: M <= 128
                    BSP_TRY(describe_plan<CfgFP4S>(N, M, K, *ctx, plan));
                    plan[6] = 1;
                    GemmArgs t{};
                    t.M = N, t.N = M, t.K = K;
                    plan[7] = use_cluster_split<CfgFP4S, CfgFP4S2>(t, *ctx) ? 1 : 0;
                    return BSP_OK;
                }
            }
        case 4: {  // masked: M = rows per expert slab; work items counted for a single expert
            BSP_TRY(describe_plan<CfgMaskedT>(M, N, K, *ctx, plan));
            plan[4] = ((M + CfgMaskedT::MCHUNK - 1) / CfgMaskedT::MCHUNK) * ((N + CfgMaskedT::BN - 1) / CfgMaskedT::BN);
            plan[6] = 1;
            return BSP_OK;
        }
        default:
            if (M / 128 <= CfgGroupedPair::MAX_PAIR_TILES)
                return grouped_wide(N) ? describe_plan<CfgGroupedPair256>(M, N, K, *ctx, plan)
                                       : describe_plan<CfgGroupedPair>(M, N, K, *ctx, plan);
            return describe_plan<CfgGrouped>(M, N, K, *ctx, plan);
    }
}

}  // extern "C"
