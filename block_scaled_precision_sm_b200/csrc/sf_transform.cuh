// sf_transform.cuh — UE8M0 scale factors [mn][kb] -> int16 words [ceil(kb/2)][ld_out],
// word(j, r) = e[r][2j] | e[r][2j+1] << 8, MN-major ("DeepSeek lanza kernels de DeepGEMM
// para Huawei Ascend 950", section "Qué incluye el lanzamiento": each pair of UE8M0
// factors along K in one 16-bit integer, MN-major).
//
// One CTA turns a tile of 128 rows x 64 scale blocks around through shared memory.  Reads run
// along K (the input's contiguous axis) in VEC-byte vectors, as wide as the input's row stride
// and base alignment allow, with every lane busy whatever kb is (the tile's (row, vector) pairs
// are numbered linearly); the exponent bytes land transposed in shared memory, K-major, so that
// each output store is one 16-byte run of eight MN-consecutive words, built from two 8-byte
// shared loads with byte permutes.  The transform moves a few bytes per scale and is bound by
// DRAM bandwidth; each thread issues all of its loads before it uses any.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace bsp {

constexpr int kSfTileMN = 128;  // rows per CTA
constexpr int kSfTileKB = 64;   // scale blocks per CTA
constexpr int kSfThreads = 256;

template <int VEC>
struct SfVec;
template <>
struct SfVec<16> {
    using T = uint4;
    static __device__ __forceinline__ uint32_t word(const T& v, int i) {
        return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
    }
};
template <>
struct SfVec<8> {
    using T = uint2;
    static __device__ __forceinline__ uint32_t word(const T& v, int i) { return i == 0 ? v.x : v.y; }
};
template <>
struct SfVec<4> {
    using T = uint32_t;
    static __device__ __forceinline__ uint32_t word(const T& v, int) { return v; }
};
template <>
struct SfVec<1> {
    using T = uint8_t;
    static __device__ __forceinline__ uint32_t word(const T& v, int) { return v; }
};

// One tensor to convert: scales [mn][kb] at `in` (row stride ld_in) -> words at `out` (ld_out).
struct SfJob {
    const void* in;
    int64_t ld_in;
    uint16_t* out;
    int64_t ld_out;
    int mn;
};
// Tensors with the same kb and input kind converted by one launch, so that independent
// conversions share one launch and one round trip; blockIdx.z picks the tensor.  Either a
// table of up to two (in_zstride == 0), or a batch: tensor z is job[0] moved by z * in_zstride
// input bytes and z * out_zstride output words.
struct SfJobs {
    SfJob job[2];
    int64_t in_zstride;
    int64_t out_zstride;
};

// IN_KIND 0: fp32 power-of-two scales (UE8M0 byte = biased fp32 exponent);
// IN_KIND 1: uint8 UE8M0 bytes.  VEC: bytes per global load (16, 8 or 4 for fp32; 16, 8, 4 or
// 1 for bytes); every job's row stride ld_in and base are multiples of VEC bytes.
template <int IN_KIND, int VEC>
__global__ void __launch_bounds__(kSfThreads) sf_transform_kernel(const SfJobs jobs, int kb, int* status) {
    SfJob jb = blockIdx.z == 0 ? jobs.job[0] : jobs.job[1];
    if (jobs.in_zstride != 0) {
        jb = jobs.job[0];
        jb.in = static_cast<const char*>(jb.in) + (int64_t)blockIdx.z * jobs.in_zstride;
        jb.out += (int64_t)blockIdx.z * jobs.out_zstride;
    }
    // the grid covers the larger job: row tiles past this job's end have nothing to do
    if ((int64_t)blockIdx.x * kSfTileMN >= jb.ld_out) return;
    const void* __restrict__ in = jb.in;
    uint16_t* __restrict__ out = jb.out;
    const int mn = jb.mn;
    const int64_t ld_in = jb.ld_in, ld_out = jb.ld_out;
    constexpr int ES = IN_KIND == 0 ? 4 : 1;       // input element bytes
    constexpr int EV = VEC / ES;                   // elements per load
    static_assert(EV >= 1 && kSfTileKB % EV == 0, "vector width");
    // Loads go in groups of four rows at one K vector ("quads"): a thread's four loads are the same
    // K range of four consecutive rows, so each K block's four exponent bytes become one 32-bit
    // shared-memory store.  Consecutive threads take consecutive vectors of a row (coalesced).
    constexpr int RQ = 4;
    constexpr int MAX_Q = (kSfTileMN / RQ * (kSfTileKB / EV) + kSfThreads - 1) / kSfThreads;  // quads per thread
    constexpr int PITCH = kSfTileMN + 16;          // bytes per K block in shared memory
    using V = typename SfVec<VEC>::T;
    __shared__ __align__(16) uint8_t eT[kSfTileKB][PITCH];

    const int r0 = blockIdx.x * kSfTileMN;
    const int k0 = blockIdx.y * kSfTileKB;
    const int kn = min(kSfTileKB, kb - k0);         // scale blocks in this tile
    const int rn = min(kSfTileMN, mn - r0);         // input rows in this tile (<= 0: padding only)
    const int vpr = (kn + EV - 1) / EV;             // loads per row
    const int quads = rn > 0 ? ((rn + RQ - 1) / RQ) * vpr : 0;
    // qidx / vpr as a multiply-high by ceil(2^32 / vpr): exact for qidx < 2^13 and 2 <= vpr <= 64
    // (vpr = 1 is qidx itself)
    const uint32_t vrec = vpr > 1 ? (uint32_t)((0x100000000ull + (uint64_t)vpr - 1) / (uint64_t)vpr) : 0u;
    const auto group_of = [&](int qidx) { return vpr > 1 ? (int)__umulhi((uint32_t)qidx, vrec) : qidx; };
    const int t = threadIdx.x;
    bool bad = false;

    // The kernel is launched with programmatic stream serialisation, so it may start while the
    // kernel before it still runs: it waits for that one before touching global memory, and only
    // then lets the next kernel launch, so whatever follows starts after everything before this
    // one has completed.
    griddep_wait();
    griddep_launch_dependents();

    // all loads first (up to MAX_Q quads in flight per thread), then the bytes into shared memory
    V v[MAX_Q][RQ];
#pragma unroll
    for (int it = 0; it < MAX_Q; ++it) {
        const int qidx = t + it * kSfThreads;
        if (qidx < quads) {
            const int g = group_of(qidx), k = (qidx - g * vpr) * EV;
#pragma unroll
            for (int q = 0; q < RQ; ++q) {
                const int i = RQ * g + q;
                const char* src = static_cast<const char*>(in) + ((int64_t)(r0 + i) * ld_in + k0 + k) * ES;
                if (i < rn && k + EV <= kn) {
                    v[it][q] = __ldg(reinterpret_cast<const V*>(src));
                } else {  // a row past the tile's, or a partial vector at the end of a row: zeros after
                    uint32_t w[VEC >= 4 ? VEC / 4 : 1] = {};
                    if (i < rn) {
#pragma unroll
                        for (int e = 0; e < EV; ++e) {
                            if (k + e < kn) {
                                const uint32_t x = ES == 4 ? __ldg(reinterpret_cast<const uint32_t*>(src) + e)
                                                           : (uint32_t)__ldg(reinterpret_cast<const uint8_t*>(src) + e);
                                if (ES == 4)
                                    w[e] = x;
                                else
                                    w[e / 4] |= x << (8 * (e % 4));
                            }
                        }
                    }
                    if constexpr (VEC == 16)
                        v[it][q] = make_uint4(w[0], w[1], w[2], w[3]);
                    else if constexpr (VEC == 8)
                        v[it][q] = make_uint2(w[0], w[1]);
                    else if constexpr (VEC == 4)
                        v[it][q] = w[0];
                    else
                        v[it][q] = (uint8_t)w[0];
                }
            }
        }
    }
#pragma unroll
    for (int it = 0; it < MAX_Q; ++it) {
        const int qidx = t + it * kSfThreads;
        if (qidx < quads) {
            const int g = group_of(qidx), k = (qidx - g * vpr) * EV;
#pragma unroll
            for (int e = 0; e < EV; ++e) {
                if (k + e < kn) {
                    uint32_t word = 0;
#pragma unroll
                    for (int q = 0; q < RQ; ++q) {
                        uint32_t b;
                        if constexpr (IN_KIND == 0) {
                            const uint32_t bits = SfVec<VEC>::word(v[it][q], e);
                            b = (bits >> 23) & 0xFFu;
                            // an exact positive normal power of two: sign 0, mantissa 0, exponent 1..254
                            // (rows past the tile's hold 0 and are not checked)
                            if (RQ * g + q < rn) bad |= (bits & 0x807FFFFFu) != 0u || b == 0u || b == 255u;
                        } else {
                            b = (SfVec<VEC>::word(v[it][q], e / 4) >> (8 * (e % 4))) & 0xFFu;
                            bad |= b == 255u;  // UE8M0 0xFF is NaN
                        }
                        word |= b << (8 * q);
                    }
                    *reinterpret_cast<uint32_t*>(&eT[k + e][RQ * g]) = word;
                }
            }
        }
    }
    __syncthreads();

    // words (k0/2 + j) for rows r0 + 8g .. r0 + 8g + 7: rows past mn and the high byte past an
    // odd kb are 0; rows past ld_out are not written (ld_out is a multiple of 8)
    const int wn = (kn + 1) / 2;
    for (int idx = t; idx < wn * (kSfTileMN / 8); idx += kSfThreads) {
        const int j = idx / (kSfTileMN / 8), g = idx - j * (kSfTileMN / 8);
        const int r = r0 + 8 * g;
        if (r >= ld_out) continue;
        const int valid = mn - r;  // rows of this run that hold scales
        const uint64_t keep = valid >= 8 ? ~0ull : valid <= 0 ? 0ull : (1ull << (8 * valid)) - 1ull;
        const uint64_t lo = *reinterpret_cast<const uint64_t*>(&eT[2 * j][8 * g]) & keep;
        const uint64_t hi = 2 * j + 1 < kn ? *reinterpret_cast<const uint64_t*>(&eT[2 * j + 1][8 * g]) & keep : 0ull;
        const uint32_t l0 = (uint32_t)lo, l1 = (uint32_t)(lo >> 32), h0 = (uint32_t)hi, h1 = (uint32_t)(hi >> 32);
        // word of row q = byte q of lo | byte q of hi << 8
        *reinterpret_cast<uint4*>(out + (int64_t)(k0 / 2 + j) * ld_out + r) =
            make_uint4(__byte_perm(l0, h0, 0x5140), __byte_perm(l0, h0, 0x7362), __byte_perm(l1, h1, 0x5140),
                       __byte_perm(l1, h1, 0x7362));
    }
    if (__any_sync(0xffffffffu, bad) && (t % 32) == 0) atomicCAS(status, 0, -7);
}

// Widest load (bytes) that the input's base address and row stride (and the stride between
// the tensors of a batch) allow.
inline int sf_transform_vec(const void* in, int in_kind, int64_t ld_in, int64_t zstride_bytes = 0) {
    const int es = in_kind == 0 ? 4 : 1;
    const uint64_t a = reinterpret_cast<uintptr_t>(in) | (uint64_t)(ld_in * es) | (uint64_t)zstride_bytes;
    for (int v : {16, 8, 4})
        if (a % (uint64_t)v == 0) return v;
    return es == 4 ? 4 : 1;
}

template <int IN_KIND, int VEC>
inline bool launch_sf_transform_vec(dim3 grid, const SfJobs& jobs, int kb, int* status, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kSfThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, sf_transform_kernel<IN_KIND, VEC>, jobs, kb, status) == cudaSuccess;
}

inline bool launch_sf_jobs(const SfJobs& jobs, dim3 grid, int vec, int in_kind, int kb, int* status,
                           cudaStream_t stream) {
    if (grid.y > 65535u || grid.z > 65535u) return false;
    bool ok;
    if (in_kind == 0)
        ok = vec == 16  ? launch_sf_transform_vec<0, 16>(grid, jobs, kb, status, stream)
             : vec == 8 ? launch_sf_transform_vec<0, 8>(grid, jobs, kb, status, stream)
                        : launch_sf_transform_vec<0, 4>(grid, jobs, kb, status, stream);
    else
        ok = vec == 16  ? launch_sf_transform_vec<1, 16>(grid, jobs, kb, status, stream)
             : vec == 8 ? launch_sf_transform_vec<1, 8>(grid, jobs, kb, status, stream)
             : vec == 4 ? launch_sf_transform_vec<1, 4>(grid, jobs, kb, status, stream)
                        : launch_sf_transform_vec<1, 1>(grid, jobs, kb, status, stream);
    return ok && cudaGetLastError() == cudaSuccess;
}

// Launch `count` (1 or 2) jobs on `stream` (programmatic serialisation: the kernel waits for
// the one before it); false if the launch failed or the grid is too large.
inline bool launch_sf_transform(const SfJob* job, int count, int in_kind, int kb, int* status, cudaStream_t stream) {
    SfJobs jobs = {};
    int64_t ld_max = 0;
    int vec = 16;
    for (int i = 0; i < count; ++i) {
        jobs.job[i] = job[i];
        ld_max = job[i].ld_out > ld_max ? job[i].ld_out : ld_max;
        const int v = sf_transform_vec(job[i].in, in_kind, job[i].ld_in);
        vec = v < vec ? v : vec;
    }
    const dim3 grid((unsigned)((ld_max + kSfTileMN - 1) / kSfTileMN), (unsigned)((kb + kSfTileKB - 1) / kSfTileKB),
                    (unsigned)count);
    return launch_sf_jobs(jobs, grid, vec, in_kind, kb, status, stream);
}

// `batch` tensors of the same shape, tensor z at job.in + z * in_zstride_bytes and job.out +
// z * out_zstride words, in one launch (batch <= 65535).
inline bool launch_sf_transform_batched(const SfJob& job, int batch, int64_t in_zstride_bytes, int64_t out_zstride,
                                        int in_kind, int kb, int* status, cudaStream_t stream) {
    SfJobs jobs = {};
    jobs.job[0] = job;
    jobs.in_zstride = batch > 1 ? in_zstride_bytes : 0;
    jobs.out_zstride = batch > 1 ? out_zstride : 0;
    const int vec = sf_transform_vec(job.in, in_kind, job.ld_in, jobs.in_zstride);
    const dim3 grid((unsigned)((job.ld_out + kSfTileMN - 1) / kSfTileMN), (unsigned)((kb + kSfTileKB - 1) / kSfTileKB),
                    (unsigned)batch);
    return launch_sf_jobs(jobs, grid, vec, in_kind, kb, status, stream);
}

inline bool launch_sf_transform(const void* in, int in_kind, int mn, int kb, int64_t ld_in, uint16_t* out,
                                int64_t ld_out, int* status, cudaStream_t stream) {
    const SfJob job{in, ld_in, out, ld_out, mn};
    return launch_sf_transform(&job, 1, in_kind, kb, status, stream);
}

}  // namespace bsp
