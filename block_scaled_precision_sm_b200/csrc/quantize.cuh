// quantize.cuh — fp32 / bf16 values to E4M3 codes with one power-of-two UE8M0 scale per block
// of 1 x 128 (activations) or 128 x 128 (weights) values, the scales written straight into the
// packed int16 MN-major layout the GEMMs read (the pages' scale-factor section, "Fatores de
// escala FP8 e o formato UE8M0" on the crazystack page: a power-of-two scale per block chosen
// so the block fits the FP8 range, stored as UE8M0 and packed in pairs along K).
//
// Per block: e = the smallest integer with 448 * 2^e >= max |x| (0 for an all-zero block),
// clamped to [-126, 127]; the UE8M0 byte is e + 127; each value becomes x * 2^-e (exact: a
// power of two) rounded to the nearest E4M3 value, ties to even, by the cvt.rn.satfinite
// instruction.  Packed word j of scale row s holds blocks 2j (low byte) and 2j + 1; words of
// scale rows past the last one, and the high byte past an odd block count, are 0.
//
// The kernel streams its input once (HBM-bound), B200 style: a persistent grid of one
// 16- or 32-warp CTA per SM walks 128-row x 512-byte tiles (128 x 128 fp32 or 128 x 256 bf16) through
// a 3-stage TMA ring in shared memory (192 KB in flight per SM), so loads for the next tiles
// are always outstanding while the current one is reduced and converted.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "ptx.cuh"

namespace bsp {

// Smallest e with 448 * 2^e >= amax for a finite amax >= 0 given as its fp32 bit pattern (0 when
// amax == 0), clamped to the UE8M0 range [-126, 127].  With amax = (1 + m / 2^23) * 2^E and
// 448 = 1.75 * 2^8, e is E - 8 when the significand is at most 1.75 (m <= 0x600000) and E - 7
// above; a subnormal amax lies below 448 * 2^-127 and takes the floor -126.
__device__ __forceinline__ int e4m3_block_exponent(uint32_t amax_bits) {
    if (amax_bits == 0u) return 0;
    const int biased = (int)(amax_bits >> 23);
    if (biased == 0) return -126;
    const int e = (biased - 127) - 8 + ((amax_bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return e < -126 ? -126 : (e > 127 ? 127 : e);
}

// 2^-e as an fp32 value, exact for e in [-126, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2_neg(int e) {
    return e == 127 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - e) << 23);
}

// Two fp32 values to two E4M3 codes, `lo` in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

template <bool BF16_>
struct QuantCfg {
    static constexpr bool BF16 = BF16_;
    static constexpr int ES = BF16 ? 2 : 4;
    static constexpr int TR = 128;                  // tile rows (one 128-row scale block)
    static constexpr int TC = 512 / ES;             // tile columns: 512 bytes per row
    static constexpr int KBT = TC / 128;            // K blocks per tile: 2 (bf16) or 1 (fp32)
    static constexpr int VPL = TC / 32;             // values per lane per row: 8 or 4 (16 bytes)
    static constexpr int LANES_PER_BLOCK = 128 / VPL;  // 16 or 32
    static constexpr int TILE_BYTES = TR * 512;     // 64 KB
    static constexpr int STAGES = 3;
    // fp32 tiles run 32 warps of 4 rows (measured 73 -> 65 us on [4096 x 16384]: more warps hide
    // the conversion's dependent latencies); bf16 tiles, with twice the values per lane, 16 of 8
    static constexpr int WARPS = BF16 ? 16 : 32;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int ROWS_PER_WARP = TR / WARPS;  // 8 or 4
    static constexpr int SMEM_BYTES = STAGES * TILE_BYTES + 128 + 1024;  // + barriers + alignment slack
};

struct QuantArgs {
    int rows, kb_count, col_tiles, num_tiles, scale_rows, block_rows;
    int64_t ld_q, ld_sf;
    uint8_t* q;
    uint8_t* sf;  // int16 words [ceil(kb_count / 2)][ld_sf], addressed by byte
    int* status;
    unsigned long long timeout_ns;
};

// Bounded wait on a TMA stage; false (status latched) past the deadline.
__device__ __forceinline__ bool quant_wait(uint64_t* bar, uint32_t parity, const QuantArgs& a) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > a.timeout_ns) {
            atomicCAS(a.status, 0, -6);  // BSP_ERR_TIMEOUT
            return false;
        }
    }
    return true;
}

// Largest magnitude among this lane's 16 bytes of a row, as fp32 bits: magnitudes order like
// their bit patterns with the sign cleared (infinities and NaNs above every finite value).
template <class C>
__device__ __forceinline__ uint32_t quant_amax_bits(uint4 u) {
    if constexpr (C::BF16) {
        uint32_t m = __vmaxu2(__vmaxu2(u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu), __vmaxu2(u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu));
        return max(m >> 16, m & 0xFFFFu) << 16;
    } else {
        return max(max(u.x & 0x7FFFFFFFu, u.y & 0x7FFFFFFFu), max(u.z & 0x7FFFFFFFu, u.w & 0x7FFFFFFFu));
    }
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d, float s) {
    return cvt_e4m3x2(a * s, b * s) | (cvt_e4m3x2(c * s, d * s) << 16);
}

// This lane's codes of one row (its 16 input bytes scaled by `scale`), stored at dst.
template <class C>
__device__ __forceinline__ void quant_store_codes(uint8_t* dst, uint4 u, float s) {
    if constexpr (C::BF16) {
        const auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
        const auto hi = [](uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); };
        *reinterpret_cast<uint2*>(dst) = make_uint2(e4m3x4(lo(u.x), hi(u.x), lo(u.y), hi(u.y), s),
                                                    e4m3x4(lo(u.z), hi(u.z), lo(u.w), hi(u.w), s));
    } else {
        *reinterpret_cast<uint32_t*>(dst) =
            e4m3x4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w), s);
    }
}

// Maximum over this lane's K-block group of lanes (all 32 lanes for fp32 tiles, 16 for bf16).
template <class C>
__device__ __forceinline__ uint32_t quant_block_max(uint32_t m, int h) {
    if constexpr (C::LANES_PER_BLOCK == 32) {
        return __reduce_max_sync(0xffffffffu, m);
    } else {
        const uint32_t m0 = __reduce_max_sync(0xffffffffu, h == 0 ? m : 0u);
        const uint32_t m1 = __reduce_max_sync(0xffffffffu, h == 1 ? m : 0u);
        return h == 0 ? m0 : m1;
    }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    quantize_kernel(const __grid_constant__ CUtensorMap tm_x, const QuantArgs a) {
    extern __shared__ __align__(128) uint8_t qsmem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::TILE_BYTES);
    __shared__ uint32_t warp_max[C::WARPS][2];
    __shared__ int stop;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int words = (a.kb_count + 1) / 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
        tma_prefetch_desc(&tm_x);
        stop = 0;
    }
    // words of the scale rows past the last one are 0
    {
        const int64_t pad_rows = a.ld_sf - a.scale_rows, n = pad_rows * words;
        uint16_t* sf16 = reinterpret_cast<uint16_t*>(a.sf);
        for (int64_t i = blockIdx.x * (int64_t)C::THREADS + threadIdx.x; i < n; i += (int64_t)gridDim.x * C::THREADS)
            sf16[(i / pad_rows) * a.ld_sf + a.scale_rows + i % pad_rows] = 0;
    }
    __syncthreads();

    const auto tile_of = [&](int t, int* rb, int* ct) {
        *rb = t / a.col_tiles;
        *ct = t - *rb * a.col_tiles;
    };
    const auto issue = [&](int i) {  // load this CTA's i-th tile into stage i % STAGES
        const int t = blockIdx.x + i * gridDim.x;
        if (t >= a.num_tiles) return;
        int rb, ct;
        tile_of(t, &rb, &ct);
        const int s = i % C::STAGES;
        mbar_arrive_expect_tx(&full[s], C::TILE_BYTES);
        tma_load_2d(smem + s * C::TILE_BYTES, &tm_x, &full[s], ct * C::TC, rb * C::TR);
    };
    if (threadIdx.x == 0)
        for (int i = 0; i < C::STAGES; ++i) issue(i);

    // this lane's K block within the tile (bf16 tiles hold two) and its lanes' shuffle group
    const int h = lane / C::LANES_PER_BLOCK;
    bool finite = true;
    int i = 0;  // tiles of this CTA consumed so far
    for (;; ++i) {
        const int t = blockIdx.x + i * gridDim.x;
        if (t >= a.num_tiles) break;
        int rb, ct;
        tile_of(t, &rb, &ct);
        const int s = i % C::STAGES;
        if (!quant_wait(&full[s], (uint32_t)(i / C::STAGES) & 1u, a)) stop = 1;
        __syncthreads();
        if (stop) break;
        const uint8_t* tile = smem + s * C::TILE_BYTES;
        const int kb = ct * C::KBT + h;                 // this lane's K block
        const bool kb_ok = kb < a.kb_count;
        const int col = ct * C::TC + lane * C::VPL;     // this lane's first column
        // the UE8M0 byte of K block kb for scale row srow (and the zero high byte of an odd count)
        const auto store_scale = [&](int srow, int e) {
            uint8_t* p = a.sf + ((int64_t)(kb / 2) * a.ld_sf + srow) * 2 + (kb & 1);
            p[0] = (uint8_t)(e + 127);
            if ((a.kb_count & 1) && kb == a.kb_count - 1) p[1] = 0;
        };
        // all rows of this warp first: loads and lane maxima, then the reductions side by side
        constexpr int R = C::ROWS_PER_WARP;
        uint4 u[R];
        uint32_t m[R];
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
            u[rr] = *reinterpret_cast<const uint4*>(tile + (warp * R + rr) * 512 + lane * 16);
            m[rr] = quant_amax_bits<C>(u[rr]);
            finite = finite && m[rr] < 0x7F800000u;
        }
        const int row0 = rb * C::TR + warp * R;
        uint8_t* qrow = a.q + (int64_t)row0 * a.ld_q + col;
        if (a.block_rows == 1) {
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                const int e = e4m3_block_exponent(quant_block_max<C>(m[rr], h));
                if (row0 + rr < a.rows && kb_ok) {
                    quant_store_codes<C>(qrow + rr * a.ld_q, u[rr], pow2_neg(e));
                    if (lane % C::LANES_PER_BLOCK == 0) store_scale(row0 + rr, e);
                }
            }
        } else {
            uint32_t mm = m[0];
#pragma unroll
            for (int rr = 1; rr < R; ++rr) mm = max(mm, m[rr]);
            mm = quant_block_max<C>(mm, h);
            if (lane % C::LANES_PER_BLOCK == 0) warp_max[warp][h] = mm;
            __syncthreads();
            mm = warp_max[0][h];
#pragma unroll
            for (int w = 1; w < C::WARPS; ++w) mm = max(mm, warp_max[w][h]);
            const int e = e4m3_block_exponent(mm);
            const float scale = pow2_neg(e);
#pragma unroll
            for (int rr = 0; rr < R; ++rr)
                if (row0 + rr < a.rows && kb_ok) quant_store_codes<C>(qrow + rr * a.ld_q, u[rr], scale);
            if (warp == 0 && lane % C::LANES_PER_BLOCK == 0 && kb_ok) store_scale(rb, e);
        }
        __syncthreads();  // every thread is done with this stage (and with warp_max)
        if (threadIdx.x == 0) issue(i + C::STAGES);
    }
    if (!__all_sync(0xffffffffu, finite) && lane == 0) atomicCAS(a.status, 0, -7);  // BSP_ERR_DEVICE_CHECK
    // wind down after a timeout: the copies issued for tiles i .. i + STAGES - 1 (not consumed)
    // land before the CTA exits, each waited for with a fixed one-second bound
    if (stop && threadIdx.x == 0) {
        for (int k = i; k < i + C::STAGES && blockIdx.x + k * gridDim.x < a.num_tiles; ++k) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[k % C::STAGES], (uint32_t)(k / C::STAGES) & 1u) &&
                   globaltimer_ns() - t0 < 1000000000ull) {
            }
        }
    }
}

}  // namespace bsp
