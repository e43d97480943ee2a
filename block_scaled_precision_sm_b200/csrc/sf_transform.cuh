// sf_transform.cuh — UE8M0 scale factors [mn][kb] -> int16 words [ceil(kb/2)][ld_out],
// word(j, r) = e[r][2j] | e[r][2j+1] << 8, MN-major ("DeepSeek lanza kernels de DeepGEMM
// para Huawei Ascend 950", section "Qué incluye el lanzamiento": each pair of UE8M0
// factors along K in one 16-bit integer, MN-major).
//
// One CTA transposes a 64-row x 64-block tile through shared memory: the reads run along
// K (the input's contiguous axis), the writes along MN (the output's contiguous axis),
// so both sides are coalesced.  The transform moves a few bytes per scale and is bound
// by DRAM bandwidth.
#pragma once

#include <cstdint>

namespace bsp {

constexpr int kSfTileMN = 64;
constexpr int kSfTileKB = 64;

// IN_KIND 0: fp32 power-of-two scales (UE8M0 byte = biased fp32 exponent);
// IN_KIND 1: uint8 UE8M0 bytes.
template <int IN_KIND>
__global__ void __launch_bounds__(256) sf_transform_kernel(const void* __restrict__ in, int mn, int kb,
                                                           int64_t ld_in, uint16_t* __restrict__ out,
                                                           int64_t ld_out, int* status) {
    __shared__ uint8_t e[kSfTileMN][kSfTileKB + 4];
    const int r0 = blockIdx.x * kSfTileMN;
    const int k0 = blockIdx.y * kSfTileKB;
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
    bool bad = false;
#pragma unroll
    for (int i = ty; i < kSfTileMN; i += 8) {
        const int r = r0 + i;
#pragma unroll
        for (int j = tx; j < kSfTileKB; j += 32) {
            const int k = k0 + j;
            uint32_t v = 0;
            if (r < mn && k < kb) {
                if constexpr (IN_KIND == 0) {
                    const uint32_t bits = __float_as_uint(__ldg(static_cast<const float*>(in) + (int64_t)r * ld_in + k));
                    v = (bits >> 23) & 0xFFu;
                    // exact positive normal power of two: sign 0, mantissa 0, exponent 1..254
                    bad |= (bits & 0x807FFFFFu) != 0u || v == 0u || v == 255u;
                } else {
                    v = __ldg(static_cast<const uint8_t*>(in) + (int64_t)r * ld_in + k);
                }
            }
            e[i][j] = static_cast<uint8_t>(v);
        }
    }
    __syncthreads();
    const int words = (kb + 1) / 2;
#pragma unroll
    for (int w = ty; w < kSfTileKB / 2; w += 8) {
        const int jw = k0 / 2 + w;
        if (jw >= words) break;
#pragma unroll
        for (int i = tx; i < kSfTileMN; i += 32) {
            const int r = r0 + i;
            if (r < ld_out)
                out[(int64_t)jw * ld_out + r] =
                    static_cast<uint16_t>(e[i][2 * w] | (static_cast<uint32_t>(e[i][2 * w + 1]) << 8));
        }
    }
    if (IN_KIND == 0 && __any_sync(0xffffffffu, bad) && tx == 0) atomicCAS(status, 0, -7);
}

}  // namespace bsp
