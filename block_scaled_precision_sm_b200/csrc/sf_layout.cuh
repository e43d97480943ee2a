// sf_layout.cuh — the packed int16 scale words rewritten into the layout the tensor cores'
// scale copy (tcgen05.cp 32x128b, replicated to the four lane quarters) reads, one chunk per
// (scale group, row tile), so the GEMM moves each chunk with a single TMA load and never
// rearranges scales on chip.
//
// Output: 32-bit words [G][Q][T][ATOMS][UT][32][4].  For a row tile t of R rows (R = 128 for
// A, the GEMM's BLOCK_N for B) atom `at` covers tile rows 128at..128at+127; lane l, column c
// of the atom holds the word of tile row 128at + 32c + l.  Word (q, u) of a row packs the
// int16 words j = 2(q*UT + u) (low half) and j + 1 (high half), i.e. four consecutive UE8M0
// K blocks, the lowest in the low byte.  Rows outside the tile or past `rows`, and words past
// `words`, are 0.  With `gran` = 128 each scale row is shared by 128 matrix rows.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace bsp {

struct SfLayout {
    int rows;        // matrix rows covered (N for 128-row B blocks, not N/128)
    int gran;        // matrix rows per scale row (1 or 128)
    int words;       // int16 words per scale row in the input
    int64_t ld;      // input leading dimension (int16 elements)
    int64_t gstride; // input elements between groups
    int tile_rows;   // R
    int atoms;       // ceil(R / 128)
    int ut;          // 32-bit words per row per scale group
    int tiles;       // T
    int q;           // Q scale groups along K
    int groups;      // G
};

__host__ __device__ inline int64_t sf_layout_words(const SfLayout& p) {
    return (int64_t)p.q * p.tiles * p.atoms * p.ut * 128 * p.groups;
}

__device__ __forceinline__ void sf_layout_word(const uint16_t* __restrict__ in, const SfLayout& p,
                                               uint32_t* __restrict__ out, int64_t idx) {
    {
        const int c = (int)(idx & 3);
        const int l = (int)((idx >> 2) & 31);
        int64_t rest = idx >> 7;
        const int u = (int)(rest % p.ut);
        rest /= p.ut;
        const int at = (int)(rest % p.atoms);
        rest /= p.atoms;
        const int t = (int)(rest % p.tiles);
        rest /= p.tiles;
        const int qq = (int)(rest % p.q);
        const int g = (int)(rest / p.q);
        const int in_tile = 128 * at + 32 * c + l;
        const int r = t * p.tile_rows + in_tile;
        uint32_t v = 0;
        if (in_tile < p.tile_rows && r < p.rows) {
            const uint16_t* src = in + (int64_t)g * p.gstride + r / p.gran;
            const int j = 2 * (qq * p.ut + u);
            const uint32_t lo = j < p.words ? __ldg(src + (int64_t)j * p.ld) : 0u;
            const uint32_t hi = j + 1 < p.words ? __ldg(src + (int64_t)(j + 1) * p.ld) : 0u;
            v = lo | (hi << 16);
        }
        out[idx] = v;
    }
}

// Both operands' chunks in one launch: words [0, total_a) of A, then those of B, then
// `zero_vecs` 16-byte zeros at `zero` (the GEMM's split-tail counters and workspace).
__global__ void __launch_bounds__(256) sf_tmem_layout_kernel(const uint16_t* __restrict__ in_a, SfLayout pa,
                                                             uint32_t* __restrict__ out_a,
                                                             const uint16_t* __restrict__ in_b, SfLayout pb,
                                                             uint32_t* __restrict__ out_b, uint4* __restrict__ zero,
                                                             int64_t zero_vecs) {
    // Launched with programmatic stream serialisation: wait for the kernel before this one (the
    // scale transforms, typically), then let the GEMM that follows start its set-up and operand
    // loads; it waits for this kernel's writes before it reads them.  Triggering only after the
    // wait means the GEMM starts after every kernel ahead of this one has completed.
    griddep_wait();
    griddep_launch_dependents();
    const int64_t na = sf_layout_words(pa), nab = na + sf_layout_words(pb), total = nab + zero_vecs;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        if (idx < na)
            sf_layout_word(in_a, pa, out_a, idx);
        else if (idx < nab)
            sf_layout_word(in_b, pb, out_b, idx - na);
        else
            zero[idx - nab] = make_uint4(0u, 0u, 0u, 0u);
    }
}

}  // namespace bsp
