// gemm.cuh — persistent, warp-specialised sm_100a GEMM D = A * B^T (NT) with optional
// UE8M0 block scales, for BF16, FP8 (E4M3) and FP4 (E2M1) inputs and the M-grouped
// (mixture-of-experts) layout.
//
// Pipeline (the pages' "operand reuse and pipelining" with staged buffers and ready
// signals, "DeepGEMM-Ascend cobre quantas operações no Ascend 950?", section "Reúso de
// operandos e pipelining na prática", rebuilt for Blackwell):
//   warp 0      TMA producer: A/B tiles (128-byte swizzle) and the packed int16 scale
//               words of each K step into an S-stage shared-memory ring; "full" mbarrier
//               per stage (transaction-counted).
//   warp 1      owns tensor memory (TMEM); per stage it rewrites the MN-major scale
//               words into the 32-row x 16-byte layout the scale copy expects, copies
//               them into TMEM (tcgen05.cp) and issues the tcgen05.mma instructions
//               (one elected lane), then commits to the stage's "empty" mbarrier.
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator (double-buffered in TMEM so
//               the next tile's MMAs overlap), round to bf16, store to D.
// Tiles: 128 x BLOCK_N output tiles, one CTA per SM walking tiles in a grouped raster.
// Every wait is bounded: past the deadline the CTA latches BSP_ERR_TIMEOUT in the status
// word, raises a shared abort flag, drains its own in-flight copies and MMAs, frees TMEM
// and returns.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace bsp {

enum class Kind : int { BF16 = 0, FP8 = 1, FP4 = 2 };

constexpr int kStatusTimeout = -6;      // BSP_ERR_TIMEOUT
constexpr int kStatusDeviceCheck = -7;  // BSP_ERR_DEVICE_CHECK

struct GemmArgs {
    int M, N, K;
    int num_kb;    // K steps of 128 bytes per row
    int m_blocks;  // ceil(M / 128)
    int n_blocks;  // ceil(N / BLOCK_N)
    int num_tiles;
    int group_m;   // raster: m-blocks per group
    __nv_bfloat16* D;
    int64_t ldd;
    const int32_t* m_indices;  // grouped layout only
    int G;
    int sfb_gran;              // 1 or 128 (FP8); 1 for FP4
    int* status;
    unsigned long long timeout_ns;
};

template <Kind KIND, int BLOCK_N_, int STAGES_, bool GROUPED_>
struct GemmCfg {
    static constexpr Kind kind = KIND;
    static constexpr int BM = 128;
    static constexpr int BN = BLOCK_N_;
    static constexpr int STAGES = STAGES_;
    static constexpr bool GROUPED = GROUPED_;
    static constexpr bool SCALED = KIND != Kind::BF16;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BLOCK_N");

    // One K step = one 128-byte swizzle row per operand row: 64 bf16, 128 E4M3, 256 E2M1.
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    // int16 scale words per row per K step: FP8 one (the word covers two 128-K blocks,
    // the step uses one byte of it); FP4 four (8 blocks of 32 K).
    static constexpr int SF_WORDS = KIND == Kind::FP4 ? 4 : 1;
    // 32-bit TMEM scale words per row per K step.
    static constexpr int UT_WORDS = KIND == Kind::FP4 ? 2 : 1;
    static constexpr int SFB_ATOMS = (BN + 127) / 128;
    static constexpr int SFA_RAW = SCALED ? ((BM * SF_WORDS * 2 + 127) / 128) * 128 : 0;
    static constexpr int SFB_RAW = SCALED ? (((BN > 16 ? BN : 16) * SF_WORDS * 2 + 127) / 128) * 128 : 0;
    static constexpr int UTA_BYTES = SCALED ? UT_WORDS * 512 : 0;
    static constexpr int UTB_BYTES = SCALED ? UT_WORDS * SFB_ATOMS * 512 : 0;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_RAW + SFB_RAW + UTA_BYTES + UTB_BYTES;

    // Tensor memory: two fp32 accumulators of BN columns, then rotating scale slots.
    static constexpr int TMEM_COLS = 512;
    static constexpr int ACC_COLS = 2 * BN;
    static constexpr int SFA_COLS = UT_WORDS * 4;
    static constexpr int SFB_COLS = UT_WORDS * SFB_ATOMS * 4;
    static constexpr int SF_SLOT_COLS = SFA_COLS + SFB_COLS;
    static constexpr int SF_SLOTS_FIT = SCALED ? (TMEM_COLS - ACC_COLS) / SF_SLOT_COLS : 1;
    static constexpr int SF_SLOTS = SF_SLOTS_FIT > 4 ? 4 : SF_SLOTS_FIT;
    static_assert(!SCALED || SF_SLOTS >= 1, "tensor memory too small for the scale slots");

    // Shared memory map (offsets from a 1024-byte aligned base).
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_RAW;
    static constexpr int OFF_UTA = OFF_SFB + STAGES * SFB_RAW;
    static constexpr int OFF_UTB = OFF_UTA + STAGES * UTA_BYTES;
    static constexpr int OFF_BAR = ((OFF_UTB + STAGES * UTB_BYTES + 7) / 8) * 8;
    static constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
    static_assert(B_BYTES % 1024 == 0, "B tile must keep 1024-byte alignment");

    static constexpr int THREADS = 192;
};

struct Tile {
    int m_blk, n_blk;
};

__device__ __forceinline__ Tile tile_of(const GemmArgs& a, int t) {
    const int per_group = a.group_m * a.n_blocks;
    const int grp = t / per_group;
    const int first_m = grp * a.group_m;
    const int rows = min(a.group_m, a.m_blocks - first_m);
    const int local = t - grp * per_group;
    return Tile{first_m + local % rows, local / rows};
}

__device__ __forceinline__ void latch_status(int* status, int code) {
    atomicCAS(status, 0, code);
}

// Bounded wait on a phase of `bar`.  False if the deadline passed (status latched and
// abort raised) or another role already aborted.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, const GemmArgs& a,
                                             volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    // try_wait itself suspends for a while before reporting "not yet", so the deadline and
    // the abort flag are checked after every failed try.
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > a.timeout_ns) {
            latch_status(a.status, kStatusTimeout);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// Bounded wait used while winding down: ignores the abort flag and uses its own fixed
// one-second limit, so that even a very short pipeline timeout never lets the CTA exit
// before its own copies and MMAs (which finish in microseconds) have landed.
constexpr unsigned long long kDrainTimeoutNs = 1000000000ull;

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, const GemmArgs& a) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kDrainTimeoutNs) {
            latch_status(a.status, kStatusTimeout);
            return;
        }
    }
}

// Whole-warp wait: every lane waits, and the outcome is voted so the warp stays converged
// (a lane that timed out takes all lanes with it).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const GemmArgs& a,
                                          volatile int* abort_flag) {
    const bool ok = bounded_wait(bar, parity, a, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                const GemmArgs args) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::STAGES;
    uint64_t* tmem_full = bars + 2 * C::STAGES;
    uint64_t* tmem_empty = bars + 2 * C::STAGES + 2;
    uint64_t* drain = bars + 2 * C::STAGES + 4;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x / 32;
    const uint32_t lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&tmem_empty[b], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        if constexpr (C::SCALED) {
            tma_prefetch_desc(&tm_sfa);
            tma_prefetch_desc(&tm_sfb);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
                const Tile tl = tile_of(args, t);
                const int m0 = tl.m_blk * C::BM;
                const int n0 = tl.n_blk * C::BN;
                int g = 0;
                if constexpr (C::GROUPED) {
                    g = __ldg(args.m_indices + m0);
                    if (g < 0 || g >= args.G) {
                        latch_status(args.status, kStatusDeviceCheck);
                        g = 0;
                    }
                }
                for (int kb = 0; kb < args.num_kb; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!bounded_wait(&empty[s], ph ^ 1u, args, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint32_t bytes = C::A_BYTES + C::B_BYTES;
                    if constexpr (C::SCALED)
                        bytes += C::BM * C::SF_WORDS * 2 +
                                 (args.sfb_gran == 1 ? C::BN * C::SF_WORDS * 2 : 16 * 2);
                    mbar_arrive_expect_tx(&full[s], bytes);
                    uint8_t* sa = smem + C::OFF_A + s * C::A_BYTES;
                    uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
                    // x coordinate in elements of the tensor map's type: 64 bf16 or 128 bytes per step
                    const int kx = kb * (C::kind == Kind::BF16 ? 64 : 128);
                    tma_load_2d(sa, &tm_a, &full[s], kx, m0);
                    if constexpr (C::GROUPED)
                        tma_load_3d(sb, &tm_b, &full[s], kx, n0, g);
                    else
                        tma_load_2d(sb, &tm_b, &full[s], kx, n0);
                    if constexpr (C::SCALED) {
                        // word row of this step: FP8 uses word kb/2 (byte kb%2); FP4 words 4kb..4kb+3
                        const int wy = C::kind == Kind::FP4 ? kb * 4 : kb / 2;
                        uint8_t* rsa = smem + C::OFF_SFA + s * C::SFA_RAW;
                        uint8_t* rsb = smem + C::OFF_SFB + s * C::SFB_RAW;
                        tma_load_2d(rsa, &tm_sfa, &full[s], m0, wy);
                        const int bx = args.sfb_gran == 1 ? n0 : ((n0 / 128) & ~7);
                        if constexpr (C::GROUPED)
                            tma_load_3d(rsb, &tm_sfb, &full[s], bx, wy, g);
                        else
                            tma_load_2d(rsb, &tm_sfb, &full[s], bx, wy);
                    }
                }
            }
            // Wind down: wait (bounded) until the copies issued for the last stages landed.
            const uint32_t last = it < (uint32_t)C::STAGES ? it : (uint32_t)C::STAGES;
            for (uint32_t j = it - last; j < it; ++j) drain_wait(&full[j % C::STAGES], (j / C::STAGES) & 1u, args);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ scale staging + MMA
        uint32_t it = 0, lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x, ++lt) {
            const Tile tl = tile_of(args, t);
            const int n0 = tl.n_blk * C::BN;
            const uint32_t buf = lt & 1u;
            const uint32_t aph = (lt >> 1) & 1u;
            if (!warp_wait(&tmem_empty[buf], aph ^ 1u, args, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + buf * C::BN;
            for (int kb = 0; kb < args.num_kb; ++kb, ++it) {
                const int s = it % C::STAGES;
                const uint32_t ph = (it / C::STAGES) & 1u;
                if (!warp_wait(&full[s], ph, args, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t slot = it % C::SF_SLOTS;
                const uint32_t sfa_col = C::ACC_COLS + slot * C::SF_SLOT_COLS;
                const uint32_t sfb_col = sfa_col + C::SFA_COLS;
                if constexpr (C::SCALED) {
                    // MN-major int16 words -> rows of 16 bytes: row l holds the 32-bit words of
                    // matrix rows l, l+32, l+64, l+96 (the layout the 32x128b scale copy reads).
                    const uint16_t* rsa = reinterpret_cast<const uint16_t*>(smem + C::OFF_SFA + s * C::SFA_RAW);
                    const uint16_t* rsb = reinterpret_cast<const uint16_t*>(smem + C::OFF_SFB + s * C::SFB_RAW);
                    uint4* uta = reinterpret_cast<uint4*>(smem + C::OFF_UTA + s * C::UTA_BYTES);
                    uint4* utb = reinterpret_cast<uint4*>(smem + C::OFF_UTB + s * C::UTB_BYTES);
                    if constexpr (C::kind == Kind::FP8) {
                        uta[lane] = make_uint4(rsa[lane], rsa[lane + 32], rsa[lane + 64], rsa[lane + 96]);
                        const int x0 = (n0 / 128) & ~7;
#pragma unroll
                        for (int at = 0; at < C::SFB_ATOMS; ++at) {
                            uint32_t w[4];
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int r = at * 128 + c * 32 + (int)lane;
                                uint32_t v = 0;
                                if (r < C::BN) v = args.sfb_gran == 1 ? rsb[r] : rsb[(n0 + r) / 128 - x0];
                                w[c] = v;
                            }
                            utb[at * 32 + lane] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    } else {  // FP4: word u of a row packs int16 words 2u (low half) and 2u+1
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            uint32_t w[4];
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int r = c * 32 + (int)lane;
                                w[c] = (uint32_t)rsa[(2 * u) * C::BM + r] | ((uint32_t)rsa[(2 * u + 1) * C::BM + r] << 16);
                            }
                            uta[u * 32 + lane] = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
                            for (int at = 0; at < C::SFB_ATOMS; ++at) {
#pragma unroll
                                for (int c = 0; c < 4; ++c) {
                                    const int r = at * 128 + c * 32 + (int)lane;
                                    w[c] = r < C::BN ? ((uint32_t)rsb[(2 * u) * C::BN + r] |
                                                        ((uint32_t)rsb[(2 * u + 1) * C::BN + r] << 16))
                                                     : 0u;
                                }
                                utb[(u * C::SFB_ATOMS + at) * 32 + lane] = make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    const uint8_t* sa = smem + C::OFF_A + s * C::A_BYTES;
                    const uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
                    const uint64_t adesc = smem_desc_k_sw128(sa);
                    const uint64_t bdesc = smem_desc_k_sw128(sb);
                    if constexpr (C::SCALED) {
                        const uint8_t* uta = smem + C::OFF_UTA + s * C::UTA_BYTES;
                        const uint8_t* utb = smem + C::OFF_UTB + s * C::UTB_BYTES;
#pragma unroll
                        for (int u = 0; u < C::UT_WORDS; ++u) {
                            tc_cp_32x128b_warpx4(tmem_base + sfa_col + 4 * u, smem_desc_rows16(uta + u * 512));
#pragma unroll
                            for (int at = 0; at < C::SFB_ATOMS; ++at)
                                tc_cp_32x128b_warpx4(tmem_base + sfb_col + 4 * (u * C::SFB_ATOMS + at),
                                                     smem_desc_rows16(utb + (u * C::SFB_ATOMS + at) * 512));
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        // 32 bytes of K per MMA: 16 bf16, 32 E4M3, 64 E2M1
                        const uint64_t ad = adesc + (uint64_t)(2 * i);
                        const uint64_t bd = bdesc + (uint64_t)(2 * i);
                        const uint32_t acc = (kb > 0 || i > 0) ? 1u : 0u;
                        if constexpr (C::kind == Kind::BF16) {
                            tc_mma_f16(d_tmem, ad, bd, idesc_bf16(C::BM, C::BN), acc);
                        } else if constexpr (C::kind == Kind::FP8) {
                            const uint32_t id = (uint32_t)(kb & 1);
                            tc_mma_mxf8(d_tmem, ad, bd, idesc_block_scaled(C::BM, C::BN, 0u, id, id),
                                        tmem_base + sfa_col, tmem_base + sfb_col, acc);
                        } else {
                            const uint32_t u = (uint32_t)(i >> 1), id = (uint32_t)((i & 1) * 2);
                            tc_mma_mxf4(d_tmem, ad, bd, idesc_block_scaled(C::BM, C::BN, 1u, id, id),
                                        tmem_base + sfa_col + 4 * u, tmem_base + sfb_col + 4 * C::SFB_ATOMS * u,
                                        acc);
                        }
                    }
                    tc_commit(&empty[s]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) tc_commit(&tmem_full[buf]);
            __syncwarp();
        }
        // Wind down: every MMA and scale copy this warp issued has completed.
        if (lane == 0) {
            tc_commit(drain);
            drain_wait(drain, 0, args);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const uint32_t quarter = warp % 4;  // TMEM lanes this warp may read
        uint32_t lt = 0;
        for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x, ++lt) {
            const Tile tl = tile_of(args, t);
            const int m0 = tl.m_blk * C::BM;
            const int n0 = tl.n_blk * C::BN;
            const uint32_t buf = lt & 1u;
            const uint32_t aph = (lt >> 1) & 1u;
            if (!warp_wait(&tmem_full[buf], aph, args, abort_flag)) break;
            tc_fence_after();
            const int row = m0 + (int)(quarter * 32 + lane);
            bool zero_row = false;
            if constexpr (C::GROUPED) {
                if (row < args.M) {
                    const int g0 = __ldg(args.m_indices + m0);
                    const int gi = __ldg(args.m_indices + row);
                    zero_row = gi < 0;
                    if (gi != g0 && gi != -1) latch_status(args.status, kStatusDeviceCheck);
                }
            }
            __nv_bfloat16* drow = args.D + (int64_t)row * args.ldd;
            const uint32_t taddr = tmem_base + ((quarter * 32) << 16) + buf * C::BN;
#pragma unroll 1
            for (int c = 0; c < C::BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(taddr + c * 32, r);
                tmem_ld_wait();
                if (c == C::BN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tmem_empty[buf]);
                }
                if (row >= args.M) continue;
                const int col0 = n0 + c * 32;
                uint32_t packed[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    __nv_bfloat162 h = __float22bfloat162_rn(
                        make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])));
                    packed[j] = zero_row ? 0u : *reinterpret_cast<uint32_t*>(&h);
                }
                if (col0 + 32 <= args.N) {
                    uint4* dst = reinterpret_cast<uint4*>(drow + col0);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                } else {
                    const uint16_t* p16 = reinterpret_cast<const uint16_t*>(packed);
                    uint16_t* d16 = reinterpret_cast<uint16_t*>(drow);
                    for (int j = 0; j < 32 && col0 + j < args.N; ++j) d16[col0 + j] = p16[j];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace bsp
