// gemm.cuh — persistent, warp-specialised sm_100a GEMM D = A * B^T (NT) with optional
// UE8M0 block scales, for BF16, FP8 (E4M3) and FP4 (E2M1) inputs and the M-grouped
// (mixture-of-experts) layout.
//
// Pipeline (the pages' "operand reuse and pipelining" with staged buffers and ready
// signals, "DeepGEMM-Ascend cobre quantas operações no Ascend 950?", section "Reúso de
// operandos e pipelining na prática", rebuilt for Blackwell):
//   warp 0      TMA producer: A/B tiles (128-byte swizzle) into an S-stage shared-memory
//               ring ("full"/"empty" mbarriers, transaction-counted); the first stage of every
//               scale group (SF_PERIOD K steps) also carries one chunk of scale words per
//               operand, laid out beforehand (sf_layout.cuh) exactly as the scale copy reads
//               them, so no thread rearranges scales on chip.
//   warp 1      owns TMEM; in the MMA-issuing CTA one lane waits on the stage barriers and
//               issues tcgen05.cp of each scale chunk into a rotating TMEM slot and the
//               tcgen05.mma instructions, committing each stage to its "empty" barrier.
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator, round to bf16, stage 32 x 32
//               blocks in a swizzled shared-memory buffer (two per warp) and TMA-store them to
//               D.  With two accumulators in TMEM the next tile's MMAs overlap the epilogue;
//               with one (256-column tiles, whose two accumulators would leave no TMEM for
//               the scales) the epilogue first drains the whole accumulator into registers.
//
// Work items: the persistent workers walk the tiles in raster order; when the last wave would
// leave most workers idle its tiles are cut along K into slices whose fp32 partial sums are
// added in slot order (deterministic) by the slices themselves, without any slice waiting on
// another that may not be resident.  The masked grouped layout
// builds its tile list on the device from the per-expert counts.  TRANS_D configurations
// compute D^T = B A^T for small M and write the result transposed.
//
// PAIR = true: a cluster of two CTAs computes a 256 x BN tile with cta_group::2 MMAs.  CTA r
// loads A rows [128r, 128r+128) and B rows [r*BN/2, (r+1)*BN/2) of the tile into its own
// shared memory (each SM streams half of B: operand reuse across the pair without
// multicast) plus its own scale chunks (its 128 A rows, all BN B rows), the leader CTA
// (rank 0) issues the MMAs and the scale copies, and the accumulator rows of CTA r land in
// its own TMEM.  All loads signal the leader's barriers; the leader's commits are multicast
// to both CTAs' barriers; the peer's epilogue arrives on the leader's barrier remotely.
//
// FP8 scales are one byte per (row, 128 K): a scale group of four K steps is one 32-bit word
// per row and the MMA of K step kb selects byte kb % 4.  FP4 scales are one byte per (row,
// 32 K): a group is one K step of 256, two words per row, and an MMA (K = 64) selects a byte
// pair.
//
// Every wait is bounded: past the deadline the CTA latches BSP_ERR_TIMEOUT in the status
// word, raises a shared abort flag, drains its own in-flight copies and MMAs, frees TMEM and
// returns.
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
    int m_blocks;  // ceil(M / tile rows)
    int n_blocks;  // ceil(N / BLOCK_N)
    int num_tiles;
    int group_m;   // raster: m-blocks per group
    __nv_bfloat16* D;
    int64_t ldd;
    const int32_t* m_indices;  // grouped layout only
    int G;
    int sfb_gran;              // 1 or 128 (FP8); 1 for FP4
    int sfa_gran;              // A-operand scale rows per matrix row block (0 or 1: per row)
    int* status;
    unsigned long long timeout_ns;
    // Split tail: the first full_tiles tiles (in raster order) are computed whole, one per
    // work item; each remaining tile is cut into `splits` slices along K.  Slice j stores its
    // fp32 partial sums in its own workspace slot (ws: [split tiles][splits][TILE_M][BN]) and
    // counts itself in tail_count ([split tiles][CTAs][4 epilogue warps], zero on entry); the
    // rows of each epilogue warp are cut into `splits` shares, each claimed once through
    // tail_claim ([split tiles][CTAs][4][splits], zero on entry) and summed over all slots in
    // slot order before the bf16 rounding.  The fixed order keeps the result identical from
    // run to run, whichever slice reduces a share.
    int full_tiles;
    int splits;
    int num_work;  // full_tiles + (num_tiles - full_tiles) * splits
    float* ws;
    int* tail_count;
    int* tail_claim;
    const int32_t* masked_m;  // masked layout: valid rows per expert [G]
    int max_m;                // masked layout: rows per expert slab
};

template <Kind KIND, int BLOCK_N_, int STAGES_, bool GROUPED_, bool PAIR_, int ACC_BUFS_ = 2, bool MASKED_ = false,
          bool TRANS_D_ = false, bool CSPLIT_ = false>
struct GemmCfg {
    static constexpr Kind kind = KIND;
    static constexpr bool PAIR = PAIR_;
    static constexpr int CTAS = PAIR ? 2 : 1;
    static constexpr int BM = 128;              // A / D rows per CTA
    static constexpr int TILE_M = BM * CTAS;    // rows per tile
    static constexpr int BN = BLOCK_N_;         // columns per tile
    static constexpr int BN_CTA = BN / CTAS;    // B rows loaded per CTA
    static constexpr int STAGES = STAGES_;
    static constexpr bool GROUPED = GROUPED_;
    // masked grouped layout: expert g owns rows [g*max_m, (g+1)*max_m) of A and D, of which
    // the first masked_m[g] (a device array) are computed; the tile list is built on the device
    static constexpr bool MASKED = MASKED_;
    static constexpr int MAX_MASKED_G = 1024;
    static_assert(!MASKED || (GROUPED && (!PAIR_ || TRANS_D_)), "masked layout: single CTAs, or transposed pairs");
    // contiguous grouped layout on CTA pairs: a pair tile is one or two consecutive 128-row blocks
    // of one expert (an expert's odd last block alone, its peer CTA's rows then not stored); the
    // list of pair tiles is built on the device at kernel start from the blocks' expert indices
    static constexpr bool PAIR_LIST = GROUPED && PAIR_ && !MASKED;
    static constexpr int MAX_PAIR_TILES = 2048;
    // the kernel computes D^T = B' A'^T with the caller's operands swapped (A' = B, B' = A) and
    // writes each accumulator element (row i, column j) to D[j][i]: small-M problems put the
    // long N dimension on the 256-row pair tiles
    static constexpr bool TRANS_D = TRANS_D_;
    static_assert(!TRANS_D || !GROUPED || MASKED, "transposed output: dense or masked configs only");
    // masked layout, transposed: per expert, D_g^T = B_g A_g^T on CTA-pair tiles of 256 rows of
    // B_g, the expert's rows of A (a chunk of up to BN of them) as the MMA's N, which is cut to
    // the chunk's valid rows (a multiple of 16) at run time; B_g is streamed once per chunk
    static constexpr bool MT = MASKED && TRANS_D;
    static_assert(!MT || (PAIR_ && ACC_BUFS_ == 1 && BLOCK_N_ == 256 && KIND == Kind::FP8), "masked transposed");
    static constexpr int MCHUNK = MT ? BN : BM;  // rows of an expert per masked work item
    // a tile's two K halves on the two CTA pairs of one 4-CTA cluster: pair 1 hands its fp32 sums
    // to pair 0 through distributed shared memory (one tile per cluster, transposed output)
    static constexpr bool CSPLIT = CSPLIT_;
    static_assert(!CSPLIT || (PAIR_ && TRANS_D_ && ACC_BUFS_ == 2 && BLOCK_N_ == 128), "cluster split");
    static constexpr int CLUSTER = CSPLIT ? 4 : (PAIR_ ? 2 : 1);  // CTAs per cluster
    static constexpr bool SCALED = KIND != Kind::BF16;
    // TMEM accumulators: two let the next tile's MMAs run under this tile's epilogue; with one,
    // the epilogue reads the whole accumulator into registers first and releases it at once
    static constexpr int ACC_BUFS = ACC_BUFS_;
    static_assert(ACC_BUFS == 1 || ACC_BUFS == 2, "accumulator buffers");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256 && BN_CTA % 8 == 0, "BLOCK_N");

    // One K step = one 128-byte swizzle row per operand row: 64 bf16, 128 E4M3, 256 E2M1.
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN_CTA * 128;
    static_assert(B_BYTES % 1024 == 0, "B tile must keep 1024-byte alignment");

    // Scale groups: every SF_PERIOD K steps, UT_WORDS 32-bit TMEM words per row; a chunk per
    // 128-row atom and word is 32 rows x 16 bytes.
    static constexpr int SF_PERIOD = KIND == Kind::FP8 ? 4 : 1;
    static constexpr int UT_WORDS = KIND == Kind::FP8 ? 1 : 2;
    static constexpr int SFB_ATOMS = (BN + 127) / 128;  // every CTA holds the scales of all BN rows
    static constexpr int SFA_CHUNK = SCALED ? UT_WORDS * 512 : 0;
    static constexpr int SFB_CHUNK = SCALED ? SFB_ATOMS * UT_WORDS * 512 : 0;
    static constexpr int SF_STAGE_BYTES = SFA_CHUNK + SFB_CHUNK;

    // Tensor memory: ACC_BUFS fp32 accumulators of BN columns, then rotating scale slots.
    // (Measured: loading the chunks of several groups at once into a separate two-slot ring and
    // copying them in one burst was slower for FP8 and FP4 than this: the ring limited how far
    // the loads could run ahead, and long bursts of copies stalled the MMAs.)
    static constexpr int TMEM_COLS = 512;
    static constexpr int ACC_COLS = ACC_BUFS * BN;
    static constexpr int SFA_COLS = UT_WORDS * 4;
    static constexpr int SFB_COLS = UT_WORDS * SFB_ATOMS * 4;
    static constexpr int SF_SLOT_COLS = SFA_COLS + SFB_COLS;
    static constexpr int SF_SLOTS_FIT = SCALED ? (TMEM_COLS - ACC_COLS) / SF_SLOT_COLS : 1;
    static constexpr int SF_SLOTS = SF_SLOTS_FIT > 4 ? 4 : SF_SLOTS_FIT;
    static_assert(!SCALED || SF_SLOTS >= 1, "tensor memory too small for the scale slots");

    // Shared memory map (offsets from a 1024-byte aligned base).
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SF = OFF_B + STAGES * B_BYTES;  // a scale chunk buffer per stage
    // epilogue staging: per epilogue warp two 32 x 32 bf16 blocks (64-byte swizzle)
    static constexpr int EPI_BLOCK = 32 * 32 * 2;
    static constexpr int OFF_EPI = ((OFF_SF + STAGES * SF_STAGE_BYTES + 1023) / 1024) * 1024;
    // full, empty [STAGES]; tmem_full, tmem_empty [2]; drain; per epilogue warp: split-tail
    // gather; cluster split, per epilogue warp: receive buffer free, columns received
    static constexpr int NUM_BARS = 2 * STAGES + 5 + 4 + (CSPLIT ? 8 : 0);
    // cluster split, per epilogue warp: the 32 x 64 fp32 columns sent and those received, then
    // its 64 x 32 bf16 block of D, in the idle A stage buffers
    static constexpr int X_COLS = BN / 2;
    static constexpr int X_BYTES = 32 * X_COLS * 4;
    static constexpr int X_WARP_BYTES = 2 * X_BYTES + X_COLS * 32 * 2;
    static_assert(!CSPLIT || 4 * X_WARP_BYTES <= STAGES * A_BYTES, "cluster-split buffers");
    static constexpr int OFF_BAR = OFF_EPI + 4 * 2 * EPI_BLOCK;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    // masked layout: valid m-blocks before each expert [G + 1] and the clamped counts [G]
    static constexpr int OFF_MASK = OFF_MISC + 16;
    static constexpr int MASK_BYTES = MASKED ? (2 * MAX_MASKED_G + 1) * 4 : 0;
    // pair-tile list of the contiguous grouped layout: [MAX_PAIR_TILES] entries, then the count
    static constexpr int OFF_LIST = OFF_MASK + MASK_BYTES;
    static constexpr int LIST_BYTES = PAIR_LIST ? (MAX_PAIR_TILES + 1) * 4 : 0;
    static_assert(!PAIR_LIST || MAX_PAIR_TILES * 4 <= STAGES * A_BYTES, "block expert scratch");
    static constexpr int SMEM_BYTES = OFF_LIST + LIST_BYTES + 1024;  // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
    // a K slice of a split tile is a worker's last work item, so its epilogue stages the
    // fp32 partial sums (BM x BN) in the then idle A/B stage buffers
    static_assert(BM * BN * 4 <= OFF_SF, "stage buffers too small for a split tile's partial sums");

    static constexpr int THREADS = 192;
};

struct Tile {
    int m_blk, n_blk;
};

// One work item: a tile and the K steps [kb0, kb1) it covers; `tail` >= 0 for a K slice of
// a split tile (its index among the split tiles).
struct Work {
    int tile, kb0, kb1, tail, slice;
};

// Slices are cut at scale-group boundaries (`period` K steps), as evenly as the groups allow.
__device__ __forceinline__ Work work_of(const GemmArgs& a, int w, int period) {
    if (w < a.full_tiles) return Work{w, 0, a.num_kb, -1, 0};
    const int u = w - a.full_tiles;
    const int tail = u / a.splits, j = u - tail * a.splits;
    const int groups = (a.num_kb + period - 1) / period;
    const int g0 = j * groups / a.splits, g1 = (j + 1) * groups / a.splits;
    return Work{a.full_tiles + tail, g0 * period, min(g1 * period, a.num_kb), tail, j};
}

// Cluster split: tile w, K half `half` (split at a scale-group boundary, as work_of cuts two slices).
__device__ __forceinline__ Work half_work(const GemmArgs& a, int w, int half, int period) {
    const int groups = (a.num_kb + period - 1) / period;
    const int mid = min(groups / 2 * period, a.num_kb);
    return half == 0 ? Work{w, 0, mid, -1, 0} : Work{w, mid, a.num_kb, -1, 1};
}

// Masked layout: work item w is n-block w % n_blocks of the (w / n_blocks)-th valid chunk of
// `chunk` rows, counting the valid chunks of expert 0 first; mprefix[g] holds the valid chunks
// before expert g.  Returns the chunk's first row (in the flattened [G * max_m] rows) and its
// expert.
template <int CHUNK>
__device__ __forceinline__ void masked_tile(const GemmArgs& a, const int* mprefix, int w, int* m0, int* n_blk,
                                            int* g) {
    const int mbi = w / a.n_blocks;
    *n_blk = w - mbi * a.n_blocks;
    int lo = 0, hi = a.G - 1;  // the expert whose blocks include mbi: smallest g with mprefix[g + 1] > mbi
    while (lo < hi) {
        const int mid = (lo + hi) / 2;
        if (mprefix[mid + 1] > mbi)
            hi = mid;
        else
            lo = mid + 1;
    }
    *g = lo;
    *m0 = lo * a.max_m + (mbi - mprefix[lo]) * CHUNK;
}

// Masked transposed tile: valid rows of the chunk at flattened row m0 of expert g, and the MMA's
// N for them (a multiple of 16, at most 256).
__device__ __forceinline__ int masked_rows(const GemmArgs& a, const int* mcount, int g, int m0) {
    return mcount[g] - (m0 - g * a.max_m);
}
__device__ __forceinline__ int masked_n(int rows) { return rows >= 256 ? 256 : (rows + 15) / 16 * 16; }

// Contiguous grouped layout on CTA pairs: the pair tiles, built by one warp of each CTA.  A
// block of 128 rows belongs to the expert of its first row (e[b] = m_indices[128 b]); a run of
// blocks of one expert is cut into pairs from its first block on, an odd last block forming a
// tile of its own.  Entry i of `list` is the tile's first block | (its block count << 24);
// list[max_tiles] is the count.  `e` is scratch for the blocks' experts (M / 128 ints).
__device__ __forceinline__ void build_pair_list(const GemmArgs& a, int* e, int* list, int max_tiles, uint32_t lane) {
    const int nb = a.M / 128;
    for (int b = (int)lane; b < nb; b += 32) e[b] = __ldg(a.m_indices + (int64_t)b * 128);
    __syncwarp();
    const int per = (nb + 31) / 32;
    const int c0 = min(nb, (int)lane * per), c1 = min(nb, c0 + per);
    const auto run_start = [&](int b) { return b == 0 || e[b] != e[b - 1]; };
    // the run start in effect where this lane's blocks begin: the last one of earlier lanes
    int last = -1;
    for (int b = c0; b < c1; ++b)
        if (run_start(b)) last = b;
    int incl = last;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if ((int)lane >= o) incl = max(incl, v);
    }
    int carry = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) carry = 0;
    // a block starts a tile when it lies an even number of blocks after its run's start
    int rs = carry, count = 0;
    for (int b = c0; b < c1; ++b) {
        if (run_start(b)) rs = b;
        count += ((b - rs) & 1) == 0;
    }
    int pos = count;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, pos, o);
        if ((int)lane >= o) pos += v;
    }
    const int total = __shfl_sync(0xffffffffu, pos, 31);
    pos -= count;
    rs = carry;
    for (int b = c0; b < c1; ++b) {
        if (run_start(b)) rs = b;
        if (((b - rs) & 1) == 0) {
            const int len = (b + 1 < nb && e[b + 1] == e[b]) ? 2 : 1;
            if (pos < max_tiles) list[pos] = b | (len << 24);
            ++pos;
        }
    }
    if (lane == 0) list[max_tiles] = min(total, max_tiles);
}

__device__ __forceinline__ void pair_tile(const GemmArgs& a, const int* list, int w, int* b0, int* len, int* n_blk) {
    const int i = w / a.n_blocks;
    *n_blk = w - i * a.n_blocks;
    *b0 = list[i] & 0xFFFFFF;
    *len = list[i] >> 24;
}

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
template <bool CLUSTER = false>
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, const GemmArgs& a,
                                             volatile int* abort_flag) {
    auto try_once = [&] { return CLUSTER ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
    if (try_once()) return true;
    // try_wait itself suspends for a while before reporting "not yet", so the deadline and
    // the abort flag are checked after every failed try.
    const uint64_t t0 = globaltimer_ns();
    while (!try_once()) {
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

// How long a slice of a split tile looks for the other slices of its tile to publish before it
// leaves the reduction of its share to the slice that publishes last.  The slices of a tile
// normally finish within a few microseconds of one another; one that is not resident (its SM
// held by another kernel) arrives later, and then reduces every open share itself.
constexpr unsigned long long kTailPollNs = 40000ull;

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
template <bool CLUSTER = false>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const GemmArgs& a,
                                          volatile int* abort_flag) {
    const bool ok = bounded_wait<CLUSTER>(bar, parity, a, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                const __grid_constant__ CUtensorMap tm_d, const __grid_constant__ CUtensorMap tm_ws,
                const GemmArgs args) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = full + C::STAGES;
    uint64_t* tmem_full = empty + C::STAGES;
    uint64_t* tmem_empty = tmem_full + 2;
    uint64_t* drain = tmem_empty + 2;
    uint64_t* gather = drain + 1;  // [4]: one per epilogue warp
    uint64_t* xready = gather + 4;  // [4] (cluster split): the other pair's receive buffer is free
    uint64_t* xfull = xready + 4;   // [4] (cluster split): the other pair's columns have arrived
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x / 32;
    const uint32_t lane = threadIdx.x % 32;
    const uint32_t crank = C::PAIR ? cluster_ctarank() : 0u;  // rank in the cluster
    const uint32_t rank = crank & 1u;                          // rank in the CTA pair
    const uint32_t pairbase = crank & ~1u;                     // cluster rank of the pair's leader
    const bool leader = rank == 0;
    const int worker = blockIdx.x / C::CLUSTER;
    const int workers = gridDim.x / C::CLUSTER;
    const uint16_t kPairMask = (uint16_t)(0x3u << pairbase);
    const int half = C::CSPLIT ? (int)(crank >> 1) : 0;  // cluster split: this pair's K half

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&tmem_empty[b], 4 * C::CTAS);
        }
        mbar_init(drain, 1);
        for (int w = 0; w < 4; ++w) mbar_init(&gather[w], 1);
        if constexpr (C::CSPLIT) {
            for (int w = 0; w < 4; ++w) {
                mbar_init(&xready[w], 1);
                mbar_init(&xfull[w], 1);
            }
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_d);
        if (args.splits > 1) tma_prefetch_desc(&tm_ws);
        if constexpr (C::SCALED) {
            tma_prefetch_desc(&tm_sfa);
            tma_prefetch_desc(&tm_sfb);
        }
    }
    if (warp == 1) {
        if constexpr (C::PAIR) {
            tmem_alloc_pair(tmem_base_slot, C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_base_slot, C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    int* mprefix = reinterpret_cast<int*>(smem + C::OFF_MASK);
    int* mcount = mprefix + C::MAX_MASKED_G + 1;
    if constexpr (C::MASKED) {
        // the tile list of the masked layout: valid row chunks per expert, prefix-summed by
        // one warp (each lane a run of experts, then an exclusive scan over the lanes)
        if (warp == 2) {
            const int G = args.G, per = (G + 31) / 32;
            const int i0 = min(G, (int)lane * per), i1 = min(G, i0 + per);
            int local = 0;
            for (int i = i0; i < i1; ++i) {
                int c = __ldg(args.masked_m + i);
                if (c < 0 || c > args.max_m) {
                    latch_status(args.status, kStatusDeviceCheck);
                    c = c < 0 ? 0 : args.max_m;
                }
                mcount[i] = c;
                local += (c + C::MCHUNK - 1) / C::MCHUNK;
            }
            int incl = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if ((int)lane >= o) incl += v;
            }
            int run = incl - local;
            for (int i = i0; i < i1; ++i) {
                mprefix[i] = run;
                run += (mcount[i] + C::MCHUNK - 1) / C::MCHUNK;
            }
            if (lane == 31) mprefix[G] = incl;
        }
    }
    int* plist = reinterpret_cast<int*>(smem + C::OFF_LIST);
    if constexpr (C::PAIR_LIST) {
        // the A stage buffers are idle until the setup barrier below: scratch for the blocks' experts
        if (warp == 2) build_pair_list(args, reinterpret_cast<int*>(smem + C::OFF_A), plist, C::MAX_PAIR_TILES, lane);
    }
    tc_fence_before();
    if constexpr (C::PAIR)
        cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;
    const int num_work = C::MASKED      ? mprefix[args.G] * args.n_blocks
                         : C::PAIR_LIST ? plist[C::MAX_PAIR_TILES] * args.n_blocks
                                        : args.num_work;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            bool prior_done = false;  // the scale chunks come from the kernel launched before
            // this CTA's rows of work item w: its K range, first A row, tile column and expert
            struct Item {
                Work wk;
                int m0, n_blk, g;
            };
            const auto item_of = [&](int w, bool check) {
                Item t{Work{0, 0, args.num_kb, -1, 0}, 0, 0, 0};
                if constexpr (C::MASKED) {
                    masked_tile<C::MCHUNK>(args, mprefix, w, &t.m0, &t.n_blk, &t.g);
                } else if constexpr (C::PAIR_LIST) {
                    int b0, len;
                    pair_tile(args, plist, w, &b0, &len, &t.n_blk);
                    t.m0 = (b0 + (int)rank) * C::BM;
                    t.g = __ldg(args.m_indices + (int64_t)b0 * C::BM);  // both CTAs multiply by this expert's B
                    if (t.g < 0 || t.g >= args.G) {
                        if (check) latch_status(args.status, kStatusDeviceCheck);
                        t.g = 0;
                    }
                } else {
                    t.wk = C::CSPLIT ? half_work(args, w, half, C::SF_PERIOD) : work_of(args, w, C::SF_PERIOD);
                    const Tile tl = tile_of(args, t.wk.tile);
                    t.m0 = tl.m_blk * C::TILE_M + (int)rank * C::BM;
                    t.n_blk = tl.n_blk;
                    if constexpr (C::GROUPED) {
                        t.g = __ldg(args.m_indices + t.m0);
                        if (t.g < 0 || t.g >= args.G) {
                            if (check) latch_status(args.status, kStatusDeviceCheck);
                            t.g = 0;
                        }
                    }
                }
                return t;
            };
            for (int w = worker; w < num_work && ok; w += workers) {
                const Item cur = item_of(w, true);
                const Work wk = cur.wk;
                const int m0 = cur.m0, n_blk = cur.n_blk, g = cur.g;
                const int n0 = n_blk * C::BN;
                const int nb0 = n0 + (int)rank * C::BN_CTA;
                for (int kb = wk.kb0; kb < wk.kb1; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!bounded_wait(&empty[s], ph ^ 1u, args, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const bool sf_here = C::SCALED && kb % C::SF_PERIOD == 0;
                    if (leader)
                        mbar_arrive_expect_tx(&full[s], C::CTAS * (C::A_BYTES + C::B_BYTES +
                                                                   (sf_here ? C::SF_STAGE_BYTES : 0)));
                    uint8_t* sa = smem + C::OFF_A + s * C::A_BYTES;
                    uint8_t* sb = smem + C::OFF_B + s * C::B_BYTES;
                    uint8_t* sf = smem + C::OFF_SF + s * C::SF_STAGE_BYTES;
                    // x coordinate in elements of the tensor map's type: 64 bf16 or 128 bytes per step
                    const int kx = kb * (C::kind == Kind::BF16 ? 64 : 128);
                    const int q = kb / C::SF_PERIOD;
                    // A and B come from before the scale layout pass; its output is read only
                    // once it has finished
                    const auto await_prior = [&] {
                        if (sf_here && !prior_done) {
                            griddep_wait();
                            prior_done = true;
                        }
                    };
                    if constexpr (C::MT) {
                        // A' = this CTA's 128 rows of B_g, B' = the chunk's rows of A, split between
                        // the two CTAs at half the tile's N; scale chunks of B_g's rows, and both
                        // 128-row atoms of the chunk's A scales
                        const uint32_t lead_full = mapa_shared(smem_u32(&full[s]), pairbase);
                        const int half_n = masked_n(masked_rows(args, mcount, g, m0)) / 2;
                        tma_load_3d_pair(sa, &tm_a, lead_full, kx, n_blk * C::TILE_M + (int)rank * C::BM, g);
                        tma_load_2d_pair(sb, &tm_b, lead_full, kx, m0 + (int)rank * half_n);
                        await_prior();
                        if (sf_here) {
                            tma_load_4d_pair(sf, &tm_sfa, lead_full, 0, n_blk * C::CTAS + (int)rank, q, g);
                            tma_load_3d_pair(sf + C::SFA_CHUNK, &tm_sfb, lead_full, 0, m0 / 128, q);
                            tma_load_3d_pair(sf + C::SFA_CHUNK + 512, &tm_sfb, lead_full, 0, m0 / 128 + 1, q);
                        }
                    } else if constexpr (C::PAIR) {
                        const uint32_t lead_full = mapa_shared(smem_u32(&full[s]), pairbase);
                        tma_load_2d_pair(sa, &tm_a, lead_full, kx, m0);
                        if constexpr (C::GROUPED)
                            tma_load_3d_pair(sb, &tm_b, lead_full, kx, nb0, g);
                        else
                            tma_load_2d_pair(sb, &tm_b, lead_full, kx, nb0);
                        await_prior();
                        if (sf_here) {
                            // scale chunks: this CTA's A rows, all BN B rows of the tile
                            tma_load_3d_pair(sf, &tm_sfa, lead_full, 0, m0 / C::BM, q);
                            if constexpr (C::GROUPED)
                                tma_load_4d_pair(sf + C::SFA_CHUNK, &tm_sfb, lead_full, 0, n_blk, q, g);
                            else
                                tma_load_3d_pair(sf + C::SFA_CHUNK, &tm_sfb, lead_full, 0, n_blk, q);
                        }
                    } else {
                        tma_load_2d(sa, &tm_a, &full[s], kx, m0);
                        if constexpr (C::GROUPED)
                            tma_load_3d(sb, &tm_b, &full[s], kx, nb0, g);
                        else
                            tma_load_2d(sb, &tm_b, &full[s], kx, nb0);
                        await_prior();
                        if (sf_here) {
                            tma_load_3d(sf, &tm_sfa, &full[s], 0, m0 / C::BM, q);
                            if constexpr (C::GROUPED)
                                tma_load_4d(sf + C::SFA_CHUNK, &tm_sfb, &full[s], 0, n_blk, q, g);
                            else
                                tma_load_3d(sf + C::SFA_CHUNK, &tm_sfb, &full[s], 0, n_blk, q);
                        }
                    }
                }
            }
            // Wind down: wait (bounded) until the copies issued for the last stages landed.
            if (leader) {
                const uint32_t last = it < (uint32_t)C::STAGES ? it : (uint32_t)C::STAGES;
                for (uint32_t j = it - last; j < it; ++j)
                    drain_wait(&full[j % C::STAGES], (j / C::STAGES) & 1u, args);
            }
        }
        __syncwarp();
    } else if (warp == 1 && leader) {
        // ------------------------------------------------------------ MMA issue (one lane)
        if (lane == 0) {
            uint32_t it = 0, lt = 0, git = 0;  // K steps, work items and scale groups issued
            bool ok = true;
            for (int w = worker; w < num_work && ok; w += workers, ++lt) {
                const Work wk =
                    (C::MASKED || C::PAIR_LIST) ? Work{0, 0, args.num_kb, -1, 0}
                    : C::CSPLIT                 ? half_work(args, w, half, C::SF_PERIOD)
                                                : work_of(args, w, C::SF_PERIOD);
                int tile_n = C::BN;  // the MMA's N (masked transposed: the chunk's valid rows)
                if constexpr (C::MT) {
                    int cm0, cnb, cg;
                    masked_tile<C::MCHUNK>(args, mprefix, w, &cm0, &cnb, &cg);
                    tile_n = masked_n(masked_rows(args, mcount, cg, cm0));
                }
                const uint32_t buf = C::ACC_BUFS == 2 ? lt & 1u : 0u;
                const uint32_t aph = C::ACC_BUFS == 2 ? (lt >> 1) & 1u : lt & 1u;
                if (!bounded_wait<C::PAIR>(&tmem_empty[buf], aph ^ 1u, args, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * C::BN;
                uint32_t slot = 0;
                for (int kb = wk.kb0; kb < wk.kb1; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!bounded_wait(&full[s], ph, args, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if constexpr (C::SCALED) {
                        if (kb % C::SF_PERIOD == 0) {
                            // copy this group's scale chunks (carried by this stage) into TMEM slot
                            // git % SF_SLOTS; copies and MMAs run in issue order on the tensor pipe
                            slot = git % C::SF_SLOTS;
                            ++git;
                            const uint32_t sfa_col = C::ACC_COLS + slot * C::SF_SLOT_COLS;
                            const uint32_t sfb_col = sfa_col + C::SFA_COLS;
                            const uint8_t* ua = smem + C::OFF_SF + s * C::SF_STAGE_BYTES;
                            const uint8_t* ub = ua + C::SFA_CHUNK;
#pragma unroll
                            for (int u = 0; u < C::UT_WORDS; ++u) {
                                if constexpr (C::PAIR)
                                    tc_cp_32x128b_warpx4_pair(tmem_base + sfa_col + 4 * u,
                                                              smem_desc_rows16(ua + u * 512));
                                else
                                    tc_cp_32x128b_warpx4(tmem_base + sfa_col + 4 * u, smem_desc_rows16(ua + u * 512));
#pragma unroll
                                for (int at = 0; at < C::SFB_ATOMS; ++at) {
                                    const uint32_t col = tmem_base + sfb_col + 4 * (u * C::SFB_ATOMS + at);
                                    const uint64_t d = smem_desc_rows16(ub + (at * C::UT_WORDS + u) * 512);
                                    if constexpr (C::PAIR)
                                        tc_cp_32x128b_warpx4_pair(col, d);
                                    else
                                        tc_cp_32x128b_warpx4(col, d);
                                }
                            }
                        }
                    }
                    const uint64_t adesc = smem_desc_k_sw128(smem + C::OFF_A + s * C::A_BYTES);
                    const uint64_t bdesc = smem_desc_k_sw128(smem + C::OFF_B + s * C::B_BYTES);
                    const uint32_t sfa_t = tmem_base + C::ACC_COLS + slot * C::SF_SLOT_COLS;
                    const uint32_t sfb_t = sfa_t + C::SFA_COLS;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        // 32 bytes of K per MMA: 16 bf16, 32 E4M3, 64 E2M1
                        const uint64_t ad = adesc + (uint64_t)(2 * i);
                        const uint64_t bd = bdesc + (uint64_t)(2 * i);
                        const uint32_t acc = (kb > wk.kb0 || i > 0) ? 1u : 0u;
                        if constexpr (C::kind == Kind::BF16) {
                            const uint32_t id = idesc_bf16(C::TILE_M, C::BN);
                            if constexpr (C::PAIR)
                                tc_mma_f16_pair(d_tmem, ad, bd, id, acc);
                            else
                                tc_mma_f16(d_tmem, ad, bd, id, acc);
                        } else if constexpr (C::kind == Kind::FP8) {
                            const uint32_t sid = (uint32_t)(kb % 4);
                            const uint32_t id = idesc_block_scaled(C::TILE_M, tile_n, 0u, sid, sid);
                            if constexpr (C::PAIR)
                                tc_mma_mxf8_pair(d_tmem, ad, bd, id, sfa_t, sfb_t, acc);
                            else
                                tc_mma_mxf8(d_tmem, ad, bd, id, sfa_t, sfb_t, acc);
                        } else {
                            const uint32_t u = (uint32_t)(i >> 1), sid = (uint32_t)((i & 1) * 2);
                            const uint32_t id = idesc_block_scaled(C::TILE_M, C::BN, 1u, sid, sid);
                            if constexpr (C::PAIR)
                                tc_mma_mxf4_pair(d_tmem, ad, bd, id, sfa_t + 4 * u, sfb_t + 4 * C::SFB_ATOMS * u, acc);
                            else
                                tc_mma_mxf4(d_tmem, ad, bd, id, sfa_t + 4 * u, sfb_t + 4 * C::SFB_ATOMS * u, acc);
                        }
                    }
                    // the stage (A, B and any scale chunk) is free once these MMAs and copies completed
                    if constexpr (C::PAIR)
                        tc_commit_pair_mc(&empty[s], kPairMask);
                    else
                        tc_commit(&empty[s]);
                }
                if (!ok) break;
                if constexpr (C::PAIR)
                    tc_commit_pair_mc(&tmem_full[buf], kPairMask);
                else
                    tc_commit(&tmem_full[buf]);
            }
            // Wind down: every MMA and scale copy this lane issued has completed.
            if constexpr (C::PAIR)
                tc_commit_pair(drain);
            else
                tc_commit(drain);
            drain_wait(drain, 0, args);
        }
        __syncwarp();
    } else if (warp == 1) {
        // peer CTA of a pair: the leader issues every tensor-core instruction
    } else {
        // ------------------------------------------------------------ epilogue
        const uint32_t quarter = warp % 4;  // TMEM lanes this warp may read
        uint8_t* epi = smem + C::OFF_EPI + (warp - 2) * 2 * C::EPI_BLOCK;
        uint32_t lt = 0, nblk = 0, gather_phase = 0;
        for (int w = C::CSPLIT ? num_work : worker; w < num_work; w += workers, ++lt) {
            Work wk{0, 0, args.num_kb, -1, 0};
            int m0, n_blk, g = 0;
            bool mine = true;  // this CTA's rows belong to the tile (false: the peer half of a one-block pair tile)
            if constexpr (C::MASKED) {
                masked_tile<C::MCHUNK>(args, mprefix, w, &m0, &n_blk, &g);
            } else if constexpr (C::PAIR_LIST) {
                int b0, len;
                pair_tile(args, plist, w, &b0, &len, &n_blk);
                m0 = (b0 + (int)rank) * C::BM;
                mine = (int)rank < len;
            } else {
                wk = work_of(args, w, C::SF_PERIOD);
                const Tile tl = tile_of(args, wk.tile);
                m0 = tl.m_blk * C::TILE_M + (int)rank * C::BM;
                n_blk = tl.n_blk;
            }
            const int n0 = n_blk * C::BN;
            const uint32_t buf = C::ACC_BUFS == 2 ? lt & 1u : 0u;
            const uint32_t aph = C::ACC_BUFS == 2 ? (lt >> 1) & 1u : lt & 1u;
            if (!warp_wait(&tmem_full[buf], aph, args, abort_flag)) break;
            tc_fence_after();
            const int row = m0 + (int)(quarter * 32 + lane);
            bool zero_row = false;
            // masked layout: only rows below the expert's count are written; a warp whose 32
            // rows are all valid stores through TMA, one with some invalid rows row by row
            bool row_valid = mine, all_valid = mine;
            if constexpr (C::MASKED && !C::MT) {
                row_valid = row - g * args.max_m < mcount[g];
                all_valid = __all_sync(0xffffffffu, row_valid);
            }
            // masked transposed: valid rows of the chunk (D rows m0 ...), and this warp's 32
            // columns of D (its TMEM lanes: rows of B_g)
            const int vrows = C::MT ? masked_rows(args, mcount, g, m0) : 0;
            const int dcol = n_blk * C::TILE_M + (int)rank * C::BM + (int)quarter * 32;
            if constexpr (C::GROUPED && !C::MASKED) {
                if (row < args.M && mine) {
                    const int g0 = __ldg(args.m_indices + m0);
                    const int gi = __ldg(args.m_indices + row);
                    zero_row = gi < 0;
                    if (gi != g0 && gi != -1) latch_status(args.status, kStatusDeviceCheck);
                }
            }
            const uint32_t taddr = tmem_base + ((quarter * 32) << 16) + buf * C::BN;
            const auto release = [&] {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(&tmem_empty[buf]);
                    else
                        mbar_arrive_remote(mapa_shared(smem_u32(&tmem_empty[buf]), pairbase));
                }
            };
            const auto pack = [&](uint32_t lo, uint32_t hi) -> uint32_t {
                __nv_bfloat162 v = __float22bfloat162_rn(make_float2(__uint_as_float(lo), __uint_as_float(hi)));
                return zero_row ? 0u : *reinterpret_cast<uint32_t*>(&v);
            };
            // one 32 x 32 block (16 packed bf16 pairs per lane) through the swizzled staging
            // buffer to D
            const auto store_block = [&](int c, const uint32_t* w16) {
                if constexpr (C::MT) {
                    // accumulator column 32c + j is D row m0 + 32c + j; lane l holds D column dcol + l
                    const int j0 = c * 32;
                    if (j0 >= vrows || dcol >= args.N) return;
                    if (j0 + 32 <= vrows) {
                        // a whole block: transposed into the 64-byte-swizzled staging buffer, then TMA
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
                        uint8_t* blk = epi + (nblk & 1u) * C::EPI_BLOCK;
                        const uint32_t b32 = smem_u32(blk) + (lane & 7u) * 2u;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            st_shared_u16(b32 + (uint32_t)(j * 64) + (((lane >> 3) ^ (uint32_t)((j >> 1) & 3)) << 4),
                                          (uint16_t)(w16[j >> 1] >> (16 * (j & 1))));
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tm_d, blk, dcol, m0 + j0);
                            bulk_commit_group();
                        }
                        ++nblk;
                    } else if (dcol + (int)lane < args.N) {
                        // the chunk's last block, rows past the count not touched: plain stores
                        __nv_bfloat16* col = args.D + (int64_t)(m0 + j0) * args.ldd + dcol + lane;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (j0 + j < vrows)
                                *reinterpret_cast<uint16_t*>(col + (int64_t)j * args.ldd) =
                                    (uint16_t)(w16[j >> 1] >> (16 * (j & 1)));
                    }
                    return;
                }
                if constexpr (C::TRANS_D) {
                    // element (row, n0 + 32c + j) goes to D[n0 + 32c + j][row]: for each j the
                    // warp writes 32 consecutive bf16 of one row of D
                    if (row < args.M) {
                        __nv_bfloat16* col = args.D + row;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int d_row = n0 + c * 32 + j;
                            if (d_row < args.N)
                                *reinterpret_cast<uint16_t*>(col + (int64_t)d_row * args.ldd) =
                                    (uint16_t)(w16[j >> 1] >> (16 * (j & 1)));
                        }
                    }
                    return;
                }
                if (!all_valid) {
                    if (row_valid) {
                        __nv_bfloat16* dst = args.D + (int64_t)row * args.ldd + n0 + c * 32;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (n0 + c * 32 + 8 * q + 8 <= args.N)
                                *reinterpret_cast<uint4*>(dst + 8 * q) =
                                    make_uint4(w16[4 * q], w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
                    }
                    return;
                }
                // a block wholly outside D is neither staged nor stored: staging it would reuse the
                // buffer of the last store issued, which may still be reading it
                if (m0 + (int)quarter * 32 >= args.M || n0 + c * 32 >= args.N) return;
                // the store issued from this buffer two blocks ago has finished reading it
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
                uint8_t* blk = epi + (nblk & 1u) * C::EPI_BLOCK;
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // 16-byte chunk q of this row (8 columns)
                    // 64-byte swizzle: chunk q of row l sits at chunk q ^ ((l >> 1) & 3)
                    const uint32_t pos = lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4);
                    *reinterpret_cast<uint4*>(blk + pos) =
                        make_uint4(w16[4 * q], w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tm_d, blk, n0 + c * 32, m0 + (int)quarter * 32);
                    bulk_commit_group();
                }
                ++nblk;
            };
            if (wk.tail >= 0) {
                // K slice of a split tile (this worker's last work item: no copy or MMA touches
                // the stage buffers any more).  Each warp lays its 32 rows of fp32 partial sums
                // out in the stage buffers as 32 x 32 blocks (128-byte swizzle) and stores them
                // with TMA in the slice's workspace slot.
                const int64_t slot_stride = (int64_t)C::TILE_M * C::BN;
                const int slot_row = (wk.tail * args.splits + wk.slice) * C::TILE_M + (int)rank * C::BM + (int)quarter * 32;
                uint8_t* stage = smem + C::OFF_A + (warp - 2) * (32 * C::BN * 4);
#pragma unroll 1
                for (int c = 0; c < C::BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, r);
                    tmem_ld_wait();
                    if (c == C::BN / 32 - 1) release();
                    uint8_t* blk = stage + c * 4096;
#pragma unroll
                    for (int v = 0; v < 8; ++v) {  // 16-byte chunk v of this row sits at chunk v ^ (row % 8)
                        const uint32_t pos = lane * 128 + ((v ^ (lane & 7)) << 4);
                        *reinterpret_cast<uint4*>(blk + pos) = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    for (int c = 0; c < C::BN / 32; ++c) tma_store_2d(&tm_ws, stage + c * 4096, c * 32, slot_row);
                    bulk_commit_group();
                    bulk_wait_group_all();  // complete in memory, not only read
                    fence_proxy_async_global();
                }
                // Publish this slice, then reduce without ever waiting on a CTA that may not be
                // resident.  Share j of these 32 rows (rows [32j/S, 32(j+1)/S)) is summed by whoever
                // claims it first: slice j itself, if it sees every slice published within a short
                // poll, or the slice that published last, which claims every share still open.  Each
                // share is reduced exactly once, always summing the slots in slot order, so the bytes
                // do not depend on who reduced it.
                const int S = args.splits;
                const int cidx = (wk.tail * C::CTAS + (int)rank) * 4 + (int)quarter;
                int* cnt = args.tail_count + cidx;
                int* claim = args.tail_claim + cidx * S;
                int state = 0;  // bit 0: every slice published; bit 1: this slice published last
                if (lane == 0) {
                    __threadfence();
                    griddep_wait();  // the counters were zeroed by the kernel launched before
                    if (atomicAdd(cnt, 1) == S - 1) {
                        state = 3;
                    } else {
                        const uint64_t t0 = globaltimer_ns();
                        const uint64_t limit = args.timeout_ns < kTailPollNs ? args.timeout_ns : kTailPollNs;
                        while (!*abort_flag) {
                            if (*reinterpret_cast<volatile int*>(cnt) >= S) {
                                state = 1;
                                break;
                            }
                            if (globaltimer_ns() - t0 > limit) break;
                            __nanosleep(64);
                        }
                    }
                    __threadfence();
                    fence_proxy_async_global();  // the other slices' stores, acquired above, before the bulk reads
                }
                state = __shfl_sync(0xffffffffu, state, 0);
                const int row_bytes = C::BN * 4;
                const float* wbase = args.ws + (int64_t)wk.tail * S * slot_stride +
                                     (int64_t)((int)rank * C::BM + (int)quarter * 32) * C::BN;
                const int P = 32 / S;  // rows per gather pass: P rows of all S slots fill the staging area
                bool ok = true;
                // shares this warp reduces (bit j: share j): its own first, claimed by lane 0; then,
                // in the slice that published last, every share still open, claimed in one round
                // (lane j tries share j) after its own is done, so the owners come first
                uint32_t todo = 0;
                if (state & 1) {
                    int won = 0;
                    if (lane == 0) won = atomicCAS(claim + wk.slice, 0, 1) == 0;
                    if (__shfl_sync(0xffffffffu, won, 0)) todo = 1u << wk.slice;
                }
                for (int round = 0; round < 2 && ok; ++round) {
                    if (round == 1) {
                        if (!(state & 2)) break;
                        const bool took = (int)lane < S && (int)lane != wk.slice && atomicCAS(claim + lane, 0, 1) == 0;
                        todo = __ballot_sync(0xffffffffu, took);
                    }
                    while (todo && ok) {
                        const int share = __ffs(todo) - 1;
                        todo &= todo - 1;
                        const int r_end = (share + 1) * 32 / S;
                        for (int rp = share * 32 / S; rp < r_end; rp += P) {
                            const int nr = r_end - rp < P ? r_end - rp : P;
                            // the staging area's previous contents have been read by every lane
                            __syncwarp();
                            fence_proxy_async_smem();
                            if (lane == 0) {
                                mbar_arrive_expect_tx(&gather[warp - 2], (uint32_t)(nr * S * row_bytes));
                                for (int r = 0; r < nr; ++r)
                                    for (int j = 0; j < S; ++j)
                                        bulk_load(stage + (r * S + j) * row_bytes, wbase + j * slot_stride + (int64_t)(rp + r) * C::BN,
                                                  (uint32_t)row_bytes, &gather[warp - 2]);
                            }
                            if (!warp_wait(&gather[warp - 2], gather_phase, args, abort_flag)) {
                                ok = false;
                                break;
                            }
                            gather_phase ^= 1u;
                            // The reduction runs once, at the end of the kernel, so its instructions are
                            // cold: compact loops, not unrolled bodies.  First every row's S copies are
                            // added, in slot order, into its slot-0 copy (16 bytes per lane, consecutive
                            // lanes on consecutive bytes); then the sums are rounded and written.
                            const uint32_t sbase = smem_u32(stage);
                            const uint32_t row_pitch = (uint32_t)(S * row_bytes);  // between gathered rows
#pragma unroll 1
                            for (int r = 0; r < nr; ++r) {
#pragma unroll 1
                                for (int c = (int)lane * 4; c < C::BN; c += 128) {
                                    const uint32_t a0 = sbase + (uint32_t)r * row_pitch + (uint32_t)c * 4u;
                                    float4 acc = ld_shared_f32x4(a0);
#pragma unroll 1
                                    for (int j = 1; j < S; ++j) {
                                        const float4 x = ld_shared_f32x4(a0 + (uint32_t)(j * row_bytes));
                                        acc.x += x.x, acc.y += x.y, acc.z += x.z, acc.w += x.w;
                                    }
                                    st_shared_f32x4(a0, acc);
                                }
                            }
                            __syncwarp();
                            if constexpr (C::TRANS_D) {
                                // element (row, n0 + c) goes to D[n0 + c][row]: lane l writes D rows n0 + l,
                                // n0 + l + 32, ..., each with the nr consecutive bf16 of its column, eight at
                                // a time (one 16-byte store where D's row allows it)
                                const int row0 = m0 + (int)quarter * 32 + rp;
#pragma unroll 1
                                for (int c = (int)lane; c < C::BN; c += 32) {
                                    const int d_row = n0 + c;
                                    if (d_row >= args.N) continue;
                                    __nv_bfloat16* dst = args.D + (int64_t)d_row * args.ldd + row0;
#pragma unroll 1
                                    for (int r8 = 0; r8 < nr; r8 += 8) {
                                        uint32_t w[4];
#pragma unroll
                                        for (int h = 0; h < 4; ++h) {
                                            const int r = r8 + 2 * h;
                                            const float lo = r < nr ? ld_shared_f32(sbase + (uint32_t)r * row_pitch + (uint32_t)c * 4u) : 0.f;
                                            const float hi = r + 1 < nr ? ld_shared_f32(sbase + (uint32_t)(r + 1) * row_pitch + (uint32_t)c * 4u) : 0.f;
                                            __nv_bfloat162 b2 = __float22bfloat162_rn(make_float2(lo, hi));
                                            w[h] = *reinterpret_cast<uint32_t*>(&b2);
                                        }
                                        __nv_bfloat16* d8 = dst + r8;
                                        if (r8 + 8 <= nr && row0 + r8 + 8 <= args.M && (reinterpret_cast<uintptr_t>(d8) & 15u) == 0) {
                                            *reinterpret_cast<uint4*>(d8) = make_uint4(w[0], w[1], w[2], w[3]);
                                        } else {
#pragma unroll
                                            for (int r = 0; r < 8; ++r)
                                                if (r8 + r < nr && row0 + r8 + r < args.M)
                                                    *reinterpret_cast<uint16_t*>(d8 + r) = (uint16_t)(w[r >> 1] >> (16 * (r & 1)));
                                        }
                                    }
                                }
                            } else {
                                const int col = (int)lane * 8;  // 8 columns per lane
                                const int n = n0 + col;
#pragma unroll 1
                                for (int r = 0; r < nr; ++r) {
                                    const int row = m0 + (int)quarter * 32 + rp + r;
                                    if (row >= args.M || col >= C::BN || n >= args.N) continue;
                                    const uint32_t a4 = sbase + (uint32_t)r * row_pitch + (uint32_t)col * 4u;
                                    const float4 x0 = ld_shared_f32x4(a4), x1 = ld_shared_f32x4(a4 + 16);
                                    const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                                    __nv_bfloat16* dst = args.D + (int64_t)row * args.ldd + n;
                                    if (n + 8 <= args.N) {
                                        uint32_t o[4];
#pragma unroll
                                        for (int e = 0; e < 4; ++e) {
                                            __nv_bfloat162 b2 = __float22bfloat162_rn(make_float2(v[2 * e], v[2 * e + 1]));
                                            o[e] = *reinterpret_cast<uint32_t*>(&b2);
                                        }
                                        *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
                                    } else {
#pragma unroll
                                        for (int e = 0; e < 8; ++e)
                                            if (n + e < args.N) dst[e] = __float2bfloat16_rn(v[e]);
                                    }
                                }
                            }
                        }
                    }
                }
                if (!ok) break;
            } else if constexpr (C::ACC_BUFS == 2) {
#pragma unroll 1
                for (int c = 0; c < C::BN / 32; ++c) {
                    uint32_t r[32], w[16];
                    tmem_ld_32x32b_x32(taddr + c * 32, r);
                    tmem_ld_wait();
                    if (c == C::BN / 32 - 1) release();
#pragma unroll
                    for (int h = 0; h < 16; ++h) w[h] = pack(r[2 * h], r[2 * h + 1]);
                    store_block(c, w);
                }
            } else {
                // drain the whole accumulator row into registers (bf16 pairs), free it, then store
                uint32_t w[C::BN / 2];
#pragma unroll
                for (int c = 0; c < C::BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 16; ++h) w[16 * c + h] = pack(r[2 * h], r[2 * h + 1]);
                }
                release();
#pragma unroll
                for (int c = 0; c < C::BN / 32; ++c) store_block(c, w + 16 * c);
            }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    if constexpr (C::CSPLIT) {
        // One tile per cluster: pair h holds the fp32 sums of K half h in TMEM and finishes
        // columns [64h, 64h + 64) of the tile.  Each epilogue warp trades 32 rows x 64 columns
        // with the warp of the same quarter in the CTA of the other pair with the same rank:
        // it announces that its receive buffer is free (its own MMAs are done, so the stage
        // buffers are idle), lays out the columns the other pair finishes in its own shared
        // memory and, once the other side's buffer is free, moves them there with one bulk copy
        // that completes on the receiver's barrier.  It then adds the received sums to its own
        // (the same fp32 sum of the two halves as the two-slice split tail), rounds to bf16 and
        // stores its 64 x 32 block of D (rows of D are the tile's columns) with TMA.
        if (warp >= 2 && worker < num_work) {
            const uint32_t quarter = warp % 4;
            const int wq = warp - 2;
            const Tile tl = tile_of(args, worker);
            const int dcol = tl.m_blk * C::TILE_M + (int)rank * C::BM + (int)quarter * 32;  // columns of D
            const int keep = half * C::X_COLS, give = (1 - half) * C::X_COLS;
            const int drow = tl.n_blk * C::BN + keep;  // rows of D
            uint8_t* sendb = smem + C::OFF_A + wq * C::X_WARP_BYTES;
            uint8_t* recvb = sendb + C::X_BYTES;
            uint8_t* outb = recvb + C::X_BYTES;
            const uint32_t other = crank ^ 2u;
            const uint32_t taddr = tmem_base + ((quarter * 32) << 16);
            bool ok = warp_wait(&tmem_full[0], 0, args, abort_flag);
            tc_fence_after();
            if (ok && lane == 0) {
                mbar_arrive_expect_tx(&xfull[wq], C::X_BYTES);
                mbar_arrive_remote(mapa_shared(smem_u32(&xready[wq]), other));
            }
            // lane l's 64 columns: 16 chunks of 16 bytes at l * 256, chunk v at v ^ (l & 15)
            const auto chunk = [&](uint8_t* base, int v) {
                return smem_u32(base) + lane * 256u + (uint32_t)((v ^ (int)(lane & 15)) << 4);
            };
            if (ok) {
#pragma unroll 1
                for (int c = 0; c < C::X_COLS / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + give + c * 32, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        st_shared_f32x4(chunk(sendb, c * 8 + v),
                                        make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                                    __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (ok && lane == 0) {
                ok = bounded_wait<true>(&xready[wq], 0, args, abort_flag);
                if (ok)
                    bulk_copy_to_cluster(mapa_shared(smem_u32(recvb), other), sendb, C::X_BYTES,
                                         mapa_shared(smem_u32(&xfull[wq]), other));
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (ok) ok = warp_wait<true>(&xfull[wq], 0, args, abort_flag);
            if (ok) {
#pragma unroll 1
                for (int c = 0; c < C::X_COLS / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + keep + c * 32, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const float4 x = ld_shared_f32x4(chunk(recvb, c * 8 + v));
                        const float s0 = __uint_as_float(r[4 * v]) + x.x, s1 = __uint_as_float(r[4 * v + 1]) + x.y;
                        const float s2 = __uint_as_float(r[4 * v + 2]) + x.z, s3 = __uint_as_float(r[4 * v + 3]) + x.w;
                        __nv_bfloat162 b0 = __float22bfloat162_rn(make_float2(s0, s1));
                        __nv_bfloat162 b1 = __float22bfloat162_rn(make_float2(s2, s3));
                        const uint32_t w0 = *reinterpret_cast<uint32_t*>(&b0), w1 = *reinterpret_cast<uint32_t*>(&b1);
                        // column 32c + 4v + i of the tile is row 32c + 4v + i of this block of D;
                        // lane l is its column l (64 bytes a row)
                        const uint32_t o = smem_u32(outb) + (uint32_t)((c * 32 + 4 * v) * 64) + lane * 2u;
                        st_shared_u16(o, (uint16_t)w0);
                        st_shared_u16(o + 64, (uint16_t)(w0 >> 16));
                        st_shared_u16(o + 128, (uint16_t)w1);
                        st_shared_u16(o + 192, (uint16_t)(w1 >> 16));
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                // rows past M and columns past N are dropped by the tensor map's bounds
                if (lane == 0 && dcol < args.M && drow < args.N) {
                    tma_store_2d(&tm_d, outb, dcol, drow);
                    bulk_commit_group();
                    bulk_wait_group_all();
                }
            }
            __syncwarp();
        }
    }

    tc_fence_before();
    if constexpr (C::PAIR)
        cluster_sync();  // the leader's MMAs into the peer's TMEM are done before either frees it
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (C::PAIR)
            tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
        else
            tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace bsp
