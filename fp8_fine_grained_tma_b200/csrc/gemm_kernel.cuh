// gemm_kernel.cuh -- persistent fine-grained-scaled FP8 GEMM for sm_100a.
//
// Computes, for each output tile,
//   D[m,n] = bf16( sum_kb (A_kb . B_kb^T)[m,n] * sfa[m,kb] * sfb[n/128,kb] )
// which is the fine-grained ("DeepSeek-V3 style") scaling of the pages
// (chujupifa.com "机器之心报道", opening summary; deepseek.csdn.net
// "DeepGEMM：简洁、高效…", section "什么是DeepGEMM呢？") with the two-level
// accumulation they describe (each 128-wide K block is accumulated by the
// tensor core, then scaled and added into FP32 on the CUDA cores;
// chujupifa.com report, opening summary; ai.abqq.net, section 1 "架构优化").
//
// B200 design (not the pages' Hopper design).  One CTA per SM, 12 warps:
//   warp 8     TMA producer: one lane streams the CTA's A [128 x 128] and B
//              [BNL x 128] E4M3 tiles into an S-stage shared-memory ring
//              (128-byte swizzle).
//   warps 9-10 MMA issuers: one lane each, taking turns by K block, issues
//              4 x tcgen05.mma kind::f8f6f4 (K=32) per K block into one of NBUF
//              (2..4) TMEM accumulators, overwriting it at the block's first MMA.
//   warps 0-7  promotion + epilogue: two warpgroups split the tile's 16-column
//              chunks; each thread owns one TMEM lane (= one output row), reads
//              the block's partial sums with tcgen05.ld, multiplies by
//              sfa[m,kb] * sfb[n/128,kb] (loaded by the thread itself a group of
//              K blocks ahead) and adds into FP32 registers; after the last
//              block it converts to BF16 and stores its 32 x 16 pieces with TMA
//              bulk tensor stores (rows that may not be written go through
//              predicated stores instead).
//   warp 11    idle (it completes the third warpgroup for the register split).
// The tensor core takes about the same time per K block for any N up to 256
// (one 128-row MMA of K=32 every ~128 cycles), so the widest block (256)
// gives the most work per K block; narrower blocks exist for small N.
// PAIR = false: the tile is 128 x BN and the CTA works alone (M=128 MMA).
// PAIR = true:  two CTAs of a cluster share a 256 x BN tile (tcgen05
//   cta_group::2, M=256): each loads its own 128 rows of A and its own half of
//   the BN rows of B, the leader CTA issues the MMAs, and each CTA's TMEM holds
//   its 128 rows x BN columns.  No load uses multicast.
// Tiles are scheduled persistently (static stride over a raster-grouped tile
// order); the contiguous and masked MoE layouts of the pages (game.3loumao.org
// explainer, section "03 DeepSeek是如何创新的？") change only the tile -> (group,
// row block, column block) mapping and which rows are stored.
#pragma once

#include <cuda_bf16.h>

#include "rtc_compat.cuh"

#include "ptx.cuh"

// K blocks of the problem as a compile-time constant when the kernel is
// compiled at run time for one shape (0: taken from the parameters).
#ifndef FG8_KB_CT
#define FG8_KB_CT 0
#endif

namespace fg8 {

constexpr int BM = 128;
constexpr int BK = 128;
constexpr int NUM_EPI_WARPS = 8;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;                        // first MMA issuer (also allocates TMEM)
constexpr int NUM_MMA_WARPS = 2;                   // warps MMA_WARP .. MMA_WARP + NUM_MMA_WARPS - 1 issue MMAs
constexpr int NUM_THREADS = 384;                   // 3 warpgroups: 2 promotion, 1 producer/MMA
// Register split (setmaxnreg, inside each role's own branch): every thread is
// launched with REGS_LAUNCH registers; the producer warpgroup (warps 8..11)
// drops to REGS_PRODUCER and the two promotion warpgroups rise to
// REGS_PROMOTION.  256 * 224 + 128 * 56 == 384 * 168, so the raise only uses
// registers the block already owns.  The host launches a build only if its
// register count is exactly REGS_LAUNCH (otherwise the raise could wait forever).
constexpr int REGS_LAUNCH = 168;
constexpr int REGS_PRODUCER = 56;
constexpr int REGS_PROMOTION = 224;
static_assert(256 * REGS_PROMOTION + 128 * REGS_PRODUCER <= NUM_THREADS * REGS_LAUNCH, "register split");
// Epilogue staging: per promotion warp EPI_SLOTS pieces of 32 rows x 16 BF16
// columns (32 bytes a row, in the 32-byte swizzle of the D tensor map: the
// 16-byte half h of row r sits at r*32 + (h ^ ((r >> 2) & 1)) * 16).
constexpr int EPI_SLOT_BYTES = 32 * 32;
constexpr int EPI_SLOTS = 2;
constexpr int EPI_WARP_BYTES = EPI_SLOTS * EPI_SLOT_BYTES;
// Scales are loaded by the promotion threads themselves, SCALE_GROUP K blocks
// at a time, one group ahead of their use.
constexpr int SCALE_GROUP = 2;
constexpr int SCALE_PREFETCH = 8;                  // K blocks between the L1 prefetch of sfa and its load
constexpr int A_TILE_BYTES = BM * BK;              // 16 KiB
// Contiguous layout, CTA pairs: the 128-row blocks that start a pair tile are
// listed in shared memory (one 16-bit block index each).
constexpr int MAX_PAIR_LIST = 4096;
constexpr int PAIR_LIST_BYTES = MAX_PAIR_LIST * 2;

enum : int { LAYOUT_NORMAL = 0, LAYOUT_CONTIGUOUS = 1, LAYOUT_MASKED = 2 };

enum : int { ERR_TIMEOUT = 6 };
enum : int { ROLE_PRODUCER = 1, ROLE_MMA = 2, ROLE_EPILOGUE = 3 };

struct GemmParams {
    int layout;
    int rows;          // rows per group: M (normal), M_tot (contiguous), M_max (masked)
    int N, K, G;
    int KB, NB;        // K / 128, ceil(N / 128)
    int num_m_tiles;   // row tiles per group: ceil(rows / (128 or 256))
    int num_n_blocks;  // ceil(N / BN)
    int raster_m;      // row tiles per raster group
    int stages;
    int sfa_ld;        // M_pad: stride (floats) between K blocks of the MN-major sfa
    const float* sfa;  // [G or 1][KB][sfa_ld]
    const float* sfb;  // [G][NB][KB]
    __nv_bfloat16* D;  // [G or 1][rows][N]
    const int* m_indices;
    const int* masked_m;
    int* status;       // [0] = first error code, [1] = (block << 8) | role
    unsigned long long wait_limit_ns;
    // Stream-K (normal layout): the first sk_dp_tiles tiles are processed whole,
    // wave by wave; the (tile, K block) iterations of the remaining tiles are
    // split evenly over the units.  sk_ws holds one FP32 partial tile slice per
    // CTA ([grid][NC][128][16]), sk_flags the epoch of the last partial each
    // promotion warp of each CTA published ([grid][8]); sk_epoch is this
    // launch's (never 0).
    // Cluster split-K (normal layout, single CTAs, one row tile): CTA u of the
    // grid handles tile u / ks, K blocks [s * ks_per, (s + 1) * ks_per) with
    // s = u % ks; the ks CTAs of a tile form one thread-block cluster and sum
    // their partials through distributed shared memory.  ks <= 1: off.
    int ks;
    int ks_per;
    int sk;                  // 1: stream-K on
    int sk_dp_tiles;         // tiles processed whole before the split ones
    long long sk_iters;      // (tiles - sk_dp_tiles) * KB
    float* sk_ws;
    unsigned* sk_flags;
    unsigned sk_epoch;
};

__host__ __device__ constexpr int ceil_div_c(int a, int b) { return (a + b - 1) / b; }

template <int BN, bool PAIR>
struct GemmShape {
    static constexpr int NC = BN / 16;                  // 16-column chunks in a tile
    static constexpr int CPW = (NC + 1) / 2;            // chunks per promotion warpgroup
    static constexpr int BNL = PAIR ? BN / 2 : BN;      // B rows this CTA loads per K block
    static constexpr int TILE_M = PAIR ? 2 * BM : BM;   // rows of a tile
    static constexpr int B_TILE_BYTES = BNL * BK;
    static constexpr int STAGE_BYTES = A_TILE_BYTES + B_TILE_BYTES;
    static constexpr int TX_BYTES = PAIR ? 2 * STAGE_BYTES : STAGE_BYTES;   // expected on the (leader's) full barrier
    static constexpr int ACC_STRIDE = (BN + 31) / 32 * 32;   // TMEM columns per accumulator
    // As many K-block accumulators as TMEM holds (at most 4): the MMA issuer may
    // run NBUF - 1 blocks ahead of the promotion warps.
    static constexpr int NBUF = (512 / ACC_STRIDE) < 4 ? (512 / ACC_STRIDE) : 4;
    static constexpr int TMEM_USED = NBUF * ACC_STRIDE;
    static constexpr int TMEM_COLS = TMEM_USED <= 32    ? 32
                                     : TMEM_USED <= 64  ? 64
                                     : TMEM_USED <= 128 ? 128
                                     : TMEM_USED <= 256 ? 256
                                                        : 512;
    static constexpr int TEMPTY_COUNT = PAIR ? 2 * NUM_EPI_WARPS : NUM_EPI_WARPS;
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "BN must be a multiple of 16 in [16, 256]");
    static_assert(!PAIR || BN >= 32, "a CTA pair needs at least 16 B rows per CTA");
    static_assert(NBUF >= 2, "need two accumulators");
    // An issuer waits on an accumulator / stage barrier for the phase right
    // after the one its previous K block used; with more issuers than
    // accumulators it could wait two phases ahead and see a stale completion.
    // (The host also keeps the stage count >= NBUF for the same reason.)
    static_assert(NUM_MMA_WARPS <= NBUF, "more MMA issuers than TMEM accumulators");
};

// Dynamic shared memory layout (after aligning the base to 1024 bytes):
//   [stages x (A tile | B tile)] [8 x epilogue staging] [pair list (pairs only)]
//   [barriers] [tmem slot, abort flag, list count]
constexpr int MAX_NBUF = 4;
__host__ __device__ constexpr size_t gemm_smem_bytes(int stage_bytes, int stages, bool pair) {
    return 1024 + static_cast<size_t>(stages) * stage_bytes + NUM_EPI_WARPS * EPI_WARP_BYTES +
           (pair ? PAIR_LIST_BYTES : 0) + (2 * stages + 2 * MAX_NBUF + 1) * 8 + 16;
}

struct TileInfo {
    int g;       // group of B / sfb (expert); for the masked layout also of A / D
    int row0;    // first row (within the group) of this CTA's 128-row slice of the tile
    int n_blk;
    int kb0, kb1;      // K blocks [kb0, kb1) of the tile processed here (0, KB unless stream-K)
    int sk_first;      // stream-K, kb0 > 0 and kb1 == KB: first unit whose partial this one adds
};

// Enumerates the tiles of this CTA (or CTA pair).  Every role builds its own
// copy and walks the same sequence, so no role tells another which tile is next.
template <bool PAIR>
struct TileScheduler {
    int next;
    int stride;
    int rank;                          // CTA rank within the pair (0 when alone)
    int mg, mbase, mtiles, mtiles_m;   // masked layout cursor
    const uint16_t* pair_list;         // contiguous layout with pairs
    int pair_count;

    long long sk_lo, sk_cur;           // stream-K: this unit's iteration range [sk_lo, sk_hi), walked backwards
    int unit_, units_;

    __device__ TileScheduler(int unit, int num_units, int rank_, const uint16_t* list, int count) {
        init(unit, num_units, rank_, list, count);
    }
    TileScheduler() = default;

    __device__ void init(int unit, int num_units, int rank_, const uint16_t* list, int count) {
        next = unit;
        stride = num_units;
        rank = rank_;
        mg = 0;
        mbase = 0;
        mtiles = -1;
        mtiles_m = 0;
        pair_list = list;
        pair_count = count;
        sk_lo = 0;
        sk_cur = 0;
        unit_ = unit;
        units_ = num_units;
    }

    // First iteration of unit u's stream-K range.
    __device__ static long long sk_start(const GemmParams& p, int u, int units) {
        return static_cast<long long>(u) * p.sk_iters / units;
    }

    // Raster-grouped tile order: tile index -> (row tile, column block).
    __device__ static void raster(const GemmParams& p, int idx, int& m_tile, int& n_blk) {
        const int per_group = p.raster_m * p.num_n_blocks;
        const int grp = idx / per_group;
        const int first_m = grp * p.raster_m;
        const int gm = min(p.raster_m, p.num_m_tiles - first_m);
        const int local = idx - grp * per_group;
        m_tile = first_m + local % gm;
        n_blk = local / gm;
    }

    __device__ bool get(const GemmParams& p, TileInfo& t) {
        constexpr int TILE_M = PAIR ? 2 * BM : BM;
        t.kb0 = 0;
        t.kb1 = FG8_KB_CT > 0 ? FG8_KB_CT : p.KB;
        t.sk_first = -1;
        if (!PAIR && p.ks > 1) {
            // One (tile, K split) per CTA.
            if (next >= p.num_m_tiles * p.num_n_blocks * p.ks) return false;
            const int tile = next / p.ks;
            const int split = next - tile * p.ks;
            next += stride;
            t.kb0 = split * p.ks_per;
            t.kb1 = min(p.KB, t.kb0 + p.ks_per);
            int m_tile;
            raster(p, tile, m_tile, t.n_blk);
            t.row0 = m_tile * BM;
            t.g = 0;
            return true;
        }
        if (p.sk) {
            // Whole tiles first (unit, unit + units, ... below sk_dp_tiles), then
            // this unit's share of the split iterations, last piece first: a
            // piece that ends inside its tile (its partial sum goes to the
            // workspace) is done before the pieces that finish tiles.
            if (next < p.sk_dp_tiles) {
                const int idx = next;
                next += stride;
                int m_tile;
                raster(p, idx, m_tile, t.n_blk);
                t.row0 = m_tile * TILE_M + rank * BM;
                t.g = 0;
                return true;
            }
            if (next != 0x7fffffff) {   // entering the split part: set up the range
                next = 0x7fffffff;
                sk_lo = sk_start(p, unit_, units_);
                sk_cur = sk_start(p, unit_ + 1, units_);
            }
            if (sk_cur <= sk_lo) return false;
            const long long last = sk_cur - 1;
            const int tile = static_cast<int>(last / p.KB);
            const long long tile_start = static_cast<long long>(tile) * p.KB;
            const long long b = max(sk_lo, tile_start);
            t.kb0 = static_cast<int>(b - tile_start);
            t.kb1 = static_cast<int>(sk_cur - tile_start);
            sk_cur = b;
            if (t.kb0 > 0 && t.kb1 == p.KB) {
                // The unit holding this tile's first iteration: the largest u
                // with sk_start(u) <= tile_start.
                int u = static_cast<int>(tile_start * units_ / max(1ll, p.sk_iters));
                while (u + 1 < units_ && sk_start(p, u + 1, units_) <= tile_start) ++u;
                while (u > 0 && sk_start(p, u, units_) > tile_start) --u;
                t.sk_first = u;
            }
            int m_tile;
            raster(p, p.sk_dp_tiles + tile, m_tile, t.n_blk);
            t.row0 = m_tile * TILE_M + rank * BM;
            t.g = 0;
            return true;
        }
        if (p.layout == LAYOUT_MASKED) {
            const int idx = next;
            while (true) {
                if (mg >= p.G) return false;
                if (mtiles < 0) {
                    int mm = __ldg(p.masked_m + mg);
                    mm = mm < 0 ? 0 : (mm > p.rows ? p.rows : mm);
                    mtiles_m = ceil_div_c(mm, TILE_M);
                    mtiles = mtiles_m * p.num_n_blocks;
                }
                if (idx < mbase + mtiles) break;
                mbase += mtiles;
                ++mg;
                mtiles = -1;
            }
            const int local = idx - mbase;
            t.g = mg;
            t.row0 = (local % mtiles_m) * TILE_M + rank * BM;   // row tiles of one column block run side by side
            t.n_blk = local / mtiles_m;
            next += stride;
            return true;
        }
        if (PAIR && p.layout == LAYOUT_CONTIGUOUS) {
            const int total = pair_count * p.num_n_blocks;
            if (next >= total) return false;
            const int idx = next;
            next += stride;
            const int per_group = p.raster_m * p.num_n_blocks;
            const int grp = idx / per_group;
            const int first_m = grp * p.raster_m;
            const int gm = min(p.raster_m, pair_count - first_m);
            const int local = idx - grp * per_group;
            const int blk = pair_list[first_m + local % gm];
            t.n_blk = local / gm;
            t.row0 = (blk + rank) * BM;
            t.g = __ldg(p.m_indices + blk * BM);
            return true;
        }
        const int total = p.num_m_tiles * p.num_n_blocks;
        while (next < total) {
            const int idx = next;
            next += stride;
            const int per_group = p.raster_m * p.num_n_blocks;
            const int grp = idx / per_group;
            const int first_m = grp * p.raster_m;
            const int gm = min(p.raster_m, p.num_m_tiles - first_m);
            const int local = idx - grp * per_group;
            const int m_tile = first_m + local % gm;
            t.n_blk = local / gm;
            t.row0 = m_tile * TILE_M + rank * BM;
            t.g = 0;
            if (p.layout == LAYOUT_CONTIGUOUS) {
                const int e = __ldg(p.m_indices + m_tile * BM);
                if (e < 0 || e >= p.G) continue;   // a block of padding rows only: nothing to do
                t.g = e;
            }
            return true;
        }
        return false;
    }
};

// Wait result: 0 = completed, 1 = another role aborted, 2 = this wait timed out.
// The thread is parked by the hardware (mbarrier suspend hint, at most 1 ms per
// try) rather than spinning, so waiting roles take no issue slots or shared
// memory bandwidth from the MMA; the abort flag and the time limit are checked
// each time a try expires.
__device__ __forceinline__ int wait_bar(uint64_t* bar, uint32_t parity, uint64_t limit_ns, volatile int* abort_flag) {
    if (ptx::mbar_test_wait(bar, parity)) return 0;   // fast path: the phase is already complete
    const uint32_t hint = limit_ns < 1000000ull ? static_cast<uint32_t>(limit_ns) : 1000000u;
    if (ptx::mbar_try_wait_suspend(bar, parity, hint)) return 0;
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
        if (ptx::mbar_try_wait_suspend(bar, parity, hint)) return 0;
        if (*abort_flag) return 1;
        if (ptx::globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            return 2;
        }
    }
}

__device__ __forceinline__ void record_error(int* status, int code, int role) {
    if (atomicCAS(status, 0, code) == 0) status[1] = (static_cast<int>(blockIdx.x) << 8) | role;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Contiguous layout with CTA pairs: list, in row order, the 128-row blocks that
// start a pair tile.  A pair starts at every even offset of a run of blocks
// carrying the same expert tag (tag of a block = tag of its first row); the
// second block of a pair may belong to another expert or be padding, and then
// that CTA's rows are simply not stored.  Run by warp 0; `tags` is scratch
// shared memory for one int per block.  Returns the number of pairs.
__device__ __forceinline__ int build_pair_list(const GemmParams& p, int* tags, uint16_t* list) {
    const int lane = threadIdx.x % 32;
    const int nblk = p.rows / BM;
    for (int b = lane; b < nblk; b += 32) {
        const int e = __ldg(p.m_indices + b * BM);
        tags[b] = (e < 0 || e >= p.G) ? -1 : e;
    }
    __syncwarp();
    int count = 0;
    for (int base = 0; base < nblk; base += 32) {
        const int b = base + lane;
        bool start = false;
        if (b < nblk && tags[b] >= 0) {
            int run = 0;   // blocks of the same tag directly before b
            while (b - run - 1 >= 0 && tags[b - run - 1] == tags[b]) ++run;
            start = (run % 2) == 0;
        }
        const uint32_t mask = __ballot_sync(0xffffffffu, start);
        const int pos = count + __popc(mask & ((1u << lane) - 1u));
        if (start && pos < MAX_PAIR_LIST) list[pos] = static_cast<uint16_t>(b);
        count += __popc(mask);
    }
    return count < MAX_PAIR_LIST ? count : MAX_PAIR_LIST;
}

// BF16 pair of (lo, hi), round to nearest even, as one 32-bit word.
__device__ __forceinline__ uint4 pack_bf16x8(const float2 (&a)[8], int q) {
    uint4 v;
    v.x = pack_bf16x2(a[4 * q + 0].x, a[4 * q + 0].y);
    v.y = pack_bf16x2(a[4 * q + 1].x, a[4 * q + 1].y);
    v.z = pack_bf16x2(a[4 * q + 2].x, a[4 * q + 2].y);
    v.w = pack_bf16x2(a[4 * q + 3].x, a[4 * q + 3].y);
    return v;
}

template <int BN, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fg8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmD, const GemmParams p) {
    using S = GemmShape<BN, PAIR>;
    constexpr int NC = S::NC;
    constexpr int CPW = S::CPW;
    constexpr int PB = CPW <= 2 ? CPW : 2;   // chunks per TMEM load batch of the promotion pipeline
    constexpr int NBATCH = (CPW + PB - 1) / PB;
    constexpr uint32_t IDESC = ptx::idesc_e4m3_f32(S::TILE_M, BN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_base = smem;
    uint8_t* epi_base = smem + static_cast<size_t>(p.stages) * S::STAGE_BYTES;
    uint16_t* pair_list = reinterpret_cast<uint16_t*>(epi_base + NUM_EPI_WARPS * EPI_WARP_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(pair_list) + (PAIR ? PAIR_LIST_BYTES : 0));
    uint64_t* empty = full + p.stages;
    uint64_t* tfull = empty + p.stages;
    uint64_t* tempty = tfull + S::NBUF;
    uint64_t* done_bar = tempty + S::NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* pair_count_slot = reinterpret_cast<int*>(tmem_slot + 2);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = p.wait_limit_ns;
    const uint64_t drain_limit = 2000000000ull;   // 2 s: copies in flight always finish
    const int rank = PAIR ? static_cast<int>(ptx::cluster_ctarank()) : 0;
    const bool leader = rank == 0;
    const int unit = PAIR ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
    const int num_units = PAIR ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);

    if (warp == PRODUCER_WARP && lane == 0) {
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < S::NBUF; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], S::TEMPTY_COUNT);
        }
        ptx::mbar_init(done_bar, NUM_MMA_WARPS);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
        ptx::prefetch_tensormap(&tmA);
        ptx::prefetch_tensormap(&tmB);
        ptx::prefetch_tensormap(&tmD);
    }
    if (warp == MMA_WARP) {
        if constexpr (PAIR) {
            ptx::tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
            ptx::tmem_relinquish_pair();
        } else {
            ptx::tmem_alloc(tmem_slot, S::TMEM_COLS);
            ptx::tmem_relinquish();
        }
    }
    // Everything above touched only this CTA's own memory; global memory is
    // read or written only after the grids this launch depends on are done.
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    if (PAIR && p.layout == LAYOUT_CONTIGUOUS && warp == 0) {
        // The stage ring is free until the roles start: use it for the tags.
        const int n = build_pair_list(p, reinterpret_cast<int*>(stage_base), pair_list);
        if (lane == 0) *pair_count_slot = n;
    }
    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) ptx::cluster_sync();   // peer barriers initialised, TMEM of both CTAs allocated
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int pair_count = (PAIR && p.layout == LAYOUT_CONTIGUOUS) ? *pair_count_slot : 0;

    if (warp >= NUM_EPI_WARPS) {
      ptx::setmaxnreg_dec<REGS_PRODUCER>();
      if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            TileScheduler<PAIR> sch(unit, num_units, rank, pair_list, pair_count);
            TileInfo t;
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;           // loads issued so far (for the drain below)
            // Normal layout: every A row panel is read by all column blocks and
            // each B panel by only the row tiles of one raster group, so A is
            // kept in L2 in preference to B (measured: 2-3 % on the prefill
            // shapes).  The grouped layouts reuse B across an expert's row
            // tiles and keep the default policy.
            const bool hinted = p.layout == LAYOUT_NORMAL;
            const uint64_t pol_a = ptx::policy_evict_last();
            const uint64_t pol_b = ptx::policy_evict_first();
            int w = 0;
            while (w == 0 && sch.get(p, t)) {
                const int a_g = p.layout == LAYOUT_MASKED ? t.g : 0;
                const int b_row = t.n_blk * BN + rank * S::BNL;
                for (int kb = t.kb0; kb < t.kb1; ++kb) {
                    w = wait_bar(&empty[stage], phase ^ 1u, limit, abort_flag);
                    if (w) break;
                    uint8_t* sa = stage_base + static_cast<size_t>(stage) * S::STAGE_BYTES;
                    if constexpr (PAIR) {
                        // Both CTAs' loads complete on the leader's full barrier.
                        const uint32_t bar = ptx::mapa_shared(ptx::smem_addr(&full[stage]), 0);
                        if (leader) ptx::mbar_arrive_expect_tx(&full[stage], S::TX_BYTES);
                        if (hinted) {
                            ptx::tma_load_3d_pair_hint(sa, &tmA, bar, kb * BK, t.row0, a_g, pol_a);
                            ptx::tma_load_3d_pair_hint(sa + A_TILE_BYTES, &tmB, bar, kb * BK, b_row, t.g, pol_b);
                        } else {
                            ptx::tma_load_3d_pair(sa, &tmA, bar, kb * BK, t.row0, a_g);
                            ptx::tma_load_3d_pair(sa + A_TILE_BYTES, &tmB, bar, kb * BK, b_row, t.g);
                        }
                    } else {
                        ptx::mbar_arrive_expect_tx(&full[stage], S::TX_BYTES);
                        if (hinted) {
                            ptx::tma_load_3d_hint(sa, &tmA, &full[stage], kb * BK, t.row0, a_g, pol_a);
                            ptx::tma_load_3d_hint(sa + A_TILE_BYTES, &tmB, &full[stage], kb * BK, b_row, t.g, pol_b);
                        } else {
                            ptx::tma_load_3d(sa, &tmA, &full[stage], kb * BK, t.row0, a_g);
                            ptx::tma_load_3d(sa + A_TILE_BYTES, &tmB, &full[stage], kb * BK, b_row, t.g);
                        }
                    }
                    ++issued;
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (w == 2) record_error(p.status, ERR_TIMEOUT, ROLE_PRODUCER);
            if (!PAIR || leader) {
                // Let every copy still in flight land before the CTA can exit:
                // walk back over the last p.stages loads (stage, parity).
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < p.stages && issued - 1 - i >= 0; ++i) {
                    if (s == 0) {
                        s = p.stages - 1;
                        ph ^= 1u;
                    } else {
                        --s;
                    }
                    ptx::mbar_wait(&full[s], ph, drain_limit);
                }
            } else if (w != 0) {
                // The peer's loads complete on the leader's barriers, which it
                // cannot wait on: after an abort give them time to land.
                for (int i = 0; i < 200; ++i) __nanosleep(1000);
            }
        }
      } else if (warp < MMA_WARP + NUM_MMA_WARPS) {
        // K blocks are independent (each accumulates into its own TMEM buffer),
        // so NUM_MMA_WARPS issuers take turns: issuer j handles the global
        // K-block sequence numbers g with g % NUM_MMA_WARPS == j.  This hides
        // the long per-thread latency of the barrier waits, the fence and each
        // tcgen05 issue behind another issuer's work.
        const int j = warp - MMA_WARP;
        if (lane == 0 && (!PAIR || leader)) {
            TileScheduler<PAIR> sch(unit, num_units, rank, pair_list, pair_count);
            TileInfo t;
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            int w = 0;
            int g = 0;
            while (w == 0 && sch.get(p, t)) {
                for (int kb = t.kb0; kb < t.kb1; ++kb, ++g) {
                    if (g % NUM_MMA_WARPS == j) {
                        // The stage is normally loaded long before the accumulator
                        // is released: wait for it first, so that nothing but the
                        // fence stands between the release and the first MMA.
                        w = wait_bar(&full[stage], phase, limit, abort_flag);
                        if (w) break;
                        w = wait_bar(&tempty[buf], bphase ^ 1u, limit, abort_flag);
                        if (w) break;
                        ptx::tc_fence_after();
                        const uint32_t a_addr =
                            ptx::smem_addr(stage_base + static_cast<size_t>(stage) * S::STAGE_BYTES);
                        const uint64_t adesc = ptx::smem_desc_sw128(a_addr);
                        const uint64_t bdesc = ptx::smem_desc_sw128(a_addr + A_TILE_BYTES);
                        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * S::ACC_STRIDE);
#pragma unroll
                        for (int k = 0; k < BK / 32; ++k) {
                            // K step k: 32 E4M3 = 32 bytes further along the swizzled 128-byte row.
                            if constexpr (PAIR)
                                ptx::mma_f8f6f4_pair(d_tmem, adesc + static_cast<uint64_t>(k * 2),
                                                     bdesc + static_cast<uint64_t>(k * 2), IDESC, k > 0 ? 1u : 0u);
                            else
                                ptx::mma_f8f6f4(d_tmem, adesc + static_cast<uint64_t>(k * 2),
                                                bdesc + static_cast<uint64_t>(k * 2), IDESC, k > 0 ? 1u : 0u);
                        }
                        if constexpr (PAIR) {
                            ptx::mma_commit_pair(&empty[stage], 0x3);
                            ptx::mma_commit_pair(&tfull[buf], 0x3);
                        } else {
                            ptx::mma_commit(&empty[stage]);
                            ptx::mma_commit(&tfull[buf]);
                        }
                    }
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++buf == S::NBUF) {
                        buf = 0;
                        bphase ^= 1u;
                    }
                }
            }
            if (w == 2) record_error(p.status, ERR_TIMEOUT, ROLE_MMA);
            // Every MMA issued above must finish before TMEM is released
            // (done_bar completes once every issuer's commit has arrived).
            if constexpr (PAIR) ptx::mma_commit_pair(done_bar, 0x1);
            else ptx::mma_commit(done_bar);
            ptx::mbar_wait(done_bar, 0, drain_limit);
        }
      }
    } else {
        ptx::setmaxnreg_inc<REGS_PROMOTION>();
        // ---- promotion + epilogue: warps 0..7 ----
        const int wg = warp / 4;
        const int quarter = warp % 4;                 // TMEM lanes 32*quarter .. +31
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int chunk0 = wg * CPW;                  // first 16-column chunk of this warpgroup
        uint8_t* stg = epi_base + warp * EPI_WARP_BYTES;
        const uint32_t tempty_peer0 = PAIR ? ptx::mapa_shared(ptx::smem_addr(&tempty[0]), 0) : 0u;

        // The tile sequence is only needed between tiles: lane 0 walks it with
        // its state in shared memory and hands each tile to the warp by
        // shuffles, which keeps the registers for the accumulators.
        __shared__ TileScheduler<PAIR> sched_store[NUM_EPI_WARPS];
        if (lane == 0) sched_store[warp].init(unit, num_units, rank, pair_list, pair_count);
        TileInfo t;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        while (ok) {
            int has = 0;
            if (lane == 0) has = sched_store[warp].get(p, t) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, has, 0)) break;
            t.g = __shfl_sync(0xffffffffu, t.g, 0);
            t.row0 = __shfl_sync(0xffffffffu, t.row0, 0);
            t.n_blk = __shfl_sync(0xffffffffu, t.n_blk, 0);
            t.kb0 = __shfl_sync(0xffffffffu, t.kb0, 0);
            t.kb1 = __shfl_sync(0xffffffffu, t.kb1, 0);
            t.sk_first = __shfl_sync(0xffffffffu, t.sk_first, 0);
            const int row = t.row0 + row_in_tile;
            const int n0 = t.n_blk * BN;
            // Scale block of this warpgroup's chunks: nb_lo for the first chunk,
            // nb_hi for the chunks whose bit is set in hi_mask (a warpgroup spans
            // <= 128 columns, so at most two blocks).  Block widths that are
            // multiples of 128 start every tile on a block boundary, so a
            // warpgroup then lies in a single block.  Blocks past the last one
            // (columns >= N, never stored) are clamped to it.
            const int nb_lo = min((n0 + chunk0 * 16) / 128, p.NB - 1);
            const int nb_hi = min(nb_lo + 1, p.NB - 1);
            uint32_t hi_mask = 0;
            if constexpr (BN % 128 != 0) {
#pragma unroll
                for (int i = 0; i < CPW; ++i)
                    if ((n0 + (chunk0 + i) * 16) / 128 > (n0 + chunk0 * 16) / 128) hi_mask |= 1u << i;
            }
            // This row's sfa (rows past the padded scale array read nothing:
            // they are never stored) and the warpgroup's sfb rows.
            const int a_g = p.layout == LAYOUT_MASKED ? t.g : 0;
            const bool row_has_scale = row < p.sfa_ld;
            const float* sfa_row = p.sfa + static_cast<size_t>(a_g) * p.KB * p.sfa_ld + (row_has_scale ? row : 0);
            const float* sfb_lo = p.sfb + (static_cast<size_t>(t.g) * p.NB + nb_lo) * p.KB;
            const float* sfb_hi = p.sfb + (static_cast<size_t>(t.g) * p.NB + nb_hi) * p.KB;

            // Column pairs: the promotion uses the packed FP32 FMA (two FMAs per
            // instruction, each rounded to nearest as a scalar fmaf would be).
            float2 acc[CPW][8];
#pragma unroll
            for (int i = 0; i < CPW; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = make_float2(0.0f, 0.0f);

            // Scales: the raw values of the next group of SCALE_GROUP K blocks are
            // loaded while the current group is promoted (their latency is
            // hidden behind a group's MMAs); at the group switch they become
            // the per-K-block factors sfa * sfb of the current group.  With two
            // accumulators the promotion's latency bounds the tensor core's
            // rate, so no load or shared-memory access of scales sits between
            // an accumulator's completion and its release.
            float na[SCALE_GROUP], nl[SCALE_GROUP], nh[SCALE_GROUP];
#define FG8_LOAD_SCALE_GROUP(KG)                                                                      \
    _Pragma("unroll") for (int u = 0; u < SCALE_GROUP; ++u) {                                         \
        const int kq = min((KG) + u, p.KB - 1);                                                       \
        na[u] = row_has_scale ? __ldg(sfa_row + static_cast<size_t>(kq) * p.sfa_ld) : 0.0f;           \
        nl[u] = __ldg(sfb_lo + kq);                                                                   \
        nh[u] = (BN % 128 == 0) ? 0.0f : __ldg(sfb_hi + kq);                                          \
    }
            if (row_has_scale) {
                for (int kq = t.kb0 + SCALE_GROUP; kq < min(t.kb1, t.kb0 + SCALE_PREFETCH); ++kq)
                    ptx::prefetch_l1(sfa_row + static_cast<size_t>(kq) * p.sfa_ld);
            }
            FG8_LOAD_SCALE_GROUP(t.kb0)
            int w = 0;
            // A kernel compiled for one shape knows the K blocks of a whole tile.
            const int kb_end = (FG8_KB_CT > 0 && !p.sk) ? FG8_KB_CT : t.kb1;
            for (int kg = t.kb0; kg < kb_end && w == 0; kg += SCALE_GROUP) {
                float s_lo[SCALE_GROUP], s_hi[SCALE_GROUP];
#pragma unroll
                for (int u = 0; u < SCALE_GROUP; ++u) {
                    s_lo[u] = na[u] * nl[u];
                    s_hi[u] = (BN % 128 == 0) ? s_lo[u] : na[u] * nh[u];
                }
                if (kg + SCALE_GROUP < kb_end) {
                    FG8_LOAD_SCALE_GROUP(kg + SCALE_GROUP)
                }
                // sfa is a new 512-byte slice per K block: bring the slices of
                // SCALE_PREFETCH K blocks ahead into L1 so that the loads above
                // find them there instead of waiting on L2 behind the operand
                // traffic.
                if (row_has_scale) {
#pragma unroll
                    for (int u = 0; u < SCALE_GROUP; ++u)
                        if (kg + SCALE_PREFETCH + u < kb_end)
                            ptx::prefetch_l1(sfa_row + static_cast<size_t>(kg + SCALE_PREFETCH + u) * p.sfa_ld);
                }
#undef FG8_LOAD_SCALE_GROUP
#pragma unroll
                for (int u = 0; u < SCALE_GROUP; ++u) {
                    if (kg + u >= kb_end) break;
                    if (lane == 0) w = wait_bar(&tfull[buf], bphase, limit, abort_flag);
                    w = __shfl_sync(0xffffffffu, w, 0);
                    if (w) break;
                    ptx::tc_fence_after();
                    const uint32_t tbase = tmem_base + lane_base + static_cast<uint32_t>(buf * S::ACC_STRIDE);
                    // Software pipeline over batches of PB chunks: the TMEM loads of
                    // batch q + 1 are in flight while batch q is scaled and added
                    // (tcgen05.wait::ld waits for all of a thread's loads, so only
                    // one batch is ever outstanding), and the accumulator is released
                    // to the MMA issuers as soon as its last batch is in registers.
                    uint32_t r[2][PB][16];
#pragma unroll
                    for (int b = 0; b < PB; ++b) {
                        const int c = chunk0 + b;
                        if (b < CPW && c < NC) ptx::tmem_ld16(tbase + static_cast<uint32_t>(c * 16), r[0][b]);
                    }
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int b = 0; b < PB; ++b) ptx::reg_fence(r[0][b]);
                    if (NBATCH == 1) {
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (PAIR) ptx::mbar_arrive_cluster(tempty_peer0 + static_cast<uint32_t>(buf * 8));
                            else ptx::mbar_arrive(&tempty[buf]);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < NBATCH; ++q) {
                        if (q + 1 < NBATCH) {
#pragma unroll
                            for (int b = 0; b < PB; ++b) {
                                const int c = chunk0 + (q + 1) * PB + b;
                                if ((q + 1) * PB + b < CPW && c < NC)
                                    ptx::tmem_ld16(tbase + static_cast<uint32_t>(c * 16), r[(q + 1) & 1][b]);
                            }
                        }
#pragma unroll
                        for (int b = 0; b < PB; ++b) {
                            const int i = q * PB + b;
                            const int c = chunk0 + i;
                            if (i < CPW && c < NC) {
                                const float sc = (BN % 128 == 0) ? s_lo[u] : (((hi_mask >> i) & 1u) ? s_hi[u] : s_lo[u]);
                                const float2 sc2 = make_float2(sc, sc);
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const float2 v = make_float2(__uint_as_float(r[q & 1][b][2 * j]),
                                                                 __uint_as_float(r[q & 1][b][2 * j + 1]));
                                    acc[i < CPW ? i : 0][j] = __ffma2_rn(v, sc2, acc[i < CPW ? i : 0][j]);
                                }
                            }
                        }
                        if (q + 1 < NBATCH) {
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int b = 0; b < PB; ++b) ptx::reg_fence(r[(q + 1) & 1][b]);
                            if (q + 2 == NBATCH) {
                                // Every partial sum of this K block is in registers.
                                ptx::tc_fence_before();
                                __syncwarp();
                                if (lane == 0) {
                                    if constexpr (PAIR) ptx::mbar_arrive_cluster(tempty_peer0 + static_cast<uint32_t>(buf * 8));
                                    else ptx::mbar_arrive(&tempty[buf]);
                                }
                            }
                        }
                    }
                    if (++buf == S::NBUF) {
                        buf = 0;
                        bphase ^= 1u;
                    }
                }
            }
            if (w) {
                if (w == 2 && lane == 0) record_error(p.status, ERR_TIMEOUT, ROLE_EPILOGUE);
                ok = false;
                break;
            }

            if (!PAIR && p.ks > 1) {
                // Cluster split-K: stage this split's FP32 partial in the (now
                // idle) stage ring as [chunk][row][16]; the cluster reduction
                // after the role branches writes D.
                float* part = reinterpret_cast<float*>(stage_base);
#pragma unroll
                for (int i = 0; i < CPW; ++i) {
                    const int c = chunk0 + i;
                    if (c >= NC) break;
                    float4* dst = reinterpret_cast<float4*>(part + (static_cast<size_t>(c) * BM + row_in_tile) * 16);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_float4(acc[i][2 * q].x, acc[i][2 * q].y, acc[i][2 * q + 1].x, acc[i][2 * q + 1].y);
                }
                continue;
            }

            // ---- stream-K: publish a partial sum, or add the earlier ones ----
            if (t.kb1 < p.KB) {
                // This piece ends inside its tile: store its FP32 partial sum in
                // this CTA's workspace slice and publish it with the epoch.
                float* ws = p.sk_ws + static_cast<size_t>(blockIdx.x) * NC * BM * 16;
#pragma unroll
                for (int i = 0; i < CPW; ++i) {
                    const int c = chunk0 + i;
                    if (c >= NC) break;
                    float4* dst = reinterpret_cast<float4*>(ws + (static_cast<size_t>(c) * BM + row_in_tile) * 16);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        __stcg(dst + q, make_float4(acc[i][2 * q].x, acc[i][2 * q].y, acc[i][2 * q + 1].x,
                                                    acc[i][2 * q + 1].y));
                }
                // Each warp publishes its own rows x columns: the warp of the same
                // position in the finishing CTA waits for exactly this flag, so no
                // warp waits on another warp of its own CTA.
                __threadfence();
                __syncwarp();
                if (lane == 0) ptx::st_release_gpu(p.sk_flags + blockIdx.x * NUM_EPI_WARPS + warp, p.sk_epoch);
                continue;
            }
            if (t.sk_first >= 0) {
                // This piece finishes its tile: add the partial sums of the units
                // that did its first K blocks, in unit order (deterministic).
                const int my_unit = PAIR ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
                for (int u = t.sk_first; u < my_unit && ok; ++u) {
                    // A unit with no split iterations published nothing.
                    if (TileScheduler<PAIR>::sk_start(p, u, num_units) == TileScheduler<PAIR>::sk_start(p, u + 1, num_units))
                        continue;
                    const int cta = PAIR ? 2 * u + rank : u;
                    const unsigned* flag = p.sk_flags + cta * NUM_EPI_WARPS + warp;
                    int w2 = 0;
                    if (lane == 0) {
                        const uint64_t t0 = ptx::globaltimer();
                        while (ptx::ld_acquire_gpu(flag) != p.sk_epoch) {
                            if (*abort_flag) {
                                w2 = 1;
                                break;
                            }
                            if (ptx::globaltimer() - t0 > limit) {
                                *abort_flag = 1;
                                w2 = 2;
                                break;
                            }
                        }
                    }
                    w2 = __shfl_sync(0xffffffffu, w2, 0);
                    if (w2) {
                        if (w2 == 2 && lane == 0) record_error(p.status, ERR_TIMEOUT, ROLE_EPILOGUE);
                        ok = false;
                        break;
                    }
                    (void)ptx::ld_acquire_gpu(flag);   // every lane acquires the published partial
                    const float* ws = p.sk_ws + static_cast<size_t>(cta) * NC * BM * 16;
#pragma unroll
                    for (int i = 0; i < CPW; ++i) {
                        const int c = chunk0 + i;
                        if (c >= NC) break;
                        const float4* src =
                            reinterpret_cast<const float4*>(ws + (static_cast<size_t>(c) * BM + row_in_tile) * 16);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 v = __ldcg(src + q);
                            acc[i][2 * q].x += v.x;
                            acc[i][2 * q].y += v.y;
                            acc[i][2 * q + 1].x += v.z;
                            acc[i][2 * q + 1].y += v.w;
                        }
                    }
                }
                if (!ok) break;
            }

            // ---- epilogue: BF16 (round to nearest even), rows that may be written only ----
            bool row_ok;
            if (p.layout == LAYOUT_NORMAL) {
                row_ok = row < p.rows;
            } else if (p.layout == LAYOUT_CONTIGUOUS) {
                row_ok = row < p.rows && __ldg(p.m_indices + row) == t.g;
            } else {
                int mm = __ldg(p.masked_m + t.g);
                mm = mm > p.rows ? p.rows : mm;
                row_ok = row < mm;
            }
            const uint32_t rows_mask = __ballot_sync(0xffffffffu, row_ok);
            if (rows_mask == 0u) continue;
            const int warp_row0 = t.row0 + quarter * 32;
            const int d_g = p.layout == LAYOUT_MASKED ? t.g : 0;
            // The staging slots may still be read by this warp's stores of the
            // previous tile.
            if (lane == 0) ptx::bulk_wait_group_read<0>();
            __syncwarp();
            const int sw = (lane >> 2) & 1;
            // The D tensor map clips rows >= its row count and columns >= N, so a
            // warp whose rows are all writable, or (normal layout) whose only
            // unwritable rows lie past M, stores whole 32 x 16 pieces by TMA.
            const bool bulk = rows_mask == 0xffffffffu || p.layout == LAYOUT_NORMAL;
            if (bulk) {
#pragma unroll
                for (int i = 0; i < CPW; ++i) {
                    const int c = chunk0 + i;
                    if (c >= NC || n0 + c * 16 >= p.N) break;
                    uint8_t* piece = stg + (i & 1) * EPI_SLOT_BYTES;
                    if (i >= EPI_SLOTS) {
                        if (lane == 0) ptx::bulk_wait_group_read<EPI_SLOTS - 1>();
                        __syncwarp();
                    }
                    *reinterpret_cast<uint4*>(piece + lane * 32 + (0 ^ sw) * 16) = pack_bf16x8(acc[i], 0);
                    *reinterpret_cast<uint4*>(piece + lane * 32 + (1 ^ sw) * 16) = pack_bf16x8(acc[i], 1);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        ptx::tma_store_3d(&tmD, piece, n0 + c * 16, warp_row0, d_g);
                        ptx::bulk_commit_group();
                    }
                }
            } else {
                __nv_bfloat16* Dg = p.D + static_cast<size_t>(d_g) * p.rows * p.N;
#pragma unroll
                for (int i = 0; i < CPW; ++i) {
                    const int c = chunk0 + i;
                    if (c >= NC || n0 + c * 16 >= p.N) break;
                    uint8_t* piece = stg;
                    *reinterpret_cast<uint4*>(piece + lane * 32 + (0 ^ sw) * 16) = pack_bf16x8(acc[i], 0);
                    *reinterpret_cast<uint4*>(piece + lane * 32 + (1 ^ sw) * 16) = pack_bf16x8(acc[i], 1);
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int u = lane + 32 * q;     // 16-byte unit: row u / 2, half u % 2
                        const int r = u >> 1;
                        const int h = u & 1;
                        if ((rows_mask >> r) & 1u) {
                            const uint4 v = *reinterpret_cast<const uint4*>(piece + r * 32 + (h ^ ((r >> 2) & 1)) * 16);
                            *reinterpret_cast<uint4*>(Dg + static_cast<size_t>(warp_row0 + r) * p.N + n0 + c * 16 + h * 8) = v;
                        }
                    }
                    __syncwarp();
                }
            }
        }
        // Every bulk store of this warp must be complete before the CTA exits.
        if (lane == 0) ptx::bulk_wait_group<0>();
    }

    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) ptx::cluster_sync();   // the leader's MMAs read the peer's shared memory until here
    if (!PAIR && p.ks > 1) {
        // Cluster split-K: once every split of the tile has staged its partial,
        // CTA r of the cluster sums a slice of the tile's rows over all splits
        // in split order (deterministic), reading the peers' shared memory, and
        // writes them as BF16; the second barrier keeps each CTA's partial
        // alive until its peers have read it.  Every thread takes both
        // barriers, also after an abort.
        ptx::cluster_sync();
        if (warp < NUM_EPI_WARPS && !*abort_flag) {
            const int S = p.ks;
            const int r = static_cast<int>(ptx::cluster_ctarank());
            int m_tile, n_blk;
            TileScheduler<PAIR>::raster(p, static_cast<int>(blockIdx.x) / S, m_tile, n_blk);
            const int row0 = m_tile * BM;
            const int n0 = n_blk * BN;
            const int rows = min(BM, p.rows - row0);
            const int rs = (rows + S - 1) / S;
            const int r0 = min(rows, r * rs);
            const int r1 = min(rows, r0 + rs);
            constexpr int Q = BN / 4;                         // 4-column groups of a row
            const uint32_t base = ptx::smem_addr(stage_base);
            for (int e = threadIdx.x; e < (r1 - r0) * Q; e += NUM_EPI_WARPS * 32) {
                const int row = r0 + e / Q;
                const int col = (e - (e / Q) * Q) * 4;
                const int n = n0 + col;
                if (n >= p.N) continue;                        // N % 16 == 0: the 4 columns are all in range
                const uint32_t off =
                    base + static_cast<uint32_t>((((col >> 4) * BM + row) * 16 + (col & 15)) * 4);
                // All splits' loads in flight together, then the sum in split order.
                float4 v[8];
#pragma unroll
                for (int sp = 0; sp < 8; ++sp)
                    if (sp < S) v[sp] = ptx::ld_shared_cluster_v4(ptx::mapa_shared(off, static_cast<uint32_t>(sp)));
                float4 sum = v[0];
#pragma unroll
                for (int sp = 1; sp < 8; ++sp) {
                    if (sp < S) {
                        sum.x += v[sp].x;
                        sum.y += v[sp].y;
                        sum.z += v[sp].z;
                        sum.w += v[sp].w;
                    }
                }
                uint2 pk;
                pk.x = pack_bf16x2(sum.x, sum.y);
                pk.y = pack_bf16x2(sum.z, sum.w);
                *reinterpret_cast<uint2*>(p.D + static_cast<size_t>(row0 + row) * p.N + n) = pk;
            }
        }
        ptx::cluster_sync();
    }
    if (warp == MMA_WARP) {
        ptx::tc_fence_after();
        if constexpr (PAIR) ptx::tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
        else ptx::tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
}

}  // namespace fg8
