// gemm_kernel.cuh -- persistent fine-grained-scaled FP8 GEMM for sm_100a.
//
// Computes, for each output tile of BM x BN,
//   D[m,n] = bf16( sum_kb (A_kb . B_kb^T)[m,n] * sfa[m,kb] * sfb[n/128,kb] )
// which is the fine-grained ("DeepSeek-V3 style") scaling of the pages
// (chujupifa.com "机器之心报道", opening summary; deepseek.csdn.net
// "DeepGEMM：简洁、高效…", section "什么是DeepGEMM呢？") with the two-level
// accumulation they describe (each 128-wide K block is accumulated by the
// tensor core, then scaled and added into FP32 on the CUDA cores;
// chujupifa.com report, opening summary; ai.abqq.net, section 1 "架构优化").
//
// B200 design (not the pages' Hopper design):
//   warp 8     TMA producer: one lane streams A [128 x 128] and B [BN x 128]
//              E4M3 tiles into an S-stage shared-memory ring (128-byte swizzle).
//   warp 9     MMA issuer: one lane issues 4 x tcgen05.mma kind::f8f6f4
//              (M=128, N=BN, K=32) per K block into one of NBUF (2..4) TMEM
//              accumulators, overwriting it at the block's first MMA.
//   warps 0-7  promotion + epilogue: two warpgroups split the tile's 16-column
//              chunks; each thread owns one TMEM lane (= one output row), reads
//              the block's partial sums with tcgen05.ld, multiplies by
//              sfa[m,kb] * sfb[n/128,kb] and adds into FP32 registers, then
//              after the last block converts to BF16 and stores the rows that
//              may be written.
// Tiles are scheduled persistently (static stride over a raster-grouped tile
// order); the contiguous and masked MoE layouts of the pages (game.3loumao.org
// explainer, section "03 DeepSeek是如何创新的？") change only the tile -> (group,
// row block, column block) mapping and which rows are stored.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace fg8 {

constexpr int BM = 128;
constexpr int BK = 128;
constexpr int NUM_EPI_WARPS = 8;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
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
constexpr int EPI_COLS = 32;                       // columns per staged piece
constexpr int EPI_PITCH = EPI_COLS * 2 + 16;       // bytes per staged row (padding kills bank conflicts)
constexpr int EPI_WARP_BYTES = 32 * EPI_PITCH;     // staging bytes per epilogue warp
constexpr int A_TILE_BYTES = BM * BK;              // 16 KiB

enum : int { LAYOUT_NORMAL = 0, LAYOUT_CONTIGUOUS = 1, LAYOUT_MASKED = 2 };

enum : int { ERR_TIMEOUT = 6 };
enum : int { ROLE_PRODUCER = 1, ROLE_MMA = 2, ROLE_EPILOGUE = 3 };

struct GemmParams {
    int layout;
    int rows;          // rows per group: M (normal), M_tot (contiguous), M_max (masked)
    int N, K, G;
    int KB, NB;        // K / 128, ceil(N / 128)
    int num_m_blocks;  // ceil(rows / BM)
    int num_n_blocks;  // ceil(N / BN)
    int raster_m;      // row blocks per raster group
    int stages;
    int sfa_ld;        // M_pad: stride (floats) between K blocks of the MN-major sfa
    const float* sfa;  // [G or 1][KB][sfa_ld]
    const float* sfb;  // [G][NB][KB]
    __nv_bfloat16* D;  // [G or 1][rows][N]
    const int* m_indices;
    const int* masked_m;
    int* status;       // [0] = first error code, [1] = (block << 8) | role
    unsigned long long wait_limit_ns;
};

__host__ __device__ constexpr int ceil_div_c(int a, int b) { return (a + b - 1) / b; }

template <int BN>
struct GemmShape {
    static constexpr int NC = BN / 16;                  // 16-column chunks in a tile
    static constexpr int CPW = (NC + 1) / 2;            // chunks per promotion warpgroup
    static constexpr int B_TILE_BYTES = BN * BK;
    static constexpr int STAGE_BYTES = A_TILE_BYTES + B_TILE_BYTES;
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
    static_assert(NBUF >= 2, "need two accumulators");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "BN must be a multiple of 16 in [16, 256]");
};

// Dynamic shared memory layout (after aligning the base to 1024 bytes):
//   [stages x (A tile | B tile)] [8 x epilogue staging] [barriers] [tmem slot, abort flag]
constexpr int MAX_NBUF = 4;
__host__ __device__ constexpr size_t gemm_smem_bytes(int stage_bytes, int stages) {
    return 1024 + static_cast<size_t>(stages) * stage_bytes + NUM_EPI_WARPS * EPI_WARP_BYTES +
           (2 * stages + 2 * MAX_NBUF + 1) * 8 + 16;
}

struct TileInfo {
    int g;       // group of B / sfb (expert); for the masked layout also of A / D
    int m_blk;
    int n_blk;
};

// Enumerates the tiles of this CTA.  Every role builds its own copy and walks
// the same sequence, so no role has to tell another which tile comes next.
struct TileScheduler {
    int next;
    int mg, mbase, mtiles, mblocks;   // masked layout cursor

    __device__ explicit TileScheduler() : next(blockIdx.x), mg(0), mbase(0), mtiles(-1), mblocks(0) {}

    __device__ bool get(const GemmParams& p, TileInfo& t) {
        if (p.layout == LAYOUT_MASKED) {
            const int idx = next;
            while (true) {
                if (mg >= p.G) return false;
                if (mtiles < 0) {
                    int mm = __ldg(p.masked_m + mg);
                    mm = mm < 0 ? 0 : (mm > p.rows ? p.rows : mm);
                    mblocks = ceil_div_c(mm, BM);
                    mtiles = mblocks * p.num_n_blocks;
                }
                if (idx < mbase + mtiles) break;
                mbase += mtiles;
                ++mg;
                mtiles = -1;
            }
            const int local = idx - mbase;
            t.g = mg;
            t.m_blk = local % mblocks;   // row blocks of one column block run side by side
            t.n_blk = local / mblocks;
            next += gridDim.x;
            return true;
        }
        const int total = p.num_m_blocks * p.num_n_blocks;
        while (next < total) {
            const int idx = next;
            next += gridDim.x;
            const int per_group = p.raster_m * p.num_n_blocks;
            const int grp = idx / per_group;
            const int first_m = grp * p.raster_m;
            const int gm = min(p.raster_m, p.num_m_blocks - first_m);
            const int local = idx - grp * per_group;
            t.m_blk = first_m + local % gm;
            t.n_blk = local / gm;
            t.g = 0;
            if (p.layout == LAYOUT_CONTIGUOUS) {
                const int e = __ldg(p.m_indices + t.m_blk * BM);
                if (e < 0 || e >= p.G) continue;   // a block of padding rows only: nothing to do
                t.g = e;
            }
            return true;
        }
        return false;
    }
};

// Wait result: 0 = completed, 1 = another role aborted, 2 = this wait timed out.
__device__ __forceinline__ int wait_bar(uint64_t* bar, uint32_t parity, uint64_t limit_ns, volatile int* abort_flag) {
    if (ptx::mbar_try_wait(bar, parity)) return 0;
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return 0;
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

template <int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fg8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const GemmParams p) {
    using S = GemmShape<BN>;
    constexpr int NC = S::NC;
    constexpr int CPW = S::CPW;
    constexpr int LB = CPW <= 4 ? CPW : 4;   // chunks read from TMEM per wait
    constexpr uint32_t IDESC = ptx::idesc_e4m3_f32(BM, BN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_base = smem;
    uint8_t* epi_base = smem + static_cast<size_t>(p.stages) * S::STAGE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(epi_base + NUM_EPI_WARPS * EPI_WARP_BYTES);
    uint64_t* empty = full + p.stages;
    uint64_t* tfull = empty + p.stages;
    uint64_t* tempty = tfull + S::NBUF;
    uint64_t* done_bar = tempty + S::NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = p.wait_limit_ns;
    const uint64_t drain_limit = 2000000000ull;   // 2 s: copies in flight always finish

    if (warp == PRODUCER_WARP && lane == 0) {
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < S::NBUF; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], NUM_EPI_WARPS);
        }
        ptx::mbar_init(done_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
        ptx::prefetch_tensormap(&tmA);
        ptx::prefetch_tensormap(&tmB);
    }
    if (warp == MMA_WARP) {
        ptx::tmem_alloc(tmem_slot, S::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp >= NUM_EPI_WARPS) {
      ptx::setmaxnreg_dec<REGS_PRODUCER>();
      if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            TileScheduler sch;
            TileInfo t;
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;           // loads issued so far (for the drain below)
            int w = 0;
            while (w == 0 && sch.get(p, t)) {
                const int a_row = t.m_blk * BM;
                const int a_g = p.layout == LAYOUT_MASKED ? t.g : 0;
                const int b_row = t.n_blk * BN;
                for (int kb = 0; kb < p.KB; ++kb) {
                    w = wait_bar(&empty[stage], phase ^ 1u, limit, abort_flag);
                    if (w) break;
                    uint8_t* sa = stage_base + static_cast<size_t>(stage) * S::STAGE_BYTES;
                    ptx::mbar_arrive_expect_tx(&full[stage], S::STAGE_BYTES);
                    ptx::tma_load_3d(sa, &tmA, &full[stage], kb * BK, a_row, a_g);
                    ptx::tma_load_3d(sa + A_TILE_BYTES, &tmB, &full[stage], kb * BK, b_row, t.g);
                    ++issued;
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (w == 2) record_error(p.status, ERR_TIMEOUT, ROLE_PRODUCER);
            // Let every copy still in flight land before the CTA can exit.
            // The last p.stages loads went to stages stage, stage+1, ... (mod p.stages)
            // with the parity of the fill they belong to.
            {
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < p.stages; ++i) {
                    // walk back: (s, ph) after the loop are those of the oldest of the last loads
                    if (s == 0) {
                        s = p.stages - 1;
                        ph ^= 1u;
                    } else {
                        --s;
                    }
                    if (issued - 1 - i < 0) break;
                    ptx::mbar_wait(&full[s], ph, drain_limit);
                }
            }
        }
      } else if (warp == MMA_WARP) {
        if (lane == 0) {
            TileScheduler sch;
            TileInfo t;
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            int w = 0;
            while (w == 0 && sch.get(p, t)) {
                for (int kb = 0; kb < p.KB; ++kb) {
                    w = wait_bar(&tempty[buf], bphase ^ 1u, limit, abort_flag);
                    if (w) break;
                    ptx::tc_fence_after();
                    w = wait_bar(&full[stage], phase, limit, abort_flag);
                    if (w) break;
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_addr(stage_base + static_cast<size_t>(stage) * S::STAGE_BYTES);
                    const uint64_t adesc = ptx::smem_desc_sw128(a_addr);
                    const uint64_t bdesc = ptx::smem_desc_sw128(a_addr + A_TILE_BYTES);
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * S::ACC_STRIDE);
#pragma unroll
                    for (int j = 0; j < BK / 32; ++j) {
                        // K step j: 32 E4M3 = 32 bytes further along the swizzled 128-byte row.
                        ptx::mma_f8f6f4(d_tmem, adesc + static_cast<uint64_t>(j * 2), bdesc + static_cast<uint64_t>(j * 2),
                                        IDESC, j > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&empty[stage]);
                    ptx::mma_commit(&tfull[buf]);
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
            // Every MMA issued above must finish before TMEM is released.
            ptx::mma_commit(done_bar);
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

        TileScheduler sch;
        TileInfo t;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        while (ok && sch.get(p, t)) {
            const int row = t.m_blk * BM + row_in_tile;
            const bool row_in = row < p.rows;
            const int a_g = p.layout == LAYOUT_MASKED ? t.g : 0;
            const float* sfa_p = p.sfa + static_cast<size_t>(a_g) * p.KB * p.sfa_ld + row;
            const float* sfb_p = p.sfb + static_cast<size_t>(t.g) * p.NB * p.KB;
            const int n0 = t.n_blk * BN;
            const int my_n0 = n0 + chunk0 * 16;
            const int nb_lo = min(my_n0 / 128, p.NB - 1);
            const int nb_hi = min(nb_lo + 1, p.NB - 1);
            const int split_col = (my_n0 / 128 + 1) * 128;   // chunk columns at or past this use nb_hi

            float acc[CPW][16];
#pragma unroll
            for (int i = 0; i < CPW; ++i)
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[i][j] = 0.0f;

            float sa_n = row_in ? __ldg(sfa_p) : 0.0f;
            float sl_n = __ldg(sfb_p + static_cast<size_t>(nb_lo) * p.KB);
            float sh_n = __ldg(sfb_p + static_cast<size_t>(nb_hi) * p.KB);
            for (int kb = 0; kb < p.KB; ++kb) {
                const float sa = sa_n, sl = sl_n, sh = sh_n;
                if (kb + 1 < p.KB) {   // prefetch the next block's scales
                    sa_n = row_in ? __ldg(sfa_p + static_cast<size_t>(kb + 1) * p.sfa_ld) : 0.0f;
                    sl_n = __ldg(sfb_p + static_cast<size_t>(nb_lo) * p.KB + kb + 1);
                    sh_n = __ldg(sfb_p + static_cast<size_t>(nb_hi) * p.KB + kb + 1);
                }
                const float s_lo = sa * sl;
                const float s_hi = sa * sh;
                int w = 0;
                if (lane == 0) w = wait_bar(&tfull[buf], bphase, limit, abort_flag);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (w) {
                    if (w == 2 && lane == 0) record_error(p.status, ERR_TIMEOUT, ROLE_EPILOGUE);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t tbase = tmem_base + lane_base + static_cast<uint32_t>(buf * S::ACC_STRIDE);
                // Read the block's partial sums in batches of LB chunks (one
                // tcgen05.wait::ld per batch), then scale and accumulate.
#pragma unroll
                for (int i0 = 0; i0 < CPW; i0 += LB) {
                    uint32_t r[LB][16];
#pragma unroll
                    for (int b = 0; b < LB; ++b) {
                        const int c = chunk0 + i0 + b;
                        if (i0 + b < CPW && c < NC) ptx::tmem_ld16(tbase + static_cast<uint32_t>(c * 16), r[b]);
                    }
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int b = 0; b < LB; ++b) ptx::reg_fence(r[b]);
#pragma unroll
                    for (int b = 0; b < LB; ++b) {
                        const int i = i0 + b;
                        const int c = chunk0 + i;
                        if (i < CPW && c < NC) {
                            const float sc = (n0 + c * 16 >= split_col) ? s_hi : s_lo;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                acc[i < CPW ? i : 0][j] = fmaf(__uint_as_float(r[b][j]), sc, acc[i < CPW ? i : 0][j]);
                        }
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
                if (++buf == S::NBUF) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
            if (!ok) break;

            // ---- epilogue: BF16 (round to nearest even), rows that may be written only ----
            bool row_ok;
            if (p.layout == LAYOUT_NORMAL) {
                row_ok = row_in;
            } else if (p.layout == LAYOUT_CONTIGUOUS) {
                row_ok = row_in && __ldg(p.m_indices + row) == t.g;
            } else {
                int mm = __ldg(p.masked_m + t.g);
                mm = mm > p.rows ? p.rows : mm;
                row_ok = row < mm;
            }
            const uint32_t rows_mask = __ballot_sync(0xffffffffu, row_ok);
            __nv_bfloat16* Dg = p.D + (p.layout == LAYOUT_MASKED ? static_cast<size_t>(t.g) * p.rows * p.N : 0);
            const int warp_row0 = t.m_blk * BM + quarter * 32;
#pragma unroll
            for (int i = 0; i < CPW; i += 2) {
                const int c0 = chunk0 + i;
                if (c0 >= NC) break;
                const bool has1 = (i + 1 < CPW) && (c0 + 1 < NC);
                uint8_t* myrow = stg + lane * EPI_PITCH;
                {
                    uint4 v0, v1;
                    v0.x = pack_bf16x2(acc[i][0], acc[i][1]);
                    v0.y = pack_bf16x2(acc[i][2], acc[i][3]);
                    v0.z = pack_bf16x2(acc[i][4], acc[i][5]);
                    v0.w = pack_bf16x2(acc[i][6], acc[i][7]);
                    v1.x = pack_bf16x2(acc[i][8], acc[i][9]);
                    v1.y = pack_bf16x2(acc[i][10], acc[i][11]);
                    v1.z = pack_bf16x2(acc[i][12], acc[i][13]);
                    v1.w = pack_bf16x2(acc[i][14], acc[i][15]);
                    *reinterpret_cast<uint4*>(myrow) = v0;
                    *reinterpret_cast<uint4*>(myrow + 16) = v1;
                }
                if (has1) {
                    const int i1 = (i + 1) < CPW ? i + 1 : i;
                    uint4 v0, v1;
                    v0.x = pack_bf16x2(acc[i1][0], acc[i1][1]);
                    v0.y = pack_bf16x2(acc[i1][2], acc[i1][3]);
                    v0.z = pack_bf16x2(acc[i1][4], acc[i1][5]);
                    v0.w = pack_bf16x2(acc[i1][6], acc[i1][7]);
                    v1.x = pack_bf16x2(acc[i1][8], acc[i1][9]);
                    v1.y = pack_bf16x2(acc[i1][10], acc[i1][11]);
                    v1.z = pack_bf16x2(acc[i1][12], acc[i1][13]);
                    v1.w = pack_bf16x2(acc[i1][14], acc[i1][15]);
                    *reinterpret_cast<uint4*>(myrow + 32) = v0;
                    *reinterpret_cast<uint4*>(myrow + 48) = v1;
                }
                __syncwarp();
                const int units = has1 ? 4 : 2;     // 16-byte units per staged row
                const int col_base = n0 + c0 * 16;
                for (int q = lane; q < 32 * units; q += 32) {
                    const int r = q / units;
                    const int u = q - r * units;
                    const int gcol = col_base + u * 8;
                    if (((rows_mask >> r) & 1u) && gcol < p.N) {
                        const uint4 v = *reinterpret_cast<const uint4*>(stg + r * EPI_PITCH + u * 16);
                        *reinterpret_cast<uint4*>(Dg + static_cast<size_t>(warp_row0 + r) * p.N + gcol) = v;
                    }
                }
                __syncwarp();
            }
        }
    }

    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
}

}  // namespace fg8
