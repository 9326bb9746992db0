// decode_kernel.cuh -- fine-grained-scaled FP8 GEMM for few rows of A (decode).
//
// Same result as the main kernel, D[m,n] = bf16(sum_kb (A_kb . B_kb^T)[m,n] *
// sfa[m,kb] * sfb[n/128,kb]), for M <= 256.  With so few rows the work is
// bound by streaming B from HBM, so the tile is turned around: the tensor
// core's 128-row side runs over 128 rows of B (n) and its N side over the
// MT >= M rows of A (m), i.e. the MMA computes D^T tiles of 128 x MT.  K is
// split over several CTAs so that enough SMs stream B at once.  The splits
// of a tile are summed in split order (deterministic) in one of two ways:
//  - cluster mode (2..8 splits, whole grid resident): the splits of a tile
//    form one thread-block cluster; each CTA stages its FP32 partial in its
//    own shared memory and then sums a slice of the tile's rows over all
//    peers through distributed shared memory;
//  - workspace mode (persistent grid): each split writes its partial to a
//    global workspace and the last CTA to arrive at a tile's counter sums them.
//
// Roles (384 threads, same register split as the main kernel):
//   warp 8      TMA producer: B tile [128 x 128] and A tile [MT x 128] per K block
//   warps 9-10  MMA issuers, taking turns by K block (M=128, N=MT, K=32 x 4)
//   warp 11     scale warp: for each K block writes scol[m] = sfa[m,kb] *
//               sfb[tile,kb] into a shared-memory ring (the B rows of a tile
//               all lie in one 128-row scale block)
//   warps 0-7   promotion (TMEM lane = row n of B, two warpgroups split the MT
//               columns), then the split-K epilogue.
// Two-level accumulation as in the pages (chujupifa.com "机器之心报道", opening
// summary; ai.abqq.net, section 1 "架构优化"): each K block's partial sums are
// scaled and added into FP32 registers.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "gemm_kernel.cuh"

namespace fg8 {

constexpr int DEC_SCALE_WARP = 11;
// Register split of this kernel (setmaxnreg, as in the main kernel):
// 256 * 208 + 128 * 88 == 384 * 168.
constexpr int DEC_REGS_PRODUCER = 88;
constexpr int DEC_REGS_PROMOTION = 208;
static_assert(256 * DEC_REGS_PROMOTION + 128 * DEC_REGS_PRODUCER <= NUM_THREADS * REGS_LAUNCH, "register split");
constexpr int DEC_SCALE_SLOTS = 8;          // scale ring depth (K blocks)
constexpr int DEC_MAX_NBUF = 8;
constexpr int DEC_MAX_CLUSTER = 8;          // largest split count reduced inside a cluster

struct DecodeParams {
    int M, N, K;
    int KB;               // K / 128
    int NB;               // ceil(N / 128) = number of tiles
    int splits;           // K splits per tile
    int kb_per_split;     // ceil(KB / splits)
    int units;            // NB * splits
    int cluster_reduce;   // 1: the splits of a tile are one cluster and reduce through DSMEM
    int stages;
    int sfa_ld;           // M_pad of the MN-major sfa
    const float* sfa;     // [KB][sfa_ld]
    const float* sfb;     // [NB][KB]
    __nv_bfloat16* D;     // [M][N]
    float* workspace;     // [units][MT][128] FP32 partials (splits > 1, no cluster)
    unsigned* counters;   // [NB] arrival counters, 0 between launches (each resets itself
                          // at its tile's last arrival; the host clears them after an abort)
    int* status;
    unsigned long long wait_limit_ns;
};

template <int MT>
struct DecodeShape {
    static constexpr int NC = MT / 16;
    static constexpr int CPW = (NC + 1) / 2;             // column chunks per promotion warpgroup
    static constexpr int B_BYTES = BM * BK;              // B (weights) tile: 128 rows
    static constexpr int A_BYTES = MT * BK;              // A (tokens) tile: MT rows
    static constexpr int STAGE_BYTES = B_BYTES + A_BYTES;
    static constexpr int NBUF = (512 / MT) < DEC_MAX_NBUF ? (512 / MT) : DEC_MAX_NBUF;
    static constexpr int TMEM_USED = NBUF * MT;
    static constexpr int TMEM_COLS = TMEM_USED <= 32    ? 32
                                     : TMEM_USED <= 64  ? 64
                                     : TMEM_USED <= 128 ? 128
                                     : TMEM_USED <= 256 ? 256
                                                        : 512;
    static_assert(MT % 32 == 0 && MT >= 32 && MT <= 256, "MT must be a multiple of 32 in [32, 256]");
    static_assert(NUM_MMA_WARPS <= NBUF, "more MMA issuers than TMEM accumulators");
};

// Shared memory: [stages x (B | A)] [scale ring DEC_SCALE_SLOTS x MT floats]
//                [barriers] [tmem slot, abort flag, broadcast word]
__host__ __device__ constexpr size_t decode_smem_bytes(int stage_bytes, int stages, int mt) {
    return 1024 + static_cast<size_t>(stages) * stage_bytes + static_cast<size_t>(DEC_SCALE_SLOTS) * mt * 4 +
           (2 * stages + 2 * DEC_MAX_NBUF + 2 * DEC_SCALE_SLOTS + 1) * 8 + 16;
}

// The unit sequence of a CTA: u = blockIdx.x, +gridDim.x, ...; unit u covers
// tile u / splits and K blocks [kb0, kb1) of split u % splits.
struct DecodeUnit {
    int tile, split, kb0, kb1;
};

__device__ __forceinline__ bool decode_unit(const DecodeParams& p, int u, DecodeUnit& d) {
    if (u >= p.units) return false;
    d.tile = u / p.splits;
    d.split = u - d.tile * p.splits;
    d.kb0 = d.split * p.kb_per_split;
    d.kb1 = min(p.KB, d.kb0 + p.kb_per_split);
    return true;
}

// Walks the flat sequence of (unit, K block) pairs of one CTA.
struct DecodeCursor {
    int u;
    int kb;
    DecodeUnit d;
    bool valid;

    __device__ DecodeCursor(const DecodeParams& p, int first_unit, int stride) : u(first_unit), kb(0), valid(false) {
        while (decode_unit(p, u, d)) {
            if (d.kb0 < d.kb1) {
                kb = d.kb0;
                valid = true;
                return;
            }
            u += stride;
        }
    }

    __device__ void advance(const DecodeParams& p, int stride) {
        if (!valid) return;
        if (++kb < d.kb1) return;
        u += stride;
        while (decode_unit(p, u, d)) {
            if (d.kb0 < d.kb1) {
                kb = d.kb0;
                return;
            }
            u += stride;
        }
        valid = false;
    }
};

// The scales of one (unit, K block) for one lane of the scale warp: sfa[m, kb]
// for m = lane + 32 i, and sfb[tile, kb].
template <int MT>
__device__ __forceinline__ void load_scales(const DecodeParams& p, const DecodeCursor& c, int lane,
                                            float (&a)[MT / 32], float& b) {
    if (!c.valid) {
#pragma unroll
        for (int i = 0; i < MT / 32; ++i) a[i] = 0.0f;
        b = 0.0f;
        return;
    }
    const float* srow = p.sfa + static_cast<size_t>(c.kb) * p.sfa_ld;
#pragma unroll
    for (int i = 0; i < MT / 32; ++i) {
        const int m = lane + 32 * i;
        a[i] = m < p.M ? __ldg(srow + m) : 0.0f;
    }
    b = __ldg(p.sfb + static_cast<size_t>(c.d.tile) * p.KB + c.kb);
}

template <int MT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fg8_decode_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const DecodeParams p) {
    using S = DecodeShape<MT>;
    constexpr int NC = S::NC;
    constexpr int CPW = S::CPW;
    constexpr int LB = CPW <= 4 ? CPW : 4;
    constexpr uint32_t IDESC = ptx::idesc_e4m3_f32(BM, MT);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_base = smem;
    float* scale_ring = reinterpret_cast<float*>(smem + static_cast<size_t>(p.stages) * S::STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(scale_ring + DEC_SCALE_SLOTS * MT);
    uint64_t* empty = full + p.stages;
    uint64_t* tfull = empty + p.stages;
    uint64_t* tempty = tfull + S::NBUF;
    uint64_t* sfull = tempty + S::NBUF;
    uint64_t* sempty = sfull + DEC_SCALE_SLOTS;
    uint64_t* done_bar = sempty + DEC_SCALE_SLOTS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* bcast = reinterpret_cast<volatile int*>(tmem_slot + 2);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint64_t limit = p.wait_limit_ns;
    const uint64_t drain_limit = 2000000000ull;

    // The producer's walk over this CTA's (unit, K block) sequence.  Its first
    // p.stages loads need no free stage, so the producer issues them right
    // after initialising the barriers, before the TMEM allocation and the
    // block-wide barrier: the first bytes are on their way during the set-up.
    DecodeCursor pcur(p, blockIdx.x, gridDim.x);
    int preloaded = 0;
    if (warp == PRODUCER_WARP && lane == 0) {
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < S::NBUF; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], NUM_EPI_WARPS);
        }
        for (int b = 0; b < DEC_SCALE_SLOTS; ++b) {
            ptx::mbar_init(&sfull[b], 1);
            ptx::mbar_init(&sempty[b], NUM_EPI_WARPS);
        }
        ptx::mbar_init(done_bar, NUM_MMA_WARPS);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
        ptx::prefetch_tensormap(&tmA);
        ptx::prefetch_tensormap(&tmB);
        ptx::griddep_wait();
        for (; pcur.valid && preloaded < p.stages; ++preloaded, pcur.advance(p, gridDim.x)) {
            uint8_t* sb = stage_base + static_cast<size_t>(preloaded) * S::STAGE_BYTES;
            ptx::mbar_arrive_expect_tx(&full[preloaded], S::STAGE_BYTES);
            ptx::tma_load_3d(sb, &tmB, &full[preloaded], pcur.kb * BK, pcur.d.tile * BM, 0);
            ptx::tma_load_3d(sb + S::B_BYTES, &tmA, &full[preloaded], pcur.kb * BK, 0, 0);
        }
    }
    if (warp == MMA_WARP) {
        ptx::tmem_alloc(tmem_slot, S::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    // Global memory is read or written only after the grids this launch
    // depends on are done (programmatic dependent launch).
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp >= NUM_EPI_WARPS) {
        ptx::setmaxnreg_dec<DEC_REGS_PRODUCER>();
        if (warp == PRODUCER_WARP) {
            if (lane == 0) {
                // Continue after the loads issued during the set-up.
                int stage = preloaded == p.stages ? 0 : preloaded;
                uint32_t phase = preloaded == p.stages ? 1u : 0u;
                int issued = preloaded;
                int w = 0;
                for (; w == 0 && pcur.valid; pcur.advance(p, gridDim.x)) {
                    w = wait_bar(&empty[stage], phase ^ 1u, limit, abort_flag);
                    if (w) break;
                    uint8_t* sb = stage_base + static_cast<size_t>(stage) * S::STAGE_BYTES;
                    ptx::mbar_arrive_expect_tx(&full[stage], S::STAGE_BYTES);
                    ptx::tma_load_3d(sb, &tmB, &full[stage], pcur.kb * BK, pcur.d.tile * BM, 0);
                    ptx::tma_load_3d(sb + S::B_BYTES, &tmA, &full[stage], pcur.kb * BK, 0, 0);
                    ++issued;
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (w == 2) record_error(p.status, ERR_TIMEOUT, ROLE_PRODUCER);
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
            }
        } else if (warp < MMA_WARP + NUM_MMA_WARPS) {
            const int j = warp - MMA_WARP;
            if (lane == 0) {
                int stage = 0;
                uint32_t phase = 0;
                int buf = 0;
                uint32_t bphase = 0;
                int w = 0;
                int g = 0;
                DecodeUnit d;
                for (int u = blockIdx.x; w == 0 && decode_unit(p, u, d); u += gridDim.x) {
                    for (int kb = d.kb0; kb < d.kb1; ++kb, ++g) {
                        if (g % NUM_MMA_WARPS == j) {
                            w = wait_bar(&full[stage], phase, limit, abort_flag);
                            if (w) break;
                            w = wait_bar(&tempty[buf], bphase ^ 1u, limit, abort_flag);
                            if (w) break;
                            ptx::tc_fence_after();
                            const uint32_t b_addr =
                                ptx::smem_addr(stage_base + static_cast<size_t>(stage) * S::STAGE_BYTES);
                            const uint64_t adesc = ptx::smem_desc_sw128(b_addr);                 // weights
                            const uint64_t bdesc = ptx::smem_desc_sw128(b_addr + S::B_BYTES);    // tokens
                            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * MT);
#pragma unroll
                            for (int k = 0; k < BK / 32; ++k)
                                ptx::mma_f8f6f4(d_tmem, adesc + static_cast<uint64_t>(k * 2),
                                                bdesc + static_cast<uint64_t>(k * 2), IDESC, k > 0 ? 1u : 0u);
                            ptx::mma_commit(&empty[stage]);
                            ptx::mma_commit(&tfull[buf]);
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
                ptx::mma_commit(done_bar);
                ptx::mbar_wait(done_bar, 0, drain_limit);
            }
        } else if (warp == DEC_SCALE_WARP) {
            // scol[m] = sfa[m, kb] * sfb[tile, kb] for every K block, in order.
            // Loads run SCALE_AHEAD K blocks ahead of the writes.  The loop is
            // unrolled by SCALE_AHEAD so that each register slot is refilled in
            // place: a rotating copy would stall on the newest load every block.
            constexpr int SCALE_AHEAD = 4;
            constexpr int PER_LANE = MT / 32;
            DecodeCursor ld(p, blockIdx.x, gridDim.x);    // next (unit, K block) to load
            DecodeCursor wr = ld;                         // next one to write
            float qa[SCALE_AHEAD][PER_LANE];
            float qb[SCALE_AHEAD];
#pragma unroll
            for (int q = 0; q < SCALE_AHEAD; ++q) {
                load_scales<MT>(p, ld, lane, qa[q], qb[q]);
                ld.advance(p, gridDim.x);
            }
            int slot = 0;
            uint32_t sphase = 0;
            int w = 0;
            while (wr.valid && w == 0) {
#pragma unroll
                for (int q = 0; q < SCALE_AHEAD; ++q) {
                    if (!wr.valid) break;
                    if (lane == 0) w = wait_bar(&sempty[slot], sphase ^ 1u, limit, abort_flag);
                    w = __shfl_sync(0xffffffffu, w, 0);
                    if (w) break;
                    float* dst = scale_ring + slot * MT;
#pragma unroll
                    for (int i = 0; i < PER_LANE; ++i) dst[lane + 32 * i] = qa[q][i] * qb[q];
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sfull[slot]);
                    load_scales<MT>(p, ld, lane, qa[q], qb[q]);
                    ld.advance(p, gridDim.x);
                    wr.advance(p, gridDim.x);
                    if (++slot == DEC_SCALE_SLOTS) {
                        slot = 0;
                        sphase ^= 1u;
                    }
                }
            }
            if (w == 2 && lane == 0) record_error(p.status, ERR_TIMEOUT, ROLE_PRODUCER);
        }
    } else {
        ptx::setmaxnreg_inc<DEC_REGS_PROMOTION>();
        const int wg = warp / 4;
        const int quarter = warp % 4;
        const int row_in_tile = quarter * 32 + lane;    // row n of B within the tile
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int chunk0 = wg * CPW;
        int buf = 0;
        uint32_t bphase = 0;
        int slot = 0;
        uint32_t sphase = 0;
        bool ok = true;
        DecodeUnit d;
        // Every promotion warp walks all of this CTA's units, even after an abort
        // (ok turns false: the warp then skips the waits and the memory work), so
        // all warps run the same sequence of named barriers in the split-K
        // epilogue: warps that saw the abort in different units still meet there.
        for (int u = blockIdx.x; decode_unit(p, u, d); u += gridDim.x) {
            float2 acc[CPW][8];
#pragma unroll
            for (int i = 0; i < CPW; ++i)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[i][q] = make_float2(0.0f, 0.0f);

            for (int kb = d.kb0; ok && kb < d.kb1; ++kb) {
                int w = 0;
                if (lane == 0) {
                    w = wait_bar(&tfull[buf], bphase, limit, abort_flag);
                    if (!w) w = wait_bar(&sfull[slot], sphase, limit, abort_flag);
                }
                w = __shfl_sync(0xffffffffu, w, 0);
                if (w) {
                    if (w == 2 && lane == 0) record_error(p.status, ERR_TIMEOUT, ROLE_EPILOGUE);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t tbase = tmem_base + lane_base + static_cast<uint32_t>(buf * MT);
                const float* scol = scale_ring + slot * MT;
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
                            const float4* sv = reinterpret_cast<const float4*>(scol + c * 16);
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4) {
                                const float4 s4 = sv[q4];
                                const float2 v0 = make_float2(__uint_as_float(r[b][4 * q4]), __uint_as_float(r[b][4 * q4 + 1]));
                                const float2 v1 =
                                    make_float2(__uint_as_float(r[b][4 * q4 + 2]), __uint_as_float(r[b][4 * q4 + 3]));
                                acc[i < CPW ? i : 0][2 * q4] =
                                    __ffma2_rn(v0, make_float2(s4.x, s4.y), acc[i < CPW ? i : 0][2 * q4]);
                                acc[i < CPW ? i : 0][2 * q4 + 1] =
                                    __ffma2_rn(v1, make_float2(s4.z, s4.w), acc[i < CPW ? i : 0][2 * q4 + 1]);
                            }
                        }
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(&tempty[buf]);
                    ptx::mbar_arrive(&sempty[slot]);
                }
                if (++buf == S::NBUF) {
                    buf = 0;
                    bphase ^= 1u;
                }
                if (++slot == DEC_SCALE_SLOTS) {
                    slot = 0;
                    sphase ^= 1u;
                }
            }
            // ---- epilogue: this split's FP32 partial, then the BF16 tile ----
            // Every promotion warp runs the same barrier sequence even after an
            // abort (it then skips the memory work), so no warp can be left
            // waiting at a barrier.
            const int n = d.tile * BM + row_in_tile;
            const bool n_ok = n < p.N;
            if (p.splits == 1) {
                if (ok) {
#pragma unroll
                    for (int i = 0; i < CPW; ++i) {
                        const int c = chunk0 + i;
                        if (c < NC) {
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const int m = c * 16 + 2 * q;
                                if (n_ok && m < p.M)
                                    p.D[static_cast<size_t>(m) * p.N + n] = __float2bfloat16_rn(acc[i][q].x);
                                if (n_ok && m + 1 < p.M)
                                    p.D[static_cast<size_t>(m + 1) * p.N + n] = __float2bfloat16_rn(acc[i][q].y);
                            }
                        }
                    }
                }
                continue;
            }
            if (p.cluster_reduce) {
                // Stage the partial in this CTA's own (now idle) stage buffers as
                // [MT][128] floats; the cluster phase below sums the splits.
                if (ok) {
                    float* stg = reinterpret_cast<float*>(stage_base);
#pragma unroll
                    for (int i = 0; i < CPW; ++i) {
                        const int c = chunk0 + i;
                        if (c < NC) {
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const int m = c * 16 + 2 * q;
                                stg[m * BM + row_in_tile] = acc[i][q].x;
                                stg[(m + 1) * BM + row_in_tile] = acc[i][q].y;
                            }
                        }
                    }
                }
                continue;
            }
            // Global workspace, layout per unit [MT][128] floats (coalesced).
            if (ok) {
                float* ws = p.workspace + static_cast<size_t>(u) * MT * BM + row_in_tile;
#pragma unroll
                for (int i = 0; i < CPW; ++i) {
                    const int c = chunk0 + i;
                    if (c < NC) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const int m = c * 16 + 2 * q;
                            __stcg(ws + static_cast<size_t>(m) * BM, acc[i][q].x);
                            __stcg(ws + static_cast<size_t>(m + 1) * BM, acc[i][q].y);
                        }
                    }
                }
            }
            ptx::named_barrier_sync(1, NUM_EPI_WARPS * 32);   // every partial of this CTA is stored
            if (threadIdx.x == 0) {
                const unsigned old = ptx::atom_inc_acq_rel_gpu(p.counters + d.tile, static_cast<unsigned>(p.splits - 1));
                *bcast = (*abort_flag) ? -1 : static_cast<int>(old) + 1;
            }
            ptx::named_barrier_sync(1, NUM_EPI_WARPS * 32);
            const int arrived = *bcast;
            ptx::named_barrier_sync(1, NUM_EPI_WARPS * 32);   // everyone has read bcast before it is reused
            if (arrived != p.splits) continue;                // another split finishes this tile (or aborted)
            // The last split sums all splits in split order 0..S-1 (its own from
            // registers), one chunk at a time with up to RB splits' loads in flight.
            constexpr int RB = MT <= 128 ? 4 : 2;
            const float* ws0 = p.workspace + static_cast<size_t>(d.tile) * p.splits * MT * BM + row_in_tile;
#pragma unroll
            for (int i = 0; i < CPW; ++i) {
                const int c = chunk0 + i;
                if (c >= NC) continue;
                float red[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) red[j] = 0.0f;
                for (int s0 = 0; s0 < p.splits; s0 += RB) {
                    float v[RB][16];
#pragma unroll
                    for (int h = 0; h < RB; ++h) {
                        const int sp = s0 + h;
                        const float* wsp = ws0 + (static_cast<size_t>(sp) * MT + c * 16) * BM;
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            v[h][j] = (sp < p.splits && sp != d.split) ? __ldcg(wsp + static_cast<size_t>(j) * BM) : 0.0f;
                        if (sp == d.split) {
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                v[h][2 * q] = acc[i][q].x;
                                v[h][2 * q + 1] = acc[i][q].y;
                            }
                        }
                    }
#pragma unroll
                    for (int h = 0; h < RB; ++h)
#pragma unroll
                        for (int j = 0; j < 16; ++j) red[j] += v[h][j];
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int m = c * 16 + j;
                    if (n_ok && m < p.M) p.D[static_cast<size_t>(m) * p.N + n] = __float2bfloat16_rn(red[j]);
                }
            }
        }
    }

    __syncwarp();
    if (p.cluster_reduce) {
        // The splits of a tile form one cluster (rank = split).  After every CTA
        // has staged its partial, CTA r sums rows [r*RS, (r+1)*RS) of the tile
        // over all splits in split order, reading the peers' shared memory, and
        // writes them; the second barrier keeps each CTA's staging alive until
        // its peers are done with it.
        ptx::cluster_sync();
        if (warp < NUM_EPI_WARPS && !*abort_flag) {
            const int S = p.splits;
            const int rank = static_cast<int>(ptx::cluster_ctarank());
            const int tile = static_cast<int>(blockIdx.x) / S;
            const int rs = ((BM + S - 1) / S + 3) & ~3;      // rows per rank, a multiple of 4
            const int r0 = min(BM, rank * rs);
            const int nq = (min(BM, r0 + rs) - r0) / 4;      // groups of 4 rows
            const uint32_t base = ptx::smem_addr(stage_base);
            for (int e = threadIdx.x; e < nq * p.M; e += NUM_EPI_WARPS * 32) {
                const int m = e / nq;
                const int row = r0 + 4 * (e - m * nq);
                const uint32_t off = base + static_cast<uint32_t>((m * BM + row) * 4);
                float4 v[DEC_MAX_CLUSTER];
#pragma unroll
                for (int sp = 0; sp < DEC_MAX_CLUSTER; ++sp)
                    if (sp < S) v[sp] = ptx::ld_shared_cluster_v4(ptx::mapa_shared(off, static_cast<uint32_t>(sp)));
                float4 sum = v[0];
#pragma unroll
                for (int sp = 1; sp < DEC_MAX_CLUSTER; ++sp) {
                    if (sp < S) {
                        sum.x += v[sp].x;
                        sum.y += v[sp].y;
                        sum.z += v[sp].z;
                        sum.w += v[sp].w;
                    }
                }
                const int nn = tile * BM + row;               // N % 16 == 0: all 4 rows in range or none
                if (nn < p.N) {
                    const __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
                    const __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
                    uint2 pk;
                    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
                    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
                    *reinterpret_cast<uint2*>(p.D + static_cast<size_t>(m) * p.N + nn) = pk;
                }
            }
        }
        ptx::cluster_sync();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
}

}  // namespace fg8
