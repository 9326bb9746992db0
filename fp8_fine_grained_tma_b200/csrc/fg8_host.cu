// fg8_host.cu -- the C ABI declared in include/fg8.h: argument checks, tile
// configuration, TMA descriptor encoding (cached), kernel launches, the scale
// layout transform and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "decode_launch.cuh"
#include "fg8.h"
#include "jit.h"
#include "launch.cuh"

namespace fg8 {

#define FG8_DECLARE_BOTH(BN)                                 \
    FG8_DECLARE_LAUNCH_ONE(BN, false) FG8_DECLARE_LAUNCH_ONE(BN, true) \
    template <>                                              \
    cudaError_t gemm_max_split_clusters<BN>(int cluster, int* out);
FG8_FOR_EACH_BN(FG8_DECLARE_BOTH)
#undef FG8_DECLARE_BOTH
FG8_FOR_EACH_MT(FG8_DECLARE_DECODE_LAUNCH)

// First error recorded by any GEMM kernel on this device: [0] = code,
// [1] = (block << 8) | role.  Cleared by fg_get_last_device_status.
__device__ int g_status[2];

namespace {

constexpr int kMaxDevices = 64;

std::atomic<int> g_num_sms{0};   // 0 = not set: use the device's SM count
std::atomic<unsigned long long> g_wait_limit_ns{1000000000ull};

struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    int cc_major = 0;
    int* status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

fg_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return FG_OK;
    if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver || e == cudaErrorInitializationError)
        return FG_ERR_NO_DEVICE;
    return FG_ERR_CUDA;
}

// Current device, checked to be an sm_100 part; fills *info.
fg_status current_device(DeviceInfo** info) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_status(e) == FG_OK ? FG_ERR_CUDA : cuda_status(e);
    }
    if (dev < 0 || dev >= kMaxDevices) return FG_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_dev_mutex);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return FG_ERR_NO_DEVICE;
        }
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_status) != cudaSuccess) {
            cudaGetLastError();
            return FG_ERR_CUDA;
        }
        d.status = static_cast<int*>(addr);
        d.ready = true;
    }
    if (d.cc_major != 10) return FG_ERR_NO_DEVICE;
    *info = &d;
    return FG_OK;
}

int effective_sms(const DeviceInfo& d) {
    int n = g_num_sms.load();
    if (n <= 0) {
        const char* env = std::getenv("FG_NUM_SMS");
        if (env) n = std::atoi(env);
    }
    if (n <= 0 || n > d.sm_count) n = d.sm_count;
    return n;
}

// ---- TMA descriptors ---------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return static_cast<EncodeTiledFn>(nullptr);
        }
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 3-D E4M3 operand [groups][rows][K] (K innermost), box 128 (K) x box_rows x 1,
// 128-byte swizzle, zero fill out of bounds.
struct MapKey {
    const void* ptr;
    uint64_t K, rows, groups;
    uint32_t box_rows;
    bool operator<(const MapKey& o) const {
        return std::tie(ptr, K, rows, groups, box_rows) < std::tie(o.ptr, o.K, o.rows, o.groups, o.box_rows);
    }
};
std::map<MapKey, CUtensorMap> g_maps;
std::mutex g_maps_mutex;

fg_status operand_map(const void* ptr, uint64_t K, uint64_t rows, uint64_t groups, uint32_t box_rows,
                      CUtensorMap* out) {
    MapKey key{ptr, K, rows, groups, box_rows};
    {
        std::lock_guard<std::mutex> lk(g_maps_mutex);
        auto it = g_maps.find(key);
        if (it != g_maps.end()) {
            *out = it->second;
            return FG_OK;
        }
    }
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return FG_ERR_NO_DEVICE;
    CUtensorMap m;
    std::memset(&m, 0, sizeof(m));
    const cuuint64_t dims[3] = {K, rows, groups};
    const cuuint64_t strides[2] = {K, K * rows};   // bytes, dims 1 and 2
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return FG_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(g_maps_mutex);
        if (g_maps.size() > 512) g_maps.clear();
        g_maps[key] = m;
    }
    *out = m;
    return FG_OK;
}

// 3-D BF16 output D [groups][rows][N] (N innermost), box 16 (N) x 32 rows x 1,
// 32-byte swizzle: the pieces the GEMM kernel's epilogue stores by TMA.  The
// map's extents clip the stores at N columns and `rows` rows.
struct OutKey {
    const void* ptr;
    uint64_t N, rows, groups;
    bool operator<(const OutKey& o) const {
        return std::tie(ptr, N, rows, groups) < std::tie(o.ptr, o.N, o.rows, o.groups);
    }
};
std::map<OutKey, CUtensorMap> g_out_maps;

fg_status output_map(void* ptr, uint64_t N, uint64_t rows, uint64_t groups, CUtensorMap* out) {
    OutKey key{ptr, N, rows, groups};
    {
        std::lock_guard<std::mutex> lk(g_maps_mutex);
        auto it = g_out_maps.find(key);
        if (it != g_out_maps.end()) {
            *out = it->second;
            return FG_OK;
        }
    }
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return FG_ERR_NO_DEVICE;
    CUtensorMap m;
    std::memset(&m, 0, sizeof(m));
    const cuuint64_t dims[3] = {N, rows, groups};
    const cuuint64_t strides[2] = {N * 2, N * 2 * rows};   // bytes, dims 1 and 2
    const cuuint32_t box[3] = {16, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return FG_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(g_maps_mutex);
        if (g_out_maps.size() > 512) g_out_maps.clear();
        g_out_maps[key] = m;
    }
    *out = m;
    return FG_OK;
}

// ---- configuration -----------------------------------------------------------
// Cost model of one candidate (block width BN, 128-row tiles on one CTA or
// 256-row tiles on a CTA pair), in SM clock cycles, from measurements on B200:
//   - the tensor core needs ~512 cycles per K block of a 128-row tile for any
//     BN <= 256 (one M=128, K=32 MMA every ~128 cycles), so wider blocks do
//     more work in the same time;
//   - with two TMEM accumulators (BN > 170) the promotion of one K block and
//     its handshake with the MMA issuers stretch that to ~700 cycles; three
//     (BN <= 170) to ~600; four (BN <= 128) to ~520;
//   - each tile adds an epilogue of ~2000 cycles that overlaps the next tile
//     only partly.
// Tiles per CTA (pair) = ceil(tiles / (SMs or SMs/2)).  The job is bounded
// below by its unique HBM bytes at ~3.3 KB/clk.
struct Choice {
    int bn = 0;
    bool pair = false;
};

// ---- stream-K (normal layout) ----------------------------------------------------
// When the tiles fill the units' last wave poorly, all but the last one or two
// waves of tiles run whole and the (tile, K block) iterations of the rest are
// split evenly over the units (see TileScheduler).  Used when that wave would
// be less than 90 % full and every unit gets at least a quarter of a tile's K
// blocks (so a tile is split over a few units at most).  FG_STREAMK=0 turns it
// off.
struct StreamKPlan {
    bool on = false;
    int dp_tiles = 0;
    long long iters = 0;
};

StreamKPlan streamk_plan(long long tiles, int units, int KB) {
    StreamKPlan sp;
    const char* env = std::getenv("FG_STREAMK");
    if ((env && std::atoi(env) == 0) || units <= 1 || tiles <= 0 || KB < 2) return sp;
    const long long waves = (tiles + units - 1) / units;
    const double fill = static_cast<double>(tiles) / static_cast<double>(waves * units);
    if (fill >= 0.9) return sp;
    const long long full_waves = tiles / units;
    const long long dp = full_waves > 1 ? (full_waves - 1) * units : 0;
    const long long iters = (tiles - dp) * KB;
    if (iters * 4 < static_cast<long long>(units) * KB) return sp;   // pieces shorter than KB / 4
    sp.on = true;
    sp.dp_tiles = static_cast<int>(dp);
    sp.iters = iters;
    return sp;
}

double estimate_cycles(int layout, bool pair, int bn, long long row_tiles, int N, int K, int num_sms,
                       double hbm_bytes) {
    const int KB = K / BK;
    const long long tiles = row_tiles * ((N + bn - 1) / bn);
    const int units = std::max(1, pair ? num_sms / 2 : num_sms);
    double waves = static_cast<double>((tiles + units - 1) / units);
    if (layout == LAYOUT_NORMAL && streamk_plan(tiles, units, KB).on)
        waves = static_cast<double>(tiles) / units + 0.05;   // split iterations, plus the partial-sum exchange
    const int acc_stride = (bn + 31) / 32 * 32;
    const int nbuf = std::min(4, 512 / acc_stride);
    double per_kb = nbuf >= 4 ? 520.0 : (nbuf == 3 ? 600.0 : 700.0);
    if (pair) per_kb *= 0.96;   // a pair's 256-row tile runs a few per cent faster than two 128-row tiles
    const double t_tiles = waves * (KB * per_kb + 2000.0);
    return std::max(t_tiles, hbm_bytes / 3300.0) + 2000.0;
}

// rows: rows per row group; groups: row groups (masked: G, else 1); valid_rows:
// expected rows that carry data per group (the masked hint, else rows).
Choice choose_config(int layout, int rows, int groups, int valid_rows, int N, int K, int num_sms, double hbm_bytes) {
    Choice best;
    const char* force = std::getenv("FG_FORCE_BLOCK_N");
    const char* force_pair = std::getenv("FG_FORCE_PAIR");
    const int fbn = force ? std::atoi(force) : 0;
    const int fpair = force_pair ? std::atoi(force_pair) : -1;
    // CTA pairs halve each SM's B loads.  Measured on B200 they win a few per
    // cent on the normal layout, tie on contiguous groups and lose on masked
    // groups (whose 256-row tiles compute rows past masked_m), so by default
    // only the normal layout considers them; FG_FORCE_PAIR=0/1 forbids/forces.
    const bool pair_ok = num_sms >= 2 && !(layout == LAYOUT_CONTIGUOUS && rows / BM > MAX_PAIR_LIST) &&
                         (fpair == 1 || (fpair != 0 && layout == LAYOUT_NORMAL));
    double best_t = 1e300;
    for (int pair = 0; pair <= 1; ++pair) {
        if (pair && !pair_ok) continue;
        if (fpair >= 0 && pair != fpair) continue;
        for (int bn = pair ? 32 : 16; bn <= 256; bn += 16) {
            if (fbn >= 16 && fbn <= 256 && fbn % 16 == 0 && bn != fbn) continue;
            const int tile_m = pair ? 2 * BM : BM;
            const long long row_tiles = static_cast<long long>(groups) * ((valid_rows + tile_m - 1) / tile_m);
            const double t = estimate_cycles(layout, pair, bn, std::max(1ll, row_tiles), N, K, num_sms, hbm_bytes);
            if (t < best_t * 0.999 || (t <= best_t * 1.001 && (pair > (best.pair ? 1 : 0) || bn > best.bn))) {
                if (t < best_t) best_t = t;
                best.bn = bn;
                best.pair = pair != 0;
            }
        }
    }
    return best;
}

int stage_bytes_for(int bn, bool pair) { return BM * BK + (pair ? bn / 2 : bn) * BK; }

// At least MAX_NBUF stages: an MMA issuer then never waits on a stage barrier
// more than one phase ahead (every block width fits 4 stages in 227 KiB).
int choose_stages(int bn, bool pair) {
    const int sb = stage_bytes_for(bn, pair);
    int s = 8;
    while (s > MAX_NBUF && gemm_smem_bytes(sb, s, pair) > static_cast<size_t>(kMaxDynamicSmem - kGemmStaticSmem)) --s;
    return s;
}

template <int BN>
cudaError_t launch_either(bool pair, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                          const GemmParams& p, int grid, size_t smem, cudaStream_t st, int cluster) {
    if constexpr (BN >= 32) {
        if (pair) return launch_gemm<BN, true>(ta, tb, td, p, grid, smem, st, 2);
    } else {
        if (pair) return cudaErrorInvalidValue;
    }
    return launch_gemm<BN, false>(ta, tb, td, p, grid, smem, st, cluster);
}

fg_status launch_bn(int bn, bool pair, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                    const GemmParams& p, int grid, size_t smem, cudaStream_t st, int cluster = 1) {
    cudaError_t e = cudaErrorInvalidValue;
    switch (bn) {
#define FG8_CASE(BNV) \
    case BNV:         \
        e = launch_either<BNV>(pair, ta, tb, td, p, grid, smem, st, cluster); \
        break;
        FG8_FOR_EACH_BN(FG8_CASE)
#undef FG8_CASE
        default:
            return FG_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return FG_ERR_CUDA;
    }
    return FG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

constexpr long long kMaxDim = (1ll << 31) - 1;

// ---- decode (few rows of A): split-K workspace ----------------------------------
// One FP32 partial buffer and one counter array per (device, stream), grown on
// demand and kept for the life of the process; launches on one stream run in
// order, so they never share a buffer concurrently.  Counters are zero between
// launches (each resets itself at its tile's last arrival); after a device-side
// abort fg_get_last_device_status clears them.
struct Workspace {
    float* partials = nullptr;
    size_t partial_bytes = 0;
    unsigned* counters = nullptr;
    size_t counter_count = 0;
};
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;
std::mutex g_ws_mutex;

fg_status get_workspace(int dev, cudaStream_t stream, size_t partial_bytes, size_t counters, float** part,
                        unsigned** ctr) {
    std::lock_guard<std::mutex> lk(g_ws_mutex);
    Workspace& w = g_ws[std::make_pair(dev, stream)];
    if (w.partial_bytes < partial_bytes) {
        if (w.partials) cudaFree(w.partials);
        w.partials = nullptr;
        w.partial_bytes = 0;
        const size_t want = std::max(partial_bytes, 2 * w.partial_bytes);
        if (cudaMalloc(&w.partials, want) != cudaSuccess) {
            cudaGetLastError();
            return FG_ERR_CUDA;
        }
        w.partial_bytes = want;
    }
    if (w.counter_count < counters) {
        if (w.counters) cudaFree(w.counters);
        w.counters = nullptr;
        w.counter_count = 0;
        const size_t want = std::max<size_t>(counters, 1024);
        if (cudaMalloc(&w.counters, want * sizeof(unsigned)) != cudaSuccess ||
            cudaMemset(w.counters, 0, want * sizeof(unsigned)) != cudaSuccess) {
            cudaGetLastError();
            return FG_ERR_CUDA;
        }
        w.counter_count = want;
    }
    *part = w.partials;
    *ctr = w.counters;
    return FG_OK;
}

// After an aborted launch some counters may hold a partial count: clear all of
// this device's counters (synchronously; the caller has synchronised).
void clear_workspace_counters(int dev) {
    std::lock_guard<std::mutex> lk(g_ws_mutex);
    for (auto& kv : g_ws)
        if (kv.first.first == dev && kv.second.counters)
            cudaMemset(kv.second.counters, 0, kv.second.counter_count * sizeof(unsigned));
}

int decode_tile_width(int M) { return std::max(32, (M + 31) / 32 * 32); }

int decode_nbuf(int mt) { return std::min(DEC_MAX_NBUF, 512 / mt); }

int decode_stages(int mt) {
    const int sb = BM * BK + mt * BK;
    int s = 8;
    while (s > 2 && decode_smem_bytes(sb, s, mt) > static_cast<size_t>(kMaxDynamicSmem)) --s;
    return s;
}

// Resident CTAs of fg8_decode_kernel<mt> when grouped in clusters of s
// (cached per device; 0 when clusters of that size cannot be launched).
int decode_cluster_slots(int dev, int mt, int s, size_t smem) {
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, int> cache;
    const auto key = std::make_tuple(dev, mt, s);
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    int mc = 0;
    cudaError_t e = cudaErrorInvalidValue;
    switch (mt) {
#define FG8_DCAP(MTV) \
    case MTV:         \
        e = decode_max_clusters<MTV>(s, smem, &mc); \
        break;
        FG8_FOR_EACH_MT(FG8_DCAP)
#undef FG8_DCAP
        default:
            break;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        mc = 0;
    }
    const int slots = std::max(0, mc) * s;
    std::lock_guard<std::mutex> lk(mu);
    cache[key] = slots;
    return slots;
}

struct DecodePlan {
    int splits;
    int cluster;   // 1, or == splits when the splits of a tile form one cluster
};

// Splits of K per 128-row tile of B, and whether they reduce inside a cluster.
// Minimises the modelled time
//   max(B bytes / HBM rate, waves * K blocks per split * t_kb) + waves * t_unit
// with t_kb = 16 KiB / 64 GB/s (one SM streaming B alone), HBM rate 6.5 TB/s
// and t_unit the pipeline ramp plus the split reduction: 1.5 us through the
// global workspace (persistent grid), 1.0 us through distributed shared memory
// (2..8 splits, every tile's cluster resident at once).
DecodePlan decode_plan(int dev, int mt, size_t smem, int stage_room, int N, int K, int num_sms) {
    const int KB = K / BK;
    const int NB = (N + BM - 1) / BM;
    const char* cenv = std::getenv("FG_DECODE_CLUSTER");
    const bool cluster_ok = !(cenv && std::atoi(cenv) == 0) && stage_room >= mt * BM * 4;
    auto cluster_fits = [&](int s) {
        if (!cluster_ok || s < 2 || s > DEC_MAX_CLUSTER) return false;
        const long long units = static_cast<long long>(NB) * s;
        return units <= std::min(num_sms, decode_cluster_slots(dev, mt, s, smem));
    };
    const char* force = std::getenv("FG_FORCE_SPLITS");
    if (force && std::atoi(force) >= 1) {
        const int f = std::min(std::atoi(force), KB);
        return DecodePlan{f, cluster_fits(f) ? f : 1};
    }
    const double t_hbm = static_cast<double>(N) * K / 6.5e12;
    const double t_kb = 16384.0 / 64e9;
    DecodePlan best{1, 1};
    double best_t = 1e300;
    for (int s = 1; s <= std::min(KB, 32); ++s) {
        const int per = (KB + s - 1) / s;
        const int used = (KB + per - 1) / per;   // splits that get work
        if (used != s) continue;
        const long long units = static_cast<long long>(NB) * s;
        const double waves = static_cast<double>((units + num_sms - 1) / num_sms);
        double t = std::max(t_hbm, waves * per * t_kb) + waves * 1.5e-6;
        int cl = 1;
        if (cluster_fits(s)) {
            const double tc = std::max(t_hbm, per * t_kb) + 1.0e-6;
            if (tc < t) {
                t = tc;
                cl = s;
            }
        }
        if (t < best_t * 0.98) {
            best_t = t;
            best = DecodePlan{s, cl};
        }
    }
    return best;
}

fg_status launch_decode_mt(int mt, const CUtensorMap& ta, const CUtensorMap& tb, const DecodeParams& p, int grid,
                           int cluster, size_t smem, cudaStream_t st) {
    cudaError_t e = cudaErrorInvalidValue;
    switch (mt) {
#define FG8_DCASE(MTV) \
    case MTV:          \
        e = launch_decode<MTV>(ta, tb, p, grid, cluster, smem, st); \
        break;
        FG8_FOR_EACH_MT(FG8_DCASE)
#undef FG8_DCASE
        default:
            return FG_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return FG_ERR_CUDA;
    }
    return FG_OK;
}

fg_status run_decode(const void* A, const float* sfa, const void* B, const float* sfb, void* D, int M, int N, int K,
                     cudaStream_t stream) {
    DeviceInfo* dev = nullptr;
    fg_status st = current_device(&dev);
    if (st != FG_OK) return st;
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    const int num_sms = effective_sms(*dev);
    const int mt = decode_tile_width(M);
    const int stages = decode_stages(mt);
    if (stages < decode_nbuf(mt)) return FG_ERR_UNSUPPORTED;   // the issuers' barrier invariant needs it
    const int stage_bytes = BM * BK + mt * BK;
    const size_t smem = decode_smem_bytes(stage_bytes, stages, mt);
    const DecodePlan plan = decode_plan(dev_id, mt, smem, stages * stage_bytes, N, K, num_sms);

    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = K;
    p.KB = K / BK;
    p.NB = (N + BM - 1) / BM;
    p.splits = plan.splits;
    p.kb_per_split = (p.KB + p.splits - 1) / p.splits;
    p.units = p.NB * p.splits;
    p.cluster_reduce = plan.cluster > 1 ? 1 : 0;
    p.stages = stages;
    p.sfa_ld = static_cast<int>(fg_get_tma_aligned_size(M, 4));
    p.sfa = sfa;
    p.sfb = sfb;
    p.D = static_cast<__nv_bfloat16*>(D);
    p.status = dev->status;
    p.wait_limit_ns = g_wait_limit_ns.load();
    if (p.splits > 1 && !p.cluster_reduce) {
        st = get_workspace(dev_id, stream, static_cast<size_t>(p.units) * mt * BM * sizeof(float), p.NB,
                           &p.workspace, &p.counters);
        if (st != FG_OK) return st;
    }
    CUtensorMap ta, tb;
    st = operand_map(A, K, M, 1, mt, &ta);
    if (st != FG_OK) return st;
    st = operand_map(B, K, N, 1, BM, &tb);
    if (st != FG_OK) return st;
    // Cluster mode: one CTA per unit (the whole grid is resident by the plan);
    // otherwise a persistent grid.
    const int grid = p.cluster_reduce ? p.units : std::max(1, std::min(p.units, num_sms));
    return launch_decode_mt(mt, ta, tb, p, grid, plan.cluster, smem, stream);
}

// Rows of A up to which the normal GEMM uses the decode kernel.
int decode_max_rows() {
    const char* env = std::getenv("FG_DECODE_MAX_M");
    return env ? std::atoi(env) : 128;
}

// Workspace of the stream-K partial sums and their flags, one per (device,
// stream), grown on demand and kept for the life of the process (launches on
// one stream run in order).  Flags hold the epoch of the launch that published
// them: each launch takes a new epoch, so stale flags never match.
struct StreamKWorkspace {
    float* ws = nullptr;
    size_t ws_bytes = 0;
    unsigned* flags = nullptr;
    size_t flag_count = 0;
    unsigned epoch = 0;
};
std::map<std::pair<int, cudaStream_t>, StreamKWorkspace> g_sk;
std::mutex g_sk_mutex;

fg_status get_streamk_workspace(int dev, cudaStream_t stream, size_t ws_bytes, size_t flags, float** ws,
                                unsigned** fl, unsigned* epoch) {
    std::lock_guard<std::mutex> lk(g_sk_mutex);
    StreamKWorkspace& w = g_sk[std::make_pair(dev, stream)];
    if (w.ws_bytes < ws_bytes) {
        if (w.ws) cudaFree(w.ws);
        w.ws = nullptr;
        w.ws_bytes = 0;
        if (cudaMalloc(&w.ws, ws_bytes) != cudaSuccess) {
            cudaGetLastError();
            return FG_ERR_CUDA;
        }
        w.ws_bytes = ws_bytes;
    }
    if (w.flag_count < flags) {
        if (w.flags) cudaFree(w.flags);
        w.flags = nullptr;
        w.flag_count = 0;
        if (cudaMalloc(&w.flags, flags * sizeof(unsigned)) != cudaSuccess ||
            cudaMemset(w.flags, 0, flags * sizeof(unsigned)) != cudaSuccess) {
            cudaGetLastError();
            return FG_ERR_CUDA;
        }
        w.flag_count = flags;
        w.epoch = 0;
    }
    if (++w.epoch == 0) w.epoch = 1;
    *ws = w.ws;
    *fl = w.flags;
    *epoch = w.epoch;
    return FG_OK;
}

// ---- cluster split-K through the tile kernel (few rows) -----------------------
// For M <= 128 the tile kernel covers all rows with one 128-row tile per column
// block; its K blocks are split over the `ks` CTAs of a thread-block cluster,
// which sum their FP32 partials through distributed shared memory.  With the
// token rows on the MMA's M side each promotion thread scales one row by two
// scalars per K block (the swap-AB decode kernel needs a scale per column).
// FG_TILE_SPLITK=0 / 1 forbids / forces it; by default it serves 64 < M <= 128
// when the splits stay long enough (see splitk_plan).
struct SplitKPlan {
    bool on = false;
    int bn = 0, ks = 0, ks_per = 0, tiles = 0;
};

cudaError_t max_split_clusters(int bn, int cluster, int* out) {
    switch (bn) {
#define FG8_CASE(BNV) \
    case BNV:         \
        return gemm_max_split_clusters<BNV>(cluster, out);
        FG8_FOR_EACH_BN(FG8_CASE)
#undef FG8_CASE
        default:
            return cudaErrorInvalidValue;
    }
}

// The largest resident split count for block width bn (0 when none >= 2).
SplitKPlan splitk_for_width(int bn, int N, int KB, int sms) {
    SplitKPlan sp;
    const int tiles = (N + bn - 1) / bn;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return sp;
    }
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, int> cache;   // (device, bn, cluster) -> resident clusters
    for (int ks = std::min({8, KB, sms / std::max(1, tiles)}); ks >= 2; --ks) {
        const int ks_per = (KB + ks - 1) / ks;
        const int ks2 = (KB + ks_per - 1) / ks_per;          // every split gets K blocks
        if (ks2 < 2) continue;
        int mc = 0;
        {
            std::lock_guard<std::mutex> lk(mu);
            auto it = cache.find({dev, bn, ks2});
            if (it != cache.end()) {
                mc = it->second;
            } else {
                if (max_split_clusters(bn, ks2, &mc) != cudaSuccess) {
                    cudaGetLastError();
                    mc = 0;
                }
                cache[{dev, bn, ks2}] = mc;
            }
        }
        if (tiles <= mc) {
            sp.on = true;
            sp.bn = bn;
            sp.ks = ks2;
            sp.ks_per = ks_per;
            sp.tiles = tiles;
            return sp;
        }
    }
    return sp;
}

SplitKPlan splitk_plan(int M, int N, int K, int sms) {
    SplitKPlan off;
    const char* env = std::getenv("FG_TILE_SPLITK");
    const int mode = env ? std::atoi(env) : -1;
    if (mode == 0 || M > BM) return off;
    if (mode < 0 && M <= 64) return off;
    const int KB = K / BK;
    const char* fbn_env = std::getenv("FG_FORCE_BLOCK_N");
    const int fbn = fbn_env ? std::atoi(fbn_env) : 0;
    if (fbn >= 16 && fbn <= 256 && fbn % 16 == 0) return splitk_for_width(fbn, N, KB, sms);
    const int wide = N >= 256 ? 256 : (N + 15) / 16 * 16;
    if (mode > 0) return splitk_for_width(wide, N, KB, sms);
    // Measured on B200 (M=128, back-to-back launches) against the swap-AB
    // decode kernel: 256-wide tiles win when every split keeps >= 24 K blocks
    // (N=7168, K=16384: 34 vs 49 us); otherwise 128-wide tiles (twice the
    // CTAs, four TMEM accumulators) win when a split keeps >= 8 K blocks
    // (N=4096, K=7168: 15.5 vs 17 us; N=7168, K=2048: 12.9 vs 13.5 us); with
    // shorter splits the set-up and the cluster reduction lose.
    const SplitKPlan w = splitk_for_width(wide, N, KB, sms);
    if (w.on && w.ks_per >= 24) return w;
    if (N >= 256) {
        const SplitKPlan h = splitk_for_width(128, N, KB, sms);
        if (h.on && h.ks_per >= 8) return h;
    }
    return off;
}

fg_status run_gemm_splitk(const SplitKPlan& sp, const void* A, const float* sfa, const void* B, const float* sfb,
                          void* D, int M, int N, int K, cudaStream_t stream) {
    DeviceInfo* dev = nullptr;
    fg_status st = current_device(&dev);
    if (st != FG_OK) return st;
    const int bn = sp.bn;
    const int stages = choose_stages(bn, false);
    const size_t smem = gemm_smem_bytes(stage_bytes_for(bn, false), stages, false);
    // The partial of a split ([128 rows][bn] FP32) is staged in the stage ring.
    if (static_cast<size_t>(BM) * bn * sizeof(float) > static_cast<size_t>(stages) * stage_bytes_for(bn, false))
        return FG_ERR_UNSUPPORTED;
    CUtensorMap ta, tb, td;
    st = operand_map(A, K, M, 1, BM, &ta);
    if (st != FG_OK) return st;
    st = operand_map(B, K, N, 1, bn, &tb);
    if (st != FG_OK) return st;
    st = output_map(D, N, M, 1, &td);
    if (st != FG_OK) return st;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.layout = LAYOUT_NORMAL;
    p.rows = M;
    p.N = N;
    p.K = K;
    p.G = 1;
    p.KB = K / BK;
    p.NB = (N + 127) / 128;
    p.num_m_tiles = 1;
    p.num_n_blocks = sp.tiles;
    p.raster_m = 1;
    p.stages = stages;
    p.sfa_ld = static_cast<int>(fg_get_tma_aligned_size(M, 4));
    p.sfa = sfa;
    p.sfb = sfb;
    p.D = static_cast<__nv_bfloat16*>(D);
    p.status = dev->status;
    p.wait_limit_ns = g_wait_limit_ns.load();
    p.ks = sp.ks;
    p.ks_per = sp.ks_per;
    return launch_bn(bn, false, ta, tb, td, p, sp.tiles * sp.ks, smem, stream, sp.ks);
}

// Shared by the three GEMM kinds once their arguments are checked.
fg_status run_gemm(int layout, const void* A, const float* sfa, const void* B, const float* sfb, void* D,
                   const int* m_indices, const int* masked_m, int rows, int N, int K, int G, int valid_rows_hint,
                   cudaStream_t stream) {
    DeviceInfo* dev = nullptr;
    fg_status st = current_device(&dev);
    if (st != FG_OK) return st;
    const int num_sms = effective_sms(*dev);
    const int KB = K / BK;
    const int NB = (N + 127) / 128;
    const int a_groups = layout == LAYOUT_MASKED ? G : 1;
    const double hbm = static_cast<double>(a_groups) * std::min(rows, std::max(1, valid_rows_hint)) * K +
                       static_cast<double>(G) * N * K + 2.0 * a_groups * rows * N;
    const Choice c = choose_config(layout, rows, a_groups, layout == LAYOUT_MASKED ? valid_rows_hint : rows, N, K,
                                   num_sms, hbm);
    const int bn = c.bn;
    const int tile_m = c.pair ? 2 * BM : BM;
    const int stages = choose_stages(bn, c.pair);
    const size_t smem = gemm_smem_bytes(stage_bytes_for(bn, c.pair), stages, c.pair);

    CUtensorMap ta, tb, td;
    st = operand_map(A, K, rows, a_groups, BM, &ta);
    if (st != FG_OK) return st;
    st = operand_map(B, K, N, G, c.pair ? bn / 2 : bn, &tb);
    if (st != FG_OK) return st;
    st = output_map(D, N, rows, a_groups, &td);
    if (st != FG_OK) return st;

    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.layout = layout;
    p.rows = rows;
    p.N = N;
    p.K = K;
    p.G = G;
    p.KB = KB;
    p.NB = NB;
    p.num_m_tiles = (rows + tile_m - 1) / tile_m;
    p.num_n_blocks = (N + bn - 1) / bn;
    p.raster_m = c.pair ? 8 : 16;
    p.stages = stages;
    p.sfa_ld = static_cast<int>(fg_get_tma_aligned_size(rows, 4));
    p.sfa = sfa;
    p.sfb = sfb;
    p.D = static_cast<__nv_bfloat16*>(D);
    p.m_indices = m_indices;
    p.masked_m = masked_m;
    p.status = dev->status;
    p.wait_limit_ns = g_wait_limit_ns.load();

    // Upper bound of the tiles (the masked and contiguous schedulers may find fewer on the device).
    const long long row_tiles = layout == LAYOUT_CONTIGUOUS ? (c.pair ? rows / BM : p.num_m_tiles)
                                                            : static_cast<long long>(a_groups) * p.num_m_tiles;
    const long long tiles = row_tiles * p.num_n_blocks;
    const int units = c.pair ? num_sms / 2 : num_sms;
    long long used = std::max<long long>(1, std::min<long long>(tiles, units));
    if (layout == LAYOUT_NORMAL) {
        const StreamKPlan sp = streamk_plan(tiles, units, KB);
        if (sp.on) {
            used = units;
            const size_t ctas = static_cast<size_t>(c.pair ? 2 * used : used);
            int dev_id = 0;
            cudaGetDevice(&dev_id);
            st = get_streamk_workspace(dev_id, stream, ctas * BM * bn * sizeof(float), ctas * NUM_EPI_WARPS, &p.sk_ws,
                                       &p.sk_flags, &p.sk_epoch);
            if (st != FG_OK) return st;
            p.sk = 1;
            p.sk_dp_tiles = sp.dp_tiles;
            p.sk_iters = sp.iters;
        }
    }
    const int grid = static_cast<int>(c.pair ? 2 * used : used);
    if (jit_enabled() && jit_launch_gemm(bn, c.pair, ta, tb, td, p, grid, smem, stream) == FG_OK) return FG_OK;
    return launch_bn(bn, c.pair, ta, tb, td, p, grid, smem, stream);
}

__global__ void sfa_transform_kernel(const float* __restrict__ in, float* __restrict__ out, int G, int M, int KB,
                                     int M_pad) {
    // One thread per output element, consecutive threads along m (coalesced stores).
    const long long total = static_cast<long long>(G) * KB * M_pad;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int m = static_cast<int>(i % M_pad);
        const long long gk = i / M_pad;
        const int kb = static_cast<int>(gk % KB);
        const int g = static_cast<int>(gk / KB);
        out[i] = m < M ? in[(static_cast<long long>(g) * M + m) * KB + kb] : 0.0f;
    }
}

struct EnvInit {
    EnvInit() {
        const char* w = std::getenv("FG_WAIT_LIMIT_NS");
        if (w) {
            unsigned long long v = std::strtoull(w, nullptr, 10);
            if (v >= 1000) g_wait_limit_ns.store(v);
        }
    }
} g_env_init;

}  // namespace
}  // namespace fg8

using namespace fg8;

extern "C" {

const char* fg_status_string(int s) {
    switch (s) {
        case FG_OK: return "FG_OK";
        case FG_ERR_INVALID_ARG: return "FG_ERR_INVALID_ARG";
        case FG_ERR_ALIGNMENT: return "FG_ERR_ALIGNMENT";
        case FG_ERR_UNSUPPORTED: return "FG_ERR_UNSUPPORTED";
        case FG_ERR_NO_DEVICE: return "FG_ERR_NO_DEVICE";
        case FG_ERR_CUDA: return "FG_ERR_CUDA";
        case FG_ERR_TIMEOUT: return "FG_ERR_TIMEOUT";
        default: return "FG_ERR_UNKNOWN";
    }
}

const char* fg_version(void) { return "fg8 0.1.0 sm_100a"; }

fg_status fg_fp8_gemm_nt(const void* A, const float* sfa, const void* B, const float* sfb, void* D, int M, int N,
                         int K, fg_stream_t stream) {
    if (M < 0 || N < 0 || K < 0) return FG_ERR_INVALID_ARG;
    if (K == 0 || K % 128 != 0 || N % 16 != 0) return FG_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return FG_OK;
    if (!A || !sfa || !B || !sfb || !D) return FG_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned4(sfb))
        return FG_ERR_ALIGNMENT;
    if (static_cast<long long>(M) * N > kMaxDim * 4 || M > kMaxDim - 128) return FG_ERR_UNSUPPORTED;
    if (M <= std::min(decode_max_rows(), 256)) {
        DeviceInfo* dev = nullptr;
        if (current_device(&dev) == FG_OK) {
            const SplitKPlan sp = splitk_plan(M, N, K, effective_sms(*dev));
            // A launch that is refused (nothing ran) falls back to the decode kernel.
            if (sp.on && run_gemm_splitk(sp, A, sfa, B, sfb, D, M, N, K, reinterpret_cast<cudaStream_t>(stream)) == FG_OK)
                return FG_OK;
        }
        return run_decode(A, sfa, B, sfb, D, M, N, K, reinterpret_cast<cudaStream_t>(stream));
    }
    return run_gemm(LAYOUT_NORMAL, A, sfa, B, sfb, D, nullptr, nullptr, M, N, K, 1, M,
                    reinterpret_cast<cudaStream_t>(stream));
}

fg_status fg_m_grouped_fp8_gemm_nt_contiguous(const void* A, const float* sfa, const void* B, const float* sfb,
                                              void* D, const int* m_indices, int M_tot, int N, int K, int G,
                                              fg_stream_t stream) {
    if (M_tot < 0 || N < 0 || K < 0 || G <= 0) return FG_ERR_INVALID_ARG;
    if (K == 0 || K % 128 != 0 || N % 16 != 0) return FG_ERR_UNSUPPORTED;
    if (M_tot % fg_get_m_alignment_for_contiguous_layout() != 0) return FG_ERR_INVALID_ARG;
    if (M_tot == 0 || N == 0) return FG_OK;
    if (!A || !sfa || !B || !sfb || !D || !m_indices) return FG_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned4(sfb) ||
        !aligned4(m_indices))
        return FG_ERR_ALIGNMENT;
    if (M_tot > kMaxDim - 128) return FG_ERR_UNSUPPORTED;
    return run_gemm(LAYOUT_CONTIGUOUS, A, sfa, B, sfb, D, m_indices, nullptr, M_tot, N, K, G, BM,
                    reinterpret_cast<cudaStream_t>(stream));
}

fg_status fg_m_grouped_fp8_gemm_nt_masked(const void* A, const float* sfa, const void* B, const float* sfb,
                                          void* D, const int* masked_m, int G, int M_max, int N, int K,
                                          int expected_m, fg_stream_t stream) {
    if (G < 0 || M_max < 0 || N < 0 || K < 0 || expected_m < 0) return FG_ERR_INVALID_ARG;
    if (K == 0 || K % 128 != 0 || N % 16 != 0) return FG_ERR_UNSUPPORTED;
    if (G == 0 || M_max == 0 || N == 0) return FG_OK;
    if (!A || !sfa || !B || !sfb || !D || !masked_m) return FG_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned4(sfb) ||
        !aligned4(masked_m))
        return FG_ERR_ALIGNMENT;
    if (static_cast<long long>(G) * M_max > kMaxDim - 128) return FG_ERR_UNSUPPORTED;
    const int hint = expected_m > 0 ? std::min(expected_m, M_max) : M_max;
    return run_gemm(LAYOUT_MASKED, A, sfa, B, sfb, D, nullptr, masked_m, M_max, N, K, G, hint,
                    reinterpret_cast<cudaStream_t>(stream));
}

int fg_get_num_sms(void) {
    const int n = g_num_sms.load();
    if (n > 0) return n;
    DeviceInfo* d = nullptr;
    if (current_device(&d) != FG_OK) {
        const char* env = std::getenv("FG_NUM_SMS");
        return env ? std::max(0, std::atoi(env)) : 0;
    }
    return effective_sms(*d);
}

fg_status fg_set_num_sms(int n) {
    if (n <= 0) return FG_ERR_INVALID_ARG;
    DeviceInfo* d = nullptr;
    const fg_status st = current_device(&d);
    if (st == FG_OK && n > d->sm_count) return FG_ERR_INVALID_ARG;
    g_num_sms.store(n);
    return FG_OK;
}

int fg_get_m_alignment_for_contiguous_layout(void) { return BM; }

size_t fg_get_tma_aligned_size(size_t n, size_t elem_bytes) {
    if (elem_bytes == 0 || 16 % elem_bytes != 0) return 0;
    const size_t a = 16 / elem_bytes;
    return (n + a - 1) / a * a;
}

fg_status fg_transform_sfa_to_tma_layout(const float* in, float* out, int G, int M, int KB, fg_stream_t stream) {
    if (G < 0 || M < 0 || KB < 0) return FG_ERR_INVALID_ARG;
    if (G == 0 || M == 0 || KB == 0) return FG_OK;
    if (!in || !out) return FG_ERR_INVALID_ARG;
    if (!aligned4(in) || !aligned16(out)) return FG_ERR_ALIGNMENT;
    DeviceInfo* d = nullptr;
    fg_status st = current_device(&d);
    if (st != FG_OK) return st;
    const int M_pad = static_cast<int>(fg_get_tma_aligned_size(M, 4));
    const long long total = static_cast<long long>(G) * KB * M_pad;
    const int threads = 256;
    const long long blocks = std::min<long long>((total + threads - 1) / threads, 8LL * d->sm_count);
    sfa_transform_kernel<<<static_cast<int>(blocks), threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        in, out, G, M, KB, M_pad);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FG_OK : FG_ERR_CUDA;
}

fg_status fg_get_last_device_status(fg_stream_t stream, int* code_out, int* detail_out) {
    if (!code_out) return FG_ERR_INVALID_ARG;
    DeviceInfo* d = nullptr;
    fg_status st = current_device(&d);
    if (st != FG_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return FG_ERR_CUDA;
    }
    int h[2] = {0, 0};
    const int zero[2] = {0, 0};
    if (cudaMemcpyFromSymbol(h, g_status, sizeof(h)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_status, zero, sizeof(zero)) != cudaSuccess) {
        cudaGetLastError();
        return FG_ERR_CUDA;
    }
    *code_out = h[0];
    if (detail_out) *detail_out = h[1];
    if (h[0] != 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        clear_workspace_counters(dev);
    }
    return FG_OK;
}

fg_status fg_set_wait_limit_ns(unsigned long long ns) {
    if (ns < 1000) return FG_ERR_INVALID_ARG;
    g_wait_limit_ns.store(ns);
    return FG_OK;
}

unsigned long long fg_get_wait_limit_ns(void) { return g_wait_limit_ns.load(); }

int fg_query_block_n(int M, int N, int K) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 128 != 0 || N % 16 != 0) return 0;
    DeviceInfo* d = nullptr;
    int sms = 148;
    if (current_device(&d) == FG_OK) sms = effective_sms(*d);
    else if (g_num_sms.load() > 0) sms = g_num_sms.load();
    const double hbm = static_cast<double>(M) * K + static_cast<double>(N) * K + 2.0 * M * N;
    const Choice c = choose_config(LAYOUT_NORMAL, M, 1, M, N, K, sms, hbm);
    return c.pair ? -c.bn : c.bn;
}

fg_status fg_query_plan(int layout, int rows, int N, int K, int G, int expected_m, int* kernel_out,
                        int* tile_n_out, int* pair_out, int* splits_out, int* cluster_out) {
    if (!kernel_out || !tile_n_out || !pair_out || !splits_out || !cluster_out) return FG_ERR_INVALID_ARG;
    if (layout < LAYOUT_NORMAL || layout > LAYOUT_MASKED || rows <= 0 || N <= 0 || K <= 0 || G <= 0 ||
        expected_m < 0)
        return FG_ERR_INVALID_ARG;
    if (K % 128 != 0 || N % 16 != 0) return FG_ERR_UNSUPPORTED;
    DeviceInfo* d = nullptr;
    int sms = 148;
    int dev_id = -1;
    if (current_device(&d) == FG_OK) {
        sms = effective_sms(*d);
        cudaGetDevice(&dev_id);
    } else if (g_num_sms.load() > 0) {
        sms = g_num_sms.load();
    }
    if (layout == LAYOUT_NORMAL && rows <= std::min(decode_max_rows(), 256)) {
        if (dev_id >= 0) {
            const SplitKPlan sk = splitk_plan(rows, N, K, sms);
            if (sk.on) {
                *kernel_out = 0;
                *tile_n_out = sk.bn;
                *pair_out = 0;
                *splits_out = sk.ks;
                *cluster_out = sk.ks;
                return FG_OK;
            }
        }
        const int mt = decode_tile_width(rows);
        const int stages = decode_stages(mt);
        const size_t smem = decode_smem_bytes(BM * BK + mt * BK, stages, mt);
        // Without a device the cluster residency cannot be queried: the plan
        // then assumes no cluster launch (the workspace reduction).
        const DecodePlan plan = dev_id >= 0 ? decode_plan(dev_id, mt, smem, stages * (BM * BK + mt * BK), N, K, sms)
                                            : decode_plan(0, mt, smem, 0, N, K, sms);
        *kernel_out = 1;
        *tile_n_out = mt;
        *pair_out = 0;
        *splits_out = plan.splits;
        *cluster_out = plan.cluster;
        return FG_OK;
    }
    const int a_groups = layout == LAYOUT_MASKED ? G : 1;
    const int hint = layout == LAYOUT_MASKED ? (expected_m > 0 ? std::min(expected_m, rows) : rows)
                     : layout == LAYOUT_CONTIGUOUS ? BM : rows;
    const double hbm = static_cast<double>(a_groups) * std::min(rows, std::max(1, hint)) * K +
                       static_cast<double>(G) * N * K + 2.0 * a_groups * rows * N;
    const Choice c = choose_config(layout, rows, a_groups, layout == LAYOUT_MASKED ? hint : rows, N, K, sms, hbm);
    *kernel_out = 0;
    *tile_n_out = c.bn;
    *pair_out = c.pair ? 1 : 0;
    *splits_out = 1;
    *cluster_out = c.pair ? 2 : 1;
    return FG_OK;
}

}  // extern "C"

// ---- few-rows GEMM on library-owned scratch (fg_fp8_gemm_nt_small_m_no_alloc) --
namespace fg8 {

// Split-K scratch of the no-allocation entry point, one copy per device:
// [FG_NO_ALLOC_MAX_N / 128 arrival counters (unsigned)]
// [FG_NO_ALLOC_PARTIAL_FLOATS partial sums (float)].
// Host code must not use this name as an address; it takes the device address
// from cudaGetSymbolAddress (no_alloc_scratch below).
constexpr size_t kNoAllocCounterBytes = static_cast<size_t>(FG_NO_ALLOC_MAX_N / BM) * sizeof(unsigned);
static_assert(kNoAllocCounterBytes % 256 == 0, "partials start 256-byte aligned");
static __device__ __align__(256) unsigned char g_no_alloc_scratch[FG_NO_ALLOC_SCRATCH_BYTES];

namespace {

unsigned char* g_no_alloc_ptr[kMaxDevices];
std::mutex g_no_alloc_mutex;

// Device address of the scratch on device `dev` (current), looked up once.
fg_status no_alloc_scratch(int dev, unsigned char** out) {
    std::lock_guard<std::mutex> lk(g_no_alloc_mutex);
    if (!g_no_alloc_ptr[dev]) {
        void* addr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&addr, g_no_alloc_scratch);
        if (e != cudaSuccess || !addr) {
            cudaGetLastError();
            return FG_ERR_CUDA;
        }
        g_no_alloc_ptr[dev] = static_cast<unsigned char*>(addr);
    }
    *out = g_no_alloc_ptr[dev];
    return FG_OK;
}

// The operand descriptor of operand_map, encoded on the stack (no cache).
fg_status operand_map_uncached(const void* ptr, uint64_t K, uint64_t rows, uint32_t box_rows, CUtensorMap* out) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return FG_ERR_NO_DEVICE;
    std::memset(out, 0, sizeof(*out));
    const cuuint64_t dims[3] = {K, rows, 1};
    const cuuint64_t strides[2] = {K, K * rows};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FG_OK : FG_ERR_CUDA;
}

// The decode kernel in workspace mode with the scratch above as workspace.
fg_status run_decode_no_alloc(const void* A, const float* sfa, const void* B, const float* sfb, void* D, int M,
                              int N, int K, cudaStream_t stream) {
    DeviceInfo* dev = nullptr;
    fg_status st = current_device(&dev);
    if (st != FG_OK) return st;
    int dev_id = 0;
    if (cudaGetDevice(&dev_id) != cudaSuccess) {
        cudaGetLastError();
        return FG_ERR_CUDA;
    }
    unsigned char* scratch = nullptr;
    st = no_alloc_scratch(dev_id, &scratch);
    if (st != FG_OK) return st;
    const int num_sms = effective_sms(*dev);
    const int mt = decode_tile_width(M);
    const int stages = decode_stages(mt);
    if (stages < decode_nbuf(mt)) return FG_ERR_UNSUPPORTED;
    const size_t smem = decode_smem_bytes(BM * BK + mt * BK, stages, mt);
    // No room for cluster staging: the plan picks the workspace reduction.
    DecodePlan plan = decode_plan(dev_id, mt, smem, 0, N, K, num_sms);
    const int KB = K / BK;
    const int NB = (N + BM - 1) / BM;
    int splits = plan.splits;
    while (splits > 1 && static_cast<size_t>(NB) * splits * mt * BM > FG_NO_ALLOC_PARTIAL_FLOATS) --splits;

    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = K;
    p.KB = KB;
    p.NB = NB;
    p.splits = splits;
    p.kb_per_split = (KB + splits - 1) / splits;
    p.units = NB * splits;
    p.cluster_reduce = 0;
    p.stages = stages;
    p.sfa_ld = static_cast<int>(fg_get_tma_aligned_size(M, 4));
    p.sfa = sfa;
    p.sfb = sfb;
    p.D = static_cast<__nv_bfloat16*>(D);
    p.status = dev->status;
    p.wait_limit_ns = g_wait_limit_ns.load();
    if (splits > 1) {
        p.counters = reinterpret_cast<unsigned*>(scratch);
        p.workspace = reinterpret_cast<float*>(scratch + kNoAllocCounterBytes);
        // The counters must start at zero; an earlier call may have left any value.
        if (cudaMemsetAsync(p.counters, 0, static_cast<size_t>(NB) * sizeof(unsigned), stream) != cudaSuccess) {
            cudaGetLastError();
            return FG_ERR_CUDA;
        }
    }
    CUtensorMap ta, tb;
    st = operand_map_uncached(A, K, M, mt, &ta);
    if (st != FG_OK) return st;
    st = operand_map_uncached(B, K, N, BM, &tb);
    if (st != FG_OK) return st;
    const int grid = std::max(1, std::min(p.units, num_sms));
    return launch_decode_mt(mt, ta, tb, p, grid, 1, smem, stream);
}

}  // namespace
}  // namespace fg8

extern "C" fg_status fg_fp8_gemm_nt_small_m_no_alloc(const void* A, const float* sfa, const void* B,
                                                     const float* sfb, void* D, int M, int N, int K,
                                                     fg_stream_t stream) {
    if (M < 0 || N < 0 || K < 0) return FG_ERR_INVALID_ARG;
    if (K == 0 || K % 128 != 0 || N % 16 != 0) return FG_ERR_UNSUPPORTED;
    if (M > FG_NO_ALLOC_MAX_M || N > FG_NO_ALLOC_MAX_N) return FG_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return FG_OK;
    if (!A || !sfa || !B || !sfb || !D) return FG_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(sfa) || !aligned4(sfb))
        return FG_ERR_ALIGNMENT;
    return run_decode_no_alloc(A, sfa, B, sfb, D, M, N, K, reinterpret_cast<cudaStream_t>(stream));
}
