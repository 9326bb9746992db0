// quant.cu -- activation quantiser: FP32 or BF16 rows -> E4M3 codes plus one
// FP32 scale per 1 x 128 block, the scales written straight into the
// MN-major, TMA-aligned layout the GEMMs read.
//
// The fine-grained scaling of the pages ("as proposed in DeepSeek-V3":
// chujupifa.com "机器之心报道", opening summary) gives each 1 x 128 block of
// an activation row its own FP32 scale; the scale layout is the one made by
// get_col_major_tma_aligned_tensor (deepseek.csdn.net "DeepGEMM：简洁、高效…",
// section "实用工具").  Per block:
//   scale = max(amax, 1e-4) / 448        (FP32; 448 = largest finite E4M3)
//   q     = E4M3(x / scale)              (the FP32 quotient rounded to nearest
//                                         even, then to E4M3, saturating at +-448)
// so the block's largest magnitude lands on 448.  The 1e-4 floor keeps an
// all-zero block finite.
//
// B200 design: the op should be HBM-bound (5 bytes per FP32 element, 3 per
// BF16), so the per-element work is kept to a few instructions: a few lanes
// share a 128-element block (16 or 32 elements each, 16-byte coalesced loads,
// a short shuffle max, 16-byte stores of codes) and a warp covers four or
// eight consecutive blocks per instruction.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fg8.h"

namespace fg8q {

constexpr int QBLK = 128;
constexpr int QTHREADS = 256;
// QL lanes quantise one 128-element block (QBLK / QL elements each), so a
// warp instruction serves 32 / QL blocks: the per-block work (the amax
// reduction, the scale, its reciprocal and the scale store) is shared by
// that many blocks.  Latency is hidden by occupancy (MB CTAs of 256 threads
// per SM), each warp with one group of blocks in flight.  Measured on B200 at
// M=4096, K=7168: FP32 input is fastest with 8 lanes and six CTAs per SM
// (0.87 of HBM; 4 lanes: 0.60), BF16 input with 4 lanes and four CTAs per SM
// (0.61; 8 lanes: 0.55, 16 lanes: 0.43).  Two groups per warp in flight, or
// the next group prefetched, were slower at both.
template <typename T>
struct QCfg;
template <>
struct QCfg<float> {
    static constexpr int QL = 8;
    static constexpr int MB = 6;
};
template <>
struct QCfg<__nv_bfloat16> {
    static constexpr int QL = 4;
    static constexpr int MB = 4;
};

// QBLK / QL consecutive elements as FP32 (streaming loads: the input is read once).
template <int N>
__device__ __forceinline__ void load_elems(const float* p, float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
        const float4 f = __ldcs(reinterpret_cast<const float4*>(p) + i);
        v[4 * i] = f.x;
        v[4 * i + 1] = f.y;
        v[4 * i + 2] = f.z;
        v[4 * i + 3] = f.w;
    }
}

template <int N>
__device__ __forceinline__ void load_elems(const __nv_bfloat16* p, float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p) + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

// x / b rounded to nearest even, given y = the correctly rounded reciprocal
// of b.  Markstein's method (P. Markstein, "IA-64 and Elementary Functions",
// 2000): with the residual r = x - b q computed exactly by an FMA, q + r y
// rounded once is the correctly rounded quotient when q is within one unit in
// the last place of x / b.  x * y alone can be 1.5 units off, so one residual
// step brings it within one unit and a second gives the correctly rounded
// result.  The sign of x is put back at the end, so that -0 / b stays -0 (a
// residual step would turn it into +0).  Used for the per-element quotients;
// valid for the normal scales and |x / b| <= 448 (plus rounding) of the
// quantiser.  The tests check the codes bit for bit against IEEE division on
// values within a few units of every E4M3 rounding boundary.
__device__ __forceinline__ float2 div_rn2(float2 x, float b, float y) {
    // Two quotients per instruction (packed FP32 multiply and FMA, each half
    // rounded to nearest as the scalar operation would be).  The steps run on
    // the signed values: round-to-nearest-even is symmetric, so the result is
    // exactly the negated quotient of |x| except for a zero, whose sign the
    // final copysign restores.
    const float2 y2 = make_float2(y, y);
    const float2 nb2 = make_float2(-b, -b);
    float2 q = __fmul2_rn(x, y2);
    float2 r = __ffma2_rn(q, nb2, x);
    q = __ffma2_rn(r, y2, q);
    r = __ffma2_rn(q, nb2, x);
    q = __ffma2_rn(r, y2, q);
    return make_float2(copysignf(q.x, x.x), copysignf(q.y, x.y));
}

// Four FP32 -> four E4M3 codes (round to nearest even, saturating), byte i = value i.
__device__ __forceinline__ uint32_t to_e4m3x4(float a, float b, float c, float d) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(a), "f"(b));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(c), "f"(d));
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

template <typename T>
__global__ void __launch_bounds__(QTHREADS, QCfg<T>::MB)
    quantize_kernel(const T* __restrict__ x, uint8_t* __restrict__ q, float* __restrict__ sfa, int M, int K, int m_pad) {
    constexpr int QL = QCfg<T>::QL;
    constexpr int QEL = QBLK / QL;                  // elements per lane
    constexpr int BPW = 32 / QL;                    // blocks per warp instruction
    const int KB = K / QBLK;
    const long long nblk = static_cast<long long>(M) * KB;
    const int lane = threadIdx.x % 32;
    const int sub = lane / QL;                      // block of the warp's group
    const int ls = lane % QL;                       // slice of that block
    const long long warps = static_cast<long long>(gridDim.x) * (QTHREADS / 32);
    const long long w0 = static_cast<long long>(blockIdx.x) * (QTHREADS / 32) + threadIdx.x / 32;
    const long long step = warps * BPW;             // blocks per sweep of the whole grid
    for (long long base = w0 * BPW; base < nblk; base += step) {
        const long long b = base + sub;
        float v[QEL];
        if (b < nblk) {
            load_elems<QEL>(x + b * QBLK + ls * QEL, v);
        } else {
#pragma unroll
            for (int i = 0; i < QEL; ++i) v[i] = 0.0f;
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < QEL; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
        for (int o = QL / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (b >= nblk) continue;
        const float scale = fmaxf(amax, 1e-4f) / 448.0f;
        const float rcp = __frcp_rn(scale);
        uint32_t c[QEL / 4];
#pragma unroll
        for (int i = 0; i < QEL / 4; ++i) {
            const float2 lo = div_rn2(make_float2(v[4 * i], v[4 * i + 1]), scale, rcp);
            const float2 hi = div_rn2(make_float2(v[4 * i + 2], v[4 * i + 3]), scale, rcp);
            c[i] = to_e4m3x4(lo.x, lo.y, hi.x, hi.y);
        }
        uint4* dst = reinterpret_cast<uint4*>(q + b * QBLK + ls * QEL);
#pragma unroll
        for (int i = 0; i < QEL / 16; ++i) __stcs(dst + i, make_uint4(c[4 * i], c[4 * i + 1], c[4 * i + 2], c[4 * i + 3]));
        if (ls == 0) {
            // Block b is row m, K block kb (32-bit division whenever the block
            // count allows it).
            long long m;
            if (nblk <= 0x7fffffffLL) m = static_cast<long long>(static_cast<unsigned>(b) / static_cast<unsigned>(KB));
            else m = b / KB;
            const int kb = static_cast<int>(b - m * KB);
            sfa[static_cast<long long>(kb) * m_pad + m] = scale;
        }
    }
    // Padding rows of the MN-major scales are zero.
    const long long npad = static_cast<long long>(m_pad - M) * KB;
    for (long long i = static_cast<long long>(blockIdx.x) * QTHREADS + threadIdx.x; i < npad;
         i += static_cast<long long>(gridDim.x) * QTHREADS) {
        const int kb = static_cast<int>(i / (m_pad - M));
        const int m = M + static_cast<int>(i - static_cast<long long>(kb) * (m_pad - M));
        sfa[static_cast<long long>(kb) * m_pad + m] = 0.0f;
    }
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 0;
    }
    if (cached[dev] == 0) {
        int n = 0, major = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cached[dev] = major == 10 ? n : -1;
    }
    return cached[dev];
}

}  // namespace fg8q

extern "C" fg_status fg_quantize_fp8_activations(const void* x, int x_is_bf16, void* q, float* sfa, int M, int K,
                                                 fg_stream_t stream) {
    using namespace fg8q;
    if (M < 0 || K < 0 || (x_is_bf16 != 0 && x_is_bf16 != 1)) return FG_ERR_INVALID_ARG;
    if (K == 0 || K % QBLK != 0) return FG_ERR_UNSUPPORTED;
    if (M == 0) return FG_OK;
    if (!x || !q || !sfa) return FG_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(q) & 15u) ||
        (reinterpret_cast<uintptr_t>(sfa) & 15u))
        return FG_ERR_ALIGNMENT;
    const int sms = sm_count();
    if (sms <= 0) return FG_ERR_NO_DEVICE;
    const int m_pad = (M + 3) / 4 * 4;
    const long long nblk = static_cast<long long>(M) * (K / QBLK);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // One group of blocks per warp, capped at the resident grid.
    auto grid_for = [&](int blocks_per_warp, int min_blocks) {
        const long long warps_needed = (nblk + blocks_per_warp - 1) / blocks_per_warp;
        const long long ctas = (warps_needed + QTHREADS / 32 - 1) / (QTHREADS / 32);
        const long long cap = static_cast<long long>(min_blocks) * sms;
        return static_cast<int>(ctas < cap ? (ctas > 0 ? ctas : 1) : cap);
    };
    if (x_is_bf16)
        quantize_kernel<__nv_bfloat16>
            <<<grid_for(32 / QCfg<__nv_bfloat16>::QL, QCfg<__nv_bfloat16>::MB), QTHREADS, 0, s>>>(
                static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(q), sfa, M, K, m_pad);
    else
        quantize_kernel<float><<<grid_for(32 / QCfg<float>::QL, QCfg<float>::MB), QTHREADS, 0, s>>>(
            static_cast<const float*>(x), static_cast<uint8_t*>(q), sfa, M, K, m_pad);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FG_OK : FG_ERR_CUDA;
}
