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
// B200 design: the op is HBM-bound (5 bytes per FP32 element, 3 per BF16), so
// one warp handles one 128-element block with 16-byte (FP32) or 8-byte (BF16)
// coalesced loads, a 5-step shuffle max, and one 4-byte store of four codes
// per lane; each warp walks several blocks with their loads issued together.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fg8.h"

namespace fg8q {

constexpr int QBLK = 128;
constexpr int QTHREADS = 256;
// Blocks per warp whose loads are in flight together: 1 KiB per warp for
// either input type, enough bytes in flight per SM to cover HBM latency.
template <typename T>
__host__ __device__ constexpr int qunroll() { return sizeof(T) == 2 ? 4 : 2; }

__device__ __forceinline__ float4 load4(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }

__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    const uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
    float4 f;
    f.x = __uint_as_float(u.x << 16);
    f.y = __uint_as_float(u.x & 0xFFFF0000u);
    f.z = __uint_as_float(u.y << 16);
    f.w = __uint_as_float(u.y & 0xFFFF0000u);
    return f;
}

// x / b rounded to nearest even, given y = the correctly rounded reciprocal
// of b.  Markstein's method (P. Markstein, "IA-64 and Elementary Functions",
// 2000): with the residual r = x - b q computed exactly by an FMA, q + r y
// rounded once is the correctly rounded quotient when q is within one unit in
// the last place of x / b.  x * y alone can be 1.5 units off, so one residual
// step brings it within one unit and a second gives the correctly rounded
// result.  Computed on |x| with the sign put back at the end, so that -0 / b
// stays -0 (a residual step would turn it into +0).  Used for the per-element
// quotients; valid for the normal scales and |x / b| <= 448 (plus rounding)
// of the quantiser.  The tests check the codes bit for bit against IEEE
// division on values within a few units of every E4M3 rounding boundary.
__device__ __forceinline__ float div_rn(float x, float b, float y) {
    const float a = fabsf(x);
    float q = a * y;
    float r = fmaf(-q, b, a);
    q = fmaf(r, y, q);
    r = fmaf(-q, b, a);
    q = fmaf(r, y, q);
    return copysignf(q, x);
}

// Four FP32 -> four E4M3 codes (round to nearest even, saturating), byte i = value i.
__device__ __forceinline__ uint32_t to_e4m3x4(float a, float b, float c, float d) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(a), "f"(b));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(c), "f"(d));
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

template <typename T>
__global__ void __launch_bounds__(QTHREADS, 8) quantize_kernel(const T* __restrict__ x, uint8_t* __restrict__ q,
                                                            float* __restrict__ sfa, int M, int K, int m_pad) {
    const int KB = K / QBLK;
    const long long nblk = static_cast<long long>(M) * KB;
    const int lane = threadIdx.x % 32;
    const long long warps = static_cast<long long>(gridDim.x) * (QTHREADS / 32);
    const long long w0 = static_cast<long long>(blockIdx.x) * (QTHREADS / 32) + threadIdx.x / 32;
    constexpr int QUNROLL = qunroll<T>();
    for (long long base = w0; base < nblk; base += warps * QUNROLL) {
        float4 v[QUNROLL];
#pragma unroll
        for (int u = 0; u < QUNROLL; ++u) {
            const long long b = base + u * warps;
            v[u] = b < nblk ? load4(x + b * QBLK + lane * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < QUNROLL; ++u) {
            const long long b = base + u * warps;
            float amax = fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            if (b >= nblk) continue;   // warp-uniform
            const float scale = fmaxf(amax, 1e-4f) / 448.0f;
            const float rcp = __frcp_rn(scale);
            const uint32_t codes = to_e4m3x4(div_rn(v[u].x, scale, rcp), div_rn(v[u].y, scale, rcp),
                                             div_rn(v[u].z, scale, rcp), div_rn(v[u].w, scale, rcp));
            __stcs(reinterpret_cast<uint32_t*>(q + b * QBLK) + lane, codes);
            if (lane == 0) {
                const long long m = b / KB;
                const int kb = static_cast<int>(b - m * KB);
                sfa[static_cast<long long>(kb) * m_pad + m] = scale;
            }
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
    const int unroll = x_is_bf16 ? qunroll<__nv_bfloat16>() : qunroll<float>();
    const long long warps_needed = (nblk + unroll - 1) / unroll;
    const long long blocks_needed = (warps_needed + QTHREADS / 32 - 1) / (QTHREADS / 32);
    const int grid = static_cast<int>(blocks_needed < 8LL * sms ? (blocks_needed > 0 ? blocks_needed : 1) : 8LL * sms);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (x_is_bf16)
        quantize_kernel<__nv_bfloat16><<<grid, QTHREADS, 0, s>>>(static_cast<const __nv_bfloat16*>(x),
                                                                 static_cast<uint8_t*>(q), sfa, M, K, m_pad);
    else
        quantize_kernel<float><<<grid, QTHREADS, 0, s>>>(static_cast<const float*>(x), static_cast<uint8_t*>(q), sfa,
                                                         M, K, m_pad);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FG_OK : FG_ERR_CUDA;
}
