// rtc_compat.cuh -- the few host-library types the kernels need, so that the
// same kernel headers compile both under nvcc (ahead of time) and under NVRTC
// (runtime specialisation), where <cstdint> and <cuda.h> are not available.
#pragma once

#ifdef __CUDACC_RTC__
typedef unsigned char uint8_t;
typedef unsigned short uint16_t;
typedef int int32_t;
typedef unsigned int uint32_t;
typedef long long int64_t;
typedef unsigned long long uint64_t;
typedef unsigned long long uintptr_t;
// Same size and alignment as the driver's opaque tensor-map type.
struct alignas(64) CUtensorMap_st {
    unsigned long long opaque[16];
};
typedef CUtensorMap_st CUtensorMap;
#else
#include <cstdint>
#include <cuda.h>
#endif
