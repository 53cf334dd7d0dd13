// kda_common.cuh -- small device helpers shared by the KDA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Sticky device status word (one per device that loads the library). A
// kernel whose bounded wait gives up ORs in a flag and records where.
struct DeviceStatus {
  int flags;   // bit 0: a bounded wait timed out
  int detail;  // code of the first wait that gave up
};

// Defined once: the library is a single translation unit (kda_lib.cu).
__device__ DeviceStatus g_status = {0, 0};

constexpr int kStatusTimeout = 1;

__device__ __forceinline__ void report_timeout(int where) {
  if (atomicOr(&g_status.flags, kStatusTimeout) == 0) g_status.detail = where;
}

// Element loads/stores for the two supported I/O types.
template <typename T> struct Io;

template <> struct Io<float> {
  static __device__ __forceinline__ float load(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
};

template <> struct Io<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
  }
};

// Sequence bounds of chain `seq`: either cu_seqlens (clamped into [0, T]) or
// the dense layout seq * T.
__device__ __forceinline__ void seq_bounds(const int32_t* cu, int seq, int T,
                                           long long* begin, long long* end) {
  if (cu) {
    int b = cu[seq], e = cu[seq + 1];
    b = b < 0 ? 0 : (b > T ? T : b);
    e = e < b ? b : (e > T ? T : e);
    *begin = b;
    *end = e;
  } else {
    *begin = (long long)seq * T;
    *end = (long long)seq * T + T;
  }
}

}  // namespace kda
