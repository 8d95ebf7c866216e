// common.cuh -- internal types shared by the sfnn CUDA sources (not part of the C ABI).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "decode1.cuh"
#include "sfnn.h"

namespace sfnn {

constexpr int kMaxBatch = 32;
constexpr int kMaxSplits = 64;  // K-splits of the down projection (partials per token)

// Device-side error word values (a subset of sfnn_status).
constexpr int kErrInvalidIdx = SFNN_ERR_INVALID_ARG;
constexpr int kErrTimeout = SFNN_ERR_TIMEOUT;

struct Layout {
  int d, n, r, nproj, act, dt, esize, vec, nwords;
  int rows_q;  // rows stored as 8- or 4-bit codes with per-row fp32 scales (0: in dt)
};

}  // namespace sfnn


namespace sfnn {

// ---------------------------------------------------------------- element helpers
template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kVec = 4;  // elements per 16-byte vector
};
template <>
struct Elem<__half> {
  static constexpr int kVec = 8;
};

// Read-only 16-byte load from global memory, not kept in L1 (weights stream once).
__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Read-only 16-byte load that may stay in L1 (activations reused by a CTA).
__device__ __forceinline__ uint4 ld_keep(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

template <typename T>
__device__ __forceinline__ void unpack(const uint4 &v, float *f);

template <>
__device__ __forceinline__ void unpack<float>(const uint4 &v, float *f) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}

template <>
__device__ __forceinline__ void unpack<__half>(const uint4 &v, float *f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h2 = *reinterpret_cast<const __half2 *>(&w[i]);
    float2 f2 = __half22float2(h2);
    f[2 * i] = f2.x;
    f[2 * i + 1] = f2.y;
  }
}

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void latch_error(int32_t *err, int code) { atomicCAS(err, 0, code); }

}  // namespace sfnn
