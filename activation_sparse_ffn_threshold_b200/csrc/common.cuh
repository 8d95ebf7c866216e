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

struct sfnn_ctx {
  sfnn::Layout L;
  int max_batch;
  int device;
  int num_sms;
  int batch_path;
  double expected_union[sfnn::kMaxBatch + 1];  // E|U|/n by batch size, from the hotness profile
  // re-laid-out weights (internal neuron order p = 0..n-1, hottest first)
  void *rows;      // [n][nproj][d]: ReLU (up, down); ReGLU (gate, up, down)
  void *At;        // [r][d]
  void *Bt;        // [n][r]
  void *cvec;      // [n]
  void *bias;      // [n]
  int32_t *perm;   // [n] internal -> original
  int32_t *iperm;  // [n] original -> internal
  // scratch
  float *h;          // [2 * max_batch][r]: the hidden layer (fused kernels: per token two half sums)
  uint32_t *mask;    // [max_batch][nwords]
  int32_t *ulist;    // [n] union list (internal positions, ascending)
  uint32_t *utok;    // [n] tokens active on each union row (bit t)
  int32_t *ucount;   // [1]
  float *acoef;      // [n][max_batch] activation of each union row for each token
  float *rscale;     // [n][nproj] scales of quantized rows (storage order), or null
  __half *hact;      // [32][n rounded up to 128] fp16 activations (tensor-core batch path) or null
  __half *hpair;     // [2][32][r] the batch's hidden layer as fp16 hi and lo parts (same path)
  float *part;       // [kMaxSplits][max_batch][d] partial sums of the down projection
  void *xin;         // [max_batch][d] wdtype: layer input inside a stack
  int32_t *err;      // [1] latched device-side error
  uint64_t *bar;     // grid barrier arrival counter of the fused kernel
  int2 *alist;       // [n] look-ahead stack: this layer's predicted active lists per tile
  int32_t *acnt;     // [G]   (storage position, bias) pairs and counts, from the launch before
  int2 *blist;       // [n] rebalancing: each tile's active (storage position, bias) pairs
  int32_t *bcnt;     // [G]   and their counts (single-token fused kernel)
  int quota;         // its per-CTA quota of own rows (0: no rebalancing)
  int quota_multi[sfnn::kMultiMaxTokens + 1];  // the same for the multi-token kernel, by batch size
  bool batch_quota_off;  // the multi-token kernel's rebalancing switched off (batch-invariant rows)
  int mdepth[4];         // the multi-token kernel's request depths (bstages, c2pre, c1depth, c2stages)
  bool auto_chunked[sfnn::kMaxBatch + 1];  // AUTO: b tokens as two few-token launches (measured faster)
  int32_t *scnt;     // [max_batch][G] per-tile counts of the sets a fused launch used (lists: ulist
                     //   for one token, acoef's words for several)
  int multi_max;     // largest batch the multi-token fused kernel serves (0: none)
  int hot_rows[sfnn::kMultiMaxTokens + 1];  // its hot prefix by batch size: ranks in the union w.p. >= 0.99
  bool hot_on;       // the hot prefix is read densely (sfnn_set_hot_prefix)
  bool fused_ok;     // the fused single-token kernel fits this layer
  bool fused_on;     // ... and is enabled (sfnn_set_fused_decode)
  sfnn::Decode1Params d1;  // its launch plan (pointers to x/y filled per call)
  int64_t weight_bytes, scratch_bytes;
  int64_t launches;  // kernels this handle has launched (or captured into a graph)
  // one-shot profiling events around the dominant kernel
  cudaEvent_t prof_before, prof_after;
};

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
