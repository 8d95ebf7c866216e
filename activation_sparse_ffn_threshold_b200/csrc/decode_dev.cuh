// decode_dev.cuh -- device helpers shared by the fused decode kernels (decode1.cu,
// decode_ahead.cu): 16-byte chunk dot products and the bounded grid barrier.
#pragma once

#include "async.cuh"
#include "common.cuh"
#include "decode1.cuh"

namespace sfnn {

// Storage of the FFN rows a decode kernel reads: the layer's element type, or codes with
// per-row scales (Q8: int8, one per byte; Q4: int4, two per byte, element 2k in the low
// nibble of byte k).
struct Q8 {};
struct Q4 {};
template <typename R>
struct RowFmt {
  static constexpr int kBits = 8 * (int)sizeof(R);
};
template <>
struct RowFmt<Q8> {
  static constexpr int kBits = 8;
};
template <>
struct RowFmt<Q4> {
  static constexpr int kBits = 4;
};

namespace {

constexpr int kT = kDecode1Threads;
constexpr int kW = kT / 32;
constexpr int kSegChunks = 256;  // 16-byte chunks of one C1 segment (8 per lane)
constexpr int kSmemCap = kDecodeSmemCap;

template <typename T>
__device__ __forceinline__ float dot_chunk(const uint4 &w, const float *h, float a) {
  constexpr int V = Elem<T>::kVec;
  float f[V];
  unpack<T>(w, f);
#pragma unroll
  for (int v = 0; v < V; ++v) a = fmaf(f[v], h[v], a);
  return a;
}

// 16 int8 codes of a row (one 16-byte chunk) against x[16 ch .. 16 ch + 15] (fp16 in
// shared memory); the row's scale is applied to the finished sum.
__device__ __forceinline__ float dot_chunk_i8(const uint4 &w, const unsigned char *xs, int ch, float a) {
  float xf[16];
  unpack<__half>(*reinterpret_cast<const uint4 *>(xs + (size_t)ch * 32), xf);
  unpack<__half>(*reinterpret_cast<const uint4 *>(xs + (size_t)ch * 32 + 16), xf + 8);
  const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaf((float)(int8_t)(q[i >> 2] >> (8 * (i & 3))), xf[i], a);
  return a;
}

// 32 int4 codes of a row (one 16-byte chunk) against x[32 ch .. 32 ch + 31] (fp16 in
// shared memory), 8 codes per 32-bit word, low nibble first; the row's scale is applied
// to the finished sum.
__device__ __forceinline__ float dot_chunk_i4(const uint4 &w, const unsigned char *xs, int ch, float a) {
  const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    float xf[8];
    unpack<__half>(*reinterpret_cast<const uint4 *>(xs + (size_t)ch * 64 + h * 16), xf);
#pragma unroll
    for (int j = 0; j < 8; ++j) a = fmaf((float)((int32_t)(q[h] << (28 - 4 * j)) >> 28), xf[j], a);
  }
  return a;
}

template <typename T>
__device__ __forceinline__ float dot_chunk_smem(const uint4 &w, const unsigned char *xs, int ch, float a) {
  constexpr int V = Elem<T>::kVec;
  float f[V], xf[V];
  unpack<T>(w, f);
  unpack<T>(*reinterpret_cast<const uint4 *>(xs + (size_t)ch * 16), xf);
#pragma unroll
  for (int v = 0; v < V; ++v) a = fmaf(f[v], xf[v], a);
  return a;
}

// Two fp16 pairs (the halves of w and x, low half first) accumulated into a by sm_100's
// mixed-precision FMA: it widens the fp16 operands exactly, their product is exact in fp32
// and the sum is rounded once -- the result of widening first and fmaf, in one instruction.
__device__ __forceinline__ float fma_h2(uint32_t w, uint32_t x, float a) {
  asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "fma.rn.f32.f16 %0, wl, xl, %0;\n\t"
      "fma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
      : "+f"(a)
      : "r"(w), "r"(x));
  return a;
}

template <>
__device__ __forceinline__ float dot_chunk_smem<__half>(const uint4 &w, const unsigned char *xs, int ch, float a) {
  const uint4 x = *reinterpret_cast<const uint4 *>(xs + (size_t)ch * 16);
  a = fma_h2(w.x, x.x, a);
  a = fma_h2(w.y, x.y, a);
  a = fma_h2(w.z, x.z, a);
  return fma_h2(w.w, x.w, a);
}

// Grid barrier by thread 0, bracketed by CTA barriers; false (and the error latched)
// if it timed out.  No separate fences: the CTA's writes happen before thread 0's
// release add through the CTA barrier, and another CTA's reads after its thread 0's
// acquire load through its CTA barrier; causality order composes the CTA-scope and
// GPU-scope synchronisations.
__device__ __forceinline__ bool cta_grid_sync(const Decode1Params &P, int *flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = grid_barrier(P.bar, (uint32_t)P.G, kWaitCycles);
    if (!ok) latch_error(P.err, kErrTimeout);
    *flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *reinterpret_cast<volatile int *>(flag) != 0;
}

// The same barrier in two halves, so that a CTA can work between them: every thread
// calls cta_grid_arrive after the CTA's writes that other CTAs read (thread 0 draws the
// ticket), and cta_grid_wait before reading theirs; `slot` keeps the target in shared
// memory.  cta_grid_wait returns false (and the error is latched) if it timed out.
__device__ __forceinline__ void cta_grid_arrive(const Decode1Params &P, unsigned long long *slot) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t ticket = atom_add_release_gpu_u64(P.bar, 1ull);
    *slot = (ticket / (uint32_t)P.G + 1) * (uint32_t)P.G;
  }
}
__device__ __forceinline__ bool cta_grid_wait(const Decode1Params &P, const unsigned long long *slot, int *flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t target = *slot;
    const uint64_t t0 = clock64();
    bool ok = true;
    while (ld_acquire_gpu_u64(P.bar) < target)
      if ((uint64_t)(clock64() - t0) > kWaitCycles) {
        ok = false;
        break;
      }
    if (!ok) latch_error(P.err, kErrTimeout);
    *flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *reinterpret_cast<volatile int *>(flag) != 0;
}

// The fused kernels' final sums.  CTA c owns the columns [c CW, c CW + ncol) of each of
// the NT outputs, CW = ceil(d / G) rounded up to a multiple of 4 so that the partials move
// as float4s.  The G partials part[(k NT + t) d + col] of a column are summed in ngu
// groups of consecutive k in parallel (ascending k within a group, 8 loads in flight),
// ngu a power of two, then the groups pairwise in a fixed tree: deterministic.  `red`
// holds blockDim.x float4s of shared memory; out(t, col, v) receives the sums of columns
// col..col+3 of output t.  The grouping depends on NTMAX (not NT), so that a kernel
// instantiated for several output counts sums each output in the same order.
template <int NT, int NTMAX, class Out>
__device__ __forceinline__ void column_sums(const float *part, int d, int G, float4 *red, Out out) {
  const int c = blockIdx.x, tid = threadIdx.x, nthr = blockDim.x;
  const int CW = (((d + G - 1) / G) + 3) & ~3;
  const int col0 = c * CW;
  const int nq = max(0, min(CW, d - col0)) / 4;  // float4 columns (d is a multiple of 4)
  const int width_all = nq * NT;
  if (width_all == 0) return;
  int ngu = 1;
  while (ngu * 2 <= G && ngu * 2 * min(nq * NTMAX, nthr) <= nthr) ngu *= 2;
  const int pass = nthr / ngu;  // (token, float4 column) pairs per pass
  const size_t kstride = (size_t)NT * d / 4;
  const int gi = tid / pass, j = tid - gi * pass;
  for (int cb = 0; cb < width_all; cb += pass) {
    const int width = min(pass, width_all - cb);
    const int e = cb + j, t = e / nq, q = e - t * nq;
    if (gi < ngu && j < width) {
      const float4 *src = reinterpret_cast<const float4 *>(part + (size_t)t * d + col0) + q;
      const int k0 = (int)(((int64_t)gi * G) / ngu), k1 = (int)(((int64_t)(gi + 1) * G) / ngu);
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int kb = k0; kb < k1; kb += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          v[u] = kb + u < k1 ? __ldcg(src + (size_t)(kb + u) * kstride) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          s.x += v[u].x;
          s.y += v[u].y;
          s.z += v[u].z;
          s.w += v[u].w;
        }
      }
      red[gi * pass + j] = s;
    }
    __syncthreads();
    for (int stride = ngu / 2; stride >= 1; stride /= 2) {  // group gi += group gi + stride
      if (gi < stride && j < width) {
        const float4 a = red[gi * pass + j], b = red[(gi + stride) * pass + j];
        red[gi * pass + j] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
      }
      __syncthreads();
    }
    if (gi == 0 && j < width) out(t, col0 + 4 * q, red[j]);
    __syncthreads();
  }
}

// The split barrier's wait by one warp, so that the CTA's other warps keep working: lane 0
// polls (bounded), and the warp's lanes read other CTAs' writes after the __syncwarp that
// follows its acquire load.  false (and the error latched) if it timed out.
__device__ __forceinline__ bool warp_grid_wait(const Decode1Params &P, const unsigned long long *slot) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    const uint64_t target = *slot;
    const uint64_t t0 = clock64();
    while (ld_acquire_gpu_u64(P.bar) < target)
      if ((uint64_t)(clock64() - t0) > kWaitCycles) {
        ok = false;
        break;
      }
    if (!ok) latch_error(P.err, kErrTimeout);
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  return ok;
}

// Rebalancing of a fused kernel's active rows, after the split barrier's wait, by one
// warp: every tile's count (P.bcnt, clamped to the tile), e_t = the rows past `quota`,
// and CTA c's even share of them, the global excess rows [floor(cE/G), floor((c+1)E/G))
// in tile order -- row g is slot quota + g - epre[t] of the tile t with
// epre[t] <= g < epre[t+1].  `scratch` holds G ints of shared memory.  take(j, entry)
// receives the CTA's j-th extra row's list entry (P.blist); returns the CTA's count of
// extra rows.  A function of the counts alone: every CTA computes the same assignment.
template <class Take>
__device__ __forceinline__ int share_excess_warp(const Decode1Params &P, int quota, int *scratch, Take take) {
  const int lane = threadIdx.x & 31;
  const int G = P.G, c = blockIdx.x;
  int *epre = scratch;
  // lane l takes the tiles [l tpl, (l + 1) tpl) (tpl <= 8: G <= 254), all its counts
  // requested at once; e_t goes to epre[t], then in place to the exclusive prefix
  const int tpl = (G + 31) / 32;
  const int tb = min(G, lane * tpl), te = min(G, tb + tpl);
  int cv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) cv[i] = tb + i < te ? __ldcg(P.bcnt + tb + i) : 0;
  int es = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = tb + i;
    if (t < te) {
      const int sz = decode1_tile_start(t + 1, P.n, G) - decode1_tile_start(t, P.n, G);
      const int e = max(0, min(max(cv[i], 0), sz) - quota);
      epre[t] = e;
      es += e;
    }
  }
  int incl = es;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int be = incl - es;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = tb + i;
    if (t < te) {
      const int e = epre[t];
      epre[t] = be;
      be += e;
    }
  }
  const int E = __shfl_sync(0xffffffffu, incl, 31);
  __syncwarp();
  // CTA c's share: [floor(cE/G), floor((c+1)E/G)), with floor(cE/G) = c q + floor(c rm / G)
  const int q = E / G, rm = E - q * G;
  const int F = c * q + (c * rm) / G;
  const int f = q + ((c + 1) * rm) / G - (c * rm) / G;
  for (int j = lane; j < f; j += 32) {
    const int g = F + j;
    int lo = 0, hi = G;  // the largest t with epre[t] <= g
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (epre[mid] <= g)
        lo = mid;
      else
        hi = mid;
    }
    take(j, __ldcg(P.blist + decode1_tile_start(lo, P.n, G) + quota + (g - epre[lo])));
  }
  __syncwarp();
  return f;
}

// The same by the whole CTA (warp 0 computes it; every thread returns the count, and the
// entries taken are visible to all after it).  `scratch` holds G + 1 ints.
template <class Take>
__device__ __forceinline__ int share_excess(const Decode1Params &P, int quota, int *scratch, Take take) {
  if (threadIdx.x < 32) {
    const int f = share_excess_warp(P, quota, scratch + 1, take);
    if (threadIdx.x == 0) scratch[0] = f;
  }
  __syncthreads();
  const int f = *reinterpret_cast<volatile int *>(scratch);
  __syncthreads();  // every thread has read the count before the scratch is reused
  return f;
}

}  // namespace
}  // namespace sfnn
