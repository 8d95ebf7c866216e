// layout.cu -- one-time re-layout of a layer's weights inside sfnn_create.
//
// Neurons are stored hottest first (internal position p holds original neuron
// perm[p]), after PowerInfer's offline split of neurons into frequently and
// rarely activated ones (53ai.com "sparsity for LLM inference" page, section
// 概述).  Each neuron's rows are stored together -- (gate,) up, and its column
// of W_down as a contiguous row -- so that one active neuron is one contiguous
// record of nproj*d elements: inactive rows are whole records that are never
// touched, the row/column-structured sparsity the same page (section 激活稀疏)
// calls hardware friendly.  These kernels only move bits; they run once.
#include "common.cuh"
#include "launch.cuh"

namespace sfnn {
namespace {

// dst row p, projection slot `slot`: copy of src row perm[p] (rows of length d).
template <typename E>
__global__ void k_gather_rows(const E *__restrict__ src, const int32_t *__restrict__ perm, E *__restrict__ rows,
                              int n, int d, int nproj, int slot) {
  int p = blockIdx.x;
  if (p >= n) return;
  const E *s = src + (size_t)perm[p] * d;
  E *o = rows + ((size_t)p * nproj + slot) * d;
  for (int k = threadIdx.x; k < d; k += blockDim.x) o[k] = s[k];
}

// dst[map(c) * dst_stride + rr] = src[rr * C + c] for a row-major src [R x C];
// map = identity when cmap is null.  32x32 tiles through shared memory.
template <typename E>
__global__ void k_transpose(const E *__restrict__ src, int R, int C, E *__restrict__ dst, int64_t dst_stride,
                            const int32_t *__restrict__ cmap) {
  __shared__ E tile[32][33];
  int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  int tx = threadIdx.x, ty = threadIdx.y;
  for (int m = ty; m < 32; m += blockDim.y) {
    int rr = r0 + m, cc = c0 + tx;
    if (rr < R && cc < C) tile[m][tx] = src[(size_t)rr * C + cc];
  }
  __syncthreads();
  for (int m = ty; m < 32; m += blockDim.y) {
    int cc = c0 + m, rr = r0 + tx;
    if (cc < C && rr < R) {
      int64_t orow = cmap ? cmap[cc] : cc;
      dst[orow * dst_stride + rr] = tile[tx][m];
    }
  }
}

template <typename E>
__global__ void k_gather_vec(const E *__restrict__ src, const int32_t *__restrict__ perm, E *__restrict__ dst,
                             int n) {
  int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p < n) dst[p] = src[perm[p]];
}

template <typename E>
cudaError_t layout_impl(sfnn_ctx *h, const sfnn_layer_desc *desc, cudaStream_t s) {
  const Layout &L = h->L;
  E *rows = static_cast<E *>(h->rows);
  const int nthr = 256;
  int slot = 0;
  if (L.act == SFNN_REGLU) {
    k_gather_rows<E><<<L.n, nthr, 0, s>>>(static_cast<const E *>(desc->w_gate), h->perm, rows, L.n, L.d, L.nproj,
                                          slot++);
  }
  k_gather_rows<E><<<L.n, nthr, 0, s>>>(static_cast<const E *>(desc->w_up), h->perm, rows, L.n, L.d, L.nproj,
                                        slot++);
  dim3 tb(32, 8);
  // W_down [d x n] -> rows[iperm[i]][slot][k]
  k_transpose<E><<<dim3((L.n + 31) / 32, (L.d + 31) / 32), tb, 0, s>>>(
      static_cast<const E *>(desc->w_down), L.d, L.n, rows + (size_t)slot * L.d, (int64_t)L.nproj * L.d, h->iperm);
  // A [d x r] -> At [r x d]
  k_transpose<E><<<dim3((L.r + 31) / 32, (L.d + 31) / 32), tb, 0, s>>>(
      static_cast<const E *>(desc->pa), L.d, L.r, static_cast<E *>(h->At), (int64_t)L.d, nullptr);
  // B [r x n] -> Bt [iperm[i]][j]
  k_transpose<E><<<dim3((L.n + 31) / 32, (L.r + 31) / 32), tb, 0, s>>>(
      static_cast<const E *>(desc->pb), L.r, L.n, static_cast<E *>(h->Bt), (int64_t)L.r, h->iperm);
  k_gather_vec<E><<<(L.n + 255) / 256, 256, 0, s>>>(static_cast<const E *>(desc->pc), h->perm,
                                                     static_cast<E *>(h->cvec), L.n);
  k_gather_vec<E><<<(L.n + 255) / 256, 256, 0, s>>>(static_cast<const E *>(desc->b), h->perm,
                                                     static_cast<E *>(h->bias), L.n);
  return cudaGetLastError();
}

// Quantized rows: one CTA per (neuron, projection) row of d fp16 values; in fp32, scale =
// max|w| / qmax and code = w / scale rounded to nearest even, clamped to +-qmax, with
// qmax = 127 (int8, one code per byte) or 7 (int4, two per byte, element 2k in the low
// nibble of byte k); an all-zero row: scale 0, codes 0.
template <int BITS>
__global__ void __launch_bounds__(256) k_quantize_rows(const __half *__restrict__ src, int d,
                                                       uint8_t *__restrict__ q, float *__restrict__ scale) {
  constexpr int QMAX = BITS == 8 ? 127 : 7;
  __shared__ float red[8];
  const size_t u = blockIdx.x;
  const __half *w = src + u * d;
  float m = 0.f;
  for (int k = threadIdx.x; k < d; k += blockDim.x) m = fmaxf(m, fabsf(__half2float(w[k])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float sc = red[0] / (float)QMAX;
  if (threadIdx.x == 0) scale[u] = sc;
  auto code = [&](int k) {
    int c = 0;
    if (sc > 0.f) {
      c = __float2int_rn(__half2float(w[k]) / sc);
      c = c > QMAX ? QMAX : (c < -QMAX ? -QMAX : c);
    }
    return c;
  };
  if (BITS == 8) {
    for (int k = threadIdx.x; k < d; k += blockDim.x) q[u * d + k] = (uint8_t)(int8_t)code(k);
  } else {  // two codes per byte, element 2k in the low nibble
    for (int k = threadIdx.x; k < d / 2; k += blockDim.x)
      q[u * (d / 2) + k] = (uint8_t)((code(2 * k) & 0xf) | ((code(2 * k + 1) & 0xf) << 4));
  }
}

}  // namespace

cudaError_t launch_layout(sfnn_ctx *h, const sfnn_layer_desc *desc, cudaStream_t s) {
  if (!h->L.rows_q) {
    if (h->L.esize == 2) return layout_impl<uint16_t>(h, desc, s);
    return layout_impl<uint32_t>(h, desc, s);
  }
  // fp16 rows in a temporary buffer, then their codes and scales
  const Layout &L = h->L;
  void *codes = h->rows, *tmp = nullptr;
  const size_t units = (size_t)L.n * L.nproj;
  cudaError_t e = cudaMalloc(&tmp, units * L.d * 2);
  if (e != cudaSuccess) return e;
  h->rows = tmp;
  e = layout_impl<uint16_t>(h, desc, s);
  h->rows = codes;
  if (e == cudaSuccess) {
    if (L.rows_q == 8)
      k_quantize_rows<8><<<(unsigned)units, 256, 0, s>>>(static_cast<const __half *>(tmp), L.d,
                                                        static_cast<uint8_t *>(codes), h->rscale);
    else
      k_quantize_rows<4><<<(unsigned)units, 256, 0, s>>>(static_cast<const __half *>(tmp), L.d,
                                                        static_cast<uint8_t *>(codes), h->rscale);
    e = cudaGetLastError();
  }
  const cudaError_t e2 = cudaStreamSynchronize(s);
  cudaFree(tmp);
  return e != cudaSuccess ? e : e2;
}

}  // namespace sfnn
