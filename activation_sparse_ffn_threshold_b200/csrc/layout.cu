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

}  // namespace

cudaError_t launch_layout(sfnn_ctx *h, const sfnn_layer_desc *desc, cudaStream_t s) {
  if (h->L.esize == 2) return layout_impl<uint16_t>(h, desc, s);
  return layout_impl<uint32_t>(h, desc, s);
}

}  // namespace sfnn
