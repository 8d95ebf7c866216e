// predict.cu -- the low-rank neuron predictor and the stream compaction of its decisions.
//
// The predictor marks neuron i active when sigmoid(relu(x.A).B + c)_i > 0.5,
// evaluated as z_i > 0 (sigmoid is increasing, sigmoid(0) = 1/2).  It stands
// for the small per-layer MLP predictors that DejaVu and PowerInfer train to
// decide which FFN neurons to compute (53ai.com "sparsity for LLM inference"
// page, sections 如何推理加速 and 自适应稀疏预测器).  h is kept in fp32; z is
// accumulated in fp32 from fp16 (or fp32) weights.
//
// Kernels:
//   k_hidden   H[t][j] = relu(At[j] . X[t])         one warp per row of At
//   k_logits   bit i of token t = (Bt[i] . H[t] + c_i > 0)   one CTA per 32 neurons
//   k_mask_from_idx   a caller-given index list as a bit mask
//   k_union    masks -> the union of a batch's sets with each row's token mask
//   k_compact  masks -> ascending index lists (per token, in caller numbering)
//              and the union of the tokens' sets with, per union row, the bit
//              set of tokens active on it (warp ballot + block prefix sum).
#include "async.cuh"
#include "common.cuh"
#include "launch.cuh"

namespace sfnn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename T, int TB>
__global__ void __launch_bounds__(kThreads) k_hidden(const T *__restrict__ At, const T *__restrict__ X,
                                                     float *__restrict__ H, int r, int d, int b) {
  constexpr int V = Elem<T>::kVec;
  constexpr int U = 4;
  const int lane = threadIdx.x & 31;
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int nch = d / V;
  for (int j = gwarp; j < r; j += nwarps) {
    const T *row = At + (size_t)j * d;
    for (int t0 = 0; t0 < b; t0 += TB) {
      float acc[TB];
#pragma unroll
      for (int t = 0; t < TB; ++t) acc[t] = 0.f;
      for (int c0 = lane; c0 < nch; c0 += 32 * U) {
        uint4 w[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (c0 + 32 * u < nch) w[u] = ld_stream(row + (size_t)(c0 + 32 * u) * V);
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + 32 * u;
          if (c < nch) {
            float wf[V];
            unpack<T>(w[u], wf);
#pragma unroll
            for (int t = 0; t < TB; ++t) {
              if (t0 + t < b) {
                float xf[V];
                unpack<T>(ld_keep(X + (size_t)(t0 + t) * d + (size_t)c * V), xf);
#pragma unroll
                for (int v = 0; v < V; ++v) acc[t] = fmaf(wf[v], xf[v], acc[t]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        if (t0 + t < b) {
          const float s = warp_sum(acc[t]);
          if (lane == 0) H[(size_t)(t0 + t) * r + j] = s > 0.f ? s : 0.f;  // NaN -> 0
        }
      }
    }
  }
}

// One CTA per mask word (32 neurons); warp w takes neurons 4w..4w+3 of the word.
template <typename T, int TB>
__global__ void __launch_bounds__(kThreads) k_logits(const T *__restrict__ Bt, const T *__restrict__ cvec,
                                                     const float *__restrict__ H, uint32_t *__restrict__ mask,
                                                     int n, int r, int b, int nwords) {
  constexpr int V = Elem<T>::kVec;
  extern __shared__ float hs[];  // [b][r]
  __shared__ uint32_t bits_s[TB];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < b * r; i += blockDim.x) hs[i] = H[i];
  const int nch = r / V;
  for (int word = blockIdx.x; word < nwords; word += gridDim.x) {
    for (int t0 = 0; t0 < b; t0 += TB) {
      if (threadIdx.x < TB) bits_s[threadIdx.x] = 0u;
      __syncthreads();
      for (int q = 0; q < 4; ++q) {
        const int i = warp * 4 + q;
        const int p = word * 32 + i;
        if (p >= n) break;  // warp-uniform
        const T *row = Bt + (size_t)p * r;
        float acc[TB];
#pragma unroll
        for (int t = 0; t < TB; ++t) acc[t] = 0.f;
#pragma unroll 4
        for (int c = lane; c < nch; c += 32) {
          float wf[V];
          unpack<T>(ld_stream(row + (size_t)c * V), wf);
#pragma unroll
          for (int t = 0; t < TB; ++t) {
            if (t0 + t < b) {
              // two 16-byte reads per chunk instead of V scalar ones (fewer bank conflicts)
              const float4 *hp4 = reinterpret_cast<const float4 *>(hs + (size_t)(t0 + t) * r + (size_t)c * V);
              float hv[V];
#pragma unroll
              for (int q = 0; q < V / 4; ++q) {
                const float4 f = hp4[q];
                hv[4 * q] = f.x;
                hv[4 * q + 1] = f.y;
                hv[4 * q + 2] = f.z;
                hv[4 * q + 3] = f.w;
              }
#pragma unroll
              for (int v = 0; v < V; ++v) acc[t] = fmaf(wf[v], hv[v], acc[t]);
            }
          }
        }
        const float cz = to_f<T>(cvec[p]);
#pragma unroll
        for (int t = 0; t < TB; ++t) {
          if (t0 + t < b) {
            const float z = warp_sum(acc[t]) + cz;
            if (lane == 0 && z > 0.f) atomicOr(&bits_s[t], 1u << i);  // NaN -> inactive
          }
        }
      }
      __syncthreads();
      if (threadIdx.x < TB && t0 + threadIdx.x < b)
        mask[(size_t)(t0 + threadIdx.x) * nwords + word] = bits_s[threadIdx.x];
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(1024) k_mask_from_idx(const int32_t *__restrict__ idx,
                                                        const int32_t *__restrict__ count,
                                                        const int32_t *__restrict__ iperm,
                                                        uint32_t *__restrict__ mask, int n, int nwords,
                                                        int32_t *err) {
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) mask[w] = 0u;
  __syncthreads();
  int k = *count;
  k = k < 0 ? 0 : (k > n ? n : k);
  for (int e = threadIdx.x; e < k; e += blockDim.x) {
    const int v = idx[e];
    if (v < 0 || v >= n) {
      latch_error(err, kErrInvalidIdx);
      continue;
    }
    const int p = iperm[v];
    atomicOr(&mask[p >> 5], 1u << (p & 31));
  }
}

// Exclusive prefix sum over the block; returns this thread's offset, *total the block sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int *total) {
  __shared__ int warp_tot[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int wt = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wt, o);
      if (lane >= o) wt += y;
    }
    if (lane < nw) warp_tot[lane] = wt;  // inclusive over warps
  }
  __syncthreads();
  const int before = warp == 0 ? 0 : warp_tot[warp - 1];
  *total = warp_tot[nw - 1];
  __syncthreads();
  return before + incl - v;
}

// The union of the b tokens' sets, ascending, with each union row's token mask (bit t:
// token t's set holds the row).  CTA k takes the 32 bit words [32k, 32k + 32), warp j word
// 32k + j: lane t loads token t's word while the CTA's threads count the union bits of all
// earlier words (each bit word's b token words OR-ed, then popc), so that no CTA waits on
// another and both are one round of loads.  A warp ORs its word's token words, takes its
// first union position from the counts (earlier words, then the CTA's earlier warps), and
// lane i, on row 32 (32k + j) + i, gathers bit i of every token's word by shuffles and
// writes the row if the union holds it.  The last CTA writes the union's size.
constexpr int kUnionThreads = 1024;

__global__ void __launch_bounds__(kUnionThreads) k_union(const uint32_t *__restrict__ mask, int nwords, int n, int b,
                                                         int32_t *__restrict__ ulist, uint32_t *__restrict__ utok,
                                                         int32_t *__restrict__ ucount) {
  __shared__ int red[32], wcnt[32];
  pdl_wait();  // the masks (the kernel before) are complete
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int w0 = blockIdx.x * 32, w = w0 + warp;
  const uint32_t full = 0xffffffffu;
  const uint32_t mine = w < nwords && lane < b ? __ldcg(mask + (size_t)lane * nwords + w) : 0u;
  int before = 0;  // union bits of the words before this CTA's
  for (int v = threadIdx.x; v < w0; v += blockDim.x) {
    uint32_t u = 0u;
#pragma unroll
    for (int t = 0; t < kMaxBatch; ++t) u |= t < b ? __ldcg(mask + (size_t)t * nwords + v) : 0u;
    before += __popc(u);  // v < w0 <= nwords - 1: never the tail word
  }
  uint32_t u = __reduce_or_sync(full, mine);
  if (w == nwords - 1 && (n & 31)) u &= (1u << (n & 31)) - 1u;  // bits of the last word below n
  before = __reduce_add_sync(full, before);
  if (lane == 0) {
    red[warp] = before;
    wcnt[warp] = __popc(u);
  }
  __syncthreads();
  const int base = __reduce_add_sync(full, red[lane]);  // 32 warps
  const int wc = wcnt[lane];
  const int first = base + __reduce_add_sync(full, lane < warp ? wc : 0);
  uint32_t tok = 0u;  // the tokens whose sets hold row 32 w + lane
  for (int t = 0; t < b; ++t) tok |= ((__shfl_sync(full, mine, t) >> lane) & 1u) << t;
  if ((u >> lane) & 1u) {
    const int pos = first + __popc(u & ((1u << lane) - 1u));
    ulist[pos] = w * 32 + lane;
    utok[pos] = tok;
  }
  if (blockIdx.x == gridDim.x - 1 && warp == 0) {
    const int total = base + __reduce_add_sync(full, wc);
    if (lane == 0) *ucount = total;
  }
}

// Block t: token t's set as indices in the caller's numbering, ascending in storage order.
__global__ void __launch_bounds__(1024) k_compact(const uint32_t *__restrict__ mask, int nwords, int n,
                                                  const int32_t *__restrict__ perm, int32_t *__restrict__ idx_out,
                                                  int32_t *__restrict__ cnt_out) {
  const int t = blockIdx.x;
  const int wpt = (nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * wpt;
  int cnt = 0;
  for (int k = 0; k < wpt; ++k) {
    const int w = w0 + k;
    if (w < nwords) cnt += __popc(mask[(size_t)t * nwords + w]);
  }
  int total;
  int pos = block_exclusive_scan(cnt, &total);
  for (int k = 0; k < wpt; ++k) {
    const int w = w0 + k;
    if (w >= nwords) break;
    uint32_t m = mask[(size_t)t * nwords + w];
    while (m) {
      const int i = __ffs(m) - 1;
      m &= m - 1u;
      if (idx_out) idx_out[(size_t)t * n + pos] = perm[w * 32 + i];
      ++pos;
    }
  }
  if (threadIdx.x == 0 && cnt_out) cnt_out[t] = total;
}

// Block c: tile c's part of a fused launch's set.  Its entries follow those of tiles
// 0..c-1 (counts clamped to each tile's size), so the list is in storage order.
__global__ void __launch_bounds__(256) k_tile_sets(const int32_t *__restrict__ list, int stride,
                                                   const int32_t *__restrict__ cnt, const int32_t *__restrict__ perm,
                                                   int n, int G, int32_t *__restrict__ idx_out,
                                                   int32_t *__restrict__ cnt_out) {
  const int c = blockIdx.x, tok = blockIdx.y;
  list += (size_t)tok * n * stride;
  cnt += (size_t)tok * G;
  if (idx_out) idx_out += (size_t)tok * n;
  if (cnt_out) cnt_out += tok;
  auto tile_count = [&](int t) {
    const int sz = decode1_tile_start(t + 1, n, G) - decode1_tile_start(t, n, G);
    return min(max(cnt[t], 0), sz);
  };
  int before = 0;
  for (int t = threadIdx.x; t < c; t += blockDim.x) before += tile_count(t);
  int total;
  block_exclusive_scan(before, &total);  // total = the entries of tiles 0..c-1
  const int own = tile_count(c);
  const int start = decode1_tile_start(c, n, G);
  if (idx_out)
    for (int k = threadIdx.x; k < own; k += blockDim.x) {
      const int pos = list[(size_t)(start + k) * stride];
      idx_out[total + k] = (unsigned)pos < (unsigned)n ? perm[pos] : -1;
    }
  if (cnt_out && c == G - 1 && threadIdx.x == 0) *cnt_out = total + own;
}

template <typename T>
cudaError_t hidden_impl(const sfnn_ctx *h, const void *X, int b, cudaStream_t s) {
  const Layout &L = h->L;
  const int grid = (L.r + kWarps - 1) / kWarps;
  const T *At = static_cast<const T *>(h->At);
  const T *Xp = static_cast<const T *>(X);
  if (b == 1)
    k_hidden<T, 1><<<grid, kThreads, 0, s>>>(At, Xp, h->h, L.r, L.d, b);
  else
    k_hidden<T, 8><<<grid, kThreads, 0, s>>>(At, Xp, h->h, L.r, L.d, b);
  return cudaGetLastError();
}

constexpr int kLogitsSmemMax = 32768 * sizeof(float);  // r * max_batch <= 32768 (checked at create)

template <typename T, int TB>
cudaError_t logits_tb(const sfnn_ctx *h, int b, cudaStream_t s) {
  const Layout &L = h->L;
  const size_t smem = (size_t)b * L.r * sizeof(float);
  auto kern = k_logits<T, TB>;
  kern<<<L.nwords, kThreads, smem, s>>>(static_cast<const T *>(h->Bt), static_cast<const T *>(h->cvec), h->h,
                                        h->mask, L.n, L.r, b, L.nwords);
  return cudaGetLastError();
}

template <typename T>
cudaError_t logits_impl(const sfnn_ctx *h, int b, cudaStream_t s) {
  if (b == 1) return logits_tb<T, 1>(h, b, s);
  if (b <= 8) return logits_tb<T, 8>(h, b, s);
  return logits_tb<T, 32>(h, b, s);
}

}  // namespace

cudaError_t configure_predict() {
  const void *ks[] = {(const void *)k_logits<float, 1>, (const void *)k_logits<float, 8>,
                      (const void *)k_logits<float, 32>, (const void *)k_logits<__half, 1>,
                      (const void *)k_logits<__half, 8>, (const void *)k_logits<__half, 32>};
  for (const void *k : ks) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kLogitsSmemMax);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_hidden(const sfnn_ctx *h, const void *X, int b, cudaStream_t s) {
  return h->L.dt == SFNN_F16 ? hidden_impl<__half>(h, X, b, s) : hidden_impl<float>(h, X, b, s);
}

cudaError_t launch_logits(const sfnn_ctx *h, int b, cudaStream_t s) {
  return h->L.dt == SFNN_F16 ? logits_impl<__half>(h, b, s) : logits_impl<float>(h, b, s);
}

cudaError_t launch_mask_from_idx(const sfnn_ctx *h, const int32_t *idx, const int32_t *count, cudaStream_t s) {
  k_mask_from_idx<<<1, 1024, 0, s>>>(idx, count, h->iperm, h->mask, h->L.n, h->L.nwords, h->err);
  return cudaGetLastError();
}

cudaError_t launch_compact(const sfnn_ctx *h, int b, bool want_union, int32_t *idx_out, int32_t *cnt_out,
                           cudaStream_t s) {
  const Layout &L = h->L;
  cudaError_t e = cudaSuccess;
  if (want_union) {
    e = launch_pdl(k_union, dim3((L.nwords + 31) / 32), dim3(kUnionThreads), 0, s, (const uint32_t *)h->mask,
                   L.nwords, L.n, b, h->ulist, h->utok, h->ucount);
  }
  if (e == cudaSuccess && (idx_out || cnt_out)) {
    k_compact<<<b, 1024, 0, s>>>(h->mask, L.nwords, L.n, h->perm, idx_out, cnt_out);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_tile_sets(const int32_t *list, int stride, const int32_t *cnt, const int32_t *perm, int n, int G,
                             int32_t *idx_out, int32_t *cnt_out, cudaStream_t s, int ntok) {
  if (!idx_out && !cnt_out) return cudaSuccess;
  k_tile_sets<<<dim3(G, ntok), 256, 0, s>>>(list, stride, cnt, perm, n, G, idx_out, cnt_out);
  return cudaGetLastError();
}

}  // namespace sfnn
