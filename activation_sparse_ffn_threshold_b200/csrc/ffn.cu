// ffn.cu -- the FFN over the predicted neurons only (multi-kernel path).
//
// Only rows of predicted-active neurons are read; an inactive neuron's row of
// the down projection would add an exact zero (53ai.com "sparsity for LLM
// inference" page, section 激活稀疏).  Rows of the union of a batch's sets are
// read once and applied to every token active on them, since the benefit of
// sparsity shrinks as a batch's sets accumulate (same page, section 工程效果).
//
//   k_up      a[u][t] = act(row_u . x_t) for union row u and the tokens active
//             on it (0 for the others); one warp per union row.
//   k_down    split-K gather-axpy over the neuron-major down rows: CTA (ds, ks)
//             owns a 32*V-column slice of y and the ks-th chunk of the union
//             list; its 8 warps take interleaved rows and are summed in a
//             fixed order through shared memory -> part[ks][t][cols].
//   k_reduce  y = sum over ks of part[ks] in ascending ks (+ residual).
// Every sum runs in a fixed order, so results are bitwise reproducible.
#include "async.cuh"
#include "common.cuh"
#include "launch.cuh"

namespace sfnn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename T, int ACT, int TB>
__global__ void __launch_bounds__(kThreads)
    k_up(const T *__restrict__ rows, const T *__restrict__ bias, const T *__restrict__ X,
         const int32_t *__restrict__ ulist, const uint32_t *__restrict__ utok, const int32_t *__restrict__ ucount,
         float *__restrict__ acoef, int d, int b, int nproj) {
  constexpr int V = Elem<T>::kVec;
  const int lane = threadIdx.x & 31;
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int U = *ucount;
  const int nch = d / V;
  for (int u = gwarp; u < U; u += nwarps) {
    const int p = ulist[u];
    const uint32_t tm = utok[u];
    const T *gate_row = rows + (size_t)p * nproj * d;
    const T *up_row = gate_row + (ACT == SFNN_REGLU ? d : 0);
    const float bval = to_f<T>(bias[p]);
    for (int t0 = 0; t0 < b; t0 += TB) {
      float au[TB], ag[TB];
#pragma unroll
      for (int t = 0; t < TB; ++t) au[t] = ag[t] = 0.f;
#pragma unroll 4
      for (int c = lane; c < nch; c += 32) {
        float wu[V], wg[V];
        unpack<T>(ld_stream(up_row + (size_t)c * V), wu);
        if (ACT == SFNN_REGLU) unpack<T>(ld_stream(gate_row + (size_t)c * V), wg);
#pragma unroll
        for (int t = 0; t < TB; ++t) {
          if (t0 + t < b && ((tm >> (t0 + t)) & 1u)) {
            float xf[V];
            unpack<T>(ld_keep(X + (size_t)(t0 + t) * d + (size_t)c * V), xf);
#pragma unroll
            for (int v = 0; v < V; ++v) {
              au[t] = fmaf(wu[v], xf[v], au[t]);
              if (ACT == SFNN_REGLU) ag[t] = fmaf(wg[v], xf[v], ag[t]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        if (t0 + t < b) {
          const float su = warp_sum(au[t]);
          float a;
          if (ACT == SFNN_RELU) {
            const float g = su + bval;
            a = g > 0.f ? g : 0.f;
          } else {
            const float g = warp_sum(ag[t]) + bval;
            a = (g > 0.f ? g : 0.f) * su;
          }
          if (!((tm >> (t0 + t)) & 1u)) a = 0.f;
          if (lane == 0) acoef[(size_t)u * b + t0 + t] = a;
        }
      }
    }
  }
}

template <typename T, int TB>
__global__ void __launch_bounds__(kThreads)
    k_down(const T *__restrict__ rows, const float *__restrict__ acoef, const int32_t *__restrict__ ulist,
           const int32_t *__restrict__ ucount, float *__restrict__ part, int d, int b, int nproj, int splits) {
  constexpr int V = Elem<T>::kVec;
  constexpr int SW = 32 * V;  // columns per CTA slice
  extern __shared__ float red[];  // [kWarps][TB][SW]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ds = blockIdx.x, ks = blockIdx.y;
  const int U = *ucount;
  const int lo = (int)(((int64_t)ks * U) / splits);
  const int hi = (int)(((int64_t)(ks + 1) * U) / splits);
  const int col = ds * SW + lane * V;
  const bool col_ok = col < d;
  for (int t0 = 0; t0 < b; t0 += TB) {
    float acc[TB][V];
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
      for (int v = 0; v < V; ++v) acc[t][v] = 0.f;
#pragma unroll 4
    for (int u = lo + warp; u < hi; u += kWarps) {
      const int p = ulist[u];
      if (col_ok) {
        float w[V];
        unpack<T>(ld_stream(rows + ((size_t)p * nproj + nproj - 1) * d + col), w);
#pragma unroll
        for (int t = 0; t < TB; ++t) {
          if (t0 + t < b) {
            const float a = acoef[(size_t)u * b + t0 + t];
#pragma unroll
            for (int v = 0; v < V; ++v) acc[t][v] = fmaf(a, w[v], acc[t][v]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
      for (int v = 0; v < V; ++v) red[((size_t)warp * TB + t) * SW + lane * V + v] = acc[t][v];
    __syncthreads();
    for (int e = threadIdx.x; e < TB * SW; e += blockDim.x) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += red[(size_t)w * TB * SW + e];
      const int t = e / SW, cc = ds * SW + (e % SW);
      if (t0 + t < b && cc < d) part[((size_t)ks * b + t0 + t) * d + cc] = s;
    }
    __syncthreads();
  }
}

template <typename OUT>
__global__ void k_reduce(const float *__restrict__ part, int splits, int64_t bd, const float *resid, float *Y,
                         OUT *__restrict__ xnext) {
  pdl_wait();  // the partials (the kernel before) are complete
  pdl_launch_dependents();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= bd) return;
  float s = 0.f;
  for (int k = 0; k < splits; ++k) s += part[(size_t)k * bd + i];
  if (resid) s = resid[i] + s;
  Y[i] = s;
  if (xnext) xnext[i] = from_f<OUT>(s);
}

template <typename OUT>
__global__ void k_round(const float *__restrict__ X, OUT *__restrict__ out, int64_t count) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < count) out[i] = from_f<OUT>(X[i]);
}

template <typename T, int ACT>
cudaError_t up_act(const sfnn_ctx *h, const void *X, int b, cudaStream_t s) {
  const Layout &L = h->L;
  const int grid = h->num_sms * 4;
  const T *rows = static_cast<const T *>(h->rows);
  const T *bias = static_cast<const T *>(h->bias);
  const T *Xp = static_cast<const T *>(X);
  if (b == 1)
    k_up<T, ACT, 1><<<grid, kThreads, 0, s>>>(rows, bias, Xp, h->ulist, h->utok, h->ucount, h->acoef, L.d, b,
                                               L.nproj);
  else
    k_up<T, ACT, 8><<<grid, kThreads, 0, s>>>(rows, bias, Xp, h->ulist, h->utok, h->ucount, h->acoef, L.d, b,
                                               L.nproj);
  return cudaGetLastError();
}

template <typename T>
cudaError_t up_impl(const sfnn_ctx *h, const void *X, int b, cudaStream_t s) {
  return h->L.act == SFNN_REGLU ? up_act<T, SFNN_REGLU>(h, X, b, s) : up_act<T, SFNN_RELU>(h, X, b, s);
}

template <typename T, int TB>
cudaError_t down_tb(const sfnn_ctx *h, int b, int *splits_out, cudaStream_t s) {
  const Layout &L = h->L;
  constexpr int SW = 32 * Elem<T>::kVec;
  const int ds = (L.d + SW - 1) / SW;
  int splits = (2 * h->num_sms + ds - 1) / ds;
  splits = splits < 1 ? 1 : (splits > kMaxSplits ? kMaxSplits : splits);
  const size_t smem = (size_t)kWarps * TB * SW * sizeof(float);
  auto kern = k_down<T, TB>;
  kern<<<dim3(ds, splits), kThreads, smem, s>>>(static_cast<const T *>(h->rows), h->acoef, h->ulist, h->ucount,
                                                h->part, L.d, b, L.nproj, splits);
  *splits_out = splits;
  return cudaGetLastError();
}

template <typename T>
cudaError_t down_impl(const sfnn_ctx *h, int b, int *splits, cudaStream_t s) {
  return b == 1 ? down_tb<T, 1>(h, b, splits, s) : down_tb<T, 8>(h, b, splits, s);
}

template <typename T, int TB>
cudaError_t configure_down() {
  constexpr int SW = 32 * Elem<T>::kVec;
  return cudaFuncSetAttribute((const void *)k_down<T, TB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(kWarps * TB * SW * sizeof(float)));
}

}  // namespace

cudaError_t configure_ffn() {
  cudaError_t e = configure_down<float, 1>();
  if (e == cudaSuccess) e = configure_down<float, 8>();
  if (e == cudaSuccess) e = configure_down<__half, 1>();
  if (e == cudaSuccess) e = configure_down<__half, 8>();
  return e;
}

cudaError_t launch_up(const sfnn_ctx *h, const void *X, int b, cudaStream_t s) {
  return h->L.dt == SFNN_F16 ? up_impl<__half>(h, X, b, s) : up_impl<float>(h, X, b, s);
}

cudaError_t launch_down(const sfnn_ctx *h, int b, int *splits, cudaStream_t s) {
  return h->L.dt == SFNN_F16 ? down_impl<__half>(h, b, splits, s) : down_impl<float>(h, b, splits, s);
}

cudaError_t launch_reduce(const sfnn_ctx *h, int b, int splits, const float *resid, float *Y, void *xnext,
                          cudaStream_t s) {
  const int64_t bd = (int64_t)b * h->L.d;
  const int grid = (int)((bd + 255) / 256);
  if (h->L.dt == SFNN_F16)
    return launch_pdl(k_reduce<__half>, dim3(grid), dim3(256), 0, s, (const float *)h->part, splits, bd, resid, Y,
                      static_cast<__half *>(xnext));
  return launch_pdl(k_reduce<float>, dim3(grid), dim3(256), 0, s, (const float *)h->part, splits, bd, resid, Y,
                    static_cast<float *>(xnext));
}

cudaError_t launch_round(const float *X, void *out, int dt, int64_t count, cudaStream_t s) {
  const int grid = (int)((count + 255) / 256);
  if (dt == SFNN_F16)
    k_round<__half><<<grid, 256, 0, s>>>(X, static_cast<__half *>(out), count);
  else
    k_round<float><<<grid, 256, 0, s>>>(X, static_cast<float *>(out), count);
  return cudaGetLastError();
}

}  // namespace sfnn
