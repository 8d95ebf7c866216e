// noalloc.cu -- sfnn_predict_noalloc: the predictor for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc: code that runs while a CUDA graph is being
// captured into (an allocation there would break or be recorded into the capture),
// runtimes whose device memory is fully owned by their own pool allocator, and
// embedded users that forbid allocation after start-up.  sfnn_create allocates the
// handle's re-laid-out weights and scratch, so those callers cannot use it.  This entry
// point needs no handle: it reads the caller's weights in PyTorch layout and keeps its
// scratch (the hidden layer h and the decision bit mask) in one file-scope device array
// of kNoAllocScratchBytes, which every GPU that loads the library holds until exit.
//
// All calls share that array and it keeps the last call's contents; every word a call
// reads is first written by the same call, so nothing needs clearing.  Calls that
// overlap on the GPU (different streams, or different host threads) race on it.
#include <mutex>

#include "common.cuh"
#include "launch.cuh"

namespace {

constexpr int kNoAllocScratchBytes = SFNN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kCols = 32;    // output columns per CTA (one mask word of decisions)
constexpr int kWarps = 8;    // warps per CTA, splitting the reduction dimension

// out[j] = sum_k v[k] * M[k][j] for j in this CTA's 32 columns (M row-major [K x J]):
// lane = column, warps split k, partial sums added in a fixed warp order.
template <typename T, typename VT>
__device__ __forceinline__ float colsum(const T *__restrict__ M, const VT *__restrict__ v, int K, int J, int j,
                                        float *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k0 = (int)(((int64_t)warp * K) / kWarps), k1 = (int)(((int64_t)(warp + 1) * K) / kWarps);
  float acc = 0.f;
  if (j < J) {
#pragma unroll 4
    for (int k = k0; k < k1; ++k) acc = fmaf(sfnn::to_f<T>(M[(size_t)k * J + j]), sfnn::to_f<VT>(v[k]), acc);
  }
  red[warp * kCols + lane] = acc;
  __syncthreads();
  float s = 0.f;
  if (warp == 0) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w * kCols + lane];
  }
  return s;  // valid in warp 0
}

// h = relu(x . A), A [d x r]
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) k_na_hidden(const T *__restrict__ x, const T *__restrict__ A, int d,
                                                          int r, float *__restrict__ h) {
  __shared__ float red[kWarps * kCols];
  const int j = blockIdx.x * kCols + (threadIdx.x & 31);
  const float s = colsum<T, T>(A, x, d, r, j, red);
  if (threadIdx.x < 32 && j < r) h[j] = s > 0.f ? s : 0.f;  // NaN -> 0
}

// bit i of the mask = (h . B[:, i] + c_i > 0), B [r x n]; one CTA per mask word
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) k_na_logits(const float *__restrict__ h, const T *__restrict__ B,
                                                          const T *__restrict__ c, int r, int n,
                                                          uint32_t *__restrict__ mask) {
  __shared__ float red[kWarps * kCols];
  const int i = blockIdx.x * kCols + (threadIdx.x & 31);
  const float s = colsum<T, float>(B, h, r, n, i, red);
  if (threadIdx.x < 32) {
    const bool on = i < n && s + sfnn::to_f<T>(c[i]) > 0.f;  // NaN -> inactive
    const uint32_t word = __ballot_sync(0xffffffffu, on);
    if (threadIdx.x == 0) mask[blockIdx.x] = word;
  }
}

// ascending index list of the set bits, and their count (one CTA)
__global__ void __launch_bounds__(1024) k_na_compact(const uint32_t *__restrict__ mask, int nwords,
                                                     int32_t *__restrict__ idx, int32_t *__restrict__ count) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int w0 = 0; w0 < nwords; w0 += blockDim.x) {
    const int w = w0 + threadIdx.x;
    const uint32_t word = w < nwords ? mask[w] : 0u;
    const int k = __popc(word);
    int incl = k;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x / 32;
      int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      if (lane < nw) warp_tot[lane] = t;
    }
    __syncthreads();
    int pos = carry + (warp ? warp_tot[warp - 1] : 0) + incl - k;
    uint32_t m = word;
    while (m) {
      idx[pos++] = w * 32 + __ffs(m) - 1;
      m &= m - 1u;
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_tot[blockDim.x / 32 - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) *count = carry;
}

// Device address of the scratch array, looked up once per device (with that device
// current).  Host code must not use the array's name as an address.
constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

cudaError_t scratch_for_current_device(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

template <typename T>
cudaError_t run(const void *x, const void *pa, const void *pb, const void *pc, int d, int r, int n, int32_t *idx,
                int32_t *count, cudaStream_t s, unsigned char *scratch) {
  float *h = reinterpret_cast<float *>(scratch);
  const size_t hbytes = ((size_t)r * 4 + 255) / 256 * 256;
  uint32_t *mask = reinterpret_cast<uint32_t *>(scratch + hbytes);
  const int nwords = (n + 31) / 32;
  k_na_hidden<T><<<(r + kCols - 1) / kCols, kWarps * 32, 0, s>>>(static_cast<const T *>(x), static_cast<const T *>(pa),
                                                                  d, r, h);
  k_na_logits<T><<<nwords, kWarps * 32, 0, s>>>(h, static_cast<const T *>(pb), static_cast<const T *>(pc), r, n,
                                                 mask);
  k_na_compact<<<1, 1024, 0, s>>>(mask, nwords, idx, count);
  return cudaGetLastError();
}

}  // namespace

extern "C" sfnn_status sfnn_predict_noalloc(const void *x, const void *pa, const void *pb, const void *pc, int32_t d,
                                            int32_t r, int32_t n, int32_t wdtype, int32_t *idx, int32_t *count,
                                            sfnn_stream_t stream) {
  if (!x || !pa || !pb || !pc || !idx || !count || d < 1 || r < 1 || n < 1) return SFNN_ERR_INVALID_ARG;
  if (wdtype != SFNN_F32 && wdtype != SFNN_F16) return SFNN_ERR_INVALID_ARG;
  const size_t need = ((size_t)r * 4 + 255) / 256 * 256 + (size_t)((n + 31) / 32) * 4;
  if (need > (size_t)kNoAllocScratchBytes) return SFNN_ERR_UNSUPPORTED;  // r and n beyond the fixed scratch
  void *scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return SFNN_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  e = wdtype == SFNN_F16 ? run<__half>(x, pa, pb, pc, d, r, n, idx, count, s, static_cast<unsigned char *>(scratch))
                         : run<float>(x, pa, pb, pc, d, r, n, idx, count, s, static_cast<unsigned char *>(scratch));
  return e == cudaSuccess ? SFNN_OK : SFNN_ERR_CUDA;
}
