// launch.cuh -- host-side launchers of the kernels (defined in the .cu files) and the
// size limits the host checks when a layer is created.
#pragma once

#include "common.cuh"
#include "context.cuh"

namespace sfnn {

constexpr int kMaxNeurons = 1 << 20;  // n at most

// Launch with programmatic stream serialization: the kernel may start while the one before
// it in the stream finishes (it reads nothing that kernel writes before griddepcontrol.wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

cudaError_t configure_predict();  // one-time kernel attributes (shared-memory limits)
cudaError_t configure_ffn();
cudaError_t launch_layout(sfnn_ctx *h, const sfnn_layer_desc *desc, cudaStream_t s);
cudaError_t launch_hidden(const sfnn_ctx *h, const void *X, int b, cudaStream_t s);
cudaError_t launch_logits(const sfnn_ctx *h, int b, cudaStream_t s);
cudaError_t launch_mask_from_idx(const sfnn_ctx *h, const int32_t *idx, const int32_t *count, cudaStream_t s);
// want_union: the batch's union list (k_union); idx_out/cnt_out: per-token lists (k_compact)
cudaError_t launch_compact(const sfnn_ctx *h, int b, bool want_union, int32_t *idx_out, int32_t *cnt_out,
                           cudaStream_t s);
cudaError_t launch_up(const sfnn_ctx *h, const void *X, int b, cudaStream_t s);
cudaError_t launch_down(const sfnn_ctx *h, int b, int *splits, cudaStream_t s);
cudaError_t launch_reduce(const sfnn_ctx *h, int b, int splits, const float *resid, float *Y, void *xnext,
                          cudaStream_t s);
// The per-tile lists of a fused launch -> one index list in caller numbering (tile order)
// and its length, for each of `ntok` tokens.  Token t's tile c holds cnt[t * G + c]
// storage positions, every `stride`-th int32 of `list` from position t * n + start(c)
// on (stride 1: plain positions; 2: the look-ahead kernel's (position, bias) pairs).
// Token t's list goes to idx_out + t * n, its length to cnt_out[t]; either may be null.
cudaError_t launch_tile_sets(const int32_t *list, int stride, const int32_t *cnt, const int32_t *perm, int n, int G,
                             int32_t *idx_out, int32_t *cnt_out, cudaStream_t s, int ntok = 1);
cudaError_t launch_round(const float *X, void *out, int dt, int64_t count, cudaStream_t s);

// Tensor-core (tcgen05) batch path: fp16 weights, d a multiple of 128.
bool tc_batch_supported(const sfnn_ctx *h);
bool tc_predict_supported(const sfnn_ctx *h);  // and r a multiple of 64
cudaError_t launch_tc_predict(const sfnn_ctx *h, const void *X, int b, cudaStream_t s);
int tc_hstride(int n);
size_t tc_up_partial_bytes(int num_sms, int max_batch);
cudaError_t configure_tc_batch();
cudaError_t launch_tc_batch(const sfnn_ctx *h, const void *X, int b, int *splits_out, cudaStream_t s);

}  // namespace sfnn
