// context.cuh -- the host-side state of one sfnn handle (not part of the C ABI); the device
// kernels do not include it.
#pragma once

#include "common.cuh"

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
  float *upart;      // tensor-core up projection: fp32 partials of tiles split between CTAs
  int32_t *tcnt;     // [n / 128 rounded up] its per-tile arrival counters (zero between launches)
  int tc_up_ctas_per_sm;  // its grid: CTAs per SM (1 or 2; at most as many as fit)
  int tc_up_kps;          // and the 64-wide K chunks of every row it stages per step (1 or 2)
  int tc_down_mps;        // the down projection's 128-column output tiles per CTA (1 or 2)
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
