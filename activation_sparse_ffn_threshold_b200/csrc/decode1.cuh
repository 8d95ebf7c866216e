// decode1.cuh -- parameters and shared-memory plan of the fused single-token decode kernel.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sfnn.h"

namespace sfnn {

constexpr int kDecode1Threads = 512;  // 16 warps per CTA, one CTA per SM
constexpr int kDecode1BStages = 4;     // B^T rows staged per warp (thread-private shared staging)
constexpr int kDecodeSmemCap = 227 * 1024;  // opt-in dynamic shared memory of one CTA

// W_down rows in flight per thread in the down phase, by 16-byte chunks per thread and row
__host__ __device__ constexpr int decode1_dstages(int maxm) { return maxm == 1 ? 8 : (maxm == 2 ? 4 : 2); }
// The single-token kernel's down phase has the whole staging region (128 KB of rows): its
// up/gate phase reads into registers.
__host__ __device__ constexpr int decode1_c2stages(int maxm) { return maxm == 1 ? 16 : (maxm == 2 ? 8 : 4); }
// 16-byte chunks of a d-vector per thread (1, 2 or 4)
__host__ __device__ inline int decode1_maxm(int nch_d) {
  return nch_d <= kDecode1Threads ? 1 : (nch_d <= 2 * kDecode1Threads ? 2 : 4);
}

struct Decode1Params {
  const void *At, *Bt, *cvec, *bias, *rows;  // re-laid-out weights
  const void *x;                             // [d] input (wdtype)
  float *y;                                  // [d] output
  const float *resid;                        // [d] or null: y = resid + FFN(x)
  void *xnext;                               // [d] or null: round(y) in wdtype
  float *hbuf;                               // [2][r] predictor hidden layer (halves; scratch)
  float *part;                               // [G][d] per-CTA partial sums (scratch)
  uint64_t *bar;                             // grid barrier arrival counter (scratch, zeroed at create)
  int32_t *err;                              // latched device error
  int d, n, r, nproj, act, dt;
  int G;         // CTAs (one per SM) = tiles of neurons
  int tile_max;  // largest tile
  int nseg;      // 4 KB segments of one projection row (C1 work items per row and projection)
  int rq;        // rows are 8- or 4-bit codes (0: dt); rscale [n][nproj] their fp32 scales
  const float *rscale;
  int quota;         // rebalancing of the active rows: own rows kept per CTA, the rest shared out
                     //   evenly after a split grid barrier (0: every CTA takes its own tile's rows)
  int2 *blist;       // [n] each tile's active (storage position, bias) pairs, at start(c)
  int32_t *bcnt;     // [G] their counts
  int hot;           // multi-token kernel: ranks of the hot prefix whose gate/up rows are read before
                     //   the sets are known (0: none); rank k is position k / G of tile k % G
  int32_t *set_pos;  // null, or [n]: tile c's active storage positions at [start(c), start(c) + cnt)
  int32_t *set_cnt;  //   and [G] their counts -- the set this launch used, for callers that ask
  // The single-token kernel's request depths: more bytes in flight than keep HBM busy only
  // queue, and delay the reads on the critical path (barrier polls, the hidden layer).
  int bstages;   // B^T rows staged per warp (1, 2, 3, 4, 6 or 8)
  int c2pre;     // W_down rows requested during C1 (0 .. the C2 stage count)
  int c1depth;   // up/gate segments in flight per warp (1 or 2)
  int c2stages;  // W_down rows in flight in C2 (1, 2, 4, 8 or 16; at most decode1_c2stages)
};

struct Decode1Layout {
  size_t x, h, bias, c, act, a, dots, red2, bits, wpref, bars, bstage, dstage, total;
};

__host__ __device__ inline size_t decode1_align(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Bytes of the staging region: B^T rows (phase B) and W_down chunks (C2) share it; the
// single-token kernel (`single`) stages more W_down rows than the others.
__host__ __device__ inline size_t decode1_stage_bytes(const Decode1Params &P, bool single = false) {
  const int vec = P.dt == SFNN_F16 ? 8 : 4;
  const int maxm = decode1_maxm(P.d / vec);
  const size_t bsz = (size_t)(kDecode1Threads / 32) * (single ? P.bstages : kDecode1BStages) * (P.r / vec) * 16;
  const size_t dsz = (size_t)(single ? decode1_c2stages(maxm) : decode1_dstages(maxm)) * maxm * kDecode1Threads * 16;
  return bsz > dsz ? bsz : dsz;
}

__host__ __device__ inline Decode1Layout decode1_layout(const Decode1Params &P, bool single = false) {
  const size_t esz = P.dt == SFNN_F16 ? 2 : 4;
  const size_t tm = (size_t)P.tile_max;
  Decode1Layout L;
  size_t o = 0;
  L.x = o;
  o = decode1_align(o + (size_t)P.d * esz, 16);
  L.h = o;  // the hidden layer, read once per CTA
  o = decode1_align(o + (size_t)P.r * 4, 16);
  L.bias = o;
  o = decode1_align(o + tm * 4, 16);
  L.c = o;
  o = decode1_align(o + tm * 4, 16);
  L.act = o;  // active positions of the tile, ascending
  o = decode1_align(o + tm * 4, 16);
  L.a = o;  // their activations
  o = decode1_align(o + tm * 4, 16);
  L.dots = o;  // segment partials of the up (and gate) dot products
  o = decode1_align(o + tm * 2 * (size_t)P.nseg * 4, 16);
  L.red2 = o;
  o = decode1_align(o + (size_t)kDecode1Threads * 4, 16);
  L.bits = o;
  o = decode1_align(o + ((tm + 31) / 32) * 4 + 16, 16);
  L.wpref = o;  // exclusive prefix of the bit words' population counts
  o = decode1_align(o + ((tm + 31) / 32 + 1) * 4, 16);
  L.bars = o;  // the active count, a flag, the split barrier's target, C1's item counter and row count
  o = decode1_align(o + 32, 16);
  // The two staging areas share one region: B^T rows are staged only in phase B, the
  // W_down chunks only after it (the CTA synchronises in between).
  L.bstage = o;  // [warp][stage][chunk of the row]: B^T rows staged per warp
  L.dstage = o;  // [stage][chunk m][thread]: W_down chunks staged per thread
  o = decode1_align(o + decode1_stage_bytes(P, single), 16);
  L.total = o;
  return L;
}

// First neuron position of tile c when n neurons are split into G contiguous tiles.
__host__ __device__ inline int decode1_tile_start(int c, int n, int G) {
  const int q = n / G, rr = n % G;
  return c * q + (c < rr ? c : rr);
}

// The look-ahead stack kernel (decode_ahead.cu): layer l's FFN on the set predicted by
// the previous launch, beside layer l+1's predictor on the same input.
struct AheadParams {
  const void *At, *Bt, *cvec, *bias;  // the next layer's predictor and gated bias (At null: none)
  float *hbuf;                        // [r] its hidden layer (scratch)
  int r, n, tile_max;                 // its sizes; it has the same G tiles as this layer
  const int2 *list_in;                // this layer's active lists: tile c's from position
  const int32_t *cnt_in;              //   start(c), (storage position, bias) pairs; [G] counts
                                      //   (list_in null: no FFN in this launch)
  int2 *list_out;                     // the next layer's lists, written for the next launch
  int32_t *cnt_out;
};

// The shared-memory plan of one look-ahead launch: the single-layer plan sized for this
// layer's d and C1 segments, the next layer's r, and the larger of the two tiles.
__host__ __device__ inline Decode1Layout decode_ahead_layout(const Decode1Params &P, const AheadParams &Q) {
  Decode1Params M = P;
  M.r = Q.At ? Q.r : (P.dt == SFNN_F16 ? 8 : 4);
  M.tile_max = P.tile_max > Q.tile_max ? P.tile_max : Q.tile_max;
  return decode1_layout(M);
}

// The multi-token fused kernel (decode_multi.cu): NB = 2..4 tokens per launch on the
// single-token kernel's tile plan.  Its shared memory: the NB inputs, their hidden
// layers, the tile's per-token decisions and the union's activations, and a staging
// region for half rows of B^T (phase B, per warp) or W_down chunks (per thread).
constexpr int kMultiMaxTokens = 4;
constexpr int kMultiBStages = 6;  // B^T half rows staged per warp

struct MultiLayout {
  size_t x, h, bias, c, act, tok, a, zpart, dots, pdots, red2, tbits, ubits, wpref, bars, stage, total;
};

// Rows of tile c in the hot prefix of `hot` ranks (ranks are dealt round-robin to G tiles).
__host__ __device__ inline int decode1_hot_rows(int hot, int c, int G) { return hot > c ? (hot - c + G - 1) / G : 0; }

__host__ __device__ inline MultiLayout decode_multi_layout(const Decode1Params &P, int nb) {
  const size_t tm = (size_t)P.tile_max;
  const size_t words = (tm + 31) / 32;
  const int vec = 8;  // fp16 only
  MultiLayout L;
  size_t o = 0;
  L.x = o;
  o = decode1_align(o + (size_t)nb * P.d * 2, 16);
  L.h = o;
  o = decode1_align(o + (size_t)nb * P.r * 4, 16);
  L.bias = o;
  o = decode1_align(o + tm * 4, 16);
  L.c = o;
  o = decode1_align(o + tm * 4, 16);
  L.act = o;  // the tile's union positions, ascending
  o = decode1_align(o + tm * 4, 16);
  L.tok = o;  // and the tokens active on each (bit t)
  o = decode1_align(o + tm * 4, 16);
  L.a = o;  // the tile's b, then the union rows' activations [k][t]
  o = decode1_align(o + tm * nb * 4, 16);
  L.zpart = o;  // the two halves of each logit [half][p][t]
  o = decode1_align(o + 2 * tm * nb * 4, 16);
  L.dots = o;  // C1 segment sums [k][proj][seg][t]
  o = decode1_align(o + tm * 2 * (size_t)P.nseg * nb * 4, 16);
  L.pdots = o;  // the same for the tile's hot prefix, by tile position
  o = decode1_align(o + (size_t)decode1_hot_rows(P.hot, 0, P.G) * 2 * (size_t)P.nseg * nb * 4, 16);
  L.red2 = o;
  o = decode1_align(o + (size_t)kDecode1Threads * 4, 16);
  L.tbits = o;  // [t][word]
  o = decode1_align(o + (size_t)nb * words * 4 + 16, 16);
  L.ubits = o;
  o = decode1_align(o + words * 4 + 16, 16);
  L.wpref = o;
  o = decode1_align(o + (words + 1) * 4, 16);
  L.bars = o;  // the union count, a flag, the split barrier's target, C1's item counter and row count
  o = decode1_align(o + 32, 16);
  L.stage = o;
  const int maxm = decode1_maxm(P.d / vec);
  const size_t bsz = (size_t)(kDecode1Threads / 32) * P.bstages * 64 * 16;  // 2 chunks per lane and stage
  const size_t dsz = (size_t)decode1_dstages(maxm) * maxm * kDecode1Threads * 16;
  o = decode1_align(o + (bsz > dsz ? bsz : dsz), 16);
  L.total = o;
  return L;
}

// Launch attributes of the persistent fused kernels: cooperative (the runtime then
// guarantees that all of a launch's CTAs are resident at once, which its grid barriers
// rely on) and, when asked, programmatic dependent launch.  Returns the count.
inline unsigned fused_launch_attrs(cudaLaunchAttribute (&attr)[2], bool pdl) {
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  return pdl ? 2u : 1u;
}

cudaError_t configure_decode_multi();
cudaError_t launch_decode_multi(const Decode1Params &P, int nb, cudaStream_t stream, bool pdl);
int decode_multi_blocks_per_sm(const Decode1Params &P, int nb);

cudaError_t configure_decode1();
cudaError_t configure_decode_ahead();
cudaError_t launch_decode_ahead(const Decode1Params &P, const AheadParams &Q, cudaStream_t stream, bool pdl);
int decode1_blocks_per_sm(const Decode1Params &P);  // co-resident CTAs per SM for this plan
cudaError_t launch_decode1(const Decode1Params &P, cudaStream_t stream, bool pdl);
cudaError_t launch_barrier_bump(uint64_t *count, cudaStream_t stream);

}  // namespace sfnn
