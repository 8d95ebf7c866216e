// decode1.cuh -- parameters and shared-memory plan of the fused single-token decode kernel.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "sfnn.h"

namespace sfnn {

constexpr int kDecode1SmemMax = 227 * 1024;  // opt-in dynamic shared memory per CTA on sm_100

struct Decode1Params {
  const void *At, *Bt, *cvec, *bias, *rows;  // re-laid-out weights
  const void *x;                             // [d] input (wdtype)
  float *y;                                  // [d] output
  const float *resid;                        // [d] or null: y = resid + FFN(x)
  void *xnext;                               // [d] or null: round(y) in wdtype
  float *hbuf;                               // [r] predictor hidden layer (scratch)
  float *part;                               // [G][d] per-CTA partial sums (scratch)
  uint32_t *bar;                             // [2] grid barrier state (scratch, zeroed at create)
  int32_t *err;                              // latched device error
  int d, n, r, nproj, act, dt;
  int G;           // CTAs (one per SM) = tiles of neurons
  int S, SB, NPC;  // ring stages, bytes per stage, neurons of B^T per stage
  int tile_max, chunks_max;
};

struct Decode1Layout {
  size_t x, h, bias, c, red, red2, bits, decided, desc, bars, total;
};

__host__ __device__ inline size_t decode1_align(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline Decode1Layout decode1_layout(const Decode1Params &P) {
  const size_t esz = P.dt == SFNN_F16 ? 2 : 4;
  Decode1Layout L;
  size_t o = (size_t)P.S * P.SB;
  L.x = o;
  o = decode1_align(o + (size_t)P.d * esz, 16);
  L.h = o;
  o = decode1_align(o + (size_t)P.r * 4, 16);
  L.bias = o;
  o = decode1_align(o + (size_t)P.tile_max * 4, 16);
  L.c = o;
  o = decode1_align(o + (size_t)P.tile_max * 4, 16);
  L.red = o;
  o = decode1_align(o + 2 * 8 * 2 * 4, 16);
  L.red2 = o;
  o = decode1_align(o + 256 * 4, 16);
  L.bits = o;
  o = decode1_align(o + (size_t)((P.tile_max + 31) / 32) * 4, 16);
  L.decided = o;
  o = decode1_align(o + (size_t)P.chunks_max * 4, 16);
  L.desc = o;
  o = decode1_align(o + (size_t)P.S * 16, 16);
  L.bars = o;
  o = decode1_align(o + (size_t)(2 * P.S + 2) * 8 + 8, 16);
  L.total = o;
  return L;
}

// First neuron position of tile c when n neurons are split into G contiguous tiles.
__host__ __device__ inline int decode1_tile_start(int c, int n, int G) {
  const int q = n / G, rr = n % G;
  return c * q + (c < rr ? c : rr);
}

cudaError_t configure_decode1();
int decode1_threads();
int decode1_blocks_per_sm(const Decode1Params &P);  // co-resident CTAs per SM for this plan
cudaError_t launch_decode1(const Decode1Params &P, cudaStream_t stream, bool pdl);

}  // namespace sfnn
