// decode_multi.cu -- the fused decode kernel for a few tokens at once (batch 2..4).
//
// As a batch's active sets accumulate, their union grows and the benefit of sparsity
// shrinks (53ai.com "sparsity for LLM inference" page, section 工程效果); a union that
// small is no dense contraction yet, so a batch of 2 to 4 tokens stays on CUDA cores and
// keeps the single-token kernel's plan -- one persistent CTA of 16 warps per SM owning a
// tile of neurons (hotness ranks dealt round-robin to the tiles, hottest first inside
// each), two bounded grid barriers -- with every weight read once for all NB tokens:
//
//   A   h_t = relu(A^T x_t) for the NB tokens: each predictor row split in halves over a
//       warp pair, read once and multiplied by the NB inputs held in shared memory.  Grid
//       barrier (split: the hot prefix below runs between its arrival and its wait).
//   B   z_t = B^T h_t + c for the tile: each neuron's B^T row is split in two halves
//       over a pair of warps (so that each lane holds the NB hidden layers' values for
//       2 chunks in registers), half rows streaming through 6 shared-memory stages per
//       warp; the halves are added in a fixed order, then c.  Token t's bit is z_t > 0
//       (sigmoid(z) > 0.5); the union of the tokens' bits is compacted in order, each
//       union row with the set of tokens active on it.
//   C1  gate/up dot products of the union rows in 4 KB segments over all warps, for the
//       tokens active on each row only; ReLU / ReGLU; the activation is 0 for a token
//       whose set does not hold the row.
//   C2  the union rows of W_down into per-thread column accumulators for the NB tokens
//       (tokens with a zero activation skipped), staged as in the single-token kernel.
//   D   per-CTA partials of the NB outputs; grid barrier; fixed-order column sums.
//
// Products are accumulated in fp32 pairs (packed two-wide FMA); every sum has a fixed
// order, so results are bitwise reproducible.
#include "async.cuh"
#include "common.cuh"
#include "decode1.cuh"
#include "decode_dev.cuh"

namespace sfnn {
namespace {


__device__ __forceinline__ void unpack2(const uint4 &v, float2 (&f)[4]) {
  const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = __half22float2(h[i]);
}

// a.x += w.lo x.lo and a.y += w.hi x.hi for one fp16 pair each, by sm_100's mixed-precision
// FMA (the fp16 operands widen exactly and the product is exact in fp32: the result of
// widening first and a packed fp32 FMA, without the conversions)
__device__ __forceinline__ float2 fma_pair_h(uint32_t w, uint32_t x, float2 a) {
  asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %2;\n\t"
      "mov.b32 {xl, xh}, %3;\n\t"
      "fma.rn.f32.f16 %0, wl, xl, %0;\n\t"
      "fma.rn.f32.f16 %1, wh, xh, %1;\n\t}"
      : "+f"(a.x), "+f"(a.y)
      : "r"(w), "r"(x));
  return a;
}

// acc[t] += w . x_t over one 16-byte chunk (8 elements), for the tokens in `tok`: even
// elements into acc[t].x, odd ones into acc[t].y, in element order
template <int NB>
__device__ __forceinline__ void dot_tokens(const uint4 &w, const unsigned char *xs, size_t tstride, int ch,
                                           uint32_t tok, float2 (&acc)[NB]) {
#pragma unroll
  for (int t = 0; t < NB; ++t) {
    if ((tok >> t) & 1u) {
      const uint4 x = *reinterpret_cast<const uint4 *>(xs + t * tstride + (size_t)ch * 16);
      acc[t] = fma_pair_h(w.x, x.x, acc[t]);
      acc[t] = fma_pair_h(w.y, x.y, acc[t]);
      acc[t] = fma_pair_h(w.z, x.z, acc[t]);
      acc[t] = fma_pair_h(w.w, x.w, acc[t]);
    }
  }
}

template <int NB, int ACT, int MAXM>
__global__ void __launch_bounds__(kT, 1) k_decode_multi(const Decode1Params P) {
  constexpr int V = 8;   // fp16 elements per 16-byte chunk
  constexpr int MH = 2;  // chunks of a half row of B^T per lane (r <= 1024)
  const int DD = min(P.c2stages, decode1_dstages(MAXM));  // W_down rows in flight: 1, 2, 4 or 8
  const int kMB = P.bstages;                               // B^T half rows per warp: 2, 4, 6 or 8
  constexpr uint32_t ALL = (1u << NB) - 1u;
  extern __shared__ __align__(16) unsigned char smem[];
  const MultiLayout L = decode_multi_layout(P, NB);
  unsigned char *xs = smem + L.x;
  float *h_s = reinterpret_cast<float *>(smem + L.h);
  float *bias_s = reinterpret_cast<float *>(smem + L.bias);
  float *c_s = reinterpret_cast<float *>(smem + L.c);
  int *act_s = reinterpret_cast<int *>(smem + L.act);
  uint32_t *tok_s = reinterpret_cast<uint32_t *>(smem + L.tok);
  float *a_s = reinterpret_cast<float *>(smem + L.a);
  float *zpart = reinterpret_cast<float *>(smem + L.zpart);
  float *dots = reinterpret_cast<float *>(smem + L.dots);
  float *pdots = reinterpret_cast<float *>(smem + L.pdots);
  float *red2 = reinterpret_cast<float *>(smem + L.red2);
  uint32_t *tbits = reinterpret_cast<uint32_t *>(smem + L.tbits);
  uint32_t *ubits = reinterpret_cast<uint32_t *>(smem + L.ubits);
  int *wpref = reinterpret_cast<int *>(smem + L.wpref);
  int *cnt_s = reinterpret_cast<int *>(smem + L.bars);
  int *flag_s = cnt_s + 1;
  unsigned long long *target_s = reinterpret_cast<unsigned long long *>(cnt_s + 2);
  int *next_s = cnt_s + 4;  // C1's next work item
  int *ext_s = cnt_s + 5;   // C1's final row count once known (-1: not yet, -2: abandoned)
  unsigned char *stage = smem + L.stage;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = P.G;
  const int t0 = decode1_tile_start(c, P.n, G);
  const int tn = decode1_tile_start(c + 1, P.n, G) - t0;
  const int d = P.d, r = P.r, nproj = P.nproj;
  const int nch_d = d / V, nch_r = r / V;
  const int hc = (nch_r + 1) / 2;  // chunks of the first half of a B^T row
  const size_t xstride = (size_t)d * 2;
  const __half *At = static_cast<const __half *>(P.At);
  const __half *Bt = static_cast<const __half *>(P.Bt);
  const unsigned char *rows = static_cast<const unsigned char *>(P.rows);
  const size_t rowB = (size_t)d * 2;
  const int words = (tn + 31) / 32;

  pdl_launch_dependents();
  // A^T rows split in halves over warp pairs (as in the single-token kernel): a lane's
  // whole share of its first half row is requested before the wait for the previous kernel
  const int apair = warp >> 1, ahalf = warp & 1;
  const int hca = (nch_d + 1) / 2;
  const int abeg = ahalf * hca, aend = ahalf ? nch_d : hca;
  const int j0 = c + G * apair;  // this warp's first row of A^T

  // ---------------------------------------------------------------- A: hidden layers
  uint4 w0[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int ch = abeg + lane + 32 * u;
    if (j0 < r && ch < aend) w0[u] = ld_stream(At + (size_t)j0 * d + (size_t)ch * V);
  }
  const __half *cp = static_cast<const __half *>(P.cvec);
  const __half *bp = static_cast<const __half *>(P.bias);
  __half c_first = __float2half(0.f), b_first = __float2half(0.f);
  if (tid < tn) {
    c_first = cp[t0 + tid];
    b_first = bp[t0 + tid];
  }

  // B^T half rows: warp w takes half (w & 1) of the tile's neurons p = (w >> 1) + 8 k;
  // each lane copies exactly the chunks it reads
  const int half = warp & 1, pair = warp >> 1;
  constexpr int kPairs = kW / 2;
  const int hbeg = half * hc, hend = half ? nch_r : hc;
  unsigned char *bst = stage + (size_t)warp * kMB * MH * 32 * 16;
  auto stage_b = [&](int s, int p) {  // neuron p's half row into stage s; always one group
    if (p < tn) {
#pragma unroll
      for (int m = 0; m < MH; ++m) {
        const int ch = hbeg + lane + 32 * m;
        if (ch < hend)
          cp_async16(bst + ((size_t)s * MH * 32 + lane + 32 * m) * 16, Bt + (size_t)(t0 + p) * r + (size_t)ch * V);
      }
    }
    cp_async_commit();
  };
  pdl_wait();  // X (and every buffer this kernel writes) belongs to earlier kernels until here
  {
    uint4 xv[NB * MAXM];  // every load of X in flight at once, then into shared memory
#pragma unroll
    for (int m = 0; m < NB * MAXM; ++m) {
      const int i = tid + kT * m;
      if (i < NB * nch_d) xv[m] = __ldcg(reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(P.x) + (size_t)i * 16));
    }
#pragma unroll
    for (int m = 0; m < NB * MAXM; ++m) {
      const int i = tid + kT * m;
      if (i < NB * nch_d) *reinterpret_cast<uint4 *>(xs + (size_t)i * 16) = xv[m];
    }
  }
  __syncthreads();
  if (j0 >= r) {
#pragma unroll 1
    for (int s = 0; s < kMB; ++s) stage_b(s, pair + kPairs * s);
  }
  // each token's half-row sums go to hbuf[t][half][j]; h is formed after the barrier
  for (int j = j0; j < r; j += G * (kW / 2)) {
    const __half *row = At + (size_t)j * d;
    float2 acc[NB];
#pragma unroll
    for (int t = 0; t < NB; ++t) acc[t] = make_float2(0.f, 0.f);
    for (int cb = abeg; cb < aend; cb += 32 * 16) {
      if (j != j0 || cb != abeg) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int ch = cb + lane + 32 * u;
          if (ch < aend) w0[u] = ld_stream(row + (size_t)ch * V);
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int ch = cb + lane + 32 * u;
        if (ch < aend) dot_tokens<NB>(w0[u], xs, xstride, ch, ALL, acc);
      }
    }
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const float hs = warp_sum(acc[t].x + acc[t].y);
      if (lane == 0) P.hbuf[((size_t)t * 2 + ahalf) * r + j] = hs;
    }
  }
  if (tid < tn) {
    c_s[tid] = __half2float(c_first);
    a_s[tid] = __half2float(b_first);
  }
  for (int i = tid + kT; i < tn; i += kT) {
    c_s[i] = __half2float(cp[t0 + i]);
    a_s[i] = __half2float(bp[t0 + i]);
  }
  constexpr int NPG = ACT == SFNN_REGLU ? 2 : 1;  // projections with a dot: (gate,) up
  constexpr int SU = kSegChunks / 32;             // chunks per lane and 4 KB segment
  const int nseg = P.nseg;
  const int per_row = NPG * nseg;
  cta_grid_arrive(P, target_s);
  // the B^T stages of the warps with an A^T row go out after the arrival: its release
  // would otherwise wait for them to land
  if (j0 < r) {
#pragma unroll 1
    for (int s = 0; s < kMB; ++s) stage_b(s, pair + kPairs * s);
  }
  // The hot prefix (the tile's first hp positions: neurons in a batch's union with
  // probability >= 0.99) is read densely: its gate/up dots for every token are computed
  // while the barrier completes, before the sets are known; a prefix row that no token's
  // set holds is dropped after phase B.
  const int hp = min(tn, decode1_hot_rows(P.hot, c, G));
  for (int it = warp; it < hp * per_row; it += kW) {
    const int q = it / per_row, pj = (it - q * per_row) / nseg, sg = it - q * per_row - pj * nseg;
    const unsigned char *row = rows + ((size_t)(t0 + q) * nproj + pj) * rowB;
    uint4 w[SU];
#pragma unroll
    for (int u = 0; u < SU; ++u) {
      const int ch = sg * kSegChunks + lane + 32 * u;
      if (ch < nch_d) w[u] = ld_stream(row + (size_t)ch * 16);
    }
    float2 acc[NB];
#pragma unroll
    for (int t = 0; t < NB; ++t) acc[t] = make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < SU; ++u) {
      const int ch = sg * kSegChunks + lane + 32 * u;
      if (ch < nch_d) dot_tokens<NB>(w[u], xs, xstride, ch, ALL, acc);
    }
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const float v = warp_sum(acc[t].x + acc[t].y);
      if (lane == 0) pdots[(((size_t)q * 2 + pj) * nseg + sg) * NB + t] = v;
    }
  }
  if (!cta_grid_wait(P, target_s, flag_s)) {
    cp_async_wait<0>();  // no copy into shared memory outlives the CTA
    return;
  }

  // ---------------------------------------------------------------- B: logits + threshold
  {
    for (int i = tid; i < NB * r / 4; i += kT) {  // h_t = relu(first half + second half); NaN -> 0
      const int t = i / (r / 4), q = i - t * (r / 4);
      const float4 a = __ldcg(reinterpret_cast<const float4 *>(P.hbuf + (size_t)t * 2 * r) + q);
      const float4 b = __ldcg(reinterpret_cast<const float4 *>(P.hbuf + ((size_t)t * 2 + 1) * r) + q);
      const float4 h4 = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
      reinterpret_cast<float4 *>(h_s)[i] = make_float4(h4.x > 0.f ? h4.x : 0.f, h4.y > 0.f ? h4.y : 0.f,
                                                       h4.z > 0.f ? h4.z : 0.f, h4.w > 0.f ? h4.w : 0.f);
    }
    __syncthreads();
    float2 hreg[NB][MH][4];
#pragma unroll
    for (int t = 0; t < NB; ++t)
#pragma unroll
      for (int m = 0; m < MH; ++m) {
        const int ch = hbeg + lane + 32 * m;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float2 q = make_float2(0.f, 0.f);
          if (ch < hend) q = *reinterpret_cast<const float2 *>(h_s + (size_t)t * r + (size_t)ch * V + 2 * i);
          hreg[t][m][i] = q;
        }
      }
    for (int pb = pair; pb < tn; pb += kMB * kPairs) {
#pragma unroll 1
      for (int s = 0; s < kMB; ++s) {
        const int p = pb + kPairs * s;
        if (p < tn) {
          switch (kMB) {  // this lane's copies of neuron p's half row have landed
            case 2: cp_async_wait<1>(); break;
            case 4: cp_async_wait<3>(); break;
            case 6: cp_async_wait<5>(); break;
            default: cp_async_wait<7>(); break;
          }
          float2 a[NB];
#pragma unroll
          for (int t = 0; t < NB; ++t) a[t] = make_float2(0.f, 0.f);
#pragma unroll
          for (int m = 0; m < MH; ++m) {
            if (hbeg + lane + 32 * m < hend) {
              float2 bf[4];
              unpack2(*reinterpret_cast<const uint4 *>(bst + ((size_t)s * MH * 32 + lane + 32 * m) * 16), bf);
#pragma unroll
              for (int t = 0; t < NB; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) a[t] = __ffma2_rn(bf[i], hreg[t][m][i], a[t]);
            }
          }
          stage_b(s, p + kMB * kPairs);
#pragma unroll
          for (int t = 0; t < NB; ++t) {
            const float z = warp_sum(a[t].x + a[t].y);
            if (lane == 0) zpart[((size_t)half * P.tile_max + p) * NB + t] = z;
          }
        }
      }
    }
    cp_async_wait<0>();
  }
  __syncthreads();
  // decisions: z_t = (first half + second half) + c; a warp's 32 positions form one word
  for (int pb = warp * 32; pb < words * 32; pb += kT) {
    const int p = pb + lane;
    uint32_t any = 0u;
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      bool on = false;
      if (p < tn) {
        const float z = (zpart[(size_t)p * NB + t] + zpart[((size_t)P.tile_max + p) * NB + t]) + c_s[p];
        on = z > 0.f;  // NaN -> inactive
      }
      const uint32_t bw = __ballot_sync(0xffffffffu, on);
      any |= bw;
      if (lane == 0) tbits[t * words + (p >> 5)] = bw;
    }
    if (lane == 0) ubits[p >> 5] = any;
  }
  __syncthreads();
  // the union's positions, ascending, each with its tokens and b
  if (warp == 0) {
    int base = 0;
    for (int wi = 0; wi < words; wi += 32) {
      const int k = wi + lane < words ? __popc(ubits[wi + lane]) : 0;
      int incl = k;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (wi + lane < words) wpref[wi + lane] = base + incl - k;
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      *cnt_s = base;
      *next_s = 0;
      *ext_s = -1;
    }
  } else if (P.set_pos && warp <= NB) {  // token (warp - 1)'s own set, for callers that ask
    const int t = warp - 1;
    int base = 0;
    for (int wi = 0; wi < words; wi += 32) {
      const uint32_t wd = wi + lane < words ? tbits[t * words + wi + lane] : 0u;
      const int k = __popc(wd);
      int incl = k;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = base + incl - k;
      uint32_t m = wd;
      while (m) {
        const int bit = __ffs(m) - 1;
        m &= m - 1u;
        P.set_pos[(size_t)t * P.n + t0 + pos++] = t0 + (wi + lane) * 32 + bit;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) P.set_cnt[t * G + c] = base;
  }
  __syncthreads();
  for (int p = tid; p < tn; p += kT) {
    const uint32_t word = ubits[p >> 5], bit = 1u << (p & 31);
    if (word & bit) {
      const int k = wpref[p >> 5] + __popc(word & (bit - 1u));
      uint32_t tm = 0u;
#pragma unroll
      for (int t = 0; t < NB; ++t) tm |= ((tbits[t * words + (p >> 5)] & bit) ? 1u : 0u) << t;
      act_s[k] = t0 + p;
      tok_s[k] = tm;
      bias_s[k] = a_s[p];
    }
  }
  const int kp = __syncthreads_count(tid < hp && ((ubits[tid >> 5] >> (tid & 31)) & 1u));  // union rows in the prefix
  const int cnt = *cnt_s;
  // Rebalancing, as in the single-token kernel: each CTA keeps its first `quota` union rows
  // (at least its hot prefix, whose dots only it holds), publishes its list (position |
  // token mask << 24, b) and arrives on a split grid barrier; one warp waits on it beside
  // the own rows' stream, and the CTA takes an even share of all tiles' rows past the quota.
  const int quota = P.quota;
  if (quota > 0) {
    for (int k = tid; k < cnt; k += kT)
      P.blist[t0 + k] = make_int2(act_s[k] | (int)(tok_s[k] << 24), __float_as_int(bias_s[k]));
    if (tid == 0) P.bcnt[c] = cnt;
    cta_grid_arrive(P, target_s);
  }
  const int own = quota > 0 ? min(cnt, quota) : cnt;
  int nrows = own;  // union rows of this CTA whose place in act_s is known

  auto dslot = [&](int s, int m) { return stage + (((size_t)s * MAXM + m) * kT + tid) * 16; };
  auto stage_d = [&](int s, int k) {  // union row k's down row into stage s; always one group
    if (k < nrows) {
      const unsigned char *row = rows + ((size_t)act_s[k] * nproj + (nproj - 1)) * rowB;
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        const int ch = tid + kT * m;
        if (ch < nch_d) cp_async16(dslot(s, m), row + (size_t)ch * 16);
      }
    }
    cp_async_commit();
  };

  // ---------------------------------------------------------------- C1: gate / up dots
  // The union rows after the hot prefix, [kp, total): their 4 KB segments are work items
  // handed out in order by a shared counter, loaded into registers (no L1 allocation), dots
  // only for the tokens active on each row; a warp keeps c1depth segments in flight.  A
  // segment's dots do not depend on the warp that computes them.  C2's first rows are
  // requested behind each warp's first segments; with rebalancing, warp 0 waits on the
  // split barrier beside the stream and appends the rows shared out to this CTA.
  int total = own;
  int lim = (own - kp) * per_row;  // items known to exist
  bool known = quota == 0;         // the final count is known
  uint4 wa[SU], wb[SU];
  auto grab = [&]() {
    int v = 0;
    if (lane == 0) v = atomicAdd(next_s, 1);
    return __shfl_sync(0xffffffffu, v, 0);
  };
  auto avail = [&](int it) {  // 1: item `it` exists, 0: past the end, -1: abandoned
    if (it < lim) return 1;
    if (known) return 0;
    int e = -1;  // the rebalancing's count: wait for warp 0 to publish it (bounded)
    if (lane == 0) {
      const uint64_t t0c = clock64();
      while ((e = *reinterpret_cast<volatile int *>(ext_s)) == -1)
        if ((uint64_t)(clock64() - t0c) > 2 * kWaitCycles) {
          latch_error(P.err, kErrTimeout);
          e = -2;
          break;
        }
      __threadfence_block();
    }
    e = __shfl_sync(0xffffffffu, e, 0);
    __syncwarp();
    if (e < 0) return -1;
    known = true;
    total = e;
    nrows = e;
    lim = (e - kp) * per_row;
    return it < lim ? 1 : 0;
  };
  auto load_c = [&](uint4 *w, int it) {  // item `it` (which exists) into registers
    const int k = kp + it / per_row, pj = (it % per_row) / nseg, sg = it % per_row - pj * nseg;
    const unsigned char *row = rows + ((size_t)act_s[k] * nproj + pj) * rowB;
#pragma unroll
    for (int u = 0; u < SU; ++u) {
      const int ch = sg * kSegChunks + lane + 32 * u;
      if (ch < nch_d) w[u] = ld_stream(row + (size_t)ch * 16);
    }
  };
  auto sum_c = [&](const uint4 *w, int it) {  // its dots into dots, for the row's tokens
    const int k = kp + it / per_row, pj = (it % per_row) / nseg, sg = it % per_row - pj * nseg;
    const uint32_t tm = tok_s[k];
    float2 acc[NB];
#pragma unroll
    for (int t = 0; t < NB; ++t) acc[t] = make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < SU; ++u) {
      const int ch = sg * kSegChunks + lane + 32 * u;
      if (ch < nch_d) dot_tokens<NB>(w[u], xs, xstride, ch, tm, acc);
    }
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      if ((tm >> t) & 1u) {  // warp-uniform: the item's row is the warp's
        const float v = warp_sum(acc[t].x + acc[t].y);
        if (lane == 0) dots[(((size_t)k * 2 + pj) * nseg + sg) * NB + t] = v;
      }
    }
  };
  const bool two = P.c1depth > 1;
  int ia = grab(), ib = two ? grab() : 0;
  int sa = ia < lim ? 1 : 2, sb = two ? (ib < lim ? 1 : 2) : 0;  // 2: not known yet
  if (sa == 1) load_c(wa, ia);
  if (sb == 1) load_c(wb, ib);
  const int pre = min(min(DD, P.c2pre), own);
  for (int s = 0; s < pre; ++s) stage_d(s, s);  // behind C1's first loads, which gate C2
  if (!known && warp == 0) {  // the split barrier's wait and the shared-out rows
    int e = -2;
    if (warp_grid_wait(P, target_s)) {
      const int f = share_excess_warp(P, quota, reinterpret_cast<int *>(red2), [&](int j, int2 en) {
        act_s[own + j] = en.x & 0xFFFFFF;
        tok_s[own + j] = (uint32_t)en.x >> 24;
        bias_s[own + j] = __int_as_float(en.y);
      });
      e = own + f;
    }
    if (lane == 0) {
      __threadfence_block();  // the rows' entries before the count
      *reinterpret_cast<volatile int *>(ext_s) = e;
    }
    __syncwarp();
  }
  if (sa == 2) {
    sa = avail(ia);
    if (sa == 1) load_c(wa, ia);
  }
  if (sb == 2 && sa >= 0) {
    sb = avail(ib);
    if (sb == 1) load_c(wb, ib);
  }
#pragma unroll 1
  while (sa > 0 || sb > 0) {
    if (sa < 0 || sb < 0) break;
    if (sa > 0) {
      sum_c(wa, ia);
      ia = grab();
      sa = avail(ia);
      if (sa > 0) load_c(wa, ia);
    }
    if (sb > 0 && sa >= 0) {
      sum_c(wb, ib);
      ib = grab();
      sb = avail(ib);
      if (sb > 0) load_c(wb, ib);
    }
  }
  if (sa < 0 || sb < 0) {  // abandoned: the split barrier timed out (every warp sees it)
    cp_async_wait<0>();
    return;
  }
  __syncthreads();
  for (int e = tid; e < total * NB; e += kT) {
    const int k = e / NB, t = e - k * NB;
    float a = 0.f;
    if ((tok_s[k] >> t) & 1u) {
      // the prefix's dots by tile position, the others' by union row
      const float *dk = k < kp ? pdots + (size_t)(act_s[k] - t0) * 2 * nseg * NB : dots + (size_t)k * 2 * nseg * NB;
      float g = 0.f, u = 0.f;  // g: the ReLU'd projection (up for ReLU, gate for ReGLU)
      for (int sg = 0; sg < nseg; ++sg) g += dk[(size_t)sg * NB + t];
      if (ACT == SFNN_REGLU)
        for (int sg = 0; sg < nseg; ++sg) u += dk[((size_t)nseg + sg) * NB + t];
      const float pre_act = g + bias_s[k];
      const float relu = pre_act > 0.f ? pre_act : 0.f;
      a = ACT == SFNN_RELU ? relu : relu * u;
    }
    a_s[e] = a;
  }
  __syncthreads();
  for (int s = pre; s < DD; ++s) stage_d(s, s);  // C2's first stages not requested yet

  // ---------------------------------------------------------------- C2: down projection
  float2 acc[MAXM][4][NB];
#pragma unroll
  for (int m = 0; m < MAXM; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < NB; ++t) acc[m][i][t] = make_float2(0.f, 0.f);
  for (int kb = 0; kb < total; kb += DD) {
#pragma unroll 1
    for (int s = 0; s < DD; ++s) {
      const int k = kb + s;
      if (k < total) {
        switch (DD) {  // this thread's chunks of row k have landed
          case 1: cp_async_wait<0>(); break;
          case 2: cp_async_wait<1>(); break;
          case 4: cp_async_wait<3>(); break;
          default: cp_async_wait<7>(); break;
        }
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
          if (tid + kT * m < nch_d) {
            float2 f[4];
            unpack2(*reinterpret_cast<const uint4 *>(dslot(s, m)), f);
#pragma unroll
            for (int t = 0; t < NB; ++t) {
              const float a = a_s[k * NB + t];
              if (a != 0.f) {  // the same for every thread: row k's activation for token t
                const float2 a2 = make_float2(a, a);
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[m][i][t] = __ffma2_rn(a2, f[i], acc[m][i][t]);
              }
            }
          }
        }
        stage_d(s, k + DD);
      }
    }
  }
  cp_async_wait<0>();

  // ---------------------------------------------------------------- D: partials, final sums
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    const int ch = tid + kT * m;
    if (ch < nch_d) {
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        float4 *dst = reinterpret_cast<float4 *>(P.part + ((size_t)c * NB + t) * d + (size_t)ch * V);
        dst[0] = make_float4(acc[m][0][t].x, acc[m][0][t].y, acc[m][1][t].x, acc[m][1][t].y);
        dst[1] = make_float4(acc[m][2][t].x, acc[m][2][t].y, acc[m][3][t].x, acc[m][3][t].y);
      }
    }
  }
  if (!cta_grid_sync(P, flag_s)) return;
  // the stage region is free again: C2's copies have all landed
  column_sums<NB, kMultiMaxTokens>(P.part, d, G, reinterpret_cast<float4 *>(stage), [&](int t, int col, float4 v) {
    const float t4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const size_t o = (size_t)t * d + col + i;
      float tot = t4[i];
      if (P.resid) tot = P.resid[o] + tot;
      P.y[o] = tot;
      if (P.xnext) static_cast<__half *>(P.xnext)[o] = __float2half_rn(tot);
    }
  });
}

template <int NB, int ACT, int MAXM>
cudaError_t launch_t(const Decode1Params &P, size_t smem, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.G);
  cfg.blockDim = dim3(kT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  cfg.numAttrs = fused_launch_attrs(attr, pdl);
  return cudaLaunchKernelEx(&cfg, k_decode_multi<NB, ACT, MAXM>, P);
}

template <int NB, int ACT>
const void *kernel_for(int nch) {
  if (nch <= kT) return (const void *)k_decode_multi<NB, ACT, 1>;
  if (nch <= 2 * kT) return (const void *)k_decode_multi<NB, ACT, 2>;
  return nullptr;
}

const void *plan_kernel(int nb, int act, int nch) {
  const bool g = act == SFNN_REGLU;
  switch (nb) {
    case 2: return g ? kernel_for<2, SFNN_REGLU>(nch) : kernel_for<2, SFNN_RELU>(nch);
    case 3: return g ? kernel_for<3, SFNN_REGLU>(nch) : kernel_for<3, SFNN_RELU>(nch);
    case 4: return g ? kernel_for<4, SFNN_REGLU>(nch) : kernel_for<4, SFNN_RELU>(nch);
  }
  return nullptr;
}

template <int NB, int ACT>
cudaError_t launch_nb(const Decode1Params &P, size_t smem, cudaStream_t stream, bool pdl) {
  const int nch = P.d / 8;
  if (nch <= kT) return launch_t<NB, ACT, 1>(P, smem, stream, pdl);
  return launch_t<NB, ACT, 2>(P, smem, stream, pdl);
}

}  // namespace

cudaError_t configure_decode_multi() {
  for (int nb = 2; nb <= kMultiMaxTokens; ++nb)
    for (int act = 0; act < 2; ++act)
      for (int nch : {kT, 2 * kT}) {
        const void *k = plan_kernel(nb, act, nch);
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCap);
        if (e != cudaSuccess) return e;
      }
  return cudaSuccess;
}

// Co-resident CTAs per SM of the multi-token kernel for NB tokens (0: it does not fit:
// fp16 only, d <= 16384 (two 16-byte chunks per thread), r <= 1024).
int decode_multi_blocks_per_sm(const Decode1Params &P, int nb) {
  if (P.dt != SFNN_F16 || P.rq || nb < 2 || nb > kMultiMaxTokens) return 0;
  if (P.r / 8 > 2 * 2 * 32 || P.d / 8 > 2 * kT) return 0;
  const size_t smem = decode_multi_layout(P, nb).total;
  if (smem > (size_t)kSmemCap) return 0;
  const void *k = plan_kernel(nb, P.act, P.d / 8);
  int blocks = 0;
  if (!k || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, k, kT, smem) != cudaSuccess) return 0;
  return blocks;
}

cudaError_t launch_decode_multi(const Decode1Params &P, int nb, cudaStream_t stream, bool pdl) {
  const size_t smem = decode_multi_layout(P, nb).total;
  const bool g = P.act == SFNN_REGLU;
  switch (nb) {
    case 2: return g ? launch_nb<2, SFNN_REGLU>(P, smem, stream, pdl) : launch_nb<2, SFNN_RELU>(P, smem, stream, pdl);
    case 3: return g ? launch_nb<3, SFNN_REGLU>(P, smem, stream, pdl) : launch_nb<3, SFNN_RELU>(P, smem, stream, pdl);
    case 4: return g ? launch_nb<4, SFNN_REGLU>(P, smem, stream, pdl) : launch_nb<4, SFNN_RELU>(P, smem, stream, pdl);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sfnn
