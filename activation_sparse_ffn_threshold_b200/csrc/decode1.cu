// decode1.cu -- the fused single-token decode kernel (batch 1): one launch per token.
//
// Decode is bound by reading weights, not by arithmetic (53ai.com "sparsity for LLM
// inference" page, its opening analysis: the I/O of loading parameters dominates token
// generation), so the kernel is a sequence of streaming phases, each keeping many
// 16-byte loads in flight per SM, inside one persistent launch:
//
//   grid: one CTA of 16 warps per SM (G CTAs, all resident).  CTA c owns a contiguous
//   tile of neurons; the storage order deals hotness ranks round-robin to the tiles,
//   so every tile holds the same mix of hot and cold neurons (equal expected work),
//   hottest first inside the tile.
//
//   A   h_j = relu(A^T[j] . x): each predictor row split in two halves over a pair of
//       warps, every chunk of the first half row requested before waiting for the
//       previous kernel; the halves' sums go to global memory; grid barrier.
//   B   z_i = B^T[i] . h + c_i for the tile, one warp per neuron (h = relu of the two
//       halves' sum, formed once per CTA); each warp's B^T rows stream through 4
//       shared-memory stages of its own (16-byte cp.async copies, the first ones requested
//       during phase A); neuron i is active iff z_i > 0 (sigmoid(z) > 0.5).  The tile's
//       active positions are compacted in order.
//   C1  up (and gate) dot products of the active rows, split in 4 KB segments dealt to
//       the warps; each warp streams its segments through 3 shared-memory slots of its
//       own (192 KB of the CTA's shared memory in flight); segment sums added in a fixed
//       order, then ReLU / ReGLU.  Rows of inactive neurons are never requested.
//   C2  the active rows of W_down (neuron-major, contiguous) are added into per-thread
//       column accumulators; each thread's chunks stream through private shared-memory
//       stages (128 KB of rows in flight per CTA).
//   D   the CTA's partial y goes to global memory; grid barrier; CTA c sums a column
//       slice of all G partials in a fixed order (two-phase, deterministic) -> y
//       (+ residual, + rounded next-layer input).
//
// Which CTA reads which active rows: the hotness deal keeps the tiles' expected counts
// equal, but the busiest tile of a token still holds ~1.5x the mean, and with its own
// tile's rows alone that CTA finishes long after the others.  With a quota (set from the
// hotness profile: 0.8 of a tile's expected count) each CTA keeps its first `quota` rows,
// publishes its tile's list and arrives on a split grid barrier; after its own rows' C1
// it waits there, and the rows past the quota in all tiles are shared out evenly over
// the CTAs in tile order -- a function of the counts alone, so every sum keeps a fixed
// order and results stay bitwise reproducible.  Without a quota every CTA takes its own
// tile's rows (two grid barriers).
//
// PDL: the kernel lets the next one launch at once and reads x, and writes anything,
// only after griddepcontrol.wait.  Every grid barrier is bounded: on a timeout the
// kernel latches SFNN_ERR_TIMEOUT and returns without a result.
#include "async.cuh"
#include "common.cuh"
#include "decode1.cuh"
#include "decode_dev.cuh"

namespace sfnn {
namespace {

template <typename T, int ACT, int MAXM, typename R>
__global__ void __launch_bounds__(kT, 1) k_decode1(const Decode1Params P) {
  constexpr int V = Elem<T>::kVec;
  constexpr int RB = RowFmt<R>::kBits;  // bits of a stored row element
  constexpr bool QR = RB <= 8;           // rows are codes with per-row scales
  constexpr int VR = 128 / RB;           // row elements per 16-byte chunk
  constexpr int MAXH = 4;  // chunks of h per lane (r <= 128 * V)
  const int DB = P.bstages;  // 1, 2, 3, 4, 6 or 8
  const int DD = min(P.c2stages, decode1_c2stages(MAXM));  // 1, 2, 4, 8 or 16
  extern __shared__ __align__(16) unsigned char smem[];
  const Decode1Layout L = decode1_layout(P, true);
  unsigned char *xs = smem + L.x;
  float *bias_s = reinterpret_cast<float *>(smem + L.bias);  // b of the active rows, in order
  float *c_s = reinterpret_cast<float *>(smem + L.c);
  int *act_s = reinterpret_cast<int *>(smem + L.act);
  float *a_s = reinterpret_cast<float *>(smem + L.a);  // b of the tile, then activations
  float *dots = reinterpret_cast<float *>(smem + L.dots);
  float *red2 = reinterpret_cast<float *>(smem + L.red2);
  uint32_t *bits = reinterpret_cast<uint32_t *>(smem + L.bits);
  int *wpref = reinterpret_cast<int *>(smem + L.wpref);
  float *h_s = reinterpret_cast<float *>(smem + L.h);
  int *cnt_s = reinterpret_cast<int *>(smem + L.bars);
  int *flag_s = cnt_s + 1;
  unsigned long long *target_s = reinterpret_cast<unsigned long long *>(cnt_s + 2);  // split barrier
  int *next_s = cnt_s + 4;  // C1's next work item
  int *ext_s = cnt_s + 5;   // C1's final row count once known (-1: not yet, -2: abandoned)
  unsigned char *bstage = smem + L.bstage;
  unsigned char *dstage = smem + L.dstage;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = P.G;
  const int t0 = decode1_tile_start(c, P.n, G);
  const int tn = decode1_tile_start(c + 1, P.n, G) - t0;
  const int d = P.d, r = P.r, nproj = P.nproj;
  const int nch_d = d / V, nch_r = r / V;
  const T *At = static_cast<const T *>(P.At);
  const T *Bt = static_cast<const T *>(P.Bt);
  const unsigned char *rows = static_cast<const unsigned char *>(P.rows);
  const size_t rowB = (size_t)P.d * RB / 8;  // bytes of one stored row

  pdl_launch_dependents();
  // The launch is cooperative: its CTAs start together once the previous kernel's CTAs
  // have left the SMs, so the wait for that kernel costs little here, and x is requested
  // first, ahead of the weights' streams.
  pdl_wait();  // x (and every buffer this kernel writes) belongs to earlier kernels until here
  uint4 xv[MAXM];
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    const int ch = tid + kT * m;
    if (ch < nch_d) xv[m] = __ldcg(reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(P.x) + (size_t)ch * 16));
  }
  // A^T rows are split in halves over warp pairs: warp w takes half (w & 1) of the rows
  // j = c + G (w >> 1) + 8 G k, so that a lane's part of its first half row (at most 16
  // chunks for d <= 8192 fp16) is requested at once.
  const int apair = warp >> 1, ahalf = warp & 1;
  const int hca = (nch_d + 1) / 2;  // chunks of a row's first half
  const int abeg = ahalf * hca, aend = ahalf ? nch_d : hca;
  const int j0 = c + G * apair;  // this warp's first row of A^T

  // ---------------------------------------------------------------- A: hidden layer
  uint4 w0[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int ch = abeg + lane + 32 * u;
    if (j0 < r && ch < aend) w0[u] = ld_stream(At + (size_t)j0 * d + (size_t)ch * V);
  }
  const T *cp = static_cast<const T *>(P.cvec);
  const T *bp = static_cast<const T *>(P.bias);
  T c_first = from_f<T>(0.f), b_first = from_f<T>(0.f);  // c and b at tile position tid
  if (tid < tn) {
    c_first = cp[t0 + tid];
    b_first = bp[t0 + tid];
  }
  for (int i = tid; i < (P.tile_max + 31) / 32; i += kT) bits[i] = 0u;

  // B^T rows of this warp's neurons stream through DB shared-memory stages private to the
  // warp; each lane copies (cp.async) exactly the chunks it will read, so only its own
  // wait is needed.  The first DB rows are requested as soon as x has landed, and land
  // while phase A and the barrier run.
  unsigned char *bst = bstage + (size_t)warp * DB * nch_r * 16;
  auto stage_b = [&](int s, int p) {  // row p of the tile into stage s; always one group
    if (p < tn) {
#pragma unroll
      for (int m = 0; m < MAXH; ++m) {
        const int ch = lane + 32 * m;
        if (ch < nch_r) cp_async16(bst + ((size_t)s * nch_r + ch) * 16, Bt + (size_t)(t0 + p) * r + (size_t)ch * V);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    const int ch = tid + kT * m;
    if (ch < nch_d) *reinterpret_cast<uint4 *>(xs + (size_t)ch * 16) = xv[m];
  }
  __syncthreads();
  // every warp requests its first two B^T rows now (x has landed), behind its first A^T half
  // row, and the rest of its DB stages once its A^T rows have landed (more requests at once
  // would only queue ahead of phase A's)
  const int db0 = min(DB, 2);
#pragma unroll 1
  for (int s = 0; s < db0; ++s) stage_b(s, warp + kW * s);
  // each half row's dot product (chunks ascending in one chain, then a butterfly sum) goes
  // to hbuf[half][j]; h_j = relu(first half + second half) is formed after the barrier
  for (int j = j0; j < r; j += G * (kW / 2)) {
    const T *row = At + (size_t)j * d;
    float acc = 0.f;
    for (int cb = abeg; cb < aend; cb += 32 * 16) {
      if (j != j0 || cb != abeg) {  // the first batch of the first row is already in w0
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int ch = cb + lane + 32 * u;
          if (ch < aend) w0[u] = ld_stream(row + (size_t)ch * V);
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int ch = cb + lane + 32 * u;
        if (ch < aend) acc = dot_chunk_smem<T>(w0[u], xs, ch, acc);
      }
    }
    const float hs = warp_sum(acc);
    if (lane == 0) P.hbuf[(size_t)ahalf * r + j] = hs;
  }
  // c and b of the tile into shared memory
  if (tid < tn) {
    c_s[tid] = to_f<T>(c_first);
    a_s[tid] = to_f<T>(b_first);
  }
  for (int i = tid + kT; i < tn; i += kT) {
    c_s[i] = to_f<T>(cp[t0 + i]);
    a_s[i] = to_f<T>(bp[t0 + i]);
  }
  cta_grid_arrive(P, target_s);
  // the rest of the first DB B^T rows go out after the arrival (its release would otherwise
  // wait for them to land), and land during the barrier
#pragma unroll 1
  for (int s = db0; s < DB; ++s) stage_b(s, warp + kW * s);
  if (!cta_grid_wait(P, target_s, flag_s)) {
    cp_async_wait<0>();  // no copy into shared memory outlives the CTA
    return;
  }

  // ---------------------------------------------------------------- B: logits + threshold
  {
    // h = relu(first half + second half) once per CTA from L2 (every warp needs all of
    // it), then into registers
    for (int i = tid; i < r / 4; i += kT) {
      const float4 a = __ldcg(reinterpret_cast<const float4 *>(P.hbuf) + i);
      const float4 b = __ldcg(reinterpret_cast<const float4 *>(P.hbuf + r) + i);
      const float4 h4 = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
      reinterpret_cast<float4 *>(h_s)[i] = make_float4(h4.x > 0.f ? h4.x : 0.f, h4.y > 0.f ? h4.y : 0.f,
                                                       h4.z > 0.f ? h4.z : 0.f, h4.w > 0.f ? h4.w : 0.f);  // NaN -> 0
    }
    __syncthreads();
    float hreg[MAXH][V];
#pragma unroll
    for (int m = 0; m < MAXH; ++m) {
      const int ch = lane + 32 * m;
#pragma unroll
      for (int v = 0; v < V; v += 4) {
        float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ch < nch_r) q = *reinterpret_cast<const float4 *>(h_s + (size_t)ch * V + v);
        hreg[m][v] = q.x;
        hreg[m][v + 1] = q.y;
        hreg[m][v + 2] = q.z;
        hreg[m][v + 3] = q.w;
      }
    }
    for (int pb = warp; pb < tn; pb += DB * kW) {
#pragma unroll 1
      for (int s = 0; s < DB; ++s) {
        const int p = pb + kW * s;
        if (p < tn) {
          switch (DB) {  // this lane's copies of row p have landed
            case 1: cp_async_wait<0>(); break;
            case 2: cp_async_wait<1>(); break;
            case 3: cp_async_wait<2>(); break;
            case 4: cp_async_wait<3>(); break;
            case 6: cp_async_wait<5>(); break;
            default: cp_async_wait<7>(); break;
          }
          float a = 0.f;
#pragma unroll
          for (int m = 0; m < MAXH; ++m) {
            const int ch = lane + 32 * m;
            if (ch < nch_r)
              a = dot_chunk<T>(*reinterpret_cast<const uint4 *>(bst + ((size_t)s * nch_r + ch) * 16), hreg[m], a);
          }
          stage_b(s, p + DB * kW);
          const float z = warp_sum(a) + c_s[p];
          if (lane == 0 && z > 0.f) atomicOr(&bits[p >> 5], 1u << (p & 31));  // NaN -> inactive
        }
      }
    }
    cp_async_wait<0>();
  }
  __syncthreads();
  // The tile's active positions, ascending: warp 0 scans the words' population counts,
  // then every thread places its own positions.  The CTA takes its own tile's active
  // rows: the hotness deal gives every tile the same expected count, and the rows stay
  // where their decisions were made (no exchange).
  const int nwords = (tn + 31) / 32;
  if (warp == 0) {
    int base = 0;
    for (int wi = 0; wi < nwords; wi += 32) {
      const int k = wi + lane < nwords ? __popc(bits[wi + lane]) : 0;
      int incl = k;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (wi + lane < nwords) wpref[wi + lane] = base + incl - k;
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      *cnt_s = base;
      *next_s = 0;
      *ext_s = -1;
    }
  }
  __syncthreads();
  for (int p = tid; p < tn; p += kT) {
    const uint32_t word = bits[p >> 5], bit = 1u << (p & 31);
    if (word & bit) {
      const int k = wpref[p >> 5] + __popc(word & (bit - 1u));
      act_s[k] = t0 + p;
      bias_s[k] = a_s[p];
    }
  }
  __syncthreads();
  const int cnt = *cnt_s;
  if (P.set_pos) {  // the tile's decisions, exactly as the rows below are read
    for (int k = tid; k < cnt; k += kT) P.set_pos[t0 + k] = act_s[k];
    if (tid == 0) P.set_cnt[c] = cnt;
  }
  // Rebalancing (quota > 0): the busiest tile of a token holds ~1.5x the mean count, and
  // the CTAs that finish their rows early would leave the HBM stream to it.  So each CTA
  // keeps the first `quota` of its tile's active rows, publishes its list, and arrives on
  // a grid barrier; one warp waits on it while the others stream the own rows, and the
  // rows past the quota in every tile are shared out evenly over all CTAs, in tile order
  // (a function of the counts alone: deterministic).
  const int quota = P.quota;
  if (quota > 0) {
    for (int k = tid; k < cnt; k += kT) P.blist[t0 + k] = make_int2(act_s[k], __float_as_int(bias_s[k]));
    if (tid == 0) P.bcnt[c] = cnt;
    cta_grid_arrive(P, target_s);  // its CTA barrier orders the list before the release
  }
  const int own = quota > 0 ? min(cnt, quota) : cnt;
  int nrows = own;  // rows of this CTA whose place in act_s is known

  // C2's rows of W_down stream through DD shared-memory stages private to each thread
  auto dslot = [&](int s, int m) { return dstage + (((size_t)s * MAXM + m) * kT + tid) * 16; };
  auto stage_d = [&](int s, int k) {  // active row k into stage s; always one group
    if (k < nrows) {
      const unsigned char *row = rows + ((size_t)act_s[k] * nproj + (nproj - 1)) * rowB;
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        const int ch = tid + kT * m;  // V columns (code rows: their V codes, 8 or 4 bytes)
        if (ch < nch_d) {
          const unsigned char *src = row + (size_t)ch * V * RB / 8;
          if (RB == 4)
            cp_async4(dslot(s, m), src);
          else if (RB == 8)
            cp_async8(dslot(s, m), src);
          else
            cp_async16(dslot(s, m), src);
        }
      }
    }
    cp_async_commit();
  };

  // ---------------------------------------------------------------- C1: up / gate dots
  constexpr int NPG = ACT == SFNN_REGLU ? 2 : 1;  // projections with a dot: (gate,) up
  constexpr int SU = kSegChunks / 32;             // chunks per lane and segment
  const int nseg = P.nseg;
  const int per_row = NPG * nseg;
  const int nch_r8 = d / VR;  // 16-byte chunks of a row
  // The rows' 4 KB segments are work items, handed out in order by a shared counter; each
  // lane loads its SU chunks of a segment into registers (no L1 allocation), and a warp
  // keeps two segments in flight: the next one's loads are issued before the current one
  // is summed.  A segment's dot product does not depend on the warp that computes it.
  int total = own;
  int lim = own * per_row;  // items known to exist
  bool known = quota == 0;  // the final count is known
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
      const uint64_t t0 = clock64();
      while ((e = *reinterpret_cast<volatile int *>(ext_s)) == -1)
        if ((uint64_t)(clock64() - t0) > 2 * kWaitCycles) {
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
    lim = e * per_row;
    return it < lim ? 1 : 0;
  };
  auto load_c = [&](uint4 *w, int it) {  // item `it` (which exists) into registers
    const int k = it / per_row, pj = (it % per_row) / nseg, sg = it % per_row - pj * nseg;
    const unsigned char *row = rows + ((size_t)act_s[k] * nproj + pj) * rowB;
#pragma unroll
    for (int u = 0; u < SU; ++u) {
      const int ch = sg * kSegChunks + lane + 32 * u;
      if (ch < nch_r8) w[u] = ld_stream(row + (size_t)ch * 16);
    }
  };
  auto sum_c = [&](const uint4 *w, int it) {  // its dot product into dots
    const int k = it / per_row, pj = (it % per_row) / nseg, sg = it % per_row - pj * nseg;
    float a = 0.f;
#pragma unroll
    for (int u = 0; u < SU; ++u) {
      const int ch = sg * kSegChunks + lane + 32 * u;
      if (ch < nch_r8) {
        if (RB == 4)
          a = dot_chunk_i4(w[u], xs, ch, a);
        else if (RB == 8)
          a = dot_chunk_i8(w[u], xs, ch, a);
        else
          a = dot_chunk_smem<T>(w[u], xs, ch, a);
      }
    }
    a = warp_sum(a);
    if (lane == 0) dots[(k * 2 + pj) * nseg + sg] = a;
  };
  // Each warp's first two segments are requested before anything else (few rows: all of
  // them), then C2's first rows: C1 reads into registers, so the staging region is free,
  // and they land while C1 streams (rows shared out by the rebalancing come after the own
  // rows; their stages follow C1).
  const bool two = P.c1depth > 1;
  int ia = grab(), ib = two ? grab() : 0;
  int sa = ia < lim ? 1 : 2, sb = two ? (ib < lim ? 1 : 2) : 0;  // 2: not known yet
  if (sa == 1) load_c(wa, ia);
  if (sb == 1) load_c(wb, ib);
  const int pre = min(min(DD, P.c2pre), own);
#pragma unroll 1
  for (int s = 0; s < pre; ++s) stage_d(s, s);
  if (!known && warp == 0) {  // the split barrier's wait and the shared-out rows
    int e = -2;
    if (warp_grid_wait(P, target_s)) {
      const int f = share_excess_warp(P, quota, reinterpret_cast<int *>(red2), [&](int j, int2 en) {
        act_s[own + j] = en.x;
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
  // two segments in flight (c1depth 2): while one is summed, the other's loads are
  // outstanding; with one (sb stays 0), the next segment is requested after the sum
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
  for (int k = tid; k < total; k += kT) {
    float g = 0.f, u = 0.f;  // g: the ReLU'd projection (up for ReLU, gate for ReGLU)
    for (int sg = 0; sg < nseg; ++sg) g += dots[(k * 2 + 0) * nseg + sg];
    if (ACT == SFNN_REGLU)
      for (int sg = 0; sg < nseg; ++sg) u += dots[(k * 2 + 1) * nseg + sg];
    float sd = 1.f;
    if (QR) {  // the codes' sums times their rows' scales; the down row's folded into a
      const float *sc = P.rscale + (size_t)act_s[k] * nproj;
      g *= sc[0];
      if (ACT == SFNN_REGLU) u *= sc[1];
      sd = sc[nproj - 1];
    }
    const float pre_act = g + bias_s[k];
    const float relu = pre_act > 0.f ? pre_act : 0.f;
    a_s[k] = ACT == SFNN_RELU ? relu : relu * u;
    if (QR) a_s[k] *= sd;
  }
  __syncthreads();
#pragma unroll 1
  for (int s = pre; s < DD; ++s) stage_d(s, s);  // the rest of C2's first stages

  // ---------------------------------------------------------------- C2: down projection
  float acc[MAXM][V];
#pragma unroll
  for (int m = 0; m < MAXM; ++m)
#pragma unroll
    for (int v = 0; v < V; ++v) acc[m][v] = 0.f;
  for (int kb = 0; kb < total; kb += DD) {
#pragma unroll 1
    for (int s = 0; s < DD; ++s) {
      const int k = kb + s;
      if (k < total) {
        switch (DD) {  // this thread's chunks of row k have landed
          case 1: cp_async_wait<0>(); break;
          case 2: cp_async_wait<1>(); break;
          case 4: cp_async_wait<3>(); break;
          case 8: cp_async_wait<7>(); break;
          default: cp_async_wait<15>(); break;
        }
        const float a = a_s[k];
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
          if (tid + kT * m < nch_d) {
            float f[V];
            if (RB == 4) {
              const uint32_t q = *reinterpret_cast<const uint32_t *>(dslot(s, m));
#pragma unroll
              for (int v = 0; v < V; ++v) f[v] = (float)((int32_t)(q << (28 - 4 * v)) >> 28);
            } else if (RB == 8) {
              const uint2 q = *reinterpret_cast<const uint2 *>(dslot(s, m));
#pragma unroll
              for (int v = 0; v < V; ++v) f[v] = (float)(int8_t)((v < 4 ? q.x : q.y) >> (8 * (v & 3)));
            } else {
              unpack<T>(*reinterpret_cast<const uint4 *>(dslot(s, m)), f);
            }
#pragma unroll
            for (int v = 0; v < V; ++v) acc[m][v] = fmaf(a, f[v], acc[m][v]);
          }
        }
        stage_d(s, k + DD);
      }
    }
  }
  cp_async_wait<0>();

  // ---------------------------------------------------------------- D: partials, final sum
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    const int ch = tid + kT * m;
    if (ch < nch_d) {
      float4 *dst = reinterpret_cast<float4 *>(P.part + (size_t)c * d + (size_t)ch * V);
#pragma unroll
      for (int v = 0; v < V; v += 4) dst[v / 4] = make_float4(acc[m][v], acc[m][v + 1], acc[m][v + 2], acc[m][v + 3]);
    }
  }
  if (!cta_grid_sync(P, flag_s)) return;
  // the stage region is free again: C2's copies have all landed
  column_sums<1, 1>(P.part, d, G, reinterpret_cast<float4 *>(dstage), [&](int, int col, float4 v) {
    const float t4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float tot = t4[i];
      if (P.resid) tot = P.resid[col + i] + tot;
      P.y[col + i] = tot;
      if (P.xnext) static_cast<T *>(P.xnext)[col + i] = from_f<T>(tot);
    }
  });
}

__global__ void k_barrier_bump(uint64_t *count) { atomicAdd(reinterpret_cast<unsigned long long *>(count), 1ull); }

template <typename T, int ACT, int MAXM, typename R>
cudaError_t launch_t(const Decode1Params &P, size_t smem, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.G);
  cfg.blockDim = dim3(kT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  cfg.numAttrs = fused_launch_attrs(attr, pdl);
  return cudaLaunchKernelEx(&cfg, k_decode1<T, ACT, MAXM, R>, P);
}

template <typename T, int ACT, typename R>
const void *pick_kernel(int nch) {
  if (nch <= kT) return (const void *)k_decode1<T, ACT, 1, R>;
  if (nch <= 2 * kT) return (const void *)k_decode1<T, ACT, 2, R>;
  return (const void *)k_decode1<T, ACT, 4, R>;
}

template <typename T, int ACT, typename R>
cudaError_t launch_act(const Decode1Params &P, size_t smem, cudaStream_t stream, bool pdl) {
  const int nch = P.d / Elem<T>::kVec;
  if (nch <= kT) return launch_t<T, ACT, 1, R>(P, smem, stream, pdl);
  if (nch <= 2 * kT) return launch_t<T, ACT, 2, R>(P, smem, stream, pdl);
  return launch_t<T, ACT, 4, R>(P, smem, stream, pdl);
}

template <typename T, int ACT, typename R>
cudaError_t config_act() {
  const void *ks[] = {(const void *)k_decode1<T, ACT, 1, R>, (const void *)k_decode1<T, ACT, 2, R>,
                      (const void *)k_decode1<T, ACT, 4, R>};
  for (const void *k : ks) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCap);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The kernel for this plan: element types (fp32, fp16, or fp16 with int8 / int4 rows) and activation.
const void *plan_kernel(const Decode1Params &P, int nch) {
  if (P.dt != SFNN_F16)
    return P.act == SFNN_REGLU ? pick_kernel<float, SFNN_REGLU, float>(nch) : pick_kernel<float, SFNN_RELU, float>(nch);
  if (P.rq == 8)
    return P.act == SFNN_REGLU ? pick_kernel<__half, SFNN_REGLU, Q8>(nch) : pick_kernel<__half, SFNN_RELU, Q8>(nch);
  if (P.rq == 4)
    return P.act == SFNN_REGLU ? pick_kernel<__half, SFNN_REGLU, Q4>(nch) : pick_kernel<__half, SFNN_RELU, Q4>(nch);
  return P.act == SFNN_REGLU ? pick_kernel<__half, SFNN_REGLU, __half>(nch)
                             : pick_kernel<__half, SFNN_RELU, __half>(nch);
}

}  // namespace

cudaError_t configure_decode1() {
  cudaError_t e = config_act<float, SFNN_RELU, float>();
  if (e == cudaSuccess) e = config_act<float, SFNN_REGLU, float>();
  if (e == cudaSuccess) e = config_act<__half, SFNN_RELU, __half>();
  if (e == cudaSuccess) e = config_act<__half, SFNN_REGLU, __half>();
  if (e == cudaSuccess) e = config_act<__half, SFNN_RELU, Q8>();
  if (e == cudaSuccess) e = config_act<__half, SFNN_REGLU, Q8>();
  if (e == cudaSuccess) e = config_act<__half, SFNN_RELU, Q4>();
  if (e == cudaSuccess) e = config_act<__half, SFNN_REGLU, Q4>();
  return e;
}

int decode1_blocks_per_sm(const Decode1Params &P) {
  const size_t smem = decode1_layout(P, true).total;
  if (smem > (size_t)kSmemCap) return 0;
  const int nch = P.d / (P.dt == SFNN_F16 ? 8 : 4);
  if (nch > 4 * kT) return 0;  // beyond the kernel's register plan
  const void *k = plan_kernel(P, nch);
  int blocks = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, k, kT, smem) != cudaSuccess) return 0;
  return blocks;
}

cudaError_t launch_barrier_bump(uint64_t *count, cudaStream_t stream) {
  k_barrier_bump<<<1, 1, 0, stream>>>(count);
  return cudaGetLastError();
}

cudaError_t launch_decode1(const Decode1Params &P, cudaStream_t stream, bool pdl) {
  const size_t smem = decode1_layout(P, true).total;
  if (P.dt != SFNN_F16)
    return P.act == SFNN_REGLU ? launch_act<float, SFNN_REGLU, float>(P, smem, stream, pdl)
                               : launch_act<float, SFNN_RELU, float>(P, smem, stream, pdl);
  if (P.rq == 8)
    return P.act == SFNN_REGLU ? launch_act<__half, SFNN_REGLU, Q8>(P, smem, stream, pdl)
                               : launch_act<__half, SFNN_RELU, Q8>(P, smem, stream, pdl);
  if (P.rq == 4)
    return P.act == SFNN_REGLU ? launch_act<__half, SFNN_REGLU, Q4>(P, smem, stream, pdl)
                               : launch_act<__half, SFNN_RELU, Q4>(P, smem, stream, pdl);
  return P.act == SFNN_REGLU ? launch_act<__half, SFNN_REGLU, __half>(P, smem, stream, pdl)
                             : launch_act<__half, SFNN_RELU, __half>(P, smem, stream, pdl);
}

}  // namespace sfnn
