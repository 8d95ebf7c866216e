// decode_ahead.cu -- the fused decode kernel of a residual stack whose active sets are
// predicted one layer ahead.
//
// DejaVu's predictor runs asynchronously: the next layer's sparsity is predicted one
// step in advance, so the prediction does not sit in front of the layer that uses it
// (53ai.com "sparsity for LLM inference" page, section "如何推理加速").  Here layer
// l+1's predictor takes layer l's input u_l, which lets one launch per layer carry both
// halves (one CTA of 16 warps per SM, as the single-layer kernel):
//
//   P1  u_l, and the active lists of layer l (written by the previous launch), into
//       shared memory; C1 / C2 on the CTA's share of layer l's active rows, as in the
//       single-layer kernel; h' = relu(A'^T u_l) for the CTA's rows of layer l+1's A'
//       (one warp per row, its first batch requested during C2: h' is needed only after
//       the barrier, while C1 needs only the lists); the CTA's partial y to global
//       memory; the first B'^T rows of layer l+1's tile requested into the staging
//       region C2 has left, after the barrier's arrival.
//   grid barrier (the launch's only one)
//   P2  the fixed-order column reduce of the partials -> y_l (+ residual), u_{l+1};
//       z' = B'^T h' + c' on layer l+1's tile -> its active list, kept in global memory
//       for the next launch.
//
// Against the single-layer kernel, each layer drops one grid barrier and the hidden
// layer's phase from its critical chain, and the column reduce overlaps the logits.
// Because all of a layer's lists are in global memory before its launch starts, the
// active rows need not stay with the tile that predicted them: every CTA takes an equal
// share (its own tile's rows up to the share, then rows the fuller tiles leave over),
// which removes the busiest tile's surplus from the critical path at the cost of one
// dependent load.  The stack's first launch runs the predictor half only (layer 0 on
// u_0); its last launch has no next predictor.  Its predictor sums each row of A'^T in
// one warp (the single-token kernel splits rows over two warps), so the two kernels' sums
// may differ in rounding.
#include "async.cuh"
#include "common.cuh"
#include "decode1.cuh"
#include "decode_dev.cuh"

namespace sfnn {
namespace {

template <typename T, int ACT, int MAXM, typename R>
__global__ void __launch_bounds__(kT, 1) k_decode_ahead(const Decode1Params P, const AheadParams Q) {
  constexpr int V = Elem<T>::kVec;
  constexpr int RB = RowFmt<R>::kBits;  // bits of a stored row element
  constexpr bool QR = RB <= 8;           // rows are codes with per-row scales
  constexpr int VR = 128 / RB;           // row elements per 16-byte chunk
  constexpr int MAXH = 4;              // chunks of h' per lane (r <= 128 * V)
  const int DB = min(P.bstages, kDecode1BStages);  // B'^T rows staged per warp: 1, 2, 3 or 4
  constexpr int DD = decode1_dstages(MAXM);
  extern __shared__ __align__(16) unsigned char smem[];
  const Decode1Layout L = decode_ahead_layout(P, Q);
  unsigned char *xs = smem + L.x;
  float *bias_s = reinterpret_cast<float *>(smem + L.bias);  // b of this layer's active rows
  float *c_s = reinterpret_cast<float *>(smem + L.c);        // c' of the next layer's tile
  int *act_s = reinterpret_cast<int *>(smem + L.act);
  float *a_s = reinterpret_cast<float *>(smem + L.a);  // activations, then b' of the next tile
  float *dots = reinterpret_cast<float *>(smem + L.dots);
  float *red2 = reinterpret_cast<float *>(smem + L.red2);
  uint32_t *bits = reinterpret_cast<uint32_t *>(smem + L.bits);
  int *wpref = reinterpret_cast<int *>(smem + L.wpref);
  float *h_s = reinterpret_cast<float *>(smem + L.h);
  int *cnt_s = reinterpret_cast<int *>(smem + L.bars);
  int *flag_s = cnt_s + 1;
  int *ncnt_s = cnt_s + 2;
  unsigned long long *target_s = reinterpret_cast<unsigned long long *>(cnt_s + 4);  // the barrier's target
  int *next_s = cnt_s + 6;  // C1's next work item
  int *ext_s = cnt_s + 7;   // C1's final row count once known (-1: not yet)
  unsigned char *bstage = smem + L.bstage;
  unsigned char *dstage = smem + L.dstage;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = P.G;
  const bool cur = Q.list_in != nullptr, next = Q.At != nullptr;
  const int t0 = decode1_tile_start(c, P.n, G);  // this layer's tile
  const int tn = decode1_tile_start(c + 1, P.n, G) - t0;
  const int u0 = decode1_tile_start(c, Q.n, G);  // the next layer's tile
  const int un = next ? decode1_tile_start(c + 1, Q.n, G) - u0 : 0;
  const int d = P.d, r = Q.r, nproj = P.nproj;
  const int nch_d = d / V, nch_r = next ? r / V : 0;
  const T *At = static_cast<const T *>(Q.At);
  const T *Bt = static_cast<const T *>(Q.Bt);
  const unsigned char *rows = static_cast<const unsigned char *>(P.rows);
  const size_t rowB = (size_t)P.d * RB / 8;  // bytes of one stored row

  pdl_launch_dependents();
  const int j0 = c + G * warp;  // this warp's first row of A'^T

  // Before griddepcontrol.wait only c', b' at tile position tid (weights); after it, u_l
  // and this layer's lists are requested first (they gate everything), then the first
  // batch of the warp's row of A'^T.
  const T *cp = static_cast<const T *>(Q.cvec);
  const T *bp = static_cast<const T *>(Q.bias);
  T c_first = from_f<T>(0.f), b_first = from_f<T>(0.f);
  if (tid < un) {
    c_first = cp[u0 + tid];
    b_first = bp[u0 + tid];
  }
  for (int i = tid; i < (Q.tile_max + 31) / 32; i += kT) bits[i] = 0u;
  if (tid == 0) {
    *next_s = 0;
    *ext_s = -1;
  }

  pdl_wait();  // u_l, this layer's lists and every buffer written here belong to earlier kernels until here
  uint4 xv[MAXM];
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    const int ch = tid + kT * m;
    if (ch < nch_d) xv[m] = __ldcg(reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(P.x) + (size_t)ch * 16));
  }
  int2 l_first = make_int2(0, 0);
  int c_tile = 0;
  if (cur && tid < tn) l_first = __ldcg(Q.list_in + t0 + tid);
  if (cur && tid < G) c_tile = __ldcg(Q.cnt_in + tid);
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    const int ch = tid + kT * m;
    if (ch < nch_d) *reinterpret_cast<uint4 *>(xs + (size_t)ch * 16) = xv[m];
  }
  // The active rows are shared out evenly: CTA c takes T_c = floor((c+1)K/G) - floor(cK/G)
  // of the layer's K rows, first o_c = min(cnt_c, T_c) of its own tile's, then f_c = T_c - o_c
  // of the rows the tiles with more than their share leave over (e_t = cnt_t - o_t each,
  // taken in tile order).  The assignment depends on the counts only: deterministic.
  int *cnt_all = reinterpret_cast<int *>(red2);  // [G] counts, [G + 1] prefix of e, o_c f_c F_c K
  int *epre = cnt_all + G;
  int *own = epre + G + 1;
  if (cur) {
    for (int i = tid; i < tn; i += kT) {  // the own tile's slots arrive with the counts
      const int2 e = i == tid ? l_first : __ldcg(Q.list_in + t0 + i);
      act_s[i] = e.x;
      bias_s[i] = __int_as_float(e.y);
    }
    for (int t = tid; t < G; t += kT) {
      const int sz = decode1_tile_start(t + 1, P.n, G) - decode1_tile_start(t, P.n, G);
      cnt_all[t] = min(max(t == tid ? c_tile : __ldcg(Q.cnt_in + t), 0), sz);
    }
  }
  __syncthreads();
  // every warp: the layer's row count K and this CTA's own rows o_c = min(cnt_c, T_c), with
  // floor(tK/G) = t q + floor(t rm / G), K = q G + rm (32-bit arithmetic)
  int K = 0, o_c = 0;
  if (cur) {
    int ks = 0;
    for (int t = lane; t < G; t += 32) ks += cnt_all[t];
    K = __reduce_add_sync(0xffffffffu, ks);
    const int q = K / G, rm = K - q * G;
    o_c = min(cnt_all[c], q + ((c + 1) * rm) / G - (c * rm) / G);
  }
  int cnt = o_c;  // this CTA's rows; the shared-out ones are appended during C1

  // C2's rows of W_down stream through DD shared-memory stages private to each thread
  auto dslot = [&](int s, int m) { return dstage + (((size_t)s * MAXM + m) * kT + tid) * 16; };
  auto stage_d = [&](int s, int k) {  // active row k into stage s; always one group
    if (k < cnt) {
      const unsigned char *row = rows + ((size_t)act_s[k] * nproj + (nproj - 1)) * rowB;
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        const int ch = tid + kT * m;
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
  float acc[MAXM][V];
#pragma unroll
  for (int m = 0; m < MAXM; ++m)
#pragma unroll
    for (int v = 0; v < V; ++v) acc[m][v] = 0.f;
  // The layer's own work comes first: C1 and C2 need only the lists, while the next
  // layer's A'^T rows are requested during C2 and summed after it (h' is needed only
  // after the grid barrier).
  uint4 w0[16];
  auto load_a = [&]() {  // the first batch of the warp's row of A'^T
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int ch = lane + 32 * u;
      if (j0 < r && ch < nch_d) w0[u] = ld_stream(At + (size_t)j0 * d + (size_t)ch * V);
    }
  };
  int cpre = 0;  // C2 stages requested during C1
  if (cur) {
    // -------------------------------------------------------------- C1: up / gate dots
    // The rows' 4 KB segments are work items handed out in order by a shared counter
    // (own rows first), loaded into registers; warp 0 meanwhile computes the share's
    // prefix, fetches the shared-out rows' entries and publishes the final count.
    constexpr int NPG = ACT == SFNN_REGLU ? 2 : 1;
    constexpr int SU = kSegChunks / 32;
    const int nseg = P.nseg;
    const int per_row = NPG * nseg;
    const int nch_r8 = d / VR;
    int lim = o_c * per_row;  // items known to exist
    bool known = false;
    uint4 wa[SU], wb[SU];
    auto grab = [&]() {
      int v = 0;
      if (lane == 0) v = atomicAdd(next_s, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    auto avail = [&](int it) {  // 1: item `it` exists, 0: past the end, -1: abandoned
      if (it < lim) return 1;
      if (known) return 0;
      int e = -1;  // the final count: wait for warp 0 to publish it (bounded)
      if (lane == 0) {
        const uint64_t tw = clock64();
        while ((e = *reinterpret_cast<volatile int *>(ext_s)) == -1)
          if ((uint64_t)(clock64() - tw) > 2 * kWaitCycles) {
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
      cnt = e;
      lim = e * per_row;
      return it < lim ? 1 : 0;
    };
    auto load_c = [&](uint4 *w, int it) {
      const int k = it / per_row, pj = (it % per_row) / nseg, sg = it % per_row - pj * nseg;
      const unsigned char *row = rows + ((size_t)act_s[k] * nproj + pj) * rowB;
#pragma unroll
      for (int u = 0; u < SU; ++u) {
        const int ch = sg * kSegChunks + lane + 32 * u;
        if (ch < nch_r8) w[u] = ld_stream(row + (size_t)ch * 16);
      }
    };
    auto sum_c = [&](const uint4 *w, int it) {
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
    const bool two = P.c1depth > 1;
    int ia = grab(), ib = two ? grab() : 0;
    int sa = ia < lim ? 1 : 2, sb = two ? (ib < lim ? 1 : 2) : 0;  // 2: not known yet
    if (sa == 1) load_c(wa, ia);
    if (sb == 1) load_c(wb, ib);
    cpre = min(DD, o_c);
#pragma unroll 1
    for (int s = 0; s < cpre; ++s) stage_d(s, s);
    if (warp == 0) {
      // Lane l walks the tiles [l tpl, (l + 1) tpl) in order, twice: once for its sums of
      // e_t and f_t, then (after a scan over the lanes) for epre[t] and this CTA's f, F.
      const int q = K / G, rm = K - q * G;
      const int tpl = (G + 31) / 32;
      const int tb = min(G, lane * tpl), te = min(G, tb + tpl);
      int es = 0, fs = 0;
      for (int t = tb, fl = (tb * rm) / G; t < te; ++t) {
        const int fh = ((t + 1) * rm) / G;
        const int share = q + fh - fl;
        fl = fh;
        const int o = min(cnt_all[t], share);
        es += cnt_all[t] - o;
        fs += share - o;
      }
      int ie = es, jf = fs;  // inclusive scans of the lanes' sums
#pragma unroll
      for (int sh = 1; sh < 32; sh <<= 1) {
        const int ye = __shfl_up_sync(0xffffffffu, ie, sh), yf = __shfl_up_sync(0xffffffffu, jf, sh);
        if (lane >= sh) {
          ie += ye;
          jf += yf;
        }
      }
      int be = ie - es, bf = jf - fs;
      for (int t = tb, fl = (tb * rm) / G; t < te; ++t) {
        const int fh = ((t + 1) * rm) / G;
        const int share = q + fh - fl;
        fl = fh;
        const int o = min(cnt_all[t], share);
        epre[t] = be;
        if (t == c) {
          own[1] = share - o;
          own[2] = bf;
        }
        be += cnt_all[t] - o;
        bf += share - o;
      }
      if (lane == 31) epre[G] = be;
      __syncwarp();
      // this CTA's excess row j is the layer's excess row g = F + j: tile t with
      // epre[t] <= g < epre[t + 1], slot o_t + g - epre[t] of that tile
      const int f_c = own[1], F_c = own[2];
      for (int j = lane; j < f_c; j += 32) {
        const int g = F_c + j;
        int lo = 0, hi = G;
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (epre[mid] <= g)
            lo = mid;
          else
            hi = mid;
        }
        const int share = q + ((lo + 1) * rm) / G - (lo * rm) / G;
        const int2 e = __ldcg(Q.list_in + decode1_tile_start(lo, P.n, G) + min(cnt_all[lo], share) + g - epre[lo]);
        act_s[o_c + j] = e.x;
        bias_s[o_c + j] = __int_as_float(e.y);
      }
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();  // the rows' entries before the count
        *reinterpret_cast<volatile int *>(ext_s) = o_c + f_c;
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
    if (sa < 0 || sb < 0) {  // abandoned (warp 0 always publishes: defensive)
      cp_async_wait<0>();
      return;
    }
    __syncthreads();
    for (int k = tid; k < cnt; k += kT) {
      float g = 0.f, u = 0.f;
      for (int sg = 0; sg < nseg; ++sg) g += dots[(k * 2 + 0) * nseg + sg];
      if (ACT == SFNN_REGLU)
        for (int sg = 0; sg < nseg; ++sg) u += dots[(k * 2 + 1) * nseg + sg];
      float sd = 1.f;
      if (QR) {
        const float *sc = P.rscale + (size_t)act_s[k] * nproj;
        g *= sc[0];
        if (ACT == SFNN_REGLU) u *= sc[1];
        sd = sc[nproj - 1];
      }
      const float pre = g + bias_s[k];
      const float relu = pre > 0.f ? pre : 0.f;
      a_s[k] = ACT == SFNN_RELU ? relu : relu * u;
      if (QR) a_s[k] *= sd;
    }
    __syncthreads();
#pragma unroll 1
    for (int s = cpre; s < DD; ++s) stage_d(s, s);  // the rest of C2's first stages
    if (next) load_a();  // lands during C2

    // -------------------------------------------------------------- C2: down projection
    for (int kb = 0; kb < cnt; kb += DD) {
#pragma unroll
      for (int s = 0; s < DD; ++s) {
        const int k = kb + s;
        if (k < cnt) {
          cp_async_wait<DD - 1>();
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
  } else if (next) {
    load_a();
  }

  // ---------------------------------------------------------------- A': next hidden layer
  if (next) {
    for (int j = j0; j < r; j += G * kW) {
      const T *row = At + (size_t)j * d;
      float acc1 = 0.f;  // one chain in ascending chunk order (the multi-kernel predictor's order)
      for (int cb = 0; cb < nch_d; cb += 32 * 16) {
        if (j != j0 || cb != 0) {
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int ch = cb + lane + 32 * u;
            if (ch < nch_d) w0[u] = ld_stream(row + (size_t)ch * V);
          }
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int ch = cb + lane + 32 * u;
          if (ch < nch_d) acc1 = dot_chunk_smem<T>(w0[u], xs, ch, acc1);
        }
      }
      const float hs = warp_sum(acc1);
      if (lane == 0) Q.hbuf[j] = hs > 0.f ? hs : 0.f;  // NaN -> 0
    }
  }
  __syncthreads();  // C2's stages and activations are consumed: the region takes B'^T rows

  // The next layer's B'^T rows stream through DB stages private to each warp, as in the
  // single-layer kernel; the first DB rows land during the partial write and the barrier.
  unsigned char *bst = bstage + (size_t)warp * DB * nch_r * 16;
  auto stage_b = [&](int s, int p) {  // row p of the next tile into stage s; always one group
    if (p < un) {
#pragma unroll
      for (int m = 0; m < MAXH; ++m) {
        const int ch = lane + 32 * m;
        if (ch < nch_r) cp_async16(bst + ((size_t)s * nch_r + ch) * 16, Bt + (size_t)(u0 + p) * r + (size_t)ch * V);
      }
    }
    cp_async_commit();
  };
  if (next) {
    if (tid < un) {
      c_s[tid] = to_f<T>(c_first);
      a_s[tid] = to_f<T>(b_first);
    }
    for (int i = tid + kT; i < un; i += kT) {
      c_s[i] = to_f<T>(cp[u0 + i]);
      a_s[i] = to_f<T>(bp[u0 + i]);
    }
  }
  if (cur) {
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int ch = tid + kT * m;
      if (ch < nch_d) {
        float4 *dst = reinterpret_cast<float4 *>(P.part + (size_t)c * d + (size_t)ch * V);
#pragma unroll
        for (int v = 0; v < V; v += 4) dst[v / 4] = make_float4(acc[m][v], acc[m][v + 1], acc[m][v + 2], acc[m][v + 3]);
      }
    }
  }
  cta_grid_arrive(P, target_s);
  // the first DB B'^T rows go out after the arrival (its release would otherwise wait for
  // them to land), and land during the barrier
  if (next) {
#pragma unroll 1
    for (int s = 0; s < DB; ++s) stage_b(s, warp + kW * s);
  }
  if (!cta_grid_wait(P, target_s, flag_s)) {
    cp_async_wait<0>();  // no copy into shared memory outlives the CTA
    return;
  }

  // ---------------------------------------------------------------- P2
  if (next)  // h' once per CTA from L2; its loads overlap the reduce's
    for (int i = tid; i < r / 4; i += kT)
      reinterpret_cast<float4 *>(h_s)[i] = __ldcg(reinterpret_cast<const float4 *>(Q.hbuf) + i);
  if (cur) {  // y_l: CTA c sums a column slice of all G partials in a fixed order
    const int CW = (d + G - 1) / G;
    const int col0 = c * CW;
    const int ncol = max(0, min(CW, d - col0));
    for (int cb = 0; cb < ncol; cb += kT) {
      const int width = min(kT, ncol - cb);
      const int gi = tid / width, j = tid % width;
      const int ngu = kT / width;
      if (gi < ngu) {
        const int k0 = (int)(((int64_t)gi * G) / ngu), k1 = (int)(((int64_t)(gi + 1) * G) / ngu);
        const float *src = P.part + col0 + cb + j;
        float sum = 0.f;  // in ascending k; the first 24 loads issued at once, then 8 at a time
        float v0[24];
#pragma unroll
        for (int u = 0; u < 24; ++u) v0[u] = k0 + u < k1 ? __ldcg(src + (size_t)(k0 + u) * d) : 0.f;
#pragma unroll
        for (int u = 0; u < 24; ++u)
          if (k0 + u < k1) sum += v0[u];
        int k = k0 + 24;
        for (; k + 8 <= k1; k += 8) {
          float v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (size_t)(k + u) * d);
#pragma unroll
          for (int u = 0; u < 8; ++u) sum += v[u];
        }
        for (; k < k1; ++k) sum += __ldcg(src + (size_t)k * d);
        red2[gi * width + j] = sum;
      }
      __syncthreads();
      if (tid < width) {
        float tot = 0.f;
        for (int g = 0; g < ngu; ++g) tot += red2[g * width + tid];
        const int col = col0 + cb + tid;
        if (P.resid) tot = P.resid[col] + tot;
        P.y[col] = tot;
        if (P.xnext) static_cast<T *>(P.xnext)[col] = from_f<T>(tot);
      }
      __syncthreads();
    }
  }
  if (!next) return;
  __syncthreads();

  // ---------------------------------------------------------------- B': next logits
  {
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
    for (int pb = warp; pb < un; pb += DB * kW) {
#pragma unroll 1
      for (int s = 0; s < DB; ++s) {
        const int p = pb + kW * s;
        if (p < un) {
          switch (DB) {  // this lane's copies of row p have landed
            case 1: cp_async_wait<0>(); break;
            case 2: cp_async_wait<1>(); break;
            case 3: cp_async_wait<2>(); break;
            default: cp_async_wait<3>(); break;
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
  // The next tile's active positions, ascending, with their biases -> the next launch
  const int nwords = (un + 31) / 32;
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
    if (lane == 0) *ncnt_s = base;
  }
  __syncthreads();
  for (int p = tid; p < un; p += kT) {
    const uint32_t word = bits[p >> 5], bit = 1u << (p & 31);
    if (word & bit) {
      const int k = wpref[p >> 5] + __popc(word & (bit - 1u));
      Q.list_out[u0 + k] = make_int2(u0 + p, __float_as_int(a_s[p]));
    }
  }
  if (tid == 0) Q.cnt_out[c] = *ncnt_s;
}

template <typename T, int ACT, int MAXM, typename R>
cudaError_t launch_t(const Decode1Params &P, const AheadParams &Q, size_t smem, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.G);
  cfg.blockDim = dim3(kT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  cfg.numAttrs = fused_launch_attrs(attr, pdl);
  return cudaLaunchKernelEx(&cfg, k_decode_ahead<T, ACT, MAXM, R>, P, Q);
}

template <typename T, int ACT, typename R>
cudaError_t launch_act(const Decode1Params &P, const AheadParams &Q, size_t smem, cudaStream_t stream, bool pdl) {
  const int nch = P.d / Elem<T>::kVec;
  if (nch <= kT) return launch_t<T, ACT, 1, R>(P, Q, smem, stream, pdl);
  if (nch <= 2 * kT) return launch_t<T, ACT, 2, R>(P, Q, smem, stream, pdl);
  return launch_t<T, ACT, 4, R>(P, Q, smem, stream, pdl);
}

template <typename T, int ACT, typename R>
cudaError_t config_act() {
  const void *ks[] = {(const void *)k_decode_ahead<T, ACT, 1, R>, (const void *)k_decode_ahead<T, ACT, 2, R>,
                      (const void *)k_decode_ahead<T, ACT, 4, R>};
  for (const void *k : ks) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCap);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t configure_decode_ahead() {
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

cudaError_t launch_decode_ahead(const Decode1Params &P, const AheadParams &Q, cudaStream_t stream, bool pdl) {
  const size_t smem = decode_ahead_layout(P, Q).total;
  if (smem > (size_t)kSmemCap || P.d / (P.dt == SFNN_F16 ? 8 : 4) > 4 * kT) return cudaErrorInvalidValue;
  if (P.dt != SFNN_F16)
    return P.act == SFNN_REGLU ? launch_act<float, SFNN_REGLU, float>(P, Q, smem, stream, pdl)
                               : launch_act<float, SFNN_RELU, float>(P, Q, smem, stream, pdl);
  if (P.rq == 8)
    return P.act == SFNN_REGLU ? launch_act<__half, SFNN_REGLU, Q8>(P, Q, smem, stream, pdl)
                               : launch_act<__half, SFNN_RELU, Q8>(P, Q, smem, stream, pdl);
  if (P.rq == 4)
    return P.act == SFNN_REGLU ? launch_act<__half, SFNN_REGLU, Q4>(P, Q, smem, stream, pdl)
                               : launch_act<__half, SFNN_RELU, Q4>(P, Q, smem, stream, pdl);
  return P.act == SFNN_REGLU ? launch_act<__half, SFNN_REGLU, __half>(P, Q, smem, stream, pdl)
                             : launch_act<__half, SFNN_RELU, __half>(P, Q, smem, stream, pdl);
}

}  // namespace sfnn
