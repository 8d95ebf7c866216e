// decode1.cu -- the fused single-token decode kernel (batch 1): one launch per token.
//
// Decode is bound by reading weights, not by arithmetic (53ai.com "sparsity for LLM
// inference" page, its opening analysis of decode latency: the I/O of loading
// parameters dominates token generation), so this kernel is organised around keeping
// HBM busy from the first cycle to the last:
//
//   grid: one persistent CTA per SM (G CTAs).  CTA c owns a contiguous tile of
//   neurons; the storage order deals hotness ranks round-robin to the tiles, so every
//   tile holds the same mix of hot and cold neurons (equal expected work), hottest
//   first inside the tile.
//
//   warp 8 (producer, one thread) streams everything the CTA reads through a ring of
//   S shared-memory stages with 1-D bulk async copies (TMA engine, cp.async.bulk,
//   mbarrier completion): first the tile's rows of the predictor's B^T (no dependence
//   on x, so they are in flight while the hidden layer is computed), then, as soon as
//   the consumers have decided a chunk of neurons, the [gate|up|down] record of every
//   active neuron of that chunk.  Inactive neurons' records are never requested.
//
//   warps 0-7 (consumers):
//     P1  h_j = relu(A^T[j] . x) for the CTA's share of the r predictor rows (one warp
//         per row, 128-bit loads), written to global; grid barrier.
//     P2  per B^T chunk: z_i = B^T[i] . h + c_i, one warp per neuron; neuron i is
//         active iff z_i > 0 (sigmoid(z) > 0.5); decisions go to a shared bit set the
//         producer reads.
//     P3  per active record: the up (and gate) dot products split over all 256
//         threads and summed in a fixed order, ReLU / ReGLU, then the axpy of the
//         neuron's contiguous W_down row into per-thread column accumulators.
//     P4  the CTA's partial y goes to global; grid barrier; CTA c sums a column slice
//         of all G partials in a fixed order (two-phase, deterministic) -> y
//         (+ residual, + rounded next-layer input).
//
// PDL: the kernel lets the next kernel in the stream launch at once and reads x, and
// writes anything, only after griddepcontrol.wait; weights are read before it.
// Every wait is bounded; on a timeout the kernel latches SFNN_ERR_TIMEOUT, lets its
// copies in flight land, and returns.
#include "async.cuh"
#include "common.cuh"
#include "decode1.cuh"

namespace sfnn {
namespace {

constexpr int kCW = 8;                 // consumer warps
constexpr int kConsumers = kCW * 32;   // consumer threads
constexpr int kThreads1 = kConsumers + 32;
constexpr uint64_t kWaitNs = 1000000000ull;  // every wait gives up after 1 s
enum : int { kItemBt = 0, kItemRow = 1, kItemEnd = 2 };

struct Smem {
  unsigned char *ring;
  unsigned char *x;
  float *h, *bias, *c, *red, *red2;
  uint32_t *bits;
  int *decided;
  int4 *desc;
  uint64_t *full, *empty, *xbar, *sync;
  int *abort_flag;
};

__device__ Smem carve(unsigned char *base, const Decode1Params &P) {
  Decode1Layout l = decode1_layout(P);
  Smem s;
  s.ring = base;
  s.x = base + l.x;
  s.h = reinterpret_cast<float *>(base + l.h);
  s.bias = reinterpret_cast<float *>(base + l.bias);
  s.c = reinterpret_cast<float *>(base + l.c);
  s.red = reinterpret_cast<float *>(base + l.red);
  s.red2 = reinterpret_cast<float *>(base + l.red2);
  s.bits = reinterpret_cast<uint32_t *>(base + l.bits);
  s.decided = reinterpret_cast<int *>(base + l.decided);
  s.desc = reinterpret_cast<int4 *>(base + l.desc);
  s.full = reinterpret_cast<uint64_t *>(base + l.bars);
  s.empty = s.full + P.S;
  s.xbar = s.empty + P.S;
  s.sync = s.xbar + 1;
  s.abort_flag = reinterpret_cast<int *>(s.sync + 1);
  return s;
}

__device__ __forceinline__ bool aborted(const Smem &s) { return *reinterpret_cast<volatile int *>(s.abort_flag); }

__device__ __forceinline__ void do_abort(const Smem &s, int32_t *err) {
  *reinterpret_cast<volatile int *>(s.abort_flag) = 1;
  latch_error(err, kErrTimeout);
}

// Bounded wait that also gives up as soon as another thread of the CTA aborted.
__device__ __forceinline__ bool wait_bar(const Smem &s, uint64_t *bar, uint32_t parity) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 63) {
      if (aborted(s)) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0)
        t0 = now;
      else if (now - t0 > kWaitNs)
        return false;
    }
  }
}

// All consumer warps meet (mbarrier with kCW arrivals, bounded).
__device__ __forceinline__ bool consumers_sync(const Smem &s, uint32_t &phase, int32_t *err) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(s.sync);
  const bool ok = wait_bar(s, s.sync, phase & 1u);
  ++phase;
  if (!ok) do_abort(s, err);
  return ok;
}

template <typename T>
__device__ __forceinline__ void load_vec_smem(const void *p, float *f) {
  unpack<T>(*reinterpret_cast<const uint4 *>(p), f);
}

template <typename T, int ACT, int MAXM>
__global__ void __launch_bounds__(kThreads1, 1) k_decode1(const Decode1Params P) {
  constexpr int V = Elem<T>::kVec;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const Smem s = carve(smem_raw, P);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = P.G;
  const int t0 = decode1_tile_start(c, P.n, G);
  const int tn = decode1_tile_start(c + 1, P.n, G) - t0;
  const int nchunks = (tn + P.NPC - 1) / P.NPC;
  const int nproj = P.nproj, d = P.d, r = P.r;
  const T *rows = static_cast<const T *>(P.rows);

  if (tid == 0) {
    for (int i = 0; i < P.S; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kCW);
    }
    mbar_init(s.xbar, 1);
    mbar_init(s.sync, kCW);
    *s.abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < (P.tile_max + 31) / 32; i += blockDim.x) s.bits[i] = 0u;
  for (int i = tid; i < P.chunks_max; i += blockDim.x) s.decided[i] = 0;
  __syncthreads();
  pdl_launch_dependents();

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    const T *Bt = static_cast<const T *>(P.Bt);
    const uint32_t rec_bytes = (uint32_t)(nproj * d * sizeof(T));
    int seq = 0, next_chunk = 0, dec = 0, cursor = 0;
    int last_item_bytes[64];  // per slot: bytes of the last item issued there (for the abort drain)
    for (int i = 0; i < P.S; ++i) last_item_bytes[i] = 0;
    bool x_issued = false, ok = true;
    uint64_t idle_since = 0;
    while (ok) {
      // the input vector, once the previous kernel's writes are visible
      if (!x_issued && (next_chunk >= P.S || next_chunk >= nchunks)) {
        pdl_wait();
        mbar_arrive_expect_tx(s.xbar, (uint32_t)(d * sizeof(T)));
        bulk_g2s(s.x, P.x, (uint32_t)(d * sizeof(T)), s.xbar);
        x_issued = true;
      }
      while (dec < next_chunk && *reinterpret_cast<volatile int *>(&s.decided[dec]) == kCW) ++dec;
      __threadfence_block();
      const int decided_upto = min(tn, dec * P.NPC);
      // next active neuron among the decided positions; every position below `cursor`
      // is decided and scanned
      int p = -1;
      while (cursor < decided_upto) {
        const uint32_t w = *reinterpret_cast<volatile uint32_t *>(&s.bits[cursor >> 5]) >> (cursor & 31);
        if (w) {
          const int q = cursor + __ffs(w) - 1;
          if (q < decided_upto)
            p = q;
          else
            cursor = decided_upto;
          break;
        }
        cursor = min((cursor | 31) + 1, decided_upto);
      }
      int4 item;
      uint32_t bytes = 0;
      const void *src = nullptr;
      if (p >= 0) {
        item = make_int4(kItemRow, p, 1, 0);
        bytes = rec_bytes;
        src = rows + (size_t)(t0 + p) * nproj * d;
        cursor = p + 1;
      } else if (next_chunk < nchunks) {
        const int p0 = next_chunk * P.NPC;
        const int cnt = min(P.NPC, tn - p0);
        item = make_int4(kItemBt, p0, cnt, next_chunk);
        bytes = (uint32_t)(cnt * r * sizeof(T));
        src = Bt + (size_t)(t0 + p0) * r;
        ++next_chunk;
      } else if (dec == nchunks && cursor >= decided_upto) {
        item = make_int4(kItemEnd, 0, 0, 0);
      } else {  // rows not decided yet: wait for the consumers
        const uint64_t now = globaltimer_ns();
        if (idle_since == 0) idle_since = now;
        if (now - idle_since > kWaitNs || aborted(s)) {
          ok = false;
          break;
        }
        __nanosleep(32);
        continue;
      }
      idle_since = 0;
      const int slot = seq % P.S;
      if (seq >= P.S && !wait_bar(s, &s.empty[slot], (uint32_t)((seq / P.S) - 1) & 1u)) {
        ok = false;
        break;
      }
      s.desc[slot] = item;
      if (bytes) {
        mbar_arrive_expect_tx(&s.full[slot], bytes);
        bulk_g2s(s.ring + (size_t)slot * P.SB, src, bytes, &s.full[slot]);
      } else {
        mbar_arrive(&s.full[slot]);
      }
      last_item_bytes[slot] = (int)bytes;
      ++seq;
      if (item.x == kItemEnd) break;
    }
    if (!x_issued) {  // keep the x barrier consistent even on the abort path
      pdl_wait();
      mbar_arrive_expect_tx(s.xbar, (uint32_t)(d * sizeof(T)));
      bulk_g2s(s.x, P.x, (uint32_t)(d * sizeof(T)), s.xbar);
    }
    if (!ok) {
      do_abort(s, P.err);
      // let every copy in flight land before the CTA's shared memory is released
      for (int k = seq - 1; k >= 0 && k >= seq - P.S; --k) {
        const int slot = k % P.S;
        if (last_item_bytes[slot]) mbar_wait(&s.full[slot], (uint32_t)(k / P.S) & 1u, kWaitNs);
      }
      mbar_wait(s.xbar, 0, kWaitNs);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  uint32_t sync_phase = 0;
  const T *At = static_cast<const T *>(P.At);
  const T *biasp = static_cast<const T *>(P.bias);
  const T *cp = static_cast<const T *>(P.cvec);
  for (int i = tid; i < tn; i += kConsumers) {
    s.bias[i] = to_f<T>(biasp[t0 + i]);
    s.c[i] = to_f<T>(cp[t0 + i]);
  }
  // P1: predictor hidden layer, rows j = c + G*(warp + kCW*k).  The weight loads are
  // issued before waiting for x.
  const int nch_d = d / V;
  bool ok = true, x_ready = false;
  for (int j = c + G * warp; ok && j < r; j += G * kCW) {
    const T *row = At + (size_t)j * d;
    float acc = 0.f;
    for (int cb = 0; cb < nch_d; cb += 32 * 16) {
      uint4 w[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int ch = cb + lane + 32 * u;
        if (ch < nch_d) w[u] = ld_stream(row + (size_t)ch * V);
      }
      if (!x_ready) {
        ok = wait_bar(s, s.xbar, 0);
        x_ready = true;
        if (!ok) {
          do_abort(s, P.err);
          break;
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int ch = cb + lane + 32 * u;
        if (ch < nch_d) {
          float wf[V], xf[V];
          unpack<T>(w[u], wf);
          load_vec_smem<T>(s.x + (size_t)ch * 16, xf);
#pragma unroll
          for (int v = 0; v < V; ++v) acc = fmaf(wf[v], xf[v], acc);
        }
      }
    }
    if (!ok) break;
    const float hs = warp_sum(acc);
    if (lane == 0) P.hbuf[j] = hs > 0.f ? hs : 0.f;  // NaN -> 0
  }
  if (ok && !x_ready) {
    ok = wait_bar(s, s.xbar, 0);
    if (!ok) do_abort(s, P.err);
  }
  __threadfence();
  ok = ok && consumers_sync(s, sync_phase, P.err);
  if (ok && tid == 0 && !grid_barrier(P.bar, (uint32_t)G, kWaitNs)) do_abort(s, P.err);
  ok = ok && consumers_sync(s, sync_phase, P.err) && !aborted(s);
  for (int i = tid; ok && i < r; i += kConsumers) s.h[i] = __ldcg(P.hbuf + i);
  ok = ok && consumers_sync(s, sync_phase, P.err);

  // P2 + P3: the stage loop
  float acc[MAXM][V];
#pragma unroll
  for (int m = 0; m < MAXM; ++m)
#pragma unroll
    for (int v = 0; v < V; ++v) acc[m][v] = 0.f;
  const int nch_r = r / V;
  int buf = 0;
  for (int seq = 0; ok; ++seq) {
    const int slot = seq % P.S;
    if (!wait_bar(s, &s.full[slot], (uint32_t)(seq / P.S) & 1u)) {
      do_abort(s, P.err);
      ok = false;
      break;
    }
    const int4 item = s.desc[slot];
    if (item.x == kItemEnd) break;
    const unsigned char *st = s.ring + (size_t)slot * P.SB;
    if (item.x == kItemBt) {
      for (int k = warp; k < item.z; k += kCW) {
        const unsigned char *brow = st + (size_t)k * r * sizeof(T);
        float a = 0.f;
#pragma unroll 4
        for (int ch = lane; ch < nch_r; ch += 32) {
          float wf[V];
          load_vec_smem<T>(brow + (size_t)ch * 16, wf);
          const float *hp = s.h + (size_t)ch * V;
#pragma unroll
          for (int v = 0; v < V; ++v) a = fmaf(wf[v], hp[v], a);
        }
        const int p = item.y + k;
        const float z = warp_sum(a) + s.c[p];
        if (lane == 0 && z > 0.f) atomicOr(&s.bits[p >> 5], 1u << (p & 31));  // NaN -> inactive
      }
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        atomicAdd(&s.decided[item.w], 1);
        mbar_arrive(&s.empty[slot]);
      }
      continue;
    }
    // a row record: [gate | up | down]
    const unsigned char *gate = st;
    const unsigned char *up = st + (ACT == SFNN_REGLU ? (size_t)d * sizeof(T) : 0);
    const unsigned char *down = st + (size_t)(nproj - 1) * d * sizeof(T);
    float su = 0.f, sg = 0.f;
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int ch = tid + kConsumers * m;
      if (ch < nch_d) {
        float xf[V], wu[V];
        load_vec_smem<T>(s.x + (size_t)ch * 16, xf);
        load_vec_smem<T>(up + (size_t)ch * 16, wu);
#pragma unroll
        for (int v = 0; v < V; ++v) su = fmaf(wu[v], xf[v], su);
        if (ACT == SFNN_REGLU) {
          float wg[V];
          load_vec_smem<T>(gate + (size_t)ch * 16, wg);
#pragma unroll
          for (int v = 0; v < V; ++v) sg = fmaf(wg[v], xf[v], sg);
        }
      }
    }
    su = warp_sum(su);
    if (ACT == SFNN_REGLU) sg = warp_sum(sg);
    if (lane == 0) {
      s.red[(buf * kCW + warp) * 2 + 0] = su;
      s.red[(buf * kCW + warp) * 2 + 1] = sg;
    }
    if (!consumers_sync(s, sync_phase, P.err)) {
      ok = false;
      break;
    }
    float tu = 0.f, tg = 0.f;
#pragma unroll
    for (int w = 0; w < kCW; ++w) {
      tu += s.red[(buf * kCW + w) * 2 + 0];
      tg += s.red[(buf * kCW + w) * 2 + 1];
    }
    const float bval = s.bias[item.y];
    float a;
    if (ACT == SFNN_RELU) {
      const float g = tu + bval;
      a = g > 0.f ? g : 0.f;
    } else {
      const float g = tg + bval;
      a = (g > 0.f ? g : 0.f) * tu;
    }
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int ch = tid + kConsumers * m;
      if (ch < nch_d) {
        float wd[V];
        load_vec_smem<T>(down + (size_t)ch * 16, wd);
#pragma unroll
        for (int v = 0; v < V; ++v) acc[m][v] = fmaf(a, wd[v], acc[m][v]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[slot]);
    buf ^= 1;
  }

  // P4: the CTA's partial, then the fixed-order column sums of all partials
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    const int ch = tid + kConsumers * m;
    if (ch < nch_d) {
      float4 *dst = reinterpret_cast<float4 *>(P.part + (size_t)c * d + (size_t)ch * V);
#pragma unroll
      for (int v = 0; v < V; v += 4) dst[v / 4] = make_float4(acc[m][v], acc[m][v + 1], acc[m][v + 2], acc[m][v + 3]);
    }
  }
  __threadfence();
  ok = ok && consumers_sync(s, sync_phase, P.err);
  if (ok && tid == 0 && !grid_barrier(P.bar, (uint32_t)G, kWaitNs)) do_abort(s, P.err);
  ok = ok && consumers_sync(s, sync_phase, P.err) && !aborted(s);
  if (!ok) return;
  const int CW = (d + G - 1) / G;
  const int col0 = c * CW;
  const int ncol = max(0, min(CW, d - col0));
  for (int cb = 0; cb < ncol; cb += kConsumers) {
    const int width = min(kConsumers, ncol - cb);
    const int gi = tid / width, j = tid % width;
    const int ngu = kConsumers / width;  // groups of partials summed in parallel
    if (gi < ngu) {
      const int k0 = (int)(((int64_t)gi * G) / ngu), k1 = (int)(((int64_t)(gi + 1) * G) / ngu);
      const float *src = P.part + col0 + cb + j;
      float sum = 0.f;
      for (int k = k0; k < k1; ++k) sum += __ldcg(src + (size_t)k * d);
      s.red2[gi * width + j] = sum;
    }
    if (!consumers_sync(s, sync_phase, P.err)) return;
    if (tid < width) {
      float tot = 0.f;
      for (int g = 0; g < ngu; ++g) tot += s.red2[g * width + tid];
      const int col = col0 + cb + tid;
      if (P.resid) tot = P.resid[col] + tot;
      P.y[col] = tot;
      if (P.xnext) static_cast<T *>(P.xnext)[col] = from_f<T>(tot);
    }
    if (!consumers_sync(s, sync_phase, P.err)) return;
  }
}

template <typename T, int ACT, int MAXM>
cudaError_t launch_t(const Decode1Params &P, size_t smem, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.G);
  cfg.blockDim = dim3(kThreads1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_decode1<T, ACT, MAXM>, P);
}

template <typename T, int ACT>
cudaError_t launch_act(const Decode1Params &P, size_t smem, cudaStream_t stream, bool pdl) {
  const int nch = P.d / Elem<T>::kVec;
  if (nch <= kConsumers * 4) return launch_t<T, ACT, 4>(P, smem, stream, pdl);
  return launch_t<T, ACT, 8>(P, smem, stream, pdl);
}

template <typename T, int ACT, int MAXM>
cudaError_t config_t() {
  return cudaFuncSetAttribute((const void *)k_decode1<T, ACT, MAXM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kDecode1SmemMax);
}

}  // namespace

cudaError_t configure_decode1() {
  cudaError_t e = config_t<float, SFNN_RELU, 4>();
  if (e == cudaSuccess) e = config_t<float, SFNN_RELU, 8>();
  if (e == cudaSuccess) e = config_t<float, SFNN_REGLU, 4>();
  if (e == cudaSuccess) e = config_t<float, SFNN_REGLU, 8>();
  if (e == cudaSuccess) e = config_t<__half, SFNN_RELU, 4>();
  if (e == cudaSuccess) e = config_t<__half, SFNN_RELU, 8>();
  if (e == cudaSuccess) e = config_t<__half, SFNN_REGLU, 4>();
  if (e == cudaSuccess) e = config_t<__half, SFNN_REGLU, 8>();
  return e;
}

int decode1_threads() { return kThreads1; }

int decode1_blocks_per_sm(const Decode1Params &P) {
  const size_t smem = decode1_layout(P).total;
  const int nch = P.d / (P.dt == SFNN_F16 ? 8 : 4);
  const bool m8 = nch > kConsumers * 4;
  const void *k;
  if (P.dt == SFNN_F16)
    k = P.act == SFNN_REGLU ? (m8 ? (const void *)k_decode1<__half, SFNN_REGLU, 8> : (const void *)k_decode1<__half, SFNN_REGLU, 4>)
                            : (m8 ? (const void *)k_decode1<__half, SFNN_RELU, 8> : (const void *)k_decode1<__half, SFNN_RELU, 4>);
  else
    k = P.act == SFNN_REGLU ? (m8 ? (const void *)k_decode1<float, SFNN_REGLU, 8> : (const void *)k_decode1<float, SFNN_REGLU, 4>)
                            : (m8 ? (const void *)k_decode1<float, SFNN_RELU, 8> : (const void *)k_decode1<float, SFNN_RELU, 4>);
  int blocks = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, k, kThreads1, smem) != cudaSuccess) return 0;
  return blocks;
}

cudaError_t launch_decode1(const Decode1Params &P, cudaStream_t stream, bool pdl) {
  const size_t smem = decode1_layout(P).total;
  if (P.dt == SFNN_F16)
    return P.act == SFNN_REGLU ? launch_act<__half, SFNN_REGLU>(P, smem, stream, pdl)
                               : launch_act<__half, SFNN_RELU>(P, smem, stream, pdl);
  return P.act == SFNN_REGLU ? launch_act<float, SFNN_REGLU>(P, smem, stream, pdl)
                             : launch_act<float, SFNN_RELU>(P, smem, stream, pdl);
}

}  // namespace sfnn
