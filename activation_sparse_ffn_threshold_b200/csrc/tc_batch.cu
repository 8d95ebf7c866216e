// tc_batch.cu -- the batched union FFN on the tensor cores (tcgen05, fp16 weights).
//
// With several tokens, the rows of the union of their sets are read once and serve every
// token (53ai.com "sparsity for LLM inference" page, section 工程效果: the union grows with
// the batch, so each row read is shared by more tokens).  At batch b the up (and gate)
// projection of a union row is b dot products and its down row feeds b outputs, so the
// work is a gathered GEMM whose arithmetic grows with b while its bytes stay the rows' ---
// at b = 32 CUDA cores fall behind HBM, tcgen05 does not.
//
//   k_tc_up    D[union row][token] = W_up[U] . X^T (and W_gate[U] . X^T): one CTA per 128
//              union rows; A = the gathered rows (K-major), B = the batch's x rows
//              (K-major), accumulators in TMEM.  Epilogue: + b, ReLU / ReGLU, zero for
//              the tokens whose set does not hold the row -> H[token][union] (fp16).
//   k_tc_down  Y^T[cols][token] = W_down[U]^T . H^T over a split of the union: A = the
//              gathered down rows, 128 (or 256) output columns each (MN-major: a row is
//              contiguous along d), B = H (K-major) -> part[split][token][cols]; k_reduce
//              adds the splits in a fixed order.
//   k_tc_hidden, k_tc_hsum, k_tc_logits  the predictor of the batch (dense GEMMs over
//              A^T and B^T), ending in the token-major decision masks k_compact reads.
//
// Operand tiles are 64 fp16 wide along K (one 128-byte swizzle row) and staged in shared
// memory with 16-byte cp.async copies (the rows are gathered by index), 128-byte
// swizzled, in the canonical layouts the MMA descriptors name.  Thread 0 issues the MMAs
// of a stage and commits them to the stage's mbarrier, which frees the stage for the copy
// of a later one.  Every wait is bounded: on a timeout the kernel latches
// SFNN_ERR_TIMEOUT, frees its tensor memory and returns.
#include <algorithm>

#include "async.cuh"
#include "common.cuh"
#include "launch.cuh"

namespace sfnn {
namespace {

constexpr int kTT = 128;  // threads per CTA (4 warps: warp w reads TMEM lanes 32w..32w+31)
constexpr int kTM = 128;  // MMA M
constexpr int kTK = 64;   // K of a stage: 64 fp16 = one 128-byte swizzle row
constexpr int kTmemCols = 64;

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void mb_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mb_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
// Wait for the phase with this parity; false after kWaitCycles.
__device__ __forceinline__ bool mb_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = clock64();
  for (;;) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((uint64_t)(clock64() - t0) > kWaitCycles) return false;
  }
}
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Make this thread's generic-proxy writes to shared memory visible to the MMA's reads.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[smem] . B[smem], one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  const uint32_t mask0 = 0, mask1 = 0, mask2 = 0, mask3 = 0;  // no output lane disabled
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(mask0), "r"(mask1), "r"(mask2),
      "r"(mask3)
      : "memory");
}
// The mbarrier gets one arrival once every MMA this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// 16 consecutive fp32 columns of this warp's 32 TMEM lanes (one lane per thread).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float v[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, 128-byte swizzle (the tile's 8-row atoms are
// 1024-byte aligned).  K-major: lbo unused (16), sbo = stride of 8-row groups.
// MN-major: lbo = stride of 64-element MN atoms, sbo = stride of 8-deep K groups.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: fp16 A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// Byte offset of 16-byte chunk c (0..7) of row `row` in a K-major 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t kmajor_off(int row, int c) {
  return (uint32_t)row * 128u + (uint32_t)((c ^ (row & 7)) << 4);
}

__device__ __forceinline__ void cp16(unsigned char *base, uint32_t off, const void *src) {
  cp_async16(base + off, src);
}

// ---------------------------------------------------------------- shared pipeline
// All threads: init the stage mbarriers, allocate tensor memory (warp 0), publish.
__device__ __forceinline__ uint32_t tc_begin(uint64_t *mbar, int stages, uint32_t *tmem_slot, int *fail) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) mb_init(&mbar[s], 1);
    mb_init_fence();
    *fail = 0;
  }
  if ((threadIdx.x >> 5) == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tmem_slot;
}
// All threads: release tensor memory once every read of it is done.
__device__ __forceinline__ void tc_end(uint32_t tmem) {
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) tmem_dealloc(tmem, kTmemCols);
}
// The K loop: `load(s, it, what)` copies iteration it's operands (`what`: kLoadA the
// weights, kLoadB the activations, kLoadAll both) into stage s (cp.async, all threads); `issue(stage_smem_addr, it)` issues its MMAs (thread 0), which are committed
// to the stage's mbarrier; the stage is refilled once they are done.  `base` counts the
// iterations this CTA ran in earlier calls (they fix the stage and mbarrier phase of
// each iteration).  Returns false if a wait ran out (then `fail` is set).  On return every
// MMA has completed (or failed) and the accumulators may be read after tc_fence_after.
constexpr int kLoadA = 1, kLoadB = 2, kLoadAll = 3;  // `load`'s operands: the weights, the activations
template <class Load, class Issue>
__device__ __forceinline__ bool tc_mainloop(unsigned char *smem, uint32_t stage_bytes, int stages, int nk,
                                            uint64_t *mbar, int *fail, Load load, Issue issue, int base = 0,
                                            int a_pre = 0) {
  const int tid = threadIdx.x;
  for (int s = 0; s < stages - 1; ++s) {  // a_pre: iterations whose weights were copied already
    if (s < nk) load((base + s) % stages, s, s < a_pre ? kLoadB : kLoadAll);
    cp_async_commit();
  }
  bool ok = true;
  for (int it = 0; it < nk && ok; ++it) {
    const int j = base + it, s = j % stages;
    // committed groups: stages - 1 + it; iteration it's is the (it + 1)-th oldest
    switch (stages) {
      case 2: cp_async_wait<0>(); break;
      case 3: cp_async_wait<1>(); break;
      default: cp_async_wait<2>(); break;
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      issue(smem_u32(smem + (size_t)s * stage_bytes), it);
      umma_commit(&mbar[s]);
    }
    const int nx = it + stages - 1;  // refill the stage iteration it - 1 read, once its MMAs are done
    if (nx < nk) {
      if (it >= 1 && !mb_wait(&mbar[(j - 1) % stages], (uint32_t)(((j - 1) / stages) & 1))) *fail = 1;
      load((base + nx) % stages, nx, kLoadAll);
    }
    cp_async_commit();
    __syncthreads();
    ok = *fail == 0;
  }
  cp_async_wait<0>();
  if (ok && nk > 0 && !mb_wait(&mbar[(base + nk - 1) % stages], (uint32_t)(((base + nk - 1) / stages) & 1)))
    *fail = 1;
  tc_fence_after();
  __syncthreads();
  return *fail == 0;
}

// ---------------------------------------------------------------- k_tc_up
// Stream-K: the union's 128-row tiles times their d/(64 kps) K steps are T iterations (a
// step stages kps 64-wide K chunks of every row: 128 kps contiguous bytes), and CTA
// g of G runs iterations [g T / G, (g + 1) T / G) -- so every SM stays busy however few
// tiles the union makes.  A CTA's range is cut at tile edges into segments.  A segment that
// is a whole tile ends in the epilogue; a part of a tile leaves its fp32 accumulators in
// upart (slot 2g for the CTA's first tile, 2g + 1 for its last) and counts itself in
// tcnt[tile]; the tile's last segment to arrive adds the tile's partials in CTA order
// (deterministic), runs the epilogue and zeroes the counter for the next launch.  No CTA
// waits for another.
// smem per stage: kps times (NP tiles of 128 rows (16 KB each) + the x tile (N rows x 128 B)).
template <int ACT>
__global__ void __launch_bounds__(kTT) k_tc_up(const __half *__restrict__ rows, const __half *__restrict__ bias,
                                               const __half *__restrict__ X, const int32_t *__restrict__ ulist,
                                               const uint32_t *__restrict__ utok, const int32_t *__restrict__ ucount,
                                               __half *__restrict__ H, int hstride, int d, int b, int N, int nproj,
                                               int stages, int kps, float *__restrict__ upart,
                                               int32_t *__restrict__ tcnt, int32_t *err) {
  constexpr int NP = ACT == SFNN_REGLU ? 2 : 1;  // projections with a dot: (gate,) up
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t mbar[8];
  __shared__ uint32_t tmem_slot;
  __shared__ int fail, last_s;
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();  // the union (the kernel before) is complete
  pdl_launch_dependents();
  const int U = *ucount;
  const int nk = d / (kTK * kps);  // K steps of a tile
  const int64_t T = (int64_t)((U + kTM - 1) / kTM) * nk;
  const int64_t G = T < (int64_t)gridDim.x ? T : (int64_t)gridDim.x;  // every range non-empty
  const int64_t g = blockIdx.x;
  if (g >= G) return;
  int64_t i0 = g * T / G;
  const int64_t i1 = (g + 1) * T / G;
  // the CTA whose range holds iteration i: the largest g' with g' T / G <= i
  auto cta_of = [&](int64_t i) { return ((i + 1) * G + T - 1) / T - 1; };
  const int first_tile = (int)(i0 / nk);
  const uint32_t chunk_bytes = NP * 16384u + (uint32_t)N * 128u;  // a multiple of 1024
  const uint32_t stage_bytes = (uint32_t)kps * chunk_bytes;
  const uint32_t tmem = tc_begin(mbar, stages, &tmem_slot, &fail);
  const uint32_t idesc = idesc_f16(kTM, N, 0, 0);
  const int c8 = tid & 7, row = warp * 32 + lane;
  const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
  bool ok = true;
  int base = 0;  // iterations run so far (stage and mbarrier phase of the next one)

  // bias + ReLU / ReGLU of this thread's row of tile m; zero for the tokens whose set
  // does not hold the row -> H[token][union] (fp16)
  auto epilogue = [&](int m, const float *gs, const float *us) {
    const int u = m * kTM + row;
    if (u < U) {
      const int p = ulist[u];
      const uint32_t tm = utok[u];
      const float bv = __half2float(bias[p]);
      for (int t = 0; t < N; ++t) {
        float a = 0.f;
        if (t < b && ((tm >> t) & 1u)) {
          const float pre = gs[t] + bv;
          a = pre > 0.f ? pre : 0.f;
          if (ACT == SFNN_REGLU) a *= us[t];
        }
        H[(size_t)t * hstride + u] = __float2half_rn(a);
      }
    } else if (u < hstride) {  // the union's padding up to the down GEMM's K chunks: zeros
      for (int t = 0; t < N; ++t) H[(size_t)t * hstride + u] = __float2half_rn(0.f);
    }
  };

  while (i0 < i1) {
    const int m = (int)(i0 / nk);
    const int k0 = (int)(i0 - (int64_t)m * nk);
    const int k1 = (int)(i1 - (int64_t)m * nk < nk ? i1 - (int64_t)m * nk : nk);
    const int u0 = m * kTM;
    // this thread's 8 rows of the tile (row = tid/8 + 16 i) and its 16-byte chunk (tid % 8)
    const __half *src[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int u = u0 + (tid >> 3) + 16 * i;
      u = u < U ? u : U - 1;  // the tile's tail repeats a row; its results are not stored
      src[i] = rows + (size_t)ulist[u] * nproj * d + c8 * 8;
    }
    auto load = [&](int s, int it, int) {
      for (int a = 0; a < kps; ++a) {
        const int kc = (k0 + it) * kps + a;
        unsigned char *st = smem + (size_t)s * stage_bytes + (size_t)a * chunk_bytes;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < NP; ++j)
            cp16(st + j * 16384, kmajor_off((tid >> 3) + 16 * i, c8), src[i] + (size_t)j * d + (size_t)kc * kTK);
        unsigned char *xt = st + NP * 16384;
        for (int q = tid; q < N * 8; q += kTT) {  // x rows: token q/8 (tokens past b repeat the last one)
          const int t = q >> 3, c = q & 7;
          const int tt = t < b ? t : b - 1;
          cp16(xt, kmajor_off(t, c), X + (size_t)tt * d + (size_t)kc * kTK + c * 8);
        }
      }
    };
    auto issue = [&](uint32_t st, int it) {
      for (int a = 0; a < kps; ++a) {
        const uint32_t at = st + (uint32_t)a * chunk_bytes, xt = at + NP * 16384;
#pragma unroll
        for (int k = 0; k < kTK / 16; ++k) {
          const uint64_t bd = sdesc_sw128(xt + k * 32, 16, 1024);
#pragma unroll
          for (int j = 0; j < NP; ++j)
            umma_f16(tmem + (uint32_t)(j * N), sdesc_sw128(at + j * 16384 + k * 32, 16, 1024), bd, idesc,
                     (it > 0 || a > 0 || k > 0) ? 1u : 0u);
        }
      }
    };
    if (ok && !tc_mainloop(smem, stage_bytes, stages, k1 - k0, mbar, &fail, load, issue, base)) {
      ok = false;
      if (tid == 0) latch_error(err, kErrTimeout);
    }
    base += k1 - k0;
    float gs[32], us[32];
    if (ok) {
      for (int c0 = 0; c0 < N; c0 += 16) tmem_ld16(lane_addr + c0, gs + c0);
      if (ACT == SFNN_REGLU)
        for (int c0 = 0; c0 < N; c0 += 16) tmem_ld16(lane_addr + N + c0, us + c0);
    } else {  // after a timeout the tile is still counted (the error is latched)
      for (int t = 0; t < 32; ++t) gs[t] = us[t] = 0.f;
    }
    tc_fence_before();
    __syncthreads();  // every TMEM read is done before the next segment's MMAs
    if (k0 == 0 && k1 == nk) {
      epilogue(m, gs, us);
    } else {
      const int slot = 2 * (int)g + (m == first_tile ? 0 : 1);
      for (int t = 0; t < b; ++t) {
        upart[((size_t)slot * NP * b + t) * kTM + row] = gs[t];
        if (ACT == SFNN_REGLU) upart[((size_t)slot * NP * b + b + t) * kTM + row] = us[t];
      }
      __threadfence();
      __syncthreads();
      const int64_t ga = cta_of((int64_t)m * nk), gb = cta_of((int64_t)m * nk + nk - 1);
      if (tid == 0) {
        const int prev = atomicAdd(&tcnt[m], 1);
        last_s = prev == (int)(gb - ga);
        if (last_s) tcnt[m] = 0;  // every segment of the tile has arrived: ready for the next launch
      }
      __syncthreads();
      if (last_s) {
        __threadfence();
        for (int t = 0; t < b; ++t) gs[t] = us[t] = 0.f;
        for (int64_t q = ga; q <= gb; ++q) {  // CTA order
          const int qs = 2 * (int)q + ((int)((q * T / G) / nk) == m ? 0 : 1);
          for (int t = 0; t < b; ++t) {
            gs[t] += __ldcg(&upart[((size_t)qs * NP * b + t) * kTM + row]);
            if (ACT == SFNN_REGLU) us[t] += __ldcg(&upart[((size_t)qs * NP * b + b + t) * kTM + row]);
          }
        }
        epilogue(m, gs, us);
      }
    }
    i0 = (int64_t)(m + 1) * nk;
  }
  tc_end(tmem);
}

// ---------------------------------------------------------------- k_tc_down
// A CTA computes mps adjacent 128-column output tiles (each a TMEM accumulator of N
// columns) over its split of the union.  smem per stage: mps A tiles (64 union rows x 128
// columns, MN-major, 16 KB each) + the H tile (N tokens x 64 union entries, K-major).  A
// warp's copy instruction covers 2 / mps union rows of 256 mps contiguous bytes.
template <int MPS>
__global__ void __launch_bounds__(kTT) k_tc_down(const __half *__restrict__ rows, const __half *__restrict__ H,
                                                 int hstride, const int32_t *__restrict__ ulist,
                                                 const int32_t *__restrict__ ucount, float *__restrict__ part, int d,
                                                 int b, int N, int nproj, int splits, int stages, int32_t *err) {
  constexpr int mps = MPS;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t mbar[8];
  __shared__ uint32_t tmem_slot;
  __shared__ int fail;
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt = blockIdx.x, ks = blockIdx.y;
  // The union (two kernels before) is complete when this grid starts: the up projection
  // lets it start only after its own griddepcontrol.wait.  Its list is read through L2.
  const int U = __ldcg(ucount);
  const int nkc = (U + kTK - 1) / kTK;
  const int c0 = (int)(((int64_t)ks * nkc) / splits), c1 = (int)(((int64_t)(ks + 1) * nkc) / splits);
  const int col0 = mt * kTM * mps;
  const uint32_t a_bytes = (uint32_t)mps * 16384u;
  const uint32_t stage_bytes = a_bytes + (uint32_t)N * 128u;

  if (c0 == c1) {  // an empty split still provides its (zero) partial
    pdl_wait();
    pdl_launch_dependents();
    for (int q = tid; q < b * kTM * mps; q += kTT)
      part[((size_t)ks * b + q / (kTM * mps)) * d + col0 + q % (kTM * mps)] = 0.f;
    return;
  }
  const uint32_t tmem = tc_begin(mbar, stages, &tmem_slot, &fail);

  // A: chunk q = tid + 128 i -> union row k = q / (16 mps) of the stage, 16-byte column
  // chunk c = q % (16 mps) of its 256 mps bytes: tile mp = c / 16, and within it MN atom
  // m' = (c % 16) / 8, chunk cc = c % 8 of its 128-byte row; k = 8 k1 + k0.
  constexpr int cpr = 16 * mps;  // 16-byte chunks of a row
  auto load = [&](int s, int it, int what) {
    const int kc = c0 + it;
    unsigned char *st = smem + (size_t)s * stage_bytes;
    if (what & kLoadA) {
#pragma unroll
      for (int i = 0; i < 8 * mps; ++i) {  // unrolled: the union indices are loaded together
        const int q = tid + kTT * i;
        const int k = q / cpr, c = q % cpr;
        int u = kc * kTK + k;
        u = u < U ? u : U - 1;  // past the union: a repeated row times H's zero padding
        const int mp = c >> 4, c16 = c & 15;
        const int k0 = k & 7, k1 = k >> 3, ma = c16 >> 3, cc = c16 & 7;
        const uint32_t off = (uint32_t)(mp * 16384 + ma * 1024 + k1 * 2048 + k0 * 128 + ((cc ^ k0) << 4));
        cp16(st, off, rows + ((size_t)__ldcg(ulist + u) * nproj + (nproj - 1)) * d + col0 + c * 8);
      }
    }
    if (what & kLoadB) {
      unsigned char *ht = st + a_bytes;
      for (int q = tid; q < N * 8; q += kTT) {
        const int t = q >> 3, c = q & 7;
        cp16(ht, kmajor_off(t, c), H + (size_t)t * hstride + (size_t)kc * kTK + c * 8);
      }
    }
  };
  const uint32_t idesc = idesc_f16(kTM, N, 1, 0);
  auto issue = [&](uint32_t st, int it) {
    const uint32_t ht = st + a_bytes;
#pragma unroll
    for (int k = 0; k < kTK / 16; ++k)
#pragma unroll
      for (int mp = 0; mp < mps; ++mp)
        umma_f16(tmem + (uint32_t)(mp * N), sdesc_sw128(st + mp * 16384 + k * 4096, 1024, 2048),
                 sdesc_sw128(ht + k * 32, 16, 1024), idesc, (it > 0 || k > 0) ? 1u : 0u);
  };
  // the first stages' W_down rows while the up projection finishes; H after it has
  const int a_pre = min(stages - 1, c1 - c0);
  for (int i = 0; i < a_pre; ++i) load(i, i, kLoadA);
  pdl_wait();
  pdl_launch_dependents();
  if (!tc_mainloop(smem, stage_bytes, stages, c1 - c0, mbar, &fail, load, issue, 0, a_pre)) {
    if (tid == 0) latch_error(err, kErrTimeout);
  } else {
    const int m = warp * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    float v[32];
#pragma unroll
    for (int mp = 0; mp < mps; ++mp) {
      for (int cb = 0; cb < N; cb += 16) tmem_ld16(lane_addr + mp * N + cb, v + cb);
      for (int t = 0; t < b; ++t) part[((size_t)ks * b + t) * d + col0 + mp * kTM + m] = v[t];
    }
  }
  tc_end(tmem);
}

// ---------------------------------------------------------------- predictor
// k_tc_hidden: partial hidden layer hp[ks][t][j] = A^T[j] . x_t over the ks-th split of d
// (A^T rows contiguous, 128 per CTA).  k_tc_hsum: h = relu(sum over ks in order), split
// into fp16 hi + lo (h - hi), the B operand pair of the logits.  k_tc_logits: z[i][t] =
// B^T[i] . (hi_t + lo_t) + c_i for 128 neurons per CTA (two MMAs per step into one fp32
// accumulator, so h keeps about 22 bits), active iff z > 0 -> one mask word per warp and
// token by ballot (token-major masks, as k_compact reads them).
__global__ void __launch_bounds__(kTT) k_tc_hidden(const __half *__restrict__ At, const __half *__restrict__ X,
                                                   float *__restrict__ hp, int d, int r, int b, int N, int splits,
                                                   int stages, int32_t *err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t mbar[8];
  __shared__ uint32_t tmem_slot;
  __shared__ int fail;
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j0 = blockIdx.x * kTM, ks = blockIdx.y;
  const int nkc = d / kTK;
  const int c0 = (int)(((int64_t)ks * nkc) / splits), c1 = (int)(((int64_t)(ks + 1) * nkc) / splits);
  const uint32_t stage_bytes = 16384u + (uint32_t)N * 128u;
  if (c0 == c1) {
    pdl_wait();
    pdl_launch_dependents();
    for (int q = tid; q < b * kTM; q += kTT) {
      const int t = q / kTM, j = j0 + q % kTM;
      if (j < r) hp[((size_t)ks * b + t) * r + j] = 0.f;
    }
    return;
  }
  const uint32_t tmem = tc_begin(mbar, stages, &tmem_slot, &fail);
  const int c8 = tid & 7;
  auto load = [&](int s, int it, int what) {
    const int kc = c0 + it;
    unsigned char *st = smem + (size_t)s * stage_bytes;
    if (what & kLoadA) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = (tid >> 3) + 16 * i;
        const int j = j0 + row < r ? j0 + row : r - 1;
        cp16(st, kmajor_off(row, c8), At + (size_t)j * d + (size_t)kc * kTK + c8 * 8);
      }
    }
    if (what & kLoadB) {
      unsigned char *xt = st + 16384;
      for (int q = tid; q < N * 8; q += kTT) {
        const int t = q >> 3, c = q & 7;
        const int tt = t < b ? t : b - 1;
        cp16(xt, kmajor_off(t, c), X + (size_t)tt * d + (size_t)kc * kTK + c * 8);
      }
    }
  };
  const uint32_t idesc = idesc_f16(kTM, N, 0, 0);
  auto issue = [&](uint32_t st, int it) {
#pragma unroll
    for (int k = 0; k < kTK / 16; ++k)
      umma_f16(tmem, sdesc_sw128(st + k * 32, 16, 1024), sdesc_sw128(st + 16384 + k * 32, 16, 1024), idesc,
               (it > 0 || k > 0) ? 1u : 0u);
  };
  // the first stages' A^T rows (weights) before the kernel before completes; x after it
  const int a_pre = min(stages - 1, c1 - c0);
  for (int i = 0; i < a_pre; ++i) load(i, i, kLoadA);
  pdl_wait();
  pdl_launch_dependents();
  if (!tc_mainloop(smem, stage_bytes, stages, c1 - c0, mbar, &fail, load, issue, 0, a_pre)) {
    if (tid == 0) latch_error(err, kErrTimeout);
  } else {
    const int j = j0 + warp * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    float v[32];
    for (int cb = 0; cb < N; cb += 16) tmem_ld16(lane_addr + cb, v + cb);
    if (j < r)
      for (int t = 0; t < b; ++t) hp[((size_t)ks * b + t) * r + j] = v[t];
  }
  tc_end(tmem);
}

__global__ void k_tc_hsum(const float *__restrict__ hp, int splits, int b, int N, int r, __half *__restrict__ hhi,
                          __half *__restrict__ hlo) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;  // t * r + j over N tokens
  if (i >= N * r) return;
  const int t = i / r;
  float h = 0.f;
  if (t < b) {
    const int j = i - t * r;
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += hp[((size_t)k * b + t) * r + j];
    h = s > 0.f ? s : 0.f;  // NaN -> 0
  }
  const __half hi = __float2half_rn(h);
  hhi[i] = hi;
  hlo[i] = __float2half_rn(h - __half2float(hi));
}

__global__ void __launch_bounds__(kTT) k_tc_logits(const __half *__restrict__ Bt, const __half *__restrict__ cvec,
                                                   const __half *__restrict__ hhi, const __half *__restrict__ hlo,
                                                   uint32_t *__restrict__ mask, int n, int r, int nwords, int b, int N,
                                                   int stages, int32_t *err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t mbar[8];
  __shared__ uint32_t tmem_slot;
  __shared__ int fail;
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = blockIdx.x * kTM;
  const uint32_t stage_bytes = 16384u + 2u * (uint32_t)N * 128u;
  const uint32_t tmem = tc_begin(mbar, stages, &tmem_slot, &fail);
  const int c8 = tid & 7;
  auto load = [&](int s, int kc, int what) {
    unsigned char *st = smem + (size_t)s * stage_bytes;
    if (what & kLoadA) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = (tid >> 3) + 16 * i;
        const int nn = i0 + row < n ? i0 + row : n - 1;
        cp16(st, kmajor_off(row, c8), Bt + (size_t)nn * r + (size_t)kc * kTK + c8 * 8);
      }
    }
    if (what & kLoadB) {
      unsigned char *ht = st + 16384;
      for (int q = tid; q < 2 * N * 8; q += kTT) {  // hi rows, then lo rows
        const int half = q / (N * 8), qq = q - half * N * 8;
        const int t = qq >> 3, c = qq & 7;
        cp16(ht + half * N * 128, kmajor_off(t, c), (half ? hlo : hhi) + (size_t)t * r + (size_t)kc * kTK + c * 8);
      }
    }
  };
  const uint32_t idesc = idesc_f16(kTM, N, 0, 0);
  auto issue = [&](uint32_t st, int it) {
    const uint32_t ht = st + 16384;
#pragma unroll
    for (int k = 0; k < kTK / 16; ++k) {
      const uint64_t ad = sdesc_sw128(st + k * 32, 16, 1024);
      umma_f16(tmem, ad, sdesc_sw128(ht + k * 32, 16, 1024), idesc, (it > 0 || k > 0) ? 1u : 0u);
      umma_f16(tmem, ad, sdesc_sw128(ht + N * 128 + k * 32, 16, 1024), idesc, 1u);
    }
  };
  // the first stages' B^T rows (weights) while the hidden layer is summed; h after it
  const int a_pre = min(stages - 1, r / kTK);
  for (int i = 0; i < a_pre; ++i) load(i, i, kLoadA);
  pdl_wait();
  pdl_launch_dependents();
  if (!tc_mainloop(smem, stage_bytes, stages, r / kTK, mbar, &fail, load, issue, 0, a_pre)) {
    if (tid == 0) latch_error(err, kErrTimeout);
  } else {
    const int i = i0 + warp * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    float v[32];
    for (int cb = 0; cb < N; cb += 16) tmem_ld16(lane_addr + cb, v + cb);
    const float cv = i < n ? __half2float(cvec[i]) : 0.f;
    const int word = (i0 + warp * 32) >> 5;
    for (int t = 0; t < b; ++t) {
      const bool on = i < n && v[t] + cv > 0.f;  // NaN -> inactive
      const uint32_t bits = __ballot_sync(0xffffffffu, on);
      if (lane == 0 && word < nwords) mask[(size_t)t * nwords + word] = bits;
    }
  }
  tc_end(tmem);
}

constexpr int kUpStages = 3, kDownStages = 3, kPredStages = 4;

size_t up_smem(int act, int N, int kps) {
  return (size_t)kUpStages * kps * ((act == SFNN_REGLU ? 2 : 1) * 16384 + N * 128) + 1024;
}
size_t down_smem(int N, int mps) { return (size_t)kDownStages * (mps * 16384 + N * 128) + 1024; }
size_t hidden_smem(int N) { return (size_t)kPredStages * (16384 + N * 128) + 1024; }
size_t logits_smem(int N) { return (size_t)kPredStages * (16384 + 2 * N * 128) + 1024; }

}  // namespace

bool tc_batch_supported(const sfnn_ctx *h) {
  return h->L.dt == SFNN_F16 && h->L.d % kTM == 0 && h->hact != nullptr;
}

bool tc_predict_supported(const sfnn_ctx *h) { return tc_batch_supported(h) && h->L.r % kTK == 0; }

int tc_hstride(int n) { return (n + kTM - 1) / kTM * kTM; }

// k_tc_up's largest grid: two CTAs per SM; its partials: two slots per CTA.
size_t tc_up_partial_bytes(int num_sms, int max_batch) {
  return (size_t)2 * (2 * num_sms) * 2 * (size_t)max_batch * kTM * sizeof(float);
}

// CTAs of `func` with `dyn` bytes of dynamic shared memory that fit on an SM at once: by
// shared memory (what the SM holds over each CTA's dynamic + static + reserved bytes), by
// registers and by tensor memory (kTmemCols of 512 columns each).  Worked out from the
// device's and the kernel's attributes: the occupancy calculator assumes a shared-memory
// carveout smaller than the one launches get.
static int fit_per_sm(const void *func, size_t dyn) {
  int dev = 0, smem_sm = 0, reserved = 0, regs_sm = 0;
  cudaFuncAttributes fa;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
      cudaFuncGetAttributes(&fa, func) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  int n = (int)((size_t)smem_sm / (dyn + fa.sharedSizeBytes + (size_t)reserved));
  const int regs_cta = ((fa.numRegs * 32 + 255) / 256 * 256) * (kTT / 32);  // per-warp granules of 256
  n = std::min(n, regs_cta > 0 ? regs_sm / regs_cta : n);
  n = std::min(n, 512 / kTmemCols);
  return n > 0 ? n : 1;
}

// k_tc_up CTAs that fit on an SM at once for this shape (worked out once per shape).
static int up_fit(int act, int N, int kps) {
  static int cache[2][2][2] = {};
  int &c = cache[act == SFNN_REGLU][N == 32][kps - 1];
  if (c == 0)
    c = act == SFNN_REGLU ? fit_per_sm((const void *)k_tc_up<SFNN_REGLU>, up_smem(act, N, kps))
                          : fit_per_sm((const void *)k_tc_up<SFNN_RELU>, up_smem(act, N, kps));
  return c;
}

// k_tc_down CTAs that fit on an SM at once (worked out once per shape).
static int down_fit(int N, int mps) {
  static int cache[2][2] = {};
  int &c = cache[N == 32][mps - 1];
  if (c == 0)
    c = fit_per_sm(mps == 2 ? (const void *)k_tc_down<2> : (const void *)k_tc_down<1>, down_smem(N, mps));
  return c;
}

cudaError_t configure_tc_batch() {
  cudaError_t e = cudaFuncSetAttribute(k_tc_up<SFNN_RELU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)up_smem(SFNN_RELU, 32, 2));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_tc_up<SFNN_REGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)up_smem(SFNN_REGLU, 32, 2));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_tc_down<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)down_smem(32, 1));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_tc_down<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)down_smem(32, 2));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_tc_hidden, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hidden_smem(32));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_tc_logits, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)logits_smem(32));
  // the CTAs per SM of every up and down shape, outside any stream capture
  for (int act : {SFNN_RELU, SFNN_REGLU})
    for (int N : {16, 32})
      for (int kps : {1, 2}) up_fit(act, N, kps);
  for (int N : {16, 32})
    for (int mps : {1, 2}) down_fit(N, mps);
  return e;
}

// The predictor of b tokens on the tensor cores -> h->mask (token-major bit words).
cudaError_t launch_tc_predict(const sfnn_ctx *h, const void *X, int b, cudaStream_t s) {
  const Layout &L = h->L;
  const int N = b <= 16 ? 16 : 32;
  const int rtiles = (L.r + kTM - 1) / kTM;
  // split d so that the hidden layer runs on about one CTA per SM; the partials fit in
  // the down projection's partial-sum buffer
  const size_t cap = (size_t)std::max<size_t>((size_t)kMaxSplits * h->max_batch, (size_t)std::min(h->num_sms, L.n)) * L.d;
  int splits = (h->num_sms + rtiles - 1) / rtiles;
  splits = std::min(splits, L.d / kTK);
  splits = std::min<int>(splits, (int)(cap / ((size_t)b * L.r)));
  splits = splits < 1 ? 1 : splits;
  // every kernel of the chain starts early (programmatic serialization) and copies its
  // first weight stages before it waits for the one before
  cudaError_t e = launch_pdl(k_tc_hidden, dim3(rtiles, splits), dim3(kTT), hidden_smem(N), s,
                             static_cast<const __half *>(h->At), static_cast<const __half *>(X), h->part, L.d, L.r,
                             b, N, splits, kPredStages, h->err);
  if (e != cudaSuccess) return e;
  __half *hhi = h->hpair, *hlo = h->hpair + (size_t)32 * L.r;
  e = launch_pdl(k_tc_hsum, dim3((N * L.r + 255) / 256), dim3(256), 0, s, (const float *)h->part, splits, b, N, L.r,
                 hhi, hlo);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_tc_logits, dim3((L.n + kTM - 1) / kTM), dim3(kTT), logits_smem(N), s,
                    static_cast<const __half *>(h->Bt), static_cast<const __half *>(h->cvec), (const __half *)hhi,
                    (const __half *)hlo, h->mask, L.n, L.r, L.nwords, b, N, kPredStages, h->err);
}

// Up / gate of the union rows for all b tokens -> h->hact; then the down projection into
// `splits` partials of h->part.
cudaError_t launch_tc_batch(const sfnn_ctx *h, const void *X, int b, int *splits_out, cudaStream_t s) {
  const Layout &L = h->L;
  const int N = b <= 16 ? 16 : 32;
  const int hs = tc_hstride(L.n);
  const __half *rows = static_cast<const __half *>(h->rows);
  const int kps = L.d % (2 * kTK) == 0 ? h->tc_up_kps : 1;
  const int up_grid = std::min(h->tc_up_ctas_per_sm, up_fit(L.act, N, kps)) * h->num_sms;
  cudaError_t e = launch_pdl(L.act == SFNN_REGLU ? k_tc_up<SFNN_REGLU> : k_tc_up<SFNN_RELU>, dim3(up_grid),
                             dim3(kTT), up_smem(L.act, N, kps), s, rows, static_cast<const __half *>(h->bias),
                             static_cast<const __half *>(X), (const int32_t *)h->ulist, (const uint32_t *)h->utok,
                             (const int32_t *)h->ucount, h->hact, hs, L.d, b, N, L.nproj, kUpStages, kps, h->upart,
                             h->tcnt, h->err);
  if (e != cudaSuccess) return e;
  const int mps = L.d % (2 * kTM) == 0 ? h->tc_down_mps : 1;
  const int mtiles = L.d / (kTM * mps);
  // one wave: the output tiles times the splits of the union fill the CTAs that fit at once
  int splits = (down_fit(N, mps) * h->num_sms) / mtiles;
  splits = splits < 1 ? 1 : (splits > kMaxSplits ? kMaxSplits : splits);
  *splits_out = splits;
  return launch_pdl(mps == 2 ? k_tc_down<2> : k_tc_down<1>, dim3(mtiles, splits), dim3(kTT), down_smem(N, mps), s,
                    rows, (const __half *)h->hact, hs, (const int32_t *)h->ulist, (const int32_t *)h->ucount, h->part,
                    L.d, b, N, L.nproj, splits, kDownStages, h->err);
}

}  // namespace sfnn
