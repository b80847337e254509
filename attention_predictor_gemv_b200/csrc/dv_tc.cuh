// Tensor-core gathered-row kernels (tcgen05 + TMA, sm_100a) for batch 3..16.
//
// At batch B the selected rows of W1, W2, W^{Q,K,V} and W^O meet B input
// vectors: a gathered row times a [d][B] block is a thin dense contraction
// (B flop per weight byte), which the CUDA cores cannot keep up with at HBM
// rate once B reaches 8-16, so these kernels hand the multiply-adds to the
// 5th-generation tensor cores and move the bytes with the tensor memory
// accelerator (TMA).
//
// Two kernel forms share one pipeline:
//   rowdot  D[m][b] = sum_c W[row(m)][c] X[b][c]    rows of W are K-major
//           (q, k, v of the selected heads; the MLP's first layer)
//   rowaxpy D[c][b] = sum_j W[row(j)][c] S[b][j]    rows of W are MN-major
//           (W^O of the selected heads; the MLP's second layer); a unit is a
//           group of rows times 128 output columns, and the groups' partials
//           are summed as 64-bit fixed-point integers (exact, so the sum does
//           not depend on the order in which CTAs finish; tc_acc_fixed) and
//           added into the output once by tc_finalize_kernel
// with M = 128 (gathered rows, or output columns), N = 16 (the batch rows,
// zero-padded) and 64 K-elements per pipeline stage.
//
// The activations enter as two bf16 arrays, hi = bf16(v) and lo =
// bf16(v - hi) (tc_split_kernel, or the W1 kernel's epilogue for the W2
// operand), so hi + lo carries 16 significant bits of every activation:
// D = W X_hi + W X_lo is accurate to about 2^-16 relative instead of the 2^-9
// of one bf16 rounding, at twice the (idle) tensor work.
//
// Per CTA (416 threads, one CTA per SM, persistent over work units), three
// roles that meet only at mbarriers:
//   * warps 0-7 fill a ring of `stages` stages, in the 128-byte swizzled
//     layout the MMA reads, completing on the stage's "full" barrier: the
//     weight tile (16 KB) as two TMA 2-D tiles of 64 rows where the rows are
//     consecutive (a head's Q/K/V or W^O rows), else (gathered W1, W2 rows)
//     by 16-byte cp.async copies of all 256 producer threads into their
//     swizzled places, each thread's completion counted on the barrier
//     (cp.async.mbarrier.arrive); and the operand blocks (16 x 64, hi and
//     lo) as TMA 2-D tiles. TMA tile::gather4 for the gathered rows was
//     measured at about 25 GB/s per SM (about 40 cycles per 4-row copy
//     however many warps issue them), below the SM's share of HBM;
//   * warp 8 (one lane) issues the MMAs of each stage (tcgen05.mma kind::f16,
//     bf16 inputs, fp32 accumulator in tensor memory) and commits them to the
//     stage's "empty" barrier, which hands the stage back to the producers;
//     at the end of a unit it commits the accumulator to the epilogue;
//   * warps 9-12 read the 128 x 16 accumulator (tcgen05.ld 32x32b; warp w
//     owns TMEM lanes 32 (w%4) ..) and run the unit's epilogue, while the
//     MMAs of the next unit already run into the second accumulator (two
//     16-column accumulators in 32 TMEM columns).
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on a timeout
// the kernel sets DV_DEV_TIMEOUT in the status word, the other roles stop at
// their next wait, the producers wait for their copies in flight, the MMA
// warp for its MMAs, the tensor memory is released and the kernel returns.
#pragma once

#include "dv_common.cuh"
#include "dv_tc_args.h"

namespace dv {

constexpr int TC_PRODUCERS = 8;                    // warps that issue the copies
constexpr int TC_MMA_WARP = TC_PRODUCERS;          // warp that issues the MMAs
constexpr int TC_EPI_WARP0 = TC_PRODUCERS + 1;     // first of the four epilogue warps
constexpr int TC_THREADS = (TC_PRODUCERS + 5) * 32;
constexpr int TC_PRODUCER_THREADS = TC_PRODUCERS * 32;
constexpr int TC_K = 64;        // K elements per stage (128 bytes of a bf16 row: one swizzle span)
constexpr int TC_STAGES_MAX = 10;  // ring stages with one CTA per SM (half with two)
constexpr int TC_A_BYTES = TC_M * TC_K * 2;  // 16 KB weight tile
constexpr int TC_B_BYTES = TC_N * TC_K * 2;  // 2 KB bf16 operand (hi or lo)
constexpr int TC_STAGE_BYTES = TC_A_BYTES + 2 * TC_B_BYTES;
__host__ __device__ constexpr size_t tc_smem(int stages) { return 1024 + (size_t)stages * TC_STAGE_BYTES; }
constexpr int TC_TMEM_COLS = 32;       // two accumulators of TC_N columns

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// One arrival that also announces `bytes` of asynchronous copies the phase
// waits for.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the phase with the given parity to complete, for at most about
// two seconds, or until *abort is set (by another role that gave up);
// false in both cases.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, const volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (abort && *abort) return false;
    if (global_ns() - t0 > 2000000000ull) return false;
  }
  return true;
}

// 2-D tensor tile load into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte copy global -> shared through L2 (cp.async), the first src_bytes
// of it read and the rest zero (src_bytes 0: nothing is read).
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// One arrival on `bar` (counted in its expected arrivals) once every
// cp.async this thread issued before has landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The MMA reads shared memory through the async proxy; the copies above
// wrote it through the generic one.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, int ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, int ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D (tensor memory) (+)= A (shared, desc) x B (shared, desc)^T; kind::f16
// with bf16 inputs and an fp32 accumulator, one CTA.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every MMA this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp gets lane
// (taddr lane + i), columns taddr col .. +15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Barrier of the four epilogue warps (named barrier 1, 128 threads), and the
// same barrier returning whether `ok` holds in all of them.
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool epi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

// Shared-memory matrix descriptor of the 128-byte swizzled layouts (rows of
// 128 bytes whose 16-byte pieces are permuted by the row index mod 8, in
// atoms of 8 rows = 1024 bytes): start address, leading-dimension byte offset
// (K-major: unused, 16; MN-major: the distance between 64-element blocks
// along M), stride-dimension byte offset (the distance between 8-row groups),
// descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, B
// K-major, A K-major (a_mn = 0) or MN-major (a_mn = 1), shape M x N.
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N, int a_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Shared-memory stage layout (offsets inside one 1024-aligned stage)
// ---------------------------------------------------------------------------
//   A    [0, 16 KB)      weight tile
//   Bhi  [16, 18 KB)     operand hi part: 16 batch rows x 64 K, K-major
//   Blo  [18, 20 KB)     operand lo part
//
// rowdot A (K-major, 128 rows x 64 K): row m at m * 128 bytes (gather4 g
// brings rows 4g..4g+3 to g * 512, a 64-row tile k to k * 8192); sbo = 1024;
// the K = 16 slice kk of the
// stage starts 32 kk bytes in (inside the swizzle span, as the hardware
// applies the permutation to the address bits).
// rowaxpy A (MN-major, 128 columns x 64 K rows): two blocks of 64 columns at
// 0 and 8 KB, K row j of a block at j * 128 bytes; lbo = 8192, sbo = 1024;
// the K = 16 slice kk starts at kk * 2048 (two 8-row groups).
// B (K-major, 16 x 64): like rowdot A with 16 rows.
constexpr int TC_OFF_BHI = TC_A_BYTES;
constexpr int TC_OFF_BLO = TC_A_BYTES + TC_B_BYTES;

// ---------------------------------------------------------------------------
// The pipeline (shared by both forms)
// ---------------------------------------------------------------------------
//
// A problem P provides:
//   static constexpr int kAMajorMN;               // 0 rowdot, 1 rowaxpy
//   static constexpr bool kGather;                // weight rows by the producers' cp.async (else TMA tiles
//                                                 // issued by producer thread 0)
//   static constexpr bool kRowsPerUnit;           // rows() depends on the unit only
//   __device__ int units() const;                 // work units in total
//   __device__ int chunks(int unit) const;        // stages of K in a unit (>= 1 for every unit)
//   __device__ bool live(int unit, int c) const;  // false: the stage is skipped (no copies, no MMA)
//   __device__ bool any(int unit) const;          // some stage of the unit is live
//   __device__ void rows(int unit, int c, int t, int (&r)[4]) const;   // producer thread t's rows (kGather;
//                                                 // -1: zero-filled)
//   __device__ void issue(uint32_t stage, uint64_t* full, int unit, int c, int t, const int (&r)[4]) const;
//                                                 // thread t's copies (kGather), and with t = 0 the stage's
//                                                 // TMA copies (tiles and operands)
//   __device__ void epilogue(int unit, int m, int q, const float (&v)[16], bool any) const;
// The epilogue runs in the four epilogue warps together (it may use
// epi_sync()); thread m holds accumulator row m (epilogue warp q = m / 32).
// `any` is false when the unit issued no MMA (its accumulator is then zero).

template <class P>
__device__ void tc_run(const P& p, int* status, int stages) {
  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[TC_STAGES_MAX];
  __shared__ __align__(8) uint64_t bar_empty[TC_STAGES_MAX];
  __shared__ __align__(8) uint64_t bar_acc_full[2];
  __shared__ __align__(8) uint64_t bar_acc_empty[2];
  __shared__ __align__(8) uint64_t bar_final;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem0 = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == TC_MMA_WARP) {
    tmem_alloc(&s_tmem, TC_TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&bar_full[s], P::kGather ? TC_PRODUCER_THREADS + 1 : 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bar_acc_full[a], 1);
      mbar_init(&bar_acc_empty[a], 4);
    }
    mbar_init(&bar_final, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int nunits = p.units();
  auto give_up = [&]() {
    if (!s_abort) raise_status(status, DV_DEV_TIMEOUT_BIT);
    s_abort = 1;
  };

  if (warp < TC_PRODUCERS) {
    // ---- producers: the CTA's live stages in order (units blockIdx.x,
    // + gridDim.x, ...); every producer warp waits for a slot; with gathered
    // rows all 256 producer threads copy (thread t), otherwise thread 0
    // alone; thread 0 also announces the stage's TMA bytes and issues those
    // copies. The rows of the next stage are loaded while waiting for its
    // slot. ----
    if (P::kGather || warp == 0) {
      const int t = tid;
      const bool active = P::kGather || lane == 0;
      int u = blockIdx.x, c = -1, nc = u < nunits ? p.chunks(u) : 0;
      auto next_live = [&](int& u, int& c) {
        while (u < nunits) {
          if (++c >= nc) {
            u += gridDim.x;
            c = -1;
            nc = u < nunits ? p.chunks(u) : 0;
            continue;
          }
          if (p.live(u, c)) return;
        }
      };
      next_live(u, c);
      int r[4] = {-1, -1, -1, -1};
      int ru = -1;
      if (u < nunits && P::kGather) {
        p.rows(u, c, t, r);
        ru = u;
      }
      int issued = 0;
      bool ok = true;
      while (u < nunits) {
        const int s = issued % stages;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_empty[s], ((issued / stages) & 1) ^ 1, &s_abort));
        if (!ok) break;
        if (tid == 0) mbar_expect_tx(&bar_full[s], P::kGather ? 2 * TC_B_BYTES : TC_STAGE_BYTES);
        if (active) p.issue(smem0 + (uint32_t)s * TC_STAGE_BYTES, &bar_full[s], u, c, t, r);
        if (P::kGather) cp_async_arrive(&bar_full[s]);
        ++issued;
        next_live(u, c);
        if (u < nunits && P::kGather && (!P::kRowsPerUnit || u != ru)) {
          p.rows(u, c, t, r);
          ru = u;
        }
      }
      if (!ok && lane == 0) give_up();
      // the copies of the last stages issued have landed before the CTA may
      // exit (at once when the MMA warp consumed them)
      if (P::kGather) cp_async_wait_all();
      if (lane == 0)
        for (int i = issued > stages ? issued - stages : 0; i < issued; ++i)
          mbar_wait(&bar_full[i % stages], (i / stages) & 1, nullptr);
    }
  } else if (warp == TC_MMA_WARP) {
    if (lane == 0) {
      // ---- MMA issuer ----
      constexpr uint32_t idesc = tc_idesc(TC_M, TC_N, P::kAMajorMN);
      int consumed = 0, n = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++n) {
        const int acc = n & 1;
        if (!mbar_wait(&bar_acc_empty[acc], ((n >> 1) & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(acc * TC_N);
        bool first = true;
        const int nc = p.chunks(u);
        for (int c = 0; c < nc; ++c) {
          if (!p.live(u, c)) continue;
          const int s = consumed % stages;
          if (!mbar_wait(&bar_full[s], (consumed / stages) & 1, &s_abort)) {
            ok = false;
            break;
          }
          if (P::kGather) fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a0 = smem0 + (uint32_t)s * TC_STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < TC_K / 16; ++kk) {
            const uint64_t ad =
                P::kAMajorMN ? tc_sdesc(a0 + kk * 2048, 8192, 1024) : tc_sdesc(a0 + kk * 32, 16, 1024);
            tc_mma(dt, ad, tc_sdesc(a0 + TC_OFF_BHI + kk * 32, 16, 1024), idesc, (!first || kk > 0) ? 1u : 0u);
            tc_mma(dt, ad, tc_sdesc(a0 + TC_OFF_BLO + kk * 32, 16, 1024), idesc, 1u);
          }
          tc_commit(&bar_empty[s]);
          ++consumed;
          first = false;
        }
        if (!ok) break;
        tc_commit(&bar_acc_full[acc]);
      }
      if (!ok) give_up();
      // every MMA issued has completed before the tensor memory is released
      tc_commit(&bar_final);
      mbar_wait(&bar_final, 0, nullptr);
    }
  } else {
    // ---- epilogue warps: accumulator quarter q = warp % 4 ----
    const int q = warp & 3;
    int n = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++n) {
      const int acc = n & 1;
      const bool ok = epi_all(mbar_wait(&bar_acc_full[acc], (n >> 1) & 1, &s_abort));
      if (!ok) {
        if (warp == TC_EPI_WARP0 && lane == 0) give_up();
        break;
      }
      tc_fence_after();
      const bool any = p.any(u);
      float v[16];
      if (any) {
        tmem_ld16(tmem + (uint32_t)(acc * TC_N) + ((uint32_t)(q * 32) << 16), v);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acc_empty[acc]);
      p.epilogue(u, q * 32 + lane, q, v, any);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == TC_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TC_TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Activations split into bf16 hi / lo rows: hi[b][j] = bf16(x), lo[b][j] =
// bf16(x - hi) for b < nb, zero for nb <= b < 16; x = src[b * ld + j].
// ---------------------------------------------------------------------------
struct TcSplitArgs {
  const float* src;
  int nb, n;
  long long ld_src;
  __nv_bfloat16* hi;
  __nv_bfloat16* lo;
  long long ld_dst;
};

__global__ void __launch_bounds__(256) tc_split_kernel(TcSplitArgs a) {
  griddep_launch();
  griddep_wait();
  const int b = blockIdx.y;
  for (int j = blockIdx.x * 256 + threadIdx.x; j < a.n; j += gridDim.x * 256) {
    const float x = b < a.nb ? a.src[(size_t)b * a.ld_src + j] : 0.f;
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    a.hi[(size_t)b * a.ld_dst + j] = h;
    a.lo[(size_t)b * a.ld_dst + j] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
}

// The operand blocks of a stage: columns x .. x+63 of the 16 hi and lo rows.
__device__ __forceinline__ void tc_issue_operand(const TcMaps& m, uint32_t stage, uint64_t* full, int x) {
  tma_load_2d(stage + TC_OFF_BHI, &m.hi, x, 0, full);
  tma_load_2d(stage + TC_OFF_BLO, &m.lo, x, 0, full);
}

// ---------------------------------------------------------------------------
// Split K for the rowdot kernels. A 128-row tile's K range is cut into ks
// parts (units tile * ks + part), so that a tile count that does not fill the
// CTAs evenly still keeps them all streaming. A CTA streams at a rate of its
// own (its producers' copies in flight), so the step takes about as long as
// the most units any CTA holds: ceil(tiles * ks / grid) / ks tiles' time. ks
// is the power of two (1, 2, 4, 8, at most the chunks of K) that minimises it,
// with 3% added per extra part for the reduction; the same in every CTA.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int tc_pick_kslog(int tiles, int C) {
  const int G = gridDim.x;
  int best_log = 0;
  float best = 3.0e38f;
  for (int lg = 0; lg <= 3 && (1 << lg) <= C; ++lg) {
    const int ks = 1 << lg, per_cta = (tiles * ks + G - 1) / G;
    const float t = (float)per_cta / (float)ks * (1.0f + 0.03f * (float)(ks - 1));
    if (t < best) {
      best = t;
      best_log = lg;
    }
  }
  return best_log;
}

// The epilogue threads' partial sums of `tile` (thread m: row m, v[b] for b <
// nb) go into this part's own slot of red ([128][16] floats, so a thread's
// values are four float4); the part that finishes the tile last (ticket)
// sums the ks slots in part order into v, resets the ticket and returns true
// in all 128 threads; the other parts return false. The sum is the same
// whichever part arrives last, so results do not depend on timing (the
// selections downstream compare scores exactly). With ks == 1 v is already
// complete.
__device__ __forceinline__ bool tc_reduce_parts(float* red, unsigned* tick, int tile, int part, int ks, int nb, int m,
                                                float (&v)[16], int* s_flag) {
  if (ks == 1) return true;
  constexpr int SLOT4 = TC_N * TC_M / 4;  // float4 per slot
  const int nq = (nb + 3) >> 2;
  float4* slot = reinterpret_cast<float4*>(red) + ((size_t)tile * ks + part) * SLOT4 + m * 4;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q < nq) slot[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __threadfence();
  epi_sync();
  if (m == 0) *s_flag = atomicAdd(tick + tile, 1u) == (unsigned)(ks - 1) ? 1 : 0;
  epi_sync();
  const bool last = *s_flag != 0;
  if (last) {
    __threadfence();
    const float4* t0 = reinterpret_cast<const float4*>(red) + (size_t)tile * ks * SLOT4 + m * 4;
    float4 sum[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) sum[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int p = 0; p < ks; ++p) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q < nq) {
          const float4 w = __ldcg(t0 + (size_t)p * SLOT4 + q);
          sum[q].x += w.x;
          sum[q].y += w.y;
          sum[q].z += w.z;
          sum[q].w += w.w;
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[4 * q] = sum[q].x;
      v[4 * q + 1] = sum[q].y;
      v[4 * q + 2] = sum[q].z;
      v[4 * q + 3] = sum[q].w;
    }
    if (m == 0) tick[tile] = 0u;
  }
  epi_sync();  // s_flag is reused by the next unit
  return last;
}

// ---------------------------------------------------------------------------
// Order-independent sums of the rowaxpy partials: each partial is rounded to
// a multiple of 2^-32 and added as a 64-bit integer (two's complement, so an
// unsigned atomic add), which is exact and associative; tc_finalize_kernel
// converts each total once (to fp64, exactly, then fp32), adds it and the bias
// into the output, and zeroes the accumulator. Partials stay far inside the
// range (|v| < 2^31).
// ---------------------------------------------------------------------------
constexpr double TC_FIXED_SCALE = 4294967296.0;  // 2^32

__device__ __forceinline__ void tc_acc_fixed(unsigned long long* acc, int d, int nb, int col, const float (&v)[16]) {
#pragma unroll
  for (int b = 0; b < TC_N; ++b) {
    if (b >= nb) break;
    const long long q = __double2ll_rn((double)v[b] * TC_FIXED_SCALE);
    atomicAdd(acc + (size_t)b * d + col, (unsigned long long)q);
  }
}

struct TcFinalizeArgs {
  unsigned long long* acc;  // [nb][d], zero on exit
  const float* bias;        // [d] or null
  float* out;               // [nb][d], accumulated into
  int nb, d;
};

__global__ void __launch_bounds__(256) tc_finalize_kernel(TcFinalizeArgs a) {
  griddep_launch();
  griddep_wait();
  const int n = a.nb * a.d;
  for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) {
    const long long q = (long long)a.acc[i];
    a.acc[i] = 0ull;
    const int col = i % a.d;
    a.out[i] += (float)((double)q / TC_FIXED_SCALE) + (a.bias ? a.bias[col] : 0.f);
  }
}

// ---------------------------------------------------------------------------
// q, k, v of the selected heads (rowdot over Wqkv rows)
// ---------------------------------------------------------------------------

struct TcQkvProblem {
  static constexpr int kAMajorMN = 0;
  static constexpr bool kGather = false;
  static constexpr bool kRowsPerUnit = true;
  const TcMaps& m;
  TcQkvArgs a;
  int nslots;      // selected heads x 3 dh
  int C, kslog;    // 64-column chunks of d; log2 of the K parts per tile
  int* s_flag;
  __device__ int units() const { return ((nslots + TC_M - 1) / TC_M) << kslog; }
  __device__ int c0(int unit) const { return ((unit & ((1 << kslog) - 1)) * C) >> kslog; }
  __device__ int chunks(int unit) const { return ((((unit & ((1 << kslog) - 1)) + 1) * C) >> kslog) - c0(unit); }
  __device__ bool live(int, int) const { return true; }
  __device__ bool any(int) const { return true; }
  __device__ void rows(int, int, int, int (&)[4]) const {}
  // the tile's 128 slots as two tiles of 64 consecutive Wqkv rows (3 dh is a
  // multiple of 64, so a tile never spans two heads); slots past the
  // selected ones, and invalid heads, read rows 0.. (their accumulator rows
  // are not used)
  __device__ void issue(uint32_t st, uint64_t* full, int unit, int c, int, const int (&)[4]) const {
    const int per = 3 * a.dh, x = (c0(unit) + c) * TC_K;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int s0 = (unit >> kslog) * TC_M + 64 * k;
      int y = 0;
      if (s0 < nslots) {
        const int head = a.head_idx[s0 / per];
        if (head >= 0 && head < a.h) y = head * per + s0 % per;
      }
      tma_load_2d(st + k * 8192, &m.w, x, y, full);
    }
    tc_issue_operand(m, st, full, x);
  }
  __device__ void epilogue(int unit, int mrow, int, const float (&v0)[16], bool) const {
    float v[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) v[b] = v0[b];
    const int tile = unit >> kslog;
    if (!tc_reduce_parts(a.red, a.tick, tile, unit & ((1 << kslog) - 1), 1 << kslog, a.nb, mrow, v, s_flag)) return;
    const int per = 3 * a.dh;
    const int s = tile * TC_M + mrow;
    if (s >= nslots) return;
    const int p = s / per, rem = s % per, which = rem / a.dh, c = rem % a.dh;
    const int head = a.head_idx[p];
    if (head < 0 || head >= a.h) {
      if (rem == 0) raise_status(a.status, 2);
      return;
    }
    const float bias = a.bqkv ? a.bqkv[(size_t)head * per + rem] : 0.f;
#pragma unroll
    for (int b = 0; b < TC_N; ++b) {
      if (b >= a.nb) break;
      const float val = v[b] + bias;
      if (which == 0) {
        a.q[((size_t)b * a.kh_max + p) * a.dh + c] = val;
      } else {
        __nv_bfloat16* cache = which == 1 ? a.Kc : a.Vc;
        cache[(((size_t)b * a.h + head) * a.cap + a.pos) * a.dh + c] = __float2bfloat16_rn(val);
      }
    }
  }
};

__global__ void __launch_bounds__(TC_THREADS, 2) tc_qkv_kernel(const __grid_constant__ TcMaps m, TcQkvArgs a) {
  __shared__ int s_flag;
  griddep_launch();
  griddep_wait();
  int hc = *a.head_count;
  if (hc > a.kh_max || hc < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, 1);
    hc = hc < 0 ? 0 : a.kh_max;
  }
  const int nslots = hc * 3 * a.dh, C = (a.d + TC_K - 1) / TC_K;
  TcQkvProblem p{m, a, nslots, C, tc_pick_kslog((nslots + TC_M - 1) / TC_M, C), &s_flag};
  tc_run(p, a.status, a.stages);
}

// ---------------------------------------------------------------------------
// The MLP: activations of the selected neurons (rowdot over W1 rows, with
// bias, activation and per-tile compaction of the nonzero ones, written as
// hi / lo bf16 rows), then the gather-axpy of their W2 rows (rowaxpy)
// ---------------------------------------------------------------------------

__device__ __forceinline__ int tc_clamped_count(const int32_t* count, int bound, int* status) {
  int c = *count;
  if (c > bound || c < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(status, 1);
    c = c < 0 ? 0 : bound;
  }
  return c;
}

struct TcW1Problem {
  static constexpr int kAMajorMN = 0;
  static constexpr bool kGather = true;
  static constexpr bool kRowsPerUnit = true;
  const TcMaps& m;
  TcMlpArgs a;
  int cnt;
  int C, kslog;  // 64-column chunks of d; log2 of the K parts per tile
  int* s_warp;   // [4] shared: nonzero counts of the epilogue warps
  int* s_flag;
  __device__ int units() const { return ((cnt + TC_M - 1) / TC_M) << kslog; }
  __device__ int c0(int unit) const { return ((unit & ((1 << kslog) - 1)) * C) >> kslog; }
  __device__ int chunks(int unit) const { return ((((unit & ((1 << kslog) - 1)) + 1) * C) >> kslog) - c0(unit); }
  __device__ bool live(int, int) const { return true; }
  __device__ bool any(int) const { return true; }
  // thread t copies 16-byte piece t % 8 of tile rows t / 8 + 32 j (j < 4);
  // slots past the count (and invalid indices) are zero-filled
  __device__ void rows(int unit, int, int t, int (&r)[4]) const {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int s = (unit >> kslog) * TC_M + (t >> 3) + 32 * j;
      const int v = s < cnt ? a.idx[s] : -1;
      r[j] = (v >= 0 && v < a.N) ? v : -1;
    }
  }
  __device__ void issue(uint32_t st, uint64_t* full, int unit, int c, int t, const int (&r)[4]) const {
    const int x = (c0(unit) + c) * TC_K, g = t & 7, row0 = t >> 3, col = x + 8 * g;
    const uint32_t dst0 = st + (uint32_t)(row0 * 128) + (uint32_t)((g ^ (row0 & 7)) << 4);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool ok = r[j] >= 0 && col < a.d;
      cp_async16_zfill(dst0 + 32 * 128 * j, ok ? (const void*)(a.W1t + (size_t)r[j] * a.d + col) : (const void*)a.W1t,
                       ok ? 16 : 0);
    }
    if (t == 0) tc_issue_operand(m, st, full, x);
  }
  __device__ void epilogue(int unit, int mrow, int q, const float (&v0)[16], bool) const {
    float v[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) v[b] = v0[b];
    const int tile = unit >> kslog;
    if (!tc_reduce_parts(a.red, a.tick, tile, unit & ((1 << kslog) - 1), 1 << kslog, a.nb, mrow, v, s_flag)) return;
    const int s = tile * TC_M + mrow;
    int r = s < cnt ? a.idx[s] : -1;
    if (s < cnt && (r < 0 || r >= a.N)) {
      raise_status(a.status, 2);
      r = -1;
    }
    const float bias = r >= 0 ? a.b1[r] : 0.f;
    float act[TC_N];
    bool nz = false;
#pragma unroll
    for (int b = 0; b < TC_N; ++b) {
      act[b] = (r >= 0 && b < a.nb) ? activate(v[b] + bias, a.act) : 0.f;
      nz = nz || act[b] != 0.f;
    }
    const int lane = threadIdx.x & 31;
    const unsigned bal = __ballot_sync(0xffffffffu, nz);
    if (lane == 0) s_warp[q] = __popc(bal);
    epi_sync();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int n = s_warp[w];
      before += w < q ? n : 0;
      total += n;
    }
    const int base = tile * TC_M;
    // all 16 rows are written (rows >= nb zero): the W2 operand loads read
    // whole 16-row blocks
    if (nz) {  // the nonzero activations at their compacted slot
      const int slot = before + __popc(bal & ((1u << lane) - 1u));
#pragma unroll
      for (int b = 0; b < TC_N; ++b) {
        const __nv_bfloat16 h = __float2bfloat16_rn(act[b]);
        a.act_hi[(size_t)b * a.KC + base + slot] = h;
        a.act_lo[(size_t)b * a.KC + base + slot] = __float2bfloat16_rn(act[b] - __bfloat162float(h));
      }
      a.rowid_c[base + slot] = r;
    }
    if (mrow >= total) {  // zeros after the tile's count (the W2 operand reads 64-slot pieces)
      const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
      for (int b = 0; b < TC_N; ++b) {
        a.act_hi[(size_t)b * a.KC + base + mrow] = z;
        a.act_lo[(size_t)b * a.KC + base + mrow] = z;
      }
    }
    if (mrow == 0) a.tile_cnt[tile] = total;
    epi_sync();  // s_warp is reused by the next unit
  }
};

__global__ void __launch_bounds__(TC_THREADS, 2) tc_w1_kernel(const __grid_constant__ TcMaps m, TcMlpArgs a) {
  __shared__ int s_warp[4];
  __shared__ int s_flag;
  griddep_launch();
  griddep_wait();
  const int cnt = tc_clamped_count(a.count, a.k_max, a.status), C = (a.d + TC_K - 1) / TC_K;
  TcW1Problem p{m, a, cnt, C, tc_pick_kslog((cnt + TC_M - 1) / TC_M, C), s_warp, &s_flag};
  tc_run(p, a.status, a.stages);
}

struct TcW2Problem {
  static constexpr int kAMajorMN = 1;
  static constexpr bool kGather = true;
  static constexpr bool kRowsPerUnit = false;
  const TcMaps& m;
  TcMlpArgs a;
  int ntiles, n_mt, n_groups;
  const int* s_cnt;  // shared: tile_cnt of every tile
  __device__ int units() const { return n_mt * n_groups; }
  __device__ int tiles_in(int g) const {
    const int t = ntiles - g * a.tiles_per_group;
    return t < 0 ? 0 : (t > a.tiles_per_group ? a.tiles_per_group : t);
  }
  __device__ int chunks(int unit) const {
    const int n = 2 * tiles_in(unit / n_mt);
    return n > 0 ? n : 1;  // group 0 always runs its epilogue (it adds b2)
  }
  __device__ bool live(int unit, int c) const {
    const int g = unit / n_mt;
    if ((c >> 1) >= tiles_in(g)) return false;
    return s_cnt[g * a.tiles_per_group + (c >> 1)] > (c & 1) * 64;
  }
  __device__ bool any(int unit) const {
    const int g = unit / n_mt, nt = tiles_in(g);
    for (int t = 0; t < nt; ++t)
      if (s_cnt[g * a.tiles_per_group + t] > 0) return true;
    return false;
  }
  // thread t copies 16-byte piece t % 8 of K rows t / 8 and t / 8 + 32 of
  // the stage (its 64 compacted slots), output columns col0 .. col0+63 and
  // col0+64 .. col0+127; slots past the tile's count are zero-filled
  __device__ void rows(int unit, int c, int t, int (&r)[4]) const {
    const int tl = (unit / n_mt) * a.tiles_per_group + (c >> 1), half = c & 1;
    const int n = s_cnt[tl] - half * 64;
    const int base = tl * TC_M + half * 64, j0 = t >> 3;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int j = j0 + 32 * i;
      const int v = j < n ? a.rowid_c[base + j] : -1;
      r[i] = (v >= 0 && v < a.N) ? v : -1;
    }
  }
  __device__ void issue(uint32_t st, uint64_t* full, int unit, int c, int t, const int (&r)[4]) const {
    const int tl = (unit / n_mt) * a.tiles_per_group + (c >> 1), half = c & 1;
    const int g = t & 7, j0 = t >> 3, col0 = (unit % n_mt) * TC_M + 8 * g;
    const uint32_t sw = (uint32_t)((g ^ (j0 & 7)) << 4);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int h = i >> 1, j = j0 + 32 * (i & 1), rid = r[i & 1], col = col0 + 64 * h;
      const bool ok = rid >= 0 && col < a.d;
      cp_async16_zfill(st + (uint32_t)(h * 8192 + j * 128) + sw,
                       ok ? (const void*)(a.W2t + (size_t)rid * a.d + col) : (const void*)a.W2t, ok ? 16 : 0);
    }
    if (t == 0) tc_issue_operand(m, st, full, tl * TC_M + half * 64);
  }
  __device__ void epilogue(int unit, int mrow, int, const float (&v)[16], bool any) const {
    const int col = (unit % n_mt) * TC_M + mrow;
    if (any && col < a.d) tc_acc_fixed(a.acc, a.d, a.nb, col, v);
  }
};

__global__ void __launch_bounds__(TC_THREADS, 2) tc_w2_kernel(const __grid_constant__ TcMaps m, TcMlpArgs a) {
  __shared__ int s_cnt[TC_MAX_TILES];
  griddep_launch();
  griddep_wait();
  const int cnt = tc_clamped_count(a.count, a.k_max, a.status);
  const int ntiles = (cnt + TC_M - 1) / TC_M;
  for (int t = threadIdx.x; t < ntiles; t += TC_THREADS) {
    int v = a.tile_cnt[t];
    s_cnt[t] = v < 0 ? 0 : (v > TC_M ? TC_M : v);
  }
  __syncthreads();
  const int n_mt = (a.d + TC_M - 1) / TC_M;
  const int n_groups = ntiles > 0 ? (ntiles + a.tiles_per_group - 1) / a.tiles_per_group : 1;
  TcW2Problem p{m, a, ntiles, n_mt, n_groups, s_cnt};
  tc_run(p, a.status, a.stages);
}

// ---------------------------------------------------------------------------
// W^O of the selected heads (rowaxpy over WOt rows; operand H as hi / lo).
// A head's dh rows are consecutive, so a stage's 64 K rows x 128 columns are
// two plain 64 x 64 tiles.
// ---------------------------------------------------------------------------

struct TcWoProblem {
  static constexpr int kAMajorMN = 1;
  static constexpr bool kGather = false;
  static constexpr bool kRowsPerUnit = true;
  const TcMaps& m;
  TcWoArgs a;
  int hc, n_mt, n_groups, cph;  // cph: 64-row chunks per head
  __device__ int units() const { return n_mt * n_groups; }
  __device__ int heads_in(int g) const {
    const int t = hc - g * a.heads_per_group;
    return t < 0 ? 0 : (t > a.heads_per_group ? a.heads_per_group : t);
  }
  __device__ int chunks(int unit) const {
    const int n = cph * heads_in(unit / n_mt);
    return n > 0 ? n : 1;
  }
  __device__ bool head_ok(int p) const {
    const int head = a.head_idx[p];
    return head >= 0 && head < a.h;
  }
  __device__ bool live(int unit, int c) const {
    const int g = unit / n_mt, j = c / cph;
    return j < heads_in(g) && head_ok(g * a.heads_per_group + j);
  }
  __device__ bool any(int unit) const {
    const int g = unit / n_mt, nh = heads_in(g);
    for (int j = 0; j < nh; ++j)
      if (head_ok(g * a.heads_per_group + j)) return true;
    return false;
  }
  __device__ void rows(int, int, int, int (&)[4]) const {}
  __device__ void issue(uint32_t st, uint64_t* full, int unit, int c, int, const int (&)[4]) const {
    const int p = (unit / n_mt) * a.heads_per_group + c / cph, part = c % cph;
    const int y = a.head_idx[p] * a.dh + part * 64, x = (unit % n_mt) * TC_M;
    tma_load_2d(st, &m.w, x, y, full);
    tma_load_2d(st + 8192, &m.w, x + 64, y, full);
    tc_issue_operand(m, st, full, p * a.dh + part * 64);
  }
  __device__ void epilogue(int unit, int mrow, int, const float (&v)[16], bool any) const {
    const int col = (unit % n_mt) * TC_M + mrow;
    if (any && col < a.d) tc_acc_fixed(a.acc, a.d, a.nb, col, v);
  }
};

__global__ void __launch_bounds__(TC_THREADS, 2) tc_wo_kernel(const __grid_constant__ TcMaps m, TcWoArgs a) {
  griddep_launch();
  griddep_wait();
  const int hc = tc_clamped_count(a.head_count, a.kh_max, a.status);
  const int n_mt = (a.d + TC_M - 1) / TC_M;
  const int n_groups = hc > 0 ? (hc + a.heads_per_group - 1) / a.heads_per_group : 1;
  TcWoProblem p{m, a, hc, n_mt, n_groups, a.dh / 64};
  tc_run(p, a.status, a.stages);
}

// ---------------------------------------------------------------------------
// Dense rowdot (rows of one or two matrices, two 64-row tiles per stage),
// with the K range of a 128-row tile split ks = 2^kslog ways: unit u is tile
// u / ks, part u % ks (the parts reduced in order by tc_reduce_parts)
// ---------------------------------------------------------------------------

struct TcDenseProblem {
  static constexpr int kAMajorMN = 0;
  static constexpr bool kGather = false;
  static constexpr bool kRowsPerUnit = true;
  const TcMaps& m;
  TcDenseArgs a;
  int C;   // 64-column chunks of K
  int p1;  // rows of the first block, padded to 64
  int* s_flag;
  __device__ int units() const { return ((p1 + a.n2 + TC_M - 1) / TC_M) << a.kslog; }
  __device__ int c0(int unit) const { return ((unit & ((1 << a.kslog) - 1)) * C) >> a.kslog; }
  __device__ int chunks(int unit) const {
    return ((((unit & ((1 << a.kslog) - 1)) + 1) * C) >> a.kslog) - c0(unit);
  }
  __device__ bool live(int, int) const { return true; }
  __device__ bool any(int) const { return true; }
  __device__ void rows(int, int, int, int (&)[4]) const {}
  __device__ void issue(uint32_t st, uint64_t* full, int unit, int c, int, const int (&)[4]) const {
    const int y = (unit >> a.kslog) * TC_M, x = (c0(unit) + c) * TC_K;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int yv = y + 64 * k;  // rows past both blocks read zeros
      if (yv < p1) tma_load_2d(st + k * 8192, &m.w, x, yv, full);
      else tma_load_2d(st + k * 8192, &m.w2, x, yv - p1, full);
    }
    tc_issue_operand(m, st, full, x);
  }
  __device__ void epilogue(int unit, int mrow, int, const float (&v0)[16], bool) const {
    float v[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) v[b] = v0[b];
    const int tile = unit >> a.kslog;
    if (!tc_reduce_parts(a.red, a.tick, tile, unit & ((1 << a.kslog) - 1), 1 << a.kslog, a.nb, mrow, v, s_flag))
      return;
    const int row = tile * TC_M + mrow;
    float* out;
    long long ld;
    float bias = 0.f;
    int i;
    if (row < p1) {
      if (row >= a.n1) return;
      i = row;
      out = a.out1;
      ld = a.ldo1;
      if (a.bias1) bias = a.bias1[i];
    } else {
      i = row - p1;
      if (i >= a.n2) return;
      out = a.out2;
      ld = a.ldo2;
      if (a.bias2) bias = a.bias2[i];
    }
#pragma unroll
    for (int b = 0; b < TC_N; ++b) {
      if (b >= a.nb) break;
      out[(size_t)b * ld + i] = v[b] + bias;
    }
  }
};

__global__ void __launch_bounds__(TC_THREADS, 2) tc_dense_kernel(const __grid_constant__ TcMaps m, TcDenseArgs a) {
  __shared__ int s_flag;
  griddep_launch();
  griddep_wait();
  TcDenseProblem p{m, a, (a.K + TC_K - 1) / TC_K, (a.n1 + 63) / 64 * 64, &s_flag};
  tc_run(p, a.status, a.stages);
}

}  // namespace dv
