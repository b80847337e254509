// Tensor-core gathered-row kernels (tcgen05, sm_100a) for batch 5..16.
//
// At batch B the selected rows of W1, W2, W^{Q,K,V} and W^O meet B input
// vectors: a gathered row times a [d][B] block is a thin dense contraction
// (B flop per weight byte), which the CUDA cores cannot keep up with at HBM
// rate once B reaches 8-16, so these kernels hand the multiply-adds to the
// 5th-generation tensor cores and keep the SMs' issue slots for the loads.
//
// Two kernel forms share one pipeline:
//   rowdot  D[m][b] = sum_c W[row(m)][c] X[b][c]    rows of W are K-major
//           (q, k, v of the selected heads; the MLP's first layer)
//   rowaxpy D[c][b] = sum_j W[row(j)][c] S[b][j]    rows of W are MN-major
//           (W^O of the selected heads; the MLP's second layer)
// with M = 128 (gathered rows, or output columns), N = 16 (the batch rows,
// zero-padded) and 64 K-elements per pipeline stage.
//
// Per CTA (128 threads, one CTA per SM, persistent over work units):
//   * all threads stage the weight tile (bf16, 16 KB) and the fp32 operand
//     block (16 x 64) of a stage with 16-byte cp.async copies, four stages
//     ahead, into the canonical no-swizzle UMMA layout (8 x 16-byte core
//     matrices);
//   * at consume time the fp32 operand block is split into two bf16 blocks,
//     hi = bf16(v) and lo = bf16(v - hi), so hi + lo carries 16 significant
//     bits of every activation: D = W (X_hi + X_lo) is fp32-accurate to about
//     2^-16 relative instead of the 2^-9 of one bf16 rounding;
//   * thread 0 issues the MMAs (tcgen05.mma kind::f16, bf16 inputs, fp32
//     accumulator in tensor memory, 32 TMEM columns) and commits them to the
//     stage's mbarrier, which frees the stage for its next copies;
//   * at the end of a unit the four warps read the 128 x 16 accumulator
//     (tcgen05.ld 32x32b, warp w owns TMEM lanes 32w..32w+31) and run the
//     unit's epilogue.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on a timeout
// the kernel sets DV_DEV_TIMEOUT in the status word, stops issuing work,
// waits for its own copies, releases its tensor memory and returns.
#pragma once

#include "dv_common.cuh"
#include "dv_tc_args.h"

namespace dv {

constexpr int TC_THREADS = 128;
constexpr int TC_K = 64;        // K elements per stage
constexpr int TC_STAGES = 6;
constexpr int TC_DIST = TC_STAGES - 2;  // stages in flight ahead of the one consumed
constexpr int TC_A_BYTES = TC_M * TC_K * 2;       // 16 KB weight tile
constexpr int TC_B_BYTES = TC_N * TC_K * 2;       // 2 KB bf16 operand (hi or lo)
constexpr int TC_S_BYTES = TC_N * TC_K * 4;       // 4 KB fp32 operand staging
constexpr int TC_STAGE_BYTES = TC_A_BYTES + 2 * TC_B_BYTES + TC_S_BYTES;
// Slack after the last stage: every descriptor's reach stays inside the
// allocation even if its two strides were read the other way round.
constexpr int TC_SLACK = 32 * 1024;
constexpr size_t TC_SMEM = 1024 + (size_t)TC_STAGES * TC_STAGE_BYTES + TC_SLACK;
constexpr int TC_TMEM_COLS = 32;
constexpr int TC_TILES_PER_GROUP = 8;  // rowdot tiles per rowaxpy unit of the MLP (1024 neurons), at most
constexpr int TC_HEADS_PER_GROUP = 4;  // heads per rowaxpy unit of W^O, at most

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_n() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_none() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the phase with the given parity to complete, for at most about
// two seconds; false on a timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > 2000000000ull) return false;
  }
  return true;
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

// Shared-memory matrix descriptor, no swizzle (canonical layout of 8-row x
// 16-byte core matrices): start address, the byte distance between core
// matrices along K (lbo) and along M/N (sbo), descriptor version 1.
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, B
// K-major, A K-major (a_mn = 0) or MN-major (a_mn = 1), shape M x N.
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N, int a_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Shared-memory stage layout (offsets inside one stage)
// ---------------------------------------------------------------------------
//   A    [0, 16 KB)      weight tile, canonical no-swizzle layout
//   Bhi  [16, 18 KB)     operand hi part, [n/8][k/8][n%8][k%8] (K-major)
//   Blo  [18, 20 KB)     operand lo part
//   S    [20, 24 KB)     fp32 operand staging, [n][64]
//
// rowdot A (K-major, 128 rows x 64 K): byte (m/8)*1024 + (k/8)*128 +
// (m%8)*16 + (k%8)*2, so lbo = 128, sbo = 1024, and the K = 16 slice kk of
// the stage starts at kk * 256.
// rowaxpy A (MN-major, 128 columns x 64 K rows): byte (k/8)*2048 +
// (m/8)*128 + (k%8)*16 + (m%8)*2, so sbo = 128, lbo = 2048, and the K = 16
// slice kk starts at kk * 4096.
// B (K-major, 16 x 64): byte (n/8)*1024 + (k/8)*128 + (n%8)*16 + (k%8)*2,
// lbo = 128, sbo = 1024, slice kk at kk * 256.
constexpr int TC_OFF_BHI = TC_A_BYTES;
constexpr int TC_OFF_BLO = TC_A_BYTES + TC_B_BYTES;
constexpr int TC_OFF_S = TC_A_BYTES + 2 * TC_B_BYTES;

// Splits the stage's fp32 staging block into the hi / lo bf16 operand
// blocks. Each thread converts exactly the pieces it copied itself
// (tc_stage_operand: batch rows t/16 and t/16 + 8, 16-byte piece t%16), so
// its own cp.async wait is all the ordering the conversion needs.
__device__ __forceinline__ void tc_split_operand(unsigned char* stage) {
  const int t = threadIdx.x;
  const int q = t & 15;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int n = (t >> 4) + 8 * h;
    const float4 a = *reinterpret_cast<const float4*>(stage + TC_OFF_S + n * 256 + q * 16);
    const float v[4] = {a.x, a.y, a.z, a.w};
    uint32_t hi[2], lo[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * i]), h1 = __float2bfloat16_rn(v[2 * i + 1]);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(v[2 * i] - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(v[2 * i + 1] - __bfloat162float(h1));
      hi[i] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lo[i] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    // elements k = 4q .. 4q+3 of row n: core matrix k/8 = q/2, bytes (k%8)*2 = (q%2)*8
    const int off = (n >> 3) * 1024 + (q >> 1) * 128 + (n & 7) * 16 + (q & 1) * 8;
    *reinterpret_cast<uint2*>(stage + TC_OFF_BHI + off) = make_uint2(hi[0], hi[1]);
    *reinterpret_cast<uint2*>(stage + TC_OFF_BLO + off) = make_uint2(lo[0], lo[1]);
  }
}

// Stages the fp32 operand block of a stage: batch row n (< nb, zero
// otherwise), 64 consecutive elements from src + n * ld, the first `valid`
// of them (the rest zero). Thread t copies rows t/16 and t/16 + 8, 16-byte
// piece t%16 of each.
__device__ __forceinline__ void tc_stage_operand(unsigned char* stage, const float* src, long long ld, int nb,
                                                 int valid) {
  const int t = threadIdx.x;
  const int q = t & 15;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int n = (t >> 4) + 8 * h;
    int bytes = 0;
    if (n < nb) {
      const int rem = valid - q * 4;
      bytes = rem >= 4 ? 16 : (rem > 0 ? rem * 4 : 0);
    }
    const float* p = bytes ? src + (long long)n * ld + q * 4 : src;
    cp_async16_zfill(stage + TC_OFF_S + n * 256 + q * 16, p, bytes);
  }
}

// ---------------------------------------------------------------------------
// The pipeline (shared by both forms)
// ---------------------------------------------------------------------------
//
// A problem P provides:
//   static constexpr int kAMajorMN;               // 0 rowdot, 1 rowaxpy
//   __device__ int units() const;                 // work units in total
//   __device__ int chunks(int unit) const;        // stages of K in a unit (>= 1 for every unit)
//   __device__ bool live(int unit, int c) const;  // false: the stage is empty (no copies, no MMA)
//   __device__ void load(unsigned char* stage, int unit, int c) const;   // issue the stage's copies
//   __device__ void epilogue(int unit, int m, const float (&v)[16], bool any) const;
// The epilogue is called by all 128 threads together (it may use
// __syncthreads); thread m holds accumulator row m. `any` is false when the
// unit issued no MMA (its accumulator is then taken as zero).
//
// Timeouts are agreed on with __syncthreads_or, so every thread leaves the
// loop at the same barrier.

template <class P>
__device__ void tc_run(const P& p, int* status) {
  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  __shared__ __align__(8) uint64_t bar_free[TC_STAGES];
  __shared__ __align__(8) uint64_t bar_done;
  __shared__ uint32_t s_tmem;
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0) {
    tmem_alloc(&s_tmem, TC_TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < TC_STAGES; ++s) mbar_init(&bar_free[s], 1);
    mbar_init(&bar_done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  constexpr uint32_t idesc = tc_idesc(TC_M, TC_N, P::kAMajorMN);
  int abort_local = 0;

  // this CTA's units are blockIdx.x, + gridDim.x, ...; its chunk sequence is
  // the concatenation of their chunks, walked by the producer TC_DIST
  // chunks ahead of the consumer
  const int nunits = p.units();
  int prod_u = blockIdx.x, prod_c = 0;
  int issued = 0;
  auto produce = [&]() {
    if (prod_u < nunits) {
      const int s = issued % TC_STAGES;
      if (issued >= TC_STAGES && !mbar_wait_bounded(&bar_free[s], ((issued / TC_STAGES) - 1) & 1)) {
        if (!abort_local) raise_status(status, DV_DEV_TIMEOUT_BIT);
        abort_local = 1;
      }
      if (!abort_local && p.live(prod_u, prod_c)) p.load(smem + (size_t)s * TC_STAGE_BYTES, prod_u, prod_c);
      if (++prod_c >= p.chunks(prod_u)) {
        prod_c = 0;
        prod_u += gridDim.x;
      }
      ++issued;
    }
    cp_async_commit();
  };
  for (int i = 0; i < TC_DIST; ++i) produce();

  int u = blockIdx.x, c = 0;
  int consumed = 0, units_done = 0;
  bool unit_any = false;  // the current unit issued an MMA
  while (u < nunits) {
    produce();
    cp_async_wait_n<TC_DIST>();
    const int s = consumed % TC_STAGES;
    unsigned char* stage = smem + (size_t)s * TC_STAGE_BYTES;
    const bool live = p.live(u, c);
    if (live) tc_split_operand(stage);
    fence_proxy_async_smem();
    tc_fence_before();
    if (__syncthreads_or(abort_local)) break;
    const bool last = c + 1 >= p.chunks(u);
    if (tid == 0) {
      tc_fence_after();
      if (live) {
        const uint32_t a0 = smem_u32(stage), b0 = smem_u32(stage + TC_OFF_BHI), l0 = smem_u32(stage + TC_OFF_BLO);
#pragma unroll
        for (int kk = 0; kk < TC_K / 16; ++kk) {
          const uint64_t ad = P::kAMajorMN ? tc_sdesc(a0 + kk * 4096, 2048, 128) : tc_sdesc(a0 + kk * 256, 128, 1024);
          tc_mma(tmem, ad, tc_sdesc(b0 + kk * 256, 128, 1024), idesc, (unit_any || kk > 0) ? 1u : 0u);
          tc_mma(tmem, ad, tc_sdesc(l0 + kk * 256, 128, 1024), idesc, 1u);
        }
      }
      tc_commit(&bar_free[s]);
      if (last) tc_commit(&bar_done);
    }
    unit_any = unit_any || live;
    ++consumed;
    if (last) {
      if (!mbar_wait_bounded(&bar_done, units_done & 1)) {
        if (!abort_local) raise_status(status, DV_DEV_TIMEOUT_BIT);
        abort_local = 1;
      }
      if (__syncthreads_or(abort_local)) break;
      tc_fence_after();
      float v[16];
      if (unit_any) {
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), v);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      p.epilogue(u, warp * 32 + lane, v, unit_any);
      tc_fence_before();
      ++units_done;
      unit_any = false;
    }
    if (++c >= p.chunks(u)) {
      c = 0;
      u += gridDim.x;
    }
  }
  cp_async_wait_none();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TC_TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Weight tiles
// ---------------------------------------------------------------------------

// rowdot tile: 128 rows (row_of(m): pointer to row m, or null for a zero
// row) x 64 columns from k0 (columns >= d zero). Thread t copies pieces
// i = t + 128 j, j < 8: row (i % 8) + 8 (i / 64), 16-byte column piece
// (i / 8) % 8, so eight consecutive threads fill one 128-byte core matrix.
template <class RowOf>
__device__ __forceinline__ void tc_load_rows_kmajor(unsigned char* stage, const RowOf& row_of, int k0, int d,
                                                    const void* dummy) {
  const int t = threadIdx.x;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = t + 128 * j;
    const int m = (i & 7) + 8 * (i >> 6), k8 = (i >> 3) & 7;
    const int col = k0 + k8 * 8;
    const __nv_bfloat16* r = row_of(m);
    const bool ok = r != nullptr && col < d;
    cp_async16_zfill(stage + (m >> 3) * 1024 + k8 * 128 + (m & 7) * 16, ok ? (const void*)(r + col) : dummy,
                     ok ? 16 : 0);
  }
}

// rowaxpy tile: 64 rows (row_of(j), null for zero) x 128 columns from col0
// (columns >= d zero), MN-major. Thread t copies pieces i = t + 128 j, j < 8:
// row (i % 8) + 8 (i / 128), 16-byte column piece (i / 8) % 16.
template <class RowOf>
__device__ __forceinline__ void tc_load_rows_mnmajor(unsigned char* stage, const RowOf& row_of, int col0, int d,
                                                     const void* dummy) {
  const int t = threadIdx.x;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = t + 128 * j;
    const int kr = (i & 7) + 8 * j, c8 = (i >> 3) & 15;
    const int col = col0 + c8 * 8;
    const __nv_bfloat16* r = row_of(kr);
    const bool ok = r != nullptr && col < d;
    cp_async16_zfill(stage + j * 2048 + c8 * 128 + (i & 7) * 16, ok ? (const void*)(r + col) : dummy, ok ? 16 : 0);
  }
}

// ---------------------------------------------------------------------------
// q, k, v of the selected heads (rowdot over Wqkv rows)
// ---------------------------------------------------------------------------


struct TcQkvProblem {
  static constexpr int kAMajorMN = 0;
  TcQkvArgs a;
  int nslots;  // selected heads x 3 dh
  __device__ int units() const { return (nslots + TC_M - 1) / TC_M; }
  __device__ int chunks(int) const { return (a.d + TC_K - 1) / TC_K; }
  __device__ bool live(int, int) const { return true; }
  __device__ const __nv_bfloat16* row(int s) const {
    if (s >= nslots) return nullptr;
    const int per = 3 * a.dh;
    const int head = a.head_idx[s / per];
    if (head < 0 || head >= a.h) return nullptr;
    return a.Wqkv + ((size_t)head * per + s % per) * a.d;
  }
  __device__ void load(unsigned char* stage, int unit, int c) const {
    const int base = unit * TC_M;
    tc_load_rows_kmajor(stage, [&](int m) { return row(base + m); }, c * TC_K, a.d, a.Wqkv);
    tc_stage_operand(stage, a.y + c * TC_K, a.d, a.nb, a.d - c * TC_K);
  }
  __device__ void epilogue(int unit, int m, const float (&v)[16], bool) const {
    const int per = 3 * a.dh;
    const int s = unit * TC_M + m;
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

__global__ void __launch_bounds__(TC_THREADS, 1) tc_qkv_kernel(TcQkvArgs a) {
  griddep_launch();
  griddep_wait();
  int hc = *a.head_count;
  if (hc > a.kh_max || hc < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, 1);
    hc = hc < 0 ? 0 : a.kh_max;
  }
  TcQkvProblem p{a, hc * 3 * a.dh};
  tc_run(p, a.status);
}

// ---------------------------------------------------------------------------
// The MLP: activations of the selected neurons (rowdot over W1 rows, with
// bias, ReLU and per-tile compaction of the nonzero ones), then the
// gather-axpy of their W2 rows (rowaxpy)
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
  TcMlpArgs a;
  int cnt;
  int* s_warp;  // [5] shared: per-warp nonzero counts
  __device__ int units() const { return (cnt + TC_M - 1) / TC_M; }
  __device__ int chunks(int) const { return (a.d + TC_K - 1) / TC_K; }
  __device__ bool live(int, int) const { return true; }
  __device__ const __nv_bfloat16* row(int s) const {
    if (s >= cnt) return nullptr;
    const int r = a.idx[s];
    return (r >= 0 && r < a.N) ? a.W1t + (size_t)r * a.d : nullptr;
  }
  __device__ void load(unsigned char* stage, int unit, int c) const {
    const int base = unit * TC_M;
    tc_load_rows_kmajor(stage, [&](int m) { return row(base + m); }, c * TC_K, a.d, a.W1t);
    tc_stage_operand(stage, a.y + c * TC_K, a.d, a.nb, a.d - c * TC_K);
  }
  __device__ void epilogue(int unit, int m, const float (&v)[16], bool) const {
    const int s = unit * TC_M + m;
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
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned bal = __ballot_sync(0xffffffffu, nz);
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < TC_THREADS / 32; ++w) {
      const int n = s_warp[w];
      before += w < warp ? n : 0;
      total += n;
    }
    const int base = unit * TC_M;
    if (nz) {
      const int pos = before + __popc(bal & ((1u << lane) - 1u));
      for (int b = 0; b < a.nb; ++b) a.act_c[(size_t)b * a.KC + base + pos] = act[b];
      a.rowid_c[base + pos] = r;
    }
    if (m >= total)  // the slots after the tile's count hold zero activations
      for (int b = 0; b < a.nb; ++b) a.act_c[(size_t)b * a.KC + base + m] = 0.f;
    if (threadIdx.x == 0) a.tile_cnt[unit] = total;
    __syncthreads();  // s_warp is reused by the next unit
  }
};

__global__ void __launch_bounds__(TC_THREADS, 1) tc_w1_kernel(TcMlpArgs a) {
  __shared__ int s_warp[TC_THREADS / 32];
  griddep_launch();
  griddep_wait();
  TcW1Problem p{a, tc_clamped_count(a.count, a.k_max, a.status), s_warp};
  tc_run(p, a.status);
}

struct TcW2Problem {
  static constexpr int kAMajorMN = 1;
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
  __device__ void load(unsigned char* stage, int unit, int c) const {
    const int g = unit / n_mt, mt = unit % n_mt;
    const int t = g * a.tiles_per_group + (c >> 1), half = c & 1;
    const int n = s_cnt[t] - half * 64;  // > 0 (live)
    const int base = t * TC_M + half * 64;
    tc_load_rows_mnmajor(stage,
                         [&](int j) -> const __nv_bfloat16* {
                           return j < n ? a.W2t + (size_t)a.rowid_c[base + j] * a.d : nullptr;
                         },
                         mt * TC_M, a.d, a.W2t);
    tc_stage_operand(stage, a.act_c + base, a.KC, a.nb, n < 64 ? n : 64);
  }
  __device__ void epilogue(int unit, int m, const float (&v)[16], bool any) const {
    const int g = unit / n_mt, mt = unit % n_mt;
    const int col = mt * TC_M + m;
    if (col >= a.d) return;
    const float bias = (g == 0 && a.b2) ? a.b2[col] : 0.f;
    if (!any && bias == 0.f) return;
#pragma unroll
    for (int b = 0; b < TC_N; ++b) {
      if (b >= a.nb) break;
      atomicAdd(a.out + (size_t)b * a.d + col, v[b] + bias);
    }
  }
};

__global__ void __launch_bounds__(TC_THREADS, 1) tc_w2_kernel(TcMlpArgs a) {
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
  TcW2Problem p{a, ntiles, n_mt, n_groups, s_cnt};
  tc_run(p, a.status);
}

// ---------------------------------------------------------------------------
// W^O of the selected heads (rowaxpy over WOt rows; operand H)
// ---------------------------------------------------------------------------


struct TcWoProblem {
  static constexpr int kAMajorMN = 1;
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
  __device__ bool live(int unit, int c) const { return c / cph < heads_in(unit / n_mt); }
  __device__ void load(unsigned char* stage, int unit, int c) const {
    const int g = unit / n_mt, mt = unit % n_mt;
    const int p = g * a.heads_per_group + c / cph, part = c % cph;
    const int head = a.head_idx[p];
    const bool ok = head >= 0 && head < a.h;
    const __nv_bfloat16* rows = a.WOt + ((size_t)(ok ? head : 0) * a.dh + part * 64) * a.d;
    tc_load_rows_mnmajor(stage, [&](int j) -> const __nv_bfloat16* { return ok ? rows + (size_t)j * a.d : nullptr; },
                         mt * TC_M, a.d, a.WOt);
    tc_stage_operand(stage, a.H + (size_t)p * a.dh + part * 64, (long long)a.kh_max * a.dh, a.nb, ok ? 64 : 0);
  }
  __device__ void epilogue(int unit, int m, const float (&v)[16], bool any) const {
    const int g = unit / n_mt, mt = unit % n_mt;
    const int col = mt * TC_M + m;
    if (col >= a.d) return;
    const float bias = (g == 0 && a.bO) ? a.bO[col] : 0.f;
    if (!any && bias == 0.f) return;
#pragma unroll
    for (int b = 0; b < TC_N; ++b) {
      if (b >= a.nb) break;
      atomicAdd(a.out + (size_t)b * a.d + col, v[b] + bias);
    }
  }
};

__global__ void __launch_bounds__(TC_THREADS, 1) tc_wo_kernel(TcWoArgs a) {
  griddep_launch();
  griddep_wait();
  const int hc = tc_clamped_count(a.head_count, a.kh_max, a.status);
  const int n_mt = (a.d + TC_M - 1) / TC_M;
  const int n_groups = hc > 0 ? (hc + a.heads_per_group - 1) / a.heads_per_group : 1;
  TcWoProblem p{a, hc, n_mt, n_groups, a.dh / 64};
  tc_run(p, a.status);
}

}  // namespace dv
