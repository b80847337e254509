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
// The activations enter as two bf16 arrays, hi = bf16(v) and lo =
// bf16(v - hi) (tc_split_kernel, or the W1 kernel's epilogue for the W2
// operand), so hi + lo carries 16 significant bits of every activation:
// D = W X_hi + W X_lo is accurate to about 2^-16 relative instead of the 2^-9
// of one bf16 rounding, at twice the (idle) tensor work.
//
// Per CTA (128 threads, one CTA per SM, persistent over work units):
//   * all threads stage the weight tile (bf16, 16 KB) and the operand blocks
//     (16 x 64, hi and lo) of a stage with 16-byte cp.async copies, six stages
//     ahead, straight into the canonical no-swizzle UMMA layout (8 x 16-byte
//     core matrices); each thread keeps the pointers of its 8 weight rows for
//     the unit (rowdot) or the chunk (rowaxpy);
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
constexpr int TC_STAGES = 8;
constexpr int TC_DIST = TC_STAGES - 2;  // stages in flight ahead of the one consumed
constexpr int TC_A_BYTES = TC_M * TC_K * 2;  // 16 KB weight tile
constexpr int TC_B_BYTES = TC_N * TC_K * 2;  // 2 KB bf16 operand (hi or lo)
constexpr int TC_STAGE_BYTES = TC_A_BYTES + 2 * TC_B_BYTES;
constexpr size_t TC_SMEM = 1024 + (size_t)TC_STAGES * TC_STAGE_BYTES;
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

// Copies the stage's operand blocks: batch row n (< nb, zero otherwise),
// elements k0 .. k0+63 of hi[n * ld] and lo[n * ld], the first `valid` of
// them (the rest zero; valid is a multiple of 8 or the tail of the row).
// Thread t copies row t/8, 16-byte piece t%8, of both.
__device__ __forceinline__ void tc_load_operand(unsigned char* stage, const __nv_bfloat16* hi,
                                                const __nv_bfloat16* lo, long long ld, int nb, int k0, int valid) {
  const int t = threadIdx.x;
  const int n = t >> 3, k8 = t & 7;
  const bool ok = n < nb && k8 * 8 < valid;
  const long long off = ok ? (long long)n * ld + k0 + k8 * 8 : 0;
  const int dst = (n >> 3) * 1024 + k8 * 128 + (n & 7) * 16;
  cp_async16_zfill(stage + TC_OFF_BHI + dst, hi + off, ok ? 16 : 0);
  cp_async16_zfill(stage + TC_OFF_BLO + dst, lo + off, ok ? 16 : 0);
}

// This thread's 8 rows of a tile (pointers; null: a zero row). rowdot:
// piece j of thread t is tile row (t%8) + 8 (t/64) + 16 j, column piece
// (t/8)%8; rowaxpy: chunk row (t%8) + 8 j, column piece (t/8)%16.
__device__ __forceinline__ int tc_rowdot_row(int j) { return (threadIdx.x & 7) + 8 * (threadIdx.x >> 6) + 16 * j; }
__device__ __forceinline__ int tc_rowaxpy_row(int j) { return (threadIdx.x & 7) + 8 * j; }

// rowdot weight tile, K-major: columns k0 .. k0+63 of the 8 rows rp[j]
// (columns >= d zero).
__device__ __forceinline__ void tc_load_tile_kmajor(unsigned char* stage, const __nv_bfloat16* const (&rp)[8], int k0,
                                                    int d, const void* dummy) {
  const int t = threadIdx.x;
  const int k8 = (t >> 3) & 7;
  const int col = k0 + k8 * 8;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int m = tc_rowdot_row(j);
    const bool ok = rp[j] != nullptr && col < d;
    cp_async16_zfill(stage + (m >> 3) * 1024 + k8 * 128 + (m & 7) * 16, ok ? (const void*)(rp[j] + col) : dummy,
                     ok ? 16 : 0);
  }
}

// rowaxpy weight tile, MN-major: columns col0 .. col0+127 of the 8 rows rp[j]
// (columns >= d zero).
__device__ __forceinline__ void tc_load_tile_mnmajor(unsigned char* stage, const __nv_bfloat16* const (&rp)[8],
                                                     int col0, int d, const void* dummy) {
  const int t = threadIdx.x;
  const int c8 = (t >> 3) & 15;
  const int col = col0 + c8 * 8;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const bool ok = rp[j] != nullptr && col < d;
    cp_async16_zfill(stage + j * 2048 + c8 * 128 + (t & 7) * 16, ok ? (const void*)(rp[j] + col) : dummy,
                     ok ? 16 : 0);
  }
}

// ---------------------------------------------------------------------------
// The pipeline (shared by both forms)
// ---------------------------------------------------------------------------
//
// A problem P provides:
//   static constexpr int kAMajorMN;               // 0 rowdot, 1 rowaxpy
//   static constexpr bool kRowsPerUnit;           // rows() depends on the unit only
//   __device__ int units() const;                 // work units in total
//   __device__ int chunks(int unit) const;        // stages of K in a unit (>= 1 for every unit)
//   __device__ bool live(int unit, int c) const;  // false: the stage is empty (no copies, no MMA)
//   __device__ void rows(int unit, int c, const bf16* (&rp)[8]) const;  // this thread's 8 weight rows
//   __device__ void load(unsigned char* stage, int unit, int c, const bf16* const (&rp)[8]) const;
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
  const __nv_bfloat16* rp[8];
  auto produce = [&]() {
    if (prod_u < nunits) {
      const int s = issued % TC_STAGES;
      if (issued >= TC_STAGES && !mbar_wait_bounded(&bar_free[s], ((issued / TC_STAGES) - 1) & 1)) {
        if (!abort_local) raise_status(status, DV_DEV_TIMEOUT_BIT);
        abort_local = 1;
      }
      if (!abort_local && p.live(prod_u, prod_c)) {
        if (!P::kRowsPerUnit || prod_c == 0) p.rows(prod_u, prod_c, rp);
        p.load(smem + (size_t)s * TC_STAGE_BYTES, prod_u, prod_c, rp);
      }
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

// ---------------------------------------------------------------------------
// q, k, v of the selected heads (rowdot over Wqkv rows)
// ---------------------------------------------------------------------------

struct TcQkvProblem {
  static constexpr int kAMajorMN = 0;
  static constexpr bool kRowsPerUnit = true;
  TcQkvArgs a;
  int nslots;  // selected heads x 3 dh
  __device__ int units() const { return (nslots + TC_M - 1) / TC_M; }
  __device__ int chunks(int) const { return (a.d + TC_K - 1) / TC_K; }
  __device__ bool live(int, int) const { return true; }
  __device__ void rows(int unit, int, const __nv_bfloat16* (&rp)[8]) const {
    const int per = 3 * a.dh;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int s = unit * TC_M + tc_rowdot_row(j);
      const __nv_bfloat16* r = nullptr;
      if (s < nslots) {
        const int head = a.head_idx[s / per];
        if (head >= 0 && head < a.h) r = a.Wqkv + ((size_t)head * per + s % per) * a.d;
      }
      rp[j] = r;
    }
  }
  __device__ void load(unsigned char* stage, int, int c, const __nv_bfloat16* const (&rp)[8]) const {
    tc_load_tile_kmajor(stage, rp, c * TC_K, a.d, a.Wqkv);
    tc_load_operand(stage, a.xhi, a.xlo, a.d, a.nb, c * TC_K, a.d - c * TC_K);
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
  static constexpr bool kRowsPerUnit = true;
  TcMlpArgs a;
  int cnt;
  int* s_warp;  // [4] shared: per-warp nonzero counts
  __device__ int units() const { return (cnt + TC_M - 1) / TC_M; }
  __device__ int chunks(int) const { return (a.d + TC_K - 1) / TC_K; }
  __device__ bool live(int, int) const { return true; }
  __device__ void rows(int unit, int, const __nv_bfloat16* (&rp)[8]) const {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int s = unit * TC_M + tc_rowdot_row(j);
      const int r = s < cnt ? a.idx[s] : -1;
      rp[j] = (r >= 0 && r < a.N) ? a.W1t + (size_t)r * a.d : nullptr;
    }
  }
  __device__ void load(unsigned char* stage, int, int c, const __nv_bfloat16* const (&rp)[8]) const {
    tc_load_tile_kmajor(stage, rp, c * TC_K, a.d, a.W1t);
    tc_load_operand(stage, a.xhi, a.xlo, a.d, a.nb, c * TC_K, a.d - c * TC_K);
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
    if (nz) {  // the nonzero activations at their compacted slot
      const int slot = before + __popc(bal & ((1u << lane) - 1u));
#pragma unroll
      for (int b = 0; b < TC_N; ++b) {
        if (b >= a.nb) break;
        const __nv_bfloat16 h = __float2bfloat16_rn(act[b]);
        a.act_hi[(size_t)b * a.KC + base + slot] = h;
        a.act_lo[(size_t)b * a.KC + base + slot] = __float2bfloat16_rn(act[b] - __bfloat162float(h));
      }
      a.rowid_c[base + slot] = r;
    }
    if (m >= total) {  // zeros after the tile's count (the W2 operand reads 8-slot pieces)
      const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
      for (int b = 0; b < TC_N; ++b) {
        if (b >= a.nb) break;
        a.act_hi[(size_t)b * a.KC + base + m] = z;
        a.act_lo[(size_t)b * a.KC + base + m] = z;
      }
    }
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
  static constexpr bool kRowsPerUnit = false;
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
  __device__ void rows(int unit, int c, const __nv_bfloat16* (&rp)[8]) const {
    const int t = (unit / n_mt) * a.tiles_per_group + (c >> 1), half = c & 1;
    const int n = s_cnt[t] - half * 64;
    const int base = t * TC_M + half * 64;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int kr = tc_rowaxpy_row(j);
      rp[j] = kr < n ? a.W2t + (size_t)a.rowid_c[base + kr] * a.d : nullptr;
    }
  }
  __device__ void load(unsigned char* stage, int unit, int c, const __nv_bfloat16* const (&rp)[8]) const {
    const int t = (unit / n_mt) * a.tiles_per_group + (c >> 1), half = c & 1;
    const int n = s_cnt[t] - half * 64;  // > 0 (live)
    tc_load_tile_mnmajor(stage, rp, (unit % n_mt) * TC_M, a.d, a.W2t);
    const int valid = n < 64 ? (n + 7) & ~7 : 64;  // the slots after the count hold zeros
    tc_load_operand(stage, a.act_hi, a.act_lo, a.KC, a.nb, t * TC_M + half * 64, valid);
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
// W^O of the selected heads (rowaxpy over WOt rows; operand H as hi / lo)
// ---------------------------------------------------------------------------

struct TcWoProblem {
  static constexpr int kAMajorMN = 1;
  static constexpr bool kRowsPerUnit = false;
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
  __device__ void rows(int unit, int c, const __nv_bfloat16* (&rp)[8]) const {
    const int p = (unit / n_mt) * a.heads_per_group + c / cph, part = c % cph;
    const int head = a.head_idx[p];
    const bool ok = head >= 0 && head < a.h;
    const __nv_bfloat16* rows0 = a.WOt + ((size_t)(ok ? head : 0) * a.dh + part * 64) * a.d;
#pragma unroll
    for (int j = 0; j < 8; ++j) rp[j] = ok ? rows0 + (size_t)tc_rowaxpy_row(j) * a.d : nullptr;
  }
  __device__ void load(unsigned char* stage, int unit, int c, const __nv_bfloat16* const (&rp)[8]) const {
    const int p = (unit / n_mt) * a.heads_per_group + c / cph, part = c % cph;
    tc_load_tile_mnmajor(stage, rp, (unit % n_mt) * TC_M, a.d, a.WOt);
    tc_load_operand(stage, a.hhi, a.hlo, (long long)a.kh_max * a.dh, a.nb, p * a.dh + part * 64, 64);
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
