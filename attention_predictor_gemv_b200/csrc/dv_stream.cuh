// Streaming variants of the column-owner kernels for long rows (16 KB and
// more: d >= 8192 in bf16), where a CTA streams tens of rows and the
// register-resident loads of dv_colowner.cuh leave the memory pipe idle
// between row groups.
//
// Rows pass through a ring of ST_SLOTS row slots in shared memory. Each of the
// CTA's 256 threads copies its own 16-byte column vectors of upcoming rows into
// the ring (cp.async, 16 bytes, through L2 only) and later reads back only what
// it copied itself, so the ring needs no CTA barrier: a thread's
// cp.async.wait_group orders its own copies. ST_SLOTS - 1 rows are in flight
// while the CTA consumes one. The partial dot products of each warp collect in
// shared memory and are summed across the CTA once per ST_RB rows.
#pragma once

#include "dv_colowner.cuh"

namespace dv {

constexpr int ST_SLOTS = 8;  // row slots of the ring
constexpr int ST_RB = 16;    // rows per CTA reduction
constexpr int ST_CH = 64;    // MLP: selection slots per chunk (W1 pass, then their W2 rows)

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Ring layout: [S][NV][CO_THREADS] 16-byte vectors (S slots, ST_SLOTS by
// default).
template <int NV, int S = ST_SLOTS>
__device__ __forceinline__ uint4* st_vec(uint4* ring, int slot, int j) {
  return ring + ((size_t)(slot % S) * NV + j) * CO_THREADS + threadIdx.x;
}

// Copies this thread's vectors of `row` (null: nothing) into `slot` and
// closes one cp.async group (empty when row is null).
template <typename T, int NV, int S = ST_SLOTS>
__device__ __forceinline__ void st_issue(uint4* ring, int slot, const T* row, int nvec) {
  constexpr int E = WT<T>::E;
  if (row) {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int v = j * CO_THREADS + threadIdx.x;
      if (v < nvec) cp_async16(st_vec<NV, S>(ring, slot, j), row + (size_t)v * E);
    }
  }
  cp_async_commit();
}

// This thread's vectors of the row in `slot` (zero past the row's end).
template <int NV, int S = ST_SLOTS>
__device__ __forceinline__ void st_read(uint4* ring, int slot, int nvec, uint4 (&w)[NV]) {
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int v = j * CO_THREADS + threadIdx.x;
    w[j] = v < nvec ? *st_vec<NV, S>(ring, slot, j) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Issues the first S - 1 rows of [r0, r1) (always S - 1 groups).
template <typename T, int NV, int S = ST_SLOTS, class RowFn>
__device__ __forceinline__ void st_prologue(uint4* ring, int r0, int r1, int nvec, RowFn row) {
#pragma unroll 1
  for (int s = 0; s < S - 1; ++s) st_issue<T, NV, S>(ring, s, r0 + s < r1 ? row(r0 + s) : nullptr, nvec);
}

// ---- the ring filled by bulk copies (the TMA engine) ----
// One thread issues each row as one cp.async.bulk into its slot, completing
// on the slot's "full" barrier (count 1, transaction bytes); every warp
// releases a slot on its "empty" barrier (count CO_WARPS) once it has read its
// vectors, and the issuing thread waits on that before reusing the slot. The
// slot layout is the row itself (vector v of the row at v * 16 bytes), which
// is the per-thread layout above, so st_read serves both forms. Every wait is
// bounded (about 2 s, DV_DEV_TIMEOUT); after a timeout the ring's waits
// return at once, so the kernel ends with incomplete outputs.
__device__ __forceinline__ uint32_t rb_smem(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t rb_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool rb_try(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(rb_smem(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}

template <typename T, int NV, int S>
struct BulkRing {
  uint4* ring;      // [S][NV][CO_THREADS] 16-byte vectors
  uint64_t* full;   // [S]
  uint64_t* empty;  // [S]
  int* abort;       // shared: a wait timed out
  int* status;
  unsigned bytes;   // bytes of a row
  unsigned fp;      // this thread's parity of each slot's next "full" phase
  unsigned ep;      // the issuing thread's parity of each slot's next "empty" wait

  __device__ void init() {  // the caller synchronises the CTA afterwards
    fp = 0u;
    ep = ~0u;  // the first wait on a slot's "empty" barrier passes at once
    if (threadIdx.x == 0) {
      for (int s = 0; s < S; ++s) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(rb_smem(&full[s])) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(rb_smem(&empty[s])), "r"(CO_WARPS) : "memory");
      }
      *abort = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  __device__ bool wait_bar(uint64_t* bar, unsigned parity) {
    if (rb_try(bar, parity)) return true;
    const uint64_t t0 = rb_ns();
    while (!rb_try(bar, parity)) {
      if (*reinterpret_cast<volatile int*>(abort)) return false;
      if (rb_ns() - t0 > 2000000000ull) {
        *reinterpret_cast<volatile int*>(abort) = 1;
        raise_status(status, 8);
        return false;
      }
    }
    return true;
  }
  // Thread 0: the row of position p (null: a row with no data, which still
  // completes the slot's phase). Every position issued is consumed once.
  __device__ void issue(int p, const T* row) {
    if (threadIdx.x != 0) return;
    const int s = p % S;
    wait_bar(&empty[s], (ep >> s) & 1u);
    ep ^= 1u << s;
    if (row) {
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(rb_smem(&full[s])), "r"(bytes)
                   : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              rb_smem(ring + (size_t)s * NV * CO_THREADS)),
          "l"(row), "r"(bytes), "r"(rb_smem(&full[s]))
          : "memory");
    } else {
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(rb_smem(&full[s])) : "memory");
    }
  }
  __device__ void wait(int p) {  // every thread, in position order
    const int s = p % S;
    wait_bar(&full[s], (fp >> s) & 1u);
    fp ^= 1u << s;
  }
  __device__ void release(int p) {  // every thread, after reading position p
    __syncwarp();
    if ((threadIdx.x & 31) == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(rb_smem(&empty[p % S])) : "memory");
  }
  template <class RowFn>
  __device__ void prologue(int r0, int r1, RowFn row) {  // positions 0 .. S - 2 of [r0, r1)
    for (int q = 0; q < S - 1 && r0 + q < r1; ++q) issue(q, row(r0 + q));
  }
};

// Streams rows [r0, r1) whose first ST_SLOTS - 1 were issued by st_prologue;
// row(i) gives row i's pointer (null: skipped). For every row and batch row
// out(i, b, s) receives the CTA-wide dot product s of the row with the input
// slices xr, called by one thread. red: [2][ST_RB][NB][CO_WARPS].
template <typename T, int NB, int NV, int S = ST_SLOTS, class RowFn, class OutFn>
__device__ __forceinline__ void st_rows_dot(uint4* ring, int r0, int r1, int nvec,
                                            const float (&xr)[NB][NV][WT<T>::E], float* red, RowFn row,
                                            OutFn out) {
  constexpr int E = WT<T>::E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = r1 - r0;
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    const int ahead = i + S - 1;
    st_issue<T, NV, S>(ring, ahead, ahead < n ? row(r0 + ahead) : nullptr, nvec);
    cp_async_wait<S - 1>();
    uint4 w[NV];
    st_read<NV, S>(ring, i, nvec, w);
    float acc[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      float wf[E];
      WT<T>::unpack(w[j], wf);
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[b] = fmaf(wf[e], xr[b][j][e], acc[b]);
    }
    const int buf = (i / ST_RB) & 1, ri = i % ST_RB;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float s = warp_sum(acc[b]);
      if (lane == 0) red[((buf * ST_RB + ri) * NB + b) * CO_WARPS + warp] = s;
    }
    if (ri == ST_RB - 1 || i == n - 1) {
      __syncthreads();
      const int nr = ri + 1;
      for (int t = threadIdx.x; t < nr * NB; t += CO_THREADS) {
        const int rr = t / NB, b = t % NB;
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < CO_WARPS; ++q) s += red[((buf * ST_RB + rr) * NB + b) * CO_WARPS + q];
        out(r0 + i - ri + rr, b, s);
      }
      // the other buffer is written next; this one again only after the
      // next reduction's barrier, which every reader above reaches first
    }
  }
}


// ----------------------------------------------------------------------------
// attn_in_stream_kernel: attn_in_kernel for long rows. CTA g streams the rows
// [g n / G, (g + 1) n / G) of the n = |S_A| * 3 dh selected Q/K/V rows
// followed by the optional rows of the next layer's predictor.
// ----------------------------------------------------------------------------
template <typename T, int NB, int NV, int S = ST_SLOTS>
__global__ void __launch_bounds__(CO_THREADS, 1) attn_in_stream_kernel(AttnInArgs a) {
  constexpr int E = WT<T>::E;
  extern __shared__ __align__(16) uint4 s_ring[];
  __shared__ float red[2 * ST_RB * NB * CO_WARPS];
  __shared__ float lnred[2 * NB * CO_WARPS];
  const T* Wqkv = static_cast<const T*>(a.Wqkv);
  const int per = 3 * a.dh, nvec = a.d / E;
  griddep_launch();
  int r0 = 0, r1 = 0, nq = 0;  // rows [0, nq): Q/K/V; [nq, nq + n2h + n2r): next layer's predictor
  auto setup = [&]() {
    int hc = *a.head_count;
    if (hc > a.kh_max || hc < 0) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, 1);
      hc = hc < 0 ? 0 : a.kh_max;
    }
    nq = hc * per;
    const long long n = (long long)nq + a.n2h + a.n2r;
    r0 = (int)(n * blockIdx.x / gridDim.x);
    r1 = (int)(n * (blockIdx.x + 1) / gridDim.x);
  };
  auto head_of = [&](int slot) {
    const int head = a.head_idx[slot / per];
    return (head < 0 || head >= a.h) ? -1 : head;
  };
  auto row = [&](int slot) -> const T* {
    if (slot >= nq) {
      const int i2 = slot - nq;
      return i2 < a.n2h ? static_cast<const T*>(a.PA2) + (size_t)i2 * a.d
                        : static_cast<const T*>(a.At2) + (size_t)(i2 - a.n2h) * a.d;
    }
    const int head = head_of(slot);
    return head < 0 ? nullptr : Wqkv + ((size_t)head * per + slot % per) * a.d;
  };
  if (a.sets_ready) {
    setup();
    st_prologue<T, NV, S>(s_ring, r0, r1, nvec, row);
  }
  griddep_wait();
  if (!a.sets_ready) {
    setup();
    st_prologue<T, NV, S>(s_ring, r0, r1, nvec, row);
  }
  float xr[NB][NV][E];
  x_slice_load<T, NB, NV>(a.x, a.d, a.nb, xr);
  x_slice_ln<T, NB, NV>(xr, a.d, a.eps, a.ln_g, a.ln_b, lnred);
  if (blockIdx.x == 0) {
    if (a.yA_out) x_slice_store<T, NB, NV>(xr, a.d, a.nb, a.yA_out);
    const int n4 = (a.nb * a.d) >> 2;
    for (int i = threadIdx.x; i < n4; i += CO_THREADS)
      reinterpret_cast<float4*>(a.t1)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  T* Kc = static_cast<T*>(a.Kc);
  T* Vc = static_cast<T*>(a.Vc);
  auto out = [&](int slot, int b, float v) {
    if (b >= a.nb) return;
    if (slot >= nq) {
      const int i2 = slot - nq;
      if (i2 < a.n2h) a.sh2[(size_t)b * a.n2h + i2] = v;
      else a.z2[(size_t)b * a.n2r + i2 - a.n2h] = v;
      return;
    }
    const int head = head_of(slot);
    if (head < 0) {
      if (threadIdx.x == 0) raise_status(a.status, 2);
      return;
    }
    const int p = slot / per, rem = slot % per, m = rem / a.dh, c = rem % a.dh;
    if (a.bqkv) v += a.bqkv[(size_t)head * per + rem];
    if (m == 0) {
      a.q[((size_t)b * a.kh_max + p) * a.dh + c] = v;
    } else {
      T* cache = (m == 1) ? Kc : Vc;
      cache[(((size_t)b * a.h + head) * a.cap + a.pos) * a.dh + c] = WT<T>::store_cvt(v);
    }
  };
  st_rows_dot<T, NB, NV, S>(s_ring, r0, r1, nvec, xr, red, row, out);
}

// ----------------------------------------------------------------------------
// predict_a_stream_kernel: predict_a_kernel for long rows (rows [0, h) of PA,
// then rows [0, r) of At).
// ----------------------------------------------------------------------------
template <typename T, int NB, int NV>
__global__ void __launch_bounds__(CO_THREADS, 1) predict_a_stream_kernel(PredictAArgs a) {
  constexpr int E = WT<T>::E;
  extern __shared__ __align__(16) uint4 s_ring[];
  __shared__ float red[2 * ST_RB * NB * CO_WARPS];
  const int nvec = a.d / E;
  const int heads = a.PA ? a.h : 0;
  const long long n = heads + (a.At ? a.r : 0);
  const int r0 = (int)(n * blockIdx.x / gridDim.x), r1 = (int)(n * (blockIdx.x + 1) / gridDim.x);
  auto row = [&](int i) -> const T* {
    return i < heads ? static_cast<const T*>(a.PA) + (size_t)i * a.d
                     : static_cast<const T*>(a.At) + (size_t)(i - heads) * a.d;
  };
  griddep_launch();
  st_prologue<T, NV>(s_ring, r0, r1, nvec, row);
  griddep_wait();  // y comes from the previous kernel
  float xr[NB][NV][E];
  x_slice_load<T, NB, NV>(a.y, a.d, a.nb, xr);
  st_rows_dot<T, NB, NV>(s_ring, r0, r1, nvec, xr, red, row, [&](int i, int b, float v) {
    if (b >= a.nb) return;
    if (i < heads) a.scores_h[(size_t)b * a.h + i] = v;
    else a.z[(size_t)b * a.r + i - heads] = v;
  });
}

// ----------------------------------------------------------------------------
// mlp_stream_kernel: mlp_block_kernel for long rows. CTA g owns selection slots
// [g cnt / G, (g + 1) cnt / G), taken ST_CH at a time: the chunk's W1 rows
// stream through the ring (dot products with LN2(t1)), one CTA reduction gives
// the activations relu(. + b1), the nonzero ones are compacted, and their W2
// rows stream through the ring into the thread's own output columns, which
// are added to x once at the end (CTA 0 also adds t1 and b2).
// ----------------------------------------------------------------------------
template <typename T, int NB, int NV, int S = ST_SLOTS, bool BULK = false>
__global__ void __launch_bounds__(CO_THREADS, 1) mlp_stream_kernel(MlpBlockArgs a) {
  constexpr int E = WT<T>::E;
  extern __shared__ __align__(16) uint4 s_ring[];
  __shared__ float red[ST_CH * NB * CO_WARPS];
  __shared__ float lnred[2 * NB * CO_WARPS];
  __shared__ int s_row[ST_CH];     // W1 rows of the chunk (-1: invalid index)
  __shared__ float s_bias[ST_CH];
  __shared__ int s_row2[ST_CH];    // W2 rows with a nonzero activation
  __shared__ float s_act2[ST_CH][NB];
  __shared__ int s_nz;
  const T* W1t = static_cast<const T*>(a.W1t);
  const T* W2t = static_cast<const T*>(a.W2t);
  const int nvec = a.d / E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ uint64_t s_full[BULK ? S : 1], s_empty[BULK ? S : 1];
  __shared__ int s_abort;
  BulkRing<T, NV, S> rb{s_ring, s_full, s_empty, &s_abort, a.status, (unsigned)nvec * 16u, 0u, 0u};
  if constexpr (BULK) {
    rb.init();
    __syncthreads();
  }
  griddep_launch();
  int j0 = 0, j1 = 0;
  auto slot_range = [&]() {
    int cnt = *a.count;
    if (cnt > a.k_max || cnt < 0) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, 1);
      cnt = cnt < 0 ? 0 : a.k_max;
    }
    j0 = (int)(((long long)cnt * blockIdx.x) / gridDim.x);
    j1 = (int)(((long long)cnt * (blockIdx.x + 1)) / gridDim.x);
  };
  // the chunk's row indices and biases into shared memory, then its first rows
  auto chunk_begin = [&](int c0, int cn) {
    if ((int)threadIdx.x < cn) {
      int rw = a.idx[c0 + threadIdx.x];
      if (rw < 0 || rw >= a.N) {
        raise_status(a.status, 2);
        rw = -1;
      }
      s_row[threadIdx.x] = rw;
      s_bias[threadIdx.x] = rw >= 0 ? a.b1[rw] : 0.f;
    }
    __syncthreads();
    auto row1 = [&](int i) -> const T* {
      const int rw = s_row[i];
      return rw >= 0 ? W1t + (size_t)rw * a.d : nullptr;
    };
    if constexpr (BULK) rb.prologue(0, cn, row1);
    else st_prologue<T, NV, S>(s_ring, 0, cn, nvec, row1);
  };
  if (a.sets_ready) {
    slot_range();
    if (j1 > j0) chunk_begin(j0, min(ST_CH, j1 - j0));
  }
  griddep_wait();
  if (!a.sets_ready) {
    slot_range();
    if (j1 > j0) chunk_begin(j0, min(ST_CH, j1 - j0));
  }
  float xr[NB][NV][E];
  x_slice_load<T, NB, NV>(a.t1, a.d, a.nb, xr);
  x_slice_ln<T, NB, NV>(xr, a.d, a.eps, a.ln_g, a.ln_b, lnred);
  if (blockIdx.x == 0 && a.yM_out) x_slice_store<T, NB, NV>(xr, a.d, a.nb, a.yM_out);

  float acc[NB][NV][E];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int j = 0; j < NV; ++j)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[b][j][e] = 0.f;
#pragma unroll 1
  for (int c0 = j0; c0 < j1; c0 += ST_CH) {
    const int cn = min(ST_CH, j1 - c0);
    if (c0 != j0) chunk_begin(c0, cn);
    // ---- W1: partial dots of the chunk's rows ----
#pragma unroll 1
    for (int i = 0; i < cn; ++i) {
      const int ahead = i + S - 1;
      const int rw = ahead < cn ? s_row[ahead] : -1;
      uint4 w[NV];
      if constexpr (BULK) {
        if (ahead < cn) rb.issue(ahead, rw >= 0 ? W1t + (size_t)rw * a.d : nullptr);
        rb.wait(i);
        st_read<NV, S>(s_ring, i, nvec, w);
        rb.release(i);
      } else {
        st_issue<T, NV, S>(s_ring, ahead, rw >= 0 ? W1t + (size_t)rw * a.d : nullptr, nvec);
        cp_async_wait<S - 1>();
        st_read<NV, S>(s_ring, i, nvec, w);
      }
      float d1[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) d1[b] = 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        float wf[E];
        WT<T>::unpack(w[j], wf);
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int e = 0; e < E; ++e) d1[b] = fmaf(wf[e], xr[b][j][e], d1[b]);
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float s = warp_sum(d1[b]);
        if (lane == 0) red[(i * NB + b) * CO_WARPS + warp] = s;
      }
    }
    __syncthreads();
    // ---- activations, nonzero ones compacted in slot order ----
    if (warp == 0) {
      int base = 0;
#pragma unroll 1
      for (int i0 = 0; i0 < cn; i0 += 32) {
        const int i = i0 + lane;
        float act[NB];
        bool nz = false;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float s = 0.f;
          if (i < cn && b < a.nb && s_row[i] >= 0) {
#pragma unroll
            for (int q = 0; q < CO_WARPS; ++q) s += red[(i * NB + b) * CO_WARPS + q];
            s = activate(s + s_bias[i], a.act);
          }
          act[b] = s;
          nz |= s != 0.f;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, nz);
        if (nz) {
          const int at = base + __popc(bal & ((1u << lane) - 1u));
          s_row2[at] = s_row[i];
#pragma unroll
          for (int b = 0; b < NB; ++b) s_act2[at][b] = act[b];
        }
        base += __popc(bal);
      }
      if (lane == 0) s_nz = base;
    }
    __syncthreads();
    // ---- W2: the nonzero rows into this thread's columns ----
    const int nl = s_nz;
    auto row2 = [&](int i) -> const T* { return W2t + (size_t)s_row2[i] * a.d; };
    if constexpr (BULK) rb.prologue(0, nl, row2);
    else st_prologue<T, NV, S>(s_ring, 0, nl, nvec, row2);
#pragma unroll 1
    for (int i = 0; i < nl; ++i) {
      const int ahead = i + S - 1;
      uint4 w[NV];
      if constexpr (BULK) {
        if (ahead < nl) rb.issue(ahead, row2(ahead));
        rb.wait(i);
        st_read<NV, S>(s_ring, i, nvec, w);
        rb.release(i);
      } else {
        st_issue<T, NV, S>(s_ring, ahead, ahead < nl ? row2(ahead) : nullptr, nvec);
        cp_async_wait<S - 1>();
        st_read<NV, S>(s_ring, i, nvec, w);
      }
      float cb[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) cb[b] = s_act2[i][b];
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        float wf[E];
        WT<T>::unpack(w[j], wf);
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int e = 0; e < E; ++e) acc[b][j][e] = fmaf(cb[b], wf[e], acc[b][j][e]);
      }
    }
    __syncthreads();  // s_row / s_row2 / s_act2 are rewritten by the next chunk
  }
  const bool residual = blockIdx.x == 0;
  if (j1 == j0 && !residual) return;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * CO_THREADS + threadIdx.x) * E;
    if (c >= a.d) continue;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b >= a.nb) continue;
      float o[E];
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = acc[b][j][e];
      if (residual) {
#pragma unroll
        for (int e4 = 0; e4 < E / 4; ++e4) {
          const float4 t = __ldcg(reinterpret_cast<const float4*>(a.t1 + (size_t)b * a.d + c) + e4);
          float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
          if (a.b2) bb = *(reinterpret_cast<const float4*>(a.b2 + c) + e4);
          o[4 * e4 + 0] += t.x + bb.x;
          o[4 * e4 + 1] += t.y + bb.y;
          o[4 * e4 + 2] += t.z + bb.z;
          o[4 * e4 + 3] += t.w + bb.w;
        }
      }
#pragma unroll
      for (int e4 = 0; e4 < E / 4; ++e4)
        red_add4(a.x + (size_t)b * a.d + c + 4 * e4,
                 make_float4(o[4 * e4], o[4 * e4 + 1], o[4 * e4 + 2], o[4 * e4 + 3]));
    }
  }
}

// ----------------------------------------------------------------------------
// wo_stream_kernel: the W^O product of eq. (2) for long rows (16-24 KB, batch
// 1-2), after attn_out_kernel stopped at H (ATTN_H_ONLY):
//   t1 += sum over the selected heads' rows (p, c) of H[b][p][c] W_i^O[c][:]
// Rows are spread evenly over one CTA per SM; each CTA streams its rows
// through the ring into its threads' own columns (no CTA reduction) and adds
// its full-width partial to t1 once. The first rows are issued before the
// dependency wait when the head set is known ahead (their W^O rows do not
// depend on the attention), so they stream while the attention runs. CTA 0
// also moves the residual: t1 += x + bO, then x = 0.
// ----------------------------------------------------------------------------
struct WoStreamArgs {
  const void* WOt;  // [h][dh][d]
  const float* bO;  // [d] or null
  const float* H;   // [nb][kh_max][dh]
  const int32_t* head_idx;
  const int32_t* head_count;
  int kh_max, h, dh, d, nb, sets_ready;
  float* x;
  float* t1;
  int* status;
};

constexpr int WO_CHUNK = 1024;  // rows whose coefficients a CTA holds at once

template <typename T, int NB, int NV, int S = ST_SLOTS>
__global__ void __launch_bounds__(CO_THREADS, 1) wo_stream_kernel(WoStreamArgs a) {
  constexpr int E = WT<T>::E;
  extern __shared__ __align__(16) uint4 s_ring[];
  __shared__ float s_coef[WO_CHUNK][NB];
  const T* WO = static_cast<const T*>(a.WOt);
  const int nvec = a.d / E;
  griddep_launch();
  int r0 = 0, r1 = 0;
  auto range = [&]() {
    int hc = *a.head_count;
    if (hc > a.kh_max || hc < 0) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, 1);
      hc = hc < 0 ? 0 : a.kh_max;
    }
    const long long nrows = (long long)hc * a.dh;
    r0 = (int)(nrows * blockIdx.x / gridDim.x);
    r1 = (int)(nrows * (blockIdx.x + 1) / gridDim.x);
  };
  auto head_of = [&](int i) {
    const int head = a.head_idx[i / a.dh];
    return (head >= 0 && head < a.h) ? head : -1;
  };
  auto row = [&](int i) -> const T* {
    const int head = head_of(i);
    return head >= 0 ? WO + ((size_t)head * a.dh + i % a.dh) * a.d : nullptr;
  };
  auto rowr = [&](int i) -> const T* { return row(r0 + i); };
  if (a.sets_ready) {
    range();
    st_prologue<T, NV, S>(s_ring, 0, r1 - r0, nvec, rowr);
  }
  griddep_wait();
  if (!a.sets_ready) {
    range();
    st_prologue<T, NV, S>(s_ring, 0, r1 - r0, nvec, rowr);
  }
  float acc[NB][NV][E];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int j = 0; j < NV; ++j)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[b][j][e] = 0.f;
  const int n = r1 - r0;
#pragma unroll 1
  for (int c0 = 0; c0 < n; c0 += WO_CHUNK) {
    const int cn = min(WO_CHUNK, n - c0);
    __syncthreads();  // the previous chunk's coefficients are consumed
    for (int t = threadIdx.x; t < cn * NB; t += CO_THREADS) {
      const int i = t / NB, b = t % NB, rr = r0 + c0 + i;
      const bool ok = b < a.nb && head_of(rr) >= 0;
      s_coef[i][b] = ok ? __ldcg(a.H + ((size_t)b * a.kh_max + rr / a.dh) * a.dh + rr % a.dh) : 0.f;
      if (b == 0 && head_of(rr) < 0 && rr % a.dh == 0) raise_status(a.status, 2);
    }
    __syncthreads();
#pragma unroll 1
    for (int i = c0; i < c0 + cn; ++i) {
      const int ahead = i + S - 1;
      st_issue<T, NV, S>(s_ring, ahead, ahead < n ? rowr(ahead) : nullptr, nvec);
      cp_async_wait<S - 1>();
      if (head_of(r0 + i) < 0) continue;  // a skipped row: its slot holds no data (same for every thread)
      uint4 w[NV];
      st_read<NV, S>(s_ring, i, nvec, w);
      float cb[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) cb[b] = s_coef[i - c0][b];
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        float wf[E];
        WT<T>::unpack(w[j], wf);
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int e = 0; e < E; ++e) acc[b][j][e] = fmaf(cb[b], wf[e], acc[b][j][e]);
      }
    }
  }
  const bool residual = blockIdx.x == 0;
  if (n == 0 && !residual) return;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * CO_THREADS + threadIdx.x) * E;
    if (c >= a.d) continue;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b >= a.nb) continue;
      float o[E];
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = acc[b][j][e];
      if (residual) {
        float* xr = a.x + (size_t)b * a.d + c;
#pragma unroll
        for (int e4 = 0; e4 < E / 4; ++e4) {
          const float4 xv = __ldcg(reinterpret_cast<const float4*>(xr) + e4);
          float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
          if (a.bO) bb = *(reinterpret_cast<const float4*>(a.bO + c) + e4);
          o[4 * e4 + 0] += xv.x + bb.x;
          o[4 * e4 + 1] += xv.y + bb.y;
          o[4 * e4 + 2] += xv.z + bb.z;
          o[4 * e4 + 3] += xv.w + bb.w;
          reinterpret_cast<float4*>(xr)[e4] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int e4 = 0; e4 < E / 4; ++e4)
        red_add4(a.t1 + (size_t)b * a.d + c + 4 * e4,
                 make_float4(o[4 * e4], o[4 * e4 + 1], o[4 * e4 + 2], o[4 * e4 + 3]));
    }
  }
}

}  // namespace dv
