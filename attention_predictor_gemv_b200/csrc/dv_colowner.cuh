// Column-owner variants of the fused kernels whose rows are d long (Q/K/V,
// W1, the predictor's first stage).
//
// Each of the CTA's 256 threads owns fixed columns of the input vector: the
// 16-byte vectors j * 256 + t (j < NV). The thread keeps its slice of the
// (normalised) input in registers for every row the CTA streams, so the input
// is read from memory once per CTA and never from shared memory; LayerNorm
// needs one block-wide reduction. A CTA streams R rows with R * NV 16-byte
// loads in flight per thread, fully coalesced (each row is read by the whole
// CTA), and reduces the R partial dot products across the CTA at the end.
// Used when NB * NV is small (batch 1-2 up to NV = 6, batch 3-4 up to NV = 2):
// the slices then fit in registers.
#pragma once

#include "dv_fused.cuh"

namespace dv {

constexpr int CO_THREADS = FUSED_THREADS;
constexpr int CO_WARPS = CO_THREADS / 32;

// Sums of N values over the CTA; every thread gets all N totals.
// red holds N * CO_WARPS floats. Ends with a barrier.
template <int N>
__device__ __forceinline__ void block_sum_n(float (&v)[N], float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float s = warp_sum(v[i]);
    if (lane == 0) red[i * CO_WARPS + w] = s;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) {
    float t = lane < CO_WARPS ? red[i * CO_WARPS + lane] : 0.f;
    v[i] = warp_sum(t);
  }
  __syncthreads();
}

// This thread's slice of x [nb][d]: xr[b][j][e] = x[b][(j*256 + t)*E + e],
// zero outside the row. One 16-byte-load pass, all loads in flight.
template <typename T, int NB, int NV>
__device__ __forceinline__ void x_slice_load(const float* __restrict__ x, int d, int nb,
                                             float (&xr)[NB][NV][WT<T>::E]) {
  constexpr int E = WT<T>::E;
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c = (j * CO_THREADS + threadIdx.x) * E;
      const bool ok = b < nb && c < d;
#pragma unroll
      for (int e4 = 0; e4 < E / 4; ++e4) {
        const float4 v = ok ? __ldcg(reinterpret_cast<const float4*>(x + (size_t)b * d + c) + e4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        xr[b][j][4 * e4 + 0] = v.x;
        xr[b][j][4 * e4 + 1] = v.y;
        xr[b][j][4 * e4 + 2] = v.z;
        xr[b][j][4 * e4 + 3] = v.w;
      }
    }
}

// LayerNorm of the slices in place: (x - mean) / sqrt(var + eps) * g + beta,
// mean and biased variance over the d columns of each batch row, both from
// one CTA reduction of the sums of x and x^2 (var = E[x^2] - mean^2 in fp32:
// the block inputs have |mean| of the order of their spread, far from the
// cancellation regime). Columns outside the row stay zero. red holds
// 2 NB CO_WARPS floats.
template <typename T, int NB, int NV>
__device__ __forceinline__ void x_slice_ln(float (&xr)[NB][NV][WT<T>::E], int d, float eps, const float* g,
                                           const float* beta, float* red) {
  constexpr int E = WT<T>::E;
  float sq[2 * NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        s1 += xr[b][j][e];
        s2 = fmaf(xr[b][j][e], xr[b][j][e], s2);
      }
    sq[b] = s1;
    sq[NB + b] = s2;
  }
  block_sum_n<2 * NB>(sq, red);
  float s[NB], q[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    s[b] = sq[b] / (float)d;
    q[b] = fmaxf(sq[NB + b] / (float)d - s[b] * s[b], 0.f) * (float)d;
  }
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int c = (j * CO_THREADS + threadIdx.x) * E;
    if (c >= d) continue;
    float gv[E], bv[E];
#pragma unroll
    for (int e4 = 0; e4 < E / 4; ++e4) {
      const float4 gg = g ? *(reinterpret_cast<const float4*>(g + c) + e4) : make_float4(1.f, 1.f, 1.f, 1.f);
      const float4 bb = beta ? *(reinterpret_cast<const float4*>(beta + c) + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
      gv[4 * e4] = gg.x; gv[4 * e4 + 1] = gg.y; gv[4 * e4 + 2] = gg.z; gv[4 * e4 + 3] = gg.w;
      bv[4 * e4] = bb.x; bv[4 * e4 + 1] = bb.y; bv[4 * e4 + 2] = bb.z; bv[4 * e4 + 3] = bb.w;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float rs = rsqrtf(q[b] / (float)d + eps);
#pragma unroll
      for (int e = 0; e < E; ++e) xr[b][j][e] = (xr[b][j][e] - s[b]) * rs * gv[e] + bv[e];
    }
  }
}

// Writes the slices back to y [nb][d] (each thread its own columns).
template <typename T, int NB, int NV>
__device__ __forceinline__ void x_slice_store(const float (&xr)[NB][NV][WT<T>::E], int d, int nb, float* y) {
  constexpr int E = WT<T>::E;
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int c = (j * CO_THREADS + threadIdx.x) * E;
      if (b < nb && c < d) {
#pragma unroll
        for (int e4 = 0; e4 < E / 4; ++e4)
          reinterpret_cast<float4*>(y + (size_t)b * d + c)[e4] =
              make_float4(xr[b][j][4 * e4], xr[b][j][4 * e4 + 1], xr[b][j][4 * e4 + 2], xr[b][j][4 * e4 + 3]);
      }
    }
}

// Issues the loads of this thread's columns of R rows.
template <typename T, int NV, int R>
__device__ __forceinline__ void co_issue(uint4 (&w)[R][NV], const T* const (&rowp)[R], const bool (&valid)[R],
                                         int nvec) {
  constexpr int E = WT<T>::E;
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int v = j * CO_THREADS + threadIdx.x;
      w[r][j] = (valid[r] && v < nvec) ? ld_stream(rowp[r] + (size_t)v * E) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// Dot products of R rows with NB input slices, summed over the CTA:
// out[r * NB + b] (shared memory) on return. red holds R * NB * CO_WARPS floats.
template <typename T, int NB, int NV, int R>
__device__ __forceinline__ void co_dot(const uint4 (&w)[R][NV], const float (&xr)[NB][NV][WT<T>::E], float* red,
                                       float* out) {
  constexpr int E = WT<T>::E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc[R][NB];
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      float wf[E];
      WT<T>::unpack(w[r][j], wf);
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[r][b] = fmaf(wf[e], xr[b][j][e], acc[r][b]);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float s = warp_sum(acc[r][b]);
      if (lane == 0) red[(r * NB + b) * CO_WARPS + warp] = s;
    }
  __syncthreads();
  for (int i = threadIdx.x; i < R * NB; i += CO_THREADS) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < CO_WARPS; ++q) s += red[i * CO_WARPS + q];
    out[i] = s;
  }
  __syncthreads();
}

// ----------------------------------------------------------------------------
// attn_in_co_kernel: attn_in_kernel (LN1, selected heads' q/k/v, KV append)
// with R output rows per CTA, column-owner layout. Slots [0, kh_max 3 dh) are
// the Q/K/V rows of the selected heads (those past the count idle), slots
// after them the optional rows of the next layer's predictor.
// ----------------------------------------------------------------------------
template <typename T, int NB, int NV, int R>
__global__ void __launch_bounds__(CO_THREADS) attn_in_co_kernel(AttnInArgs a) {
  constexpr int E = WT<T>::E;
  __shared__ float red[(R * NB > 2 * NB ? R * NB : 2 * NB) * CO_WARPS];
  __shared__ float s_out[R * NB];
  const T* Wqkv = static_cast<const T*>(a.Wqkv);
  const int per = 3 * a.dh;
  const int nvec = a.d / E;
  const int qrows = a.kh_max * per, n2 = a.n2h + a.n2r;
  const int ngroups = (qrows + n2 + R - 1) / R;
  int slot0 = blockIdx.x * R;
  griddep_launch();
  const T* rowp[R];
  bool valid[R];
  int heads[R];
  int nslot = 0;
  auto count_slots = [&]() {
    int hc = *a.head_count;
    if (hc > a.kh_max || hc < 0) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, 1);
      hc = hc < 0 ? 0 : a.kh_max;
    }
    nslot = hc * per;
  };
  auto setup = [&]() {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int slot = slot0 + r;
      int head = -1;  // >= 0: a Q/K/V row of that head; <= -2: predictor row -2 - head
      const T* rp = Wqkv;
      if (slot < nslot) {
        head = a.head_idx[slot / per];
        if (head < 0 || head >= a.h) {
          if (threadIdx.x == 0) raise_status(a.status, 2);
          head = -1;
        } else {
          rp = Wqkv + ((size_t)head * per + (slot % per)) * a.d;
        }
      } else if (slot >= qrows && slot < qrows + n2) {
        const int i2 = slot - qrows;
        head = -2 - i2;
        rp = i2 < a.n2h ? static_cast<const T*>(a.PA2) + (size_t)i2 * a.d
                        : static_cast<const T*>(a.At2) + (size_t)(i2 - a.n2h) * a.d;
      }
      heads[r] = head;
      valid[r] = head != -1;
      rowp[r] = rp;
    }
  };
  uint4 w[R][NV];
  if (a.sets_ready) {
    count_slots();
    setup();
    co_issue<T, NV, R>(w, rowp, valid, nvec);
  }
  griddep_wait();
  if (!a.sets_ready) {
    count_slots();
    setup();
    co_issue<T, NV, R>(w, rowp, valid, nvec);
  }
  float xr[NB][NV][E];
  x_slice_load<T, NB, NV>(a.x, a.d, a.nb, xr);
  x_slice_ln<T, NB, NV>(xr, a.d, a.eps, a.ln_g, a.ln_b, red);
  if (blockIdx.x == 0) {
    if (a.yA_out) x_slice_store<T, NB, NV>(xr, a.d, a.nb, a.yA_out);
    const int n4 = (a.nb * a.d) >> 2;
    for (int i = threadIdx.x; i < n4; i += CO_THREADS)
      reinterpret_cast<float4*>(a.t1)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  T* Kc = static_cast<T*>(a.Kc);
  T* Vc = static_cast<T*>(a.Vc);
  for (int g = blockIdx.x; g < ngroups; g += gridDim.x) {
    if (g != (int)blockIdx.x) {
      slot0 = g * R;
      setup();
      co_issue<T, NV, R>(w, rowp, valid, nvec);
    }
    co_dot<T, NB, NV, R>(w, xr, red, s_out);
    for (int i = threadIdx.x; i < R * NB; i += CO_THREADS) {
      const int r = i / NB, b = i % NB;
      bool ok = false;
      int head = 0;
#pragma unroll
      for (int rr = 0; rr < R; ++rr)
        if (rr == r) {
          ok = valid[rr];
          head = heads[rr];
        }
      if (!ok || b >= a.nb) continue;
      float v = s_out[i];
      if (head <= -2) {
        const int i2 = -2 - head;
        if (i2 < a.n2h) a.sh2[(size_t)b * a.n2h + i2] = v;
        else a.z2[(size_t)b * a.n2r + i2 - a.n2h] = v;
        continue;
      }
      const int slot = slot0 + r;
      const int p = slot / per, rem = slot % per, m = rem / a.dh, c = rem % a.dh;
      if (a.bqkv) v += a.bqkv[(size_t)head * per + rem];
      if (m == 0) {
        a.q[((size_t)b * a.kh_max + p) * a.dh + c] = v;
      } else {
        T* cache = (m == 1) ? Kc : Vc;
        cache[(((size_t)b * a.h + head) * a.cap + a.pos) * a.dh + c] = WT<T>::store_cvt(v);
      }
    }
  }
}

// ----------------------------------------------------------------------------
// mlp_block_co_kernel: mlp_block_kernel (LN2, W1 + b1 + ReLU, W2 gather-axpy,
// residual) in the column-owner layout. CTA g owns selection slots
// [g*cnt/G, (g+1)*cnt/G), taken R at a time. A chunk's W2 rows are loaded
// together with its W1 rows (before griddep_wait for the first chunk), not
// after the activations are known: the predictor selects the neurons it
// expects to be active, so their W2 rows are needed, and at these row
// lengths the kernel is bound by the latency of dependent loads, not by
// bytes. The W2 rows of nonzero activations accumulate into the thread's own
// columns across all chunks and are added to x once at the end; CTA 0 also
// adds t1 and b2.
// ----------------------------------------------------------------------------
template <typename T, int NB, int NV, int R>
__global__ void __launch_bounds__(CO_THREADS) mlp_block_co_kernel(MlpBlockArgs a) {
  constexpr int E = WT<T>::E;
  __shared__ float red[(R * NB > 2 * NB ? R * NB : 2 * NB) * CO_WARPS];
  __shared__ float s_out[R * NB];
  __shared__ float s_act[R][NB];
  const T* W1t = static_cast<const T*>(a.W1t);
  const T* W2t = static_cast<const T*>(a.W2t);
  const int nvec = a.d / E;
  griddep_launch();
  int cnt = 0, j0 = 0, j1 = 0;
  auto slot_range = [&]() {
    cnt = *a.count;
    if (cnt > a.k_max || cnt < 0) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, 1);
      cnt = cnt < 0 ? 0 : a.k_max;
    }
    j0 = (int)(((long long)cnt * blockIdx.x) / a.G);
    j1 = (int)(((long long)cnt * (blockIdx.x + 1)) / a.G);
  };
  const T* rowp[R];
  const T* rowp2[R];
  bool valid[R];
  float bias[R];
  auto setup_rows = [&](int base) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = base + r;
      int row = j < j1 ? a.idx[j] : -1;
      if (j < j1 && (row < 0 || row >= a.N)) {
        if (threadIdx.x == 0) raise_status(a.status, 2);
        row = -1;
      }
      valid[r] = row >= 0;
      rowp[r] = W1t + (size_t)(row >= 0 ? row : 0) * a.d;
      rowp2[r] = W2t + (size_t)(row >= 0 ? row : 0) * a.d;
      bias[r] = row >= 0 ? a.b1[row] : 0.f;
    }
  };
  uint4 w[R][NV], w2[R][NV];
  auto issue = [&]() {
    co_issue<T, NV, R>(w, rowp, valid, nvec);
    co_issue<T, NV, R>(w2, rowp2, valid, nvec);
  };
  if (a.sets_ready) {
    slot_range();
    setup_rows(j0);
    issue();
  }
  griddep_wait();
  if (!a.sets_ready) {
    slot_range();
    setup_rows(j0);
    issue();
  }
  float xr[NB][NV][E];
  x_slice_load<T, NB, NV>(a.t1, a.d, a.nb, xr);
  x_slice_ln<T, NB, NV>(xr, a.d, a.eps, a.ln_g, a.ln_b, red);
  if (blockIdx.x == 0 && a.yM_out) x_slice_store<T, NB, NV>(xr, a.d, a.nb, a.yM_out);

  float acc[NB][NV][E];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int j = 0; j < NV; ++j)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[b][j][e] = 0.f;
  for (int c0 = j0; c0 < j1; c0 += R) {
    if (c0 != j0) {
      setup_rows(c0);
      issue();
    }
    co_dot<T, NB, NV, R>(w, xr, red, s_out);
    if (threadIdx.x < R * NB) {
      const int r = threadIdx.x / NB, b = threadIdx.x % NB;
      float v = 0.f;
#pragma unroll
      for (int rr = 0; rr < R; ++rr)
        if (rr == r) v = (valid[rr] && b < a.nb) ? activate(s_out[r * NB + b] + bias[rr], a.act) : 0.f;
      s_act[r][b] = v;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r) {
      bool nz = false;
#pragma unroll
      for (int b = 0; b < NB; ++b) nz |= s_act[r][b] != 0.f;
      if (nz) {  // the same for every thread: zero activations add nothing
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          float wf[E];
          WT<T>::unpack(w2[r][j], wf);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const float cb = s_act[r][b];
#pragma unroll
            for (int e = 0; e < E; ++e) acc[b][j][e] = fmaf(cb, wf[e], acc[b][j][e]);
          }
        }
      }
    }
    __syncthreads();  // s_act is rewritten by the next chunk
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
// predict_a_co_kernel: predict_a_kernel (head scores, z = y A) in the
// column-owner layout: R rows of [PA; At] per CTA.
// ----------------------------------------------------------------------------
template <typename T, int NB, int NV, int R>
__global__ void __launch_bounds__(CO_THREADS) predict_a_co_kernel(PredictAArgs a) {
  constexpr int E = WT<T>::E;
  __shared__ float red[R * NB * CO_WARPS];
  __shared__ float s_out[R * NB];
  griddep_launch();
  const int heads = a.PA ? a.h : 0;
  const int nrows = heads + (a.At ? a.r : 0);
  const int ngroups = (nrows + R - 1) / R;
  const T* rowp[R];
  bool valid[R];
  auto setup = [&](int row0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int row = row0 + r;
      valid[r] = row < nrows;
      const T* base = row < heads ? static_cast<const T*>(a.PA) + (size_t)row * a.d
                                  : static_cast<const T*>(a.At) + (size_t)(valid[r] ? row - heads : 0) * a.d;
      rowp[r] = valid[r] ? base : static_cast<const T*>(heads ? a.PA : a.At);
    }
  };
  uint4 w[R][NV];
  setup(blockIdx.x * R);
  co_issue<T, NV, R>(w, rowp, valid, a.d / E);
  griddep_wait();  // y comes from the previous kernel
  float xr[NB][NV][E];
  x_slice_load<T, NB, NV>(a.y, a.d, a.nb, xr);
  for (int g = blockIdx.x; g < ngroups; g += gridDim.x) {
    const int row0 = g * R;
    if (g != (int)blockIdx.x) {
      setup(row0);
      co_issue<T, NV, R>(w, rowp, valid, a.d / E);
    }
    co_dot<T, NB, NV, R>(w, xr, red, s_out);
    for (int i = threadIdx.x; i < R * NB; i += CO_THREADS) {
      const int r = i / NB, b = i % NB;
      const int row = row0 + r;
      if (row >= nrows || b >= a.nb) continue;
      if (row < heads) a.scores_h[(size_t)b * a.h + row] = s_out[i];
      else a.z[(size_t)b * a.r + row - heads] = s_out[i];
    }
  }
}

}  // namespace dv
