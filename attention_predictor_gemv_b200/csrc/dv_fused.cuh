// Fused per-layer kernels of the decode step.
//
// One layer runs as three kernels on the main stream:
//   attn_in_kernel    LN1(x), Q/K/V of the selected heads, KV append
//                     (column-owner and ring variants: dv_colowner.cuh,
//                     dv_stream.cuh; they can also carry the next layer's
//                     predictor first stage)
//   attn_out_kernel   split attention + combine + W^O, one thread-block
//                     cluster per selected head (DSMEM combine)
//   mlp_block_kernel  LN2, W1 gather + b1 + ReLU, W2 gather-axpy
//                     (column-owner and ring variants as above)
// and the look-ahead predictor as kernels on side streams:
//   predict_a_kernel  head scores and z = y A (when not carried by attn_in)
//   predict_b_kernel  neuron scores z B^T + b1
//   select_rows_kernel, select_heads_kernel and gate_kernel
//                     (dv_api_kernels.cuh): the exact neuron and head
//                     selections, and the ordering gate
//
// The residual stream moves x -> t1 -> x through the three main kernels:
// attn_in zeroes t1, attn_out adds x + MHA(yA) into t1 and zeroes x, and
// mlp_block adds t1 + MLP(yM) into x. Every block output is accumulated with
// vector float reductions; one CTA per column (a column slice's owner, or
// CTA 0 when CTAs take whole rows) adds the residual (and the bias) exactly
// once.
#pragma once

#include <cooperative_groups.h>

#include "dv_kernels.cuh"

namespace dv {

namespace cg = cooperative_groups;

constexpr int FUSED_THREADS = 256;
constexpr int FUSED_WARPS = FUSED_THREADS / 32;
constexpr int HSEL_MAX = 1024;  // heads handled by the in-kernel head selection

// LayerNorm of every batch row of x [nb][d] into dst [nb][d] (shared
// memory): one pass of 16-byte loads brings x in (all loads in flight, one
// global round trip), then mean and biased variance are reduced from shared
// memory and dst is normalised in place: (x - mean) / sqrt(var + eps) * g + beta.
template <int NB>
__device__ __forceinline__ void ln_to_smem(const float* __restrict__ x, int d, int nb, float eps,
                                           const float* __restrict__ g, const float* __restrict__ beta,
                                           float* __restrict__ dst, float* red) {
  const int n4 = (nb * d) >> 2, d4 = d >> 2;
  const float4* xs = reinterpret_cast<const float4*>(x);
  float4* ds = reinterpret_cast<float4*>(dst);
  constexpr int UNR = 4;
  for (int i0 = threadIdx.x; i0 < n4; i0 += FUSED_THREADS * UNR) {
    float4 v[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = i0 + u * FUSED_THREADS;
      if (i < n4) v[u] = __ldcg(xs + i);
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = i0 + u * FUSED_THREADS;
      if (i < n4) ds[i] = v[u];
    }
  }
  __syncthreads();
  for (int b = 0; b < nb && b < NB; ++b) {
    const float4* xr = ds + (size_t)b * d4;
    float s = 0.f;
    for (int i = threadIdx.x; i < d4; i += FUSED_THREADS) {
      const float4 v = xr[i];
      s += (v.x + v.y) + (v.z + v.w);
    }
    const float m = block_sum<FUSED_THREADS>(s, red) / (float)d;
    float q = 0.f;
    for (int i = threadIdx.x; i < d4; i += FUSED_THREADS) {
      const float4 v = xr[i];
      const float a = v.x - m, c = v.y - m, e = v.z - m, f = v.w - m;
      q += (a * a + c * c) + (e * e + f * f);
    }
    const float rs = rsqrtf(block_sum<FUSED_THREADS>(q, red) / (float)d + eps);
    float4* yr = ds + (size_t)b * d4;
    for (int i = threadIdx.x; i < d4; i += FUSED_THREADS) {
      const float4 v = yr[i];
      float4 o = make_float4((v.x - m) * rs, (v.y - m) * rs, (v.z - m) * rs, (v.w - m) * rs);
      if (g) {
        const float4 gg = __ldg(reinterpret_cast<const float4*>(g) + i);
        o.x *= gg.x; o.y *= gg.y; o.z *= gg.z; o.w *= gg.w;
      }
      if (beta) {
        const float4 bb = __ldg(reinterpret_cast<const float4*>(beta) + i);
        o.x += bb.x; o.y += bb.y; o.z += bb.z; o.w += bb.w;
      }
      yr[i] = o;
    }
  }
  __syncthreads();
}

// ----------------------------------------------------------------------------
// Row dots against a normalised input held in shared memory. Same load
// pattern as warp_rows_dot (RPW rows, U column steps, 8 loads in flight per
// lane), with the first column step optionally issued before the caller's
// griddep_wait (its rows do not depend on the previous kernel).
// ----------------------------------------------------------------------------
template <typename T, int RPW, int U>
struct RowLoads {
  uint4 w[U][RPW];
};

template <typename T, int RPW, int U>
__device__ __forceinline__ void issue_row_loads(RowLoads<T, RPW, U>& L, const T* const (&rowp)[RPW],
                                                const bool (&valid)[RPW], int nvec, int v0) {
  constexpr int E = WT<T>::E;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int v = v0 + u * 32;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
      L.w[u][r] = (valid[r] && v < nvec) ? ld_stream(rowp[r] + (size_t)v * E) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <typename T, int NB, int RPW, int U>
__device__ __forceinline__ void consume_row_loads(const RowLoads<T, RPW, U>& L, const float* __restrict__ ys, int d,
                                                  int nb, int nvec, int v0, float (&acc)[RPW][NB]) {
  constexpr int E = WT<T>::E;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int v = v0 + u * 32;
    if (v < nvec) {
      float wf[RPW][E];
#pragma unroll
      for (int r = 0; r < RPW; ++r) WT<T>::unpack(L.w[u][r], wf[r]);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b < nb) {
          float xv[E];
          const float4* xp = reinterpret_cast<const float4*>(ys + (size_t)b * d + (size_t)v * E);
#pragma unroll
          for (int e4 = 0; e4 < E / 4; ++e4) {
            const float4 t = xp[e4];
            xv[4 * e4 + 0] = t.x;
            xv[4 * e4 + 1] = t.y;
            xv[4 * e4 + 2] = t.z;
            xv[4 * e4 + 3] = t.w;
          }
#pragma unroll
          for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int e = 0; e < E; ++e) acc[r][b] = fmaf(wf[r][e], xv[e], acc[r][b]);
        }
      }
    }
  }
}

// Full dot of RPW rows with ys, where the loads of the first column step
// (v0 = lane) were already issued into L.
template <typename T, int NB, int RPW, int U>
__device__ __forceinline__ void finish_rows_dot(RowLoads<T, RPW, U>& L, const T* const (&rowp)[RPW],
                                                const bool (&valid)[RPW], const float* __restrict__ ys, int d,
                                                int nb, float (&acc)[RPW][NB]) {
  constexpr int E = WT<T>::E;
  const int lane = threadIdx.x & 31;
  const int nvec = d / E;
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
  consume_row_loads<T, NB, RPW, U>(L, ys, d, nb, nvec, lane, acc);
  for (int v0 = lane + 32 * U; v0 < nvec; v0 += 32 * U) {
    issue_row_loads<T, RPW, U>(L, rowp, valid, nvec, v0);
    consume_row_loads<T, NB, RPW, U>(L, ys, d, nb, nvec, v0, acc);
  }
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = warp_sum(acc[r][b]);
}

// ----------------------------------------------------------------------------
// mlp_block_kernel: x (+)= t1 + sum_j relu(yM . W1t[idx_j] + b1[idx_j]) W2t[idx_j]
// (+ b2), yM = LN2(t1) (eq. (1)). CTA g owns selection slots
// [g*cnt/G, (g+1)*cnt/G): it forms their activations (warp per row), keeps
// the nonzero ones, streams their W2 rows over all d columns and adds its
// partial sums to x. CTA 0 also adds t1 and b2. x must be zero on entry.
// ----------------------------------------------------------------------------
struct MlpBlockArgs {
  const float* t1;  // [B][d] block input (residual after attention)
  float* x;         // [B][d] output, zero on entry
  const float* ln_g;
  const float* ln_b;
  float eps;
  const void* W1t;
  const float* b1;
  const void* W2t;
  const float* b2;
  const int32_t* idx;
  const int32_t* count;
  int k_max, d, N, nb, G, sets_ready;
  float* yM_out;  // optional copy of LN2(t1), written by CTA 0
  int* status;
  int act;        // ACT_RELU or ACT_GELU
};

constexpr int MLP_MAX_ROWS = 64;  // selection slots per CTA held in shared memory at once

template <typename T, int NB, int RPW, int U>
__global__ void __launch_bounds__(FUSED_THREADS) mlp_block_kernel(MlpBlockArgs a) {
  constexpr int E = WT<T>::E;
  extern __shared__ __align__(16) float s_y[];  // [nb][d] normalised input
  __shared__ float red[FUSED_WARPS];
  __shared__ float s_act[MLP_MAX_ROWS][NB];
  __shared__ int s_row[MLP_MAX_ROWS];
  __shared__ int s_nz[MLP_MAX_ROWS];
  __shared__ int s_list[MLP_MAX_ROWS];
  __shared__ int s_nlist;
  const T* W1t = static_cast<const T*>(a.W1t);
  const T* W2t = static_cast<const T*>(a.W2t);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
  // rows of the first chunk handled by this warp
  const T* rowp[RPW];
  bool valid[RPW];
  int rows[RPW];
  float bias[RPW];
  auto setup_rows = [&](int base, int limit) {
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int j = base + warp * RPW + r;
      int row = j < limit ? a.idx[j] : -1;
      if (j < limit && (row < 0 || row >= a.N)) {
        if (lane == 0) raise_status(a.status, 2);
        row = -1;
      }
      rows[r] = row;
      valid[r] = row >= 0;
      rowp[r] = W1t + (size_t)(row >= 0 ? row : 0) * a.d;
      bias[r] = row >= 0 ? a.b1[row] : 0.f;
    }
  };
  RowLoads<T, RPW, U> L;
  if (a.sets_ready) {  // the sets were made before the previous kernel: start streaming W1 now
    slot_range();
    setup_rows(j0, min(j1, j0 + MLP_MAX_ROWS));
    issue_row_loads<T, RPW, U>(L, rowp, valid, nvec, lane);
  }
  griddep_wait();
  if (!a.sets_ready) {
    slot_range();
    setup_rows(j0, min(j1, j0 + MLP_MAX_ROWS));
    issue_row_loads<T, RPW, U>(L, rowp, valid, nvec, lane);
  }
  ln_to_smem<NB>(a.t1, a.d, a.nb, a.eps, a.ln_g, a.ln_b, s_y, red);
  if (blockIdx.x == 0 && a.yM_out) {
    const int n4 = (a.nb * a.d) >> 2;
    for (int i = threadIdx.x; i < n4; i += FUSED_THREADS)
      reinterpret_cast<float4*>(a.yM_out)[i] = reinterpret_cast<const float4*>(s_y)[i];
  }

  const int col = threadIdx.x * E;  // first column of this thread in each 256*E tile
  for (int c0 = j0; c0 < j1 || (c0 == j0 && blockIdx.x == 0); c0 += MLP_MAX_ROWS) {
    const int nrows = max(0, min(MLP_MAX_ROWS, j1 - c0));
    // activations of this chunk: warp w handles slots w*RPW .. (then strided)
    for (int base = 0; base < nrows; base += FUSED_WARPS * RPW) {
      if (!(c0 == j0 && base == 0)) {
        setup_rows(c0 + base, c0 + nrows);
        issue_row_loads<T, RPW, U>(L, rowp, valid, nvec, lane);
      }
      float acc[RPW][NB];
      finish_rows_dot<T, NB, RPW, U>(L, rowp, valid, s_y, a.d, a.nb, acc);
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const int s = base + warp * RPW + r;
          if (s < nrows) {
            int nz = 0;
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              const float v = (valid[r] && b < a.nb) ? activate(acc[r][b] + bias[r], a.act) : 0.f;
              s_act[s][b] = v;
              nz |= v != 0.f;
            }
            s_nz[s] = nz;
            s_row[s] = rows[r];
          }
        }
      }
    }
    __syncthreads();
    if (warp == 0) {  // compact the nonzero slots, in slot order
      int base = 0;
      for (int s0 = 0; s0 < nrows; s0 += 32) {
        const int s = s0 + lane;
        const int nz = s < nrows ? s_nz[s] : 0;
        const unsigned bal = __ballot_sync(0xffffffffu, nz);
        if (nz) s_list[base + __popc(bal & ((1u << lane) - 1u))] = s;
        base += __popc(bal);
      }
      if (lane == 0) s_nlist = base;
    }
    __syncthreads();
    const int nl = s_nlist;
    const bool add_residual = blockIdx.x == 0 && c0 == j0;
    // W2 rows of the nonzero slots, accumulated over all d columns
    for (int t0 = 0; t0 < a.d; t0 += FUSED_THREADS * E) {
      const int c = t0 + col;
      const bool colok = c < a.d;
      float acc[NB][E];
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[b][e] = 0.f;
      if (add_residual && colok) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < a.nb) {
#pragma unroll
            for (int e4 = 0; e4 < E / 4; ++e4) {
              const float4 t = __ldcg(reinterpret_cast<const float4*>(a.t1 + (size_t)b * a.d + c) + e4);
              float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
              if (a.b2) bb = __ldg(reinterpret_cast<const float4*>(a.b2 + c) + e4);
              acc[b][4 * e4 + 0] = t.x + bb.x;
              acc[b][4 * e4 + 1] = t.y + bb.y;
              acc[b][4 * e4 + 2] = t.z + bb.z;
              acc[b][4 * e4 + 3] = t.w + bb.w;
            }
          }
        }
      }
      for (int i0 = 0; i0 < nl; i0 += AX_U) {
        uint4 w[AX_U];
#pragma unroll
        for (int u = 0; u < AX_U; ++u) {
          const int i = i0 + u;
          w[u] = (colok && i < nl) ? ld_stream(W2t + (size_t)s_row[s_list[i]] * a.d + c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < AX_U; ++u) {
          const int i = i0 + u;
          if (i < nl) {
            float wf[E];
            WT<T>::unpack(w[u], wf);
            const int s = s_list[i];
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              const float cb = s_act[s][b];
#pragma unroll
              for (int e = 0; e < E; ++e) acc[b][e] = fmaf(cb, wf[e], acc[b][e]);
            }
          }
        }
      }
      if (colok && (nl > 0 || add_residual)) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < a.nb) {
#pragma unroll
            for (int e4 = 0; e4 < E / 4; ++e4)
              red_add4(a.x + (size_t)b * a.d + c + 4 * e4,
                        make_float4(acc[b][4 * e4], acc[b][4 * e4 + 1], acc[b][4 * e4 + 2], acc[b][4 * e4 + 3]));
          }
        }
      }
    }
    __syncthreads();
    if (nrows == 0) break;
  }
}

// ----------------------------------------------------------------------------
// attn_in_kernel: yA = LN1(x); for the selected heads q, k, v = yA Wqkv[i]^T
// (+ bqkv); q -> workspace, k and v -> KV cache slot pos (eq. (2); KV-cache
// figure (b)). Warp per output row, as qkv_kernel. CTA 0 also writes yA (for
// the look-ahead predictor) and zeroes t1 (the next kernel accumulates into
// it).
// ----------------------------------------------------------------------------
struct AttnInArgs {
  const float* x;
  float* t1;
  float* yA_out;
  const float* ln_g;
  const float* ln_b;
  float eps;
  const void* Wqkv;
  const float* bqkv;
  const int32_t* head_idx;
  const int32_t* head_count;
  int kh_max;
  float* q;
  void* Kc;
  void* Vc;
  int h, dh, d, cap, pos, nb, sets_ready;
  int* status;
  // optional rows of the next layer's predictor, dotted with the same yA
  // (column-owner and streaming kernels): PA2 [n2h][d] -> sh2 [nb][n2h],
  // At2 [n2r][d] -> z2 [nb][n2r]
  const void* PA2;
  const void* At2;
  float* sh2;
  float* z2;
  int n2h, n2r;
};

template <typename T, int NB, int RPW, int U>
__global__ void __launch_bounds__(FUSED_THREADS) attn_in_kernel(AttnInArgs a) {
  constexpr int E = WT<T>::E;
  extern __shared__ __align__(16) float s_y[];
  __shared__ float red[FUSED_WARPS];
  const T* Wqkv = static_cast<const T*>(a.Wqkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = 3 * a.dh;
  const int nvec = a.d / E;
  const int slot0 = (blockIdx.x * FUSED_WARPS + warp) * RPW;
  griddep_launch();
  const T* rowp[RPW];
  bool valid[RPW];
  int heads[RPW];
  auto setup = [&]() {
    int hc = *a.head_count;
    if (hc > a.kh_max || hc < 0) {
      if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(a.status, 1);
      hc = hc < 0 ? 0 : a.kh_max;
    }
    const int nslot = hc * per;
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int slot = slot0 + r;
      int head = -1;
      if (slot < nslot) {
        head = a.head_idx[slot / per];
        if (head < 0 || head >= a.h) {
          if (lane == 0) raise_status(a.status, 2);
          head = -1;
        }
      }
      heads[r] = head;
      valid[r] = head >= 0;
      rowp[r] = Wqkv + ((size_t)(head >= 0 ? head : 0) * per + (slot % per)) * a.d;
    }
  };
  RowLoads<T, RPW, U> L;
  if (a.sets_ready) {
    setup();
    issue_row_loads<T, RPW, U>(L, rowp, valid, nvec, lane);
  }
  griddep_wait();
  if (!a.sets_ready) {
    setup();
    issue_row_loads<T, RPW, U>(L, rowp, valid, nvec, lane);
  }
  ln_to_smem<NB>(a.x, a.d, a.nb, a.eps, a.ln_g, a.ln_b, s_y, red);
  if (blockIdx.x == 0) {
    const int n4 = (a.nb * a.d) >> 2;
    for (int i = threadIdx.x; i < n4; i += FUSED_THREADS) {
      reinterpret_cast<float4*>(a.t1)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (a.yA_out) reinterpret_cast<float4*>(a.yA_out)[i] = reinterpret_cast<const float4*>(s_y)[i];
    }
  }
  float acc[RPW][NB];
  finish_rows_dot<T, NB, RPW, U>(L, rowp, valid, s_y, a.d, a.nb, acc);
  T* Kc = static_cast<T*>(a.Kc);
  T* Vc = static_cast<T*>(a.Vc);
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (lane == ((r * NB + b) & 31) && valid[r] && b < a.nb) {
        const int slot = slot0 + r;
        const int p = slot / per, rem = slot % per, m = rem / a.dh, c = rem % a.dh;
        float v = acc[r][b];
        if (a.bqkv) v += a.bqkv[(size_t)heads[r] * per + rem];
        if (m == 0) {
          a.q[((size_t)b * a.kh_max + p) * a.dh + c] = v;
        } else {
          T* cache = (m == 1) ? Kc : Vc;
          cache[(((size_t)b * a.h + heads[r]) * a.cap + a.pos) * a.dh + c] = WT<T>::store_cvt(v);
        }
      }
    }
  }
}

// ----------------------------------------------------------------------------
// attn_out_kernel: for selected head slot p (grid y) a cluster of CS CTAs
// splits the keys 0..pos: CTA c stages its K/V range in shared memory (slots
// below pos before griddep_wait: they do not depend on attn_in) and forms
// the partial (m, l, acc) of the max-subtracted softmax (eq. (2):
// D_i^{-1} exp(.) X W_i^V), each warp over its own keys with a running max,
// then merged across the CTA's warps. Every CTA stores its partial into the
// shared memory of all CS CTAs of the cluster (distributed shared memory), so
// after one cluster barrier each CTA combines the CS partials into H locally.
// CTA c then multiplies H by its column slice of W_i^O and adds the result to
// t1. With WV > 0 the slice (WV 16-byte vectors per thread) is loaded into
// registers before griddep_wait; with WV = 0 it is streamed afterwards. The
// cluster of slot 0 also moves the residual: t1 += x (+ bO) on its slices,
// then x = 0. With WV = ATTN_H_ONLY the kernel stops at H, which CTA 0 of
// the cluster stores to memory (the W^O product and the residual are then
// wo_stream_kernel's). With WV < 0 (long rows, batch 1-2) CTA c instead multiplies H
// by whole rows c, c + CS, ... of W_i^O (each thread -WV 16-byte vectors of a
// row) and adds its full-width partial to t1: on B200 a CTA streaming whole
// 16-24 KB rows reaches about three times the bandwidth of CTAs that each
// read a 2-3 KB column slice of every row. CTA 0 of slot 0's cluster then
// moves the residual over all columns.
// ----------------------------------------------------------------------------
struct AttnOutArgs {
  const float* q;
  const void* Kc;
  const void* Vc;
  const void* WOt;
  const float* bO;
  const int32_t* head_idx;
  const int32_t* head_count;
  int kh_max;
  float* x;
  float* t1;
  int h, dh, d, cap, pos, nb, S, sets_ready;
  float scale;
  int* status;
  int stage_rows;  // batch rows whose K/V tiles fit in shared memory at once: nb, or 1
  float* H_out;    // [nb][kh_max][dh]: the attention outputs (only with WV = ATTN_H_ONLY)
};

// attn_out_kernel's WV for "attention only": H goes to memory and
// wo_stream_kernel (dv_stream.cuh) multiplies it by the W^O rows
constexpr int ATTN_H_ONLY = 1;

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Merges the softmax partial (mo, lo, ao) into (m, l, acc).
template <int E>
__device__ __forceinline__ void softmax_merge(float& m, float& l, float (&acc)[E], float mo, float lo,
                                              const float (&ao)[E]) {
  const float M = fmaxf(m, mo);
  if (M == -INFINITY) return;  // both empty
  const float c1 = __expf(m - M), c2 = __expf(mo - M);
  l = l * c1 + lo * c2;
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = acc[e] * c1 + ao[e] * c2;
  m = M;
}

template <typename KT, int DH, int CS, int NB, int WV, int NT = FUSED_THREADS>
__global__ void __launch_bounds__(NT) attn_out_kernel(AttnOutArgs a) {
  constexpr int NW = NT / 32;  // warps
  constexpr int E = WT<KT>::E;
  constexpr int G = DH / E;    // lanes per key row
  constexpr int KPW = 32 / G;  // keys per warp step
  constexpr int PW = DH + 2;   // partial: m, l, acc[DH]
  constexpr bool H_ONLY = WV == ATTN_H_ONLY;  // H to global memory; W^O in wo_stream_kernel
  constexpr int RG = (WV > 0 && !H_ONLY) ? DH / WV : 1;  // W^O row groups (register path)
  extern __shared__ __align__(16) unsigned char s_dyn[];
  const int SR = a.stage_rows;
  KT* sK = reinterpret_cast<KT*>(s_dyn);                               // [SR][S][DH]
  KT* sV = sK + (size_t)SR * a.S * DH;                                 // [SR][S][DH]
  float* s_all = reinterpret_cast<float*>(sV + (size_t)SR * a.S * DH);  // [nb][CS][PW]
  float* s_q = s_all + (size_t)a.nb * CS * PW;                          // [nb][DH], scaled q
  __shared__ __align__(16) float s_w[NW][PW];
  __shared__ __align__(16) float s_H[NB][DH];
  __shared__ float s_red[WV != 0 ? 1 : NT * E];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const int p = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const KT* Kc = static_cast<const KT*>(a.Kc);
  const KT* Vc = static_cast<const KT*>(a.Vc);
  const KT* WO = static_cast<const KT*>(a.WOt);
  const int nkeys = a.pos + 1;
  const int t0 = crank * a.S;
  const int nk = max(0, min(a.S, nkeys - t0));
  const int cols = a.d / CS;  // d % (8 CS) == 0 is checked on the host
  const int c_lo = crank * cols;
  griddep_launch();
  cluster_arrive_relaxed();  // waited on before the first store into another CTA

  int hc = 0, head = -1;
  auto read_head = [&]() {
    hc = *a.head_count;
    hc = hc < 0 ? 0 : (hc > a.kh_max ? a.kh_max : hc);
    head = p < hc ? a.head_idx[p] : -1;
    if (p < hc && (head < 0 || head >= a.h)) {
      if (tid == 0 && crank == 0) raise_status(a.status, 2);
      head = -1;
    }
  };
  // stage K/V of batch row b, keys [t0, t0+nk) except slot pos when `old_only`
  auto stage = [&](int b, bool old_only, bool new_only) {
    const int lo = new_only ? (a.pos - t0) : 0;
    const int hi = old_only ? min(nk, a.pos - t0) : nk;
    if (hi <= lo) return;
    const size_t base = (((size_t)b * a.h + head) * a.cap + t0) * DH;
    const size_t tile = (size_t)(b % SR) * a.S * DH;
    const int v0 = lo * DH / E, v1 = hi * DH / E;
    for (int v = v0 + tid; v < v1; v += NT) {
      cp_async16(sK + tile + v * E, Kc + base + (size_t)v * E);
      cp_async16(sV + tile + v * E, Vc + base + (size_t)v * E);
    }
  };
  const bool pos_in_chunk = a.pos >= t0 && a.pos < t0 + nk;
  // register path: thread (cgi, rg) holds rows rg + i RG of column vector cgi
  const int cgi = tid / RG, rg = tid % RG;
  uint4 wo[(WV > 0 && !H_ONLY) ? WV : 1];
  // whole-row path: rows crank + CS u, u < WU, of W_i^O are this CTA's first
  // group; they are loaded into registers at the start, so they arrive while
  // the attention runs
  constexpr int WU = WV < 0 ? (NB == 1 ? 4 : 2) : 1;
  constexpr int NVO = WV < 0 ? -WV : 1;
  uint4 wfirst[WU][NVO];
  auto load_wo = [&]() {
    if constexpr (WV > 0 && !H_ONLY) {
      const KT* Wh = WO + (size_t)head * DH * a.d + c_lo + cgi * E;
#pragma unroll
      for (int i = 0; i < WV; ++i) wo[i] = ld_stream(Wh + (size_t)(rg + i * RG) * a.d);
    } else if constexpr (WV < 0) {
      const KT* Wh = WO + (size_t)head * DH * a.d;
#pragma unroll
      for (int u = 0; u < WU; ++u)
#pragma unroll
        for (int j = 0; j < NVO; ++j) {
          const int r = crank + u * CS, v = tid + j * NT;
          wfirst[u][j] = (r < DH && v * E < a.d) ? ld_stream(Wh + (size_t)r * a.d + (size_t)v * E)
                                                 : make_uint4(0u, 0u, 0u, 0u);
        }
    }
  };
  auto prefetch_wo = [&]() {
    if constexpr (WV == 0) {
      const char* base = reinterpret_cast<const char*>(WO + (size_t)head * DH * a.d + c_lo);
      for (int i = tid; i < DH; i += NT) prefetch_l2(base + (size_t)i * a.d * sizeof(KT), cols * sizeof(KT));
    } else if constexpr (WV < 0) {
      const char* base = reinterpret_cast<const char*>(WO + (size_t)head * DH * a.d);
      for (int i = crank + tid * CS; i < DH; i += NT * CS)
        prefetch_l2(base + (size_t)i * a.d * sizeof(KT), a.d * sizeof(KT));
    }
  };
  // the slots below pos of every batch row whose tiles fit (all rows, or row 0)
  auto stage_old = [&]() {
    for (int b = 0; b < (SR == a.nb ? a.nb : 1); ++b) stage(b, true, false);
  };
  if (a.sets_ready) {
    read_head();
    if (head >= 0) {
      stage_old();
      load_wo();
      prefetch_wo();
    }
  }
  griddep_wait();
  if (!a.sets_ready) {
    read_head();
    if (head >= 0) {
      stage_old();
      load_wo();
    }
  }
  const bool active = head >= 0;
  cluster_wait();  // every CTA of the cluster runs: its shared memory may be written
  // ---- partial attention over this CTA's keys, per batch row ----
  if (active) {
    const int g = lane % G, kq = lane / G;
    const int KW = (nk + NW - 1) / NW;
    const int kw0 = min(nk, warp * KW), kw1 = min(nk, kw0 + KW);
    if (SR == a.nb && pos_in_chunk)
      for (int b = 0; b < a.nb; ++b) stage(b, false, true);  // slot pos of every row, written by attn_in
    // q of every batch row (written by attn_in) in one round of loads
    for (int i = tid; i < a.nb * DH / 4; i += NT) {
      const int b = i / (DH / 4), c4 = i % (DH / 4);
      const float4 v = __ldcg(reinterpret_cast<const float4*>(a.q + ((size_t)b * a.kh_max + p) * DH) + c4);
      reinterpret_cast<float4*>(s_q + (size_t)b * DH)[c4] =
          make_float4(v.x * a.scale, v.y * a.scale, v.z * a.scale, v.w * a.scale);
    }
    for (int b = 0; b < a.nb; ++b) {
      if (b > 0) __syncthreads();  // previous row's s_w (and tiles, when staged row by row) are consumed
      if (SR == 1) {
        if (b > 0) stage(b, false, false);
        else if (pos_in_chunk) stage(0, false, true);  // slot pos, written by attn_in
      }
      const KT* tK = sK + (size_t)(b % SR) * a.S * DH;
      const KT* tV = sV + (size_t)(b % SR) * a.S * DH;
      cp_async_wait_all();
      if (b == 0 || SR == 1) __syncthreads();  // tiles and s_q complete (all rows' tiles land before row 0)
      float qv[E];
#pragma unroll
      for (int e = 0; e < E; ++e) qv[e] = s_q[(size_t)b * DH + g * E + e];
      float m = -INFINITY, l = 0.f, acc[E];
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = 0.f;
      // two key groups per trip (warp-uniform trip count): both dot products
      // and their shuffle reductions are independent, so their latencies
      // overlap; the running-max updates then follow in key order
      for (int tb = kw0; tb < kw1; tb += 2 * KPW) {
        float dot[2];
        bool ok[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int t = tb + u * KPW + kq;
          ok[u] = t < kw1;
          dot[u] = 0.f;
          if (ok[u]) {
            float kf[E];
            WT<KT>::unpack(*reinterpret_cast<const uint4*>(tK + t * DH + g * E), kf);
#pragma unroll
            for (int e = 0; e < E; ++e) dot[u] = fmaf(qv[e], kf[e], dot[u]);
          }
        }
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) {
          dot[0] += __shfl_xor_sync(0xffffffffu, dot[0], o);
          dot[1] += __shfl_xor_sync(0xffffffffu, dot[1], o);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (ok[u]) {
            const int t = tb + u * KPW + kq;
            float vf[E];
            WT<KT>::unpack(*reinterpret_cast<const uint4*>(tV + t * DH + g * E), vf);
            const float mn = fmaxf(m, dot[u]);
            const float c = __expf(m - mn), pe = __expf(dot[u] - mn);
            l = l * c + pe;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = fmaf(pe, vf[e], acc[e] * c);
            m = mn;
          }
        }
      }
      // merge the warp's KPW key groups (lanes g, g + G, ... hold the same dims)
#pragma unroll
      for (int o = G; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o), lo = __shfl_xor_sync(0xffffffffu, l, o);
        float ao[E];
#pragma unroll
        for (int e = 0; e < E; ++e) ao[e] = __shfl_xor_sync(0xffffffffu, acc[e], o);
        softmax_merge<E>(m, l, acc, mo, lo, ao);
      }
      if (kq == 0) {
        if (g == 0) {
          s_w[warp][0] = m;
          s_w[warp][1] = l;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) s_w[warp][2 + g * E + e] = acc[e];
      }
      __syncthreads();
      // this CTA's partial, stored into every CTA of the cluster
      for (int c = tid; c < PW; c += NT) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, s_w[w][0]);
        float v = 0.f;
        if (M != -INFINITY) {
          if (c == 0) {
            v = M;
          } else {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
              const float mw = s_w[w][0];
              v += (mw == -INFINITY) ? 0.f : __expf(mw - M) * s_w[w][c];
            }
          }
        } else {
          v = (c == 0) ? -INFINITY : 0.f;
        }
        const int off = (b * CS + crank) * PW + c;
#pragma unroll
        for (int r = 0; r < CS; ++r) cluster.map_shared_rank(s_all, r)[off] = v;
      }
    }
  }
  cluster.sync();  // every partial has reached every CTA
  if (active) {
    // ---- combine the CS partials of each batch row (local shared memory) ----
    for (int i = tid; i < a.nb * DH; i += NT) {
      const int b = i / DH, c = i % DH;
      const float* pb = s_all + (size_t)b * CS * PW;
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < CS; ++r) M = fmaxf(M, pb[r * PW]);
      float den = 0.f, num = 0.f;
#pragma unroll
      for (int r = 0; r < CS; ++r) {
        const float mr = pb[r * PW];
        const float f = (mr == -INFINITY) ? 0.f : __expf(mr - M);
        den += f * pb[r * PW + 1];
        num += f * pb[r * PW + 2 + c];
      }
      s_H[b][c] = num / den;
    }
  }
  __syncthreads();
  if constexpr (H_ONLY) {  // H of the head to global memory (CTA 0 of the cluster)
    if (active && crank == 0)
      for (int i = tid; i < a.nb * DH; i += NT)
        a.H_out[((size_t)(i / DH) * a.kh_max + p) * DH + i % DH] = s_H[i / DH][i % DH];
    return;
  }
  // slot 0's cluster moves the residual: every CTA on its own column slice,
  // or CTA 0 on all columns when CTAs take whole rows
  const bool residual = (p == 0) && (WV >= 0 || crank == 0);
  if (!active && !residual) return;
  // residual (slot 0's cluster): o += x + bO at columns c..c+E-1, then x = 0
  auto add_residual = [&](float (&o)[E], int b, int c) {
    float* xr = a.x + (size_t)b * a.d + c;
#pragma unroll
    for (int e4 = 0; e4 < E / 4; ++e4) {
      const float4 xv = __ldcg(reinterpret_cast<const float4*>(xr) + e4);
      float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
      if (a.bO) bb = __ldg(reinterpret_cast<const float4*>(a.bO + c) + e4);
      o[4 * e4 + 0] += xv.x + bb.x;
      o[4 * e4 + 1] += xv.y + bb.y;
      o[4 * e4 + 2] += xv.z + bb.z;
      o[4 * e4 + 3] += xv.w + bb.w;
      reinterpret_cast<float4*>(xr)[e4] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  if constexpr (WV < 0) {
    // ---- whole rows crank, crank + CS, ... of W_i^O; this thread's vectors
    // tid + 256 j of each row; U rows in flight, the first group loaded at
    // the start of the kernel ----
    constexpr int U = WU;
    const KT* Wh = WO + (size_t)head * DH * a.d;
    float o[NB][NVO][E];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int j = 0; j < NVO; ++j)
#pragma unroll
        for (int e = 0; e < E; ++e) o[b][j][e] = 0.f;
    auto consume = [&](const uint4 (&w)[U][NVO], int r0) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int r = r0 + u * CS;
        if (r < DH) {
#pragma unroll
          for (int j = 0; j < NVO; ++j) {
            float wf[E];
            WT<KT>::unpack(w[u][j], wf);
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              const float hv = b < a.nb ? s_H[b][r] : 0.f;
#pragma unroll
              for (int e = 0; e < E; ++e) o[b][j][e] = fmaf(hv, wf[e], o[b][j][e]);
            }
          }
        }
      }
    };
    if (active) {
      consume(wfirst, crank);
#pragma unroll 1
      for (int r0 = crank + CS * U; r0 < DH; r0 += CS * U) {
        uint4 w[U][NVO];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int j = 0; j < NVO; ++j) {
            const int r = r0 + u * CS, v = tid + j * NT;
            w[u][j] = (r < DH && v * E < a.d) ? ld_stream(Wh + (size_t)r * a.d + (size_t)v * E)
                                              : make_uint4(0u, 0u, 0u, 0u);
          }
        consume(w, r0);
      }
    }
#pragma unroll
    for (int j = 0; j < NVO; ++j) {
      const int c = (tid + j * NT) * E;
      if (c >= a.d) continue;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b >= a.nb) break;
        if (residual) add_residual(o[b][j], b, c);
#pragma unroll
        for (int e4 = 0; e4 < E / 4; ++e4)
          red_add4(a.t1 + (size_t)b * a.d + c + 4 * e4,
                   make_float4(o[b][j][4 * e4], o[b][j][4 * e4 + 1], o[b][j][4 * e4 + 2], o[b][j][4 * e4 + 3]));
      }
    }
  } else if constexpr (WV > 0 && !H_ONLY) {
    // ---- W^O slice from registers; row groups reduced across RG lanes ----
    float o[NB][E];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < E; ++e) o[b][e] = 0.f;
    if (active) {
#pragma unroll
      for (int i = 0; i < WV; ++i) {
        float wf[E];
        WT<KT>::unpack(wo[i], wf);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float hv = b < a.nb ? s_H[b][rg + i * RG] : 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) o[b][e] = fmaf(hv, wf[e], o[b][e]);
        }
      }
    }
#pragma unroll
    for (int sh = RG / 2; sh > 0; sh >>= 1)
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < E; ++e) o[b][e] += __shfl_xor_sync(0xffffffffu, o[b][e], sh);
    if (rg == 0) {
      const int c = c_lo + cgi * E;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b >= a.nb) break;
        if (residual) add_residual(o[b], b, c);
#pragma unroll
        for (int e4 = 0; e4 < E / 4; ++e4)
          red_add4(a.t1 + (size_t)b * a.d + c + 4 * e4,
                   make_float4(o[b][4 * e4], o[b][4 * e4 + 1], o[b][4 * e4 + 2], o[b][4 * e4 + 3]));
      }
    }
  } else {
    // ---- W^O slice streamed: columns [c_lo, c_lo + cols) ----
    const int ncg = cols / E;
    for (int cg0 = 0; cg0 < ncg; cg0 += NT) {
      const int ngrp = min(NT, ncg - cg0);
      const int nrg = max(1, NT / ngrp);  // row groups
      const int cgj = tid % ngrp, rgj = tid / ngrp;
      const bool thr_ok = rgj < nrg && tid < ngrp * nrg;
      const int c = c_lo + (cg0 + cgj) * E;
      float acc[NB][E];
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[b][e] = 0.f;
      if (active && thr_ok) {
        constexpr int WO_U = 16;  // rows of W^O in flight per thread
        const KT* Wh = WO + (size_t)head * DH * a.d + c;
        for (int i0 = rgj; i0 < DH; i0 += nrg * WO_U) {
          uint4 w[WO_U];
#pragma unroll
          for (int u = 0; u < WO_U; ++u) {
            const int i = i0 + u * nrg;
            w[u] = i < DH ? ld_stream(Wh + (size_t)i * a.d) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int u = 0; u < WO_U; ++u) {
            const int i = i0 + u * nrg;
            if (i < DH) {
              float wf[E];
              WT<KT>::unpack(w[u], wf);
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                if (b < a.nb) {
                  const float hv = s_H[b][i];
#pragma unroll
                  for (int e = 0; e < E; ++e) acc[b][e] = fmaf(hv, wf[e], acc[b][e]);
                }
              }
            }
          }
        }
      }
      // reduce the row groups, one batch row at a time (unrolled, so that
      // acc keeps static indices and stays in registers)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b >= a.nb) break;
        if (nrg > 1) {
          __syncthreads();
          if (thr_ok) {
#pragma unroll
            for (int e = 0; e < E; ++e) s_red[(rgj * ngrp + cgj) * E + e] = acc[b][e];
          }
          __syncthreads();
        }
        if (rgj == 0 && thr_ok) {
          float o[E];
#pragma unroll
          for (int e = 0; e < E; ++e) {
            float sum = acc[b][e];
            for (int r2 = 1; r2 < nrg; ++r2) sum += s_red[(r2 * ngrp + cgj) * E + e];
            o[e] = sum;
          }
          if (residual) add_residual(o, b, c);
#pragma unroll
          for (int e4 = 0; e4 < E / 4; ++e4)
            red_add4(a.t1 + (size_t)b * a.d + c + 4 * e4,
                     make_float4(o[4 * e4], o[4 * e4 + 1], o[4 * e4 + 2], o[4 * e4 + 3]));
        }
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Look-ahead predictor, first kernel: rows [0, h) of PA give the head scores
// s_A[b][i] = y[b] . PA[i]; rows [h, h + r) of At give z[b][c] = y[b] . At[c]
// (the first factor of the neuron predictor). The weight rows do not depend
// on the previous kernel, so their first loads go out before griddep_wait.
// ----------------------------------------------------------------------------
struct PredictAArgs {
  const float* y;  // [B][d]
  const void* PA;  // [h][d] (null when heads are not predicted)
  const void* At;  // [r][d] (null when z is not needed)
  int h, r, d, nb;
  float* scores_h;  // [B][h]
  float* z;         // [B][r]
};

template <typename T, int NB, int RPW, int U>
__global__ void __launch_bounds__(FUSED_THREADS) predict_a_kernel(PredictAArgs a) {
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int heads = a.PA ? a.h : 0;
  const int nrows = heads + (a.At ? a.r : 0);
  const int row0 = (blockIdx.x * FUSED_WARPS + warp) * RPW;
  const T* rowp[RPW];
  bool valid[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int row = row0 + r;
    valid[r] = row < nrows;
    const T* base = row < heads ? static_cast<const T*>(a.PA) + (size_t)row * a.d
                                : static_cast<const T*>(a.At) + (size_t)(valid[r] ? row - heads : 0) * a.d;
    rowp[r] = valid[r] ? base : static_cast<const T*>(heads ? a.PA : a.At);
  }
  RowLoads<T, RPW, U> L;
  issue_row_loads<T, RPW, U>(L, rowp, valid, a.d / WT<T>::E, lane);
  griddep_wait();  // y comes from the previous kernel
  float acc[RPW][NB];
  finish_rows_dot<T, NB, RPW, U>(L, rowp, valid, a.y, a.d, a.nb, acc);
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b)
      if (lane == ((r * NB + b) & 31) && valid[r] && b < a.nb) {
        const int row = row0 + r;
        if (row < heads) a.scores_h[(size_t)b * a.h + row] = acc[r][b];
        else a.z[(size_t)b * a.r + row - heads] = acc[r][b];
      }
}

// ----------------------------------------------------------------------------
// Look-ahead predictor, second kernel: neuron scores s[b][i] = z[b] . Bm[i] +
// b1[i] (rows of length r). Persistent grid: warp w of CTA c takes row
// groups (c * FUSED_WARPS + w) RPW + k (grid size) RPW, and issues the loads
// of its next group before it reduces the current one, so two groups per
// warp are always in flight.
// ----------------------------------------------------------------------------
struct PredictBArgs {
  const float* z;  // [B][r]
  const void* Bm;  // [N][r]
  const float* b1; // [N]
  int N, r, nb;
  float* scores;   // [B][N]
};

template <typename T, int NB, int RPW, int U, int MINB = 1>
__global__ void __launch_bounds__(FUSED_THREADS, MINB) predict_b_kernel(PredictBArgs a) {
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = a.r / WT<T>::E;
  const int stride = gridDim.x * FUSED_WARPS * RPW;
  const T* Bm = static_cast<const T*>(a.Bm);
  auto setup = [&](int r0, const T* (&rowp)[RPW], bool (&valid)[RPW]) {
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      valid[r] = r0 + r < a.N;
      rowp[r] = Bm + (size_t)(valid[r] ? r0 + r : 0) * a.r;
    }
  };
  int row0 = (blockIdx.x * FUSED_WARPS + warp) * RPW;
  const T* rp[RPW];
  bool vd[RPW];
  RowLoads<T, RPW, U> L;
  setup(row0, rp, vd);
  issue_row_loads<T, RPW, U>(L, rp, vd, nvec, lane);  // Bm does not depend on the previous kernel
  griddep_wait();                                     // z does
#pragma unroll 1
  for (; row0 < a.N; row0 += stride) {
    const T* rpn[RPW];
    bool vn[RPW];
    RowLoads<T, RPW, U> Ln;
    setup(row0 + stride, rpn, vn);
    issue_row_loads<T, RPW, U>(Ln, rpn, vn, nvec, lane);
    float acc[RPW][NB];
    finish_rows_dot<T, NB, RPW, U>(L, rp, vd, a.z, a.r, a.nb, acc);
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (lane == ((r * NB + b) & 31) && vd[r] && b < a.nb)
          a.scores[(size_t)b * a.N + row0 + r] = acc[r][b] + a.b1[row0 + r];
    L = Ln;
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      rp[r] = rpn[r];
      vd[r] = vn[r];
    }
  }
}


}  // namespace dv
