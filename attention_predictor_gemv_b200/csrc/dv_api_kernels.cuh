// Kernels that the C ABI layer launches itself: LayerNorm, the exact
// selection that ends the look-ahead predictor, its gate, and the L2
// prefetch of a layer's selected rows. Included by one translation unit.
#pragma once

#include "dv_fused.cuh"

namespace dv {

// ----------------------------------------------------------------------------
// LayerNorm: y = (x - mean) / sqrt(var + eps) * g + b, biased variance, one CTA
// per batch row.
// ----------------------------------------------------------------------------
constexpr int LN_THREADS = 512;

__global__ void __launch_bounds__(LN_THREADS)
    layernorm_kernel(const float* __restrict__ x, float* __restrict__ y, int d, const float* __restrict__ g,
                     const float* __restrict__ bta, float eps) {
  __shared__ float red[LN_THREADS / 32];
  griddep_launch();
  griddep_wait();
  const int b = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)b * d);
  float4* yr = reinterpret_cast<float4*>(y + (size_t)b * d);
  const int n4 = d >> 2;
  float s = 0.f;
  for (int i = threadIdx.x; i < n4; i += LN_THREADS) {
    float4 v = xr[i];
    s += (v.x + v.y) + (v.z + v.w);
  }
  const float mean = block_sum<LN_THREADS>(s, red) / (float)d;
  float q = 0.f;
  for (int i = threadIdx.x; i < n4; i += LN_THREADS) {
    float4 v = xr[i];
    float a = v.x - mean, c = v.y - mean, e = v.z - mean, f = v.w - mean;
    q += (a * a + c * c) + (e * e + f * f);
  }
  const float var = block_sum<LN_THREADS>(q, red) / (float)d;
  const float rstd = rsqrtf(var + eps);
  for (int i = threadIdx.x; i < n4; i += LN_THREADS) {
    float4 v = xr[i];
    float4 o = make_float4((v.x - mean) * rstd, (v.y - mean) * rstd, (v.z - mean) * rstd, (v.w - mean) * rstd);
    if (g) {
      float4 gg = reinterpret_cast<const float4*>(g)[i];
      o.x *= gg.x; o.y *= gg.y; o.z *= gg.z; o.w *= gg.w;
    }
    if (bta) {
      float4 bb = reinterpret_cast<const float4*>(bta)[i];
      o.x += bb.x; o.y += bb.y; o.z += bb.z; o.w += bb.w;
    }
    yr[i] = o;
  }
}

// ----------------------------------------------------------------------------
// L2 prefetch of one layer's selected parameters. With the look-ahead
// predictor the sets of layer l+1 are known while layer l runs; this kernel
// (on the side stream) asks the bulk-copy engine to bring layer l+1's
// selected Q/K/V and W^O blocks, the selected heads' KV entries and the
// selected W1 (and optionally W2) rows into L2, so layer l+1's kernels read
// them from L2. Fire-and-forget: no data moves through the SMs.
// ----------------------------------------------------------------------------
struct PrefetchArgs {
  const char* Wqkv;
  const char* WOt;
  const char* Kc;
  const char* Vc;
  const char* W1t;
  const char* W2t;
  const int32_t* head_idx;
  const int32_t* head_count;
  const int32_t* idx;
  const int32_t* count;
  int kh_max, k_max, B, h, dh, d, N, cap, pos, wbytes, kvbytes, with_w2;
};

__device__ __forceinline__ void prefetch_range(const char* base, size_t bytes, int chunk) {
  const size_t off = (size_t)chunk * PF_CHUNK;
  if (off < bytes) prefetch_l2(base + off, (uint32_t)min((size_t)PF_CHUNK, bytes - off));
}

__global__ void __launch_bounds__(256) prefetch_layer_kernel(PrefetchArgs a) {
  griddep_launch();
  griddep_wait();
  int hc = *a.head_count, cnt = *a.count;
  hc = hc < 0 ? 0 : (hc > a.kh_max ? a.kh_max : hc);
  cnt = cnt < 0 ? 0 : (cnt > a.k_max ? a.k_max : cnt);
  const size_t qkv = (size_t)3 * a.dh * a.d * a.wbytes, wo = (size_t)a.dh * a.d * a.wbytes;
  const size_t kv = (size_t)a.pos * a.dh * a.kvbytes, row = (size_t)a.d * a.wbytes;
  const int nq = (int)((qkv + PF_CHUNK - 1) / PF_CHUNK), nwo = (int)((wo + PF_CHUNK - 1) / PF_CHUNK);
  const int nkv = (int)((kv + PF_CHUNK - 1) / PF_CHUNK), nrow = (int)((row + PF_CHUNK - 1) / PF_CHUNK);
  const int per_head = nq + nwo + 2 * a.B * nkv;
  const int per_neuron = nrow * (a.with_w2 ? 2 : 1);
  const long long total = (long long)hc * per_head + (long long)cnt * per_neuron;
  for (long long it = blockIdx.x * 256ll + threadIdx.x; it < total; it += (long long)gridDim.x * 256) {
    if (it < (long long)hc * per_head) {
      const int p = (int)(it / per_head);
      int c = (int)(it % per_head);
      const int head = a.head_idx[p];
      if (head < 0 || head >= a.h) continue;
      if (c < nq) {
        prefetch_range(a.Wqkv + (size_t)head * qkv, qkv, c);
      } else if ((c -= nq) < nwo) {
        prefetch_range(a.WOt + (size_t)head * wo, wo, c);
      } else {
        c -= nwo;
        const int which = c / (a.B * nkv);  // 0: K, 1: V
        c %= a.B * nkv;
        const int b = c / nkv;
        const size_t cache_off = (((size_t)b * a.h + head) * a.cap) * a.dh * a.kvbytes;
        prefetch_range((which ? a.Vc : a.Kc) + cache_off, kv, c % nkv);
      }
    } else {
      const long long r = it - (long long)hc * per_head;
      const int j = (int)(r / per_neuron);
      int c = (int)(r % per_neuron);
      const int neuron = a.idx[j];
      if (neuron < 0 || neuron >= a.N) continue;
      const char* base = (c < nrow ? a.W1t : a.W2t) + (size_t)neuron * row;
      prefetch_range(base, row, c % nrow);
    }
  }
}

// ----------------------------------------------------------------------------
// Head selection from the head scores of B rows: the union over the rows of
// each row's k_h best (ties to the lower index) or of its scores > tau. Few
// heads (h <= HSEL_MAX): every thread ranks its head by direct comparison
// with all others. One CTA.
// ----------------------------------------------------------------------------
struct SelectHeadsArgs {
  const float* scores_h;  // [B][h]
  int nb, h, k_h, mode_h;
  float tau_h;
  int32_t* head_idx;
  int32_t* head_count;
};

__global__ void __launch_bounds__(SEL_THREADS) select_heads_kernel(SelectHeadsArgs a) {
  extern __shared__ uint32_t s_keys[];  // [h]
  __shared__ uint32_t s_hsel[HSEL_MAX / 32];
  griddep_launch();
  griddep_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = a.h, nw = (h + 31) >> 5;
  for (int w = tid; w < nw; w += SEL_THREADS) s_hsel[w] = 0u;
  for (int b = 0; b < a.nb; ++b) {
    __syncthreads();
    for (int i = tid; i < h; i += SEL_THREADS) s_keys[i] = ord_key(a.scores_h[(size_t)b * h + i]);
    __syncthreads();
    for (int i = tid; i < h; i += SEL_THREADS) {
      bool take;
      if (a.mode_h == 1) {
        take = a.scores_h[(size_t)b * h + i] > a.tau_h;
      } else {
        const uint32_t ki = s_keys[i];
        int rank = 0;
        for (int j = 0; j < h; ++j) {
          const uint32_t kj = s_keys[j];
          rank += (kj > ki) || (kj == ki && j < i);
        }
        take = rank < a.k_h;
      }
      if (take) atomicOr(&s_hsel[i >> 5], 1u << (i & 31));
    }
  }
  __syncthreads();
  if (warp == 0) {
    unsigned base = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t u = w < nw ? s_hsel[w] : 0u;
      const unsigned c = __popc(u);
      unsigned incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      unsigned off = base + incl - c;
      uint32_t v = u;
      while (v) {
        const int jb = __ffs(v) - 1;
        v &= v - 1u;
        a.head_idx[off++] = w * 32 + jb;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *a.head_count = (int32_t)base;
  }
}

// ----------------------------------------------------------------------------
// select_rows_kernel: the selected set of B score rows of length n (top-k per
// row, ties to the lower index, or s > tau), united over the rows, as an
// ascending index list. One thread-block cluster of SR_CS CTAs per row; CTA
// c holds the keys of a contiguous index range of the row in registers
// (order-preserving 32-bit keys: NaN lowest, -0 == +0), SR_KPT per thread.
//
// Top-k: the k-th largest key T is found exactly by four radix passes of 8
// bits, most significant first. In each pass every warp counts the digits of
// its keys that match the prefix found so far into its own 256-bin
// histogram in shared memory; the CTA sums its 8 warp histograms, publishes
// the sum, and after one cluster barrier every CTA reads the SR_CS sums
// through distributed shared memory and picks the same digit. The keys above
// T are taken, and of the keys equal to T the kk lowest-index ones (their
// rank is the count of equal keys in lower-indexed words: in the warp, the
// CTA's earlier warps, and the cluster's earlier CTAs).
//
// The row's bitmap: with one row each CTA writes its own indices at its
// offset in the cluster; with several rows every cluster stores its bitmap,
// and the last cluster to finish (ticket) ORs the rows and writes the union.
// ----------------------------------------------------------------------------
constexpr int SR_CS = 8;
constexpr int SR_THREADS = 256;
constexpr int SR_WARPS = SR_THREADS / 32;
constexpr int SR_KPT = 24;
constexpr int SR_MAX_N = SR_CS * SR_THREADS * SR_KPT;  // 49152
constexpr int SR_MAX_WPC = SR_MAX_N / 32 / SR_CS;      // bitmap words per CTA

struct SelectRowsArgs {
  const float* scores;  // [nrows][n]
  int n, nrows, k, mode;
  float tau;
  uint32_t* bitmaps;    // [nrows][(n + 31) / 32] (used when nrows > 1)
  unsigned* ticket;     // zero on entry, left zero
  int32_t* idx;
  int32_t* count;
};

__global__ void __launch_bounds__(SR_THREADS) select_rows_kernel(SelectRowsArgs a) {
  __shared__ unsigned s_wh[SR_WARPS][256];  // per-warp digit histograms
  __shared__ unsigned s_cnt[2][256];        // this CTA's digit counts (read by the cluster)
  __shared__ uint32_t s_bm[SR_MAX_WPC];     // this CTA's bitmap words
  __shared__ unsigned s_wv[SR_WARPS];       // per-warp counts
  __shared__ unsigned sc[SR_WARPS + 1];
  __shared__ unsigned s_ceq, s_csel, s_digit, s_kk;  // s_ceq, s_csel: read by the cluster
  __shared__ int s_last;
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  griddep_launch();
  griddep_wait();
  const int n = a.n, nw = (n + 31) >> 5;
  const int wpc = (nw + SR_CS - 1) / SR_CS;
  const int cw0 = crank * wpc, cw1 = min(nw, cw0 + wpc);
  const int wpw = (wpc + SR_WARPS - 1) / SR_WARPS;  // <= SR_KPT (n <= SR_MAX_N, checked on the host)
  const int ww0 = cw0 + warp * wpw, ww1 = min(cw1, ww0 + wpw);
  const float* srow = a.scores + (size_t)row * n;

  uint32_t key[SR_KPT];
  unsigned vmask = 0u;  // bit j: key j exists
#pragma unroll
  for (int j = 0; j < SR_KPT; ++j) {
    const int w = ww0 + j, i = w * 32 + lane;
    const bool v = w < ww1 && i < n;
    key[j] = v ? ord_key(srow[i]) : 0u;
    vmask |= (v ? 1u : 0u) << j;
  }

  const bool topk = a.mode == 0 && a.k > 0 && a.k < n;
  uint32_t T = 0u;
  unsigned kk = 0u;
  if (topk) {
    uint32_t prefix = 0u, mask = 0u;
    kk = (unsigned)a.k;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
#pragma unroll
      for (int w = 0; w < SR_WARPS; ++w) s_wh[w][tid] = 0u;
      __syncthreads();
      // per-key adds; grouping a warp's equal digits first (__match_any_sync)
      // made the whole look-ahead step 20 us per layer slower when this kernel
      // ran beside the main-stream kernels (measured at N = 49152), though it
      // was not slower alone
#pragma unroll
      for (int j = 0; j < SR_KPT; ++j)
        if (((vmask >> j) & 1u) && (key[j] & mask) == prefix) atomicAdd(&s_wh[warp][(key[j] >> shift) & 255u], 1u);
      __syncthreads();
      unsigned c = 0u;
#pragma unroll
      for (int w = 0; w < SR_WARPS; ++w) c += s_wh[w][255 - tid];  // thread t: bin 255 - t (descending)
      s_cnt[pass & 1][tid] = c;
      cluster.sync();
      unsigned tot = 0u;
#pragma unroll
      for (int r = 0; r < SR_CS; ++r) tot += cluster.map_shared_rank(&s_cnt[pass & 1][0], r)[tid];
      unsigned total;
      const unsigned above = block_exclusive_scan<SR_THREADS>(tot, sc, &total);
      if (above < kk && kk <= above + tot) {
        s_digit = 255u - (unsigned)tid;
        s_kk = kk - above;
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= 0xffu << shift;
      kk = s_kk;
    }
    T = prefix;  // the k-th largest key; kk of the keys equal to it are taken
  }

  // ---- this CTA's bitmap words ----
  unsigned rank = 0u;  // keys equal to T in lower-indexed words of the row
  if (topk) {
    unsigned eq = 0u;
#pragma unroll
    for (int j = 0; j < SR_KPT; ++j) eq += __popc(__ballot_sync(0xffffffffu, ((vmask >> j) & 1u) && key[j] == T));
    if (lane == 0) s_wv[warp] = eq;
    __syncthreads();
    unsigned ctot = 0u, wbefore = 0u;
#pragma unroll
    for (int w = 0; w < SR_WARPS; ++w) {
      wbefore += w < warp ? s_wv[w] : 0u;
      ctot += s_wv[w];
    }
    if (tid == 0) s_ceq = ctot;
    cluster.sync();
    unsigned cbefore = 0u;
    for (int r = 0; r < crank; ++r) cbefore += *cluster.map_shared_rank(&s_ceq, r);
    rank = cbefore + wbefore;
  }
  const uint32_t tau_key = ord_key(a.tau);
  const bool tau_nan = a.tau != a.tau;
  unsigned nsel = 0u;
#pragma unroll
  for (int j = 0; j < SR_KPT; ++j) {
    const bool v = (vmask >> j) & 1u;
    bool take;
    if (topk) {
      const bool e = v && key[j] == T;
      const unsigned em = __ballot_sync(0xffffffffu, e);
      take = v && (key[j] > T || (e && rank + __popc(em & lt) < kk));
      rank += __popc(em);
    } else if (a.mode == 1) {
      take = v && !tau_nan && key[j] != 0u && key[j] > tau_key;  // NaN (key 0) never passes
    } else {
      take = v && a.k >= n;
    }
    const uint32_t word = __ballot_sync(0xffffffffu, take);
    const int w = ww0 + j;
    if (lane == 0 && w < ww1) s_bm[w - cw0] = word;
    nsel += __popc(word);
  }
  __syncthreads();

  // ---- several rows: store the bitmap; the last cluster forms the union ----
  if (a.nrows > 1) {
    uint32_t* bm = a.bitmaps + (size_t)row * nw;
    for (int w = cw0 + tid; w < cw1; w += SR_THREADS) bm[w] = s_bm[w - cw0];
    __threadfence();
    cluster.sync();  // every CTA of the row has stored its words
    if (crank == 0 && tid == 0) {
      const int last = atomicAdd(a.ticket, 1u) == (unsigned)a.nrows - 1u;
#pragma unroll
      for (int r = 0; r < SR_CS; ++r) *cluster.map_shared_rank(&s_last, r) = last;
    }
    cluster.sync();
    if (!s_last) return;
    __threadfence();
    nsel = 0u;
    for (int w = cw0 + tid; w < cw1; w += SR_THREADS) {
      uint32_t u = 0u;
      for (int rr = 0; rr < a.nrows; ++rr) u |= __ldcg(a.bitmaps + (size_t)rr * nw + w);
      s_bm[w - cw0] = u;
    }
    __syncthreads();
    if (crank == 0 && tid == 0) *a.ticket = 0u;
    for (int w = ww0; w < ww1; ++w) nsel += __popc(s_bm[w - cw0]) * (lane == 0 ? 1u : 0u);
    nsel = __reduce_add_sync(0xffffffffu, nsel);
  } else {
    nsel = __shfl_sync(0xffffffffu, nsel, 0);
  }
  // ---- the index list: warp offsets in the CTA, CTA offsets in the cluster ----
  if (lane == 0) s_wv[warp] = nsel;
  __syncthreads();
  unsigned ctot = 0u, wbefore = 0u;
#pragma unroll
  for (int w = 0; w < SR_WARPS; ++w) {
    wbefore += w < warp ? s_wv[w] : 0u;
    ctot += s_wv[w];
  }
  if (tid == 0) s_csel = ctot;
  cluster.sync();
  unsigned off = wbefore;
  for (int r = 0; r < crank; ++r) off += *cluster.map_shared_rank(&s_csel, r);
  if (crank == SR_CS - 1 && tid == 0) *a.count = (int32_t)(off - wbefore + ctot);
  for (int w = ww0; w < ww1; ++w) {
    const uint32_t u = s_bm[w - cw0];
    if ((u >> lane) & 1u) a.idx[off + __popc(u & lt)] = w * 32 + lane;
    off += __popc(u);
  }
  cluster.sync();  // no CTA exits while another may still read its shared memory
}

// ----------------------------------------------------------------------------
// Gate: returns once the previous kernel on its stream has completed and its
// writes are visible. Ends the look-ahead predictor so that a kernel on
// another stream that depends on it through an event, and that may be
// launched early by programmatic dependent launch (stream capture can give
// such a cross-stream edge the programmatic type), cannot start before the
// predicted sets are complete: it starts at the earliest when the gate has
// exited.
// ----------------------------------------------------------------------------
__global__ void gate_kernel() { griddep_wait(); }

}  // namespace dv
