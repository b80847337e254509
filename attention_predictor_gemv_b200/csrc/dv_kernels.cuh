// Decode-step kernels: LayerNorm, row GEMVs (dense and gathered), selection,
// split-K decode attention and gather-axpy accumulation.
//
// Everything here is HBM-bound GEMV work at small batch: each weight byte is
// used for B multiply-adds. The kernels stream whole rows with 16-byte loads,
// keep 8 loads in flight per lane, reduce with warp shuffles, and never wait
// on another CTA (cross-CTA steps use a last-CTA-done ticket).
#pragma once

#include "dv_common.cuh"

namespace dv {

// ----------------------------------------------------------------------------
// Warp row-dot: one warp forms the dot products of RPW weight rows (K elements
// each, 16-byte aligned) with nb <= NB fp32 input vectors X[b][0..K). U column
// steps of RPW loads each are issued before any use: RPW * U = 8 loads of 16
// bytes in flight per lane. On return every lane holds the full sums.
// ----------------------------------------------------------------------------
template <typename T, int NB, int RPW, int U>
__device__ __forceinline__ void warp_rows_dot(const T* const (&rowp)[RPW], const bool (&valid)[RPW], int K,
                                              const float* __restrict__ X, int ldx, int nb,
                                              float (&acc)[RPW][NB]) {
  constexpr int E = WT<T>::E;
  const int lane = threadIdx.x & 31;
  const int nvec = K / E;
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
  for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
    uint4 w[U][RPW];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * 32;
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        if (valid[r] && v < nvec) w[u][r] = ld_stream(rowp[r] + (size_t)v * E);
        else w[u][r] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * 32;
      if (v < nvec) {
        float wf[RPW][E];
#pragma unroll
        for (int r = 0; r < RPW; ++r) WT<T>::unpack(w[u][r], wf[r]);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < nb) {
            float xv[E];
            const float4* xp = reinterpret_cast<const float4*>(X + (size_t)b * ldx + (size_t)v * E);
#pragma unroll
            for (int e4 = 0; e4 < E / 4; ++e4) {
              float4 t = __ldg(xp + e4);
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
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = warp_sum(acc[r][b]);
}

constexpr int GEMV_WARPS = 8;
constexpr int GEMV_THREADS = GEMV_WARPS * 32;

// Dense GEMV over rows 0..nrows-1 of W [nrows][K]: out[b][i] = W[i] . X[b] + bias[i].
template <typename T, int NB, int RPW, int U>
__global__ void __launch_bounds__(GEMV_THREADS)
    dense_gemv_kernel(const T* __restrict__ W, int nrows, int K, const float* __restrict__ X, int ldx, int nb,
                      const float* __restrict__ bias, float* __restrict__ out, int ldo) {
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * GEMV_WARPS + warp) * RPW;
  const T* rowp[RPW];
  bool valid[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    valid[r] = row0 + r < nrows;
    rowp[r] = W + (size_t)(valid[r] ? row0 + r : 0) * K;
  }
  griddep_wait();  // X comes from the previous kernel
  float acc[RPW][NB];
  warp_rows_dot<T, NB, RPW, U>(rowp, valid, K, X, ldx, nb, acc);
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b)
      if (lane == ((r * NB + b) & 31) && valid[r] && b < nb)
        out[(size_t)b * ldo + row0 + r] = acc[r][b] + (bias ? bias[row0 + r] : 0.f);
}

// ----------------------------------------------------------------------------
// Sparse W1 GEMV + b1 + ReLU + compaction (eq. (1), first factor).
// CTA c owns selection slots [c*SEG, (c+1)*SEG), SEG = GEMV_WARPS * RPW. It
// writes the slots whose activation is nonzero in some batch row, in slot
// order, to seg_idx / seg_a at the segment's base and their number to
// seg_cnt[c]. Compaction is thus deterministic: the consumer forms the
// prefix sum over seg_cnt.
// ----------------------------------------------------------------------------
template <typename T, int NB, int RPW, int U>
__global__ void __launch_bounds__(GEMV_THREADS)
    mlp_up_kernel(const T* __restrict__ W1t, int d, int N, const float* __restrict__ X, int nb,
                  const float* __restrict__ b1, const int32_t* __restrict__ idx, const int32_t* __restrict__ count_dev,
                  int k_max, int32_t* __restrict__ seg_idx, float* __restrict__ seg_a, int32_t* __restrict__ seg_cnt,
                  int* __restrict__ status, int act, const float* __restrict__ wscale) {
  constexpr int SEG = GEMV_WARPS * RPW;
  __shared__ float s_a[SEG][NB];
  __shared__ int s_row[SEG];
  __shared__ int s_nz[SEG];
  griddep_launch();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int cnt = *count_dev;
  if (cnt > k_max || cnt < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(status, 1);
    cnt = cnt < 0 ? 0 : k_max;
  }
  const int slot0 = blockIdx.x * SEG + warp * RPW;
  const T* rowp[RPW];
  bool valid[RPW];
  int rows[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int slot = slot0 + r;
    int row = slot < cnt ? idx[slot] : -1;
    if (slot < cnt && (row < 0 || row >= N)) {
      if (lane == 0) raise_status(status, 2);
      row = -1;
    }
    rows[r] = row;
    valid[r] = row >= 0;
    rowp[r] = W1t + (size_t)(row >= 0 ? row : 0) * d;
  }
  float acc[RPW][NB];
  warp_rows_dot<T, NB, RPW, U>(rowp, valid, d, X, d, nb, acc);
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      int nz = 0;
      const float bias = valid[r] ? b1[rows[r]] : 0.f;
      const float sc = (valid[r] && wscale) ? wscale[rows[r]] : 1.f;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float a = (valid[r] && b < nb) ? activate(acc[r][b] * sc + bias, act) : 0.f;
        s_a[warp * RPW + r][b] = a;
        nz |= a != 0.f;
      }
      s_nz[warp * RPW + r] = nz;
      s_row[warp * RPW + r] = rows[r];
    }
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0;
#pragma unroll
    for (int c0 = 0; c0 < SEG; c0 += 32) {
      const int j = c0 + lane;
      const int nz = (j < SEG) ? s_nz[j] : 0;
      const unsigned bal = __ballot_sync(0xffffffffu, nz);
      if (nz) {
        const int p = blockIdx.x * SEG + base + __popc(bal & ((1u << lane) - 1u));
        seg_idx[p] = s_row[j];
        for (int b = 0; b < nb; ++b) seg_a[(size_t)p * nb + b] = s_a[j][b];
      }
      base += __popc(bal);
    }
    if (lane == 0) seg_cnt[blockIdx.x] = base;
  }
}

// ----------------------------------------------------------------------------
// Sparse-head Q/K/V projection + KV append (eq. (2); the itpub KV-cache figure).
// Slot s in [0, hc*3*dh): p = s / (3 dh) indexes head_idx, m = (s / dh) % 3
// picks q/k/v, c = s % dh the channel. q goes to the workspace (fp32); k and v
// are rounded to the cache dtype and written at slot `pos`.
// ----------------------------------------------------------------------------
template <typename T, typename KT, int NB, int RPW, int U>
__global__ void __launch_bounds__(GEMV_THREADS)
    qkv_kernel(const T* __restrict__ Wqkv, int d, int h, int dh, const float* __restrict__ X, int nb,
               const float* __restrict__ bqkv, const int32_t* __restrict__ head_idx,
               const int32_t* __restrict__ head_count, int kh_max, float* __restrict__ q, KT* __restrict__ Kc,
               KT* __restrict__ Vc, int cap, int pos, int* __restrict__ status, const float* __restrict__ wscale) {
  griddep_launch();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int hc = *head_count;
  if (hc > kh_max || hc < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(status, 1);
    hc = hc < 0 ? 0 : kh_max;
  }
  const int per = 3 * dh;
  const int nslot = hc * per;
  const int slot0 = (blockIdx.x * GEMV_WARPS + warp) * RPW;
  const T* rowp[RPW];
  bool valid[RPW];
  int heads[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int slot = slot0 + r;
    int head = -1;
    if (slot < nslot) {
      head = head_idx[slot / per];
      if (head < 0 || head >= h) {
        if (lane == 0) raise_status(status, 2);
        head = -1;
      }
    }
    heads[r] = head;
    valid[r] = head >= 0;
    rowp[r] = Wqkv + ((size_t)(head >= 0 ? head : 0) * per + (slot % per)) * d;
  }
  float acc[RPW][NB];
  warp_rows_dot<T, NB, RPW, U>(rowp, valid, d, X, d, nb, acc);
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (lane == ((r * NB + b) & 31) && valid[r] && b < nb) {
        const int slot = slot0 + r;
        const int p = slot / per, rem = slot % per, m = rem / dh, c = rem % dh;
        float v = acc[r][b];
        if (wscale) v *= wscale[(size_t)heads[r] * per + rem];
        if (bqkv) v += bqkv[(size_t)heads[r] * per + rem];
        if (m == 0) {
          q[((size_t)b * kh_max + p) * dh + c] = v;
        } else {
          KT* cache = (m == 1) ? Kc : Vc;
          cache[(((size_t)b * h + heads[r]) * cap + pos) * dh + c] = WT<KT>::store_cvt(v);
        }
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Exact KV maintenance: k and v at slot `pos` for the heads NOT in the
// selected set (the KV-cache figure (b): every step appends the new token's
// key and value for every head), so later steps attend over true keys and
// values. Every CTA rebuilds the ascending list of unselected heads from
// head_idx in shared memory. Slot s in [0, (h - hc) * 2 dh): p = s / (2 dh)
// indexes that list, m = 1 + (s / dh) % 2 picks k / v, c = s % dh.
// ----------------------------------------------------------------------------
constexpr int KV_REST_MAX_H = 1024;

template <typename T, int NB, int RPW, int U>
__global__ void __launch_bounds__(GEMV_THREADS)
    kv_rest_kernel(const T* __restrict__ Wqkv, int d, int h, int dh, const float* __restrict__ X, int nb,
                   const float* __restrict__ bqkv, const int32_t* __restrict__ head_idx,
                   const int32_t* __restrict__ head_count, int kh_max, T* __restrict__ Kc, T* __restrict__ Vc, int cap,
                   int pos, int* __restrict__ status) {
  __shared__ int s_rest[KV_REST_MAX_H];
  __shared__ unsigned char s_sel[KV_REST_MAX_H];
  __shared__ int s_nrest;
  griddep_launch();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int hc = *head_count;
  if (hc > kh_max || hc < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(status, 1);
    hc = hc < 0 ? 0 : kh_max;
  }
  for (int i = threadIdx.x; i < h; i += GEMV_THREADS) s_sel[i] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < hc; p += GEMV_THREADS) {
    const int head = head_idx[p];
    if (head >= 0 && head < h) s_sel[head] = 1;
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0;
    for (int i0 = 0; i0 < h; i0 += 32) {
      const int i = i0 + lane;
      const bool rest = i < h && !s_sel[i];
      const unsigned bal = __ballot_sync(0xffffffffu, rest);
      if (rest) s_rest[base + __popc(bal & ((1u << lane) - 1u))] = i;
      base += __popc(bal);
    }
    if (lane == 0) s_nrest = base;
  }
  __syncthreads();
  const int per = 2 * dh;
  const int nslot = s_nrest * per;
  const int slot0 = (blockIdx.x * GEMV_WARPS + warp) * RPW;
  if (slot0 >= nslot) return;
  const T* rowp[RPW];
  bool valid[RPW];
  int heads[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int slot = slot0 + r;
    valid[r] = slot < nslot;
    heads[r] = valid[r] ? s_rest[slot / per] : 0;
    rowp[r] = Wqkv + ((size_t)heads[r] * 3 * dh + dh + (valid[r] ? slot % per : 0)) * d;
  }
  float acc[RPW][NB];
  warp_rows_dot<T, NB, RPW, U>(rowp, valid, d, X, d, nb, acc);
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (lane == ((r * NB + b) & 31) && valid[r] && b < nb) {
        const int rem = (slot0 + r) % per, c = rem % dh;
        float v = acc[r][b];
        if (bqkv) v += bqkv[(size_t)heads[r] * 3 * dh + dh + rem];
        T* cache = rem < dh ? Kc : Vc;
        cache[(((size_t)b * h + heads[r]) * cap + pos) * dh + c] = WT<T>::store_cvt(v);
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Selection: per-row top-k by radix select on order-preserving keys, or a
// strict threshold; the union over rows, compacted to ascending indices.
// One CTA per score row writes its selection bitmap; the last CTA to finish
// (ticket) ORs the bitmaps and writes idx / count, then resets the ticket.
//
// The k-th largest key is found in three digit passes (11, 11, 10 bits): a
// shared-memory histogram of the digits of the keys that still match the
// prefix, then a block-wide suffix scan over the bins. The flag and
// compaction passes are warp-cooperative (one ballot per 32 indices), so the
// result comes out in index order: keys above the threshold, then the
// lowest-index copies of the threshold key.
// ----------------------------------------------------------------------------
constexpr int SEL_THREADS = 1024;
constexpr int SEL_WARPS = SEL_THREADS / 32;
constexpr int SEL_SMEM_KEYS = 49152;  // rows up to this length keep keys in shared memory
constexpr int SEL_BINS = 2048;

// Order-preserving map float -> uint32: larger float, larger key. -0.0 maps
// like +0.0; every NaN maps to 0, below -inf (0x007fffff).
__device__ __forceinline__ uint32_t ord_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (s != s) return 0u;
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <bool KEYS_IN_SMEM>
__device__ __forceinline__ uint32_t sel_key(const uint32_t* s_keys, const float* row, int i) {
  return KEYS_IN_SMEM ? s_keys[i] : ord_key(__ldcg(row + i));
}

template <bool KEYS_IN_SMEM>
__global__ void __launch_bounds__(SEL_THREADS)
    select_kernel(const float* __restrict__ scores, int n, int nrows, int k, float tau, int mode,
                  uint32_t* __restrict__ bitmaps, unsigned* __restrict__ ticket, int32_t* __restrict__ idx,
                  int32_t* __restrict__ count) {
  extern __shared__ uint32_t s_keys[];
  __shared__ unsigned hist[SEL_BINS];
  __shared__ unsigned sc[SEL_WARPS + 1];
  __shared__ unsigned s_digit, s_kk, s_last;
  griddep_launch();
  griddep_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x;
  const float* row = scores + (size_t)b * n;
  const int nw = (n + 31) >> 5;
  uint32_t* bm = bitmaps + (size_t)b * nw;
  const int wpw = (nw + SEL_WARPS - 1) / SEL_WARPS;  // bitmap words per warp
  const int w0 = warp * wpw, w1 = min(nw, w0 + wpw);

  if (mode == 1 || k >= n || k <= 0) {
    // threshold s > tau (NaN fails), or all / none
    for (int w = w0; w < w1; ++w) {
      const int i = w * 32 + lane;
      bool sel;
      if (mode == 1) sel = i < n && row[i] > tau;
      else sel = i < n && k > 0;
      const unsigned word = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) bm[w] = word;
    }
  } else {
    if (KEYS_IN_SMEM) {
      for (int i = tid; i < n; i += SEL_THREADS) s_keys[i] = ord_key(row[i]);
    }
    uint32_t prefix = 0, mask = 0;
    unsigned kk = (unsigned)k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);  // digits: bits 31..21, 20..10, 9..0
      const unsigned dmask = pass == 2 ? 0x3ffu : 0x7ffu;
      for (int i = tid; i < SEL_BINS; i += SEL_THREADS) hist[i] = 0;
      __syncthreads();
      // keys of a warp that share a bin add once (scores crowd into few
      // top-digit bins, where per-key atomics would serialise)
      for (int i0 = 0; i0 < n; i0 += SEL_THREADS) {
        const int i = i0 + tid;
        const uint32_t key = i < n ? sel_key<KEYS_IN_SMEM>(s_keys, row, i) : 0u;
        const bool in = i < n && (key & mask) == prefix;
        const unsigned bin = in ? (key >> shift) & dmask : 0xffffffffu;
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (in && (__ffs(peers) - 1) == lane) atomicAdd(&hist[bin], (unsigned)__popc(peers));
      }
      __syncthreads();
      // thread t owns bins 2047-2t and 2046-2t (descending); an exclusive scan
      // in thread order counts the keys in higher bins
      const unsigned c0 = hist[SEL_BINS - 1 - 2 * tid], c1 = hist[SEL_BINS - 2 - 2 * tid];
      unsigned tot;
      const unsigned above = block_exclusive_scan<SEL_THREADS>(c0 + c1, sc, &tot);
      if (above < kk && kk <= above + c0 + c1) {
        if (kk <= above + c0) {
          s_digit = SEL_BINS - 1 - 2 * tid;
          s_kk = kk - above;
        } else {
          s_digit = SEL_BINS - 2 - 2 * tid;
          s_kk = kk - above - c0;
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= dmask << shift;
      kk = s_kk;
    }
    // prefix is the k-th largest key; kk of its copies are taken, lowest
    // indices first
    unsigned eq = 0;
    for (int w = w0; w < w1; ++w) {
      const int i = w * 32 + lane;
      const bool e = i < n && sel_key<KEYS_IN_SMEM>(s_keys, row, i) == prefix;
      eq += __popc(__ballot_sync(0xffffffffu, e));
    }
    if (lane == 0) sc[warp] = eq;
    __syncthreads();
    if (warp == 0) {
      const unsigned v = sc[lane];
      unsigned incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      sc[lane] = incl - v;
    }
    __syncthreads();
    unsigned rank = sc[warp];
    for (int w = w0; w < w1; ++w) {
      const int i = w * 32 + lane;
      uint32_t key = 0;
      bool valid = i < n;
      if (valid) key = sel_key<KEYS_IN_SMEM>(s_keys, row, i);
      const bool e = valid && key == prefix;
      const unsigned em = __ballot_sync(0xffffffffu, e);
      const unsigned r = rank + __popc(em & ((1u << lane) - 1u));
      const bool sel = valid && (key > prefix || (e && r < kk));
      const unsigned word = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) bm[w] = word;
      rank += __popc(em);
    }
  }
  // union over rows by the last CTA
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(ticket, 1u) == (unsigned)nrows - 1u);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // the union of the rows' bitmaps, every word loaded at once, kept in the
  // (now free) key buffer or, for long rows, re-read below
  uint32_t* s_u = s_keys;
  const bool u_in_smem = KEYS_IN_SMEM || nw <= 0;
  unsigned pc = 0;
  if (u_in_smem) {
    for (int w = tid; w < nw; w += SEL_THREADS) {
      uint32_t u = 0;
      for (int rr = 0; rr < nrows; ++rr) u |= __ldcg(bitmaps + (size_t)rr * nw + w);
      s_u[w] = u;
    }
    __syncthreads();
    for (int w = w0; w < w1; ++w) pc += __popc(s_u[w]);
  } else {
    for (int w = w0; w < w1; ++w) {
      uint32_t u = 0;
      for (int rr = lane; rr < nrows; rr += 32) u |= __ldcg(bitmaps + (size_t)rr * nw + w);
      pc += __popc(__reduce_or_sync(0xffffffffu, u));
    }
  }
  if (lane == 0) sc[warp] = pc;
  __syncthreads();
  if (warp == 0) {
    const unsigned v = sc[lane];
    unsigned incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    sc[lane] = incl - v;
    if (lane == 31) sc[SEL_WARPS] = incl;
  }
  __syncthreads();
  unsigned off = sc[warp];
  for (int w = w0; w < w1; ++w) {
    uint32_t u = 0;
    if (u_in_smem) {
      u = s_u[w];
    } else {
      for (int rr = lane; rr < nrows; rr += 32) u |= __ldcg(bitmaps + (size_t)rr * nw + w);
      u = __reduce_or_sync(0xffffffffu, u);
    }
    if ((u >> lane) & 1u) idx[off + __popc(u & ((1u << lane) - 1u))] = w * 32 + lane;
    off += __popc(u);
  }
  if (tid == 0) {
    *count = (int32_t)sc[SEL_WARPS];
    *ticket = 0u;
  }
}

// ----------------------------------------------------------------------------
// Split-K decode attention over the selected heads (eq. (2), D_i normalised,
// max-subtracted). CTA (s, p, b) handles keys [s*S, min(s*S+S, pos+1)) of
// head head_idx[p], batch row b: it stages its K and V tiles in shared memory
// with cp.async (all loads in flight at once), forms the scores, and writes
// the partial (m, l, acc[dh]). The last split to finish for (b, p) combines
// the partials into H[b][p][:].
// ----------------------------------------------------------------------------
constexpr int ATTN_THREADS = 128;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

template <typename KT, int DH, int S>
__global__ void __launch_bounds__(ATTN_THREADS)
    attn_split_kernel(const float* __restrict__ q, const KT* __restrict__ Kc, const KT* __restrict__ Vc, int h, int cap,
                      int pos, float scale, const int32_t* __restrict__ head_idx,
                      const int32_t* __restrict__ head_count, int kh_max, int nsplit, float* __restrict__ part,
                      unsigned* __restrict__ ctr, float* __restrict__ H, int* __restrict__ status) {
  constexpr int E = WT<KT>::E;        // elements per 16-byte vector
  constexpr int G = DH / E;           // lanes per key row
  constexpr int KPP = ATTN_THREADS / G;  // keys per pass
  __shared__ __align__(16) KT sK[S * DH];
  __shared__ __align__(16) KT sV[S * DH];
  __shared__ float sE[S];
  __shared__ float sRed[KPP * DH];
  __shared__ float red[ATTN_THREADS / 32];
  __shared__ unsigned s_last;
  griddep_launch();
  griddep_wait();
  const int s = blockIdx.x, p = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  int hc = *head_count;
  hc = hc < 0 ? 0 : (hc > kh_max ? kh_max : hc);
  if (p >= hc) return;
  const int head = head_idx[p];
  if (head < 0 || head >= h) {
    if (tid == 0 && s == 0) raise_status(status, 2);
    return;
  }
  const int t0 = s * S;
  const int nk = min(S, pos + 1 - t0);
  const size_t base = (((size_t)b * h + head) * cap + t0) * DH;
  {
    const int nvec = nk * DH / E;
    for (int v = tid; v < nvec; v += ATTN_THREADS) {
      cp_async16(sK + v * E, Kc + base + (size_t)v * E);
      cp_async16(sV + v * E, Vc + base + (size_t)v * E);
    }
  }
  const int g = tid % G, j = tid / G;
  float qv[E];
  {
    const float* qp = q + ((size_t)b * kh_max + p) * DH + g * E;
#pragma unroll
    for (int e = 0; e < E; ++e) qv[e] = qp[e] * scale;
  }
  cp_async_wait_all();
  __syncthreads();
  // scores; every thread runs the same trip count so the group shuffles
  // below always see all 32 lanes of the warp
  for (int tb = 0; tb < nk; tb += KPP) {
    const int t = tb + j;
    float dot = 0.f;
    if (t < nk) {
      float kf[E];
      WT<KT>::unpack(*reinterpret_cast<const uint4*>(sK + t * DH + g * E), kf);
#pragma unroll
      for (int e = 0; e < E; ++e) dot = fmaf(qv[e], kf[e], dot);
    }
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (g == 0 && t < nk) sE[t] = dot;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int t = tid; t < nk; t += ATTN_THREADS) m = fmaxf(m, sE[t]);
  m = block_max<ATTN_THREADS>(m, red);
  float l = 0.f;
  for (int t = tid; t < nk; t += ATTN_THREADS) {
    const float pe = __expf(sE[t] - m);
    sE[t] = pe;
    l += pe;
  }
  l = block_sum<ATTN_THREADS>(l, red);  // ends with a barrier: sE is final
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int t = j; t < nk; t += KPP) {
    float vf[E];
    WT<KT>::unpack(*reinterpret_cast<const uint4*>(sV + t * DH + g * E), vf);
    const float pe = sE[t];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(pe, vf[e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < E; ++e) sRed[j * DH + g * E + e] = acc[e];
  __syncthreads();
  float* pp = part + (((size_t)b * kh_max + p) * nsplit + s) * (DH + 2);
  for (int c = tid; c < DH; c += ATTN_THREADS) {
    float a = 0.f;
#pragma unroll
    for (int jj = 0; jj < KPP; ++jj) a += sRed[jj * DH + c];
    pp[2 + c] = a;
  }
  if (tid == 0) {
    pp[0] = m;
    pp[1] = l;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(ctr + (size_t)b * kh_max + p, 1u) == (unsigned)nsplit - 1u);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* p0 = part + ((size_t)b * kh_max + p) * nsplit * (DH + 2);
  float M = -INFINITY;
  for (int ss = 0; ss < nsplit; ++ss) M = fmaxf(M, __ldcg(p0 + (size_t)ss * (DH + 2)));
  float den = 0.f;
  for (int ss = 0; ss < nsplit; ++ss) {
    const float* ps = p0 + (size_t)ss * (DH + 2);
    den += __expf(__ldcg(ps) - M) * __ldcg(ps + 1);
  }
  for (int c = tid; c < DH; c += ATTN_THREADS) {
    float num = 0.f;
    for (int ss = 0; ss < nsplit; ++ss) {
      const float* ps = p0 + (size_t)ss * (DH + 2);
      num += __expf(__ldcg(ps) - M) * __ldcg(ps + 2 + c);
    }
    H[((size_t)b * kh_max + p) * DH + c] = num / den;
  }
  if (tid == 0) ctr[(size_t)b * kh_max + p] = 0u;
}

// ----------------------------------------------------------------------------
// Gather-axpy: out[b][:] += sum_p coef[p][b] * W[row(p)][:] over a device-sized
// list of rows. Grid (column tiles, G): CTA (x, y) owns columns
// [x*AX_THREADS*E, ...) and list positions [total*y/G, total*(y+1)/G). Rows are
// streamed with U 16-byte loads in flight per thread; the CTA's partial sums
// are added to out with vector float atomics. The CTA with y == 0 adds bias.
//
// Row sources: RowsMlp (compacted neurons from mlp_up_kernel's segments; eq.
// (1), second factor) and RowsHeads (rows c of W_i^O for i in S_A; eq. (2)).
// ----------------------------------------------------------------------------
constexpr int AX_THREADS = 128;
constexpr int AX_CHUNK = 256;
constexpr int AX_U = 8;

struct RowsMlp {
  const int32_t* seg_idx;
  const float* seg_a;
  const int32_t* seg_cnt;
  int nseg, SEG;
  const float* wscale = nullptr;  // per-row scale of int8 weights, or null
  // Builds the prefix sums of the segment counts in s_off[0..nseg]; returns the total.
  __device__ int prologue(int* s_off, unsigned* sc) const {
    unsigned run = 0;
    for (int base = 0; base < nseg; base += AX_THREADS) {
      const int i = base + threadIdx.x;
      const unsigned c = i < nseg ? (unsigned)seg_cnt[i] : 0u;
      unsigned tot;
      const unsigned ex = block_exclusive_scan<AX_THREADS>(c, sc, &tot);
      if (i < nseg) s_off[i] = (int)(run + ex);
      run += tot;
    }
    if (threadIdx.x == 0) s_off[nseg] = (int)run;
    __syncthreads();
    return (int)run;
  }
  __device__ int row(int pidx, const int* s_off) const {
    int lo = 0, hi = nseg - 1;  // last segment with s_off[seg] <= pidx
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= pidx) lo = mid;
      else hi = mid - 1;
    }
    return lo * SEG + (pidx - s_off[lo]);  // slot
  }
  __device__ int row_of_slot(int slot) const { return seg_idx[slot]; }
  __device__ float coef(int slot, int b, int nb) const { return seg_a[(size_t)slot * nb + b]; }
};

struct RowsHeads {
  const int32_t* head_idx;
  const int32_t* head_count;
  const float* Hbuf;  // [B][kh_max][dh]
  int kh_max, dh, h;
  const float* wscale = nullptr;  // per-row scale of int8 weights, or null
  __device__ int prologue(int*, unsigned*) const {
    int hc = *head_count;
    hc = hc < 0 ? 0 : (hc > kh_max ? kh_max : hc);
    return hc * dh;
  }
  __device__ int row(int pidx, const int*) const { return pidx; }
  __device__ int row_of_slot(int slot) const {
    const int head = head_idx[slot / dh];
    return (head < 0 || head >= h) ? -1 : head * dh + slot % dh;
  }
  __device__ float coef(int slot, int b, int) const {
    return Hbuf[((size_t)b * kh_max + slot / dh) * dh + slot % dh];
  }
};

template <typename T, int NB, class Src>
__global__ void __launch_bounds__(AX_THREADS)
    axpy_rows_kernel(const T* __restrict__ W, int d, int nrows_w, Src src, const float* __restrict__ bias,
                     float* __restrict__ out, int nb, int G, int* __restrict__ status) {
  constexpr int E = WT<T>::E;
  extern __shared__ int s_off[];
  __shared__ int s_rows[AX_CHUNK];
  __shared__ float s_coef[AX_CHUNK][NB];
  __shared__ unsigned sc[AX_THREADS / 32 + 1];
  griddep_launch();
  griddep_wait();
  const int tid = threadIdx.x;
  const int total = src.prologue(s_off, sc);
  const int p0 = (int)(((long long)total * blockIdx.y) / G);
  const int p1 = (int)(((long long)total * (blockIdx.y + 1)) / G);
  const int col = (blockIdx.x * AX_THREADS + tid) * E;
  const bool colok = col < d;
  float acc[NB][E];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int e = 0; e < E; ++e) acc[b][e] = (bias && blockIdx.y == 0 && colok && b < nb) ? bias[col + e] : 0.f;
  for (int c0 = p0; c0 < p1; c0 += AX_CHUNK) {
    const int n = min(AX_CHUNK, p1 - c0);
    for (int i = tid; i < n; i += AX_THREADS) {
      const int slot = src.row(c0 + i, s_off);
      int row = src.row_of_slot(slot);
      if (row < 0 || row >= nrows_w) {
        raise_status(status, 2);
        row = -1;
      }
      s_rows[i] = row;
      const float sc = (row >= 0 && src.wscale) ? src.wscale[row] : 1.f;
#pragma unroll
      for (int b = 0; b < NB; ++b) s_coef[i][b] = (row >= 0 && b < nb) ? src.coef(slot, b, nb) * sc : 0.f;
    }
    __syncthreads();
    for (int i0 = 0; i0 < n; i0 += AX_U) {
      uint4 w[AX_U];
#pragma unroll
      for (int u = 0; u < AX_U; ++u) {
        const int i = i0 + u;
        const int row = (i < n) ? s_rows[i] : -1;
        w[u] = (colok && row >= 0) ? ld_stream(W + (size_t)row * d + col) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < AX_U; ++u) {
        const int i = i0 + u;
        if (i < n) {
          float wf[E];
          WT<T>::unpack(w[u], wf);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const float cb = s_coef[i][b];
#pragma unroll
            for (int e = 0; e < E; ++e) acc[b][e] = fmaf(cb, wf[e], acc[b][e]);
          }
        }
      }
    }
    __syncthreads();
  }
  if (colok && (p1 > p0 || (bias && blockIdx.y == 0))) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < nb) {
#pragma unroll
        for (int e4 = 0; e4 < E / 4; ++e4) {
          float4 v = make_float4(acc[b][4 * e4], acc[b][4 * e4 + 1], acc[b][4 * e4 + 2], acc[b][4 * e4 + 3]);
          red_add4(out + (size_t)b * d + col + 4 * e4, v);
        }
      }
    }
  }
}

// Asks the bulk-copy engine to bring [p, p + bytes) into L2; no data moves
// through the SM.
constexpr uint32_t PF_CHUNK = 16384;  // bytes per prefetch request

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

}  // namespace dv
