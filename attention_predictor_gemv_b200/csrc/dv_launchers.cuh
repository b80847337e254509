// Kernel launchers: grid shapes and template dispatch. The function
// templates named at the end are instantiated once, each in its own
// translation unit (dv_inst_*.cu), so the kernels compile in parallel.
#pragma once

#include "../../include/dejavu.h"
#include "dv_stream.cuh"
#include "dv_launch.cuh"

namespace dv {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------------------
// Launchers (arguments already checked)
// ---------------------------------------------------------------------------

template <typename T, int NB>
cudaError_t run_dense_gemv_nb(const void* W, int nrows, int K, const float* X, int ldx, int nb, const float* bias,
                              float* out, int ldo, cudaStream_t st) {
  const T* w = static_cast<const T*>(W);
  const int rpw = rpw_for(K, WT<T>::E);
  const int rows_per_cta = GEMV_WARPS * rpw;
  dim3 grid((nrows + rows_per_cta - 1) / rows_per_cta);
  switch (rpw) {
    case 1: return launch(dense_gemv_kernel<T, NB, 1, 8>, grid, GEMV_THREADS, 0, st, w, nrows, K, X, ldx, nb, bias, out, ldo);
    case 2: return launch(dense_gemv_kernel<T, NB, 2, 4>, grid, GEMV_THREADS, 0, st, w, nrows, K, X, ldx, nb, bias, out, ldo);
    case 4: return launch(dense_gemv_kernel<T, NB, 4, 2>, grid, GEMV_THREADS, 0, st, w, nrows, K, X, ldx, nb, bias, out, ldo);
    default: return launch(dense_gemv_kernel<T, NB, 8, 1>, grid, GEMV_THREADS, 0, st, w, nrows, K, X, ldx, nb, bias, out, ldo);
  }
}

template <typename T>
cudaError_t run_dense_gemv(const void* W, int nrows, int K, const float* X, int ldx, int nb, const float* bias,
                           float* out, int ldo, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_dense_gemv_nb<T, 1>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
    case 2: return run_dense_gemv_nb<T, 2>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
    case 4: return run_dense_gemv_nb<T, 4>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
    case 8: return run_dense_gemv_nb<T, 8>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
    default: return run_dense_gemv_nb<T, 16>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
  }
}

cudaError_t run_gemv(dv_dtype dt, const void* W, int nrows, int K, const float* X, int ldx, int nb, const float* bias,
                     float* out, int ldo, cudaStream_t st);

cudaError_t run_select(const float* scores, int nrows, int n, int k, float tau, int mode, uint32_t* bm,
                       unsigned* ticket, int32_t* idx, int32_t* count, cudaStream_t st);

template <typename T, int NB>
cudaError_t run_mlp_up_nb(const void* W1t, int d, int N, const float* y, int nb, const float* b1, const int32_t* idx,
                          const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a, int32_t* seg_cnt,
                          int* status, int nseg, int act, cudaStream_t st) {
  const T* w = static_cast<const T*>(W1t);
  dim3 grid(nseg > 0 ? nseg : 1);
  switch (rpw_for(d, WT<T>::E)) {
    case 1: return launch(mlp_up_kernel<T, NB, 1, 8>, grid, GEMV_THREADS, 0, st, w, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, act, (const float*)nullptr);
    case 2: return launch(mlp_up_kernel<T, NB, 2, 4>, grid, GEMV_THREADS, 0, st, w, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, act, (const float*)nullptr);
    case 4: return launch(mlp_up_kernel<T, NB, 4, 2>, grid, GEMV_THREADS, 0, st, w, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, act, (const float*)nullptr);
    default: return launch(mlp_up_kernel<T, NB, 8, 1>, grid, GEMV_THREADS, 0, st, w, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, act, (const float*)nullptr);
  }
}

template <typename T, int NB, class Src>
cudaError_t run_axpy_st(const void* W, int d, int nrows_w, Src src, const float* bias, float* out, int nb, int k_max,
                        size_t smem, int* status, cudaStream_t st) {
  constexpr int E = WT<T>::E;
  const int tiles = (d + AX_THREADS * E - 1) / (AX_THREADS * E);
  int G = (2 * sm_count() + tiles - 1) / tiles;
  const int gmax = (k_max + 3) / 4;
  if (G > gmax) G = gmax;
  if (G < 1) G = 1;
  cudaError_t e = allow_smem(axpy_rows_kernel<T, NB, Src>, smem);
  if (e != cudaSuccess) return e;
  return launch(axpy_rows_kernel<T, NB, Src>, dim3(tiles, G), AX_THREADS, smem, st, static_cast<const T*>(W), d,
                nrows_w, src, bias, out, nb, G, status);
}

template <typename T, class Src>
cudaError_t run_axpy(const void* W, int d, int nrows_w, Src src, const float* bias, float* out, int nb, int k_max,
                     size_t smem, int* status, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_axpy_st<T, 1>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    case 2: return run_axpy_st<T, 2>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    case 4: return run_axpy_st<T, 4>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    case 8: return run_axpy_st<T, 8>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    default: return run_axpy_st<T, 16>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
  }
}

template <typename T>
cudaError_t run_mlp_up(const void* W1t, int d, int N, const float* y, int nb, const float* b1, const int32_t* idx,
                       const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a, int32_t* seg_cnt, int* status,
                       int nseg, int act, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_mlp_up_nb<T, 1>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st);
    case 2: return run_mlp_up_nb<T, 2>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st);
    case 4: return run_mlp_up_nb<T, 4>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st);
    case 8: return run_mlp_up_nb<T, 8>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st);
    default: return run_mlp_up_nb<T, 16>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st);
  }
}

template <typename T, int NB>
cudaError_t run_qkv_nb(const void* Wqkv, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                       const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, void* Kc, void* Vc,
                       int cap, int pos, int* status, cudaStream_t st) {
  const T* w = static_cast<const T*>(Wqkv);
  const int rpw = rpw_for(d, WT<T>::E);
  const int slots = kh_max * 3 * dh;
  const int per_cta = GEMV_WARPS * rpw;
  dim3 grid((slots + per_cta - 1) / per_cta > 0 ? (slots + per_cta - 1) / per_cta : 1);
  T* K = static_cast<T*>(Kc);
  T* V = static_cast<T*>(Vc);
  switch (rpw) {
    case 1: return launch(qkv_kernel<T, T, NB, 1, 8>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, (const float*)nullptr);
    case 2: return launch(qkv_kernel<T, T, NB, 2, 4>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, (const float*)nullptr);
    case 4: return launch(qkv_kernel<T, T, NB, 4, 2>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, (const float*)nullptr);
    default: return launch(qkv_kernel<T, T, NB, 8, 1>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, (const float*)nullptr);
  }
}

template <typename T>
cudaError_t run_qkv(const void* Wqkv, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                    const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, void* Kc, void* Vc,
                    int cap, int pos, int* status, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_qkv_nb<T, 1>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
    case 2: return run_qkv_nb<T, 2>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
    case 4: return run_qkv_nb<T, 4>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
    case 8: return run_qkv_nb<T, 8>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
    default: return run_qkv_nb<T, 16>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos, status, st);
  }
}

template <typename T, int NB>
cudaError_t run_kv_rest_nb(const void* Wqkv, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                           const int32_t* head_idx, const int32_t* head_count, int kh_max, void* Kc, void* Vc, int cap,
                           int pos, int* status, cudaStream_t st) {
  const T* w = static_cast<const T*>(Wqkv);
  const int rpw = rpw_for(d, WT<T>::E);
  const int per_cta = GEMV_WARPS * rpw;
  const int slots = h * 2 * dh;  // every head unselected, at most
  dim3 grid((slots + per_cta - 1) / per_cta > 0 ? (slots + per_cta - 1) / per_cta : 1);
  T* K = static_cast<T*>(Kc);
  T* V = static_cast<T*>(Vc);
  switch (rpw) {
    case 1: return launch(kv_rest_kernel<T, NB, 1, 8>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, K, V, cap, pos, status);
    case 2: return launch(kv_rest_kernel<T, NB, 2, 4>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, K, V, cap, pos, status);
    case 4: return launch(kv_rest_kernel<T, NB, 4, 2>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, K, V, cap, pos, status);
    default: return launch(kv_rest_kernel<T, NB, 8, 1>, grid, GEMV_THREADS, 0, st, w, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, K, V, cap, pos, status);
  }
}

template <typename T>
cudaError_t run_kv_rest(const void* Wqkv, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                        const int32_t* head_idx, const int32_t* head_count, int kh_max, void* Kc, void* Vc, int cap,
                        int pos, int* status, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_kv_rest_nb<T, 1>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, Kc, Vc, cap, pos, status, st);
    case 2: return run_kv_rest_nb<T, 2>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, Kc, Vc, cap, pos, status, st);
    case 4: return run_kv_rest_nb<T, 4>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, Kc, Vc, cap, pos, status, st);
    case 8: return run_kv_rest_nb<T, 8>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, Kc, Vc, cap, pos, status, st);
    default: return run_kv_rest_nb<T, 16>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, Kc, Vc, cap, pos, status, st);
  }
}

// Keys per split: the largest of 64 / 32 that still gives >= 2 CTAs per SM.
inline int attn_split_len(int B, int kh_max, int pos) {
  const int want = 2 * sm_count();
  if ((long long)B * kh_max * ((pos + 1 + 63) / 64) >= want) return 64;
  return 32;
}

template <typename KT, int DH>
cudaError_t run_attn_dh(const float* q, const void* Kc, const void* Vc, int B, int h, int cap, int pos, float scale,
                        const int32_t* head_idx, const int32_t* head_count, int kh_max, float* part, unsigned* ctr,
                        float* H, int* status, cudaStream_t st) {
  const int S = (sizeof(KT) * DH * 64 * 2 <= 32768) ? attn_split_len(B, kh_max, pos) : 32;
  const int nsplit = (pos + 1 + S - 1) / S;
  dim3 grid(nsplit, kh_max, B);
  const KT* K = static_cast<const KT*>(Kc);
  const KT* V = static_cast<const KT*>(Vc);
  if constexpr (sizeof(KT) * DH * 64 * 2 <= 32768) {  // K and V tiles in static shared memory
    if (S == 64)
      return launch(attn_split_kernel<KT, DH, 64>, grid, ATTN_THREADS, 0, st, q, K, V, h, cap, pos, scale, head_idx,
                    head_count, kh_max, nsplit, part, ctr, H, status);
  }
  return launch(attn_split_kernel<KT, DH, 32>, grid, ATTN_THREADS, 0, st, q, K, V, h, cap, pos, scale, head_idx,
                head_count, kh_max, nsplit, part, ctr, H, status);
}

template <typename KT>
cudaError_t run_attn(int dh, const float* q, const void* Kc, const void* Vc, int B, int h, int cap, int pos,
                     float scale, const int32_t* head_idx, const int32_t* head_count, int kh_max, float* part,
                     unsigned* ctr, float* H, int* status, cudaStream_t st) {
  if (dh == 64)
    return run_attn_dh<KT, 64>(q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, part, ctr, H, status, st);
  return run_attn_dh<KT, 128>(q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, part, ctr, H, status, st);
}


constexpr int ATTN_CS = 8;  // CTAs per cluster (per selected head) in attn_out_kernel

inline int attn_out_S(int pos, int cs = ATTN_CS) { return (pos + 1 + cs - 1) / cs; }
// K/V tiles of S keys, the cluster's partials (m, l, acc[dh]) and q of nb rows.
inline size_t attn_out_smem(int S, int dh, int kvbytes, int nb, int cs = ATTN_CS) {
  return 2ull * S * dh * kvbytes + 4ull * nb * cs * (dh + 2) + 4ull * nb * dh;
}
// CTAs per cluster (per selected head) of the attention-only form: 8 at
// batch 1, 16 (a non-portable cluster size, half the keys per CTA) at batch
// 2, where each CTA holds two rows' K/V tiles (measured at the OPT-175B
// shape: 249 against 259 us per layer at batch 2, 119 against 118 at batch
// 1). DV_ATTN_CS=8 or 16 overrides.
inline int attn_h_cs(int nb) {
  static const int env = [] {
    const char* e = std::getenv("DV_ATTN_CS");
    return !e ? 0 : (e[0] == '1' && e[1] == '6' ? 16 : 8);
  }();
  return env ? env : (nb >= 2 ? 16 : 8);
}
constexpr size_t ATTN_SMEM_MAX = 204 * 1024;  // dynamic part; the static part stays below 21 KB

// W^O vectors per thread when a CTA's W^O slice (dh rows of d / ATTN_CS
// columns) fits in registers: dh / (256 / column vectors); 0 streams it.
inline int attn_out_wv(int d, int dh, int E, int nb) {
  const int ncg = d / ATTN_CS / E;
  if (nb > 4 || ncg < 8 || ncg > 256 || 256 % ncg != 0) return 0;
  const int rg = 256 / ncg;
  if (dh % rg != 0) return 0;
  const int wv = dh / rg;
  return (wv == 8 || wv == 16) ? wv : 0;
}

template <typename K, typename A>
cudaError_t launch_fused(K kern, dim3 grid, size_t smem, cudaStream_t st, const A& a) {
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  return launch_main(kern, grid, FUSED_THREADS, smem, st, a);
}

template <typename T, int NB>
cudaError_t run_attn_in_nb(const AttnInArgs& a, cudaStream_t st) {
  const int rpw = rpw_for(a.d, WT<T>::E);
  const int slots = a.kh_max * 3 * a.dh, per = FUSED_WARPS * rpw;
  const dim3 grid(slots > 0 ? (slots + per - 1) / per : 1);
  const size_t smem = 4ull * a.nb * a.d;
  switch (rpw) {
    case 1: return launch_fused(attn_in_kernel<T, NB, 1, 8>, grid, smem, st, a);
    case 2: return launch_fused(attn_in_kernel<T, NB, 2, 4>, grid, smem, st, a);
    case 4: return launch_fused(attn_in_kernel<T, NB, 4, 2>, grid, smem, st, a);
    default: return launch_fused(attn_in_kernel<T, NB, 8, 1>, grid, smem, st, a);
  }
}

template <typename T>
cudaError_t run_attn_in(const AttnInArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_attn_in_nb<T, 1>(a, st);
    case 2: return run_attn_in_nb<T, 2>(a, st);
    case 4: return run_attn_in_nb<T, 4>(a, st);
    case 8: return run_attn_in_nb<T, 8>(a, st);
    default: return run_attn_in_nb<T, 16>(a, st);
  }
}

template <typename KT, int DH, int NB, int WV, int CS = ATTN_CS, int NT = FUSED_THREADS>
cudaError_t run_attn_out_nbw(AttnOutArgs a, cudaStream_t st) {
  // K/V tiles of every batch row at once when they fit, else row by row; and
  // row by row too when the grid is larger than the SMs and holding every
  // row would leave one CTA per SM (a second wave costs more than staging
  // the rows one after the other)
  a.S = attn_out_S(a.pos, CS);
  const size_t tiles = 2ull * a.S * DH * sizeof(KT);
  const size_t all_rows = attn_out_smem(a.S, DH, sizeof(KT), a.nb, CS) + (a.nb - 1) * tiles;
  const bool waves = (long long)CS * (a.kh_max > 0 ? a.kh_max : 1) > sm_count();
  a.stage_rows = (all_rows <= ATTN_SMEM_MAX && !(waves && all_rows > 110 * 1024)) ? a.nb : 1;
  const size_t smem = attn_out_smem(a.S, DH, sizeof(KT), a.nb, CS) + (a.stage_rows - 1) * tiles;
  auto kern = attn_out_kernel<KT, DH, CS, NB, WV, NT>;
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  if constexpr (CS > 8) {
    static const cudaError_t np = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (np != cudaSuccess) return np;
  }
  return launch_cluster(kern, dim3(CS, a.kh_max > 0 ? a.kh_max : 1), NT, smem, st, CS, a);
}

// Whole-row W^O (long rows, bf16, batch 1-2): 16-byte vectors per thread
// per row, 4-6 (d = 8192-12288); 0 when the path does not apply.
inline int attn_out_whole_rows(int d, int E, int kvbytes, int nb) {
  if (nb > 2 || kvbytes != 2 || d % (256 * E) != 0) return 0;
  const int nvo = d / (256 * E);
  return (nvo >= 4 && nvo <= 6) ? nvo : 0;
}

template <typename KT, int DH, int NB>
cudaError_t run_attn_out_nb(const AttnOutArgs& a, cudaStream_t st) {
  if constexpr (NB <= 2 && sizeof(KT) == 2) {
    if (a.H_out) {  // W^O in wo_stream_kernel
      if (attn_h_cs(a.nb) == 16) return run_attn_out_nbw<KT, DH, NB, ATTN_H_ONLY, 16>(a, st);
      // batch 1: 512 threads per CTA (16 warps over the CTA's keys: the
      // attention is bound by issue latency at 8 warps per SM); measured at
      // the OPT-175B shape 109.6-110.0 against 111.2 us per layer-step.
      // DV_ATTN_NT=256 or 512 overrides.
      static const int nt_env = [] {
        const char* e = std::getenv("DV_ATTN_NT");
        return !e ? 0 : (e[0] == '5' ? 512 : 256);
      }();
      const int nt = nt_env ? nt_env : (a.nb == 1 ? 512 : 256);
      if (nt == 512) return run_attn_out_nbw<KT, DH, NB, ATTN_H_ONLY, ATTN_CS, 512>(a, st);
      return run_attn_out_nbw<KT, DH, NB, ATTN_H_ONLY>(a, st);
    }
    switch (attn_out_whole_rows(a.d, WT<KT>::E, sizeof(KT), a.nb)) {
      case 4: return run_attn_out_nbw<KT, DH, NB, -4>(a, st);
      case 5: return run_attn_out_nbw<KT, DH, NB, -5>(a, st);
      case 6: return run_attn_out_nbw<KT, DH, NB, -6>(a, st);
      default: break;
    }
  }
  if constexpr (NB <= 4) {
    switch (attn_out_wv(a.d, DH, WT<KT>::E, a.nb)) {
      case 8: return run_attn_out_nbw<KT, DH, NB, 8>(a, st);
      case 16: return run_attn_out_nbw<KT, DH, NB, 16>(a, st);
      default: break;
    }
  }
  return run_attn_out_nbw<KT, DH, NB, 0>(a, st);
}

template <typename KT, int DH>
cudaError_t run_attn_out_dh(const AttnOutArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_attn_out_nb<KT, DH, 1>(a, st);
    case 2: return run_attn_out_nb<KT, DH, 2>(a, st);
    case 4: return run_attn_out_nb<KT, DH, 4>(a, st);
    case 8: return run_attn_out_nb<KT, DH, 8>(a, st);
    default: return run_attn_out_nb<KT, DH, 16>(a, st);
  }
}

template <typename KT>
cudaError_t run_attn_out(const AttnOutArgs& a, cudaStream_t st) {
  return a.dh == 64 ? run_attn_out_dh<KT, 64>(a, st) : run_attn_out_dh<KT, 128>(a, st);
}

inline int mlp_block_grid(int k_max) {
  const int g = (k_max + 7) / 8;
  return g < 1 ? 1 : (g > sm_count() ? sm_count() : g);
}

template <typename T, int NB>
cudaError_t run_mlp_block_nb(const MlpBlockArgs& a, cudaStream_t st) {
  const int rpw = rpw_for(a.d, WT<T>::E);
  const dim3 grid(a.G);
  const size_t smem = 4ull * a.nb * a.d;
  switch (rpw) {
    case 1: return launch_fused(mlp_block_kernel<T, NB, 1, 8>, grid, smem, st, a);
    case 2: return launch_fused(mlp_block_kernel<T, NB, 2, 4>, grid, smem, st, a);
    case 4: return launch_fused(mlp_block_kernel<T, NB, 4, 2>, grid, smem, st, a);
    default: return launch_fused(mlp_block_kernel<T, NB, 8, 1>, grid, smem, st, a);
  }
}

template <typename T>
cudaError_t run_mlp_block(const MlpBlockArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_mlp_block_nb<T, 1>(a, st);
    case 2: return run_mlp_block_nb<T, 2>(a, st);
    case 4: return run_mlp_block_nb<T, 4>(a, st);
    case 8: return run_mlp_block_nb<T, 8>(a, st);
    default: return run_mlp_block_nb<T, 16>(a, st);
  }
}

template <typename T, int NB>
cudaError_t run_predict_a_nb(const PredictAArgs& a, cudaStream_t st) {
  const int rows = (a.PA ? a.h : 0) + (a.At ? a.r : 0);
  const int rpw = rpw_for(a.d, WT<T>::E), per = FUSED_WARPS * rpw;
  const dim3 grid(rows > 0 ? (rows + per - 1) / per : 1);
  switch (rpw) {
    case 1: return launch(predict_a_kernel<T, NB, 1, 8>, grid, FUSED_THREADS, 0, st, a);
    case 2: return launch(predict_a_kernel<T, NB, 2, 4>, grid, FUSED_THREADS, 0, st, a);
    case 4: return launch(predict_a_kernel<T, NB, 4, 2>, grid, FUSED_THREADS, 0, st, a);
    default: return launch(predict_a_kernel<T, NB, 8, 1>, grid, FUSED_THREADS, 0, st, a);
  }
}

template <typename T>
cudaError_t run_predict_a(const PredictAArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_predict_a_nb<T, 1>(a, st);
    case 2: return run_predict_a_nb<T, 2>(a, st);
    case 4: return run_predict_a_nb<T, 4>(a, st);
    case 8: return run_predict_a_nb<T, 8>(a, st);
    default: return run_predict_a_nb<T, 16>(a, st);
  }
}

template <typename T, int NB>
cudaError_t run_predict_b_nb(const PredictBArgs& a, cudaStream_t st) {
  const int rpw = rpw_for(a.r, WT<T>::E), per = FUSED_WARPS * rpw;
  const int groups = (a.N + per - 1) / per;
  if constexpr (NB <= 2) {
    // one row per warp and four CTAs per SM (registers capped at 64): twice
    // the warps of the two-rows-per-warp form, which the memory pipe needs
    // to keep enough 16-byte loads in flight for rows of 4 vectors per lane
    if (a.r / WT<T>::E == 128) {
      const int g1 = (a.N + FUSED_WARPS - 1) / FUSED_WARPS, cap = pb_ctas();
      const dim3 grid1(g1 < cap ? g1 : cap);
      return launch(predict_b_kernel<T, NB, 1, 4, 4>, grid1, FUSED_THREADS, 0, st, a);
    }
  }
  const dim3 grid(groups < 2 * sm_count() ? groups : 2 * sm_count());  // persistent: two CTAs per SM
  switch (rpw) {
    case 1: return launch(predict_b_kernel<T, NB, 1, 8>, grid, FUSED_THREADS, 0, st, a);
    case 2: return launch(predict_b_kernel<T, NB, 2, 4>, grid, FUSED_THREADS, 0, st, a);
    case 4: return launch(predict_b_kernel<T, NB, 4, 2>, grid, FUSED_THREADS, 0, st, a);
    default: return launch(predict_b_kernel<T, NB, 8, 1>, grid, FUSED_THREADS, 0, st, a);
  }
}

template <typename T>
cudaError_t run_predict_b(const PredictBArgs& a, cudaStream_t st) {
  switch (nb_bucket(a.nb)) {
    case 1: return run_predict_b_nb<T, 1>(a, st);
    case 2: return run_predict_b_nb<T, 2>(a, st);
    case 4: return run_predict_b_nb<T, 4>(a, st);
    case 8: return run_predict_b_nb<T, 8>(a, st);
    default: return run_predict_b_nb<T, 16>(a, st);
  }
}

// ---------------------------------------------------------------------------
// Column-owner kernels (dv_colowner.cuh) for batch 1-4
// ---------------------------------------------------------------------------

inline int co_nv(int d, int E) { return (d + CO_THREADS * E - 1) / (CO_THREADS * E); }
// Rows per group: 8 or more 16-byte loads in flight per thread. The MLP
// kernel also holds the W2 rows and its output slice, so it keeps fewer.
inline int co_r(int nv) { return nv == 1 ? 8 : nv == 2 ? 4 : nv == 3 ? 3 : 4; }
inline int co_r_mlp(int nv) { return nv == 1 ? 8 : nv == 2 ? 4 : nv == 3 ? 3 : 2; }
// batch 1-2 up to 6 vectors per thread per row (d <= 12288 bf16); batch 3-4
// up to 2 (the input slices and the MLP's output columns of 4 rows stay in
// registers)
inline bool co_ok(int nb, int d, int E) {
  const int nv = co_nv(d, E);
  return (nb <= 2 && nv <= 6) || (nb <= 4 && nv <= 2);
}
inline int co_grid(long long groups) {
  const long long cap = 2ll * sm_count();
  return (int)(groups < 1 ? 1 : (groups > cap ? cap : groups));
}

#define DV_CO_SWITCH(KERN, NB, grid, st, a, LAUNCH)                           \
  switch (nv) {                                                              \
    case 1: return LAUNCH(KERN<T, NB, 1, 8>, grid, CO_THREADS, 0, st, a);    \
    case 2: return LAUNCH(KERN<T, NB, 2, 4>, grid, CO_THREADS, 0, st, a);    \
    case 3: return LAUNCH(KERN<T, NB, 3, 3>, grid, CO_THREADS, 0, st, a);    \
    case 4: return LAUNCH(KERN<T, NB, 4, 4>, grid, CO_THREADS, 0, st, a);    \
    case 5: return LAUNCH(KERN<T, NB, 5, 4>, grid, CO_THREADS, 0, st, a);    \
    default: return LAUNCH(KERN<T, NB, 6, 4>, grid, CO_THREADS, 0, st, a);   \
  }
#define DV_CO_SWITCH_MLP(KERN, NB, grid, st, a)                               \
  switch (nv) {                                                              \
    case 1: return launch_main(KERN<T, NB, 1, 8>, grid, CO_THREADS, 0, st, a); \
    case 2: return launch_main(KERN<T, NB, 2, 4>, grid, CO_THREADS, 0, st, a); \
    case 3: return launch_main(KERN<T, NB, 3, 3>, grid, CO_THREADS, 0, st, a); \
    case 4: return launch_main(KERN<T, NB, 4, 2>, grid, CO_THREADS, 0, st, a); \
    case 5: return launch_main(KERN<T, NB, 5, 2>, grid, CO_THREADS, 0, st, a); \
    default: return launch_main(KERN<T, NB, 6, 2>, grid, CO_THREADS, 0, st, a); \
  }

// batch 3-4: vectors per thread 1 or 2 only
#define DV_CO_SWITCH4(KERN, grid, st, a, LAUNCH)                              \
  if (nv == 1) return LAUNCH(KERN<T, 4, 1, 8>, grid, CO_THREADS, 0, st, a);  \
  return LAUNCH(KERN<T, 4, 2, 4>, grid, CO_THREADS, 0, st, a);

template <typename T, int NB>
cudaError_t run_attn_in_co_nb(const AttnInArgs& a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E), R = co_r(nv);
  const dim3 grid(co_grid(((long long)a.kh_max * 3 * a.dh + a.n2h + a.n2r + R - 1) / R));
  if constexpr (NB == 4) {
    DV_CO_SWITCH4(attn_in_co_kernel, grid, st, a, launch_main)
  } else {
    DV_CO_SWITCH(attn_in_co_kernel, NB, grid, st, a, launch_main)
  }
}

template <typename T, int NB>
cudaError_t run_mlp_block_co_nb(MlpBlockArgs a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E), R = co_r_mlp(nv);
  a.G = co_grid(((long long)a.k_max + R - 1) / R);
  const dim3 grid(a.G);
  if constexpr (NB == 4) {
    DV_CO_SWITCH4(mlp_block_co_kernel, grid, st, a, launch_main)
  } else {
    DV_CO_SWITCH_MLP(mlp_block_co_kernel, NB, grid, st, a)
  }
}

template <typename T, int NB>
cudaError_t run_predict_a_co_nb(const PredictAArgs& a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E), R = co_r(nv);
  const int rows = (a.PA ? a.h : 0) + (a.At ? a.r : 0);
  const dim3 grid(co_grid((rows + R - 1) / R));
  if constexpr (NB == 4) {
    DV_CO_SWITCH4(predict_a_co_kernel, grid, st, a, launch)
  } else {
    DV_CO_SWITCH(predict_a_co_kernel, NB, grid, st, a, launch)
  }
}
#undef DV_CO_SWITCH
#undef DV_CO_SWITCH_MLP
#undef DV_CO_SWITCH4

// ---------------------------------------------------------------------------
// Streaming kernels (dv_stream.cuh) for rows of 16 KB and more, batch 1-2
// ---------------------------------------------------------------------------

inline bool stream_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DV_STREAM");
    return !(e && e[0] == '0');
  }();
  return on;
}
inline bool st_ok(int nb, int d, int E) {
  const int nv = co_nv(d, E);
  return stream_enabled() && nb <= 2 && nv >= 4 && nv <= 6;
}
inline size_t st_smem(int nv) { return (size_t)ST_SLOTS * nv * CO_THREADS * 16; }
inline int st_grid(long long rows) {
  const long long cap = sm_count();
  return (int)(rows < 1 ? 1 : (rows > cap ? cap : rows));
}

#define DV_ST_SWITCH(KERN, NB, grid, st, a)                                         \
  switch (nv) {                                                                    \
    case 4: return launch_fused_co(KERN<T, NB, 4>, grid, st_smem(4), st, a);        \
    case 5: return launch_fused_co(KERN<T, NB, 5>, grid, st_smem(5), st, a);        \
    default: return launch_fused_co(KERN<T, NB, 6>, grid, st_smem(6), st, a);       \
  }

template <typename K, typename A>
cudaError_t launch_fused_co(K kern, dim3 grid, size_t smem, cudaStream_t st, const A& a) {
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  return launch_main(kern, grid, CO_THREADS, smem, st, a);
}

// Whether the MLP ring kernel fills its ring by bulk copies instead of
// per-thread cp.async: at batch 1 (DV_BULK=0 or 1 overrides). Measured at the
// OPT-175B shape: the MLP kernel alone 36.1 against 40.7 us at batch 1, but
// 74.1 against 71.6 at batch 2; the Q/K/V kernel was slower with bulk copies
// at both batches (30.0 against 25.2 us at batch 1), so it keeps cp.async.
inline bool st_bulk(int nb) {
  static const int env = [] {
    const char* e = std::getenv("DV_BULK");
    return !e ? -1 : (e[0] == '1' ? 1 : 0);
  }();
  return env >= 0 ? env == 1 : nb == 1;
}

#define DV_ST_SWITCH_BULK(KERN, NB, grid, st, a)                                              \
  switch (nv) {                                                                              \
    case 4: return launch_fused_co(KERN<T, NB, 4, ST_SLOTS, true>, grid, st_smem(4), st, a);  \
    case 5: return launch_fused_co(KERN<T, NB, 5, ST_SLOTS, true>, grid, st_smem(5), st, a);  \
    default: return launch_fused_co(KERN<T, NB, 6, ST_SLOTS, true>, grid, st_smem(6), st, a); \
  }

template <typename T, int NB>
cudaError_t run_attn_in_st_nb(const AttnInArgs& a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E);
  const dim3 grid(st_grid((long long)a.kh_max * 3 * a.dh + a.n2h + a.n2r));
  DV_ST_SWITCH(attn_in_stream_kernel, NB, grid, st, a)
}

template <typename T, int NB>
cudaError_t run_mlp_block_st_nb(MlpBlockArgs a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E);
  a.G = st_grid(a.k_max);
  const dim3 grid(a.G);
  if (st_bulk(a.nb)) DV_ST_SWITCH_BULK(mlp_stream_kernel, NB, grid, st, a)
  DV_ST_SWITCH(mlp_stream_kernel, NB, grid, st, a)
}
#undef DV_ST_SWITCH_BULK

template <typename T, int NB>
cudaError_t run_predict_a_st_nb(const PredictAArgs& a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E);
  const dim3 grid(st_grid((a.PA ? a.h : 0) + (a.At ? a.r : 0)));
  DV_ST_SWITCH(predict_a_stream_kernel, NB, grid, st, a)
}
template <typename T, int NB>
cudaError_t run_wo_stream_nb(const WoStreamArgs& a, cudaStream_t st) {
  const int nv = co_nv(a.d, WT<T>::E);
  const dim3 grid(sm_count());
  // ring slots: 4 at batch 1, 8 at batch 2 (DV_WO_SLOTS = 4 or 8
  // overrides; 5 and 6 measured no better). At the OPT-175B shape the smaller ring made the look-ahead
  // step faster at batch 1 (117.0-117.4 against 118.1-118.2 us per layer,
  // two runs each) although the kernel alone is slower (20.5 against 19.1
  // us with the attention); at batch 2 it was slower (250.5 against 248.9).
  static const int env_slots = [] {
    const char* e = std::getenv("DV_WO_SLOTS");
    const int v = e ? std::atoi(e) : 0;
    return (v == 4 || v == 8) ? v : 0;
  }();
  const int slots = env_slots ? env_slots : (a.nb == 1 ? 4 : 8);
  auto go = [&](auto kern, int s) {
    return launch_fused_co(kern, grid, (size_t)s * nv * CO_THREADS * 16, st, a);
  };
#define DV_WO_CASE(S)                                                      \
  if (slots == S) switch (nv) {                                           \
      case 4: return go(wo_stream_kernel<T, NB, 4, S>, S);                 \
      case 5: return go(wo_stream_kernel<T, NB, 5, S>, S);                 \
      default: return go(wo_stream_kernel<T, NB, 6, S>, S);                \
    }
  DV_WO_CASE(4)
  DV_WO_CASE(8)
#undef DV_WO_CASE
  return cudaErrorInvalidValue;
}
#undef DV_ST_SWITCH

// The W^O product in its own ring kernel after an attention-only attn_out:
// long rows (16-24 KB, bf16), batch 1-2, and DV_WOSPLIT not 0.
inline bool wo_split_ok(int nb, int d, int E, int kvbytes) {
  static const bool on = [] {
    const char* e = std::getenv("DV_WOSPLIT");
    return !(e && e[0] == '0');
  }();
  return on && attn_out_whole_rows(d, E, kvbytes, nb) != 0 && st_ok(nb, d, E);
}

// Whether run_attn_in_any picks a kernel that also takes the next layer's
// predictor rows (the column-owner and streaming kernels).
inline bool attn_in_takes_rows(int nb, int d, int E) { return st_ok(nb, d, E) || co_ok(nb, d, E); }

template <typename T>
cudaError_t run_attn_in_any(const AttnInArgs& a, cudaStream_t st) {
  if (st_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_attn_in_st_nb<T, 1>(a, st) : run_attn_in_st_nb<T, 2>(a, st);
  if (co_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_attn_in_co_nb<T, 1>(a, st) : a.nb == 2 ? run_attn_in_co_nb<T, 2>(a, st) : run_attn_in_co_nb<T, 4>(a, st);
  return run_attn_in<T>(a, st);
}

template <typename T>
cudaError_t run_mlp_block_any(const MlpBlockArgs& a, cudaStream_t st) {
  if (st_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_mlp_block_st_nb<T, 1>(a, st) : run_mlp_block_st_nb<T, 2>(a, st);
  // batch 3-4: the union set spans several row groups per CTA, which the
  // column-owner MLP kernel takes one after the other (measured slower than
  // the row kernel there), so only batch 1-2 use it
  if (a.nb <= 2 && co_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_mlp_block_co_nb<T, 1>(a, st) : run_mlp_block_co_nb<T, 2>(a, st);
  return run_mlp_block<T>(a, st);
}

template <typename T>
cudaError_t run_predict_a_any(const PredictAArgs& a, cudaStream_t st) {
  if (st_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_predict_a_st_nb<T, 1>(a, st) : run_predict_a_st_nb<T, 2>(a, st);
  if (co_ok(a.nb, a.d, WT<T>::E))
    return a.nb == 1 ? run_predict_a_co_nb<T, 1>(a, st) : a.nb == 2 ? run_predict_a_co_nb<T, 2>(a, st) : run_predict_a_co_nb<T, 4>(a, st);
  return run_predict_a<T>(a, st);
}

// ---------------------------------------------------------------------------
// Entry points of the per-family translation units: element-type dispatch.
// ---------------------------------------------------------------------------

cudaError_t run_mlp_up_dt(dv_dtype dt, const void* W1t, int d, int N, const float* y, int nb, const float* b1,
                          const int32_t* idx, const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a,
                          int32_t* seg_cnt, int* status, int nseg, int act, cudaStream_t st);
cudaError_t run_axpy_dt(dv_dtype dt, const void* W, int d, int nrows_w, RowsHeads src, const float* bias, float* out,
                        int nb, int k_max, size_t smem, int* status, cudaStream_t st);
cudaError_t run_axpy_dt(dv_dtype dt, const void* W, int d, int nrows_w, RowsMlp src, const float* bias, float* out,
                        int nb, int k_max, size_t smem, int* status, cudaStream_t st);
cudaError_t run_qkv_dt(dv_dtype dt, const void* Wqkv, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                       const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, void* Kc, void* Vc,
                       int cap, int pos, int* status, cudaStream_t st);
cudaError_t run_kv_rest_dt(dv_dtype dt, const void* Wqkv, int d, int h, int dh, const float* y, int nb,
                           const float* bqkv, const int32_t* head_idx, const int32_t* head_count, int kh_max, void* Kc,
                           void* Vc, int cap, int pos, int* status, cudaStream_t st);
cudaError_t run_attn_dt(dv_dtype kvdt, int dh, const float* q, const void* Kc, const void* Vc, int B, int h, int cap,
                        int pos, float scale, const int32_t* head_idx, const int32_t* head_count, int kh_max,
                        float* part, unsigned* ctr, float* H, int* status, cudaStream_t st);
cudaError_t run_attn_in_any_dt(dv_dtype wdt, const AttnInArgs& a, cudaStream_t st);
// weight-only int8 (dv_inst_q8.cu), batch 1-4
cudaError_t run_mlp_up_q8(const int8_t* W1, const float* s1, int d, int N, const float* y, int nb, const float* b1,
                          const int32_t* idx, const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a,
                          int32_t* seg_cnt, int* status, int nseg, int act, cudaStream_t st);
cudaError_t run_qkv_q8(const int8_t* W, const float* s, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                       const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, void* Kc, void* Vc,
                       int cap, int pos, int* status, cudaStream_t st);
cudaError_t run_axpy_q8(const int8_t* W, int d, int nrows_w, RowsMlp src, const float* bias, float* out, int nb,
                        int k_max, size_t smem, int* status, cudaStream_t st);
cudaError_t run_axpy_q8(const int8_t* W, int d, int nrows_w, RowsHeads src, const float* bias, float* out, int nb,
                        int k_max, size_t smem, int* status, cudaStream_t st);
cudaError_t run_attn_out_dt(dv_dtype kvdt, const AttnOutArgs& a, cudaStream_t st);
cudaError_t run_attn_out_bf16(const AttnOutArgs& a, cudaStream_t st);
cudaError_t run_attn_out_f32(const AttnOutArgs& a, cudaStream_t st);
cudaError_t run_wo_stream_dt(dv_dtype wdt, const WoStreamArgs& a, cudaStream_t st);
cudaError_t run_mlp_block_any_dt(dv_dtype wdt, const MlpBlockArgs& a, cudaStream_t st);
cudaError_t run_predict_a_any_dt(dv_dtype wdt, const PredictAArgs& a, cudaStream_t st);
cudaError_t run_predict_b_dt(dv_dtype wdt, const PredictBArgs& a, cudaStream_t st);

}  // namespace dv
