// Launchers of the weight-only int8 gathered-row kernels (per-row fp32
// scales): W1 + bias + activation + compaction, the W2 and W^O gather-axpys
// and the selected heads' q, k, v into a bf16 KV cache. Batch 1-4.
#include "dv_launchers.cuh"

namespace dv {

namespace {

using i8 = int8_t;

template <int NB>
cudaError_t mlp_up_q8_nb(const i8* W1, const float* s1, int d, int N, const float* y, int nb, const float* b1,
                         const int32_t* idx, const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a,
                         int32_t* seg_cnt, int* status, int nseg, int act, cudaStream_t st) {
  const dim3 grid(nseg > 0 ? nseg : 1);
  switch (rpw_for(d, WT<i8>::E)) {
    case 1: return launch(mlp_up_kernel<i8, NB, 1, 8>, grid, GEMV_THREADS, 0, st, W1, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, act, s1);
    case 2: return launch(mlp_up_kernel<i8, NB, 2, 4>, grid, GEMV_THREADS, 0, st, W1, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, act, s1);
    case 4: return launch(mlp_up_kernel<i8, NB, 4, 2>, grid, GEMV_THREADS, 0, st, W1, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, act, s1);
    default: return launch(mlp_up_kernel<i8, NB, 8, 1>, grid, GEMV_THREADS, 0, st, W1, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, act, s1);
  }
}

template <int NB>
cudaError_t qkv_q8_nb(const i8* W, const float* s, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                      const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, bf16* K, bf16* V,
                      int cap, int pos, int* status, cudaStream_t st) {
  const int rpw = rpw_for(d, WT<i8>::E);
  const int slots = kh_max * 3 * dh, per_cta = GEMV_WARPS * rpw;
  const dim3 grid(slots > 0 ? (slots + per_cta - 1) / per_cta : 1);
  switch (rpw) {
    case 1: return launch(qkv_kernel<i8, bf16, NB, 1, 8>, grid, GEMV_THREADS, 0, st, W, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, s);
    case 2: return launch(qkv_kernel<i8, bf16, NB, 2, 4>, grid, GEMV_THREADS, 0, st, W, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, s);
    case 4: return launch(qkv_kernel<i8, bf16, NB, 4, 2>, grid, GEMV_THREADS, 0, st, W, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, s);
    default: return launch(qkv_kernel<i8, bf16, NB, 8, 1>, grid, GEMV_THREADS, 0, st, W, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, s);
  }
}

}  // namespace

cudaError_t run_mlp_up_q8(const int8_t* W1, const float* s1, int d, int N, const float* y, int nb, const float* b1,
                          const int32_t* idx, const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a,
                          int32_t* seg_cnt, int* status, int nseg, int act, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return mlp_up_q8_nb<1>(W1, s1, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st);
    case 2: return mlp_up_q8_nb<2>(W1, s1, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st);
    default: return mlp_up_q8_nb<4>(W1, s1, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st);
  }
}

cudaError_t run_qkv_q8(const int8_t* W, const float* s, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                       const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, void* Kc, void* Vc,
                       int cap, int pos, int* status, cudaStream_t st) {
  bf16* K = static_cast<bf16*>(Kc);
  bf16* V = static_cast<bf16*>(Vc);
  switch (nb_bucket(nb)) {
    case 1: return qkv_q8_nb<1>(W, s, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, st);
    case 2: return qkv_q8_nb<2>(W, s, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, st);
    default: return qkv_q8_nb<4>(W, s, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, K, V, cap, pos, status, st);
  }
}

template <class Src>
cudaError_t run_axpy_q8_src(const int8_t* W, int d, int nrows_w, Src src, const float* bias, float* out, int nb,
                            int k_max, size_t smem, int* status, cudaStream_t st) {
  switch (nb_bucket(nb)) {
    case 1: return run_axpy_st<i8, 1>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    case 2: return run_axpy_st<i8, 2>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
    default: return run_axpy_st<i8, 4>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
  }
}

cudaError_t run_axpy_q8(const int8_t* W, int d, int nrows_w, RowsMlp src, const float* bias, float* out, int nb,
                        int k_max, size_t smem, int* status, cudaStream_t st) {
  return run_axpy_q8_src(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
}

cudaError_t run_axpy_q8(const int8_t* W, int d, int nrows_w, RowsHeads src, const float* bias, float* out, int nb,
                        int k_max, size_t smem, int* status, cudaStream_t st) {
  return run_axpy_q8_src(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
}

}  // namespace dv
