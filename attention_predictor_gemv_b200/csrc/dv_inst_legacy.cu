// Instantiates the launchers of the kernel-per-step path (dv_kernels.cuh).
#include "dv_launchers.cuh"

namespace dv {

cudaError_t run_gemv(dv_dtype dt, const void* W, int nrows, int K, const float* X, int ldx, int nb, const float* bias,
                     float* out, int ldo, cudaStream_t st) {
  return dt == DV_BF16 ? run_dense_gemv<bf16>(W, nrows, K, X, ldx, nb, bias, out, ldo, st)
                       : run_dense_gemv<float>(W, nrows, K, X, ldx, nb, bias, out, ldo, st);
}

cudaError_t run_select(const float* scores, int nrows, int n, int k, float tau, int mode, uint32_t* bm,
                       unsigned* ticket, int32_t* idx, int32_t* count, cudaStream_t st) {
  if (n <= SEL_SMEM_KEYS) {  // keys (top-k) and the union bitmap in shared memory
    const size_t smem = 4ull * n;
    cudaError_t e = allow_smem(select_kernel<true>, smem);
    if (e != cudaSuccess) return e;
    return launch(select_kernel<true>, dim3(nrows), SEL_THREADS, smem, st, scores, n, nrows, k, tau, mode, bm, ticket,
                  idx, count);
  }
  return launch(select_kernel<false>, dim3(nrows), SEL_THREADS, 0, st, scores, n, nrows, k, tau, mode, bm, ticket, idx,
                count);
}

cudaError_t run_mlp_up_dt(dv_dtype dt, const void* W1t, int d, int N, const float* y, int nb, const float* b1,
                          const int32_t* idx, const int32_t* count, int k_max, int32_t* seg_idx, float* seg_a,
                          int32_t* seg_cnt, int* status, int nseg, int act, cudaStream_t st) {
  return dt == DV_BF16
             ? run_mlp_up<bf16>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act, st)
             : run_mlp_up<float>(W1t, d, N, y, nb, b1, idx, count, k_max, seg_idx, seg_a, seg_cnt, status, nseg, act,
                                 st);
}

cudaError_t run_axpy_dt(dv_dtype dt, const void* W, int d, int nrows_w, RowsHeads src, const float* bias, float* out,
                        int nb, int k_max, size_t smem, int* status, cudaStream_t st) {
  return dt == DV_BF16 ? run_axpy<bf16>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st)
                       : run_axpy<float>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
}

cudaError_t run_axpy_dt(dv_dtype dt, const void* W, int d, int nrows_w, RowsMlp src, const float* bias, float* out,
                        int nb, int k_max, size_t smem, int* status, cudaStream_t st) {
  return dt == DV_BF16 ? run_axpy<bf16>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st)
                       : run_axpy<float>(W, d, nrows_w, src, bias, out, nb, k_max, smem, status, st);
}

}  // namespace dv
