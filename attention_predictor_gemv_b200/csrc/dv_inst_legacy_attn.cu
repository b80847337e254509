// Instantiates the launchers of the kernel-per-step attention (dv_kernels.cuh).
#include "dv_launchers.cuh"

namespace dv {

cudaError_t run_qkv_dt(dv_dtype dt, const void* Wqkv, int d, int h, int dh, const float* y, int nb, const float* bqkv,
                       const int32_t* head_idx, const int32_t* head_count, int kh_max, float* q, void* Kc, void* Vc,
                       int cap, int pos, int* status, cudaStream_t st) {
  return dt == DV_BF16 ? run_qkv<bf16>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos,
                                       status, st)
                       : run_qkv<float>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, q, Kc, Vc, cap, pos,
                                        status, st);
}

cudaError_t run_kv_rest_dt(dv_dtype dt, const void* Wqkv, int d, int h, int dh, const float* y, int nb,
                           const float* bqkv, const int32_t* head_idx, const int32_t* head_count, int kh_max, void* Kc,
                           void* Vc, int cap, int pos, int* status, cudaStream_t st) {
  return dt == DV_BF16 ? run_kv_rest<bf16>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, Kc, Vc, cap, pos,
                                           status, st)
                       : run_kv_rest<float>(Wqkv, d, h, dh, y, nb, bqkv, head_idx, head_count, kh_max, Kc, Vc, cap,
                                            pos, status, st);
}

cudaError_t run_attn_dt(dv_dtype kvdt, int dh, const float* q, const void* Kc, const void* Vc, int B, int h, int cap,
                        int pos, float scale, const int32_t* head_idx, const int32_t* head_count, int kh_max,
                        float* part, unsigned* ctr, float* H, int* status, cudaStream_t st) {
  return kvdt == DV_BF16 ? run_attn<bf16>(dh, q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, part, ctr,
                                          H, status, st)
                         : run_attn<float>(dh, q, Kc, Vc, B, h, cap, pos, scale, head_idx, head_count, kh_max, part,
                                           ctr, H, status, st);
}

}  // namespace dv
