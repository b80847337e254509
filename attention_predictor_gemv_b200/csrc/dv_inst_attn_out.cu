// Instantiates the launchers of attn_out (split attention + W^O), bf16.
#include "dv_launchers.cuh"

namespace dv {

cudaError_t run_attn_out_dt(dv_dtype kvdt, const AttnOutArgs& a, cudaStream_t st) {
  return kvdt == DV_BF16 ? run_attn_out_bf16(a, st) : run_attn_out_f32(a, st);
}

cudaError_t run_attn_out_bf16(const AttnOutArgs& a, cudaStream_t st) { return run_attn_out<bf16>(a, st); }

cudaError_t run_wo_stream_dt(dv_dtype wdt, const WoStreamArgs& a, cudaStream_t st) {
  if (wdt != DV_BF16) return cudaErrorInvalidValue;  // long-row kernels are bf16 only
  return a.nb == 1 ? run_wo_stream_nb<bf16, 1>(a, st) : run_wo_stream_nb<bf16, 2>(a, st);
}

}  // namespace dv
