// Instantiates the launchers of attn_in (LN1 + Q/K/V + KV append).
#include "dv_launchers.cuh"

namespace dv {

cudaError_t run_attn_in_any_dt(dv_dtype wdt, const AttnInArgs& a, cudaStream_t st) {
  return wdt == DV_BF16 ? run_attn_in_any<bf16>(a, st) : run_attn_in_any<float>(a, st);
}

}  // namespace dv
