// Instantiates the launchers of mlp_block (LN2 + W1 + ReLU + W2).
#include "dv_launchers.cuh"

namespace dv {

cudaError_t run_mlp_block_any_dt(dv_dtype wdt, const MlpBlockArgs& a, cudaStream_t st) {
  return wdt == DV_BF16 ? run_mlp_block_any<bf16>(a, st) : run_mlp_block_any<float>(a, st);
}

}  // namespace dv
