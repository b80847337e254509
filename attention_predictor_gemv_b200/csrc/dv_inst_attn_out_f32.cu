// Instantiates the launchers of attn_out (split attention + W^O), fp32.
#include "dv_launchers.cuh"

namespace dv {

cudaError_t run_attn_out_f32(const AttnOutArgs& a, cudaStream_t st) { return run_attn_out<float>(a, st); }

}  // namespace dv
