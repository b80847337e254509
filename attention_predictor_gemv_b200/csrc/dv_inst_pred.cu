// Instantiates the launchers of the look-ahead predictor (predict_a, predict_b).
#include "dv_launchers.cuh"

namespace dv {

cudaError_t run_predict_a_any_dt(dv_dtype wdt, const PredictAArgs& a, cudaStream_t st) {
  return wdt == DV_BF16 ? run_predict_a_any<bf16>(a, st) : run_predict_a_any<float>(a, st);
}

cudaError_t run_predict_b_dt(dv_dtype wdt, const PredictBArgs& a, cudaStream_t st) {
  return wdt == DV_BF16 ? run_predict_b<bf16>(a, st) : run_predict_b<float>(a, st);
}

}  // namespace dv
