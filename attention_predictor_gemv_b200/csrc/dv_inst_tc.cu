// Launchers of the tensor-core gathered-row kernels (dv_tc.cuh).
#include "dv_launch.cuh"
#include "dv_tc.cuh"
#include "dv_tc_launch.h"

namespace dv {

namespace {

template <typename K, typename A>
cudaError_t launch_tc(K kern, int grid, cudaStream_t st, const A& a) {
  cudaError_t e = allow_smem(kern, TC_SMEM);
  if (e != cudaSuccess) return e;
  return launch_main(kern, dim3(grid < 1 ? 1 : grid), dim3(TC_THREADS), TC_SMEM, st, a);
}

int clamp_grid(long long units) {
  const long long cap = sm_count();
  return (int)(units < 1 ? 1 : (units > cap ? cap : units));
}

// Rows (tiles, heads) per rowaxpy unit: as many as still give every SM two
// units at the largest count, at most `most`.
int per_group(long long items_max, long long n_mt, int most) {
  long long g = items_max * n_mt / (2ll * sm_count());
  return (int)(g < 1 ? 1 : (g > most ? most : g));
}

}  // namespace

bool tc_shape_ok(int B, int wbytes, int dh, int k_max) {
  return wbytes == 2 && B >= 1 && B <= TC_N && dh % 64 == 0 && (k_max + TC_M - 1) / TC_M <= TC_MAX_TILES;
}

int tc_tiles(int k_max) { return (k_max + TC_M - 1) / TC_M; }

cudaError_t run_tc_split(const float* x, int nb, int n, long long ld_src, __nv_bfloat16* hi, __nv_bfloat16* lo,
                         long long ld_dst, cudaStream_t st) {
  TcSplitArgs a{x, nb, n, ld_src, hi, lo, ld_dst};
  const int gx = (n + 255) / 256 < 64 ? (n + 255) / 256 : 64;
  return launch_main(tc_split_kernel, dim3(gx > 0 ? gx : 1, TC_N), dim3(256), 0, st, a);
}

cudaError_t run_tc_qkv(const TcQkvArgs& a, cudaStream_t st) {
  const long long units = ((long long)a.kh_max * 3 * a.dh + TC_M - 1) / TC_M;
  if (units == 0) return cudaSuccess;
  return launch_tc(tc_qkv_kernel, clamp_grid(units), st, a);
}

cudaError_t run_tc_mlp(TcMlpArgs a, cudaStream_t st) {
  const int tiles = tc_tiles(a.k_max);
  const int n_mt = (a.d + TC_M - 1) / TC_M;
  a.tiles_per_group = per_group(tiles, n_mt, TC_TILES_PER_GROUP);
  if (tiles > 0) {
    cudaError_t e = launch_tc(tc_w1_kernel, clamp_grid(tiles), st, a);
    if (e != cudaSuccess) return e;
  }
  const long long groups = tiles > 0 ? (tiles + a.tiles_per_group - 1) / a.tiles_per_group : 1;
  return launch_tc(tc_w2_kernel, clamp_grid(groups * n_mt), st, a);
}

cudaError_t run_tc_wo(TcWoArgs a, cudaStream_t st) {
  const int n_mt = (a.d + TC_M - 1) / TC_M;
  a.heads_per_group = per_group(a.kh_max, n_mt, TC_HEADS_PER_GROUP);
  const long long groups = a.kh_max > 0 ? (a.kh_max + a.heads_per_group - 1) / a.heads_per_group : 1;
  return launch_tc(tc_wo_kernel, clamp_grid(groups * n_mt), st, a);
}

}  // namespace dv
