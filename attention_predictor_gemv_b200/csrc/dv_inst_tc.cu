// Launchers of the tensor-core gathered-row kernels (dv_tc.cuh), and the
// TMA descriptors they read.
#include <cudaTypedefs.h>

#include <cstdlib>

#include "dv_launch.cuh"
#include "dv_tc.cuh"
#include "dv_tc_launch.h"

namespace dv {

namespace {

// CTAs per SM: one with a TC_STAGES_MAX-stage ring, or two with half the
// ring each (DV_TC_CTAS=1 / 2).
int tc_ctas_per_sm() {
  static const int n = [] {
    const char* e = std::getenv("DV_TC_CTAS");
    return (e && e[0] == '1') ? 1 : 2;
  }();
  return n;
}
int tc_stages() { return TC_STAGES_MAX / tc_ctas_per_sm(); }

template <typename K, typename A>
cudaError_t launch_tc(K kern, int grid, cudaStream_t st, const TcMaps& m, A a) {
  a.stages = tc_stages();
  const size_t smem = tc_smem(a.stages);
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  return launch_main(kern, dim3(grid < 1 ? 1 : grid), dim3(TC_THREADS), smem, st, m, a);
}

int clamp_grid(long long units) {
  const long long cap = (long long)tc_ctas_per_sm() * sm_count();
  return (int)(units < 1 ? 1 : (units > cap ? cap : units));
}


// cuTensorMapEncodeTiled, from the driver the runtime is bound to (no link
// against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// A bf16 matrix [rows][cols] with row stride ld elements, read in boxes of
// box_cols x box_rows into the 128-byte swizzled shared layout; reads past
// the matrix return zeros.
cudaError_t tc_map(CUtensorMap* m, const void* base, long long cols, long long rows, long long ld, int box_cols,
                   int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  if (!aligned16(base) || (ld * 2) % 16 != 0 || cols < 1 || rows < 1 || ld < cols) return cudaErrorInvalidValue;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Maps of one kernel: gathered weight rows (or W^O in 64-row tiles) and the
// operand's hi / lo rows [16][ld] of which the first `cols` are used.
cudaError_t tc_maps(TcMaps* m, const __nv_bfloat16* W, long long w_rows, int d, int w_box_rows,
                    const __nv_bfloat16* hi, const __nv_bfloat16* lo, long long cols, long long ld) {
  cudaError_t e = tc_map(&m->w, W, d, w_rows, d, TC_K, w_box_rows);
  if (e == cudaSuccess) e = tc_map(&m->hi, hi, cols, TC_N, ld, TC_K, TC_N);
  if (e == cudaSuccess) e = tc_map(&m->lo, lo, cols, TC_N, ld, TC_K, TC_N);
  return e;
}

}  // namespace

bool tc_shape_ok(int B, int d, int wbytes, int dh, int k_max) {
  return wbytes == 2 && B >= 1 && B <= TC_N && d >= TC_K && d % 8 == 0 && dh % 64 == 0 &&
         (k_max + TC_M - 1) / TC_M <= TC_MAX_TILES && encode_fn() != nullptr;
}

int tc_tiles(int k_max) { return (k_max + TC_M - 1) / TC_M; }

int tc_axpy_group(int items_max, int d, int most) {
  const long long n_mt = (d + TC_M - 1) / TC_M;
  const long long g = (long long)items_max * n_mt / (2ll * tc_ctas_per_sm() * sm_count());
  return (int)(g < 1 ? 1 : (g > most ? most : g));
}

size_t tc_red_floats(int k_max, int kh_max, int dh, int d) {
  const long long tiles = tc_tiles(k_max), qkv = ((long long)kh_max * 3 * dh + TC_M - 1) / TC_M;
  long long slots = TC_DENSE_PARTS;
  if (8 * tiles > slots) slots = 8 * tiles;
  if (8 * qkv > slots) slots = 8 * qkv;
  (void)d;
  return (size_t)slots * TC_N * TC_M;
}

size_t tc_tick_count(int k_max, int kh_max, int dh, int d) {
  long long n = TC_DENSE_PARTS;
  const long long cand[2] = {tc_tiles(k_max), ((long long)kh_max * 3 * dh + TC_M - 1) / TC_M};
  for (long long c : cand) n = c > n ? c : n;
  (void)d;
  return (size_t)n;
}

namespace {
// out[b][:] += the fixed-point totals in acc (+ bias); acc back to zero
cudaError_t run_tc_finalize(unsigned long long* acc, const float* bias, float* out, int nb, int d, cudaStream_t st) {
  TcFinalizeArgs f{acc, bias, out, nb, d};
  const long long n = (long long)nb * d, cap = 2ll * sm_count();
  const long long g = (n + 255) / 256;
  return launch_main(tc_finalize_kernel, dim3((unsigned)(g < 1 ? 1 : (g > cap ? cap : g))), dim3(256), 0, st, f);
}
}  // namespace

cudaError_t run_tc_split(const float* x, int nb, int n, long long ld_src, __nv_bfloat16* hi, __nv_bfloat16* lo,
                         long long ld_dst, cudaStream_t st) {
  TcSplitArgs a{x, nb, n, ld_src, hi, lo, ld_dst};
  const int gx = (n + 255) / 256 < 64 ? (n + 255) / 256 : 64;
  return launch_main(tc_split_kernel, dim3(gx > 0 ? gx : 1, TC_N), dim3(256), 0, st, a);
}

// The rowdot kernels split K on the device (tc_pick_kslog, up to 8 parts):
// the grid covers up to eight units per tile.
cudaError_t run_tc_qkv(TcQkvArgs a, cudaStream_t st) {
  const long long tiles = ((long long)a.kh_max * 3 * a.dh + TC_M - 1) / TC_M;
  if (tiles == 0) return cudaSuccess;
  TcMaps m;
  cudaError_t e = tc_maps(&m, a.Wqkv, (long long)a.h * 3 * a.dh, a.d, 64, a.xhi, a.xlo, a.d, a.d);
  if (e != cudaSuccess) return e;
  return launch_tc(tc_qkv_kernel, clamp_grid(tiles * 8), st, m, a);
}

cudaError_t run_tc_mlp(TcMlpArgs a, cudaStream_t st) {
  const int tiles = tc_tiles(a.k_max);
  const int n_mt = (a.d + TC_M - 1) / TC_M;
  a.tiles_per_group = tc_axpy_group(tiles, a.d, 8);
  if (tiles > 0) {
    TcMaps m1;
    cudaError_t e = tc_maps(&m1, a.W1t, a.N, a.d, 1, a.xhi, a.xlo, a.d, a.d);
    if (e == cudaSuccess) e = launch_tc(tc_w1_kernel, clamp_grid(8ll * tiles), st, m1, a);
    if (e != cudaSuccess) return e;
  }
  TcMaps m2;
  cudaError_t e = tc_maps(&m2, a.W2t, a.N, a.d, 1, a.act_hi, a.act_lo, a.KC > 0 ? a.KC : TC_M, a.KC > 0 ? a.KC : TC_M);
  if (e != cudaSuccess) return e;
  const long long groups = tiles > 0 ? (tiles + a.tiles_per_group - 1) / a.tiles_per_group : 1;
  e = launch_tc(tc_w2_kernel, clamp_grid(groups * n_mt), st, m2, a);
  if (e != cudaSuccess) return e;
  return run_tc_finalize(a.acc, a.b2, a.out, a.nb, a.d, st);
}

cudaError_t run_tc_wo(TcWoArgs a, cudaStream_t st) {
  const int n_mt = (a.d + TC_M - 1) / TC_M;
  a.heads_per_group = tc_axpy_group(a.kh_max, a.d, 4);
  const long long groups = a.kh_max > 0 ? (a.kh_max + a.heads_per_group - 1) / a.heads_per_group : 1;
  const long long ldh = (long long)(a.kh_max > 0 ? a.kh_max : 1) * a.dh;
  TcMaps m;
  cudaError_t e = tc_maps(&m, a.WOt, (long long)a.h * a.dh, a.d, 64, a.hhi, a.hlo, ldh, ldh);
  if (e != cudaSuccess) return e;
  e = launch_tc(tc_wo_kernel, clamp_grid(groups * n_mt), st, m, a);
  if (e != cudaSuccess) return e;
  return run_tc_finalize(a.acc, a.bO, a.out, a.nb, a.d, st);
}

bool tc_dense_ok(int B, int wbytes, int nrows, int K) {
  return wbytes == 2 && B >= 1 && B <= TC_N && nrows >= 64 && K >= TC_K && K % 8 == 0 && encode_fn() != nullptr;
}


cudaError_t run_tc_dense(const __nv_bfloat16* W1, int n1, const float* bias1, float* out1, long long ldo1,
                         const __nv_bfloat16* W2, int n2, const float* bias2, float* out2, long long ldo2, int K,
                         const __nv_bfloat16* xhi, const __nv_bfloat16* xlo, int nb, float* red, unsigned* tick,
                         int* status, cudaStream_t st) {
  if (n1 < 0 || n2 < 1) return cudaErrorInvalidValue;
  const long long p1 = (n1 + 63) / 64 * 64;
  const long long tiles = (p1 + n2 + TC_M - 1) / TC_M, C = (K + TC_K - 1) / TC_K;
  const long long slots = (long long)tc_ctas_per_sm() * sm_count();
  long long want = (slots + tiles - 1) / tiles;
  if (want > C) want = C;
  if (want > TC_DENSE_PARTS / tiles) want = TC_DENSE_PARTS / tiles;
  if (want > TC_DENSE_MAX_KS) want = TC_DENSE_MAX_KS;
  int kslog = 0;  // the largest power of two not above want
  while ((2ll << kslog) <= want) ++kslog;
  const long long ks = 1ll << kslog;
  TcDenseArgs a = {};
  a.bias1 = bias1;
  a.bias2 = bias2;
  a.n1 = n1;
  a.n2 = n2;
  a.K = K;
  a.nb = nb;
  a.kslog = kslog;
  a.out1 = out1;
  a.out2 = out2;
  a.ldo1 = ldo1;
  a.ldo2 = ldo2;
  a.status = status;
  a.red = red;
  a.tick = tick;
  TcMaps m;
  cudaError_t e = tc_maps(&m, W2, n2, K, 64, xhi, xlo, K, K);
  if (e != cudaSuccess) return e;
  m.w2 = m.w;
  if (n1 > 0) {
    e = tc_map(&m.w, W1, K, n1, K, TC_K, 64);
    if (e != cudaSuccess) return e;
  }
  return launch_tc(tc_dense_kernel, clamp_grid(tiles * ks), st, m, a);
}

}  // namespace dv
