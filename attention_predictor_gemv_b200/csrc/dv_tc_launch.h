// Host-side declarations of the tensor-core kernel launchers (dv_inst_tc.cu).
#pragma once

#include <cuda_runtime.h>

#include "dv_tc_args.h"

namespace dv {

constexpr int TC_DENSE_PARTS = 512;  // dense rowdot units (tiles x K parts) with partial-sum slots, at most

// Shapes the tensor-core path takes: bf16 weights, at most 16 batch rows,
// d >= 64 and a multiple of 8, dh a multiple of 64, at most 1024 tiles of 128
// selected neurons; and a driver that encodes TMA descriptors.
bool tc_shape_ok(int B, int d, int wbytes, int dh, int k_max);
// Tiles of 128 selected neurons for a bound of k_max.
int tc_tiles(int k_max);
// Rows per rowaxpy group (tiles of W2 rows, heads of W^O) for at most
// items_max of them: as many as still give every CTA two units of a group x
// 128 columns, at most `most`.
int tc_axpy_group(int items_max, int d, int most);
// Workspace the tensor-core kernels' reductions need: floats of partial-sum
// slots and per-tile tickets, for the largest sets of a call.
size_t tc_red_floats(int k_max, int kh_max, int dh, int d);
size_t tc_tick_count(int k_max, int kh_max, int dh, int d);

// hi / lo bf16 rows [16][ld_dst] of x [nb][n] (row stride ld_src); rows >= nb zero.
cudaError_t run_tc_split(const float* x, int nb, int n, long long ld_src, __nv_bfloat16* hi, __nv_bfloat16* lo,
                         long long ld_dst, cudaStream_t st);
cudaError_t run_tc_qkv(TcQkvArgs a, cudaStream_t st);
// W1 + bias + ReLU with per-tile compaction, then the W2 gather-axpy into out.
cudaError_t run_tc_mlp(TcMlpArgs a, cudaStream_t st);
cudaError_t run_tc_wo(TcWoArgs a, cudaStream_t st);

// The dense rowdot: out[b][row] = W[row] . x[b] (+ bias[row]) for the rows
// of W [nrows][K] (bf16) and the operand split into xhi / xlo [16][K]; out
// [nb][ldo]. When the K range is split across CTAs (at most TC_DENSE_PARTS
// units of tiles x parts) the partial sums go through red [units][16][128]
// and the per-tile tickets tick [tiles] (zero between calls).
bool tc_dense_ok(int B, int wbytes, int nrows, int K);
cudaError_t run_tc_dense(const __nv_bfloat16* W, int nrows, int K, const float* bias, const __nv_bfloat16* xhi,
                         const __nv_bfloat16* xlo, int nb, float* out, long long ldo, float* red, unsigned* tick,
                         int* status, cudaStream_t st);

}  // namespace dv
