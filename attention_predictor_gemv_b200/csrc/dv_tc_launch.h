// Host-side declarations of the tensor-core kernel launchers (dv_inst_tc.cu).
#pragma once

#include <cuda_runtime.h>

#include "dv_tc_args.h"

namespace dv {

constexpr int TC_DENSE_PARTS = 512;  // dense rowdot units (tiles x K parts) with partial-sum slots, at most
constexpr int TC_DENSE_MAX_KS = 32;  // K parts per dense tile, at most (the last part sums them)

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

// The dense rowdot over one or two matrices sharing the operand x (split
// into xhi / xlo [16][K]): out1[b][i] = W1[i] . x[b] (+ bias1[i]) for the n1
// rows of W1 [n1][K] (n1 = 0: none), and out2[b][i] = W2[i] . x[b] (+
// bias2[i]) for the n2 rows of W2, bf16. When the K range is split across
// CTAs (at most TC_DENSE_PARTS units of tiles x parts) the partial sums go
// through red [units][128][16] and the per-tile tickets tick (zero between
// calls).
bool tc_dense_ok(int B, int wbytes, int nrows, int K);
cudaError_t run_tc_dense(const __nv_bfloat16* W1, int n1, const float* bias1, float* out1, long long ldo1,
                         const __nv_bfloat16* W2, int n2, const float* bias2, float* out2, long long ldo2, int K,
                         const __nv_bfloat16* xhi, const __nv_bfloat16* xlo, int nb, float* red, unsigned* tick,
                         int* status, cudaStream_t st);

}  // namespace dv
